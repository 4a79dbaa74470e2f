"""Key blocks of 64 (block_k = 64, block_q = 128) against the oracle (needs
a B200).

The pages expose the query and key chunk sizes of the blockwise sweep as
separate knobs ("LWM：突破 100 万 Token 的开源大模型", 配置参数:
scan_query_chunk_size, scan_key_chunk_size). With key blocks half as tall
as query blocks, the first key block a query block visits (the one holding
its last row) is fully masked for the block's first 64 rows, so their
running max is still -inf after it: the forward must not subtract an
infinite max. The result is the same attention for every block size.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

OUT_TOL, LSE_TOL = 2e-2, 1e-3
BWD_REL = 2e-2


def _inputs(name, seed, dev, dout=False, seg_kind=None, **kw):
    w = wl.WORKLOADS[name]
    if seg_kind:
        w = wl.Workload(w.name, w.B, w.N, w.H, w.D, w.theta, seg_kind,
                        w.scale, w.backward, seg_args=kw.pop("seg_args"))
    return wl.make_inputs(w, seed, device=dev, with_dout=dout, **kw)


def _fwd(t, qkp, block_k, dtype_check=True):
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], t["theta"], qk_precision=qkp,
                       block_k=block_k)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    return out, lse


def _check_full(t, out, lse, out_tol, lse_tol):
    h = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in t.items()}
    ro, rl = oracle.attn_fwd(h["q"], h["k"], h["v"], h["segment_ids"],
                             h["positions"], t["theta"])
    eo = np.abs(out.float().cpu().numpy() - ro).max()
    el = np.abs(lse.cpu().numpy() - rl).max()
    assert eo <= out_tol and el <= lse_tol, (eo, el)


def test_block64_tiny2k_split_qk(cuda_dev):
    t = _inputs("tiny2k", 0, cuda_dev)
    _check_full(t, *_fwd(t, "bf16x3", 64), OUT_TOL, LSE_TOL)


@pytest.mark.parametrize("N,B,H,lo,hi", [(3000, 2, 3, 1, 900),
                                         (1024, 1, 2, 1, 3),
                                         (777, 1, 2, 60, 70)])
def test_block64_packed_small(cuda_dev, N, B, H, lo, hi):
    t = _inputs("packed128k", 7, cuda_dev, N=N, B=B, H=H, seg_kind="uniform",
                seg_args={"lo": lo, "hi": hi})
    _check_full(t, *_fwd(t, "bf16", 64), OUT_TOL, LSE_TOL)


@pytest.mark.parametrize("N", [1, 63, 64, 65, 129, 200])
def test_block64_edge_sizes(cuda_dev, N):
    t = _inputs("tiny2k", 3, cuda_dev, N=N, H=2, B=2)
    _check_full(t, *_fwd(t, "bf16x3", 64), OUT_TOL, LSE_TOL)


def test_block64_equals_block128_up_to_rounding(cuda_dev):
    # the same attention: the two tilings differ only in summation order
    t = _inputs("packed128k", 2, cuda_dev, N=5000, H=4, seg_kind="uniform",
                seg_args={"lo": 1, "hi": 2000})
    o64, l64 = _fwd(t, "bf16", 64)
    o128, l128 = _fwd(t, "bf16", 128)
    assert (o64.float() - o128.float()).abs().max().item() <= 2 * 2 ** -8
    assert (l64 - l128).abs().max().item() <= 1e-4


def test_block64_packed128k_full_size_sampled_rows(cuda_dev):
    t = _inputs("packed128k", 0, cuda_dev)
    out, lse = _fwd(t, "bf16", 64)
    N = t["q"].shape[1]
    rng = np.random.default_rng(13)
    L = t["lengths"][0]
    starts = np.r_[0, np.cumsum(L)[:-1]]
    rows = np.unique(np.r_[starts, starts + L - 1, rng.integers(0, N, 60)])
    h = {k: (v.cpu() if k in ("segment_ids", "positions") else v)
         for k, v in t.items()}
    idx = torch.from_numpy(rows).to(out.device)
    go = out[0, idx].float().cpu().numpy()
    gl = lse[0][:, idx].cpu().numpy()
    for hh in (0, 11, 31):
        ro, rl = oracle.attn_fwd_rows(h["q"], h["k"], h["v"],
                                      h["segment_ids"], h["positions"],
                                      t["theta"], 0, hh, rows)
        assert np.abs(go[:, hh] - ro).max() <= OUT_TOL
        assert np.abs(gl[hh] - rl).max() <= LSE_TOL


def test_block64_backward(cuda_dev):
    # the key-major backward runs 128-key units for either key block size
    # (an exact reorganisation); block_k = 64 is accepted and gives the
    # same gradients as the oracle
    t = _inputs("packed128k", 8, cuda_dev, N=1500, H=2, dout=True,
                seg_kind="uniform", seg_args={"lo": 1, "hi": 700})
    out, lse = _fwd(t, "bf16", 64)
    dq, dk, dv = ops.bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                         t["segment_ids"], t["positions"], t["theta"],
                         block_k=64)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    h = {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in t.items()}
    ref = oracle.attn_bwd(h["q"], h["k"], h["v"], h["dout"],
                          h["segment_ids"], h["positions"], t["theta"])
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        r = ref[name]
        err = np.abs(g.float().cpu().numpy() - r).max()
        assert err <= BWD_REL * np.abs(r).max(), (name, err)


@pytest.mark.parametrize("name", ["tiny2k", "packed128k", "vl256k"])
def test_block64_visibility_bit_exact(cuda_dev, name):
    # the forward's tile classification at block_k = 64, rebuilt from the
    # metadata it runs on, against the oracle's classes of 128 x 64 tiles
    w = wl.WORKLOADS[name]
    seg, _, _ = wl.make_segments(w, 0)
    v = {k: x.cpu().numpy().astype(np.int64) for k, x in ops.visibility(
        torch.from_numpy(seg).to(cuda_dev), key_view=False,
        block_k=64).items()}
    kv_lo, kv_hi, cls = oracle.classify_count(seg, 128, 64)
    Tk = cls.shape[2]
    j = np.arange(Tk)
    k0 = 64 * j
    visited = (j >= v["kv_lo"][..., None]) & (j <= v["kv_hi"][..., None])
    full = (v["lo_max"][..., None] <= k0) & (v["hi_min"][..., None]
                                             >= k0 + 63)
    got = np.where(visited, np.where(full, oracle.TILE_FULL,
                                     oracle.TILE_PARTIAL), oracle.TILE_EMPTY)
    np.testing.assert_array_equal(got, cls)
    np.testing.assert_array_equal(v["kv_lo"], kv_lo)
    np.testing.assert_array_equal(v["kv_hi"], kv_hi)
