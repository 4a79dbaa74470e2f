"""CUDA path vs the fp64 oracle on identical seeded inputs (needs a B200).

Tolerances (max abs error):
  bf16 I/O, fp32 accumulate: out <= 2e-2, lse <= 1e-3;
  fp32 I/O: out, lse <= 1e-4;
  backward bf16: dq, dk, dv <= 2e-2 * max|ref| of the tensor;
  backward fp32: <= 1e-4 * max(1, max|ref|);
  classification: bit-exact.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

OUT_TOL_BF16, LSE_TOL_BF16 = 2e-2, 1e-3
TOL_FP32 = 1e-4
BWD_REL_BF16 = 2e-2


def inputs(name, seed, dev, N=None, H=None, B=None, dtype=torch.bfloat16,
           dout=False, seg_kind=None, **seg_args):
    w = wl.WORKLOADS[name]
    if seg_kind is not None:
        w = wl.Workload(w.name, w.B, w.N, w.H, w.D, w.theta, seg_kind,
                        w.scale, w.backward, seg_args=seg_args)
    return wl.make_inputs(w, seed, device=dev, dtype=dtype, N=N, H=H, B=B,
                          with_dout=dout)


def host(t):
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in t.items()}


def run_fwd(t, qkp="bf16"):
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], t["theta"], qk_precision=qkp)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    return out, lse


def check_fwd_full(t, out, lse, out_tol, lse_tol):
    h = host(t)
    ro, rl = oracle.attn_fwd(h["q"], h["k"], h["v"], h["segment_ids"],
                             h["positions"], t["theta"])
    go = out.float().cpu().numpy()
    gl = lse.cpu().numpy()
    eo = np.abs(go - ro).max()
    el = np.abs(gl - rl).max()
    assert np.isfinite(go).all() and np.isfinite(gl).all()
    assert eo <= out_tol, f"max|out-ref|={eo}"
    assert el <= lse_tol, f"max|lse-ref|={el}"
    return eo, el


# ------------------------------------------------------------ aux kernels

@pytest.mark.parametrize("theta,max_pos", [(1e4, 4096), (5e7, 70000),
                                           (1e6, 1)])
def test_rope_table_matches_oracle(cuda_dev, theta, max_pos):
    t = ops.rope_table(theta, max_pos, device=cuda_dev).cpu().numpy()
    ang = oracle.rope_angles(np.arange(max_pos), theta, 128)
    ref = np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32)
    # both round an fp64 value to fp32; a 1-ulp fp64 difference may flip it
    assert np.abs(t - ref).max() <= 1.2e-7


@pytest.mark.parametrize("seed,N,B,bq,bk,lo,hi", [
    (0, 2048, 1, 128, 128, 64, 1024),
    (1, 3001, 2, 128, 128, 1, 700),
    (2, 2500, 1, 128, 64, 1, 300),
    (3, 1000, 3, 64, 64, 1, 50),
    (4, 4096, 1, 256, 128, 100, 2000),
    (5, 77, 1, 128, 128, 1, 10),
])
def test_classify_bit_exact_vs_bruteforce(cuda_dev, seed, N, B, bq, bk, lo,
                                          hi):
    segs = []
    for b in range(B):
        L = wl.segment_lengths("uniform", N, seed * 10 + b, lo=lo, hi=hi)
        segs.append(wl.segments_from_lengths(L)[0])
    seg = np.stack(segs)
    g = ops.classify(torch.from_numpy(seg).to(cuda_dev), bq, bk)
    r = oracle.classify_bruteforce(seg, bq, bk)
    for x, y in zip(g, r):
        np.testing.assert_array_equal(x.cpu().numpy(), y)


@pytest.mark.parametrize("name", ["text32k", "packed128k", "vl256k"])
def test_classify_bit_exact_full_size(cuda_dev, name):
    w = wl.WORKLOADS[name]
    seg, _, _ = wl.make_segments(w, 0)
    g = ops.classify(torch.from_numpy(seg).to(cuda_dev))
    r = oracle.classify_count(seg, 128, 128)
    for x, y in zip(g, r):
        np.testing.assert_array_equal(x.cpu().numpy(), y)


def test_check_inputs(cuda_dev):
    L = wl.segment_lengths("uniform", 5000, 3, lo=1, hi=900)
    seg, pos = wl.segments_from_lengths(L)
    s = torch.from_numpy(seg[None]).to(cuda_dev)
    p = torch.from_numpy(pos[None]).to(cuda_dev)
    ok, mp = ops.check_inputs(s, p, 10 ** 6)
    assert ok and mp == int(pos.max()) + 1
    ok, _ = ops.check_inputs(s, p, int(pos.max()))  # a position == max_pos
    assert not ok
    s2 = s.clone()
    s2[0, 100] = s2[0, 99] - 1
    ok, _ = ops.check_inputs(s2, p, 10 ** 6)
    assert not ok
    p2 = p.clone()
    p2[0, 7] = -1
    ok, _ = ops.check_inputs(s, p2, 10 ** 6)
    assert not ok


# --------------------------------------------------------------- forward

def test_fwd_tiny2k_split_qk_full(cuda_dev):
    # N(0,1) inputs: scores need the hi/lo split of rotated q, k
    t = inputs("tiny2k", 0, cuda_dev)
    out, lse = run_fwd(t, "bf16x3")
    check_fwd_full(t, out, lse, OUT_TOL_BF16, LSE_TOL_BF16)


@pytest.mark.parametrize("seed", [1, 2])
def test_fwd_tiny2k_split_qk_other_seeds(cuda_dev, seed):
    t = inputs("tiny2k", seed, cuda_dev)
    out, lse = run_fwd(t, "bf16x3")
    check_fwd_full(t, out, lse, OUT_TOL_BF16, LSE_TOL_BF16)


@pytest.mark.parametrize("N,B,H,lo,hi", [
    (3000, 2, 3, 1, 900),      # ragged tail, several batch rows
    (4096, 1, 4, 512, 4096),   # several tiles, long segments
    (1024, 1, 2, 1, 3),        # many tiny segments
])
def test_fwd_bf16_scaled_full(cuda_dev, N, B, H, lo, hi):
    t = inputs("packed128k", 7, cuda_dev, N=N, H=H, B=B, seg_kind="uniform",
               lo=lo, hi=hi)
    out, lse = run_fwd(t, "bf16")
    check_fwd_full(t, out, lse, OUT_TOL_BF16, LSE_TOL_BF16)


@pytest.mark.parametrize("N", [1, 2, 127, 128, 129, 255, 257])
def test_fwd_edge_sizes(cuda_dev, N):
    t = inputs("tiny2k", 3, cuda_dev, N=N, H=2, B=2)
    out, lse = run_fwd(t, "bf16x3")
    check_fwd_full(t, out, lse, OUT_TOL_BF16, LSE_TOL_BF16)


def test_fwd_every_token_its_own_segment(cuda_dev):
    t = inputs("tiny2k", 4, cuda_dev, N=300, H=2, seg_kind="fixed", length=1)
    out, lse = run_fwd(t, "bf16x3")
    check_fwd_full(t, out, lse, OUT_TOL_BF16, LSE_TOL_BF16)
    # a length-1 segment returns its own v row exactly (up to bf16 output)
    torch.testing.assert_close(out, t["v"], atol=0, rtol=0)


def test_fwd_fp32(cuda_dev):
    t = inputs("tiny2k", 5, cuda_dev, N=700, H=2, B=2, dtype=torch.float32)
    out, lse = run_fwd(t)
    check_fwd_full(t, out, lse, TOL_FP32, TOL_FP32)


def test_fwd_empty_batch_is_a_no_op(cuda_dev):
    t = inputs("tiny2k", 0, cuda_dev, N=0, H=2, B=1)
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], 1e4, max_pos=1)
    assert out.numel() == 0 and lse.numel() == 0


@pytest.mark.parametrize("name,rows,heads", [
    ("text32k", 128, None),
    ("packed128k", 128, None),
    ("vl256k", 64, None),
])
def test_fwd_full_size_sampled_rows(cuda_dev, name, rows, heads):
    w = wl.WORKLOADS[name]
    t = inputs(name, 0, cuda_dev)
    out, lse = run_fwd(t, "bf16")
    check_sampled_rows(t, out, lse, rows, heads, seed=11)


def check_sampled_rows(t, out, lse, nrows, heads, seed):
    # the oracle pulls one head of K/V (and the sampled Q rows) at a time,
    # so no full host copy of the 1M-token inputs is made
    N = t["q"].shape[1]
    H = t["q"].shape[2]
    rng = np.random.default_rng(seed)
    rows = np.unique(np.r_[0, N - 1, rng.integers(0, N, nrows - 2)])
    h = {k: (v.cpu() if k in ("segment_ids", "positions") else v)
         for k, v in t.items()}
    heads = range(H) if heads is None else heads
    go = out[0, torch.from_numpy(rows).to(out.device)].float().cpu().numpy()
    gl = lse[0][:, torch.from_numpy(rows).to(lse.device)].cpu().numpy()
    eo = el = 0.0
    for hh in heads:
        ro, rl = oracle.attn_fwd_rows(h["q"], h["k"], h["v"],
                                      h["segment_ids"], h["positions"],
                                      t["theta"], 0, hh, rows)
        eo = max(eo, np.abs(go[:, hh] - ro).max())
        el = max(el, np.abs(gl[hh] - rl).max())
    assert eo <= OUT_TOL_BF16, eo
    assert el <= LSE_TOL_BF16, el


def test_fwd_1m_sampled_rows(cuda_dev):
    t = inputs("stress1m", 0, cuda_dev)
    out, lse = run_fwd(t, "bf16")
    check_sampled_rows(t, out, lse, 24, [0, 13, 31], seed=12)


# -------------------------------------------------------------- backward

def run_bwd(t, qkp="bf16"):
    out, lse = run_fwd(t, qkp)
    dq, dk, dv = ops.bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                         t["segment_ids"], t["positions"], t["theta"],
                         qk_precision=qkp)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    return dq, dk, dv


def check_bwd_full(t, grads, rel, floor):
    h = host(t)
    ref = oracle.attn_bwd(h["q"], h["k"], h["v"], h["dout"],
                          h["segment_ids"], h["positions"], t["theta"])
    for name, g in zip(("dq", "dk", "dv"), grads):
        gg = g.float().cpu().numpy()
        r = ref[name]
        assert np.isfinite(gg).all(), name
        tol = rel * max(floor, np.abs(r).max())
        err = np.abs(gg - r).max()
        assert err <= tol, f"{name}: max err {err} > {tol}"


@pytest.mark.parametrize("N,H,lo,hi", [(1500, 2, 1, 700), (1024, 2, 1024,
                                                            1024),
                                       (777, 1, 1, 40)])
def test_bwd_bf16_full(cuda_dev, N, H, lo, hi):
    t = inputs("packed128k", 8, cuda_dev, N=N, H=H, seg_kind="uniform",
               lo=lo, hi=hi, dout=True)
    check_bwd_full(t, run_bwd(t), BWD_REL_BF16, 0.0)


def test_bwd_fp32(cuda_dev):
    t = inputs("tiny2k", 9, cuda_dev, N=400, H=2, B=2, dtype=torch.float32,
               dout=True)
    check_bwd_full(t, run_bwd(t), TOL_FP32, 1.0)


def test_bwd_bf16_split_qk_tiny(cuda_dev):
    t = inputs("tiny2k", 10, cuda_dev, N=600, H=2, dout=True)
    check_bwd_full(t, run_bwd(t, "bf16x3"), BWD_REL_BF16, 0.0)


def check_bwd_rows(h, t, dq, rows, heads):
    idx = torch.from_numpy(rows).to(dq.device)
    gq = dq[0, idx].float().cpu().numpy()
    for hh in heads:
        r = oracle.attn_bwd_rows(h["q"], h["k"], h["v"], h["dout"],
                                 h["segment_ids"], h["positions"],
                                 t["theta"], 0, hh, rows)
        err = np.abs(gq[:, hh] - r).max()
        assert err <= BWD_REL_BF16 * np.abs(r).max(), (hh, err)


def check_bwd_cols(h, t, dk, dv, a, z, cols, heads):
    """dk, dv at keys ``cols`` (global indices in [a, z)) against the oracle
    run on tokens [a, z). With a, z the bounds of the packed example that
    holds the keys (or the whole row) nothing outside [a, z) sees them or
    is seen by the rows that do, so the oracle on that slice is the oracle
    on the whole row."""
    sl = {k_: h[k_][:, a:z] for k_ in ("q", "k", "v", "dout", "segment_ids",
                                       "positions")}
    idx = torch.from_numpy(cols).to(dk.device)
    gk = dk[0, idx].float().cpu().numpy()
    gv = dv[0, idx].float().cpu().numpy()
    for hh in heads:
        rk, rv = oracle.attn_bwd_cols(sl["q"], sl["k"], sl["v"], sl["dout"],
                                      sl["segment_ids"], sl["positions"],
                                      t["theta"], 0, hh, cols - a,
                                      row_block=1024)
        ek = np.abs(gk[:, hh] - rk).max()
        ev = np.abs(gv[:, hh] - rv).max()
        assert ek <= BWD_REL_BF16 * np.abs(rk).max(), (hh, ek)
        assert ev <= BWD_REL_BF16 * np.abs(rv).max(), (hh, ev)


def test_bwd_text32k_full_size_sampled(cuda_dev):
    # the 32K workload at full size: dq on 64 rows of 2 heads, dk and dv on
    # 64 keys of 4 heads (each key column needs the whole head's forward)
    t = inputs("text32k", 0, cuda_dev, dout=True)
    dq, dk, dv = run_bwd(t)
    h = host(t)
    N = t["q"].shape[1]
    rng = np.random.default_rng(21)
    rows = np.unique(np.r_[0, N - 1, rng.integers(0, N, 62)])
    check_bwd_rows(h, t, dq, rows, (0, 17))
    check_bwd_cols(h, t, dk, dv, 0, N, rows, (5, 12, 20, 31))


def test_bwd_packed128k_full_size_sampled(cuda_dev):
    # the 128K packed workload (seed 0) in the benchmark's launch
    # configuration: dq on the first and last token of every example plus
    # random rows; dk, dv on the first and last key and random keys of six
    # examples (short to 22.8K tokens); four heads each
    t = inputs("packed128k", 0, cuda_dev, dout=True)
    dq, dk, dv = run_bwd(t)
    h = host(t)
    L = t["lengths"][0]
    starts = np.r_[0, np.cumsum(L)[:-1]]
    ends = starts + L - 1
    rng = np.random.default_rng(31)
    N = t["q"].shape[1]
    rows = np.unique(np.r_[starts, ends, rng.integers(0, N, 40)])
    assert len(rows) >= 64
    check_bwd_rows(h, t, dq, rows, (0, 9, 22, 31))
    picked = [i for i in np.argsort(L) if L[i] <= 23000]
    docs = picked[:4] + picked[-2:]  # the four shortest and two long ones
    ncols = 0
    for i in docs:
        a, z = int(starts[i]), int(ends[i]) + 1
        cols = np.unique(np.r_[a, z - 1, rng.integers(a, z, 10)])
        check_bwd_cols(h, t, dk, dv, a, z, cols, (0, 9, 22, 31))
        ncols += len(cols)
    assert ncols >= 64
