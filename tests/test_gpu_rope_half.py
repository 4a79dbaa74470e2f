"""The rotate-half RoPE layout (Hugging Face Llama checkpoints; "LWM：突破
100 万 Token 的开源大模型", 脚本运行说明) on the GPU, against the fp64
oracle. The oracle pins (tests/test_oracle.py) show that attention on
rotate-half inputs equals the oracle on inputs permuted to the interleaved
layout, with gradients permuted back; these tests use that reading."""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops, ring
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

OUT_TOL, LSE_TOL, BWD_REL = 2e-2, 1e-3, 2e-2
H2I = oracle.half_to_interleaved
I2H = oracle.interleaved_to_half


def _case(name, N, H, B, seed, dtype=torch.bfloat16, **seg):
    base = wl.WORKLOADS[name]
    w = wl.Workload("half", B, N, H, 128, base.theta, "uniform", base.scale,
                    True, seg_args=seg or {"lo": 1, "hi": 700})
    return wl.make_inputs(w, seed, device="cuda", dtype=dtype,
                          with_dout=True)


def _host(t):
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in t.items()}


def _np(x):
    return x.float().cpu().numpy() if torch.is_tensor(x) else x


def test_rope_apply_half_matches_oracle(cuda_dev):
    t = _case("packed128k", 600, 3, 2, 1)
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp)
    kr = _np(ops.rope_apply(t["k"], t["positions"], table, rope_layout="half"))
    k, pos = _np(t["k"]), t["positions"].cpu().numpy()
    for b in range(2):
        for h in range(3):
            ref = oracle.rope_rotate_half(k[b, :, h], pos[b], t["theta"])
            assert np.abs(kr[b, :, h] - ref).max() <= 2 ** -8 * np.abs(ref).max()


@pytest.mark.parametrize("qkp,name", [("bf16", "packed128k"),
                                      ("bf16x3", "tiny2k")])
def test_forward_half_matches_oracle(cuda_dev, qkp, name):
    t = _case(name, 1500, 2, 2, 2)
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], t["theta"], qk_precision=qkp,
                       rope_layout="half")
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    h = _host(t)
    ro, rl = oracle.attn_fwd(H2I(_np(h["q"])), H2I(_np(h["k"])), h["v"],
                             h["segment_ids"], h["positions"], t["theta"])
    assert np.abs(_np(out) - ro).max() <= OUT_TOL
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_TOL


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_backward_half_matches_oracle(cuda_dev, dtype):
    t = _case("packed128k", 900, 2, 1, 3, dtype=dtype)
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], t["theta"], rope_layout="half")
    dq, dk, dv = ops.bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                         t["segment_ids"], t["positions"], t["theta"],
                         rope_layout="half")
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    h = _host(t)
    ref = oracle.attn_bwd(H2I(_np(h["q"])), H2I(_np(h["k"])), _np(h["v"]),
                          _np(h["dout"]), h["segment_ids"], h["positions"],
                          t["theta"])
    rel = BWD_REL if dtype == torch.bfloat16 else 1e-4
    for name, g, r in (("dq", dq, I2H(ref["dq"])), ("dk", dk, I2H(ref["dk"])),
                       ("dv", dv, ref["dv"])):
        err = np.abs(_np(g) - r).max()
        assert err <= rel * max(1.0 if dtype == torch.float32 else 0.0,
                                np.abs(r).max()), f"{name}: {err}"


def _decode_half_check(N, lengths, lo, hi):
    B = len(lengths)
    t = _case("packed128k", N, 2, B, 4, lo=lo, hi=hi)
    seg = t["segment_ids"].cpu().numpy()
    pos = t["positions"].cpu().numpy()
    mp = int(pos.max()) + 1
    table = ops.rope_table(t["theta"], mp)
    k_rot = ops.rope_apply(t["k"], t["positions"], table, rope_layout="half")
    qi = [L - 1 for L in lengths]
    q = torch.stack([t["q"][b, qi[b]] for b in range(B)])
    start = [int(np.flatnonzero(seg[b] == seg[b, qi[b]])[0]) for b in range(B)]
    kv_start = torch.tensor(start, dtype=torch.int32, device="cuda")
    kv_len = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    q_pos = torch.tensor([pos[b, qi[b]] for b in range(B)], dtype=torch.int32,
                         device="cuda")
    out, lse = ops.decode(q, k_rot, t["v"], kv_start, kv_len, q_pos, table,
                          rope_layout="half")
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    h = _host(t)
    for b in range(B):
        for hh in range(2):
            o, l_ = oracle.attn_fwd_rows(H2I(_np(h["q"])), H2I(_np(h["k"])),
                                         h["v"], h["segment_ids"],
                                         h["positions"], t["theta"], b, hh,
                                         [qi[b]])
            assert np.abs(_np(out[b, hh]) - o[0]).max() <= OUT_TOL
            assert abs(float(lse[b, hh]) - l_[0]) <= LSE_TOL


def test_decode_half_matches_oracle(cuda_dev):
    _decode_half_check(700, [700, 531], 100, 400)


def test_decode_half_several_chunks(cuda_dev):
    # 20000-key caches: three chunks per (row, head), ragged last steps,
    # examples long enough to span chunk boundaries
    _decode_half_check(20000, [20000, 17001], 3000, 12000)


def test_ring_half_matches_oracle(cuda_dev):
    t = _case("packed128k", 1200, 2, 1, 5)
    mp = int(t["positions"].max()) + 1
    be = ring.CudaBackend(t["theta"], mp, rope_layout="half")
    out, lse = ring.simulate_ring_fwd(t["q"], t["k"], t["v"],
                                      t["segment_ids"], t["positions"], 3, be)
    dq, dk, dv = ring.simulate_ring_bwd(t["q"], t["k"], t["v"], out,
                                        t["dout"], lse, t["segment_ids"],
                                        t["positions"], 3, be)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    h = _host(t)
    ref = oracle.attn_bwd(H2I(_np(h["q"])), H2I(_np(h["k"])), _np(h["v"]),
                          _np(h["dout"]), h["segment_ids"], h["positions"],
                          t["theta"])
    assert np.abs(_np(out) - ref["out"]).max() <= OUT_TOL
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= LSE_TOL
    for name, g, r in (("dq", dq, I2H(ref["dq"])), ("dk", dk, I2H(ref["dk"])),
                       ("dv", dv, ref["dv"])):
        err = np.abs(_np(g) - r).max()
        assert err <= BWD_REL * np.abs(r).max(), f"{name}: {err}"
