"""Decode attention (one query token against a long cache of rotated keys)
vs the fp64 oracle, and the key-rotation entry point (needs a B200).

The decode query is the last token of a packed row: its oracle result is
the oracle's forward at that row (attn_fwd_rows), which sees exactly the
keys of its own example.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

OUT_TOL, LSE_TOL = 2e-2, 1e-3


def _case(N, H, B, seed, seg_kind="uniform", dev="cuda", **kw):
    base = wl.WORKLOADS["packed128k"]
    w = wl.Workload("dec", B, N, H, 128, base.theta, seg_kind, base.scale,
                    False, seg_args=kw)
    return wl.make_inputs(w, seed, device=dev)


def test_rope_apply_matches_oracle(cuda_dev):
    t = _case(700, 3, 2, 1, lo=1, hi=300)
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp, device=cuda_dev)
    kr = ops.rope_apply(t["k"], t["positions"], table).float().cpu().numpy()
    pos = t["positions"].cpu().numpy()
    k = t["k"].float().cpu().numpy()
    for b in range(2):
        for h in range(3):
            ref = oracle.rope_rotate(k[b, :, h], pos[b], t["theta"])
            # fp32 rotation then one bf16 rounding: within 2^-8 relative
            assert np.abs(kr[b, :, h] - ref).max() <= 2 ** -8 * np.abs(ref).max()


def _decode_check(t, lengths, heads=None):
    """Query = token lengths[b]-1 of row b; compare with the oracle."""
    B, N, H, D = t["q"].shape
    seg = t["segment_ids"].cpu().numpy()
    pos = t["positions"].cpu().numpy()
    mp = int(pos.max()) + 1
    dev = t["q"].device
    table = ops.rope_table(t["theta"], mp, device=dev)
    k_rot = ops.rope_apply(t["k"], t["positions"], table)
    qi = [L - 1 for L in lengths]
    q = torch.stack([t["q"][b, qi[b]] for b in range(B)])          # [B,H,D]
    start = [int(np.flatnonzero(seg[b] == seg[b, qi[b]])[0]) for b in range(B)]
    kv_start = torch.tensor(start, dtype=torch.int32, device=dev)
    kv_len = torch.tensor(lengths, dtype=torch.int32, device=dev)
    q_pos = torch.tensor([pos[b, qi[b]] for b in range(B)], dtype=torch.int32,
                         device=dev)
    out, lse = ops.decode(q, k_rot, t["v"], kv_start, kv_len, q_pos, table)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    go, gl = out.float().cpu().numpy(), lse.cpu().numpy()
    for b in range(B):
        for h in (range(H) if heads is None else heads):
            ro, rl = oracle.attn_fwd_rows(t["q"], t["k"], t["v"],
                                          t["segment_ids"].cpu(),
                                          t["positions"].cpu(), t["theta"],
                                          b, h, [qi[b]])
            assert np.abs(go[b, h] - ro[0]).max() <= OUT_TOL
            assert abs(gl[b, h] - rl[0]) <= LSE_TOL


def test_decode_packed_rows(cuda_dev):
    t = _case(5000, 4, 2, 2, lo=1, hi=3000)
    _decode_check(t, [5000, 3777])


def test_decode_short_and_single_key(cuda_dev):
    t = _case(300, 2, 2, 3, seg_kind="fixed", length=1)
    _decode_check(t, [300, 1])           # every token its own example


def test_decode_several_chunks_ragged(cuda_dev):
    # caches of 20000 keys: three chunks per (row, head), each streamed in
    # 128-key steps with a ragged last step; the rows' examples start at
    # different offsets, so chunks of one row begin mid-step
    t = _case(20000, 3, 3, 6, lo=1, hi=14000)
    _decode_check(t, [20000, 16385, 9001])


def test_decode_empty_range(cuda_dev):
    t = _case(256, 2, 1, 4, seg_kind="single")
    mp = 256
    table = ops.rope_table(t["theta"], mp, device=cuda_dev)
    k_rot = ops.rope_apply(t["k"], t["positions"], table)
    z = torch.zeros(1, dtype=torch.int32, device=cuda_dev)
    out, lse = ops.decode(t["q"][:, 0], k_rot, t["v"], z + 10, z + 10, z,
                          table)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isinf(lse))


def test_decode_1m_cache(cuda_dev):
    w = wl.WORKLOADS["stress1m"]
    t = wl.make_inputs(w, 5, device=cuda_dev)
    _decode_check(t, [w.N], heads=[0, 31])
