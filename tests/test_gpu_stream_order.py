"""Stream order around the library's calls (needs a B200).

The kernels of one call are launched as programmatic dependent launches:
each may be scheduled while the kernel before it on the stream still runs,
and waits (griddepcontrol) before it touches memory. These tests put a
torch kernel that rewrites the inputs directly before each call on the same
stream, and one that reads the outputs directly after it, with no host
synchronisation in between, and require the results to be bit-identical to
the same calls made after a full device synchronisation. The forward,
backward and decode kernels are deterministic for fixed inputs (atomics
only hand out work or add fp32 dQ partials, whose order the tests do not
rely on: dQ is compared within the bf16 tolerance).
"""

import pytest
import torch

from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _case(dev, seed=3):
    base = wl.WORKLOADS["packed128k"]
    w = wl.Workload("order", 2, 3000, 4, 128, base.theta, "uniform",
                    base.scale, True, seg_args={"lo": 100, "hi": 1500})
    return wl.make_inputs(w, seed, device=dev)


def _fwd(t, q):
    return ops.fwd(q, t["k"], t["v"], t["segment_ids"], t["positions"],
                   t["theta"], max_pos=int(t["positions"].max()) + 1)


def test_fwd_sees_inputs_written_just_before_it(cuda_dev):
    t = _case(cuda_dev)
    q = t["q"].clone()
    # reference: each call on inputs that are settled on the device
    refs = []
    for step in range(3):
        torch.cuda.synchronize()
        q_step = (t["q"] * (1.0 - 0.25 * step)).contiguous()
        torch.cuda.synchronize()
        out, lse = _fwd(t, q_step)
        torch.cuda.synchronize()
        refs.append((out.clone(), lse.clone()))
    # the same calls, each right after a torch kernel that rewrites q, and
    # followed by a torch kernel that reads the result, all on one stream
    outs = []
    for step in range(3):
        torch.mul(t["q"], 1.0 - 0.25 * step, out=q)
        out, lse = _fwd(t, q)
        outs.append((out.float().sum(), out, lse))
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    for (s, out, lse), (r_out, r_lse) in zip(outs, refs):
        assert torch.equal(out, r_out)
        assert torch.equal(lse, r_lse)
        assert torch.equal(s, r_out.float().sum())


def test_bwd_sees_gradients_written_just_before_it(cuda_dev):
    t = _case(cuda_dev, seed=4)
    mp = int(t["positions"].max()) + 1
    out, lse = _fwd(t, t["q"])
    torch.cuda.synchronize()
    dout = torch.empty_like(t["dout"])

    def bwd():
        return ops.bwd(t["q"], t["k"], t["v"], out, dout, lse,
                       t["segment_ids"], t["positions"], t["theta"],
                       max_pos=mp)

    dout.copy_(t["dout"] * 0.5)
    torch.cuda.synchronize()
    ref = [g.clone() for g in bwd()]
    torch.cuda.synchronize()
    dout.zero_()
    torch.cuda.synchronize()
    # rewrite dO on the stream and call at once
    torch.mul(t["dout"], 0.5, out=dout)
    got = bwd()
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    dq, dk, dv = got
    # dK and dV are accumulated in TMEM per key block: bit-identical
    assert torch.equal(dk, ref[1])
    assert torch.equal(dv, ref[2])
    # dQ sums fp32 partials from several key blocks in arrival order
    tol = 2e-2 * ref[0].float().abs().max().item()
    assert (dq.float() - ref[0].float()).abs().max().item() <= tol


def test_decode_sees_cache_written_just_before_it(cuda_dev):
    t = _case(cuda_dev, seed=5)
    B, N, H, D = t["q"].shape
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp, device=cuda_dev)
    k_rot = ops.rope_apply(t["k"], t["positions"], table)
    start = torch.zeros(B, dtype=torch.int32, device=cuda_dev)
    length = torch.full((B,), N, dtype=torch.int32, device=cuda_dev)
    q_pos = t["positions"][:, -1].contiguous()
    q = t["q"][:, -1].contiguous()
    v = t["v"].clone()
    torch.cuda.synchronize()
    v.mul_(2.0)
    torch.cuda.synchronize()
    ref_out, ref_lse = ops.decode(q, k_rot, v, start, length, q_pos, table)
    torch.cuda.synchronize()
    v.copy_(t["v"])
    torch.cuda.synchronize()
    v.mul_(2.0)  # on the stream, immediately before the call
    out, lse = ops.decode(q, k_rot, v, start, length, q_pos, table)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)
