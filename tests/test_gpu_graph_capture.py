"""The forward and backward calls inside a CUDA graph (needs a B200).

With max_pos, the outputs and the workspace given by the caller, a call
does no host synchronisation and no allocation, so it can be captured into
a CUDA graph (stream capture) and replayed; the replay must give the same
bits as the eager calls on the same inputs (the forward is deterministic;
dK, dV accumulate per key block in TMEM; dQ sums fp32 partials in arrival
order and is compared within the bf16 tolerance). The launch-bound small
calls are where replay pays: it removes the host work per call.
"""

import pytest
import torch

from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _case(dev):
    base = wl.WORKLOADS["packed128k"]
    w = wl.Workload("graph", 1, 4096, 4, 128, base.theta, "uniform",
                    base.scale, True, seg_args={"lo": 200, "hi": 2500})
    return wl.make_inputs(w, 7, device=dev)


def test_fwd_bwd_replay_matches_eager(cuda_dev):
    t = _case(cuda_dev)
    B, N, H, D = t["q"].shape
    mp = int(t["positions"].max()) + 1
    ws = torch.empty(max(ops.fwd_workspace_size(B, N, H, mp),
                         ops.bwd_workspace_size(B, N, H, mp)),
                     dtype=torch.uint8, device=cuda_dev)
    out = torch.empty_like(t["q"])
    lse = torch.empty((B, H, N), dtype=torch.float32, device=cuda_dev)
    dq, dk, dv = (torch.empty_like(t["q"]) for _ in range(3))

    def step(stream=None):
        ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"], t["positions"],
                t["theta"], max_pos=mp, out=out, lse=lse, workspace=ws,
                stream=stream)
        ops.bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                t["segment_ids"], t["positions"], t["theta"], max_pos=mp,
                dq=dq, dk=dk, dv=dv, workspace=ws, stream=stream)

    step()
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    ref = [x.clone() for x in (out, lse, dq, dk, dv)]

    s = torch.cuda.Stream(cuda_dev)
    with torch.cuda.stream(s):
        step(stream=s)  # warm the side stream before capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        step(stream=s)
    torch.cuda.synchronize()
    for x in (out, lse, dq, dk, dv):
        x.zero_()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    assert torch.equal(out, ref[0])
    assert torch.equal(lse, ref[1])
    assert torch.equal(dk, ref[3])
    assert torch.equal(dv, ref[4])
    tol = 2e-2 * ref[2].float().abs().max().item()
    assert (dq.float() - ref[2].float()).abs().max().item() <= tol
