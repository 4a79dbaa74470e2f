"""Failure detection on the GPU without a GPU fault (needs a B200).

A kernel whose bounded mbarrier wait can never complete must give up after
its limit, record LWM_ERR_TIMEOUT in the device status word, and leave the
CUDA context usable: the status is read and cleared on the host, and the
next attention call runs normally.
"""

import pytest
import torch

from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_dev):
    assert ops.last_status() == ops.OK
    ops.selftest_wait_timeout(20_000_000)          # 20 ms, nothing arrives
    assert ops.last_status() == ops.ERR_TIMEOUT    # reported ...
    assert ops.last_status() == ops.OK             # ... and cleared
    w = wl.WORKLOADS["packed128k"]
    t = wl.make_inputs(w, 1, device=cuda_dev, N=512, H=2)
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], w.theta)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()


def test_invalid_arguments_launch_nothing(cuda_dev):
    w = wl.WORKLOADS["packed128k"]
    t = wl.make_inputs(w, 2, device=cuda_dev, N=256, H=1)
    before = ops.kernel_launches()
    with pytest.raises(ops.LwmError) as e:
        ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"], t["positions"],
                -1.0)                                # theta must be > 0
    assert e.value.status == ops.ERR_INVALID_ARG
    with pytest.raises(ops.LwmError) as e:
        ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"], t["positions"],
                w.theta, workspace=torch.empty(16, dtype=torch.uint8,
                                               device=cuda_dev))
    assert e.value.status == ops.ERR_WORKSPACE
    assert ops.kernel_launches() == before
