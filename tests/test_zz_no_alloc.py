"""lwm_blockattn_fwd_noalloc against the regular forward (needs a B200).

Some callers cannot allocate device memory while they run (a serving loop
that must not let cudaMalloc synchronise the device, or a C host with no
device allocator). For them the library keeps its forward scratch in one
fixed device array. These checks call that entry point through the C ABI
three times in a row, on different inputs and modes, and compare each
result with the regular lwm_blockattn_fwd on the same inputs. Both run the
same deterministic kernels, so the results must be identical bit for bit:
a later call must not be disturbed in the least by what an earlier one
left in the shared array.

This file is named so that pytest collects it last.
"""

import ctypes

import pytest
import torch

from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

def _inputs(name, seed, dev, **kw):
    w = wl.WORKLOADS[name]
    seg_kind = kw.pop("seg_kind", None)
    if seg_kind:
        w = wl.Workload(w.name, w.B, w.N, w.H, w.D, w.theta, seg_kind,
                        w.scale, w.backward, seg_args=kw.pop("seg_args"))
    return wl.make_inputs(w, seed, device=dev, **kw)


def _compare(t, qkp, layout="interleaved"):
    max_pos = int(t["positions"].max().item()) + 1
    ref_out, ref_lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                               t["positions"], t["theta"], max_pos=max_pos,
                               qk_precision=qkp, rope_layout=layout)
    out = torch.full_like(t["q"], float("nan"))
    lse = torch.full_like(ref_lse, float("nan"))
    ops.fwd_noalloc(t["q"], t["k"], t["v"], t["segment_ids"],
                    t["positions"], t["theta"], max_pos, qk_precision=qkp,
                    out=out, lse=lse, rope_layout=layout)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    assert torch.isfinite(out.float()).all() and torch.isfinite(lse).all()
    assert torch.equal(out, ref_out)
    assert torch.equal(lse, ref_lse)


def test_noalloc_forward_equals_regular_forward_over_calls(cuda_dev):
    # call 1: the small N(0,1) case in the split-QK mode
    _compare(_inputs("tiny2k", 0, cuda_dev), "bf16x3")
    # call 2: a different shape, packing and mode; the shared scratch still
    # holds call 1's tables
    _compare(_inputs("packed128k", 3, cuda_dev, N=1500, H=3, B=2,
                     seg_kind="uniform", seg_args={"lo": 1, "hi": 600}),
             "bf16")
    # call 3: fp32 I/O (the CUDA-core path, which carves and reads the
    # array differently) with the rotate-half layout, after two calls have
    # left their metadata and rotated keys in it
    _compare(_inputs("tiny2k", 5, cuda_dev, N=700, H=2, B=2,
                     dtype=torch.float32), "bf16", layout="half")


def test_noalloc_rejects_sizes_beyond_its_scratch(cuda_dev):
    # a 256K x 32-head forward needs far more than the fixed array; the
    # call must refuse before touching any pointer or launching anything
    fake = ctypes.c_void_p(1 << 20)
    st = ops.lib().lwm_blockattn_fwd_noalloc(
        fake, fake, fake, fake, fake, 5e7, 128, 128, 262144, 1, 262144, 32,
        128, ops.DTYPE_BF16, ops.QK_BF16, ops.ROPE_INTERLEAVED, fake, fake,
        None)
    assert st == ops.ERR_WORKSPACE
