"""Blockwise SwiGLU feed-forward on the GPU vs the fp64 oracle.

Tolerance from the arithmetic: the tensor cores form the bf16 x bf16
products exactly and add them in fp32; the intermediate act is rounded to
bf16 once (|d act| <= 2^-9 |act|) and so is y (2^-9 |y|). So per output
element |y - y_ref| <= 2^-9 |y_ref| + 2^-9 sum_k |act_k| |Wd_jk| plus fp32
summation terms far below these; the tests allow twice that."""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _bound_check(y, t, rows=None):
    h = {k: v.float().cpu().numpy().astype(np.float64) for k, v in t.items()}
    x = h["x"] if rows is None else h["x"][rows]
    act = oracle.swiglu_intermediate(x, h["w_gate"], h["w_up"])
    ref = act @ h["w_down"].T
    tol = 2.0 * 2 ** -9 * (np.abs(ref) + np.abs(act) @ np.abs(h["w_down"]).T)
    got = y.float().cpu().numpy()
    if rows is not None:
        got = got[rows]
    err = np.abs(got - ref)
    assert np.all(err <= tol), float((err / np.maximum(tol, 1e-30)).max())
    return err.max(), np.abs(ref).max()


@pytest.mark.parametrize("T,Dm,F,chunk", [(1000, 512, 1536, 384),
                                          (1000, 512, 1536, 1000),
                                          (129, 256, 640, 8192),
                                          (1, 128, 128, 8192)])
def test_ffn_matches_oracle(cuda_dev, T, Dm, F, chunk):
    t = wl.make_ffn_inputs(T, Dm, F, seed=1, device="cuda", w_std=0.05)
    y = ops.ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], chunk=chunk)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    _bound_check(y, t)


def test_ffn_chunking_changes_nothing(cuda_dev):
    # every output row depends on its own token only and each tile sums K
    # in the same order: any chunk size gives the same bits
    t = wl.make_ffn_inputs(1100, 256, 768, seed=2, device="cuda", w_std=0.05)
    args = (t["x"], t["w_gate"], t["w_up"], t["w_down"])
    ys = [ops.ffn_fwd(*args, chunk=c) for c in (128, 300, 1100)]
    torch.cuda.synchronize()
    assert torch.equal(ys[0], ys[1]) and torch.equal(ys[0], ys[2])


def test_ffn_empty_and_rejects(cuda_dev):
    t = wl.make_ffn_inputs(0, 128, 128, seed=3, device="cuda")
    assert ops.ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"]).numel() == 0
    t = wl.make_ffn_inputs(4, 96, 128, seed=3, device="cuda")
    with pytest.raises(ops.LwmError):
        ops.ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"])


def test_ffn_llama_shape_sampled_rows(cuda_dev):
    # the bench configuration: Llama-2-7B MLP (4096 -> 11008 -> 4096) over
    # 32K tokens in chunks of 8192
    w = wl.FFN_WORKLOADS["mlp32k"]
    t = wl.make_ffn_inputs(w.T, w.Dm, w.F, seed=0, device="cuda",
                           w_std=w.w_std)
    y = ops.ffn_fwd(t["x"], t["w_gate"], t["w_up"], t["w_down"],
                    chunk=w.chunk)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    rng = np.random.default_rng(5)
    rows = np.unique(np.r_[0, w.chunk - 1, w.chunk, w.T - 1,
                           rng.integers(0, w.T, 28)])
    _bound_check(y, {k: v for k, v in t.items()}, rows=rows)
