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


# ------------------------------------------------------------ backward

def _bwd_inputs(T, Dm, F, seed, w_std=0.05):
    t = wl.make_ffn_inputs(T, Dm, F, seed=seed, device="cuda", w_std=w_std)
    g = torch.Generator(device="cuda").manual_seed(seed * 16 + 9)
    t["dy"] = torch.randn((T, Dm), generator=g, device="cuda").to(torch.bfloat16)
    return t


def _host64(t):
    return {k: v.float().cpu().numpy().astype(np.float64) for k, v in t.items()}


def _check_bwd_full(t, got):
    """Every element within twice the rounding bound of the bf16
    intermediates: dact, dh, dg and act are rounded once (2^-9 relative),
    and dh, dg also carry dact's rounding; dx is rounded once more."""
    h = _host64(t)
    ref = oracle.swiglu_mlp_bwd(h["x"], h["w_gate"], h["w_up"], h["w_down"],
                                h["dy"])
    A = np.abs
    u = 2.0 ** -9
    bounds = {
        "dx": 2 * (u * A(ref["dx"]) + 2 * u * (A(ref["dh"]) @ A(h["w_gate"])
                                              + A(ref["dg"]) @ A(h["w_up"]))),
        "dw_gate": 2 * 2 * u * (A(ref["dh"]).T @ A(h["x"])),
        "dw_up": 2 * 2 * u * (A(ref["dg"]).T @ A(h["x"])),
        "dw_down": 2 * u * (A(h["dy"]).T @ A(ref["act"])),
    }
    for name, g in zip(("dx", "dw_gate", "dw_up", "dw_down"), got):
        gg = g.float().cpu().numpy()
        err = np.abs(gg - ref[name])
        tol = bounds[name] + 1e-6
        assert np.all(err <= tol), (name, float((err / tol).max()))


@pytest.mark.parametrize("T,Dm,F,chunk", [(1000, 256, 640, 384),
                                          (129, 128, 128, 8192),
                                          (300, 192, 320, 64)])
def test_ffn_backward_matches_oracle(cuda_dev, T, Dm, F, chunk):
    t = _bwd_inputs(T, Dm, F, seed=4)
    got = ops.ffn_bwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], t["dy"],
                      chunk=chunk)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    _check_bwd_full(t, got)


def test_ffn_backward_chunking_changes_only_weight_sum_order(cuda_dev):
    # dx rows depend on their own token only: identical bits for any chunk;
    # the weight gradients are sums over chunks, equal up to fp32 order
    t = _bwd_inputs(1100, 256, 384, seed=5)
    a = ops.ffn_bwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], t["dy"],
                    chunk=256)
    b = ops.ffn_bwd(t["x"], t["w_gate"], t["w_up"], t["w_down"], t["dy"],
                    chunk=1100)
    torch.cuda.synchronize()
    assert torch.equal(a[0], b[0])
    for x, y in zip(a[1:], b[1:]):
        assert (x - y).abs().max().item() <= 1e-5 * y.abs().max().item()


def test_ffn_backward_llama_shape_sampled(cuda_dev):
    # one 8192-token chunk of the Llama-2-7B MLP: dx on sampled rows, the
    # weight gradients on sampled rows, each computed by the oracle over
    # every token
    w = wl.FFN_WORKLOADS["mlp8k"]
    t = _bwd_inputs(w.T, w.Dm, w.F, seed=6, w_std=w.w_std)
    dx, dwg, dwu, dwd = ops.ffn_bwd(t["x"], t["w_gate"], t["w_up"],
                                    t["w_down"], t["dy"], chunk=w.chunk)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    h = _host64(t)
    rng = np.random.default_rng(7)
    rows = np.unique(np.r_[0, w.T - 1, rng.integers(0, w.T, 14)])
    ref = oracle.swiglu_mlp_bwd(h["x"][rows], h["w_gate"], h["w_up"],
                                h["w_down"], h["dy"][rows])
    err = np.abs(dx.float().cpu().numpy()[rows] - ref["dx"])
    assert err.max() <= 2 ** -6 * np.abs(ref["dx"]).max()
    fr = np.unique(np.r_[0, w.F - 1, rng.integers(0, w.F, 6)])
    dr = np.unique(np.r_[0, w.Dm - 1, rng.integers(0, w.Dm, 6)])
    x, dy = h["x"], h["dy"]
    hg = x @ h["w_gate"][fr].T          # [T, |fr|]
    gg = x @ h["w_up"][fr].T
    dact = dy @ h["w_down"][:, fr]
    dh = dact * gg * oracle.silu_grad(hg)
    dg = dact * oracle.silu(hg)
    for got, ref_rows in ((dwg, dh.T @ x), (dwu, dg.T @ x)):
        g_ = got.cpu().numpy()[fr]
        assert np.abs(g_ - ref_rows).max() <= 2 ** -6 * np.abs(ref_rows).max()
    act = oracle.swiglu_intermediate(x, h["w_gate"], h["w_up"])
    ref_d = dy[:, dr].T @ act
    g_ = dwd.cpu().numpy()[dr]
    assert np.abs(g_ - ref_d).max() <= 2 ** -6 * np.abs(ref_d).max()
