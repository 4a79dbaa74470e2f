"""Pins of the blockwise feed-forward oracle (CPU, fp64): SiLU against
torch, the whole MLP against transformers' LlamaMLP with the same weights,
chunking as an exact re-organisation, and closed forms."""

import numpy as np
import pytest
import torch

import oracle


def _weights(seed, T=37, Dm=16, F=40, std=0.3):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, Dm))
    wg = rng.standard_normal((F, Dm)) * std
    wu = rng.standard_normal((F, Dm)) * std
    wd = rng.standard_normal((Dm, F)) * std
    return x, wg, wu, wd


def test_silu_matches_torch():
    h = np.linspace(-60, 60, 1001)
    ref = torch.nn.functional.silu(torch.from_numpy(h)).numpy()
    np.testing.assert_allclose(oracle.silu(h), ref, atol=1e-15, rtol=1e-14)


def test_mlp_matches_transformers_llama_mlp():
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaMLP
    x, wg, wu, wd = _weights(1)
    cfg = LlamaConfig(hidden_size=16, intermediate_size=40, hidden_act="silu",
                      mlp_bias=False, num_attention_heads=2,
                      num_key_value_heads=2)
    mlp = LlamaMLP(cfg).double()
    with torch.no_grad():
        mlp.gate_proj.weight.copy_(torch.from_numpy(wg))
        mlp.up_proj.weight.copy_(torch.from_numpy(wu))
        mlp.down_proj.weight.copy_(torch.from_numpy(wd))
        ref = mlp(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(oracle.swiglu_mlp(x, wg, wu, wd), ref,
                               atol=1e-12, rtol=0)


@pytest.mark.parametrize("chunk", [1, 5, 16, 37, 100])
def test_chunking_is_exact(chunk):
    x, wg, wu, wd = _weights(2)
    np.testing.assert_allclose(oracle.blockwise_mlp(x, wg, wu, wd, chunk),
                               oracle.swiglu_mlp(x, wg, wu, wd), atol=1e-13)


def test_closed_forms():
    x, wg, wu, wd = _weights(3)
    # x = 0 -> y = 0
    assert not oracle.swiglu_mlp(np.zeros_like(x), wg, wu, wd).any()
    # Wu = 0 -> y = 0 whatever the gate
    assert not oracle.swiglu_mlp(x, wg, np.zeros_like(wu), wd).any()
    # one feature, gate weight picks x[0], up picks x[1], down copies to
    # output 2: y[:, 2] = silu(x0) * x1, everything else 0
    Dm, F = 4, 1
    xs = np.random.default_rng(4).standard_normal((9, Dm))
    g = np.zeros((F, Dm)); g[0, 0] = 1.0
    u = np.zeros((F, Dm)); u[0, 1] = 1.0
    d = np.zeros((Dm, F)); d[2, 0] = 1.0
    y = oracle.swiglu_mlp(xs, g, u, d)
    expect = np.zeros_like(xs)
    expect[:, 2] = xs[:, 0] / (1 + np.exp(-xs[:, 0])) * xs[:, 1]
    np.testing.assert_allclose(y, expect, atol=1e-15)


def test_silu_grad_matches_torch_autograd():
    h = torch.linspace(-30, 30, 601, dtype=torch.float64, requires_grad=True)
    torch.nn.functional.silu(h).sum().backward()
    np.testing.assert_allclose(oracle.silu_grad(h.detach().numpy()),
                               h.grad.numpy(), atol=1e-14, rtol=1e-12)


def test_mlp_backward_matches_torch_autograd_of_llama_mlp():
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import LlamaMLP
    x, wg, wu, wd = _weights(5)
    dy = np.random.default_rng(6).standard_normal((x.shape[0], wd.shape[0]))
    cfg = LlamaConfig(hidden_size=16, intermediate_size=40, hidden_act="silu",
                      mlp_bias=False, num_attention_heads=2,
                      num_key_value_heads=2)
    mlp = LlamaMLP(cfg).double()
    with torch.no_grad():
        mlp.gate_proj.weight.copy_(torch.from_numpy(wg))
        mlp.up_proj.weight.copy_(torch.from_numpy(wu))
        mlp.down_proj.weight.copy_(torch.from_numpy(wd))
    xt = torch.from_numpy(x).requires_grad_(True)
    (mlp(xt) * torch.from_numpy(dy)).sum().backward()
    ref = oracle.swiglu_mlp_bwd(x, wg, wu, wd, dy)
    np.testing.assert_allclose(ref["dx"], xt.grad.numpy(), atol=1e-12)
    np.testing.assert_allclose(ref["dw_gate"], mlp.gate_proj.weight.grad.numpy(),
                               atol=1e-12)
    np.testing.assert_allclose(ref["dw_up"], mlp.up_proj.weight.grad.numpy(),
                               atol=1e-12)
    np.testing.assert_allclose(ref["dw_down"], mlp.down_proj.weight.grad.numpy(),
                               atol=1e-12)


def test_mlp_backward_finite_differences():
    x, wg, wu, wd = _weights(7, T=5, Dm=6, F=8)
    dy = np.random.default_rng(8).standard_normal((5, 6))
    ref = oracle.swiglu_mlp_bwd(x, wg, wu, wd, dy)
    f = lambda x_, g_, u_, d_: float((oracle.swiglu_mlp(x_, g_, u_, d_) * dy).sum())
    rng = np.random.default_rng(9)
    eps = 1e-6
    for name, idx in (("dx", 0), ("dw_gate", 1), ("dw_up", 2), ("dw_down", 3)):
        args = [x, wg, wu, wd]
        u = rng.standard_normal(args[idx].shape)
        plus = list(args); plus[idx] = args[idx] + eps * u
        minus = list(args); minus[idx] = args[idx] - eps * u
        num = (f(*plus) - f(*minus)) / (2 * eps)
        assert abs(num - float((ref[name] * u).sum())) <= 1e-6 * max(1, abs(num))
