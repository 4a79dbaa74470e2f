"""Blockwise SwiGLU feed-forward network in fp64 (oracle; test infra only).

The MLP half of the blockwise transformer runs over the sequence in chunks
of scan_mlp_chunk_size tokens ("LWM：突破 100 万 Token 的开源大模型",
配置参数: scan_mlp, scan_mlp_chunk_size = 8192); the block is Llama-2's
("Inside Large World Model", Core Architecture): gate and up projections, a
SiLU gate, a down projection. Chunking is an exact re-organisation: every
token's output depends on that token alone.

Readings (the pages name the model, not the formula): Llama's MLP,
y = (silu(x Wg^T) * (x Wu^T)) Wd^T with silu(h) = h / (1 + e^-h), weights in
nn.Linear layout (row = output feature), no biases.
"""

import numpy as np

from .attention import _f64


def silu(h):
    """h * sigmoid(h), written as h / (1 + e^-h)."""
    h = np.asarray(h, dtype=np.float64)
    return h / (1.0 + np.exp(-h))


def swiglu_intermediate(x, w_gate, w_up):
    """act [T, F] = silu(x Wg^T) * (x Wu^T)."""
    x = _f64(x)
    return silu(x @ _f64(w_gate).T) * (x @ _f64(w_up).T)


def swiglu_mlp(x, w_gate, w_up, w_down):
    """y [T, Dm] for x [T, Dm], Wg, Wu [F, Dm], Wd [Dm, F]."""
    return swiglu_intermediate(x, w_gate, w_up) @ _f64(w_down).T


def blockwise_mlp(x, w_gate, w_up, w_down, chunk):
    """The same MLP over `chunk` tokens at a time, outputs concatenated."""
    x = _f64(x)
    parts = [swiglu_mlp(x[t0:t0 + chunk], w_gate, w_up, w_down)
             for t0 in range(0, x.shape[0], chunk)]
    if not parts:
        return np.zeros((0, _f64(w_down).shape[0]))
    return np.concatenate(parts, axis=0)


def silu_grad(h):
    """d silu / dh = s (1 + h (1 - s)) with s the logistic sigmoid."""
    h = np.asarray(h, dtype=np.float64)
    s = 1.0 / (1.0 + np.exp(-h))
    return s * (1.0 + h * (1.0 - s))


def swiglu_mlp_bwd(x, w_gate, w_up, w_down, dy):
    """Chain rule of swiglu_mlp. Returns dict with dx [T, Dm], dw_gate,
    dw_up [F, Dm], dw_down [Dm, F] and the intermediates act, dact, dh, dg
    [T, F]."""
    x, wg, wu, wd, dy = (_f64(t) for t in (x, w_gate, w_up, w_down, dy))
    h = x @ wg.T
    g = x @ wu.T
    act = silu(h) * g
    dact = dy @ wd
    dh = dact * g * silu_grad(h)
    dg = dact * silu(h)
    return {"dx": dh @ wg + dg @ wu, "dw_gate": dh.T @ x, "dw_up": dg.T @ x,
            "dw_down": dy.T @ act, "act": act, "dact": dact, "dh": dh,
            "dg": dg}
