"""RoPE in fp64 (oracle; test infrastructure only).

Source: "[论文解读] World Model on Million-Length Video And Language With
Blockwise RingAttention", 提出的方法 -- RoPE is extended to long context by
scaling its theta with the context length; the theta values themselves
(e.g. 5e7 at 32K) appear in "LWM：突破 100 万 Token 的开源大模型",
脚本运行说明 (the update_llama_config example).

The pages do not print the rotation. Readings taken here (the Llama-2
convention, which the pages name as the backbone in "Inside Large World
Model", Stage I / Core Architecture):

* pair k of a head vector is the interleaved pair (x[2k], x[2k+1]),
  k = 0 .. D/2-1;
* its frequency is theta ** (-2k / D);
* the angle is position * frequency, evaluated in fp64 (at position 1e6 an
  fp32 product would be off by ~0.03 rad);
* R(p) rotates each pair counter-clockwise by its angle:
  (a, b) -> (a cos - b sin, a sin + b cos).
"""

import numpy as np


def rope_inv_freq(theta: float, head_dim: int) -> np.ndarray:
    """Frequencies theta ** (-2k / D) for k = 0 .. D/2-1, fp64."""
    if head_dim % 2:
        raise ValueError("head_dim must be even")
    k = np.arange(head_dim // 2, dtype=np.float64)
    return np.power(np.float64(theta), -2.0 * k / head_dim)


def rope_angles(positions, theta: float, head_dim: int) -> np.ndarray:
    """Angles [..., D/2] = position * frequency, fp64."""
    p = np.asarray(positions, dtype=np.float64)
    return p[..., None] * rope_inv_freq(theta, head_dim)


def rope_rotate(x, positions, theta: float, sign: int = 1) -> np.ndarray:
    """Apply R(sign * position) to the last axis of ``x``.

    x: [..., N, D] (any float dtype, promoted to fp64); positions: [N].
    sign=-1 gives the inverse rotation R(-p) used to map gradients taken
    with respect to rotated vectors back to the un-rotated inputs.
    """
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = float(sign) * rope_angles(positions, theta, d)  # [N, D/2]
    c = np.cos(ang)
    s = np.sin(ang)
    a = x[..., 0::2]
    b = x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = a * c - b * s
    out[..., 1::2] = a * s + b * c
    return out


def rope_rotate_half(x, positions, theta: float, sign: int = 1) -> np.ndarray:
    """RoPE in the rotate-half layout: pair k is (x[k], x[k + D/2]) with the
    same frequency theta ** (-2k / D); this is how Hugging Face Llama
    checkpoints (the PyTorch form of the models, "LWM：突破 100 万 Token 的开
    源大模型", 脚本运行说明) lay out q and k."""
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    ang = float(sign) * rope_angles(positions, theta, d)
    c = np.cos(ang)
    s = np.sin(ang)
    a = x[..., : d // 2]
    b = x[..., d // 2:]
    out = np.empty_like(x)
    out[..., : d // 2] = a * c - b * s
    out[..., d // 2:] = a * s + b * c
    return out


def half_to_interleaved(x) -> np.ndarray:
    """Permute the last axis from the rotate-half layout to the interleaved
    one: out[2k] = x[k], out[2k+1] = x[k + D/2]."""
    x = np.asarray(x)
    d = x.shape[-1]
    out = np.empty_like(x)
    out[..., 0::2] = x[..., : d // 2]
    out[..., 1::2] = x[..., d // 2:]
    return out


def interleaved_to_half(x) -> np.ndarray:
    """Inverse of half_to_interleaved."""
    x = np.asarray(x)
    return np.concatenate([x[..., 0::2], x[..., 1::2]], axis=-1)
