"""Seeded synthetic inputs for blockwise packed causal RoPE attention.

This module only draws inputs (segment lengths, segment ids, positions and
random Q/K/V/dO tensors). It holds none of the attention arithmetic and is
shared by the tests, the benchmark and the smoke check, which hand the same
arrays to the CUDA path and to the oracle.

Workload shapes follow the pages: 32 heads x head_dim 128 (the Llama-2-7B
backbone, "Inside Large World Model", Stage I), 32K-1M contexts ("LWM：突破
100 万 Token 的开源大模型", 模型和上下文大小), theta values such as 5e7
(same page, 脚本运行说明), block size 128 for queries and keys (same page,
配置参数 / the scan chunk sizes), and video frames of 256 VQ tokens plus one
delimiter ("[论文解读] World Model on Million-Length Video And Language With
Blockwise RingAttention", 提出的方法; "开源巨兽LWM...", 2.1).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

HEAD_DIM = 128
TOKENS_PER_FRAME = 256 + 1  # 256 VQ tokens + 1 frame delimiter


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    N: int
    H: int
    D: int
    theta: float
    segments: str           # "uniform" | "single" | "loguniform" | "vision_text"
    scale: float            # Q/K/V ~ N(0, 1) * scale
    backward: bool
    block_q: int = 128
    block_k: int = 128
    seg_args: dict = field(default_factory=dict)


WORKLOADS = {
    # small case the oracle finishes in seconds
    "tiny2k": Workload("tiny2k", 1, 2048, 4, HEAD_DIM, 1e4, "uniform", 1.0,
                       False, seg_args={"lo": 64, "hi": 1024}),
    # Llama-2-7B attention layer shape at 32K, one causal segment
    "text32k": Workload("text32k", 1, 32768, 32, HEAD_DIM, 1e6, "single",
                        1.0 / math.sqrt(HEAD_DIM), True),
    # packed documents, log-uniform lengths in [512, 32768]
    "packed128k": Workload("packed128k", 1, 131072, 32, HEAD_DIM, 1e7,
                           "loguniform", 1.0 / math.sqrt(HEAD_DIM), True,
                           seg_args={"lo": 512, "hi": 32768}),
    # text runs and video clips, one example per segment
    "vl256k": Workload("vl256k", 1, 262144, 32, HEAD_DIM, 5e7,
                       "vision_text", 1.0 / math.sqrt(HEAD_DIM), False,
                       seg_args={"text_lo": 32, "text_hi": 2048,
                                 "frames_lo": 8, "frames_hi": 64}),
    # single-GPU 1M-token stress, one causal segment
    "stress1m": Workload("stress1m", 1, 1048576, 32, HEAD_DIM, 5e7, "single",
                         1.0 / math.sqrt(HEAD_DIM), False),
}


def segment_lengths(kind: str, n: int, seed: int, **kw) -> np.ndarray:
    """Lengths of the packed examples of one row; they sum to n.

    The last example is truncated so the row is exactly n tokens.
    """
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    rng = np.random.default_rng(seed)
    out = []
    total = 0
    while total < n:
        if kind == "single":
            L = n
        elif kind == "uniform":
            L = int(rng.integers(kw["lo"], kw["hi"] + 1))
        elif kind == "loguniform":
            L = int(round(math.exp(rng.uniform(math.log(kw["lo"]),
                                               math.log(kw["hi"])))))
        elif kind == "vision_text":
            if rng.random() < 0.5:
                L = int(rng.integers(kw["text_lo"], kw["text_hi"] + 1))
            else:
                L = int(rng.integers(kw["frames_lo"], kw["frames_hi"] + 1)) \
                    * TOKENS_PER_FRAME
        elif kind == "fixed":
            L = int(kw["length"])
        else:
            raise ValueError(f"unknown segment kind {kind!r}")
        L = max(1, min(L, n - total))
        out.append(L)
        total += L
    return np.asarray(out, dtype=np.int64)


def segments_from_lengths(lengths: np.ndarray):
    """segment ids counting up from 0, positions reset at each start."""
    lengths = np.asarray(lengths, dtype=np.int64)
    n = int(lengths.sum())
    seg = np.repeat(np.arange(len(lengths), dtype=np.int32), lengths)
    starts = np.repeat(np.cumsum(lengths) - lengths, lengths)
    pos = (np.arange(n, dtype=np.int64) - starts).astype(np.int32)
    return seg, pos


def make_segments(w: Workload, seed: int, N: int | None = None,
                  B: int | None = None):
    """segment_ids, positions [B, N] int32 and per-row lengths."""
    N = w.N if N is None else N
    B = w.B if B is None else B
    segs, poss, lens = [], [], []
    for b in range(B):
        L = segment_lengths(w.segments, N, seed * 1000 + b, **w.seg_args)
        s, p = segments_from_lengths(L)
        segs.append(s)
        poss.append(p)
        lens.append(L)
    return (np.stack(segs) if B else np.zeros((0, N), np.int32),
            np.stack(poss) if B else np.zeros((0, N), np.int32), lens)


def visible_pairs(lengths_per_row) -> int:
    """Exact number of allowed (query, key) pairs: sum over runs L(L+1)/2."""
    return int(sum(int((L * (L + 1) // 2).sum()) for L in lengths_per_row))


def random_tensor(shape, seed: int, scale: float, dtype, device,
                  chunk_elems: int = 1 << 26, n_tokens: int | None = None):
    """N(0,1)*scale rounded to ``dtype``, drawn in chunks along dim 1.

    Chunking bounds the fp32 scratch for the 1M-token case; the values are
    a deterministic function of (shape, seed, chunk_elems). ``n_tokens``
    returns only the first n_tokens along dim 1 (the same values as that
    prefix of the full tensor, drawing only the chunks it needs).
    """
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    n = shape[1] if n_tokens is None else min(int(n_tokens), shape[1])
    out = torch.empty((shape[0], n) + tuple(shape[2:]), dtype=dtype,
                      device=device)
    if out.numel() == 0:
        return out
    per_tok = int(np.prod(shape[2:])) * shape[0]
    step = max(1, chunk_elems // max(1, per_tok))
    for s in range(0, n, step):
        e = min(shape[1], s + step)
        sub = (shape[0], e - s) + tuple(shape[2:])
        x = torch.randn(sub, generator=g, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        e = min(e, n)
        out[:, s:e].copy_(x[:, :e - s].to(dtype))
    return out


def make_inputs(w: Workload, seed: int, device="cpu", dtype=None,
                N: int | None = None, B: int | None = None, H: int | None = None,
                with_dout: bool | None = None, prefix: int | None = None):
    """All inputs of one workload as torch tensors on ``device``.

    ``prefix`` keeps only the first ``prefix`` tokens of every row (the
    same values as the full draw; "lengths" still describes the full
    rows)."""
    import torch

    dtype = torch.bfloat16 if dtype is None else dtype
    N = w.N if N is None else N
    B = w.B if B is None else B
    H = w.H if H is None else H
    seg, pos, lens = make_segments(w, seed, N=N, B=B)
    shape = (B, N, H, w.D)
    n = N if prefix is None else min(N, int(prefix))
    draw = lambda k: random_tensor(shape, seed * 16 + k, w.scale, dtype,
                                   device, n_tokens=n)
    t = {
        "q": draw(1),
        "k": draw(2),
        "v": draw(3),
        "segment_ids": torch.from_numpy(np.ascontiguousarray(seg[:, :n])).to(
            device),
        "positions": torch.from_numpy(np.ascontiguousarray(pos[:, :n])).to(
            device),
        "lengths": lens,
        "theta": w.theta,
    }
    if w.backward if with_dout is None else with_dout:
        t["dout"] = draw(4)
    return t


# ------------------------------------------------ blockwise feed-forward
@dataclass(frozen=True)
class FfnWorkload:
    """The Llama-2-7B MLP over T tokens in chunks of `chunk` (the pages'
    scan_mlp_chunk_size); activations N(0,1), weights N(0, 0.02^2) (the
    Llama initialiser's std), bf16."""
    name: str
    T: int
    Dm: int
    F: int
    chunk: int
    w_std: float = 0.02


FFN_WORKLOADS = {
    # one 32K-token sequence of LWM-Text-32K through one MLP block
    "mlp32k": FfnWorkload("mlp32k", 32768, 4096, 11008, 8192),
    # a single chunk (the unit the pages' scan_mlp processes)
    "mlp8k": FfnWorkload("mlp8k", 8192, 4096, 11008, 8192),
}


def ffn_flops(T: int, Dm: int, F: int) -> int:
    """Multiply-adds x2 of the three projections (the SwiGLU itself is
    O(T F) and not counted)."""
    return 2 * T * Dm * F * 3


def make_ffn_inputs(T: int, Dm: int, F: int, seed: int, device="cpu",
                    w_std: float = 0.02, dtype=None):
    """x [T, Dm]; w_gate, w_up [F, Dm]; w_down [Dm, F] (nn.Linear layout)."""
    import torch

    dtype = torch.bfloat16 if dtype is None else dtype
    s = seed * 16
    return {
        "x": random_tensor((1, T, Dm), s + 5, 1.0, dtype, device)[0],
        "w_gate": random_tensor((1, F, Dm), s + 6, w_std, dtype, device)[0],
        "w_up": random_tensor((1, F, Dm), s + 7, w_std, dtype, device)[0],
        "w_down": random_tensor((1, Dm, F), s + 8, w_std, dtype, device)[0],
    }
