"""The tile classification the attention kernels run on, bit-exact against
the oracle's mask definition (needs a B200).

The forward and backward kernels do not store tile classes: they visit the
key blocks [kv_lo, kv_hi] of each query block (the query blocks [q_lo, q_hi]
of each key block, backward) and take the mask-free path on a tile iff
every row's visible key range covers it (lo_max <= k0 and
hi_min >= k0 + 127). lwm_blockattn_visibility runs the very launches that
produce those arrays; here the class each tile gets from them is rebuilt by
that rule and compared with the oracle's brute-force / counting classes,
element by element. Packing and causality: "LWM：突破 100 万 Token 的开源大
模型", 概述 (b); tiles: 配置参数; the ring's chunk pairs: "开源巨兽LWM：如何用
RingAttention撬动百万Token多模态世界", 3.1.
"""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BLK = 128


def classes_from_query_view(v, k_off, Tk):
    """[B, Tq, Tk] classes as the forward kernel takes them."""
    j = np.arange(Tk)
    k0 = k_off + BLK * j
    lo, hi = v["kv_lo"][..., None], v["kv_hi"][..., None]
    visited = (j >= lo) & (j <= hi)
    full = (v["lo_max"][..., None] <= k0) & (v["hi_min"][..., None]
                                             >= k0 + BLK - 1)
    return np.where(visited, np.where(full, oracle.TILE_FULL,
                                      oracle.TILE_PARTIAL),
                    oracle.TILE_EMPTY).astype(np.uint8)


def classes_from_key_view(v, q_off, Tq):
    """[B, Tk, Tq] classes as the key-major backward kernel takes them."""
    t = np.arange(Tq)
    q0 = q_off + BLK * t
    lo, hi = v["q_lo"][..., None], v["q_hi"][..., None]
    visited = (t >= lo) & (t <= hi)
    full = (v["klo_max"][..., None] <= q0) & (v["khi_min"][..., None]
                                              >= q0 + BLK - 1)
    return np.where(visited, np.where(full, oracle.TILE_FULL,
                                      oracle.TILE_PARTIAL),
                    oracle.TILE_EMPTY).astype(np.uint8)


def to_np(v):
    return {k: x.cpu().numpy().astype(np.int64) for k, x in v.items()}


def check_ranges(lo_gpu, hi_gpu, lo_ref, hi_ref):
    """Equal ranges; an empty one (the oracle writes (-1, -2) for a row and
    (T, -1) for a block) only has to be empty on the GPU too."""
    empty = lo_ref > hi_ref
    np.testing.assert_array_equal(lo_gpu > hi_gpu, empty)
    np.testing.assert_array_equal(lo_gpu[~empty], lo_ref[~empty])
    np.testing.assert_array_equal(hi_gpu[~empty], hi_ref[~empty])


@pytest.mark.parametrize("name", ["tiny2k", "text32k", "packed128k",
                                  "vl256k"])
def test_visibility_self_attention_full_size(cuda_dev, name):
    w = wl.WORKLOADS[name]
    seg, _, _ = wl.make_segments(w, 0)
    v = to_np(ops.visibility(torch.from_numpy(seg).to(cuda_dev)))
    torch.cuda.synchronize()
    N = seg.shape[1]
    kv_lo, kv_hi, cls = oracle.classify_count(seg, BLK, BLK)
    Tq = Tk = cls.shape[1]
    check_ranges(v["kv_lo"], v["kv_hi"], kv_lo.astype(np.int64),
                 kv_hi.astype(np.int64))
    np.testing.assert_array_equal(classes_from_query_view(v, 0, Tk), cls)
    np.testing.assert_array_equal(classes_from_key_view(v, 0, Tq),
                                  cls.transpose(0, 2, 1))
    # per-row and per-key ranges on sampled indices, incl. every example's
    # first and last token for the packed rows (capped)
    rng = np.random.default_rng(5)
    starts = np.r_[0, np.flatnonzero(np.diff(seg[0])) + 1]
    edges = np.unique(np.r_[starts, starts - 1, N - 1].clip(0, N - 1))[:200]
    idx = np.unique(np.r_[edges, rng.integers(0, N, 200)])
    lo, hi = oracle.visible_key_ranges(seg[0], idx, 0, N)
    check_ranges(v["row_lo"][0, idx], v["row_hi"][0, idx], lo, hi)
    lo, hi = oracle.visible_query_ranges(seg[0], idx, 0, N)
    check_ranges(v["col_lo"][0, idx], v["col_hi"][0, idx], lo, hi)


def ring_chunks(N, P):
    b = np.linspace(0, N, P + 1).astype(int)
    return list(zip(b[:-1], b[1:] - b[:-1]))


@pytest.mark.parametrize("P,layout", [(3, "contiguous"), (4, "contiguous"),
                                      (2, "zigzag")])
def test_visibility_ring_chunk_pairs(cuda_dev, P, layout):
    # every (query chunk, key chunk) pair a ring step can meet, offsets
    # non-zero and chunk lengths not multiples of 128
    N, B = 3001, 2
    segs = [wl.segments_from_lengths(
        wl.segment_lengths("uniform", N, 40 + b, lo=1, hi=700))[0]
        for b in range(B)]
    seg = np.stack(segs)
    seg_d = torch.from_numpy(seg).to(cuda_dev)
    chunks = ring_chunks(N, 2 * P if layout == "zigzag" else P)
    for q_off, Nq in chunks:
        for k_off, Nk in chunks:
            v = to_np(ops.visibility(seg_d[:, q_off:q_off + Nq].contiguous(),
                                     seg_d[:, k_off:k_off + Nk].contiguous(),
                                     q_off=q_off, k_off=k_off))
            kv_lo, kv_hi, cls = oracle.classify_cross(seg, q_off, Nq, k_off,
                                                      Nk, BLK, BLK)
            Tq, Tk = cls.shape[1:]
            check_ranges(v["kv_lo"], v["kv_hi"], kv_lo.astype(np.int64),
                         kv_hi.astype(np.int64))
            np.testing.assert_array_equal(
                classes_from_query_view(v, k_off, Tk), cls)
            np.testing.assert_array_equal(
                classes_from_key_view(v, q_off, Tq), cls.transpose(0, 2, 1))
            for b in range(B):
                lo, hi = oracle.visible_key_ranges(
                    seg[b], np.arange(q_off, q_off + Nq), k_off, Nk)
                check_ranges(v["row_lo"][b], v["row_hi"][b], lo, hi)
                lo, hi = oracle.visible_query_ranges(
                    seg[b], np.arange(k_off, k_off + Nk), q_off, Nq)
                check_ranges(v["col_lo"][b], v["col_hi"][b], lo, hi)


def test_visibility_every_token_alone_and_ragged(cuda_dev):
    # degenerate packing: each token its own example (only diagonal tiles,
    # all PARTIAL), and N = 1, 129 (ragged blocks are never FULL)
    for seg in (np.arange(700, dtype=np.int32)[None],
                np.zeros((1, 1), np.int32), np.zeros((3, 129), np.int32)):
        v = to_np(ops.visibility(torch.from_numpy(seg).to(cuda_dev)))
        _, _, cls = oracle.classify_bruteforce(seg, BLK, BLK)
        np.testing.assert_array_equal(
            classes_from_query_view(v, 0, cls.shape[2]), cls)
        np.testing.assert_array_equal(
            classes_from_key_view(v, 0, cls.shape[1]),
            cls.transpose(0, 2, 1))
