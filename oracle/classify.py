"""Tile classification from the mask definition (oracle; test infra only).

Blockwise attention visits (query block, key block) tiles ("LWM：突破 100 万
Token 的开源大模型", 配置参数: query and key chunk sizes). Under packing plus
causality ("LWM：突破 100 万 Token 的开源大模型", 概述 (b)) a tile is

* EMPTY   (0) if no (i, j) pair in it is allowed,
* FULL    (2) if every pair in it is allowed,
* PARTIAL (1) otherwise.

Indices at or beyond N (the ragged tail of the last block) count as not
allowed, so a tile that reaches past N is never FULL. kv_lo / kv_hi of a
query block are the smallest / largest key block that is not EMPTY.

Two forms:
* ``classify_bruteforce`` builds the allowed mask of each tile and looks at
  it -- the definition itself, for small N;
* ``classify_count`` counts allowed pairs per tile from the contiguous
  segment runs (row i sees columns [start of its run, i]); it is pinned to
  the brute force on small inputs and used where N*N booleans do not fit.
"""

import numpy as np

from .attention import _i64, allowed_mask

TILE_EMPTY = 0
TILE_PARTIAL = 1
TILE_FULL = 2


def _result(counts, block_q, block_k):
    full = counts == block_q * block_k
    cls = np.where(counts == 0, TILE_EMPTY,
                   np.where(full, TILE_FULL, TILE_PARTIAL)).astype(np.uint8)
    nz = counts > 0
    tk = counts.shape[-1]
    idx = np.arange(tk)
    kv_lo = np.where(nz, idx, tk).min(axis=-1).astype(np.int32)
    kv_hi = np.where(nz, idx, -1).max(axis=-1).astype(np.int32)
    return kv_lo, kv_hi, cls


def classify_bruteforce(segment_ids, block_q, block_k):
    """segment_ids [B, N] -> kv_lo, kv_hi [B, Tq] int32; cls [B, Tq, Tk] u8."""
    seg_all = _i64(segment_ids)
    B, N = seg_all.shape
    tq = -(-N // block_q)
    tk = -(-N // block_k)
    counts = np.zeros((B, tq, tk), dtype=np.int64)
    for b in range(B):
        seg = seg_all[b]
        for t in range(tq):
            rows = np.arange(t * block_q, min((t + 1) * block_q, N))
            for j in range(tk):
                cols = np.arange(j * block_k, min((j + 1) * block_k, N))
                counts[b, t, j] = allowed_mask(seg, rows, cols).sum()
    return _result(counts, block_q, block_k)


def classify_count(segment_ids, block_q, block_k, q_tiles=None):
    """Same result as the brute force, by counting allowed pairs per tile.

    Row i of a contiguous run starting at r(i) sees columns [r(i), i]; the
    number of them inside key block [ks, ke] is
    max(0, min(i, ke) - max(ks, r(i)) + 1).  ``q_tiles`` restricts the work
    to some query blocks (the other rows of the result are left at -1 / 0).
    """
    seg_all = _i64(segment_ids)
    B, N = seg_all.shape
    tq = -(-N // block_q)
    tk = -(-N // block_k)
    q_tiles = range(tq) if q_tiles is None else q_tiles
    counts = np.zeros((B, tq, tk), dtype=np.int64)
    for b in range(B):
        seg = seg_all[b]
        starts = np.r_[0, np.flatnonzero(seg[1:] != seg[:-1]) + 1]
        run_of = np.repeat(np.arange(len(starts)),
                           np.diff(np.r_[starts, N]))
        r = starts[run_of]  # start of each row's run
        for t in q_tiles:
            i = np.arange(t * block_q, min((t + 1) * block_q, N))
            j_lo = r[i].min() // block_k
            j_hi = i.max() // block_k
            js = np.arange(j_lo, j_hi + 1)
            ks = js * block_k
            ke = np.minimum(ks + block_k - 1, N - 1)
            hi = np.minimum(i[:, None], ke[None, :])
            lo = np.maximum(ks[None, :], r[i][:, None])
            counts[b, t, j_lo:j_hi + 1] = np.maximum(0, hi - lo + 1).sum(0)
    return _result(counts, block_q, block_k)


def _chunk_tiles(q_off, Nq, k_off, Nk, block_q, block_k):
    tq = -(-Nq // block_q)
    tk = -(-Nk // block_k)
    q_blocks = [np.arange(q_off + t * block_q, q_off + min((t + 1) * block_q,
                                                           Nq))
                for t in range(tq)]
    k_blocks = [np.arange(k_off + j * block_k, k_off + min((j + 1) * block_k,
                                                           Nk))
                for j in range(tk)]
    return q_blocks, k_blocks


def classify_cross(segment_ids, q_off, Nq, k_off, Nk, block_q, block_k):
    """Tile classes of one query chunk against one key chunk of the same
    packed rows (a step of RingAttention: "开源巨兽LWM：如何用RingAttention
    撬动百万Token多模态世界", 3.1).

    Queries are the global token indices [q_off, q_off + Nq), keys
    [k_off, k_off + Nk); tiles are block_q x block_k blocks counted from the
    start of each chunk. A pair is allowed by the mask definition
    (``allowed_mask`` on global indices); indices past a chunk's end are
    never allowed. Returns kv_lo, kv_hi [B, Tq] (Tk / -1 for a query block
    that sees nothing) and cls [B, Tq, Tk], all from the brute-force count
    of allowed pairs per tile.
    """
    seg_all = _i64(segment_ids)
    B = seg_all.shape[0]
    q_blocks, k_blocks = _chunk_tiles(q_off, Nq, k_off, Nk, block_q, block_k)
    counts = np.zeros((B, len(q_blocks), len(k_blocks)), dtype=np.int64)
    for b in range(B):
        seg = seg_all[b]
        for t, rows in enumerate(q_blocks):
            for j, cols in enumerate(k_blocks):
                counts[b, t, j] = allowed_mask(seg, rows, cols).sum()
    return _result(counts, block_q, block_k)


def visible_key_ranges(segment_ids_row, rows, k_off, Nk):
    """For each global query index in ``rows`` of one packed row: the first
    and last key in [k_off, k_off + Nk) that the mask definition allows it
    to see. Those keys form one contiguous run (ids are non-decreasing), so
    the pair describes the whole set; a row that sees none of the keys gets
    (-1, -2) -- test infrastructure, compared element-wise."""
    seg = _i64(segment_ids_row)
    cols = np.arange(k_off, k_off + Nk)
    lo = np.full(len(rows), -1, dtype=np.int64)
    hi = np.full(len(rows), -2, dtype=np.int64)
    for n, i in enumerate(np.asarray(rows, dtype=np.int64)):
        ok = cols[allowed_mask(seg, [i], cols)[0]] if Nk else cols
        if ok.size:
            lo[n], hi[n] = ok.min(), ok.max()
            assert ok.size == hi[n] - lo[n] + 1  # contiguous
    return lo, hi


def visible_query_ranges(segment_ids_row, cols, q_off, Nq):
    """The key-side view: for each global key index in ``cols``, the first
    and last query in [q_off, q_off + Nq) allowed to see it ((-1, -2) if
    none)."""
    seg = _i64(segment_ids_row)
    rows = np.arange(q_off, q_off + Nq)
    lo = np.full(len(cols), -1, dtype=np.int64)
    hi = np.full(len(cols), -2, dtype=np.int64)
    for n, j in enumerate(np.asarray(cols, dtype=np.int64)):
        ok = rows[allowed_mask(seg, rows, [j])[:, 0]] if Nq else rows
        if ok.size:
            lo[n], hi[n] = ok.min(), ok.max()
            assert ok.size == hi[n] - lo[n] + 1
    return lo, hi
