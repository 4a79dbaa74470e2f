"""RingAttention forward across ranks ("开源巨兽LWM：如何用RingAttention撬动
百万Token多模态世界", 3.1; the ring of devices behind the 1M-token context in
"[论文解读] World Model on Million-Length Video And Language With Blockwise
RingAttention", 提出的方法).

The packed sequence of N tokens is cut into contiguous chunks, one per rank
(the first N % P ranks hold one token more). Each rank keeps its queries;
its rotated keys, values and segment ids travel around the ring: at step s
rank r holds the key/value chunk of rank (r - s) mod P, computes the
partial attention of its queries over it (``lwm_blockattn_fwd_block``) and
folds it into its running (out, lse) (``lwm_blockattn_merge``), while the
chunk it holds is already on its way to rank r + 1 and the next one is
arriving from rank r - 1. A chunk lying wholly after the local queries is
passed on without compute (causality).

The backward runs the same ring ("the gradients of a block travel with
it"): each rank rotates its queries once, computes D = rowsum(dO * O) of
its finished forward, and at each step adds the visiting block's share to
its fp32 dQ accumulator and to the block's dK / dV accumulators
(``lwm_blockattn_bwd_block``); the accumulators move on with the block,
one hop behind the keys and values, and a last hop brings every block's
dK / dV home, where ``lwm_blockattn_grad_finish`` rotates them back.

The arithmetic lives behind a small backend object, so the same schedule
drives the CUDA kernels (``CudaBackend``) and, in the CPU tests, any other
implementation of the same calls.
"""

from __future__ import annotations

import numpy as np
import torch

from . import ops


def ring_chunk(N: int, world: int, rank: int) -> tuple[int, int]:
    """(offset, length) of rank's contiguous chunk of an N-token sequence."""
    if world <= 0 or not (0 <= rank < world) or N < 0:
        raise ValueError("bad N/world/rank")
    base, extra = divmod(N, world)
    off = rank * base + min(rank, extra)
    return off, base + (1 if rank < extra else 0)


LAYOUTS = ("contiguous", "zigzag")


def ring_parts(N: int, world: int, rank: int,
               layout: str = "contiguous") -> list[tuple[int, int]]:
    """The token ranges [(offset, length), ...] rank holds, in the order its
    local tensors concatenate them. "contiguous": one chunk of N/world
    tokens, as on the pages. "zigzag": chunks r and 2P-1-r of N/(2P), so
    that under the causal mask every rank has the same amount of work (the
    plain ring leaves the last rank with the most)."""
    if layout == "contiguous":
        return [ring_chunk(N, world, rank)]
    if layout == "zigzag":
        return [ring_chunk(N, 2 * world, rank),
                ring_chunk(N, 2 * world, 2 * world - 1 - rank)]
    raise ValueError(f"layout {layout!r}")


def ring_sources(rank: int, world: int) -> list[int]:
    """Rank whose key/value chunk rank `rank` holds at each step."""
    return [(rank - s) % world for s in range(world)]


def causally_visible(q_off: int, nq: int, k_off: int, nk: int) -> bool:
    """Whether any key of [k_off, k_off+nk) precedes or equals any query of
    [q_off, q_off+nq) (otherwise the partial is empty by causality)."""
    return nq > 0 and nk > 0 and k_off <= q_off + nq - 1


def _own(x):
    """A part in its own allocation, as a rank would hold it (slices of one
    tensor may start off the 16-byte boundary the library requires)."""
    return x.clone(memory_format=torch.contiguous_format)


def _split(x, parts, dim=1):
    """The local tensor x cut into its parts (each in its own allocation)."""
    out, o = [], 0
    for _, n in parts:
        out.append(_own(x.narrow(dim, o, n)))
        o += n
    return out


def _check_local(x, parts, rank):
    n = sum(m for _, m in parts)
    if x.shape[1] != n:
        raise ValueError(f"rank {rank} holds {x.shape[1]} tokens, its parts "
                         f"{parts} hold {n}")


class CudaBackend:
    """The ring's calls on this library's kernels (bf16, D = 128)."""

    def __init__(self, theta: float, max_pos: int, device=None,
                 rope_layout="interleaved"):
        self.theta = float(theta)
        self.max_pos = int(max_pos)
        self.layout = rope_layout
        self.table = ops.rope_table(self.theta, self.max_pos,
                                    device=device or "cuda")

    def rotate(self, k, positions):
        return ops.rope_apply(k, positions, self.table,
                              rope_layout=self.layout)

    def partial(self, q, k_rot, v, seg_q, pos_q, seg_k, q_off, k_off):
        return ops.fwd_block(q, k_rot, v, seg_q, pos_q, seg_k, q_off, k_off,
                             self.theta, self.max_pos,
                             rope_layout=self.layout, table=self.table)

    def merge(self, out, lse, out_part, lse_part):
        return ops.merge(out, lse, out_part, lse_part)

    def empty(self, q):
        B, N, H, _ = q.shape
        return (torch.zeros_like(q),
                torch.full((B, H, N), float("-inf"), dtype=torch.float32,
                           device=q.device))

    # backward
    def delta(self, out, dout):
        return ops.bwd_delta(out, dout)

    def zeros_acc(self, like):
        return torch.zeros(like.shape, dtype=torch.float32,
                           device=like.device)

    def partial_bwd(self, q_rot, k_rot, v, dout, lse, delta, seg_q, seg_k,
                    q_off, k_off, dq_acc, dk_acc, dv_acc):
        ops.bwd_block(q_rot, k_rot, v, dout, lse, delta, seg_q, seg_k, q_off,
                      k_off, dq_acc, dk_acc, dv_acc)

    def finish(self, acc, positions):
        return ops.grad_finish(acc, positions, self.table,
                               rope_layout=self.layout)

    def finish_v(self, acc):
        return ops.grad_finish(acc)


def _fold(backend, acc, part):
    if acc is None:
        return part
    return backend.merge(acc[0], acc[1], part[0], part[1])


def _p2p_exchange(tensors, shapes_like, nxt, prv, group):
    """Post sends of `tensors` to nxt and receives of same-typed tensors of
    the given shapes from prv; returns (requests, received tensors)."""
    import torch.distributed as dist
    incoming = [t.new_empty(shape) for t, shape in shapes_like]
    ops_ = [dist.P2POp(dist.isend, t, nxt, group) for t in tensors]
    ops_ += [dist.P2POp(dist.irecv, t, prv, group) for t in incoming]
    return dist.batch_isend_irecv(ops_), incoming


def _kv_shapes(cur, parts):
    """(template tensor, shape) of a held key/value set with the given
    parts: per part (rotated keys, values, segment ids)."""
    out = []
    k0, v0, s0 = cur[0]
    B, _, H, D = k0.shape
    for _, n in parts:
        out += [(k0, (B, n, H, D)), (v0, (B, n, H, D)), (s0, (B, n))]
    return out


def _group(flat, nparts, width):
    return [tuple(flat[i * width:(i + 1) * width]) for i in range(nparts)]


def ring_fwd(q, k, v, segment_ids, positions, N: int, backend, group=None,
             layout: str = "contiguous"):
    """Forward of this rank's queries over the whole ring.

    q, k, v [B, n, H, D] and segment_ids, positions [B, n] are this rank's
    tokens: the concatenation of its parts ``ring_parts(N, world, rank,
    layout)`` of an N-token packed sequence. Returns this rank's
    (out [B, n, H, D], lse [B, H, n]) in the same order.
    """
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    parts = ring_parts(N, world, rank, layout)
    _check_local(q, parts, rank)
    glob = (lambda r: r) if group is None else \
        (lambda r: dist.get_global_rank(group, r))
    nxt, prv = glob((rank + 1) % world), glob((rank - 1) % world)
    qs, segs, poss = (_split(x, parts) for x in (q, segment_ids, positions))
    k_rot = backend.rotate(k, positions)
    cur = list(zip(_split(k_rot, parts), _split(v, parts), segs))
    acc = [None] * len(parts)
    for s, src in enumerate(ring_sources(rank, world)):
        reqs, incoming = [], None
        if s + 1 < world:  # pass the held chunks on, take the next ones in
            nparts = ring_parts(N, world, (rank - s - 1) % world, layout)
            reqs, flat = _p2p_exchange([t for kv in cur for t in kv],
                                       _kv_shapes(cur, nparts), nxt, prv,
                                       group)
            incoming = _group(flat, len(nparts), 3)
        for i, (q_off, nq) in enumerate(parts):
            for j, (k_off, nk) in enumerate(ring_parts(N, world, src,
                                                       layout)):
                if causally_visible(q_off, nq, k_off, nk):
                    acc[i] = _fold(backend, acc[i], backend.partial(
                        qs[i], cur[j][0], cur[j][1], segs[i], poss[i],
                        cur[j][2], q_off, k_off))
        for r in reqs:
            r.wait()
        if incoming is not None:
            cur = incoming
    res = [a if a is not None else backend.empty(qs[i])
           for i, a in enumerate(acc)]
    return (torch.cat([o for o, _ in res], dim=1),
            torch.cat([l_ for _, l_ in res], dim=2))


def ring_bwd(q, k, v, out, dout, lse, segment_ids, positions, N: int,
             backend, group=None, layout: str = "contiguous"):
    """Backward of this rank's tokens over the whole ring, given its part of
    the finished forward (out, lse over all keys) and of dout, laid out as
    in ``ring_fwd``. Returns this rank's (dq, dk, dv)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    parts = ring_parts(N, world, rank, layout)
    _check_local(q, parts, rank)
    glob = (lambda r: r) if group is None else \
        (lambda r: dist.get_global_rank(group, r))
    nxt, prv = glob((rank + 1) % world), glob((rank - 1) % world)
    q_rot = _split(backend.rotate(q, positions), parts)
    delta = backend.delta(out, dout)
    loc = [int(o) for o in np.cumsum([0] + [m for _, m in parts[:-1]])]
    dls = [_own(delta.narrow(2, o, m)) for o, (_, m) in zip(loc, parts)]
    lses = [_own(lse.narrow(2, o, m)) for o, (_, m) in zip(loc, parts)]
    douts, segs, poss = (_split(x, parts) for x in (dout, segment_ids,
                                                     positions))
    dq_acc = [backend.zeros_acc(x) for x in q_rot]
    k_parts = _split(backend.rotate(k, positions), parts)
    cur = list(zip(k_parts, _split(v, parts), segs))
    # gradients of the held key/value parts: they travel with them
    grads = [(backend.zeros_acc(kk), backend.zeros_acc(kk)) for kk in k_parts]
    for s, src in enumerate(ring_sources(rank, world)):
        kv_reqs, incoming = [], None
        nparts = ring_parts(N, world, (rank - s - 1) % world, layout)
        if s + 1 < world:  # keys and values run one step ahead
            kv_reqs, flat = _p2p_exchange([t for kv in cur for t in kv],
                                          _kv_shapes(cur, nparts), nxt, prv,
                                          group)
            incoming = _group(flat, len(nparts), 3)
        for i, (q_off, nq) in enumerate(parts):
            for j, (k_off, nk) in enumerate(ring_parts(N, world, src,
                                                       layout)):
                if causally_visible(q_off, nq, k_off, nk):
                    backend.partial_bwd(q_rot[i], cur[j][0], cur[j][1],
                                        douts[i], lses[i], dls[i], segs[i],
                                        cur[j][2], q_off, k_off, dq_acc[i],
                                        grads[j][0], grads[j][1])
        if world > 1:  # the held parts' gradients follow them (last: home)
            g0 = grads[0][0]
            B, _, H, D = g0.shape
            shapes = [(g0, (B, n, H, D)) for _, n in nparts for _ in (0, 1)]
            reqs, flat = _p2p_exchange([t for gr in grads for t in gr],
                                       shapes, nxt, prv, group)
            for r in reqs:
                r.wait()
            grads = _group(flat, len(nparts), 2)
        for r in kv_reqs:
            r.wait()
        if incoming is not None:
            cur = incoming
    dq = torch.cat([backend.finish(dq_acc[i], poss[i])
                    for i in range(len(parts))], dim=1)
    dk = torch.cat([backend.finish(grads[i][0], poss[i])
                    for i in range(len(parts))], dim=1)
    dv = torch.cat([backend.finish_v(grads[i][1])
                    for i in range(len(parts))], dim=1)
    return dq, dk, dv


def simulate_ring_fwd(q, k, v, segment_ids, positions, world: int, backend,
                      layout: str = "contiguous"):
    """Every rank of a `world`-rank ring, one after the other on one device,
    in the order ``ring_fwd`` computes them (no exchange: the parts are
    sliced from the full tensors). Returns the full (out, lse) in global
    token order."""
    B, N, H, _ = q.shape
    rot = backend.rotate(k, positions)
    placed = []
    for rank in range(world):
        parts = ring_parts(N, world, rank, layout)
        for q_off, nq in parts:
            qs = slice(q_off, q_off + nq)
            acc = None
            for src in ring_sources(rank, world):
                for k_off, nk in ring_parts(N, world, src, layout):
                    if not causally_visible(q_off, nq, k_off, nk):
                        continue
                    ks = slice(k_off, k_off + nk)
                    acc = _fold(backend, acc, backend.partial(
                        _own(q[:, qs]), _own(rot[:, ks]), _own(v[:, ks]),
                        _own(segment_ids[:, qs]), _own(positions[:, qs]),
                        _own(segment_ids[:, ks]), q_off, k_off))
            if acc is None:
                acc = backend.empty(_own(q[:, qs]))
            placed.append((q_off, acc))
    placed.sort(key=lambda t: t[0])
    return (torch.cat([a[0] for _, a in placed], dim=1),
            torch.cat([a[1] for _, a in placed], dim=2))


def simulate_ring_bwd(q, k, v, out, dout, lse, segment_ids, positions,
                      world: int, backend, layout: str = "contiguous"):
    """Backward of every rank of a `world`-rank ring on one device, in the
    order ``ring_bwd`` computes them. Returns the full (dq, dk, dv) in
    global token order."""
    B, N, H, _ = q.shape
    q_rot = backend.rotate(q, positions)
    k_rot = backend.rotate(k, positions)
    delta = backend.delta(out, dout)
    all_parts = sorted({pt for r in range(world)
                        for pt in ring_parts(N, world, r, layout)})

    def part(x, o, n):
        return _own(x[:, o:o + n])

    def part_h(x, o, n):  # [B, H, N] tensors
        return _own(x[:, :, o:o + n])

    dq_acc = {pt: backend.zeros_acc(part(q, *pt)) for pt in all_parts}
    dk_acc = {pt: backend.zeros_acc(part(k, *pt)) for pt in all_parts}
    dv_acc = {pt: backend.zeros_acc(part(v, *pt)) for pt in all_parts}
    for rank in range(world):
        for qp in ring_parts(N, world, rank, layout):
            q_off, nq = qp
            for src in ring_sources(rank, world):
                for kp in ring_parts(N, world, src, layout):
                    k_off, nk = kp
                    if not causally_visible(q_off, nq, k_off, nk):
                        continue
                    backend.partial_bwd(
                        part(q_rot, *qp), part(k_rot, *kp), part(v, *kp),
                        part(dout, *qp), part_h(lse, *qp),
                        part_h(delta, *qp), part(segment_ids, *qp),
                        part(segment_ids, *kp), q_off, k_off, dq_acc[qp],
                        dk_acc[kp], dv_acc[kp])
    dq = torch.cat([backend.finish(dq_acc[pt], part(positions, *pt))
                    for pt in all_parts], dim=1)
    dk = torch.cat([backend.finish(dk_acc[pt], part(positions, *pt))
                    for pt in all_parts], dim=1)
    dv = torch.cat([backend.finish_v(dv_acc[pt]) for pt in all_parts],
                   dim=1)
    return dq, dk, dv
