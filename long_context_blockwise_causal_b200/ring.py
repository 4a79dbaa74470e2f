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

import torch

from . import ops


def ring_chunk(N: int, world: int, rank: int) -> tuple[int, int]:
    """(offset, length) of rank's contiguous chunk of an N-token sequence."""
    if world <= 0 or not (0 <= rank < world) or N < 0:
        raise ValueError("bad N/world/rank")
    base, extra = divmod(N, world)
    off = rank * base + min(rank, extra)
    return off, base + (1 if rank < extra else 0)


def ring_sources(rank: int, world: int) -> list[int]:
    """Rank whose key/value chunk rank `rank` holds at each step."""
    return [(rank - s) % world for s in range(world)]


def causally_visible(q_off: int, nq: int, k_off: int, nk: int) -> bool:
    """Whether any key of [k_off, k_off+nk) precedes or equals any query of
    [q_off, q_off+nq) (otherwise the partial is empty by causality)."""
    return nq > 0 and nk > 0 and k_off <= q_off + nq - 1


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
                             rope_layout=self.layout)

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


def ring_fwd(q, k, v, segment_ids, positions, N: int, backend, group=None):
    """Forward of this rank's queries over the whole ring.

    q, k, v [B, n, H, D] and segment_ids, positions [B, n] are this rank's
    chunk (``ring_chunk(N, world, rank)``) of an N-token packed sequence.
    Returns this rank's (out [B, n, H, D], lse [B, H, n]).
    """
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    q_off, n = ring_chunk(N, world, rank)
    if q.shape[1] != n:
        raise ValueError(f"rank {rank} holds {q.shape[1]} tokens, its chunk "
                         f"of {N} over {world} ranks is {n}")
    glob = (lambda r: r) if group is None else \
        (lambda r: dist.get_global_rank(group, r))
    nxt, prv = glob((rank + 1) % world), glob((rank - 1) % world)
    cur = (backend.rotate(k, positions), v, segment_ids)
    acc = None
    for s, src in enumerate(ring_sources(rank, world)):
        reqs, incoming = [], None
        if s + 1 < world:  # pass the held chunk on, take the next one in
            _, n_in = ring_chunk(N, world, (rank - s - 1) % world)
            B, _, H, D = k.shape
            incoming = (cur[0].new_empty((B, n_in, H, D)),
                        cur[1].new_empty((B, n_in, H, D)),
                        cur[2].new_empty((B, n_in)))
            ops_ = [dist.P2POp(dist.isend, t, nxt, group) for t in cur]
            ops_ += [dist.P2POp(dist.irecv, t, prv, group) for t in incoming]
            reqs = dist.batch_isend_irecv(ops_)
        k_off, nk = ring_chunk(N, world, src)
        if causally_visible(q_off, n, k_off, nk):
            acc = _fold(backend, acc, backend.partial(
                q, cur[0], cur[1], segment_ids, positions, cur[2], q_off,
                k_off))
        for r in reqs:
            r.wait()
        if incoming is not None:
            cur = incoming
    return acc if acc is not None else backend.empty(q)


def ring_bwd(q, k, v, out, dout, lse, segment_ids, positions, N: int,
             backend, group=None):
    """Backward of this rank's chunk over the whole ring, given its chunk of
    the finished forward (out, lse over all keys) and of dout. Returns this
    rank's (dq, dk, dv)."""
    import torch.distributed as dist

    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    q_off, n = ring_chunk(N, world, rank)
    if q.shape[1] != n:
        raise ValueError(f"rank {rank} holds {q.shape[1]} tokens, its chunk "
                         f"of {N} over {world} ranks is {n}")
    glob = (lambda r: r) if group is None else \
        (lambda r: dist.get_global_rank(group, r))
    nxt, prv = glob((rank + 1) % world), glob((rank - 1) % world)
    q_rot = backend.rotate(q, positions)
    delta = backend.delta(out, dout)
    dq_acc = backend.zeros_acc(q)
    cur = (backend.rotate(k, positions), v, segment_ids)
    grads = (backend.zeros_acc(k), backend.zeros_acc(v))  # of the held block
    B, _, H, D = k.shape
    for s, src in enumerate(ring_sources(rank, world)):
        kv_reqs, incoming = [], None
        if s + 1 < world:  # keys and values run one step ahead
            _, n_in = ring_chunk(N, world, (rank - s - 1) % world)
            incoming = (cur[0].new_empty((B, n_in, H, D)),
                        cur[1].new_empty((B, n_in, H, D)),
                        cur[2].new_empty((B, n_in)))
            p2p = [dist.P2POp(dist.isend, t, nxt, group) for t in cur]
            p2p += [dist.P2POp(dist.irecv, t, prv, group) for t in incoming]
            kv_reqs = dist.batch_isend_irecv(p2p)
        k_off, nk = ring_chunk(N, world, src)
        if causally_visible(q_off, n, k_off, nk):
            backend.partial_bwd(q_rot, cur[0], cur[1], dout, lse, delta,
                                segment_ids, cur[2], q_off, k_off, dq_acc,
                                grads[0], grads[1])
        if world > 1:  # the held block's gradients follow it (last: home)
            _, n_in = ring_chunk(N, world, (rank - s - 1) % world)
            g_in = tuple(g.new_empty((B, n_in, H, D)) for g in grads)
            p2p = [dist.P2POp(dist.isend, t, nxt, group) for t in grads]
            p2p += [dist.P2POp(dist.irecv, t, prv, group) for t in g_in]
            for r in dist.batch_isend_irecv(p2p):
                r.wait()
            grads = g_in
        for r in kv_reqs:
            r.wait()
        if incoming is not None:
            cur = incoming
    return (backend.finish(dq_acc, positions),
            backend.finish(grads[0], positions), backend.finish_v(grads[1]))


def _own(x):
    """A chunk in its own allocation, as a rank would hold it (slices of one
    tensor may start off the 16-byte boundary the library requires)."""
    return x.clone(memory_format=torch.contiguous_format)


def simulate_ring_fwd(q, k, v, segment_ids, positions, world: int, backend):
    """Every rank of a `world`-rank ring, one after the other on one device,
    in the order ``ring_fwd`` computes them (no exchange: the chunks are
    sliced from the full tensors). Returns the full (out, lse)."""
    B, N, H, _ = q.shape
    outs, lses = [], []
    rot = backend.rotate(k, positions)
    for rank in range(world):
        q_off, n = ring_chunk(N, world, rank)
        qs = slice(q_off, q_off + n)
        acc = None
        for src in ring_sources(rank, world):
            k_off, nk = ring_chunk(N, world, src)
            if not causally_visible(q_off, n, k_off, nk):
                continue
            ks = slice(k_off, k_off + nk)
            acc = _fold(backend, acc, backend.partial(
                _own(q[:, qs]), _own(rot[:, ks]), _own(v[:, ks]),
                _own(segment_ids[:, qs]), _own(positions[:, qs]),
                _own(segment_ids[:, ks]), q_off, k_off))
        if acc is None:
            acc = backend.empty(_own(q[:, qs]))
        outs.append(acc[0])
        lses.append(acc[1])
    return torch.cat(outs, dim=1), torch.cat(lses, dim=2)


def simulate_ring_bwd(q, k, v, out, dout, lse, segment_ids, positions,
                      world: int, backend):
    """Backward of every rank of a `world`-rank ring on one device, in the
    order ``ring_bwd`` computes them. Returns the full (dq, dk, dv)."""
    B, N, H, _ = q.shape
    chunks = [ring_chunk(N, world, r) for r in range(world)]
    sl = [slice(o, o + n) for o, n in chunks]
    q_rot = backend.rotate(q, positions)
    k_rot = backend.rotate(k, positions)
    delta = backend.delta(out, dout)

    def part(x, r):
        return _own(x[:, sl[r]])

    def part_h(x, r):  # [B, H, N] tensors
        return _own(x[:, :, sl[r]])

    dq_acc = [backend.zeros_acc(part(q, r)) for r in range(world)]
    dk_acc = [backend.zeros_acc(part(k, r)) for r in range(world)]
    dv_acc = [backend.zeros_acc(part(v, r)) for r in range(world)]
    for rank in range(world):
        q_off, n = chunks[rank]
        for src in ring_sources(rank, world):
            k_off, nk = chunks[src]
            if not causally_visible(q_off, n, k_off, nk):
                continue
            backend.partial_bwd(
                part(q_rot, rank), part(k_rot, src), part(v, src),
                part(dout, rank), part_h(lse, rank), part_h(delta, rank),
                part(segment_ids, rank), part(segment_ids, src), q_off, k_off,
                dq_acc[rank], dk_acc[src], dv_acc[src])
    dq = torch.cat([backend.finish(dq_acc[r], part(positions, r))
                    for r in range(world)], dim=1)
    dk = torch.cat([backend.finish(dk_acc[r], part(positions, r))
                    for r in range(world)], dim=1)
    dv = torch.cat([backend.finish_v(dv_acc[r]) for r in range(world)],
                   dim=1)
    return dq, dk, dv
