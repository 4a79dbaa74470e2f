"""Ring schedule (host logic) on CPU: the chunk split, the source order, the
causal skip, and a whole ring over 2 and 3 gloo ranks whose per-step
arithmetic is the oracle's. Gathering every rank's result must reproduce
the dense oracle ("开源巨兽LWM：如何用RingAttention撬动百万Token多模态世界",
3.1: the ring is an exact re-organisation of attention)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
from long_context_blockwise_causal_b200 import ring
from long_context_blockwise_causal_b200 import workloads as wl

from ring_backend_oracle import OracleBackend

THETA = 1e5


def _inputs(N=200, H=2, D=16, seed=7):
    w = wl.Workload("ring", 2, N, H, D, THETA, "uniform", 1.0, False,
                    seg_args={"lo": 1, "hi": 90})
    return wl.make_inputs(w, seed, device="cpu", dtype=torch.float32)


def test_chunks_match_oracle_split():
    for N, P in [(200, 3), (7, 8), (1 << 20, 8), (0, 2), (129, 4)]:
        assert [ring.ring_chunk(N, P, r) for r in range(P)] == \
            oracle.ring_chunks(N, P)
    with pytest.raises(ValueError):
        ring.ring_chunk(10, 2, 2)


def test_sources_visit_every_rank_once_own_first():
    for P in (1, 2, 5, 8):
        for r in range(P):
            src = ring.ring_sources(r, P)
            assert src[0] == r and sorted(src) == list(range(P))
            # the next step's chunk is the one the left neighbour held now
            left = ring.ring_sources((r - 1) % P, P)
            assert src[1:] == left[:-1]


def test_causal_skip():
    assert ring.causally_visible(100, 50, 100, 50)
    assert ring.causally_visible(100, 50, 0, 50)
    assert ring.causally_visible(100, 50, 149, 10)
    assert not ring.causally_visible(100, 50, 150, 10)
    assert not ring.causally_visible(100, 0, 0, 10)
    assert not ring.causally_visible(100, 10, 0, 0)


@pytest.mark.parametrize("P", [1, 3, 4, 7])
def test_simulated_ring_with_oracle_steps_equals_dense(P):
    t = _inputs()
    out, lse = oracle.attn_fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                               t["positions"], THETA)
    ro, rl = ring.simulate_ring_fwd(t["q"], t["k"], t["v"],
                                    t["segment_ids"], t["positions"], P,
                                    OracleBackend(THETA))
    np.testing.assert_allclose(ro.numpy(), out, atol=1e-12)
    np.testing.assert_allclose(rl.numpy(), lse, atol=1e-12)


@pytest.mark.parametrize("P", [1, 2, 3, 5])
def test_simulated_ring_backward_with_oracle_steps_equals_dense(P):
    t = _inputs(N=150, seed=8)
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(t["q"].shape, generator=g, dtype=torch.float64)
    ref = oracle.attn_bwd(t["q"], t["k"], t["v"], dout, t["segment_ids"],
                          t["positions"], THETA)
    out = torch.from_numpy(ref["out"])
    lse = torch.from_numpy(ref["lse"])
    dq, dk, dv = ring.simulate_ring_bwd(
        t["q"].double(), t["k"].double(), t["v"].double(), out, dout, lse,
        t["segment_ids"], t["positions"], P, OracleBackend(THETA))
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got.numpy(), ref[name], atol=1e-11)


def test_zigzag_parts_cover_the_sequence_once():
    for N, P in [(200, 3), (1 << 15, 8), (17, 4), (8, 4)]:
        got = sorted(pt for r in range(P) for pt in ring.ring_parts(N, P, r,
                                                                    "zigzag"))
        off = 0
        for o, n in got:
            assert o == off
            off += n
        assert off == N
        # rank r holds chunk r and its mirror 2P-1-r
        for r in range(P):
            (a, _), (b, _) = ring.ring_parts(N, P, r, "zigzag")
            assert (a, b) == (ring.ring_chunk(N, 2 * P, r)[0],
                              ring.ring_chunk(N, 2 * P, 2 * P - 1 - r)[0])


def _causal_pairs(parts, N, P, layout):
    """Visible (query, key) pairs of one causal sequence a rank computes."""
    tot = 0
    for q_off, nq in parts:
        for src in range(P):
            for k_off, nk in ring.ring_parts(N, P, src, layout):
                for i in range(q_off, q_off + nq):
                    tot += max(0, min(i, k_off + nk - 1) - k_off + 1)
    return tot


def test_zigzag_balances_the_causal_ring():
    N, P = 512, 4
    work = {lay: [_causal_pairs(ring.ring_parts(N, P, r, lay), N, P, lay)
                  for r in range(P)] for lay in ring.LAYOUTS}
    total = N * (N + 1) // 2
    for lay in ring.LAYOUTS:
        assert sum(work[lay]) == total
    c, z = work["contiguous"], work["zigzag"]
    assert max(c) / min(c) > 5          # the plain ring: last rank >> first
    assert max(z) / min(z) < 1.01       # zigzag: equal shares


@pytest.mark.parametrize("P", [1, 2, 3, 4])
def test_simulated_zigzag_ring_with_oracle_steps_equals_dense(P):
    t = _inputs(N=150, seed=9)
    g = torch.Generator().manual_seed(4)
    dout = torch.randn(t["q"].shape, generator=g, dtype=torch.float64)
    ref = oracle.attn_bwd(t["q"], t["k"], t["v"], dout, t["segment_ids"],
                          t["positions"], THETA)
    be = OracleBackend(THETA)
    ro, rl = ring.simulate_ring_fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                                    t["positions"], P, be, layout="zigzag")
    np.testing.assert_allclose(ro.numpy(), ref["out"], atol=1e-12)
    np.testing.assert_allclose(rl.numpy(), ref["lse"], atol=1e-12)
    dq, dk, dv = ring.simulate_ring_bwd(
        t["q"].double(), t["k"].double(), t["v"].double(),
        torch.from_numpy(ref["out"]), dout, torch.from_numpy(ref["lse"]),
        t["segment_ids"], t["positions"], P, be, layout="zigzag")
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got.numpy(), ref[name], atol=1e-11)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, layout="contiguous"):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from long_context_blockwise_causal_b200 import dist as ldist
    ldist.init_from_env("gloo", timeout_s=60)
    t = _inputs()
    N = t["q"].shape[1]
    parts = ring.ring_parts(N, world, rank, layout)

    def mine(x):  # this rank's tokens: its parts, concatenated
        return torch.cat([x[:, o:o + n] for o, n in parts], dim=1)

    def mine_h(x):  # the same along the last axis of [B, H, N]
        return torch.cat([x[:, :, o:o + n] for o, n in parts], dim=2)

    out, lse = ring.ring_fwd(
        mine(t["q"]), mine(t["k"]), mine(t["v"]), mine(t["segment_ids"]),
        mine(t["positions"]), N, OracleBackend(THETA), layout=layout)
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(t["q"].shape, generator=g, dtype=torch.float64)
    grads = ring.ring_bwd(
        mine(t["q"]).double(), mine(t["k"]).double(), mine(t["v"]).double(),
        out, mine(dout), lse, mine(t["segment_ids"]), mine(t["positions"]),
        N, OracleBackend(THETA), layout=layout)
    outs = [None] * world
    torch.distributed.all_gather_object(
        outs, (parts, out.numpy(), lse.numpy())
        + tuple(x.numpy() for x in grads))
    if rank == 0:
        # put every rank's parts back in global order
        def glob(i, axis):
            full = None
            for o in outs:
                x, off = o[i], 0
                for po, pn in o[0]:
                    sl = [slice(None)] * x.ndim
                    sl[axis] = slice(off, off + pn)
                    if full is None:
                        shape = list(x.shape)
                        shape[axis] = N
                        full = np.zeros(shape)
                    fs = [slice(None)] * x.ndim
                    fs[axis] = slice(po, po + pn)
                    full[tuple(fs)] = x[tuple(sl)]
                    off += pn
            return full
        outs = [(glob(1, 1), glob(2, 2), glob(3, 1), glob(4, 1), glob(5, 1))]
        ref = oracle.attn_bwd(t["q"], t["k"], t["v"], dout,
                              t["segment_ids"], t["positions"], THETA)
        o = outs[0]
        errs = [float(np.abs(o[0] - ref["out"]).max()),
                float(np.abs(o[1] - ref["lse"]).max())]
        for i, name in ((2, "dq"), (3, "dk"), (4, "dv")):
            errs.append(float(np.abs(o[i] - ref[name]).max()))
        q.put(errs)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world,layout", [(2, "contiguous"),
                                          (3, "contiguous"), (2, "zigzag"),
                                          (3, "zigzag")])
def test_ring_forward_and_backward_over_gloo_ranks_equals_dense(world,
                                                                layout):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, layout))
             for r in range(world)]
    for p in procs:
        p.start()
    errs = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # forward out, lse; then dq, dk, dv after the ring backward
    assert max(errs[:2]) < 1e-12 and max(errs[2:]) < 1e-11, errs
