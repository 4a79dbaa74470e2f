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


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    from long_context_blockwise_causal_b200 import dist as ldist
    ldist.init_from_env("gloo", timeout_s=60)
    t = _inputs()
    N = t["q"].shape[1]
    off, n = ring.ring_chunk(N, world, rank)
    sl = slice(off, off + n)
    out, lse = ring.ring_fwd(
        t["q"][:, sl].contiguous(), t["k"][:, sl].contiguous(),
        t["v"][:, sl].contiguous(), t["segment_ids"][:, sl].contiguous(),
        t["positions"][:, sl].contiguous(), N, OracleBackend(THETA))
    g = torch.Generator().manual_seed(3)
    dout = torch.randn(t["q"].shape, generator=g, dtype=torch.float64)
    grads = ring.ring_bwd(
        t["q"][:, sl].double().contiguous(), t["k"][:, sl].double().contiguous(),
        t["v"][:, sl].double().contiguous(), out, dout[:, sl].contiguous(),
        lse, t["segment_ids"][:, sl].contiguous(),
        t["positions"][:, sl].contiguous(), N, OracleBackend(THETA))
    outs = [None] * world
    torch.distributed.all_gather_object(
        outs, (out.numpy(), lse.numpy()) + tuple(x.numpy() for x in grads))
    if rank == 0:
        ref = oracle.attn_bwd(t["q"], t["k"], t["v"], dout,
                              t["segment_ids"], t["positions"], THETA)
        errs = [float(np.abs(np.concatenate([o[0] for o in outs], axis=1)
                             - ref["out"]).max()),
                float(np.abs(np.concatenate([o[1] for o in outs], axis=2)
                             - ref["lse"]).max())]
        for i, name in ((2, "dq"), (3, "dk"), (4, "dv")):
            errs.append(float(np.abs(np.concatenate([o[i] for o in outs],
                                                    axis=1)
                                     - ref[name]).max()))
        q.put(errs)
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ring_forward_and_backward_over_gloo_ranks_equals_dense(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q))
             for r in range(world)]
    for p in procs:
        p.start()
    errs = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # forward out, lse; then dq, dk, dv after the ring backward
    assert max(errs[:2]) < 1e-12 and max(errs[2:]) < 1e-11, errs
