"""Multi-rank host logic on CPU (gloo, world size 2): head sharding and the
max-over-ranks timing reduction. Each rank computes its head slice with the
fp64 oracle; gathering the slices must reproduce the single-process result.
"""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from long_context_blockwise_causal_b200 import dist


def test_head_shard_covers_every_head_once():
    for H in (1, 2, 3, 7, 32):
        for world in (1, 2, 3, 4, 8):
            got = [dist.head_shard(H, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == H
            for (a, b), (c, d) in zip(got, got[1:]):
                assert b == c and a <= b
            sizes = [b - a for a, b in got]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        dist.head_shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import oracle
    from long_context_blockwise_causal_b200 import workloads as wl
    w, r, _ = dist.init_from_env("gloo", timeout_s=60)
    assert (w, r) == (world, rank)
    wk = wl.Workload("t", 1, 96, 5, 16, 1e4, "uniform", 1.0, False,
                     seg_args={"lo": 1, "hi": 40})
    t = wl.make_inputs(wk, 3, device="cpu", dtype=torch.float32)
    h0, h1 = dist.head_shard(wk.H, world, rank)
    out, lse = oracle.attn_fwd(t["q"][:, :, h0:h1], t["k"][:, :, h0:h1],
                               t["v"][:, :, h0:h1], t["segment_ids"],
                               t["positions"], wk.theta)
    # gather every rank's slice (padded to the largest slice)
    hmax = -(-wk.H // world)
    pad = np.zeros((1, wk.N, hmax, wk.D))
    pad[:, :, :h1 - h0] = out
    bufs = [torch.zeros_like(torch.from_numpy(pad)) for _ in range(world)]
    torch.distributed.all_gather(bufs, torch.from_numpy(pad))
    slowest = dist.max_over_ranks(float(rank + 1), world, "cpu")
    if rank == 0:
        full, _ = oracle.attn_fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                                  t["positions"], wk.theta)
        parts = [bufs[r_].numpy()[:, :, :b - a] for r_, (a, b) in
                 enumerate(dist.head_shard(wk.H, world, x)
                           for x in range(world))]
        q.put((np.abs(np.concatenate(parts, axis=2) - full).max(), slowest))
    torch.distributed.barrier()
    torch.distributed.destroy_process_group()


def test_head_sharded_job_over_two_gloo_ranks_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q))
             for r in range(2)]
    for p in procs:
        p.start()
    err, slowest = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert err < 1e-12
    assert slowest == 2.0
