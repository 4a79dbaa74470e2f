"""Ring-attention building blocks on the GPU vs the fp64 oracle: the
partial forward of a query chunk over a key chunk (any offsets, ragged
sizes, empty results), the log-sum-exp merge, and a whole ring of P ranks
run one after the other on one device ("开源巨兽LWM：如何用RingAttention
撬动百万Token多模态世界", 3.1)."""

import numpy as np
import pytest
import torch

import oracle
from long_context_blockwise_causal_b200 import ops, ring
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.gpu

OUT_TOL, LSE_TOL = 2e-2, 1e-3


def _case(N, H, B, seed, lo=1, hi=600, scale=None):
    base = wl.WORKLOADS["packed128k"]
    w = wl.Workload("ring", B, N, H, 128, base.theta, "uniform",
                    base.scale if scale is None else scale, False,
                    seg_args={"lo": lo, "hi": hi})
    return wl.make_inputs(w, seed, device="cuda")


def _partial_check(t, q_off, nq, k_off, nk):
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp)
    qs, ks = slice(q_off, q_off + nq), slice(k_off, k_off + nk)
    q = t["q"][:, qs].contiguous()
    k_rot = ops.rope_apply(t["k"][:, ks].contiguous(),
                           t["positions"][:, ks].contiguous(), table)
    v = t["v"][:, ks].contiguous()
    seg, pos = t["segment_ids"], t["positions"]
    out, lse = ops.fwd_block(q, k_rot, v, seg[:, qs].contiguous(),
                             pos[:, qs].contiguous(), seg[:, ks].contiguous(),
                             q_off, k_off, t["theta"], mp)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd_partial(
        t["q"][:, qs], t["k"][:, ks], t["v"][:, ks], seg[:, qs], seg[:, ks],
        pos[:, qs], pos[:, ks], q_off, k_off, t["theta"])
    o, l_ = out.float().cpu().numpy(), lse.cpu().numpy()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(l_), fin)
    assert np.all(o[~np.transpose(fin, (0, 2, 1))] == 0)
    assert np.abs(o - ro).max() <= OUT_TOL
    if fin.any():
        assert np.abs(l_[fin] - rl[fin]).max() <= LSE_TOL
    return fin


@pytest.mark.parametrize("q_off,nq,k_off,nk", [
    (0, 700, 0, 700),          # diagonal chunk, ragged
    (700, 700, 0, 700),        # strictly earlier keys
    (1000, 333, 517, 300),     # unaligned offsets, keys end before queries
    (384, 256, 256, 512),      # keys straddle the queries
    (0, 300, 300, 300),        # keys all in the future: empty
    (1500, 1, 0, 1501),        # one query row
    (1400, 100, 1499, 1),      # one key
])
def test_partial_matches_oracle(cuda_dev, q_off, nq, k_off, nk):
    t = _case(1600, 3, 2, 11)
    _partial_check(t, q_off, nq, k_off, nk)


def test_partial_across_examples_is_empty(cuda_dev):
    # one example per 128 tokens: queries of chunk 3 see nothing of chunk 0
    t = _case(1024, 2, 1, 12, lo=128, hi=128)
    fin = _partial_check(t, 384, 128, 0, 128)
    assert not fin.any()


def test_partial_with_no_keys(cuda_dev):
    t = _case(256, 2, 1, 13)
    mp = int(t["positions"].max()) + 1
    q = t["q"][:, :128].contiguous()
    empty = t["k"][:, :0].contiguous()
    seg = t["segment_ids"][:, :128].contiguous()
    out, lse = ops.fwd_block(q, empty, empty, seg,
                             t["positions"][:, :128].contiguous(),
                             t["segment_ids"][:, :0].contiguous(), 0, 0,
                             t["theta"], mp)
    torch.cuda.synchronize()
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))


def test_merge_matches_oracle(cuda_dev):
    g = torch.Generator().manual_seed(5)
    B, N, H = 2, 300, 3
    oa = torch.randn((B, N, H, 128), generator=g).bfloat16()
    ob = torch.randn((B, N, H, 128), generator=g).bfloat16()
    la = torch.randn((B, H, N), generator=g) * 4
    lb = torch.randn((B, H, N), generator=g) * 4
    la[0, 1, :40] = float("-inf")
    oa[0, :40, 1] = 0
    lb[1, 2, 100:] = float("-inf")
    ob[1, 100:, 2] = 0
    la[1, 0, 7] = lb[1, 0, 7] = float("-inf")
    oa[1, 7, 0] = ob[1, 7, 0] = 0
    ro, rl = oracle.merge_partials(oa.double().numpy(), la.double().numpy(),
                                   ob.double().numpy(), lb.double().numpy())
    out, lse = oa.cuda(), la.cuda()
    ops.merge(out, lse, ob.cuda(), lb.cuda())
    torch.cuda.synchronize()
    o, l_ = out.float().cpu().numpy(), lse.cpu().numpy()
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(l_), fin)
    assert o[1, 7, 0].max() == 0 and o[1, 7, 0].min() == 0
    # one bf16 rounding of a convex combination of bf16 values
    assert np.abs(o - ro).max() <= 2 ** -8 * max(1.0, np.abs(ro).max())
    assert np.abs(l_[fin] - rl[fin]).max() <= 1e-5 * max(1.0, np.abs(rl[fin]).max())


@pytest.mark.parametrize("P", [2, 3, 8])
def test_simulated_ring_matches_dense_oracle(cuda_dev, P):
    t = _case(2000, 2, 2, 14)
    mp = int(t["positions"].max()) + 1
    be = ring.CudaBackend(t["theta"], mp)
    out, lse = ring.simulate_ring_fwd(t["q"], t["k"], t["v"],
                                      t["segment_ids"], t["positions"], P, be)
    torch.cuda.synchronize()
    ro, rl = oracle.attn_fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                             t["positions"], t["theta"])
    # each of up to P merges rounds out to bf16 once more
    assert np.abs(out.float().cpu().numpy() - ro).max() <= OUT_TOL
    assert np.abs(lse.cpu().numpy() - rl).max() <= LSE_TOL


def test_ring_of_one_equals_full_forward(cuda_dev):
    t = _case(1000, 2, 1, 15)
    mp = int(t["positions"].max()) + 1
    be = ring.CudaBackend(t["theta"], mp)
    o1, l1 = ring.simulate_ring_fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                                    t["positions"], 1, be)
    o2, l2 = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"], t["positions"],
                     t["theta"], mp)
    torch.cuda.synchronize()
    # the same kernel over the same tiles: identical results
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
