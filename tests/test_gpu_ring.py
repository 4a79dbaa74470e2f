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


# ------------------------------------------------------------ backward

BWD_REL = 2e-2   # of max |reference|, as for the full backward


def _with_dout(t, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    t["dout"] = torch.randn(t["q"].shape, generator=g, device="cuda",
                            dtype=torch.float32).to(torch.bfloat16)
    return t


def _final_lse_delta(t):
    """lse and D of the finished dense forward (oracle, fp64 -> fp32); both
    sides of a partial-backward check receive these same values."""
    out, lse = oracle.attn_fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                               t["positions"], t["theta"])
    delta = oracle.bwd_delta(out, t["dout"])
    return (np.ascontiguousarray(lse, dtype=np.float32),
            np.ascontiguousarray(delta, dtype=np.float32))


@pytest.mark.parametrize("q_off,nq,k_off,nk", [
    (0, 700, 0, 700),          # diagonal chunk, ragged
    (700, 700, 0, 700),        # strictly earlier keys
    (1000, 333, 517, 300),     # unaligned offsets
    (384, 256, 256, 512),      # keys straddle the queries
    (0, 300, 300, 300),        # keys all in the future: nothing added
])
def test_partial_backward_matches_oracle(cuda_dev, q_off, nq, k_off, nk):
    t = _with_dout(_case(1600, 2, 2, 21), 22)
    lse, delta = _final_lse_delta(t)
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp)
    qs, ks = slice(q_off, q_off + nq), slice(k_off, k_off + nk)
    seg, pos = t["segment_ids"], t["positions"]

    def c(x, s):
        return x[:, s].contiguous()

    q_rot = ops.rope_apply(c(t["q"], qs), c(pos, qs), table)
    k_rot = ops.rope_apply(c(t["k"], ks), c(pos, ks), table)
    lse_q = torch.from_numpy(np.ascontiguousarray(lse[:, :, qs])).cuda()
    del_q = torch.from_numpy(np.ascontiguousarray(delta[:, :, qs])).cuda()
    dq_acc = torch.zeros(q_rot.shape, dtype=torch.float32, device="cuda")
    dk_acc = torch.zeros(k_rot.shape, dtype=torch.float32, device="cuda")
    dv_acc = torch.zeros(k_rot.shape, dtype=torch.float32, device="cuda")
    ops.bwd_block(q_rot, k_rot, c(t["v"], ks), c(t["dout"], qs), lse_q,
                  del_q, c(seg, qs), c(seg, ks), q_off, k_off, dq_acc,
                  dk_acc, dv_acc)
    dq = ops.grad_finish(dq_acc, c(pos, qs), table)
    dk = ops.grad_finish(dk_acc, c(pos, ks), table)
    dv = ops.grad_finish(dv_acc)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    ref = oracle.attn_bwd_partial(
        t["q"][:, qs], t["k"][:, ks], t["v"][:, ks], t["dout"][:, qs],
        lse[:, :, qs], delta[:, :, qs], seg[:, qs], seg[:, ks], pos[:, qs],
        pos[:, ks], q_off, k_off, t["theta"])
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        gg = g.float().cpu().numpy()
        if not r.any():
            assert not gg.any(), name
            continue
        err = np.abs(gg - r).max()
        assert err <= BWD_REL * np.abs(r).max(), f"{name}: {err}"


def test_partial_backward_many_items_per_cta(cuda_dev):
    # adjacent chunks of a packed row: only the example that straddles the
    # boundary links them, so most key blocks are seen by no query. Eight
    # heads give each CTA several items, empty ones (sorted last) after
    # non-empty ones.
    t = _with_dout(_case(8192, 8, 1, 29, lo=300, hi=2500), 30)
    lse, delta = _final_lse_delta(t)
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp)
    qs, ks = slice(4096, 8192), slice(0, 4096)
    seg, pos = t["segment_ids"], t["positions"]

    def c(x, s):
        return x[:, s].contiguous()

    q_rot = ops.rope_apply(c(t["q"], qs), c(pos, qs), table)
    k_rot = ops.rope_apply(c(t["k"], ks), c(pos, ks), table)
    acc = [torch.zeros(x.shape, dtype=torch.float32, device="cuda")
           for x in (q_rot, k_rot, k_rot)]
    ops.bwd_block(q_rot, k_rot, c(t["v"], ks), c(t["dout"], qs),
                  torch.from_numpy(np.ascontiguousarray(lse[:, :, qs])).cuda(),
                  torch.from_numpy(np.ascontiguousarray(delta[:, :, qs])).cuda(),
                  c(seg, qs), c(seg, ks), 4096, 0, *acc)
    o, l_ = ops.fwd_block(c(t["q"], qs), k_rot, c(t["v"], ks), c(seg, qs),
                          c(pos, qs), c(seg, ks), 4096, 0, t["theta"], mp)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    # the reference, on the two heads and the rows / keys that matter
    for h in (0, 5):
        sl = slice(h, h + 1)
        ro, rl = oracle.attn_fwd_partial(
            t["q"][:, qs, sl], t["k"][:, ks, sl], t["v"][:, ks, sl],
            seg[:, qs], seg[:, ks], pos[:, qs], pos[:, ks], 4096, 0,
            t["theta"])
        assert np.abs(o[:, :, sl].float().cpu().numpy() - ro).max() <= OUT_TOL
        fin = np.isfinite(rl)
        assert np.array_equal(np.isfinite(l_[:, sl].cpu().numpy()), fin)
        ref = oracle.attn_bwd_partial(
            t["q"][:, qs, sl], t["k"][:, ks, sl], t["v"][:, ks, sl],
            t["dout"][:, qs, sl], lse[:, sl, qs], delta[:, sl, qs],
            seg[:, qs], seg[:, ks], pos[:, qs], pos[:, ks], 4096, 0,
            t["theta"])
        got = (ops.grad_finish(acc[0][:, :, sl].contiguous(), c(pos, qs),
                               table),
               ops.grad_finish(acc[1][:, :, sl].contiguous(), c(pos, ks),
                               table),
               ops.grad_finish(acc[2][:, :, sl].contiguous()))
        for name, g, r in zip(("dq", "dk", "dv"), got, ref):
            gg = g.float().cpu().numpy()
            assert not gg[:, np.abs(r).max(axis=(0, 2, 3)) == 0].any(), name
            err = np.abs(gg - r).max()
            assert err <= BWD_REL * np.abs(r).max(), f"{name} h{h}: {err}"


def test_partial_backward_accumulates(cuda_dev):
    # two calls over two halves of the keys add up to one call over all
    t = _with_dout(_case(900, 2, 1, 23), 24)
    lse, delta = _final_lse_delta(t)
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp)
    q_rot = ops.rope_apply(t["q"], t["positions"], table)
    k_rot = ops.rope_apply(t["k"], t["positions"], table)
    lse_d = torch.from_numpy(lse).cuda()
    del_d = torch.from_numpy(delta).cuda()
    seg = t["segment_ids"]

    def acc():
        return [torch.zeros(t["q"].shape, dtype=torch.float32, device="cuda")
                for _ in range(3)]

    whole = acc()
    ops.bwd_block(q_rot, k_rot, t["v"], t["dout"], lse_d, del_d, seg, seg, 0,
                  0, *whole)
    halves = acc()
    dk_parts = []
    for k0, k1 in ((0, 384), (384, 900)):
        dk_p = torch.zeros((1, k1 - k0, 2, 128), dtype=torch.float32,
                           device="cuda")
        dv_p = torch.zeros_like(dk_p)
        ops.bwd_block(q_rot, k_rot[:, k0:k1].contiguous(),
                      t["v"][:, k0:k1].contiguous(), t["dout"], lse_d, del_d,
                      seg, seg[:, k0:k1].contiguous(), 0, k0, halves[0], dk_p,
                      dv_p)
        dk_parts.append((dk_p, dv_p))
    torch.cuda.synchronize()
    dk_cat = torch.cat([p[0] for p in dk_parts], dim=1)
    dv_cat = torch.cat([p[1] for p in dk_parts], dim=1)
    # same tiles, same per-key order: dK and dV are identical; dQ is
    # summed in another order across the two calls
    assert torch.equal(dk_cat, whole[1]) and torch.equal(dv_cat, whole[2])
    scale = whole[0].abs().max().item()
    assert (halves[0] - whole[0]).abs().max().item() <= 1e-5 * scale


@pytest.mark.parametrize("P", [2, 3])
def test_simulated_ring_backward_matches_dense_oracle(cuda_dev, P):
    t = _with_dout(_case(1500, 2, 1, 25), 26)
    mp = int(t["positions"].max()) + 1
    be = ring.CudaBackend(t["theta"], mp)
    out, lse = ring.simulate_ring_fwd(t["q"], t["k"], t["v"],
                                      t["segment_ids"], t["positions"], P, be)
    dq, dk, dv = ring.simulate_ring_bwd(t["q"], t["k"], t["v"], out,
                                        t["dout"], lse, t["segment_ids"],
                                        t["positions"], P, be)
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    ref = oracle.attn_bwd(t["q"], t["k"], t["v"], t["dout"],
                          t["segment_ids"], t["positions"], t["theta"])
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        gg = g.float().cpu().numpy()
        err = np.abs(gg - ref[name]).max()
        assert err <= BWD_REL * np.abs(ref[name]).max(), f"{name}: {err}"


def test_ring_of_one_backward_equals_full_backward(cuda_dev):
    t = _with_dout(_case(1000, 2, 1, 27), 28)
    mp = int(t["positions"].max()) + 1
    out, lse = ops.fwd(t["q"], t["k"], t["v"], t["segment_ids"],
                       t["positions"], t["theta"], mp)
    full = ops.bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                   t["segment_ids"], t["positions"], t["theta"], mp)
    be = ring.CudaBackend(t["theta"], mp)
    one = ring.simulate_ring_bwd(t["q"], t["k"], t["v"], out, t["dout"], lse,
                                 t["segment_ids"], t["positions"], 1, be)
    torch.cuda.synchronize()
    # dK and dV: the same kernel over the same tiles, rounded once (here
    # through the fp32 accumulator); dQ differs by summation order only
    for name, a, b in zip(("dq", "dk", "dv"), full, one):
        scale = a.float().abs().max().item()
        err = (a.float() - b.float()).abs().max().item()
        assert err <= 2 ** -7 * scale, f"{name}: {err}"


@pytest.mark.parametrize("P", [2, 4])
def test_simulated_zigzag_ring_matches_dense_oracle(cuda_dev, P):
    t = _with_dout(_case(1500, 2, 1, 31), 32)
    mp = int(t["positions"].max()) + 1
    be = ring.CudaBackend(t["theta"], mp)
    out, lse = ring.simulate_ring_fwd(t["q"], t["k"], t["v"],
                                      t["segment_ids"], t["positions"], P, be,
                                      layout="zigzag")
    dq, dk, dv = ring.simulate_ring_bwd(t["q"], t["k"], t["v"], out,
                                        t["dout"], lse, t["segment_ids"],
                                        t["positions"], P, be,
                                        layout="zigzag")
    torch.cuda.synchronize()
    assert ops.last_status() == ops.OK
    ref = oracle.attn_bwd(t["q"], t["k"], t["v"], t["dout"],
                          t["segment_ids"], t["positions"], t["theta"])
    assert np.abs(out.float().cpu().numpy() - ref["out"]).max() <= OUT_TOL
    assert np.abs(lse.cpu().numpy() - ref["lse"]).max() <= LSE_TOL
    for name, g in (("dq", dq), ("dk", dk), ("dv", dv)):
        err = np.abs(g.float().cpu().numpy() - ref[name]).max()
        assert err <= BWD_REL * np.abs(ref[name]).max(), f"{name}: {err}"


def test_partial_with_caller_table_is_identical(cuda_dev):
    # the ring passes one table to every step; the result must not change
    t = _case(900, 2, 1, 33)
    mp = int(t["positions"].max()) + 1
    table = ops.rope_table(t["theta"], mp)
    qs, ks = slice(450, 900), slice(0, 450)
    # each piece in its own allocation (the library wants 16-byte aligned
    # pointers, which slices of a B = 1 tensor need not be)
    c = lambda x, s: x[:, s].clone(memory_format=torch.contiguous_format)
    k_rot = ops.rope_apply(c(t["k"], ks), c(t["positions"], ks), table)
    args = (c(t["q"], qs), k_rot, c(t["v"], ks), c(t["segment_ids"], qs),
            c(t["positions"], qs), c(t["segment_ids"], ks), 450, 0,
            t["theta"], mp)
    o1, l1 = ops.fwd_block(*args)
    o2, l2 = ops.fwd_block(*args, table=table)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
