"""Pins of the ring-attention oracle (CPU, fp64).

A ring of P devices must reproduce dense attention exactly for every P and
every split (RingAttention is an exact re-organisation: "开源巨兽LWM：如何用
RingAttention撬动百万Token多模态世界", 3.1). The dense oracle itself is
pinned to torch SDPA and transformers' RoPE in test_oracle.py.
"""

import numpy as np
import pytest

import oracle
from long_context_blockwise_causal_b200 import workloads as wl


def _case(seed, B=2, N=200, H=2, D=16, lo=1, hi=90):
    rng = np.random.default_rng(seed)
    segs, poss = [], []
    for b in range(B):
        L = wl.segment_lengths("uniform", N, seed * 5 + b, lo=lo, hi=hi)
        s, p = wl.segments_from_lengths(L)
        segs.append(s)
        poss.append(p)
    q = rng.standard_normal((B, N, H, D))
    k = rng.standard_normal((B, N, H, D))
    v = rng.standard_normal((B, N, H, D))
    return q, k, v, np.stack(segs), np.stack(poss)


@pytest.mark.parametrize("P", [1, 2, 3, 5, 8])
def test_ring_equals_dense(P):
    q, k, v, seg, pos = _case(1)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e5)
    ro, rl = oracle.ring_fwd(q, k, v, seg, pos, 1e5, P)
    np.testing.assert_allclose(ro, out, atol=1e-12)
    np.testing.assert_allclose(rl, lse, atol=1e-12)


def test_ring_chunks_cover_sequence_in_order():
    for N, P in [(200, 3), (7, 8), (1024, 4), (0, 2)]:
        ch = oracle.ring_chunks(N, P)
        assert len(ch) == P
        assert sum(n for _, n in ch) == N
        off = 0
        for o, n in ch:
            assert o == off and n >= 0
            off += n
        assert max(n for _, n in ch) - min(n for _, n in ch) <= 1


def test_partial_over_everything_is_dense():
    q, k, v, seg, pos = _case(2, N=90)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    po, pl = oracle.attn_fwd_partial(q, k, v, seg, seg, pos, pos, 0, 0, 1e4)
    np.testing.assert_allclose(po, out, atol=1e-12)
    np.testing.assert_allclose(pl, lse, atol=1e-12)


def test_partial_over_future_keys_is_empty():
    q, k, v, seg, pos = _case(3, N=120)
    # queries 0..59 against keys 60..119: all keys lie in the future
    po, pl = oracle.attn_fwd_partial(q[:, :60], k[:, 60:], v[:, 60:],
                                     seg[:, :60], seg[:, 60:], pos[:, :60],
                                     pos[:, 60:], 0, 60, 1e4)
    assert np.all(po == 0) and np.all(np.isneginf(pl))


def test_partial_of_other_example_is_empty():
    # two examples of 50 tokens: the second's queries see none of the first's
    # keys, so (queries 50..99) x (keys 0..49) is empty
    B, N, H, D = 1, 100, 1, 8
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    seg = np.repeat([0, 1], 50)[None]
    pos = np.concatenate([np.arange(50), np.arange(50)])[None]
    po, pl = oracle.attn_fwd_partial(q[:, 50:], k[:, :50], v[:, :50],
                                     seg[:, 50:], seg[:, :50], pos[:, 50:],
                                     pos[:, :50], 50, 0, 1e4)
    assert np.all(po == 0) and np.all(np.isneginf(pl))


def test_partial_single_visible_key_returns_its_value():
    # a query that sees exactly one key of the block: out = that value row,
    # lse = its scaled score
    B, N, H, D = 1, 4, 1, 8
    rng = np.random.default_rng(5)
    q, k, v = (rng.standard_normal((B, N, H, D)) for _ in range(3))
    seg = np.zeros((1, N), dtype=np.int64)
    pos = np.arange(N)[None]
    # query 2 against the key block {2, 3}: only key 2 is visible
    po, pl = oracle.attn_fwd_partial(q[:, 2:3], k[:, 2:], v[:, 2:],
                                     seg[:, 2:3], seg[:, 2:], pos[:, 2:3],
                                     pos[:, 2:], 2, 2, 1e4)
    np.testing.assert_allclose(po[0, 0, 0], v[0, 2, 0], atol=1e-14)
    qr = oracle.rope_rotate(q[0, 2:3, 0], pos[0, 2:3], 1e4)
    kr = oracle.rope_rotate(k[0, 2:3, 0], pos[0, 2:3], 1e4)
    np.testing.assert_allclose(pl[0, 0, 0], float((qr @ kr.T)[0, 0]) / np.sqrt(D),
                               atol=1e-13)


def test_merge_identity_and_symmetry():
    rng = np.random.default_rng(6)
    oa = rng.standard_normal((2, 5, 3, 4))
    ob = rng.standard_normal((2, 5, 3, 4))
    la = rng.standard_normal((2, 3, 5))
    lb = rng.standard_normal((2, 3, 5))
    lb[0, 1, 2] = -np.inf
    ob[0, 2, 1] = 0.0
    empty_o, empty_l = np.zeros_like(oa), np.full_like(la, -np.inf)
    o, l_ = oracle.merge_partials(oa, la, empty_o, empty_l)
    np.testing.assert_allclose(o, oa, atol=1e-15)
    np.testing.assert_allclose(l_, la, atol=1e-15)
    o1, l1 = oracle.merge_partials(oa, la, ob, lb)
    o2, l2 = oracle.merge_partials(ob, lb, oa, la)
    np.testing.assert_allclose(o1, o2, atol=1e-14)
    np.testing.assert_allclose(l1, l2, atol=1e-14)
    # a row empty in b keeps a's values
    np.testing.assert_allclose(o1[0, 2, 1], oa[0, 2, 1], atol=1e-15)
    o, l_ = oracle.merge_partials(empty_o, empty_l, empty_o, empty_l)
    assert np.all(o == 0) and np.all(np.isneginf(l_))


@pytest.mark.parametrize("P", [1, 2, 3, 5])
def test_ring_backward_equals_dense(P):
    q, k, v, seg, pos = _case(8, N=150)
    dout = np.random.default_rng(9).standard_normal(q.shape)
    ref = oracle.attn_bwd(q, k, v, dout, seg, pos, 1e5)
    dq, dk, dv = oracle.ring_bwd(q, k, v, dout, seg, pos, 1e5, P)
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv")):
        np.testing.assert_allclose(got, ref[name], atol=1e-11)


def test_backward_partial_of_future_block_is_zero():
    q, k, v, seg, pos = _case(10, N=120)
    dout = np.random.default_rng(11).standard_normal(q.shape)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    delta = oracle.bwd_delta(out, dout)
    dq, dk, dv = oracle.attn_bwd_partial(
        q[:, :60], k[:, 60:], v[:, 60:], dout[:, :60], lse[:, :, :60],
        delta[:, :, :60], seg[:, :60], seg[:, 60:], pos[:, :60], pos[:, 60:],
        0, 60, 1e4)
    assert not dq.any() and not dk.any() and not dv.any()
