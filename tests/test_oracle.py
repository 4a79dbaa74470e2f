"""Pins for the fp64 oracle, independent of the oracle itself (CPU only).

Each test ties the oracle to something it does not compute the same way:
a library routine (torch SDPA, the transformers Llama RoPE), a closed form,
an invariant, a brute-force enumeration or finite differences. A plausible
mistake (dropped 1/sqrt(D), wrong rotation sign or pair layout, a
transposed operand, an off-by-one in the causal rule, a missed segment
boundary, a wrong backward term) fails at least one of them.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F
import yaml

import oracle
from oracle import rope as orope
from long_context_blockwise_causal_b200 import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def rand_case(seed, B=1, N=96, H=2, D=16, seg_kind="uniform", lo=1, hi=40,
              scale=1.0):
    rng = np.random.default_rng(seed)
    segs, poss = [], []
    for b in range(B):
        L = wl.segment_lengths(seg_kind, N, seed * 7 + b, lo=lo, hi=hi)
        s, p = wl.segments_from_lengths(L)
        segs.append(s)
        poss.append(p)
    q = rng.standard_normal((B, N, H, D)) * scale
    k = rng.standard_normal((B, N, H, D)) * scale
    v = rng.standard_normal((B, N, H, D))
    return q, k, v, np.stack(segs), np.stack(poss)


# ---------------------------------------------------------------- RoPE pins

def _hf_rope(x_half, positions, theta):
    """transformers' Llama RoPE (rotate-half layout), fp64 math."""
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import (
        LlamaRotaryEmbedding, apply_rotary_pos_emb)
    n, d = x_half.shape
    cfg = LlamaConfig(hidden_size=2 * d, num_attention_heads=2, head_dim=d,
                      rope_theta=float(theta),
                      max_position_embeddings=int(max(positions)) + 1)
    emb = LlamaRotaryEmbedding(cfg)
    xt = torch.from_numpy(x_half)[None, None]  # [1,1,n,d]
    cos, sin = emb(xt, torch.from_numpy(np.asarray(positions))[None])
    out, _ = apply_rotary_pos_emb(xt, xt, cos, sin)
    return out[0, 0].numpy()


def test_rope_matches_transformers_llama_up_to_pair_permutation():
    # interleaved pair (2k, 2k+1) <-> rotate-half pair (k, k + D/2)
    d, n, theta = 128, 64, 1e4
    rng = np.random.default_rng(0)
    x = rng.standard_normal((n, d))
    pos = rng.integers(0, 200, n)
    perm = np.r_[np.arange(0, d, 2), np.arange(1, d, 2)]  # half <- inter
    ours = orope.rope_rotate(x, pos, theta)
    hf = _hf_rope(x[:, perm], pos, theta)
    # transformers keeps its frequencies in fp32: angle error <= 200 * 2^-24
    # per unit |x|, so allow 1e-4 absolute
    np.testing.assert_allclose(ours[:, perm], hf, atol=1e-4, rtol=0)


def test_rope_is_complex_multiplication():
    d, theta = 32, 5e7
    rng = np.random.default_rng(1)
    x = rng.standard_normal((10, d))
    pos = np.array([0, 1, 2, 7, 100, 4096, 32767, 65536, 999_999, 1_048_575])
    z = (x[:, 0::2] + 1j * x[:, 1::2]) * np.exp(
        1j * pos[:, None] * theta ** (-np.arange(0, d, 2) / d))
    r = orope.rope_rotate(x, pos, theta)
    np.testing.assert_allclose(r[:, 0::2], z.real, atol=1e-9)
    np.testing.assert_allclose(r[:, 1::2], z.imag, atol=1e-9)


def test_rope_norm_inverse_and_zero_position():
    d, theta = 128, 1e7
    rng = np.random.default_rng(2)
    x = rng.standard_normal((50, d))
    pos = rng.integers(0, 1 << 20, 50)
    r = orope.rope_rotate(x, pos, theta)
    np.testing.assert_allclose(np.linalg.norm(r, axis=1),
                               np.linalg.norm(x, axis=1), rtol=1e-12)
    back = orope.rope_rotate(r, pos, theta, sign=-1)
    np.testing.assert_allclose(back, x, atol=1e-10)
    # position 0 is the identity whatever theta is
    z = np.zeros(50, dtype=np.int64)
    for th in (1e4, 1e6, 5e7):
        np.testing.assert_array_equal(orope.rope_rotate(x, z, th), x)


def test_rope_frequencies_span_one_to_theta_inverse():
    d, theta = 128, 5e7
    f = orope.rope_inv_freq(theta, d)
    assert f[0] == 1.0 and len(f) == d // 2
    assert f[-1] == pytest.approx(theta ** (-(d - 2) / d), rel=1e-14)
    assert np.all(np.diff(f) < 0)


# -------------------------------------------------------- forward pins

def _sdpa(q, k, v, mask=None, causal=False):
    # q,k,v [n, d] fp64 -> [n, d]
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a))[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    return F.scaled_dot_product_attention(t(q), t(k), t(v), attn_mask=m,
                                          is_causal=causal)[0, 0].numpy()


def test_forward_matches_sdpa_causal_without_rotation():
    # all positions 0: no rotation; one segment: plain causal attention
    N, D = 80, 32
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, N, 1, D)) for _ in range(3))
    seg = np.zeros((1, N), np.int32)
    pos = np.zeros((1, N), np.int32)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    ref = _sdpa(q[0, :, 0], k[0, :, 0], v[0, :, 0], causal=True)
    np.testing.assert_allclose(out[0, :, 0], ref, atol=1e-12)


def test_forward_matches_sdpa_with_transformers_rope():
    N, D, theta = 64, 128, 1e6
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, N, 1, D)) for _ in range(3))
    seg = np.zeros((1, N), np.int32)
    pos = np.arange(N, dtype=np.int32)[None] + 17
    perm = np.r_[np.arange(0, D, 2), np.arange(1, D, 2)]
    qh = _hf_rope(q[0, :, 0][:, perm], pos[0], theta)
    kh = _hf_rope(k[0, :, 0][:, perm], pos[0], theta)
    ref = _sdpa(qh, kh, v[0, :, 0], causal=True)
    out, _ = oracle.attn_fwd(q, k, v, seg, pos, theta)
    np.testing.assert_allclose(out[0, :, 0], ref, atol=1e-4)


def test_packed_row_equals_each_segment_alone():
    q, k, v, seg, pos = rand_case(5, N=120, H=2, D=32, lo=1, hi=50)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    starts = np.r_[0, np.flatnonzero(np.diff(seg[0])) + 1, 120]
    for a, b in zip(starts[:-1], starts[1:]):
        # the same example alone, positions starting at 0, via SDPA
        for h in range(2):
            qr = orope.rope_rotate(q[0, a:b, h], np.arange(b - a), 1e4)
            kr = orope.rope_rotate(k[0, a:b, h], np.arange(b - a), 1e4)
            ref = _sdpa(qr, kr, v[0, a:b, h], causal=True)
            np.testing.assert_allclose(out[0, a:b, h], ref, atol=1e-12)


def test_zero_queries_give_mean_of_allowed_values_and_log_count():
    q, k, v, seg, pos = rand_case(6, N=100, H=3, D=16)
    q[:] = 0.0
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    s = seg[0]
    for i in range(100):
        allowed = [j for j in range(i + 1) if s[j] == s[i]]
        for h in range(3):
            np.testing.assert_allclose(out[0, i, h], v[0, allowed, h].mean(0),
                                       atol=1e-12)
            assert lse[0, h, i] == pytest.approx(math.log(len(allowed)),
                                                 abs=1e-12)


def test_length_one_segment_returns_own_value_and_self_score():
    # rotation by one common angle keeps dot products, so the self score
    # is q.k / sqrt(D) for any position
    N, D = 40, 64
    rng = np.random.default_rng(7)
    q, k, v = (rng.standard_normal((1, N, 2, D)) for _ in range(3))
    seg = np.arange(N, dtype=np.int32)[None]  # every token its own example
    pos = rng.integers(0, 10 ** 6, (1, N)).astype(np.int32)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 5e7)
    np.testing.assert_allclose(out, v, atol=1e-12)
    self_score = (q * k).sum(-1) / math.sqrt(D)  # [1, N, 2]
    np.testing.assert_allclose(lse, self_score.transpose(0, 2, 1), atol=1e-9)


def test_unit_values_give_unit_output():
    q, k, v, seg, pos = rand_case(8, N=90, H=2, D=16, scale=3.0)
    v[:] = 1.0
    out, _ = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    np.testing.assert_allclose(out, 1.0, atol=1e-12)


def test_shift_of_all_positions_changes_nothing():
    # scores depend only on p_i - p_j
    q, k, v, seg, _ = rand_case(9, N=64, H=2, D=32, lo=64, hi=64)
    pos = np.arange(64, dtype=np.int32)[None]
    o1, l1 = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    o2, l2 = oracle.attn_fwd(q, k, v, seg, pos + 12345, 1e4)
    np.testing.assert_allclose(o1, o2, atol=1e-9)
    np.testing.assert_allclose(l1, l2, atol=1e-9)


def test_mask_against_enumeration():
    seg = np.array([0, 0, 0, 1, 1, 2, 3, 3, 3, 3, 4])
    n = len(seg)
    rows = np.arange(n)
    m = oracle.allowed_mask(seg, rows, rows)
    for i in range(n):
        for j in range(n):
            assert m[i, j] == (seg[i] == seg[j] and j <= i)


def test_sampled_rows_equal_full_forward():
    q, k, v, seg, pos = rand_case(10, N=77, H=2, D=16)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e6)
    rows = np.array([0, 5, 31, 76])
    o, l_ = oracle.attention.attn_fwd_rows(q, k, v, seg, pos, 1e6, 0, 1,
                                           rows, row_block=3)
    np.testing.assert_allclose(o, out[0, rows, 1], atol=1e-13)
    np.testing.assert_allclose(l_, lse[0, 1, rows], atol=1e-13)


@pytest.mark.parametrize("bq,bk", [(16, 16), (32, 32), (64, 64), (128, 128),
                                   (32, 16), (64, 32)])
def test_blockwise_online_softmax_equals_dense(bq, bk):
    # N not a multiple of the block: a ragged tail block
    q, k, v, seg, pos = rand_case(11, B=2, N=200, H=2, D=16, lo=1, hi=90)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    ob, lb = oracle.blockwise_fwd(q, k, v, seg, pos, 1e4, bq, bk)
    np.testing.assert_allclose(ob, out, atol=1e-12)
    np.testing.assert_allclose(lb, lse, atol=1e-12)


# -------------------------------------------------------- backward pins

def _loss(q, k, v, seg, pos, theta, g):
    out, _ = oracle.attn_fwd(q, k, v, seg, pos, theta)
    return float((out * g).sum())


def test_backward_finite_differences():
    q, k, v, seg, pos = rand_case(12, N=40, H=2, D=8, lo=1, hi=25)
    theta = 1e4
    rng = np.random.default_rng(13)
    g = rng.standard_normal(q.shape)
    res = oracle.attn_bwd(q, k, v, g, seg, pos, theta)
    eps = 1e-6
    for name, x in (("dq", q), ("dk", k), ("dv", v)):
        for trial in range(3):
            u = rng.standard_normal(x.shape)
            xp, xm = x + eps * u, x - eps * u
            args = {"dq": (0,), "dk": (1,), "dv": (2,)}[name][0]
            ins_p = [q, k, v]
            ins_m = [q, k, v]
            ins_p[args] = xp
            ins_m[args] = xm
            fd = (_loss(*ins_p, seg, pos, theta, g)
                  - _loss(*ins_m, seg, pos, theta, g)) / (2 * eps)
            an = float((res[name] * u).sum())
            assert an == pytest.approx(fd, rel=1e-6, abs=1e-8), name


def test_backward_matches_torch_autograd_of_library_ops():
    # rotation from transformers' Llama RoPE (permuted), attention from SDPA
    # with a boolean packing+causal mask, gradients from autograd
    from transformers import LlamaConfig
    from transformers.models.llama.modeling_llama import (
        LlamaRotaryEmbedding, apply_rotary_pos_emb)
    B, N, H, D, theta = 1, 70, 2, 32, 1e5
    q, k, v, seg, pos = rand_case(14, B=B, N=N, H=H, D=D, lo=1, hi=40)
    rng = np.random.default_rng(15)
    g = rng.standard_normal(q.shape)
    perm = np.r_[np.arange(0, D, 2), np.arange(1, D, 2)]
    cfg = LlamaConfig(hidden_size=2 * D, num_attention_heads=2, head_dim=D,
                      rope_theta=theta, max_position_embeddings=N)
    emb = LlamaRotaryEmbedding(cfg)
    tq = torch.tensor(q[..., perm], requires_grad=True)
    tk = torch.tensor(k[..., perm], requires_grad=True)
    tv = torch.tensor(v, requires_grad=True)
    cos, sin = emb(tq, torch.from_numpy(pos.astype(np.int64)))
    qt, kt = apply_rotary_pos_emb(tq.transpose(1, 2), tk.transpose(1, 2),
                                  cos, sin)
    mask = torch.from_numpy(oracle.allowed_mask(seg[0], np.arange(N),
                                                np.arange(N)))
    o = F.scaled_dot_product_attention(qt, kt, tv.transpose(1, 2),
                                       attn_mask=mask)
    (o.transpose(1, 2) * torch.from_numpy(g)).sum().backward()
    res = oracle.attn_bwd(q, k, v, g, seg, pos, theta)
    inv = np.argsort(perm)
    # transformers' fp32 frequencies put ~1e-5 relative error on the
    # rotation; gradients of size ~3 then differ by up to ~5e-4
    np.testing.assert_allclose(res["dq"], tq.grad.numpy()[..., inv],
                               atol=5e-4)
    np.testing.assert_allclose(res["dk"], tk.grad.numpy()[..., inv],
                               atol=5e-4)
    np.testing.assert_allclose(res["dv"], tv.grad.numpy(), atol=1e-5)


def test_backward_forward_outputs_match_forward():
    q, k, v, seg, pos = rand_case(16, N=50, H=2, D=16)
    g = np.ones_like(q)
    res = oracle.attn_bwd(q, k, v, g, seg, pos, 1e4, row_block=7)
    out, lse = oracle.attn_fwd(q, k, v, seg, pos, 1e4)
    np.testing.assert_allclose(res["out"], out, atol=1e-13)
    np.testing.assert_allclose(res["lse"], lse, atol=1e-13)


# ------------------------------------------------------ classifier pins

def test_classifier_plain_causal_closed_form():
    N, b = 1024, 128
    seg = np.zeros((1, N), np.int32)
    lo, hi, cls = oracle.classify_bruteforce(seg, b, b)
    t = np.arange(N // b)
    np.testing.assert_array_equal(lo[0], 0)
    np.testing.assert_array_equal(hi[0], t)
    expect = np.where(t[None, :] < t[:, None], oracle.TILE_FULL,
                      np.where(t[None, :] == t[:, None], oracle.TILE_PARTIAL,
                               oracle.TILE_EMPTY))
    np.testing.assert_array_equal(cls[0], expect)
    # key blocks half as tall: both halves of the diagonal are PARTIAL
    lo, hi, cls = oracle.classify_bruteforce(seg, 128, 64)
    np.testing.assert_array_equal(hi[0], 2 * t + 1)
    assert cls[0, 3, 6] == oracle.TILE_PARTIAL
    assert cls[0, 3, 7] == oracle.TILE_PARTIAL
    assert cls[0, 3, 5] == oracle.TILE_FULL


def test_classifier_each_token_alone_is_diagonal_only():
    N = 300
    seg = np.arange(N, dtype=np.int32)[None]
    lo, hi, cls = oracle.classify_bruteforce(seg, 64, 64)
    t = np.arange(-(-N // 64))
    np.testing.assert_array_equal(lo[0], t)
    np.testing.assert_array_equal(hi[0], t)
    assert (cls[0][np.eye(len(t), dtype=bool)] == oracle.TILE_PARTIAL).all()
    assert (cls[0][~np.eye(len(t), dtype=bool)] == oracle.TILE_EMPTY).all()


@pytest.mark.parametrize("seed,N,bq,bk", [(0, 1000, 128, 128),
                                          (1, 777, 128, 64),
                                          (2, 2048, 128, 128),
                                          (3, 1536, 64, 64)])
def test_classifier_count_equals_bruteforce(seed, N, bq, bk):
    L = wl.segment_lengths("uniform", N, seed, lo=1, hi=400)
    seg, _ = wl.segments_from_lengths(L)
    a = oracle.classify_bruteforce(seg[None], bq, bk)
    c = oracle.classify_count(seg[None], bq, bk)
    for x, y in zip(a, c):
        np.testing.assert_array_equal(x, y)


def test_ragged_tail_tile_is_never_full():
    N = 200  # last block rows/cols 128..199 of a 128 block
    seg = np.zeros((1, N), np.int32)
    _, _, cls = oracle.classify_bruteforce(seg, 128, 128)
    # rows 200..255 of query block 1 lie past N: not allowed, so not FULL
    assert cls[0, 1, 0] == oracle.TILE_PARTIAL
    assert cls[0, 1, 1] == oracle.TILE_PARTIAL
    _, _, cls = oracle.classify_bruteforce(np.zeros((1, 256), np.int32),
                                           128, 128)
    assert cls[0, 1, 0] == oracle.TILE_FULL


def test_cross_classification_of_the_whole_row_is_the_square_one():
    L = wl.segment_lengths("uniform", 700, 5, lo=1, hi=250)
    seg, _ = wl.segments_from_lengths(L)
    seg = np.stack([seg, np.repeat(np.arange(3, dtype=np.int32),
                                   [100, 300, 300])])
    a = oracle.classify_bruteforce(seg, 128, 128)
    c = oracle.classify_cross(seg, 0, 700, 0, 700, 128, 128)
    for x, y in zip(a, c):
        np.testing.assert_array_equal(x, y)


@pytest.mark.parametrize("q_off,Nq,k_off,Nk", [(300, 500, 0, 300),
                                               (256, 384, 256, 384),
                                               (0, 200, 500, 300),
                                               (130, 333, 7, 250)])
def test_cross_classification_single_segment_closed_form(q_off, Nq, k_off,
                                                         Nk):
    # one causal segment: key c visible to row r iff c <= r
    N = 1000
    seg = np.zeros((1, N), np.int32)
    lo, hi, cls = oracle.classify_cross(seg, q_off, Nq, k_off, Nk, 128, 128)
    for t in range(-(-Nq // 128)):
        r0, r1 = q_off + 128 * t, q_off + min(128 * (t + 1), Nq) - 1
        for s in range(-(-Nk // 128)):
            c0, c1 = k_off + 128 * s, k_off + min(128 * (s + 1), Nk) - 1
            whole = (r1 - r0 == 127) and (c1 - c0 == 127)
            want = (oracle.TILE_EMPTY if c0 > r1 else
                    oracle.TILE_FULL if whole and c1 <= r0 else
                    oracle.TILE_PARTIAL)
            assert cls[0, t, s] == want, (t, s)


def test_visible_ranges_closed_forms():
    N = 600
    one = np.zeros(N, np.int32)
    rows = np.arange(N)
    lo, hi = oracle.visible_key_ranges(one, rows, 200, 250)
    seen = rows >= 200
    np.testing.assert_array_equal(lo[seen], 200)
    np.testing.assert_array_equal(hi[seen], np.minimum(rows[seen], 449))
    assert (lo[~seen] == -1).all() and (hi[~seen] == -2).all()
    ql, qh = oracle.visible_query_ranges(one, rows, 100, 300)
    seen = rows <= 399
    np.testing.assert_array_equal(ql[seen], np.maximum(rows[seen], 100))
    np.testing.assert_array_equal(qh[seen], 399)
    assert (ql[~seen] == -1).all()
    alone = np.arange(N, dtype=np.int32)
    lo, hi = oracle.visible_key_ranges(alone, rows, 0, N)
    np.testing.assert_array_equal(lo, rows)
    np.testing.assert_array_equal(hi, rows)


@pytest.mark.parametrize("P", [1, 3, 4])
def test_visible_ranges_over_ring_chunks_count_every_pair_once(P):
    # summed over the P key chunks of a ring, the row ranges (and the
    # key-side ranges) cover exactly the sum over examples of L(L+1)/2
    L = wl.segment_lengths("uniform", 900, 11, lo=1, hi=300)
    seg, _ = wl.segments_from_lengths(L)
    bounds = np.linspace(0, 900, P + 1).astype(int)
    rows = np.arange(900)
    tot_r = tot_c = 0
    for a, z in zip(bounds[:-1], bounds[1:]):
        lo, hi = oracle.visible_key_ranges(seg, rows, a, z - a)
        tot_r += int(np.maximum(hi - lo + 1, 0).sum())
        ql, qh = oracle.visible_query_ranges(seg, rows, a, z - a)
        tot_c += int(np.maximum(qh - ql + 1, 0).sum())
    want = int((L * (L + 1) // 2).sum())
    assert tot_r == want and tot_c == want


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_cross_classification_agrees_with_row_ranges(seed):
    # a tile is EMPTY iff no row range meets its key block, FULL iff the
    # block is whole and every row range covers its key block
    N = 1100
    L = wl.segment_lengths("uniform", N, 20 + seed, lo=1, hi=400)
    seg, _ = wl.segments_from_lengths(L)
    q_off, Nq, k_off, Nk = [(0, N, 0, N), (400, 700, 100, 500),
                            (520, 580, 390, 260)][seed]
    lo_, hi_, cls = oracle.classify_cross(seg[None], q_off, Nq, k_off, Nk,
                                          128, 128)
    lo, hi = oracle.visible_key_ranges(seg, np.arange(q_off, q_off + Nq),
                                       k_off, Nk)
    for t in range(cls.shape[1]):
        r = slice(128 * t, min(128 * (t + 1), Nq))
        for s in range(cls.shape[2]):
            c0, c1 = k_off + 128 * s, k_off + min(128 * (s + 1), Nk) - 1
            meet = (lo[r] <= c1) & (hi[r] >= c0) & (lo[r] <= hi[r])
            cover = (lo[r] <= c0) & (hi[r] >= c1)
            whole = (r.stop - r.start == 128) and (c1 - c0 == 127)
            want = (oracle.TILE_EMPTY if not meet.any() else
                    oracle.TILE_FULL if whole and cover.all() else
                    oracle.TILE_PARTIAL)
            assert cls[0, t, s] == want, (t, s)


# ------------------------------------------------- workloads and page facts

def test_workloads_use_page_facts():
    facts = yaml.safe_load(open(
        __file__.rsplit("/", 1)[0] + "/golden/page_facts.yaml"))
    w = wl.WORKLOADS
    assert w["tiny2k"].block_q == facts["scan_query_chunk_size"]["value"]
    assert w["tiny2k"].block_k == facts["scan_key_chunk_size"]["value"]
    assert w["vl256k"].theta == facts["theta_vision_32k"]["value"]
    assert w["stress1m"].theta == facts["theta_vision_32k"]["value"]
    assert wl.TOKENS_PER_FRAME == facts["vq_tokens_per_frame"]["value"] + 1
    assert [w[n].N for n in ("text32k", "packed128k", "vl256k",
                             "stress1m")] == facts["context_sizes"]["value"]


def test_segment_generators_shapes():
    for name, w in wl.WORKLOADS.items():
        if w.N > 300_000:
            continue
        L = wl.segment_lengths(w.segments, w.N, 0, **w.seg_args)
        assert L.sum() == w.N and (L > 0).all()
        seg, pos = wl.segments_from_lengths(L)
        assert (np.diff(seg) >= 0).all()
        assert (pos[np.r_[0, np.cumsum(L)[:-1]]] == 0).all()
    L = wl.segment_lengths("vision_text", 262144, 0,
                           **wl.WORKLOADS["vl256k"].seg_args)
    video = L[L % wl.TOKENS_PER_FRAME == 0]
    assert len(video) > 0
    assert wl.visible_pairs([np.array([3, 1])]) == 7


def test_sampled_backward_rows_and_cols_equal_full_backward():
    q, k, v, seg, pos = rand_case(17, N=90, H=2, D=16, lo=1, hi=40)
    g = np.random.default_rng(18).standard_normal(q.shape)
    full = oracle.attn_bwd(q, k, v, g, seg, pos, 1e5)
    rows = np.array([0, 3, 44, 89])
    dq = oracle.attn_bwd_rows(q, k, v, g, seg, pos, 1e5, 0, 1, rows,
                              row_block=3)
    np.testing.assert_allclose(dq, full["dq"][0, rows, 1], atol=1e-12)
    dk, dv = oracle.attn_bwd_cols(q, k, v, g, seg, pos, 1e5, 0, 0, rows,
                                  row_block=7)
    np.testing.assert_allclose(dk, full["dk"][0, rows, 0], atol=1e-12)
    np.testing.assert_allclose(dv, full["dv"][0, rows, 0], atol=1e-12)


# ------------------------------------------------- rotate-half layout pins

def test_rope_rotate_half_matches_transformers_llama():
    d, n, theta = 128, 64, 1e6
    rng = np.random.default_rng(30)
    x = rng.standard_normal((n, d))
    pos = rng.integers(0, 300, n)
    # fp32 frequencies inside transformers: angle error <= 300 * 2^-24
    np.testing.assert_allclose(orope.rope_rotate_half(x, pos, theta),
                               _hf_rope(x, pos, theta), atol=1e-4, rtol=0)


def test_rotate_half_is_interleaved_rope_under_the_permutation():
    d, n, theta = 128, 50, 5e7
    rng = np.random.default_rng(31)
    x = rng.standard_normal((3, n, d))
    pos = rng.integers(0, 10 ** 6, n)
    for sign in (1, -1):
        via = orope.interleaved_to_half(
            orope.rope_rotate(orope.half_to_interleaved(x), pos, theta, sign))
        np.testing.assert_allclose(orope.rope_rotate_half(x, pos, theta, sign),
                                   via, atol=1e-12, rtol=0)
    y = rng.standard_normal((4, d))
    assert np.array_equal(orope.interleaved_to_half(orope.half_to_interleaved(y)), y)
    assert np.array_equal(orope.half_to_interleaved(y)[:, 1], y[:, d // 2])


def test_attention_in_rotate_half_layout_equals_permuted_interleaved():
    # scores only see dot products of q and k rotated in one layout, so
    # attention on rotate-half inputs equals the oracle on permuted inputs
    q, k, v, seg, pos = rand_case(32, N=90, H=2, D=16)
    theta = 1e4
    out, lse = oracle.attn_fwd(orope.half_to_interleaved(q),
                               orope.half_to_interleaved(k), v, seg, pos,
                               theta)
    b, h = 0, 1
    qr = orope.rope_rotate_half(q[b, :, h], pos[b], theta)
    kr = orope.rope_rotate_half(k[b, :, h], pos[b], theta)
    rows = np.arange(90)
    s = np.where(oracle.allowed_mask(seg[b], rows, rows), qr @ kr.T / 4.0,
                 -np.inf)
    ref_lse = np.log(np.exp(s - s.max(1, keepdims=True)).sum(1)) + s.max(1)
    ref_out = np.exp(s - ref_lse[:, None]) @ v[b, :, h]
    np.testing.assert_allclose(out[b, :, h], ref_out, atol=1e-12)
    np.testing.assert_allclose(lse[b, h], ref_lse, atol=1e-12)


def test_input_prefix_draw_equals_full_draw_prefix():
    # the generator's prefix mode (used to time the oracle on a sample) must
    # give exactly the first tokens of the full draw, across chunk borders
    w = wl.Workload("t", 2, 300, 3, 16, 1e4, "uniform", 0.5, True,
                    seg_args={"lo": 1, "hi": 50})
    full = wl.make_inputs(w, 4)
    for n in (1, 77, 300):
        part = wl.make_inputs(w, 4, prefix=n)
        for k in ("q", "k", "v", "dout", "segment_ids", "positions"):
            assert torch.equal(part[k], full[k][:, :n]), (k, n)
    x = wl.random_tensor((1, 50, 2, 8), 9, 1.0, torch.float32, "cpu",
                         chunk_elems=64)
    y = wl.random_tensor((1, 50, 2, 8), 9, 1.0, torch.float32, "cpu",
                         chunk_elems=64, n_tokens=13)
    assert torch.equal(x[:, :13], y)
