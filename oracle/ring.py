"""Ring attention restated on the CPU in fp64 (oracle; test infra only).

"开源巨兽LWM：如何用RingAttention撬动百万Token多模态世界", 3.1: the sequence
is cut into contiguous blocks, one per device; each device keeps its query
block while the key/value blocks travel around a ring, so that at step s
device i holds the key/value block of device (i - s) mod P. Each step
computes the attention of the local queries over the visiting keys only,
and the partial results are combined exactly with the log-sum-exp rule
(the same online-softmax identity as "LWM：突破 100 万 Token 的开源大模型",
配置参数, blockwise attention).

The backward follows the same ring: every step applies the chain rule of
the dense forward to the pairs of the visiting block only, with the final
lse and D_i = rowsum(dO * O) of the finished forward; dq collects at the
query's device, dk and dv travel with their block and are back at its
owner after the last step. The gradient is linear in the pairs, so the
block sums equal the dense gradient.

Readings: the mask of a partial is the dense one (same packed example,
key token index <= query token index) restricted to the visiting keys; a
row with no visible key in a partial has out = 0 and lse = -inf, and
contributes nothing when merged.
"""

import numpy as np

from .attention import _f64, _i64
from .rope import rope_rotate


def attn_fwd_partial(q, k, v, seg_q, seg_k, pos_q, pos_k, q_off, k_off,
                     theta):
    """Attention of query rows [q_off, q_off+Nq) over the keys
    [k_off, k_off+Nk) only. q [B,Nq,H,D]; k, v [B,Nk,H,D]; seg_*/pos_* per
    block. Returns out [B,Nq,H,D] and lse [B,H,Nq] (fp64)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    seg_q, seg_k, pos_q, pos_k = (_i64(x) for x in (seg_q, seg_k, pos_q,
                                                    pos_k))
    B, Nq, H, D = q.shape
    Nk = k.shape[1]
    scale = 1.0 / np.sqrt(D)
    out = np.zeros((B, Nq, H, D))
    lse = np.full((B, H, Nq), -np.inf)
    gi = q_off + np.arange(Nq)
    gj = k_off + np.arange(Nk)
    for b in range(B):
        mask = (seg_q[b][:, None] == seg_k[b][None, :]) & \
               (gj[None, :] <= gi[:, None])
        live = mask.any(axis=1)
        if not live.any():
            continue
        for h in range(H):
            qr = rope_rotate(q[b, :, h], pos_q[b], theta)
            kr = rope_rotate(k[b, :, h], pos_k[b], theta)
            s = np.where(mask, (qr @ kr.T) * scale, -np.inf)
            mx = np.where(live, s.max(axis=1), 0.0)
            e = np.exp(s - mx[:, None])          # 0 where masked
            l_ = e.sum(axis=1)
            o = np.zeros((Nq, D))
            o[live] = (e[live] @ v[b, :, h]) / l_[live, None]
            out[b, :, h] = o
            lse[b, h, live] = mx[live] + np.log(l_[live])
    return out, lse


def merge_partials(out_a, lse_a, out_b, lse_b):
    """Combine two partials over disjoint key sets: lse = log(e^a + e^b),
    out = e^(lse_a - lse) out_a + e^(lse_b - lse) out_b; rows where both are
    -inf give (0, -inf). Shapes as attn_fwd_partial's outputs."""
    lse = np.logaddexp(lse_a, lse_b)
    fin = np.isfinite(lse)
    safe = np.where(fin, lse, 0.0)
    wa = np.where(fin, np.exp(lse_a - safe), 0.0)   # [B,H,N]
    wb = np.where(fin, np.exp(lse_b - safe), 0.0)
    wa = np.transpose(wa, (0, 2, 1))[..., None]       # [B,N,H,1]
    wb = np.transpose(wb, (0, 2, 1))[..., None]
    return wa * out_a + wb * out_b, lse


def ring_chunks(N, P):
    """Contiguous split of N tokens over P devices: the first N % P devices
    hold one token more (the pages split evenly; this covers N % P != 0)."""
    base, extra = divmod(N, P)
    sizes = [base + (1 if i < extra else 0) for i in range(P)]
    offs = np.concatenate([[0], np.cumsum(sizes)]).astype(int)
    return [(int(offs[i]), sizes[i]) for i in range(P)]


def ring_fwd(q, k, v, segment_ids, positions, theta, P):
    """Every device of a P-device ring, in ring order, on the CPU.
    Returns out [B,N,H,D], lse [B,H,N] for the whole sequence."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    seg, pos = _i64(segment_ids), _i64(positions)
    B, N, H, D = q.shape
    out = np.zeros((B, N, H, D))
    lse = np.full((B, H, N), -np.inf)
    chunks = ring_chunks(N, P)
    for i, (qo, qn) in enumerate(chunks):
        o = np.zeros((B, qn, H, D))
        l_ = np.full((B, H, qn), -np.inf)
        for s in range(P):
            ko, kn = chunks[(i - s) % P]
            po, pl = attn_fwd_partial(
                q[:, qo:qo + qn], k[:, ko:ko + kn], v[:, ko:ko + kn],
                seg[:, qo:qo + qn], seg[:, ko:ko + kn], pos[:, qo:qo + qn],
                pos[:, ko:ko + kn], qo, ko, theta)
            o, l_ = merge_partials(o, l_, po, pl)
        out[:, qo:qo + qn] = o
        lse[:, :, qo:qo + qn] = l_
    return out, lse


def bwd_delta(out, dout):
    """D [B,H,N] = sum over d of dout * out (the finished forward's out)."""
    return np.einsum("bnhd,bnhd->bhn", _f64(out), _f64(dout))


def attn_bwd_partial(q, k, v, dout, lse, delta, seg_q, seg_k, pos_q, pos_k,
                     q_off, k_off, theta):
    """Gradient contributions of the pairs (query of [q_off, q_off+Nq), key
    of [k_off, k_off+Nk)) given the final lse and D of the queries.
    Returns dq [B,Nq,H,D], dk, dv [B,Nk,H,D] (w.r.t. un-rotated q, k)."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    lse, delta = _f64(lse), _f64(delta)
    seg_q, seg_k, pos_q, pos_k = (_i64(x) for x in (seg_q, seg_k, pos_q,
                                                    pos_k))
    B, Nq, H, D = q.shape
    Nk = k.shape[1]
    scale = 1.0 / np.sqrt(D)
    dq = np.zeros((B, Nq, H, D))
    dk = np.zeros((B, Nk, H, D))
    dv = np.zeros((B, Nk, H, D))
    gi = q_off + np.arange(Nq)
    gj = k_off + np.arange(Nk)
    for b in range(B):
        mask = (seg_q[b][:, None] == seg_k[b][None, :]) & \
               (gj[None, :] <= gi[:, None])
        for h in range(H):
            qr = rope_rotate(q[b, :, h], pos_q[b], theta)
            kr = rope_rotate(k[b, :, h], pos_k[b], theta)
            s = (qr @ kr.T) * scale
            p = np.where(mask, np.exp(np.where(mask, s, 0.0)
                                      - lse[b, h][:, None]), 0.0)
            dv[b, :, h] = p.T @ dout[b, :, h]
            dp = dout[b, :, h] @ v[b, :, h].T
            ds = p * (dp - delta[b, h][:, None])
            dq[b, :, h] = rope_rotate((ds @ kr) * scale, pos_q[b], theta,
                                      sign=-1)
            dk[b, :, h] = rope_rotate((ds.T @ qr) * scale, pos_k[b], theta,
                                      sign=-1)
    return dq, dk, dv


def ring_bwd(q, k, v, dout, segment_ids, positions, theta, P):
    """Backward of a P-device ring, every device in ring order, on the CPU.
    Returns dq, dk, dv [B,N,H,D]."""
    q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
    seg, pos = _i64(segment_ids), _i64(positions)
    out, lse = ring_fwd(q, k, v, seg, pos, theta, P)
    delta = bwd_delta(out, dout)
    dq, dk, dv = (np.zeros_like(q) for _ in range(3))
    chunks = ring_chunks(q.shape[1], P)
    for i, (qo, qn) in enumerate(chunks):
        qs = slice(qo, qo + qn)
        for s in range(P):
            ko, kn = chunks[(i - s) % P]
            ks = slice(ko, ko + kn)
            a, b_, c = attn_bwd_partial(
                q[:, qs], k[:, ks], v[:, ks], dout[:, qs], lse[:, :, qs],
                delta[:, :, qs], seg[:, qs], seg[:, ks], pos[:, qs],
                pos[:, ks], qo, ko, theta)
            dq[:, qs] += a
            dk[:, ks] += b_
            dv[:, ks] += c
    return dq, dk, dv
