"""Dense masked RoPE attention in fp64 (oracle; test infrastructure only).

This is the plain definition the blockwise kernels re-organise: the whole
masked score row is materialised (in blocks of rows, each block still spans
every one of the N columns, -inf included), then softmax-normalised.

Sources:
* causal autoregressive transformer -- "LWM：突破 100 万 Token 的开源大模型",
  概述; "Inside Large World Model", Core Architecture;
* masked sequence packing (a token sees only tokens of its own packed
  example) -- "LWM：突破 100 万 Token 的开源大模型", 概述 (b); "[论文解读]
  World Model on Million-Length Video And Language With Blockwise
  RingAttention", 提出的方法;
* RoPE with a context-scaled theta -- same review, 提出的方法;
* blockwise computation is an exact re-organisation, used for memory --
  "LWM：突破 100 万 Token 的开源大模型", 配置参数; "开源巨兽LWM：如何用
  RingAttention撬动百万Token多模态世界", 3.1.

Readings (the pages are silent on them):
* softmax scale 1/sqrt(D) (Llama-2 backbone, "Inside Large World Model",
  Stage I);
* the causal rule compares token indices inside the packed row; positions
  only drive RoPE;
* segment ids are contiguous runs (what packing produces);
* lse is the natural-log logsumexp of the scaled scores;
* the backward pass is the chain rule of this forward, with gradients taken
  with respect to the un-rotated q and k.

Layouts: q, k, v, dout [B, N, H, D]; segment_ids, positions [B, N];
out [B, N, H, D]; lse [B, H, N].
"""

import numpy as np

from .rope import rope_rotate

SOFTMAX_SCALE_RULE = "1/sqrt(D)"


def _f64(x):
    if hasattr(x, "detach"):  # a torch tensor: go through fp32 exactly
        x = x.detach().cpu()
        if str(x.dtype) in ("torch.bfloat16", "torch.float16"):
            x = x.float()
        x = x.numpy()
    return np.asarray(x, dtype=np.float64)


def _i64(x):
    if hasattr(x, "detach"):
        x = x.detach().cpu().numpy()
    return np.asarray(x, dtype=np.int64)


def allowed_mask(seg, rows, cols):
    """A(i) membership: seg[j] == seg[i] and j <= i (token index)."""
    seg = np.asarray(seg)
    rows = np.asarray(rows)
    cols = np.asarray(cols)
    same = seg[rows][:, None] == seg[cols][None, :]
    causal = cols[None, :] <= rows[:, None]
    return same & causal


def _scores(qr_blk, kr, scale, mask):
    s = (qr_blk @ kr.T) * scale
    return np.where(mask, s, -np.inf)


def attn_fwd_rows(q, k, v, segment_ids, positions, theta, b, h, rows,
                  row_block=256):
    """Forward for query rows ``rows`` of batch b, head h.

    Returns (out [len(rows), D], lse [len(rows)]), both fp64.
    """
    seg = _i64(segment_ids)[b]
    pos = _i64(positions)[b]
    rows = np.asarray(rows, dtype=np.int64)
    kb = _f64(k[b, :, h, :])
    vb = _f64(v[b, :, h, :])
    n, d = kb.shape
    scale = 1.0 / np.sqrt(d)
    kr = rope_rotate(kb, pos, theta)
    cols = np.arange(n)
    out = np.empty((len(rows), d), dtype=np.float64)
    lse = np.empty(len(rows), dtype=np.float64)
    for s0 in range(0, len(rows), row_block):
        r = rows[s0:s0 + row_block]
        qr = rope_rotate(_f64(q[b, r, h, :]), pos[r], theta)
        s = _scores(qr, kr, scale, allowed_mask(seg, r, cols))
        mx = s.max(axis=1, keepdims=True)  # finite: every row sees itself
        l_ = np.log(np.exp(s - mx).sum(axis=1, keepdims=True)) + mx
        p = np.exp(s - l_)
        out[s0:s0 + len(r)] = p @ vb
        lse[s0:s0 + len(r)] = l_[:, 0]
    return out, lse


def attn_fwd(q, k, v, segment_ids, positions, theta, heads=None,
             row_block=256):
    """Full forward. Returns out [B,N,H,D] and lse [B,H,N] in fp64.

    ``heads`` restricts the computation to a subset of heads (the others
    are left at NaN so a caller cannot mistake them for results).
    """
    B, N, H, D = q.shape
    heads = range(H) if heads is None else heads
    out = np.full((B, N, H, D), np.nan)
    lse = np.full((B, H, N), np.nan)
    rows = np.arange(N)
    for b in range(B):
        for h in heads:
            o, l_ = attn_fwd_rows(q, k, v, segment_ids, positions, theta, b,
                                  h, rows, row_block)
            out[b, :, h, :] = o
            lse[b, h, :] = l_
    return out, lse


def attn_bwd(q, k, v, dout, segment_ids, positions, theta, heads=None,
             row_block=256):
    """Chain rule of the forward, fp64.

    Returns dict with dq, dk, dv [B,N,H,D] and the forward's out, lse.
    With P = exp(S - lse): dV = P^T dO; dP = dO V^T;
    dS = P * (dP - rowsum(dO * O)); dq~ = dS k~ / sqrt(D);
    dk~ = dS^T q~ / sqrt(D); dq = R(-pos) dq~; dk = R(-pos) dk~.
    """
    B, N, H, D = q.shape
    heads = list(range(H)) if heads is None else list(heads)
    seg_all = _i64(segment_ids)
    pos_all = _i64(positions)
    dq = np.full((B, N, H, D), np.nan)
    dk = np.full((B, N, H, D), np.nan)
    dv = np.full((B, N, H, D), np.nan)
    out = np.full((B, N, H, D), np.nan)
    lse = np.full((B, H, N), np.nan)
    scale = 1.0 / np.sqrt(D)
    cols = np.arange(N)
    for b in range(B):
        seg = seg_all[b]
        pos = pos_all[b]
        for h in heads:
            qr = rope_rotate(_f64(q[b, :, h, :]), pos, theta)
            kr = rope_rotate(_f64(k[b, :, h, :]), pos, theta)
            vb = _f64(v[b, :, h, :])
            dob = _f64(dout[b, :, h, :])
            o = np.empty((N, D))
            ls = np.empty(N)
            for s0 in range(0, N, row_block):
                r = cols[s0:s0 + row_block]
                s = _scores(qr[r], kr, scale, allowed_mask(seg, r, cols))
                mx = s.max(axis=1, keepdims=True)
                l_ = np.log(np.exp(s - mx).sum(axis=1, keepdims=True)) + mx
                o[r] = np.exp(s - l_) @ vb
                ls[r] = l_[:, 0]
            delta = (dob * o).sum(axis=1)
            dqr = np.empty((N, D))
            dkr = np.zeros((N, D))
            dvb = np.zeros((N, D))
            for s0 in range(0, N, row_block):
                r = cols[s0:s0 + row_block]
                s = _scores(qr[r], kr, scale, allowed_mask(seg, r, cols))
                p = np.exp(s - ls[r][:, None])
                dvb += p.T @ dob[r]
                dp = dob[r] @ vb.T
                ds = p * (dp - delta[r][:, None])
                dqr[r] = (ds @ kr) * scale
                dkr += (ds.T @ qr[r]) * scale
            dq[b, :, h, :] = rope_rotate(dqr, pos, theta, sign=-1)
            dk[b, :, h, :] = rope_rotate(dkr, pos, theta, sign=-1)
            dv[b, :, h, :] = dvb
            out[b, :, h, :] = o
            lse[b, h, :] = ls
    return {"dq": dq, "dk": dk, "dv": dv, "out": out, "lse": lse}


def attn_bwd_rows(q, k, v, dout, segment_ids, positions, theta, b, h, rows,
                  row_block=256):
    """dq at query rows ``rows`` of (b, h), fp64 [len(rows), D].

    Only row i's own softmax enters dq_i: dq~_i = sum_j dS_ij k~_j / sqrt(D)
    with dS_ij = P_ij (dP_ij - dO_i . O_i), so the rows can be computed one
    by one at any sequence length.
    """
    seg = _i64(segment_ids)[b]
    pos = _i64(positions)[b]
    rows = np.asarray(rows, dtype=np.int64)
    kb = _f64(k[b, :, h, :])
    vb = _f64(v[b, :, h, :])
    n, d = kb.shape
    scale = 1.0 / np.sqrt(d)
    kr = rope_rotate(kb, pos, theta)
    cols = np.arange(n)
    dq = np.empty((len(rows), d))
    for s0 in range(0, len(rows), row_block):
        r = rows[s0:s0 + row_block]
        qr = rope_rotate(_f64(q[b, r, h, :]), pos[r], theta)
        s = _scores(qr, kr, scale, allowed_mask(seg, r, cols))
        mx = s.max(axis=1, keepdims=True)
        l_ = np.log(np.exp(s - mx).sum(axis=1, keepdims=True)) + mx
        p = np.exp(s - l_)
        o = p @ vb
        dob = _f64(dout[b, r, h, :])
        delta = (dob * o).sum(axis=1, keepdims=True)
        ds = p * (dob @ vb.T - delta)
        dq[s0:s0 + len(r)] = rope_rotate((ds @ kr) * scale, pos[r], theta,
                                         sign=-1)
    return dq


def attn_bwd_cols(q, k, v, dout, segment_ids, positions, theta, b, h, cols,
                  row_block=256):
    """dk, dv at key columns ``cols`` of (b, h), fp64 [len(cols), D] each.

    Key j collects from every query i that sees it, so the forward of the
    whole head (lse_i, O_i for all i) is computed first.
    """
    seg = _i64(segment_ids)[b]
    pos = _i64(positions)[b]
    cols = np.asarray(cols, dtype=np.int64)
    qb = _f64(q[b, :, h, :])
    kb = _f64(k[b, :, h, :])
    vb = _f64(v[b, :, h, :])
    dob = _f64(dout[b, :, h, :])
    n, d = kb.shape
    scale = 1.0 / np.sqrt(d)
    qr = rope_rotate(qb, pos, theta)
    kr = rope_rotate(kb, pos, theta)
    allc = np.arange(n)
    dk_r = np.zeros((len(cols), d))
    dv_ = np.zeros((len(cols), d))
    for s0 in range(0, n, row_block):
        r = allc[s0:s0 + row_block]
        s = _scores(qr[r], kr, scale, allowed_mask(seg, r, allc))
        mx = s.max(axis=1, keepdims=True)
        l_ = np.log(np.exp(s - mx).sum(axis=1, keepdims=True)) + mx
        p_all = np.exp(s - l_)
        o = p_all @ vb
        delta = (dob[r] * o).sum(axis=1, keepdims=True)
        p = p_all[:, cols]
        ds = p * (dob[r] @ vb[cols].T - delta)
        dv_ += p.T @ dob[r]
        dk_r += (ds.T @ qr[r]) * scale
    return rope_rotate(dk_r, pos[cols], theta, sign=-1), dv_
