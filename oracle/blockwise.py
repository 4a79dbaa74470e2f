"""CPU online-softmax restatement in ring order (oracle; test infra only).

Used only to pin the dense oracle: the blockwise computation must equal the
dense one for every block size. Sources: blockwise attention with query and
key chunk sizes, "LWM：突破 100 万 Token 的开源大模型", 配置参数; the ring
sweep (a device's own block first, then the blocks passed to it by its
predecessors), "开源巨兽LWM：如何用RingAttention撬动百万Token多模态世界", 3.1;
FlashAttention-style online softmax, same page 3.2 and "Inside Large World
Model", Stage I.

Per query block: running max m, running sum l and accumulator acc. For each
key block j taken from the block holding the diagonal down to block 0
(key blocks with no allowed pair are skipped):
    m' = max(m, rowmax(S_j));  P = exp(S_j - m');
    l  = l * exp(m - m') + rowsum(P);  acc = acc * exp(m - m') + P V_j.
At the end out = acc / l and lse = m + log(l).
"""

import numpy as np

from .attention import _f64, _i64, allowed_mask
from .rope import rope_rotate


def blockwise_fwd(q, k, v, segment_ids, positions, theta, block_q, block_k):
    B, N, H, D = q.shape
    seg_all = _i64(segment_ids)
    pos_all = _i64(positions)
    out = np.empty((B, N, H, D))
    lse = np.empty((B, H, N))
    scale = 1.0 / np.sqrt(D)
    for b in range(B):
        seg = seg_all[b]
        pos = pos_all[b]
        for h in range(H):
            qr = rope_rotate(_f64(q[b, :, h, :]), pos, theta)
            kr = rope_rotate(_f64(k[b, :, h, :]), pos, theta)
            vb = _f64(v[b, :, h, :])
            for q0 in range(0, N, block_q):
                rows = np.arange(q0, min(q0 + block_q, N))
                m = np.full(len(rows), -np.inf)
                l_ = np.zeros(len(rows))
                acc = np.zeros((len(rows), D))
                j_diag = rows[-1] // block_k
                for j in range(j_diag, -1, -1):
                    cols = np.arange(j * block_k, min((j + 1) * block_k, N))
                    mask = allowed_mask(seg, rows, cols)
                    if not mask.any():
                        continue
                    s = np.where(mask, (qr[rows] @ kr[cols].T) * scale,
                                 -np.inf)
                    m_new = np.maximum(m, s.max(axis=1))
                    # rows with nothing allowed so far keep m = -inf
                    live = np.isfinite(m_new)
                    seen = live & np.isfinite(m)
                    alpha = np.where(
                        seen, np.exp(np.where(seen, m, 0.0)
                                     - np.where(seen, m_new, 0.0)), 0.0)
                    p = np.where(live[:, None],
                                 np.exp(s - np.where(live, m_new, 0.0)[:, None]),
                                 0.0)
                    l_ = l_ * alpha + p.sum(axis=1)
                    acc = acc * alpha[:, None] + p @ vb[cols]
                    m = m_new
                out[b, rows, h, :] = acc / l_[:, None]
                lse[b, h, rows] = m + np.log(l_)
    return out, lse
