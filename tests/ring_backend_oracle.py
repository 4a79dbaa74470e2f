"""A ring backend made of oracle calls on CPU torch tensors (fp64), for the
ring-schedule tests that run without a GPU. Keys travel already rotated, so
the partial is asked to rotate them by position 0 (the identity)."""

import numpy as np
import torch

import oracle


class OracleBackend:
    def __init__(self, theta):
        self.theta = float(theta)

    def rotate(self, k, positions):
        k = k.double().numpy()
        pos = positions.numpy()
        out = np.empty_like(k)
        for b in range(k.shape[0]):
            for h in range(k.shape[2]):
                out[b, :, h] = oracle.rope_rotate(k[b, :, h], pos[b],
                                                  self.theta)
        return torch.from_numpy(out)

    def partial(self, q, k_rot, v, seg_q, pos_q, seg_k, q_off, k_off):
        zeros = np.zeros(tuple(seg_k.shape), dtype=np.int64)
        o, l_ = oracle.attn_fwd_partial(q, k_rot, v, seg_q, seg_k, pos_q,
                                        zeros, q_off, k_off, self.theta)
        return torch.from_numpy(o), torch.from_numpy(l_)

    def merge(self, out, lse, out_part, lse_part):
        o, l_ = oracle.merge_partials(out.numpy(), lse.numpy(),
                                      out_part.numpy(), lse_part.numpy())
        return torch.from_numpy(o), torch.from_numpy(l_)

    # backward: accumulators hold gradients w.r.t. the rotated q and k
    # (scaled), so finish only rotates back
    def delta(self, out, dout):
        return torch.from_numpy(oracle.bwd_delta(out, dout))

    def zeros_acc(self, like):
        return torch.zeros(like.shape, dtype=torch.float64)

    def partial_bwd(self, q_rot, k_rot, v, dout, lse, delta, seg_q, seg_k,
                    q_off, k_off, dq_acc, dk_acc, dv_acc):
        zq = np.zeros(tuple(seg_q.shape), dtype=np.int64)
        zk = np.zeros(tuple(seg_k.shape), dtype=np.int64)
        a, b, c = oracle.attn_bwd_partial(q_rot, k_rot, v, dout, lse, delta,
                                          seg_q, seg_k, zq, zk, q_off, k_off,
                                          self.theta)
        dq_acc += torch.from_numpy(a)
        dk_acc += torch.from_numpy(b)
        dv_acc += torch.from_numpy(c)

    def finish(self, acc, positions):
        x = acc.numpy()
        pos = positions.numpy()
        out = np.empty_like(x)
        for b in range(x.shape[0]):
            for h in range(x.shape[2]):
                out[b, :, h] = oracle.rope_rotate(x[b, :, h], pos[b],
                                                  self.theta, sign=-1)
        return torch.from_numpy(out)

    def finish_v(self, acc):
        return acc.clone()

    def empty(self, q):
        B, N, H, _ = q.shape
        return (torch.zeros(q.shape, dtype=torch.float64),
                torch.full((B, H, N), float("-inf"), dtype=torch.float64))
