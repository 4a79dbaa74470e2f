"""ctypes binding of liblwm_blockattn.so (argument marshalling only).

Every step of the attention path runs in the library's CUDA kernels; this
module turns torch tensors into device pointers, sizes and the current
stream, and turns status codes into exceptions. It never computes
anything itself and has no fallback: without the built library (or on a
tensor that is not on a CUDA device) it raises.
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "liblwm_blockattn.so")
_lib = None

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, \
    ERR_TIMEOUT, ERR_PRECONDITION = range(7)
DTYPE_BF16, DTYPE_FP32 = 0, 1
QK_BF16, QK_BF16X3 = 0, 1
ROPE_INTERLEAVED, ROPE_HALF = 0, 1
TILE_EMPTY, TILE_PARTIAL, TILE_FULL = 0, 1, 2
BLOCK = 128
HEAD_DIM = 128

_vp = ctypes.c_void_p
_i = ctypes.c_int
_sz = ctypes.c_size_t
_d = ctypes.c_double

_SIGS = {
    "lwm_blockattn_fwd_workspace_size": (_sz, [_i] * 9),
    "lwm_blockattn_bwd_workspace_size": (_sz, [_i] * 9),
    "lwm_blockattn_fwd": (_i, [_vp, _vp, _vp, _vp, _vp, _d, _i, _i, _i,
                               _i, _i, _i, _i, _i, _i, _i, _vp, _vp, _vp,
                               _sz, _vp]),
    "lwm_blockattn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _d,
                               _i, _i, _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                               _vp, _vp, _vp, _sz, _vp]),
    "lwm_blockattn_classify": (_i, [_vp, _i, _i, _i, _i, _vp, _vp, _vp,
                                    _vp]),
    "lwm_blockattn_rope_table": (_i, [_d, _i, _i, _vp, _vp]),
    "lwm_blockattn_visibility": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _i, _i]
                                 + [_vp] * 13),
    "lwm_blockattn_check_inputs": (_i, [_vp, _vp, _i, _i, _i,
                                        ctypes.POINTER(_i), _vp]),
    "lwm_blockattn_last_status": (_i, [_vp]),
    "lwm_status_string": (ctypes.c_char_p, [_i]),
    "lwm_blockattn_version": (_i, []),
    "lwm_blockattn_kernel_launches": (ctypes.c_uint64, []),
    "lwm_blockattn_selftest_wait_timeout": (_i, [ctypes.c_uint64, _vp]),
    "lwm_blockattn_rope_apply": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                      _i, _vp, _vp]),
    "lwm_blockattn_decode_workspace_size": (_sz, [_i, _i, _i, _i]),
    "lwm_blockattn_decode": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i,
                                  _i, _i, _i, _i, _i, _vp, _vp, _vp, _sz,
                                  _vp]),
    "lwm_blockattn_fwd_noalloc": (_i, [_vp, _vp, _vp, _vp, _vp, _d, _i, _i,
                                       _i, _i, _i, _i, _i, _i, _i, _i, _vp,
                                       _vp, _vp]),
    "lwm_blockattn_fwd_block_workspace_size": (_sz, [_i] * 6),
    "lwm_blockattn_fwd_block": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i,
                                     _d, _i, _vp, _i, _i, _i, _i, _i, _i,
                                     _vp, _vp, _vp, _sz, _vp]),
    "lwm_blockattn_merge": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                                 _vp]),
    "lwm_blockattn_bwd_delta": (_i, [_vp, _vp, _i, _i, _i, _i, _i, _vp,
                                     _vp]),
    "lwm_blockattn_bwd_block_workspace_size": (_sz, [_i] * 5),
    "lwm_blockattn_bwd_block": (_i, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                     _i, _i, _i, _i, _i, _i, _i, _vp, _vp,
                                     _vp, _vp, _sz, _vp]),
    "lwm_blockattn_grad_finish": (_i, [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i,
                                       _i, _vp, _vp]),
    "lwm_blockffn_workspace_size": (_sz, [_i, _i]),
    "lwm_blockffn_fwd": (_i, [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp,
                              _vp, _sz, _vp]),
    "lwm_blockffn_bwd_workspace_size": (_sz, [_i, _i]),
    "lwm_blockffn_bwd": (_i, [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i,
                              _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
}


class LwmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def lib() -> ctypes.CDLL:
    """Load the shared library once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing; build it with "
                "`python -m long_context_blockwise_causal_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in _SIGS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def exported_symbols():
    return list(_SIGS)


def status_string(status: int) -> str:
    return lib().lwm_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != OK:
        raise LwmError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code_of(dtype) -> int:
    if dtype == torch.bfloat16:
        return DTYPE_BF16
    if dtype == torch.float32:
        return DTYPE_FP32
    raise TypeError(f"unsupported dtype {dtype}")


def _dtype_code(t: torch.Tensor) -> int:
    return _dtype_code_of(t.dtype)


def _qk_code(qk_precision) -> int:
    if qk_precision in (QK_BF16, "bf16"):
        return QK_BF16
    if qk_precision in (QK_BF16X3, "bf16x3"):
        return QK_BF16X3
    raise ValueError(f"qk_precision {qk_precision!r}")


def _layout_code(rope_layout) -> int:
    if rope_layout in (ROPE_INTERLEAVED, "interleaved"):
        return ROPE_INTERLEAVED
    if rope_layout in (ROPE_HALF, "half", "rotate_half"):
        return ROPE_HALF
    raise ValueError(f"rope_layout {rope_layout!r}")


def _expect(where, name, t, shape, dtype=None):
    """Shapes and dtypes are checked here, before any pointer reaches the
    library: the C calls take sizes from q (or x) and trust every other
    buffer to match them."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape) or (dtype is not None
                                          and t.dtype != dtype):
        raise LwmError(ERR_INVALID_ARG,
                       f"{where}: {name} is {tuple(t.shape)} {t.dtype}, "
                       f"expected {tuple(shape)}"
                       + ("" if dtype is None else f" {dtype}"))


def _expect_dims(where, name, t, dims):
    if t.dim() != dims:
        raise LwmError(ERR_INVALID_ARG,
                       f"{where}: {name} must have {dims} dimensions")


def _same_device(where, *ts):
    devs = {t.device for t in ts if t is not None}
    if len(devs) > 1:
        raise LwmError(ERR_INVALID_ARG, f"{where}: tensors on {sorted(map(str, devs))}")


def _check_attn(where, q, k, v, segment_ids, positions, lse=None,
                like_q=()):
    """q, k, v (and like_q) [B,N,H,D] of one dtype; ids and positions
    [B,N] int32; lse [B,H,N] fp32."""
    _expect_dims(where, "q", q, 4)
    B, N, H, _ = q.shape
    for name, t in (("k", k), ("v", v)) + tuple(like_q):
        _expect(where, name, t, q.shape, q.dtype)
    _expect(where, "segment_ids", segment_ids, (B, N), torch.int32)
    _expect(where, "positions", positions, (B, N), torch.int32)
    _expect(where, "lse", lse, (B, H, N), torch.float32)
    _same_device(where, q, k, v, segment_ids, positions, lse,
                 *(t for _, t in like_q))


def _need_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")


def fwd_workspace_size(B, N, H, max_pos, dtype=torch.bfloat16,
                       qk_precision="bf16", D=HEAD_DIM, block_q=BLOCK,
                       block_k=BLOCK) -> int:
    return int(lib().lwm_blockattn_fwd_workspace_size(
        B, N, H, D, block_q, block_k, max_pos, _dtype_code_of(dtype),
        _qk_code(qk_precision)))


def bwd_workspace_size(B, N, H, max_pos, dtype=torch.bfloat16,
                       qk_precision="bf16", D=HEAD_DIM, block_q=BLOCK,
                       block_k=BLOCK) -> int:
    return int(lib().lwm_blockattn_bwd_workspace_size(
        B, N, H, D, block_q, block_k, max_pos, _dtype_code_of(dtype),
        _qk_code(qk_precision)))


def _workspace(nbytes, device, workspace):
    if workspace is None:
        return torch.empty(max(nbytes, 1), dtype=torch.uint8, device=device)
    if workspace.numel() * workspace.element_size() < nbytes:
        raise LwmError(ERR_WORKSPACE, "workspace")
    return workspace


def fwd(q, k, v, segment_ids, positions, theta, max_pos=None,
        qk_precision="bf16", out=None, lse=None, workspace=None,
        stream=None, block_q=BLOCK, block_k=BLOCK, rope_layout="interleaved"):
    """Forward pass. Returns (out [B,N,H,D] in q's dtype, lse [B,H,N] fp32).
    ``rope_layout``: "interleaved" pairs (2k, 2k+1) or "half" (k, k+D/2),
    the rotate-half layout of Hugging Face Llama checkpoints."""
    _check_attn("fwd", q, k, v, segment_ids, positions, lse,
                like_q=(("out", out),))
    _need_cuda(q, k, v, segment_ids, positions, out, lse, workspace)
    B, N, H, D = q.shape
    if max_pos is None:
        max_pos = int(positions.max().item()) + 1 if positions.numel() else 1
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    ws = _workspace(fwd_workspace_size(B, N, H, max_pos, q.dtype,
                                       qk_precision, D, block_q, block_k),
                    q.device, workspace)
    st = lib().lwm_blockattn_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(segment_ids), _ptr(positions),
        float(theta), block_q, block_k, int(max_pos), B, N, H, D,
        _dtype_code(q), _qk_code(qk_precision), _layout_code(rope_layout),
        _ptr(out), _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lwm_blockattn_fwd")
    return out, lse


def fwd_noalloc(q, k, v, segment_ids, positions, theta, max_pos,
                qk_precision="bf16", out=None, lse=None, stream=None,
                block_q=BLOCK, block_k=BLOCK, rope_layout="interleaved"):
    """Forward through lwm_blockattn_fwd_noalloc: the library's own fixed
    scratch array replaces the workspace (see the header for its limits).
    ``out``/``lse`` are allocated here only if the caller passes none."""
    _check_attn("fwd_noalloc", q, k, v, segment_ids, positions, lse,
                like_q=(("out", out),))
    _need_cuda(q, k, v, segment_ids, positions, out, lse)
    B, N, H, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    # the library uses the scratch array of the current device: make it the
    # tensors' device (and take that device's stream by default)
    with torch.cuda.device(q.device):
        st = lib().lwm_blockattn_fwd_noalloc(
            _ptr(q), _ptr(k), _ptr(v), _ptr(segment_ids), _ptr(positions),
            float(theta), block_q, block_k, int(max_pos), B, N, H, D,
            _dtype_code(q), _qk_code(qk_precision),
            _layout_code(rope_layout), _ptr(out), _ptr(lse),
            _stream(stream))
    _check(st, "lwm_blockattn_fwd_noalloc")
    return out, lse


def bwd(q, k, v, out, dout, lse, segment_ids, positions, theta,
        max_pos=None, qk_precision="bf16", dq=None, dk=None, dv=None,
        workspace=None, stream=None, block_q=BLOCK, block_k=BLOCK,
        rope_layout="interleaved"):
    """Backward pass. Returns (dq, dk, dv) in q's dtype (dq, dk in the
    layout q and k came in)."""
    _check_attn("bwd", q, k, v, segment_ids, positions, lse,
                like_q=(("out", out), ("dout", dout), ("dq", dq), ("dk", dk),
                        ("dv", dv)))
    _need_cuda(q, k, v, out, dout, lse, segment_ids, positions, dq, dk, dv,
               workspace)
    B, N, H, D = q.shape
    if max_pos is None:
        max_pos = int(positions.max().item()) + 1 if positions.numel() else 1
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    ws = _workspace(bwd_workspace_size(B, N, H, max_pos, q.dtype,
                                       qk_precision, D, block_q, block_k),
                    q.device, workspace)
    st = lib().lwm_blockattn_bwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(dout), _ptr(lse),
        _ptr(segment_ids), _ptr(positions), float(theta), block_q, block_k,
        int(max_pos), B, N, H, D, _dtype_code(q), _qk_code(qk_precision),
        _layout_code(rope_layout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
        ws.numel(), _stream(stream))
    _check(st, "lwm_blockattn_bwd")
    return dq, dk, dv


def fwd_block_workspace_size(B, Nq, Nk, H, max_pos, D=HEAD_DIM) -> int:
    return int(lib().lwm_blockattn_fwd_block_workspace_size(
        B, Nq, Nk, H, D, max_pos))


def fwd_block(q, k_rot, v, seg_q, pos_q, seg_k, q_off, k_off, theta,
              max_pos, out=None, lse=None, workspace=None, stream=None,
              rope_layout="interleaved", table=None):
    """Partial forward of query rows [q_off, q_off+Nq) against the rotated
    key / value rows [k_off, k_off+Nk) of the same packed sequence (one step
    of a ring). Returns (out [B,Nq,H,D] bf16, lse [B,H,Nq] fp32); rows that
    see no key get (0, -inf)."""
    _need_cuda(q, k_rot, v, seg_q, pos_q, seg_k, out, lse, workspace, table)
    B, Nq, H, D = q.shape
    Nk = k_rot.shape[1]
    if table is not None and table.shape[0] < max_pos:
        raise ValueError("rope table shorter than max_pos")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    ws = _workspace(fwd_block_workspace_size(B, Nq, Nk, H, max_pos, D),
                    q.device, workspace)
    st = lib().lwm_blockattn_fwd_block(
        _ptr(q), _ptr(k_rot), _ptr(v), _ptr(seg_q), _ptr(pos_q), _ptr(seg_k),
        int(q_off), int(k_off), float(theta), int(max_pos), _ptr(table), B,
        Nq, Nk, H, D, _layout_code(rope_layout), _ptr(out), _ptr(lse),
        _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lwm_blockattn_fwd_block")
    return out, lse


def merge(out, lse, out_part, lse_part, stream=None):
    """In place: fold the partial (out_part, lse_part) over another key set
    into (out, lse) with the log-sum-exp rule. Returns (out, lse)."""
    _need_cuda(out, lse, out_part, lse_part)
    B, N, H, D = out.shape
    st = lib().lwm_blockattn_merge(_ptr(out), _ptr(lse), _ptr(out_part),
                                   _ptr(lse_part), B, N, H, D,
                                   _dtype_code(out), _stream(stream))
    _check(st, "lwm_blockattn_merge")
    return out, lse


def bwd_delta(out, dout, delta=None, stream=None):
    """D = rowsum(dout * out) as fp32 [B,H,N]."""
    _need_cuda(out, dout, delta)
    B, N, H, D = out.shape
    if delta is None:
        delta = torch.empty((B, H, N), dtype=torch.float32, device=out.device)
    st = lib().lwm_blockattn_bwd_delta(_ptr(out), _ptr(dout), B, N, H, D,
                                       _dtype_code(out), _ptr(delta),
                                       _stream(stream))
    _check(st, "lwm_blockattn_bwd_delta")
    return delta


def bwd_block_workspace_size(B, Nq, Nk, H, D=HEAD_DIM) -> int:
    return int(lib().lwm_blockattn_bwd_block_workspace_size(B, Nq, Nk, H, D))


def bwd_block(q_rot, k_rot, v, dout, lse, delta, seg_q, seg_k, q_off, k_off,
              dq_acc, dk_acc, dv_acc, workspace=None, stream=None):
    """Partial backward of a query chunk against a key chunk: adds into the
    fp32 accumulators dq_acc [B,Nq,H,D], dk_acc and dv_acc [B,Nk,H,D]
    (rotated frame, no 1/sqrt(D); finish them with grad_finish)."""
    _need_cuda(q_rot, k_rot, v, dout, lse, delta, seg_q, seg_k, dq_acc,
               dk_acc, dv_acc, workspace)
    B, Nq, H, D = q_rot.shape
    Nk = k_rot.shape[1]
    ws = _workspace(bwd_block_workspace_size(B, Nq, Nk, H, D), q_rot.device,
                    workspace)
    st = lib().lwm_blockattn_bwd_block(
        _ptr(q_rot), _ptr(k_rot), _ptr(v), _ptr(dout), _ptr(lse),
        _ptr(delta), _ptr(seg_q), _ptr(seg_k), int(q_off), int(k_off), B, Nq,
        Nk, H, D, _ptr(dq_acc), _ptr(dk_acc), _ptr(dv_acc), _ptr(ws),
        ws.numel(), _stream(stream))
    _check(st, "lwm_blockattn_bwd_block")
    return dq_acc, dk_acc, dv_acc


def grad_finish(acc, positions=None, table=None, out=None, stream=None,
                rope_layout="interleaved"):
    """bf16 gradient from an fp32 accumulator: R(-pos) acc / sqrt(D) when
    positions are given (dq, dk), else acc (dv)."""
    _need_cuda(acc, positions, table, out)
    B, N, H, D = acc.shape
    if out is None:
        out = torch.empty(acc.shape, dtype=torch.bfloat16, device=acc.device)
    st = lib().lwm_blockattn_grad_finish(
        _ptr(acc), _ptr(positions), _ptr(table),
        0 if table is None else table.shape[0], B, N, H, D, DTYPE_BF16,
        _layout_code(rope_layout), _ptr(out), _stream(stream))
    _check(st, "lwm_blockattn_grad_finish")
    return out


def _check_ffn(where, x, w_gate, w_up, w_down, like_x=(), grads=()):
    """x (and like_x) [T, Dm]; Wg, Wu [F, Dm] and Wd [Dm, F] of x's dtype;
    grads: (name, tensor, shape) in fp32."""
    _expect_dims(where, "x", x, 2)
    _expect_dims(where, "w_gate", w_gate, 2)
    T, Dm = x.shape
    F = w_gate.shape[0]
    _expect(where, "w_gate", w_gate, (F, Dm), x.dtype)
    _expect(where, "w_up", w_up, (F, Dm), x.dtype)
    _expect(where, "w_down", w_down, (Dm, F), x.dtype)
    for name, t in like_x:
        _expect(where, name, t, (T, Dm), x.dtype)
    for name, t, shape in grads:
        _expect(where, name, t, shape, torch.float32)
    _same_device(where, x, w_gate, w_up, w_down, *(t for _, t in like_x),
                 *(t for _, t, _ in grads))


def ffn_workspace_size(chunk, F) -> int:
    return int(lib().lwm_blockffn_workspace_size(chunk, F))


def ffn_fwd(x, w_gate, w_up, w_down, chunk=8192, y=None, workspace=None,
            stream=None):
    """Blockwise SwiGLU MLP: y = (silu(x Wg^T) * (x Wu^T)) Wd^T, `chunk`
    tokens at a time. x [T, Dm]; Wg, Wu [F, Dm]; Wd [Dm, F]; bf16."""
    _check_ffn("ffn_fwd", x, w_gate, w_up, w_down, like_x=(("y", y),))
    _need_cuda(x, w_gate, w_up, w_down, y, workspace)
    T, Dm = x.shape
    F = w_gate.shape[0]
    y = torch.empty_like(x) if y is None else y
    c = max(1, min(int(chunk), T))
    ws = _workspace(ffn_workspace_size(c, F), x.device, workspace)
    st = lib().lwm_blockffn_fwd(
        _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down), T, Dm, F, int(chunk),
        _dtype_code(x), _ptr(y), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lwm_blockffn_fwd")
    return y


def ffn_bwd_workspace_size(chunk, F) -> int:
    return int(lib().lwm_blockffn_bwd_workspace_size(chunk, F))


def ffn_bwd(x, w_gate, w_up, w_down, dy, chunk=8192, dx=None, dw_gate=None,
            dw_up=None, dw_down=None, workspace=None, stream=None):
    """Backward of ffn_fwd: returns (dx bf16 [T, Dm], dWg, dWu fp32 [F, Dm],
    dWd fp32 [Dm, F]); h and g are recomputed chunk by chunk."""
    if x.dim() == 2 and w_gate.dim() == 2:
        Fg, Dmx = w_gate.shape[0], x.shape[1]
        _check_ffn("ffn_bwd", x, w_gate, w_up, w_down,
                   like_x=(("dy", dy), ("dx", dx)),
                   grads=(("dw_gate", dw_gate, (Fg, Dmx)),
                          ("dw_up", dw_up, (Fg, Dmx)),
                          ("dw_down", dw_down, (Dmx, Fg))))
    else:
        _check_ffn("ffn_bwd", x, w_gate, w_up, w_down)
    _need_cuda(x, w_gate, w_up, w_down, dy, dx, dw_gate, dw_up, dw_down,
               workspace)
    T, Dm = x.shape
    F = w_gate.shape[0]
    dev = x.device
    dx = torch.empty_like(x) if dx is None else dx
    f32 = dict(dtype=torch.float32, device=dev)
    dw_gate = torch.empty((F, Dm), **f32) if dw_gate is None else dw_gate
    dw_up = torch.empty((F, Dm), **f32) if dw_up is None else dw_up
    dw_down = torch.empty((Dm, F), **f32) if dw_down is None else dw_down
    c = max(1, min(int(chunk), T))
    ws = _workspace(ffn_bwd_workspace_size(c, F), dev, workspace)
    st = lib().lwm_blockffn_bwd(
        _ptr(x), _ptr(w_gate), _ptr(w_up), _ptr(w_down), _ptr(dy), T, Dm, F,
        int(chunk), _dtype_code(x), _ptr(dx), _ptr(dw_gate), _ptr(dw_up),
        _ptr(dw_down), _ptr(ws), ws.numel(), _stream(stream))
    _check(st, "lwm_blockffn_bwd")
    return dx, dw_gate, dw_up, dw_down


def classify(segment_ids, block_q=BLOCK, block_k=BLOCK, with_class=True,
             stream=None):
    """Returns kv_lo, kv_hi [B,Tq] int32 and tile_class [B,Tq,Tk] uint8."""
    _need_cuda(segment_ids)
    B, N = segment_ids.shape
    tq = -(-N // block_q)
    tk = -(-N // block_k)
    dev = segment_ids.device
    lo = torch.empty((B, tq), dtype=torch.int32, device=dev)
    hi = torch.empty((B, tq), dtype=torch.int32, device=dev)
    cls = torch.empty((B, tq, tk), dtype=torch.uint8, device=dev) \
        if with_class else None
    st = lib().lwm_blockattn_classify(_ptr(segment_ids), B, N, block_q,
                                      block_k, _ptr(lo), _ptr(hi), _ptr(cls),
                                      _stream(stream))
    _check(st, "lwm_blockattn_classify")
    return lo, hi, cls


VISIBILITY_QUERY_VIEW = ("row_lo", "row_hi", "kv_lo", "kv_hi", "lo_max",
                         "hi_min")
VISIBILITY_KEY_VIEW = ("col_lo", "col_hi", "q_lo", "q_hi", "klo_max",
                       "khi_min")


def visibility(seg_q, seg_k=None, q_off=0, k_off=0, query_view=True,
               key_view=True, block_q=BLOCK, block_k=BLOCK, stream=None):
    """The metadata the attention kernels classify tiles with (see
    lwm_blockattn_visibility). seg_q [B,Nq] int32 ids of queries
    [q_off, q_off+Nq); seg_k [B,Nk] of keys [k_off, k_off+Nk) (default:
    seg_q, self-attention). Returns a dict of int32 tensors: per query row
    and per query block (query view), per key and per key block (key
    view)."""
    seg_k = seg_q if seg_k is None else seg_k
    _need_cuda(seg_q, seg_k)
    _expect_dims("visibility", "seg_q", seg_q, 2)
    _expect_dims("visibility", "seg_k", seg_k, 2)
    B, Nq = seg_q.shape
    Nk = seg_k.shape[1]
    _expect("visibility", "seg_q", seg_q, (B, Nq), torch.int32)
    _expect("visibility", "seg_k", seg_k, (B, Nk), torch.int32)
    _same_device("visibility", seg_q, seg_k)
    dev = seg_q.device
    tq, tk = -(-Nq // block_q), -(-Nk // block_k)
    shapes = dict(zip(VISIBILITY_QUERY_VIEW,
                      [(B, Nq)] * 2 + [(B, tq)] * 4))
    shapes.update(zip(VISIBILITY_KEY_VIEW, [(B, Nk)] * 2 + [(B, tk)] * 4))
    want = (VISIBILITY_QUERY_VIEW if query_view else ()) + \
        (VISIBILITY_KEY_VIEW if key_view else ())
    res = {n: torch.empty(shapes[n], dtype=torch.int32, device=dev)
           for n in want}
    ptrs = [_ptr(res.get(n)) for n in VISIBILITY_QUERY_VIEW +
            VISIBILITY_KEY_VIEW]
    st = lib().lwm_blockattn_visibility(_ptr(seg_q), _ptr(seg_k), B, Nq, Nk,
                                        int(q_off), int(k_off), block_q,
                                        block_k, *ptrs, _stream(stream))
    _check(st, "lwm_blockattn_visibility")
    return res


def rope_table(theta, max_pos, D=HEAD_DIM, device="cuda", stream=None):
    """The fp32 (cos, sin) table [max_pos, D/2, 2] the kernels use."""
    t = torch.empty((max_pos, D // 2, 2), dtype=torch.float32, device=device)
    st = lib().lwm_blockattn_rope_table(float(theta), D, max_pos, _ptr(t),
                                        _stream(stream))
    _check(st, "lwm_blockattn_rope_table")
    return t


def rope_apply(x, positions, table, stream=None, out=None,
               rope_layout="interleaved"):
    """R(pos) x (bf16 [B,N,H,D]) with a table from rope_table(), pairs as
    ``rope_layout`` says (the output keeps that layout)."""
    _need_cuda(x, positions, table, out)
    B, N, H, D = x.shape
    out = torch.empty_like(x) if out is None else out
    st = lib().lwm_blockattn_rope_apply(
        _ptr(x), _ptr(positions), _ptr(table), table.shape[0], B, N, H, D,
        _dtype_code(x), _layout_code(rope_layout), _ptr(out), _stream(stream))
    _check(st, "lwm_blockattn_rope_apply")
    return out


def decode_workspace_size(B, H, L, D=HEAD_DIM) -> int:
    return int(lib().lwm_blockattn_decode_workspace_size(B, H, D, L))


def decode(q, k_rot, v, kv_start, kv_len, q_pos, table, out=None, lse=None,
           workspace=None, stream=None, rope_layout="interleaved"):
    """One query token per (b, h) [B,H,D] against a cache of rotated keys
    and values [B,L,H,D]; returns (out [B,H,D], lse [B,H])."""
    _expect_dims("decode", "q", q, 3)
    _expect_dims("decode", "k_rot", k_rot, 4)
    _expect_dims("decode", "table", table, 3)
    Bq, Hq, Dq = q.shape
    kshape = (Bq, k_rot.shape[1], Hq, Dq)
    _expect("decode", "k_rot", k_rot, kshape, q.dtype)
    _expect("decode", "v", v, kshape, q.dtype)
    for name, t in (("kv_start", kv_start), ("kv_len", kv_len),
                    ("q_pos", q_pos)):
        _expect("decode", name, t, (Bq,), torch.int32)
    _expect("decode", "table", table, (table.shape[0], Dq // 2, 2),
            torch.float32)
    _expect("decode", "out", out, q.shape, q.dtype)
    _expect("decode", "lse", lse, (Bq, Hq), torch.float32)
    _same_device("decode", q, k_rot, v, kv_start, kv_len, q_pos, table, out,
                 lse)
    _need_cuda(q, k_rot, v, kv_start, kv_len, q_pos, table, out, lse,
               workspace)
    B, H, D = q.shape
    L = k_rot.shape[1]
    out = torch.empty_like(q) if out is None else out
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    ws = _workspace(decode_workspace_size(B, H, L, D), q.device, workspace)
    st = lib().lwm_blockattn_decode(
        _ptr(q), _ptr(k_rot), _ptr(v), _ptr(kv_start), _ptr(kv_len),
        _ptr(q_pos), _ptr(table), table.shape[0], B, L, H, D, _dtype_code(q),
        _layout_code(rope_layout), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
        _stream(stream))
    _check(st, "lwm_blockattn_decode")
    return out, lse


def check_inputs(segment_ids, positions, max_pos, stream=None):
    """(ok, 1 + largest position). Synchronous."""
    _need_cuda(segment_ids, positions)
    B, N = segment_ids.shape
    mp = ctypes.c_int(0)
    st = lib().lwm_blockattn_check_inputs(_ptr(segment_ids), _ptr(positions),
                                          B, N, int(max_pos),
                                          ctypes.byref(mp), _stream(stream))
    if st not in (OK, ERR_PRECONDITION):
        _check(st, "lwm_blockattn_check_inputs")
    return st == OK, mp.value


def kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(lib().lwm_blockattn_kernel_launches())


def selftest_wait_timeout(limit_ns=20_000_000, stream=None):
    """Launch the bounded-wait self-test kernel (see the header)."""
    _check(lib().lwm_blockattn_selftest_wait_timeout(int(limit_ns),
                                                     _stream(stream)),
           "lwm_blockattn_selftest_wait_timeout")


def last_status(stream=None) -> int:
    return int(lib().lwm_blockattn_last_status(_stream(stream)))
