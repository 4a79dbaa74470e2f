"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point the header declares, sizes workspaces, and rejects bad
arguments with status codes before touching the device."""

import ctypes
import os
import re

import pytest
import torch

from long_context_blockwise_causal_b200 import ops

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            txt = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"LWM_API\s+[\w\s\*]+?\b(lwm_\w+)\s*\(", txt)
    return names


def test_header_declares_the_bound_entry_points():
    declared = set(header_functions())
    assert declared, "no LWM_API declarations found"
    assert declared == set(ops.exported_symbols())


def test_library_exports_every_declared_symbol():
    L = ops.lib()
    for name in header_functions():
        assert hasattr(L, name), name
    assert L.lwm_blockattn_version() == 1


def test_status_strings():
    assert ops.status_string(ops.OK) == "ok"
    assert "workspace" in ops.status_string(ops.ERR_WORKSPACE)
    assert ops.status_string(99) == "unknown status"


def test_workspace_sizes_grow_with_inputs():
    a = ops.fwd_workspace_size(1, 2048, 4, 2048)
    b = ops.fwd_workspace_size(1, 65536, 4, 2048)
    c = ops.fwd_workspace_size(1, 2048, 4, 4096)
    assert 0 < a < b and a < c
    # table dominates: max_pos * D floats
    assert c - a >= (4096 - 2048) * 128 * 4
    bw = ops.bwd_workspace_size(1, 2048, 4, 2048)
    assert bw >= a + 2048 * 4 * 128 * 4  # + fp32 dq accumulator
    # split-QK mode keeps the bf16 residual of the rotated keys
    x3 = ops.fwd_workspace_size(1, 2048, 4, 2048, qk_precision="bf16x3")
    assert x3 >= a + 2048 * 4 * 128 * 2
    # fp32 I/O needs no rotated-key scratch
    f32 = ops.fwd_workspace_size(1, 2048, 4, 2048, dtype=torch.float32)
    assert f32 <= a - 2048 * 4 * 128 * 2
    assert ops.fwd_workspace_size(-1, 2048, 4, 2048) == 0
    assert ops.bwd_workspace_size(1, -5, 4, 2048) == 0


def _fwd_raw(**kw):
    args = dict(q=1 << 20, k=1 << 20, v=1 << 20, seg=1 << 20, pos=1 << 20,
                theta=1e4, bq=128, bk=128, max_pos=16, B=1, N=16, H=1, D=128,
                dtype=0, qkp=0, layout=0, out=1 << 20, lse=1 << 20, ws=1 << 20,
                wsb=1 << 40, stream=None)
    args.update(kw)
    v = lambda x: None if x is None else ctypes.c_void_p(x)
    return ops.lib().lwm_blockattn_fwd(
        v(args["q"]), v(args["k"]), v(args["v"]), v(args["seg"]),
        v(args["pos"]), args["theta"], args["bq"], args["bk"],
        args["max_pos"], args["B"], args["N"], args["H"], args["D"],
        args["dtype"], args["qkp"], args["layout"], v(args["out"]),
        v(args["lse"]),
        v(args["ws"]), args["wsb"], v(args["stream"]))


@pytest.mark.parametrize("kw,status", [
    ({"q": None}, ops.ERR_INVALID_ARG),
    ({"lse": None}, ops.ERR_INVALID_ARG),
    ({"ws": None}, ops.ERR_INVALID_ARG),
    ({"k": (1 << 20) + 2}, ops.ERR_INVALID_ARG),     # misaligned
    ({"theta": -1.0}, ops.ERR_INVALID_ARG),
    ({"theta": float("nan")}, ops.ERR_INVALID_ARG),
    ({"dtype": 7}, ops.ERR_INVALID_ARG),
    ({"qkp": 5}, ops.ERR_INVALID_ARG),
    ({"layout": 2}, ops.ERR_INVALID_ARG),
    ({"N": -1}, ops.ERR_INVALID_ARG),
    ({"max_pos": 0}, ops.ERR_INVALID_ARG),
    ({"D": 64}, ops.ERR_UNSUPPORTED),
    ({"bq": 64}, ops.ERR_UNSUPPORTED),
    ({"bk": 32}, ops.ERR_UNSUPPORTED),
    ({"bk": 256}, ops.ERR_UNSUPPORTED),
    ({"wsb": 100}, ops.ERR_WORKSPACE),
    ({"N": 0, "q": None}, ops.OK),                    # empty: no work
    ({"H": 0}, ops.OK),
    ({"B": 0}, ops.OK),
])
def test_fwd_rejects_bad_arguments_before_launch(kw, status):
    assert _fwd_raw(**kw) == status


def test_visibility_rejects_bad_arguments_before_launch():
    L = ops.lib()
    p = ctypes.c_void_p(1 << 20)
    six = [p] * 6
    none6 = [None] * 6

    def call(*views, B=1, Nq=16, Nk=16, q_off=0, k_off=0, bq=128, bk=128,
             seg=p):
        ptrs = [x for view in views for x in view]
        return L.lwm_blockattn_visibility(seg, seg, B, Nq, Nk, q_off, k_off,
                                          bq, bk, *ptrs, None)

    # a view given in part is refused (it would leave the rest unwritten)
    assert call([p, None] + [p] * 4, none6) == ops.ERR_INVALID_ARG
    assert call(none6, [p] * 5 + [None]) == ops.ERR_INVALID_ARG
    assert call(six, six, bk=32) == ops.ERR_UNSUPPORTED
    # 64-key blocks: the forward's query view only
    assert call(six, six, bk=64) == ops.ERR_UNSUPPORTED
    assert call(six, six, q_off=-1) == ops.ERR_INVALID_ARG
    assert call(six, six, Nk=-3) == ops.ERR_INVALID_ARG
    assert call(six, six, seg=None) == ops.ERR_INVALID_ARG
    # nothing to do: no launch, no pointer touched
    assert call(none6, none6) == ops.OK
    assert call(six, six, Nq=0) == ops.OK
    assert call(six, six, B=0) == ops.OK


def test_noalloc_checks_arguments_before_its_scratch_size():
    # an invalid or unsupported call too large for the fixed scratch must
    # report what is wrong with it, not the scratch size (no CUDA call is
    # made on any of these paths)
    L = ops.lib()
    p = ctypes.c_void_p(1 << 20)

    def call(N=262144, H=32, D=128, dtype=0, qkp=0, layout=0, bk=128,
             theta=5e7, q=p):
        return L.lwm_blockattn_fwd_noalloc(q, p, p, p, p, theta, 128, bk,
                                           N, 1, N, H, D, dtype, qkp, layout,
                                           p, p, None)

    assert call() == ops.ERR_WORKSPACE              # valid, too large
    assert call(bk=64) == ops.ERR_WORKSPACE         # 64-key blocks: valid
    assert call(D=64) == ops.ERR_UNSUPPORTED
    assert call(bk=32) == ops.ERR_UNSUPPORTED
    assert call(dtype=9) == ops.ERR_INVALID_ARG
    assert call(qkp=4) == ops.ERR_INVALID_ARG
    assert call(layout=3) == ops.ERR_INVALID_ARG
    assert call(theta=0.0) == ops.ERR_INVALID_ARG
    assert call(q=None) == ops.ERR_INVALID_ARG
    assert call(q=ctypes.c_void_p((1 << 20) + 4)) == ops.ERR_INVALID_ARG
    assert call(H=0) == ops.OK                      # nothing to do


def test_bwd_and_classify_reject_bad_arguments():
    L = ops.lib()
    v = ctypes.c_void_p
    p = v(1 << 20)
    st = L.lwm_blockattn_bwd(p, p, p, p, p, p, p, p, 1e4, 128, 128, 16, 1, 16,
                             1, 128, 0, 0, 0, p, p, None, p, 1 << 40, None)
    assert st == ops.ERR_INVALID_ARG  # dv is NULL
    st = L.lwm_blockattn_bwd(p, p, p, p, p, p, p, p, 1e4, 128, 128, 16, 1, 16,
                             1, 128, 0, 0, 0, p, p, p, p, 10, None)
    assert st == ops.ERR_WORKSPACE
    st = L.lwm_blockattn_bwd(p, p, p, p, p, p, p, p, 1e4, 128, 128, 16, 1, 16,
                             1, 128, 0, 0, 3, p, p, p, p, 1 << 40, None)
    assert st == ops.ERR_INVALID_ARG  # unknown RoPE layout
    assert L.lwm_blockattn_classify(p, 1, 16, 128, 48, p, p, None,
                                    None) == ops.ERR_UNSUPPORTED
    assert L.lwm_blockattn_classify(None, 1, 16, 128, 128, p, p, None,
                                    None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_classify(None, 0, 16, 128, 128, None, None, None,
                                    None) == ops.OK
    assert L.lwm_blockattn_rope_table(0.0, 128, 10, p, None) == \
        ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_rope_table(1e4, 127, 10, p, None) == \
        ops.ERR_INVALID_ARG


def test_ring_and_layout_entry_points_reject_bad_arguments():
    L = ops.lib()
    v = ctypes.c_void_p
    p = v(1 << 20)
    big = 1 << 40
    # fwd_block: null q, unknown layout, misaligned seg_k
    assert L.lwm_blockattn_fwd_block(None, p, p, p, p, p, 0, 0, 1e4, 16, None, 1,
                                     16, 16, 1, 128, 0, p, p, p, big,
                                     None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_fwd_block(p, p, p, p, p, p, 0, 0, 1e4, 16, None, 1, 16,
                                     16, 1, 128, 9, p, p, p, big,
                                     None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_fwd_block(p, p, p, p, p, v((1 << 20) + 4), 0, 0,
                                     1e4, 16, None, 1, 16, 16, 1, 128, 0, p,
                                     p, p, big, None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_fwd_block(p, p, p, p, p, p, -1, 0, 1e4, 16, None, 1,
                                     16, 16, 1, 128, 0, p, p, p, big,
                                     None) == ops.ERR_INVALID_ARG
    # bwd_block: null accumulator; D != 128
    assert L.lwm_blockattn_bwd_block(p, p, p, p, p, p, p, p, 0, 0, 1, 16, 16,
                                     1, 128, p, None, p, p, big,
                                     None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_bwd_block(p, p, p, p, p, p, p, p, 0, 0, 1, 16, 16,
                                     1, 64, p, p, p, p, big,
                                     None) == ops.ERR_UNSUPPORTED
    # merge / bwd_delta: fp32 I/O is not offered
    assert L.lwm_blockattn_merge(p, p, p, p, 1, 16, 1, 128, 1,
                                 None) == ops.ERR_UNSUPPORTED
    assert L.lwm_blockattn_bwd_delta(p, p, 1, 16, 1, 128, 1, p,
                                     None) == ops.ERR_UNSUPPORTED
    # grad_finish: positions without a table
    assert L.lwm_blockattn_grad_finish(p, p, None, 16, 1, 16, 1, 128, 0, 0,
                                       p, None) == ops.ERR_INVALID_ARG
    # rope_apply and decode: unknown layout
    assert L.lwm_blockattn_rope_apply(p, p, p, 16, 1, 16, 1, 128, 0, 5, p,
                                      None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockattn_decode(p, p, p, p, p, p, p, 16, 1, 16, 1, 128, 0,
                                  5, p, p, p, big,
                                  None) == ops.ERR_INVALID_ARG
    # empty problems launch nothing and succeed
    assert L.lwm_blockattn_fwd_block(None, None, None, None, None, None, 0, 0,
                                     1e4, 16, None, 1, 0, 16, 1, 128, 0, None,
                                     None, None, 0, None) == ops.OK
    assert L.lwm_blockattn_bwd_block(None, None, None, None, None, None, None,
                                     None, 0, 0, 1, 16, 0, 1, 128, None, None,
                                     None, None, 0, None) == ops.OK


def test_ffn_entry_points_reject_bad_arguments_before_any_launch():
    L = ops.lib()
    v = ctypes.c_void_p
    p = v(1 << 20)
    big = 1 << 40
    T, Dm, F, c = 256, 128, 192, 128
    # forward: null input, unsupported width / dtype, small workspace
    assert L.lwm_blockffn_fwd(None, p, p, p, T, Dm, F, c, 0, p, p, big,
                              None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockffn_fwd(p, p, p, p, T, 100, F, c, 0, p, p, big,
                              None) == ops.ERR_UNSUPPORTED
    assert L.lwm_blockffn_fwd(p, p, p, p, T, Dm, F, c, 1, p, p, big,
                              None) == ops.ERR_UNSUPPORTED
    assert L.lwm_blockffn_fwd(p, p, p, p, T, Dm, F, 0, 0, p, p, big,
                              None) == ops.ERR_INVALID_ARG
    need = L.lwm_blockffn_workspace_size(c, F)
    assert need >= c * F * 2
    assert L.lwm_blockffn_fwd(p, p, p, p, T, Dm, F, c, 0, p, p, need - 1,
                              None) == ops.ERR_WORKSPACE
    assert L.lwm_blockffn_fwd(None, None, None, None, 0, Dm, F, c, 0, None,
                              None, 0, None) == ops.OK
    # backward: every check happens before the weight gradients are zeroed,
    # so these return their own code (a launch here, with no GPU, would
    # turn into LWM_ERR_CUDA)
    need_b = L.lwm_blockffn_bwd_workspace_size(c, F)
    assert need_b >= 4 * c * F * 2
    assert L.lwm_blockffn_bwd(p, p, p, p, p, T, Dm, F, c, 0, p, p, p, p, p,
                              need_b - 1, None) == ops.ERR_WORKSPACE
    assert L.lwm_blockffn_bwd(p, p, p, p, None, T, Dm, F, c, 0, p, p, p, p,
                              p, big, None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockffn_bwd(p, p, p, p, p, T, Dm, F, c, 0, None, p, p, p,
                              p, big, None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockffn_bwd(p, p, p, p, p, T, Dm, F, c, 0, p, None, p, p,
                              p, big, None) == ops.ERR_INVALID_ARG
    assert L.lwm_blockffn_bwd(p, p, p, p, p, T, Dm, 96, c, 0, p, p, p, p, p,
                              big, None) == ops.ERR_UNSUPPORTED


def _attn_cpu(B=1, N=8, H=2, D=128, dtype=torch.bfloat16):
    q = torch.zeros(B, N, H, D, dtype=dtype)
    seg = torch.zeros(B, N, dtype=torch.int32)
    pos = torch.arange(N, dtype=torch.int32)[None].repeat(B, 1)
    return q, q.clone(), q.clone(), seg, pos


def _invalid(fn, *a, **kw):
    with pytest.raises(ops.LwmError) as e:
        fn(*a, **kw)
    assert e.value.status == ops.ERR_INVALID_ARG
    return str(e.value)


def test_bindings_check_shapes_and_dtypes_before_the_library():
    """The C calls take their sizes from q (or x) and trust every other
    buffer; the bindings refuse mismatched tensors before any pointer is
    passed (on CPU tensors the shape check fires before the device one)."""
    q, k, v, seg, pos = _attn_cpu()
    assert "k is" in _invalid(ops.fwd, q, k[:, :4], v, seg, pos, 1e4)
    assert "v is" in _invalid(ops.fwd, q, k, v.float(), seg, pos, 1e4)
    _invalid(ops.fwd, q, k, v, seg.long(), pos, 1e4)
    _invalid(ops.fwd, q, k, v, seg, pos[:, :4], 1e4)
    _invalid(ops.fwd, q[0], k, v, seg, pos, 1e4)
    _invalid(ops.fwd, q, k, v, seg, pos, 1e4,
             lse=torch.zeros(1, 8, 2))                 # [B,N,H]: transposed
    _invalid(ops.fwd, q, k, v, seg, pos, 1e4, out=torch.zeros_like(q).float())
    _invalid(ops.fwd_noalloc, q, k, v, seg, pos, 1e4, 8, out=q[:, :2])
    lse = torch.zeros(1, 2, 8)
    _invalid(ops.bwd, q, k, v, q, q.float(), lse, seg, pos, 1e4)   # dout
    _invalid(ops.bwd, q, k, v, q, q, lse, seg, pos, 1e4, dk=q[:, :3])
    # consistent shapes: only the device check is left
    with pytest.raises(ValueError, match="CUDA"):
        ops.fwd(q, k, v, seg, pos, 1e4)
    with pytest.raises(ValueError, match="CUDA"):
        ops.bwd(q, k, v, q, q, lse, seg, pos, 1e4)

    T, Dm, F = 16, 64, 128
    x = torch.zeros(T, Dm, dtype=torch.bfloat16)
    wg = torch.zeros(F, Dm, dtype=torch.bfloat16)
    wd = torch.zeros(Dm, F, dtype=torch.bfloat16)
    _invalid(ops.ffn_fwd, x, wg, wg, wg)                 # w_down [F, Dm]
    _invalid(ops.ffn_fwd, x, wg, wg[:, :32], wd)
    _invalid(ops.ffn_fwd, x, wg, wg, wd, y=x[:8])
    _invalid(ops.ffn_bwd, x, wg, wg, wd, x[:8])          # dy
    _invalid(ops.ffn_bwd, x, wg, wg, wd, x, dw_gate=wg)  # bf16 gradient
    _invalid(ops.ffn_bwd, x, wg, wg, wd, x,
             dw_down=torch.zeros(F, Dm))                # transposed
    with pytest.raises(ValueError, match="CUDA"):
        ops.ffn_bwd(x, wg, wg, wd, x)

    B, L, H = 2, 64, 2
    qd = torch.zeros(B, H, 128, dtype=torch.bfloat16)
    kc = torch.zeros(B, L, H, 128, dtype=torch.bfloat16)
    i32 = torch.zeros(B, dtype=torch.int32)
    table = torch.zeros(L, 64, 2)
    _invalid(ops.decode, qd, kc, kc, i32, i32.long(), i32, table)
    _invalid(ops.decode, qd, kc, kc[:, :, :1], i32, i32, i32, table)
    _invalid(ops.decode, qd, kc, kc, i32, i32, i32, torch.zeros(L, 128))
    _invalid(ops.decode, qd, kc, kc, i32, i32, i32, table.double())
    _invalid(ops.decode, qd, kc, kc, i32, i32, i32, table,
             lse=torch.zeros(B, H, 1))
    with pytest.raises(ValueError, match="CUDA"):
        ops.decode(qd, kc, kc, i32, i32, i32, table)


def test_binding_checks_accept_the_workloads_tensors():
    from long_context_blockwise_causal_b200 import workloads as wl
    for name, w in wl.WORKLOADS.items():
        t = wl.make_inputs(w, 0, device="cpu", N=min(w.N, 512), with_dout=True)
        B, N, H, D = t["q"].shape
        lse = torch.empty(B, H, N)
        ops._check_attn("fwd", t["q"], t["k"], t["v"], t["segment_ids"],
                        t["positions"], lse,
                        like_q=(("out", torch.empty_like(t["q"])),
                                ("dout", t["dout"])))
    for name, w in wl.FFN_WORKLOADS.items():
        t = wl.make_ffn_inputs(256, w.Dm, w.F, 0, device="cpu")
        ops._check_ffn("ffn_bwd", t["x"], t["w_gate"], t["w_up"], t["w_down"],
                       like_x=(("dy", t["x"]), ("dx", t["x"])),
                       grads=(("dw_gate", torch.empty(w.F, w.Dm), (w.F, w.Dm)),
                              ("dw_down", torch.empty(w.Dm, w.F), (w.Dm, w.F))))


def test_plain_c_client_links_and_runs(tmp_path):
    """The boundary is a C ABI: a C99 program that includes only the header
    and links only the library builds with -Werror and runs (no Python, no
    torch; the calls it makes need no GPU)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    libdir = os.path.dirname(ops._LIB_PATH)
    exe = tmp_path / "c_abi_client"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror",
                    "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_client.c"),
                    "-o", str(exe), "-L", libdir, "-l:liblwm_blockattn.so",
                    f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True,
                       timeout=60)
    assert r.returncode == 0, r.stderr
    assert "c client ok" in r.stdout
