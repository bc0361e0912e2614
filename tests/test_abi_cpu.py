"""The C ABI without a GPU: the library loads, exports every entry point that
include/sva.h declares, and rejects bad arguments on the host before any CUDA
call."""
import ctypes
import os
import re

import pytest

import softmax_attention_video_gated_b200 as sva

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    src = open(os.path.join(ROOT, "include", "sva.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(sva_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_entry_point():
    lib = sva._lib()
    names = header_functions()
    assert len(names) >= 17
    for n in names:
        assert hasattr(lib, n), n
        assert n in sva.exported_symbols(), f"binding lacks {n}"
    assert sva.sva_version() == 1


def test_status_strings():
    for code in range(6):
        assert sva.status_string(code)
    assert "timed out" in sva.status_string(sva.SVA_ERR_DEVICE_TIMEOUT)


def _args(**kw):
    a = sva.AttnArgs()
    a.B, a.N, a.H, a.d, a.dtype = 1, 256, 2, 128, sva.SVA_BF16
    for f in ("q", "k", "v", "gate", "out"):
        setattr(a, f, 0x10000)
    a.ldq = a.ldk = a.ldv = a.ldg = a.ldo = 256
    a.eps = 1e-6
    for k, v in kw.items():
        setattr(a, k, v)
    return a


@pytest.mark.parametrize("bad, expect", [
    (dict(q=None), sva.SVA_ERR_INVALID_ARGUMENT),
    (dict(N=0), sva.SVA_ERR_INVALID_ARGUMENT),
    (dict(ldk=100), sva.SVA_ERR_INVALID_ARGUMENT),           # < D
    (dict(ldk=260), sva.SVA_ERR_INVALID_ARGUMENT),           # not 16-byte rows
    (dict(v=0x10002), sva.SVA_ERR_INVALID_ARGUMENT),         # misaligned
    (dict(d=64, ldq=128, ldk=128, ldv=128, ldg=128, ldo=128), sva.SVA_ERR_UNSUPPORTED),
    (dict(eps=-1.0), sva.SVA_ERR_INVALID_ARGUMENT),
    (dict(dtype=7), sva.SVA_ERR_INVALID_ARGUMENT),
    (dict(wgate=0x30000, ldw=1), sva.SVA_ERR_INVALID_ARGUMENT),  # write gate: ldw < H
    (dict(wgate=0x30001, ldw=8), sva.SVA_ERR_INVALID_ARGUMENT),  # not element-aligned
    (dict(n_keys=500), sva.SVA_ERR_INVALID_ARGUMENT),           # keys count: anchors only
])
def test_linear_attn_rejects_bad_arguments_on_host(bad, expect):
    a = _args(**bad)
    st = sva._lib().sva_linear_attn_fwd(ctypes.byref(a), 0x20000, 1 << 30, None)
    assert st == expect
    # the allocation-free entry point validates the same way
    assert sva._lib().sva_linear_attn_fwd_noalloc(ctypes.byref(a), None) == expect


def test_phase_and_key_count_host_validation():
    lib = sva._lib()
    st = 0x50000
    # the state phase needs k and v but not q, gate, out; the read-out the reverse
    a = _args(q=None, gate=None, out=None)
    assert lib.sva_linear_attn_state_fwd(ctypes.byref(a), None, 0x20000, 1 << 30,
                                         None) == sva.SVA_ERR_INVALID_ARGUMENT   # no state
    a = _args(k=None)
    assert lib.sva_linear_attn_state_fwd(ctypes.byref(a), st, 0x20000, 1 << 30,
                                         None) == sva.SVA_ERR_INVALID_ARGUMENT
    a = _args(out=None)
    assert lib.sva_linear_attn_readout_fwd(ctypes.byref(a), st, 0x20000, 1 << 30,
                                           None) == sva.SVA_ERR_INVALID_ARGUMENT
    a = _args(k=None, v=None)
    assert lib.sva_linear_attn_readout_fwd(ctypes.byref(a), st, 0x20000, 16,
                                           None) == sva.SVA_ERR_WORKSPACE    # k, v not needed
    assert lib.sva_linear_attn_state_bytes(1, 24, 128) == 24 * (128 * 128 + 128) * 4
    a = _args(n_keys=-1)
    assert lib.sva_softmax_anchor_fwd(ctypes.byref(a), 0x20000, 256,
                                      None) == sva.SVA_ERR_INVALID_ARGUMENT


def test_sizes_past_the_index_range_are_refused_on_host():
    # token counts and GEMM extents are indexed in 32 bits inside the kernels:
    # B*N, B*n_keys or an extent above 2^31 is refused before anything launches
    lib = sva._lib()
    a = _args(B=3, N=1 << 30)
    assert lib.sva_linear_attn_fwd(ctypes.byref(a), 0x20000, 1 << 62, None) == sva.SVA_ERR_UNSUPPORTED
    assert lib.sva_softmax_anchor_fwd(ctypes.byref(a), 0x20000, 1 << 62,
                                      None) == sva.SVA_ERR_UNSUPPORTED
    a = _args(B=3, N=1000, n_keys=1 << 30)
    assert lib.sva_softmax_anchor_fwd(ctypes.byref(a), 0x20000, 1 << 62,
                                      None) == sva.SVA_ERR_UNSUPPORTED
    assert lib.sva_projection_fwd(0x10000, 64, 0x20000, (1 << 31) + 1, 64, 64, 0x30000, 64, 0,
                                  sva.SVA_BF16, 0x40000, 256, None) == sva.SVA_ERR_UNSUPPORTED


def test_workspace_checks_happen_before_launch():
    a = _args()
    assert sva._lib().sva_linear_attn_fwd(ctypes.byref(a), None, 0, None) == sva.SVA_ERR_WORKSPACE
    assert sva._lib().sva_linear_attn_fwd(ctypes.byref(a), 0x20000, 16, None) == sva.SVA_ERR_WORKSPACE
    assert sva._lib().sva_softmax_anchor_fwd(ctypes.byref(a), 0x20000, 8, None) == sva.SVA_ERR_WORKSPACE
    assert sva._lib().sva_softmax_anchor_fwd(None, 0x20000, 256, None) == sva.SVA_ERR_INVALID_ARGUMENT


def test_projection_and_router_host_validation():
    lib = sva._lib()
    # K not a multiple of 16 bytes
    assert lib.sva_projection_fwd(0x10000, 100, 0x20000, 8, 64, 100, 0x30000, 64, 0,
                                  sva.SVA_BF16, 0x40000, 256, None) == sva.SVA_ERR_INVALID_ARGUMENT
    assert lib.sva_projection_fwd(0x10000, 64, 0x20000, 0, 64, 64, 0x30000, 64, 0,
                                  sva.SVA_BF16, 0x40000, 256, None) == sva.SVA_ERR_INVALID_ARGUMENT
    null = (ctypes.c_void_p * 1)(None)
    ok = (ctypes.c_void_p * 1)(0x50000)
    assert lib.sva_attnres_route(0x10000, null, ok, 1, 0x30000, None, 8, 64, sva.SVA_BF16,
                                 None) == sva.SVA_ERR_INVALID_ARGUMENT
    assert lib.sva_attnres_route(0x10000, ok, ok, 9, 0x30000, None, 8, 64, sva.SVA_BF16,
                                 None) == sva.SVA_ERR_INVALID_ARGUMENT


def test_stack_workspace_query_and_validation():
    lib = sva._lib()
    L = 24
    w = (ctypes.c_void_p * L)(*([0x100000] * L))
    d = sva.StackDesc()
    d.B, d.N, d.H, d.d, d.L, d.dtype = 1, 19320, 24, 128, L, sva.SVA_BF16
    d.softmax_period, d.attnres_block = 4, 8
    d.w_qkvg = ctypes.cast(w, ctypes.POINTER(ctypes.c_void_p))
    d.w_o = ctypes.cast(w, ctypes.POINTER(ctypes.c_void_p))
    d.w_r = 0x200000
    d.eps = 1e-6
    n = lib.sva_hybrid_stack_workspace_bytes(ctypes.byref(d))
    rows, D = 19320, 3072
    # fp32 stream + u + qkvg + y + 2 summaries + 2 keys + W_r^T, at least
    assert n >= rows * D * (4 + 2 + 8 + 2 + 4 * 2) + D * D * 2
    assert n < 4 * 2**30
    d.w_r = None        # routed layers exist, so W_r is required
    assert lib.sva_hybrid_stack_workspace_bytes(ctypes.byref(d)) == 0
    assert lib.sva_hybrid_stack_fwd(ctypes.byref(d), 0x10000, 0x20000, 0x30000, 1 << 40,
                                    None) == sva.SVA_ERR_INVALID_ARGUMENT
    d.attnres_block = 0  # AttnRes off: no router projection needed
    n0 = lib.sva_hybrid_stack_workspace_bytes(ctypes.byref(d))
    assert n0 > 0
    # write-gated linear layers: the fused projection output gains 24 columns; anchors' entries
    # may be NULL, linear layers' may not
    wg = (ctypes.c_void_p * L)(*[None if l % 4 == 3 else 0x300000 for l in range(L)])
    d.w_wg = ctypes.cast(wg, ctypes.POINTER(ctypes.c_void_p))
    n1 = lib.sva_hybrid_stack_workspace_bytes(ctypes.byref(d))
    assert rows * 24 * 2 <= n1 - n0 <= rows * 24 * 2 + 2048
    wg[0] = None
    assert lib.sva_hybrid_stack_workspace_bytes(ctypes.byref(d)) == 0
    d.w_wg = None


def test_stack_host_batches_host_validation():
    # all checks run before any stream, event or copy is made
    lib = sva._lib()
    L = 8
    w = (ctypes.c_void_p * L)(*([0x100000] * L))
    d = sva.StackDesc()
    d.B, d.N, d.H, d.d, d.L, d.dtype = 1, 1000, 2, 128, L, sva.SVA_BF16
    d.softmax_period, d.attnres_block = 4, 8
    d.w_qkvg = ctypes.cast(w, ctypes.POINTER(ctypes.c_void_p))
    d.w_o = ctypes.cast(w, ctypes.POINTER(ctypes.c_void_p))
    d.eps = 1e-6
    need = lib.sva_hybrid_stack_host_staging_bytes(ctypes.byref(d))
    assert need >= 4 * 1000 * 256 * 2 and need % 256 == 0
    ws = lib.sva_hybrid_stack_workspace_bytes(ctypes.byref(d))
    hx = (ctypes.c_void_p * 2)(0x1000, 0x2000)
    hy = (ctypes.c_void_p * 2)(0x3000, None)
    pp = lambda a: ctypes.cast(a, ctypes.POINTER(ctypes.c_void_p))  # noqa: E731
    call = lambda xs, ys, n, sb: lib.sva_hybrid_stack_fwd_host(  # noqa: E731
        ctypes.byref(d), xs, ys, n, 0x40000, ws, 0x80000, sb, None)
    assert call(pp(hx), pp(hy), -1, need) == sva.SVA_ERR_INVALID_ARGUMENT
    assert call(None, pp(hy), 1, need) == sva.SVA_ERR_INVALID_ARGUMENT
    assert call(pp(hx), pp(hy), 2, need) == sva.SVA_ERR_INVALID_ARGUMENT   # y_host[1] is NULL
    assert call(pp(hx), pp(hy), 1, need - 256) == sva.SVA_ERR_WORKSPACE
    assert lib.sva_hybrid_stack_fwd_host(ctypes.byref(d), pp(hx), pp(hy), 1, 0x40000, ws - 1024,
                                         0x80000, need, None) == sva.SVA_ERR_WORKSPACE
