"""Python binding of libsva.so, the sm_100a kernel library of the hybrid
linear/softmax token mixer (gated linear attention, gated softmax anchors,
Block Attention Residuals with a shared-query router).

Argument marshalling only: every function below forwards torch tensors to the
C entry point of the same name in include/sva.h as raw device pointers, sizes
and the current CUDA stream. All arithmetic runs in the library's kernels.
There is no fallback: if libsva.so is missing or a call fails, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsva.so")

SVA_OK, SVA_ERR_INVALID_ARGUMENT, SVA_ERR_UNSUPPORTED = 0, 1, 2
SVA_ERR_WORKSPACE, SVA_ERR_CUDA, SVA_ERR_DEVICE_TIMEOUT = 3, 4, 5
SVA_F32, SVA_BF16 = 0, 1
SVA_STATUS_BYTES = 256
SVA_FLAG_QK_FEATURES = 1
KERNEL_CLASSES = ("proj_qkvg", "proj_out", "linear_state", "linear_readout", "anchor", "route",
                  "keys", "other", "linear_reduce")

_c_void_p_p = ctypes.POINTER(ctypes.c_void_p)


class SvaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = f"{where}: {status_string(status)}"
        if status == SVA_ERR_CUDA:
            msg += f" ({_lib().sva_last_cuda_error().decode()})"
        super().__init__(msg)


class AttnArgs(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("q", ctypes.c_void_p), ("ldq", ctypes.c_int64),
        ("k", ctypes.c_void_p), ("ldk", ctypes.c_int64),
        ("v", ctypes.c_void_p), ("ldv", ctypes.c_int64),
        ("gate", ctypes.c_void_p), ("ldg", ctypes.c_int64),
        ("residual", ctypes.c_void_p), ("ldr", ctypes.c_int64),
        ("out", ctypes.c_void_p), ("ldo", ctypes.c_int64),
        ("eps", ctypes.c_float), ("scale", ctypes.c_float), ("flags", ctypes.c_uint),
        ("wgate", ctypes.c_void_p), ("ldw", ctypes.c_int64),
        ("n_keys", ctypes.c_int),
    ]


class StackDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
        ("L", ctypes.c_int), ("dtype", ctypes.c_int),
        ("softmax_period", ctypes.c_int), ("attnres_block", ctypes.c_int),
        ("all_softmax", ctypes.c_int),
        ("w_qkvg", _c_void_p_p), ("w_o", _c_void_p_p), ("w_r", ctypes.c_void_p),
        ("eps", ctypes.c_float),
        ("trace_o", _c_void_p_p), ("trace_y", _c_void_p_p), ("trace_alpha", _c_void_p_p),
        ("prof_events", _c_void_p_p), ("prof_capacity", ctypes.c_int),
        ("prof_kind", ctypes.POINTER(ctypes.c_int)), ("prof_count", ctypes.POINTER(ctypes.c_int)),
        ("w_wg", _c_void_p_p),
        ("launch_count", ctypes.POINTER(ctypes.c_int)),
    ]


_LIB = None

_SIGS = {
    "sva_linear_attn_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 4 + [ctypes.c_int]),
    "sva_linear_attn_fwd": (ctypes.c_int, [ctypes.POINTER(AttnArgs), ctypes.c_void_p,
                                           ctypes.c_size_t, ctypes.c_void_p]),
    "sva_linear_attn_fwd_noalloc": (ctypes.c_int, [ctypes.POINTER(AttnArgs), ctypes.c_void_p]),
    "sva_linear_attn_state_bytes": (ctypes.c_size_t, [ctypes.c_int] * 3),
    "sva_linear_attn_state_fwd": (ctypes.c_int, [ctypes.POINTER(AttnArgs), ctypes.c_void_p,
                                                 ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_void_p]),
    "sva_linear_attn_readout_fwd": (ctypes.c_int, [ctypes.POINTER(AttnArgs), ctypes.c_void_p,
                                                   ctypes.c_void_p, ctypes.c_size_t,
                                                   ctypes.c_void_p]),
    "sva_softmax_anchor_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int] * 5),
    "sva_softmax_anchor_fwd": (ctypes.c_int, [ctypes.POINTER(AttnArgs), ctypes.c_void_p,
                                              ctypes.c_size_t, ctypes.c_void_p]),
    "sva_projection_workspace_bytes": (ctypes.c_size_t, []),
    "sva_projection_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                          ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                          ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t,
                                          ctypes.c_void_p]),
    "sva_projection_residual_fwd": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                   ctypes.c_void_p, ctypes.c_int64,
                                                   ctypes.c_int64, ctypes.c_int64,
                                                   ctypes.c_void_p, ctypes.c_int64,
                                                   ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,
                                                   ctypes.c_void_p, ctypes.c_size_t,
                                                   ctypes.c_void_p]),
    "sva_attnres_keys_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int]),
    "sva_attnres_keys": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                        ctypes.c_int64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "sva_attnres_route": (ctypes.c_int, [ctypes.c_void_p, _c_void_p_p, _c_void_p_p, ctypes.c_int,
                                         ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_void_p]),
    "sva_hybrid_stack_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(StackDesc)]),
    "sva_hybrid_stack_fwd": (ctypes.c_int, [ctypes.POINTER(StackDesc), ctypes.c_void_p,
                                            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                            ctypes.c_void_p]),
    "sva_hybrid_stack_host_staging_bytes": (ctypes.c_size_t, [ctypes.POINTER(StackDesc)]),
    "sva_hybrid_stack_fwd_host": (ctypes.c_int, [ctypes.POINTER(StackDesc), _c_void_p_p,
                                                 _c_void_p_p, ctypes.c_int, ctypes.c_void_p,
                                                 ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t,
                                                 ctypes.c_void_p]),
    "sva_check_device_status": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p]),
    "sva_selftest_bounded_wait": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint,
                                                 ctypes.c_void_p]),
    "sva_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sva_last_cuda_error": (ctypes.c_char_p, []),
    "sva_version": (ctypes.c_int, []),
}


def _lib() -> ctypes.CDLL:
    """Load libsva.so (no fallback: a missing library is an error)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m softmax_attention_video_gated_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def exported_symbols() -> List[str]:
    return list(_SIGS)


def status_string(status: int) -> str:
    return _lib().sva_status_string(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != SVA_OK:
        raise SvaError(status, where)


# ---------------------------------------------------------------------------
# tensor marshalling
# ---------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return SVA_BF16
    if t.dtype == torch.float32:
        return SVA_F32
    raise TypeError(f"unsupported dtype {t.dtype}; use torch.bfloat16 or torch.float32")


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _rows(t, B: int, N: int):
    """Row stride of a [B, N, W] activation whose rows are ld elements apart and
    whose batches are N*ld elements apart (a column slice of a contiguous
    [B, N, ld] buffer is accepted)."""
    if t.dim() != 3 or t.shape[0] != B or t.shape[1] != N:
        raise ValueError(f"expected a [B={B}, N={N}, W] tensor, got {tuple(t.shape)}")
    if t.stride(2) != 1 or t.stride(0) != N * t.stride(1):
        raise ValueError("activation rows must be unit-stride with batches N*ld apart")
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    return t.stride(1)


def workspace(nbytes: int, device=None):
    torch = _torch()
    return torch.empty(max(int(nbytes), SVA_STATUS_BYTES), dtype=torch.uint8,
                       device=device if device is not None else "cuda")


def _attn_args(q, k, v, gate, out, H, residual, eps, scale, flags, wgate=None) -> AttnArgs:
    """Marshals an attention call. Operands a call does not use may be None (the
    linear-attention phases); k and v may hold more rows than q (the anchor over
    all keys for one shard's queries), which sets n_keys."""
    lead = q if q is not None else k
    B, N, D = lead.shape
    if D % H:
        raise ValueError(f"width {D} is not a multiple of H={H}")
    dt = _dtype_code(lead)
    for t in (q, k, v, gate, out, residual):
        if t is not None and _dtype_code(t) != dt:
            raise TypeError("q, k, v, gate, out and residual must share one dtype")
    a = AttnArgs()
    a.B, a.N, a.H, a.d, a.dtype = B, N, H, D // H, dt
    if q is not None:
        a.q, a.ldq = _ptr(q), _rows(q, B, N)
    if k is not None:
        Nk = k.shape[1]
        a.k, a.ldk = _ptr(k), _rows(k, B, Nk)
        a.v, a.ldv = _ptr(v), _rows(v, B, Nk)
        if Nk != N:
            a.n_keys = Nk
    if gate is not None:
        a.gate, a.ldg = _ptr(gate), _rows(gate, B, N)
    if out is not None:
        a.out, a.ldo = _ptr(out), _rows(out, B, N)
    if residual is not None:
        a.residual, a.ldr = _ptr(residual), _rows(residual, B, N)
    a.eps, a.scale, a.flags = float(eps), float(scale), int(flags)
    if wgate is not None:
        # [B, N, >=H] logits, one per token and head; rows ldw elements apart
        if _dtype_code(wgate) != dt:
            raise TypeError("wgate must have the dtype of q")
        if wgate.dim() != 3 or wgate.shape[:2] != (B, N) or wgate.shape[2] < H:
            raise ValueError(f"expected wgate [B={B}, N={N}, >={H}], got {tuple(wgate.shape)}")
        a.wgate, a.ldw = _ptr(wgate), _rows(wgate, B, N)
    return a


# ---------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def sva_linear_attn_workspace_bytes(B: int, N: int, H: int, d: int, dtype: int) -> int:
    return int(_lib().sva_linear_attn_workspace_bytes(B, N, H, d, dtype))


def sva_linear_attn_fwd(q, k, v, gate, out, H: int, residual=None, eps: float = 1e-6,
                        flags: int = 0, ws=None, stream=None, wgate=None):
    """Gated linear attention: out = phi(Q) S / (phi(Q).z + eps) * sigmoid(G) (+ residual).
    wgate [B, N, >=H] (optional): write-gate logits; token t's terms of S and z
    are scaled by sigmoid(wgate[b, t, h])."""
    a = _attn_args(q, k, v, gate, out, H, residual, eps, 0.0, flags, wgate)
    need = sva_linear_attn_workspace_bytes(a.B, a.N, a.H, a.d, a.dtype)
    ws = workspace(need, q.device) if ws is None else ws
    _check(_lib().sva_linear_attn_fwd(ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream)),
           "sva_linear_attn_fwd")
    return ws


def sva_linear_attn_state_bytes(B: int, H: int, d: int) -> int:
    return int(_lib().sva_linear_attn_state_bytes(B, H, d))


def sva_linear_attn_state_fwd(k, v, state, H: int, flags: int = 0, wgate=None, ws=None,
                              stream=None):
    """The fp32 state [B*H][d*d + d] (S, then z) of the tokens in k and v."""
    a = _attn_args(None, k, v, None, None, H, None, 0.0, 0.0, flags, wgate)
    _check_state(state, a)
    need = sva_linear_attn_workspace_bytes(a.B, a.N, a.H, a.d, a.dtype)
    ws = workspace(need, k.device) if ws is None else ws
    _check(_lib().sva_linear_attn_state_fwd(ctypes.byref(a), _ptr(state), _ptr(ws), ws.numel(),
                                            _stream(stream)), "sva_linear_attn_state_fwd")
    return ws


def sva_linear_attn_readout_fwd(q, gate, out, state, H: int, residual=None, eps: float = 1e-6,
                                flags: int = 0, ws=None, stream=None):
    """Y of the query tokens in q against a given fp32 state (e.g. summed over shards)."""
    a = _attn_args(q, None, None, gate, out, H, residual, eps, 0.0, flags)
    _check_state(state, a)
    need = sva_linear_attn_workspace_bytes(a.B, a.N, a.H, a.d, a.dtype)
    ws = workspace(need, q.device) if ws is None else ws
    _check(_lib().sva_linear_attn_readout_fwd(ctypes.byref(a), _ptr(state), _ptr(ws), ws.numel(),
                                              _stream(stream)), "sva_linear_attn_readout_fwd")
    return ws


def _check_state(state, a):
    torch = _torch()
    need = sva_linear_attn_state_bytes(a.B, a.H, a.d) // 4
    if state.dtype != torch.float32 or not state.is_contiguous() or state.numel() < need:
        raise ValueError(f"state must be a contiguous fp32 tensor of >= {need} values")


def sva_linear_attn_fwd_noalloc(q, k, v, gate, out, H: int, residual=None, eps: float = 1e-6,
                                flags: int = 0, stream=None, wgate=None):
    """sva_linear_attn_fwd without a workspace, for callers that cannot allocate
    device memory: the library's fixed 16 MiB device scratch is used instead.
    Calls that overlap on the GPU share that scratch and must be serialised."""
    a = _attn_args(q, k, v, gate, out, H, residual, eps, 0.0, flags, wgate)
    _check(_lib().sva_linear_attn_fwd_noalloc(ctypes.byref(a), _stream(stream)),
           "sva_linear_attn_fwd_noalloc")


def sva_softmax_anchor_fwd(q, k, v, gate, out, H: int, residual=None, scale: float = 0.0,
                           ws=None, stream=None):
    """Gated softmax anchor: out = softmax(scale Q K^T) V * sigmoid(G) (+ residual)."""
    a = _attn_args(q, k, v, gate, out, H, residual, 0.0, scale, 0)
    need = int(_lib().sva_softmax_anchor_workspace_bytes(a.B, a.N, a.H, a.d, a.dtype))
    ws = workspace(need, q.device) if ws is None else ws
    _check(_lib().sva_softmax_anchor_fwd(ctypes.byref(a), _ptr(ws), ws.numel(), _stream(stream)),
           "sva_softmax_anchor_fwd")
    return ws


def sva_projection_fwd(x, w, y, relu_cols: int = 0, ws=None, stream=None):
    """y = x W^T; x [M, K] (row stride allowed), W [Nout, K] contiguous, y [M, Nout]."""
    M, K = x.shape
    Nout = w.shape[0]
    if w.shape[1] != K or not w.is_contiguous() or y.shape != (M, Nout):
        raise ValueError("shape mismatch")
    ws = workspace(SVA_STATUS_BYTES, x.device) if ws is None else ws
    _check(_lib().sva_projection_fwd(_ptr(x), x.stride(0), _ptr(w), M, Nout, K, _ptr(y),
                                     y.stride(0), relu_cols, _dtype_code(x), _ptr(ws), ws.numel(),
                                     _stream(stream)), "sva_projection_fwd")
    return ws


def sva_projection_residual_fwd(x, w, h, h_copy=None, ws=None, stream=None):
    """h += x W^T (h fp32); h_copy = dtype(h) when given."""
    M, K = x.shape
    Nout = w.shape[0]
    ws = workspace(SVA_STATUS_BYTES, x.device) if ws is None else ws
    _check(_lib().sva_projection_residual_fwd(
        _ptr(x), x.stride(0), _ptr(w), M, Nout, K, _ptr(h), h.stride(0), _ptr(h_copy),
        h_copy.stride(0) if h_copy is not None else 0, _dtype_code(x), _ptr(ws), ws.numel(),
        _stream(stream)), "sva_projection_residual_fwd")
    return ws


def sva_attnres_keys(s_b, w_r, k_b, ws=None, stream=None):
    """k_b = s_b W_r for one completed block (s_b, k_b [rows, D] contiguous)."""
    rows, D = s_b.shape
    dt = _dtype_code(s_b)
    need = int(_lib().sva_attnres_keys_workspace_bytes(D, dt))
    ws = workspace(need, s_b.device) if ws is None else ws
    _check(_lib().sva_attnres_keys(_ptr(s_b), _ptr(w_r), _ptr(k_b), rows, D, dt, _ptr(ws),
                                   ws.numel(), _stream(stream)), "sva_attnres_keys")
    return ws


def sva_attnres_route(h, keys: Sequence, summaries: Sequence, u, alpha=None, stream=None):
    """u = h + sum_b softmax_b(h.k_b / sqrt(D)) s_b; alpha [rows, n] optional fp32 output."""
    rows, D = h.shape
    n = len(keys)
    kp = (ctypes.c_void_p * n)(*[_ptr(t) for t in keys])
    sp = (ctypes.c_void_p * n)(*[_ptr(t) for t in summaries])
    _check(_lib().sva_attnres_route(_ptr(h), kp, sp, n, _ptr(u), _ptr(alpha), rows, D,
                                    _dtype_code(u), _stream(stream)), "sva_attnres_route")


def _ptr_array(ts):
    if ts is None:
        return None, None
    arr = (ctypes.c_void_p * len(ts))(*[_ptr(t) for t in ts])
    return ctypes.cast(arr, _c_void_p_p), arr


class Stack:
    """Marshalled description of one hybrid stack (keeps the pointer arrays alive)."""

    def __init__(self, w_qkvg: Sequence, w_o: Sequence, w_r, B: int, N: int, H: int,
                 softmax_period: int = 4, attnres_block: int = 8, all_softmax: bool = False,
                 eps: float = 1e-6, trace_o=None, trace_y=None, trace_alpha=None, w_wg=None):
        L = len(w_qkvg)
        D = w_qkvg[0].shape[1]
        d = StackDesc()
        d.B, d.N, d.H, d.d, d.L = B, N, H, D // H, L
        d.dtype = _dtype_code(w_qkvg[0])
        d.softmax_period, d.attnres_block, d.all_softmax = softmax_period, attnres_block, int(all_softmax)
        self._keep = []
        d.w_qkvg, a = _ptr_array(list(w_qkvg)); self._keep.append(a)
        d.w_o, a = _ptr_array(list(w_o)); self._keep.append(a)
        d.w_r = _ptr(w_r)
        d.eps = float(eps)
        for name, ts in (("trace_o", trace_o), ("trace_y", trace_y), ("trace_alpha", trace_alpha),
                         ("w_wg", w_wg)):
            p, a = _ptr_array(ts)
            if p is not None:
                setattr(d, name, p)
                self._keep.append(a)
        self.desc = d
        self.tensors = (w_qkvg, w_o, w_r, trace_o, trace_y, trace_alpha, w_wg)
        self.prof_count = ctypes.c_int(0)
        self.launch_count = ctypes.c_int(0)

    def set_profile(self, events: Sequence, kinds_capacity: int):
        """events: 2*capacity torch.cuda.Event(enable_timing=True), already recorded once."""
        cap = kinds_capacity
        arr = (ctypes.c_void_p * (2 * cap))(*[ev.cuda_event for ev in events])
        self._prof_arr = arr
        self.prof_kind = (ctypes.c_int * cap)()
        self.desc.prof_events = ctypes.cast(arr, _c_void_p_p)
        self.desc.prof_capacity = cap
        self.desc.prof_kind = ctypes.cast(self.prof_kind, ctypes.POINTER(ctypes.c_int))
        self.desc.prof_count = ctypes.pointer(self.prof_count)
        self.desc.launch_count = ctypes.pointer(self.launch_count)

    def count_launches(self):
        """Have each later call write the number of kernels it launched to
        self.launch_count (no events recorded)."""
        self.desc.launch_count = ctypes.pointer(self.launch_count)

    def clear_profile(self):
        self.desc.prof_events = None
        self.desc.prof_capacity = 0
        self.desc.prof_kind = None
        self.desc.prof_count = None
        self.desc.launch_count = None

    def workspace_bytes(self) -> int:
        n = int(_lib().sva_hybrid_stack_workspace_bytes(ctypes.byref(self.desc)))
        if n == 0:
            raise SvaError(SVA_ERR_INVALID_ARGUMENT, "sva_hybrid_stack_workspace_bytes")
        return n


def sva_hybrid_stack_workspace_bytes(stack: Stack) -> int:
    return stack.workspace_bytes()


def sva_hybrid_stack_fwd(stack: Stack, x, y, ws=None, stream=None):
    """y = the hybrid stack applied to x ([B, N, D], contiguous, dtype of the weights)."""
    if not (x.is_contiguous() and y.is_contiguous()):
        raise ValueError("x and y must be contiguous [B, N, D]")
    ws = workspace(stack.workspace_bytes(), x.device) if ws is None else ws
    _check(_lib().sva_hybrid_stack_fwd(ctypes.byref(stack.desc), _ptr(x), _ptr(y), _ptr(ws),
                                       ws.numel(), _stream(stream)), "sva_hybrid_stack_fwd")
    return ws


def sva_hybrid_stack_host_staging_bytes(stack: Stack) -> int:
    return int(_lib().sva_hybrid_stack_host_staging_bytes(ctypes.byref(stack.desc)))


def sva_hybrid_stack_fwd_host(stack: Stack, xs_host: Sequence, ys_host: Sequence, ws=None,
                              staging=None, stream=None):
    """The stack over host batches: ys_host[i] = stack(xs_host[i]), copies in and
    out overlapped with the passes (CPU tensors [B, N, D], contiguous; pin them
    for the overlap). Asynchronous on `stream`. Returns (ws, staging)."""
    if len(xs_host) != len(ys_host):
        raise ValueError("one output per input")
    for t in list(xs_host) + list(ys_host):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("host batches must be contiguous CPU tensors")
    torch = _torch()
    dev = torch.device("cuda", torch.cuda.current_device())
    ws = workspace(stack.workspace_bytes(), dev) if ws is None else ws
    if staging is None:
        staging = workspace(sva_hybrid_stack_host_staging_bytes(stack), dev)
    n = len(xs_host)
    xp = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in xs_host])
    yp = (ctypes.c_void_p * max(n, 1))(*[t.data_ptr() for t in ys_host])
    _check(_lib().sva_hybrid_stack_fwd_host(
        ctypes.byref(stack.desc), ctypes.cast(xp, _c_void_p_p), ctypes.cast(yp, _c_void_p_p), n,
        _ptr(ws), ws.numel(), _ptr(staging), staging.numel(), _stream(stream)),
        "sva_hybrid_stack_fwd_host")
    return ws, staging


def sva_check_device_status(ws, stream=None) -> int:
    return int(_lib().sva_check_device_status(_ptr(ws), _stream(stream)))


def sva_selftest_bounded_wait(ws, timeout_us: int, stream=None):
    _check(_lib().sva_selftest_bounded_wait(_ptr(ws), ws.numel(), timeout_us, _stream(stream)),
           "sva_selftest_bounded_wait")


def sva_version() -> int:
    return int(_lib().sva_version())
