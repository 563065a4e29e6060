"""Thin ctypes binding over libgdn.so: the C ABI of include/gdn.h with the same names.

Only argument marshalling happens here: shapes, dtypes and devices of torch tensors are
checked, outputs and the workspace are allocated with torch when the caller passes none,
and raw device pointers plus the current CUDA stream go to the library.  Every step of
the mixer runs in the library's CUDA kernels; there is no CPU or eager fallback.  If the
library is missing this module raises on first use.
"""
from __future__ import annotations

import ctypes
import os

import torch

GDN_OK = 0
GDN_ERR_INDEX = -8
GDN_ERR_DEVICE_TIMEOUT = -7
GDN_DTYPE_F32 = 0
GDN_DTYPE_BF16 = 1
# path options (gdn_set_options): slower alternatives with the same results, for comparisons
GDN_OPT_FORCE_FP32_PATH = 1
GDN_OPT_SEPARATE_NORM = 2
GDN_OPT_NO_PDL = 4
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libgdn.so")
_lib = None


class GdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where} failed: {gdn_status_string(code)} ({code})")


class gdn_dims_t(ctypes.Structure):
    _fields_ = [
        ("n_seqs", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("h_qk", ctypes.c_int32),
        ("h_v", ctypes.c_int32),
        ("d_k", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("in_dtype", ctypes.c_int32),
        ("out_dtype", ctypes.c_int32),
        ("q_scale", ctypes.c_float),
        ("l2_eps", ctypes.c_float),
        ("rms_eps", ctypes.c_float),
    ]


class gdn_kernel_time_t(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


def lib() -> ctypes.CDLL:
    """Load libgdn.so (built by __graft_entry__.build() or gated_deltanet_token_b200._build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"libgdn.so not found at {_LIB_PATH}: build it first "
                               "(python -m gated_deltanet_token_b200._build)")
        L = ctypes.CDLL(_LIB_PATH)
        vp, dp = ctypes.c_void_p, ctypes.POINTER(gdn_dims_t)
        L.gdn_prefill_workspace_size.restype = ctypes.c_size_t
        L.gdn_prefill_workspace_size.argtypes = [dp]
        L.gdn_prefill.restype = ctypes.c_int
        L.gdn_prefill.argtypes = [dp] + [vp] * 14 + [vp, ctypes.c_size_t, vp]
        L.gdn_prefill_noalloc.restype = ctypes.c_int
        L.gdn_prefill_noalloc.argtypes = [dp] + [vp] * 14 + [vp]
        L.gdn_decode.restype = ctypes.c_int
        L.gdn_decode.argtypes = [dp] + [vp] * 13 + [vp]
        L.gdn_decode_slots.restype = ctypes.c_int
        L.gdn_decode_slots.argtypes = [dp] + [vp] * 12 + [ctypes.c_int32, vp, vp, vp]
        L.gdn_decode_multi.restype = ctypes.c_int
        L.gdn_decode_multi.argtypes = [dp, ctypes.c_int32] + [vp] * 13 + [vp]
        L.gdn_in_proj.restype = ctypes.c_int
        L.gdn_in_proj.argtypes = [dp, ctypes.c_int32] + [vp] * 8 + [vp]
        L.gdn_out_proj.restype = ctypes.c_int
        L.gdn_out_proj.argtypes = [dp, ctypes.c_int32] + [vp] * 3 + [vp]
        L.gdn_recurrence_backward_workspace_size.restype = ctypes.c_size_t
        L.gdn_recurrence_backward_workspace_size.argtypes = [dp]
        L.gdn_recurrence_backward.restype = ctypes.c_int
        L.gdn_recurrence_backward.argtypes = [dp] + [vp] * 15 + [vp, ctypes.c_size_t, vp]
        L.gdn_prefill_conv_state.restype = ctypes.c_int
        L.gdn_prefill_conv_state.argtypes = [dp] + [vp] * 5 + [vp]
        L.gdn_status_string.restype = ctypes.c_char_p
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_read_device_status.restype = ctypes.c_int
        L.gdn_read_device_status.argtypes = [vp]
        L.gdn_profile_enable.restype = ctypes.c_int
        L.gdn_profile_enable.argtypes = [ctypes.c_int]
        L.gdn_profile_read.restype = ctypes.c_int
        L.gdn_profile_read.argtypes = [ctypes.POINTER(gdn_kernel_time_t), ctypes.c_int]
        L.gdn_selftest_tc.restype = ctypes.c_int
        L.gdn_selftest_tc.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_float)]
        L.gdn_version.restype = ctypes.c_int
        L.gdn_version.argtypes = []
        L.gdn_set_options.restype = ctypes.c_uint32
        L.gdn_set_options.argtypes = [ctypes.c_uint32]
        L.gdn_get_options.restype = ctypes.c_uint32
        L.gdn_get_options.argtypes = []
        L.gdn_set_wait_limit_ns.restype = ctypes.c_int
        L.gdn_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
        L.gdn_selftest_wait_timeout.restype = ctypes.c_int
        L.gdn_selftest_wait_timeout.argtypes = [vp]
        _lib = L
    return _lib


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return GDN_DTYPE_BF16
    if t.dtype == torch.float32:
        return GDN_DTYPE_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch tensor")
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("tensors must be contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def make_dims(n_seqs, total_tokens, h_qk, h_v, in_dtype, out_dtype, d_k=128, d_v=128,
              q_scale=1.0, l2_eps=1e-6, rms_eps=1e-6) -> gdn_dims_t:
    return gdn_dims_t(n_seqs, total_tokens, h_qk, h_v, d_k, d_v, in_dtype, out_dtype, q_scale,
                      l2_eps, rms_eps)


def gdn_status_string(code: int) -> str:
    return lib().gdn_status_string(code).decode()


def gdn_version() -> int:
    return lib().gdn_version()


def gdn_read_device_status(stream=None) -> int:
    return lib().gdn_read_device_status(_stream(stream))


def gdn_set_options(flags: int) -> int:
    """Replace the process-wide path options; returns the previous word."""
    return int(lib().gdn_set_options(int(flags)))


def gdn_get_options() -> int:
    return int(lib().gdn_get_options())


def gdn_set_wait_limit_ns(ns: int) -> None:
    rc = lib().gdn_set_wait_limit_ns(int(ns))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_set_wait_limit_ns")


def gdn_selftest_wait_timeout(stream=None) -> None:
    """Launch the bounded-wait diagnostic (read its result with gdn_read_device_status)."""
    rc = lib().gdn_selftest_wait_timeout(_stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_selftest_wait_timeout")


def gdn_selftest_tc(case_id: int) -> tuple[float, float]:
    """(max |tensor-core - CUDA-core|, max |reference|) for one operand-layout case."""
    out = (ctypes.c_float * 2)()
    rc = lib().gdn_selftest_tc(int(case_id), out)
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_selftest_tc")
    return float(out[0]), float(out[1])


def gdn_profile_enable(on: bool) -> None:
    rc = lib().gdn_profile_enable(int(bool(on)))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_profile_enable")


def gdn_profile_read() -> dict:
    """{kernel name: (launches, total_ms)} since the last read."""
    buf = (gdn_kernel_time_t * 64)()
    m = lib().gdn_profile_read(buf, 64)
    if m < 0:
        raise GdnError(m, "gdn_profile_read")
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(m)}


def gdn_prefill_workspace_size(dims: gdn_dims_t) -> int:
    return lib().gdn_prefill_workspace_size(ctypes.byref(dims))


def gdn_prefill(q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, init_state=None,
                cu_seqlens=None, *, out_dtype=None, y=None, final_state=None, workspace=None,
                q_scale=1.0, l2_eps=1e-6, rms_eps=1e-6, stream=None):
    """Prefill over packed sequences.  q, k [T, h_qk, 128]; v, z [T, h_v, 128]; a, b [T, h_v];
    cu_seqlens int32 [N+1] on the device (None = one sequence).  Returns (y, final_state)."""
    T, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    n = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if out_dtype is None:
        out_dtype = q.dtype
    dims = make_dims(n, T, h_qk, h_v, _dt(q), _dt(torch.empty(0, dtype=out_dtype)), d_k, d_v, q_scale,
                     l2_eps, rms_eps)
    dev = q.device
    if y is None:
        y = torch.empty((T, h_v, d_v), dtype=out_dtype, device=dev)
    if final_state is None:
        final_state = torch.empty((n, h_v, d_v, d_k), dtype=torch.float32, device=dev)
    need = gdn_prefill_workspace_size(dims)
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=dev)
    rc = lib().gdn_prefill(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(a), _ptr(b),
                           _ptr(A_log), _ptr(dt_bias), _ptr(conv_w), _ptr(norm_w), _ptr(init_state),
                           _ptr(cu_seqlens), _ptr(y), _ptr(final_state), _ptr(workspace),
                           workspace.numel() * workspace.element_size(), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_prefill")
    return y, final_state


def gdn_prefill_noalloc(q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, init_state=None,
                        cu_seqlens=None, *, out_dtype=None, y=None, final_state=None,
                        q_scale=1.0, l2_eps=1e-6, rms_eps=1e-6, stream=None):
    """gdn_prefill on the library's built-in scratch (no workspace argument).  For callers
    that cannot allocate device memory at call time; outputs must then be passed in.
    Dims whose workspace exceeds the built-in scratch raise GdnError(GDN_ERR_WORKSPACE)."""
    T, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    n = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if out_dtype is None:
        out_dtype = y.dtype if y is not None else q.dtype
    dims = make_dims(n, T, h_qk, h_v, _dt(q), _dt(torch.empty(0, dtype=out_dtype)), d_k, d_v, q_scale,
                     l2_eps, rms_eps)
    if y is None:
        y = torch.empty((T, h_v, d_v), dtype=out_dtype, device=q.device)
    if final_state is None:
        final_state = torch.empty((n, h_v, d_v, d_k), dtype=torch.float32, device=q.device)
    rc = lib().gdn_prefill_noalloc(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(a),
                                   _ptr(b), _ptr(A_log), _ptr(dt_bias), _ptr(conv_w), _ptr(norm_w),
                                   _ptr(init_state), _ptr(cu_seqlens), _ptr(y), _ptr(final_state),
                                   _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_prefill_noalloc")
    return y, final_state


def gdn_decode(q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state, state, *,
               out_dtype=None, y=None, q_scale=1.0, l2_eps=1e-6, rms_eps=1e-6, stream=None):
    """One decode step.  conv_state [N, 3, C_conv] and state [N, h_v, 128, 128] are updated in
    place.  Returns y [N, h_v, 128]."""
    N, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    if out_dtype is None:
        out_dtype = q.dtype
    dims = make_dims(N, N, h_qk, h_v, _dt(q), _dt(torch.empty(0, dtype=out_dtype)), d_k, d_v, q_scale,
                     l2_eps, rms_eps)
    if y is None:
        y = torch.empty((N, h_v, d_v), dtype=out_dtype, device=q.device)
    rc = lib().gdn_decode(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(a), _ptr(b),
                          _ptr(A_log), _ptr(dt_bias), _ptr(conv_w), _ptr(norm_w), _ptr(conv_state),
                          _ptr(state), _ptr(y), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode")
    return y


def gdn_prefill_conv_state(q, k, v, cu_seqlens=None, *, conv_state=None, stream=None):
    """The decode conv history after a prefill over the same packed q, k, v: per sequence the
    raw q | k | v channels of its last three tokens (zeros before its first token).  Returns
    conv_state [N, 3, C_conv] in the inputs' dtype."""
    T, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    n = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    if cu_seqlens is not None and cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    dims = make_dims(n, T, h_qk, h_v, _dt(q), _dt(q), d_k, d_v)
    if conv_state is None:
        conv_state = torch.empty((n, 3, (2 * h_qk + h_v) * d_k), dtype=q.dtype, device=q.device)
    rc = lib().gdn_prefill_conv_state(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(cu_seqlens),
                                      _ptr(conv_state), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_prefill_conv_state")
    return conv_state


def gdn_decode_slots(q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state_pool, state_pool,
                     slot_ids, *, out_dtype=None, y=None, q_scale=1.0, l2_eps=1e-6, rms_eps=1e-6,
                     stream=None):
    """One decode step on resident pools: sequence n updates conv_state_pool[slot_ids[n]] and
    state_pool[slot_ids[n]] in place (slot_ids int32 on the device; a negative id is a padding
    entry).  Returns y [N, h_v, 128]."""
    N, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    if slot_ids.dtype != torch.int32 or slot_ids.numel() != N:
        raise TypeError("slot_ids must be int32 with one entry per sequence")
    if conv_state_pool.shape[0] != state_pool.shape[0]:
        raise ValueError("conv_state_pool and state_pool must have the same number of slots")
    if out_dtype is None:
        out_dtype = q.dtype
    dims = make_dims(N, N, h_qk, h_v, _dt(q), _dt(torch.empty(0, dtype=out_dtype)), d_k, d_v, q_scale,
                     l2_eps, rms_eps)
    if y is None:
        y = torch.empty((N, h_v, d_v), dtype=out_dtype, device=q.device)
    rc = lib().gdn_decode_slots(ctypes.byref(dims), _ptr(q), _ptr(k), _ptr(v), _ptr(z), _ptr(a), _ptr(b),
                                _ptr(A_log), _ptr(dt_bias), _ptr(conv_w), _ptr(norm_w), _ptr(conv_state_pool),
                                _ptr(state_pool), ctypes.c_int32(state_pool.shape[0]), _ptr(slot_ids), _ptr(y),
                                _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_slots")
    return y


def gdn_decode_multi(q, k, v, z, a, b, A_log, dt_bias, conv_w, norm_w, conv_state, state, *,
                     out_dtype=None, y=None, q_scale=1.0, l2_eps=1e-6, rms_eps=1e-6, stream=None):
    """n_tokens decode steps per sequence in one call: q, k [N, n_tokens, h_qk, 128]; v, z
    [N, n_tokens, h_v, 128]; a, b [N, n_tokens, h_v].  conv_state [N, 3, C_conv] and state
    [N, h_v, 128, 128] are updated in place.  Returns y [N, n_tokens, h_v, 128]."""
    N, K, h_qk, d_k = q.shape
    h_v, d_v = v.shape[2], v.shape[3]
    if out_dtype is None:
        out_dtype = q.dtype
    dims = make_dims(N, N * K, h_qk, h_v, _dt(q), _dt(torch.empty(0, dtype=out_dtype)), d_k, d_v, q_scale,
                     l2_eps, rms_eps)
    if y is None:
        y = torch.empty((N, K, h_v, d_v), dtype=out_dtype, device=q.device)
    rc = lib().gdn_decode_multi(ctypes.byref(dims), ctypes.c_int32(K), _ptr(q), _ptr(k), _ptr(v), _ptr(z),
                                _ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), _ptr(conv_w), _ptr(norm_w),
                                _ptr(conv_state), _ptr(state), _ptr(y), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_decode_multi")
    return y


def gdn_in_proj(x, w_in, h_qk, h_v, *, d_k=128, d_v=128, out=None, stream=None):
    """[q | k | v | z | a | b] = x w_in^T for x [T, hidden] bf16 and w_in [N_in, hidden] bf16.
    Returns (q [T, h_qk, d_k], k, v [T, h_v, d_v], z, a [T, h_v] fp32, b); `out` may hold
    preallocated tensors in that order."""
    T, hidden = x.shape
    if w_in.dtype != torch.bfloat16 or x.dtype != torch.bfloat16:
        raise TypeError("x and w_in must be bf16")
    if w_in.shape != (2 * h_qk * d_k + 2 * h_v * d_v + 2 * h_v, hidden):
        raise ValueError("w_in must be [2 h_qk d_k + 2 h_v d_v + 2 h_v, hidden]")
    if out is None:
        dev = x.device
        out = (torch.empty((T, h_qk, d_k), dtype=torch.bfloat16, device=dev),
               torch.empty((T, h_qk, d_k), dtype=torch.bfloat16, device=dev),
               torch.empty((T, h_v, d_v), dtype=torch.bfloat16, device=dev),
               torch.empty((T, h_v, d_v), dtype=torch.bfloat16, device=dev),
               torch.empty((T, h_v), dtype=torch.float32, device=dev),
               torch.empty((T, h_v), dtype=torch.float32, device=dev))
    dims = make_dims(1, T, h_qk, h_v, GDN_DTYPE_BF16, GDN_DTYPE_BF16, d_k, d_v)
    rc = lib().gdn_in_proj(ctypes.byref(dims), ctypes.c_int32(hidden), _ptr(x), _ptr(w_in),
                           *[_ptr(t) for t in out], _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_in_proj")
    return out


def gdn_out_proj(y, w_out, h_qk, h_v, *, d_v=128, out=None, stream=None):
    """out = y w_out^T for y [T, h_v, d_v] (or [T, h_v d_v]) bf16 and w_out [hidden, h_v d_v] bf16;
    returns out [T, hidden] bf16."""
    T = y.shape[0]
    hidden = w_out.shape[0]
    if y.dtype != torch.bfloat16 or w_out.dtype != torch.bfloat16:
        raise TypeError("y and w_out must be bf16")
    if w_out.shape[1] != h_v * d_v or y.numel() != T * h_v * d_v:
        raise ValueError("w_out must be [hidden, h_v d_v] and y [T, h_v, d_v]")
    if out is None:
        out = torch.empty((T, hidden), dtype=torch.bfloat16, device=y.device)
    dims = make_dims(1, T, h_qk, h_v, GDN_DTYPE_BF16, GDN_DTYPE_BF16, 128, d_v)
    rc = lib().gdn_out_proj(ctypes.byref(dims), ctypes.c_int32(hidden), _ptr(y), _ptr(w_out), _ptr(out),
                            _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_out_proj")
    return out


def gdn_recurrence_backward(qh, kh, v, g, beta, init_state, cu_seqlens, dy, dS_final, *, workspace=None,
                            stream=None):
    """Gradients of the recurrence core: qh, kh [T, h_qk, d_k], v [T, h_v, d_v], g, beta [T, h_v],
    init_state [N, h_v, d_v, d_k] or None, cu_seqlens [N + 1] int32 or None (one sequence), dy
    [T, h_v, d_v] (dL/dy before the output norm), dS_final [N, h_v, d_v, d_k] or None.  All fp32.
    Returns (dq, dk, dv, dg, dbeta, dS_init)."""
    T, h_qk, d_k = qh.shape
    h_v, d_v = v.shape[1], v.shape[2]
    N = 1 if cu_seqlens is None else cu_seqlens.numel() - 1
    for t in (qh, kh, v, g, beta, dy):
        if t.dtype != torch.float32:
            raise TypeError("the backward takes fp32 tensors")
    dims = make_dims(N, T, h_qk, h_v, GDN_DTYPE_F32, GDN_DTYPE_F32, d_k, d_v)
    dev = qh.device
    dq, dk = torch.empty_like(qh), torch.empty_like(kh)
    dv = torch.empty_like(v)
    dg, dbeta = torch.empty_like(g), torch.empty_like(beta)
    dS_init = torch.empty((N, h_v, d_v, d_k), dtype=torch.float32, device=dev)
    need = lib().gdn_recurrence_backward_workspace_size(ctypes.byref(dims))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    rc = lib().gdn_recurrence_backward(ctypes.byref(dims), _ptr(qh), _ptr(kh), _ptr(v), _ptr(g), _ptr(beta),
                                       _ptr(init_state), _ptr(cu_seqlens), _ptr(dy), _ptr(dS_final), _ptr(dq),
                                       _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(dS_init), _ptr(workspace),
                                       ctypes.c_size_t(workspace.numel()), _stream(stream))
    if rc != GDN_OK:
        raise GdnError(rc, "gdn_recurrence_backward")
    return dq, dk, dv, dg, dbeta, dS_init
