"""fp64 CPU oracle for the Gated DeltaNet token mixer -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py``
may import this package.  The CUDA library never calls it, and it shares no code with
the CUDA library: the mixer's arithmetic lives in ``gdn_oracle.c`` (plain C, fp64) and this
module marshals numpy arrays through ctypes; the two projections around the mixer are one
fp64 matrix product each (``in_proj``, ``out_proj`` below, numpy).

Element encodings: numpy ``float32`` arrays are fp32 inputs, ``uint16`` arrays are raw
bf16 bits.  Both are widened exactly to fp64 inside the C code.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# A test may point this at a separately built copy of the oracle (the planted-mistake test).
_LIB_OVERRIDE = os.environ.get("GDN_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

ENC_F32 = 0
ENC_BF16 = 1


class OracleDims(ctypes.Structure):
    _fields_ = [
        ("n_seqs", ctypes.c_int32),
        ("total_tokens", ctypes.c_int32),
        ("h_qk", ctypes.c_int32),
        ("h_v", ctypes.c_int32),
        ("d_k", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
        ("in_enc", ctypes.c_int32),
        ("q_scale", ctypes.c_double),
        ("l2_eps", ctypes.c_double),
        ("rms_eps", ctypes.c_double),
        ("chunk", ctypes.c_int32),
        ("n_threads", ctypes.c_int32),
    ]


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into liboracle.so (plain -O2, no fast-math, OpenMP threads)."""
    with _lock:
        if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            tmp = _LIB + f".{os.getpid()}.tmp"
            subprocess.check_call(
                ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-o", tmp, _SRC, "-lm"]
            )
            os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    if _lib is None:
        if _LIB_OVERRIDE:
            L = ctypes.CDLL(_LIB_OVERRIDE)
        else:
            build()
            L = ctypes.CDLL(_LIB)
        d = ctypes.c_double
        dp = ctypes.POINTER(ctypes.c_double)
        vp = ctypes.c_void_p
        for name in ("oracle_softplus", "oracle_sigmoid", "oracle_silu"):
            f = getattr(L, name)
            f.restype, f.argtypes = d, [d]
        L.oracle_decay_gate.restype, L.oracle_decay_gate.argtypes = d, [d, d, d]
        L.oracle_conv_silu_channel.restype = None
        L.oracle_conv_silu_channel.argtypes = [vp, ctypes.c_long, ctypes.c_long, vp, vp, vp]
        L.oracle_l2norm.restype, L.oracle_l2norm.argtypes = None, [vp, ctypes.c_int, d]
        L.oracle_gated_rmsnorm.restype = None
        L.oracle_gated_rmsnorm.argtypes = [vp, vp, vp, ctypes.c_int, d, vp]
        for name in ("oracle_recurrence_token",):
            f = getattr(L, name)
            f.restype = None
            f.argtypes = [ctypes.c_long, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, d, vp, vp]
        L.oracle_recurrence_chunked.restype = None
        L.oracle_recurrence_chunked.argtypes = [
            ctypes.c_long, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, d, vp, vp]
        L.oracle_prefill.restype = ctypes.c_int
        L.oracle_prefill.argtypes = [ctypes.POINTER(OracleDims)] + [vp] * 12 + [
            ctypes.c_int, ctypes.c_int, vp, vp, vp]
        L.oracle_decode.restype = ctypes.c_int
        L.oracle_decode.argtypes = [ctypes.POINTER(OracleDims)] + [vp] * 16
        _ = dp
        _lib = L
    return _lib


def _p(x):
    return None if x is None else ctypes.c_void_p(x.ctypes.data)


def _c64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _enc(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return ENC_BF16
    if x.dtype == np.float32:
        return ENC_F32
    raise TypeError(f"oracle inputs must be float32 or uint16 (bf16 bits), got {x.dtype}")


# ---- scalar and stage functions -------------------------------------------------------

def softplus(x: float) -> float:
    return lib().oracle_softplus(float(x))


def sigmoid(x: float) -> float:
    return lib().oracle_sigmoid(float(x))


def silu(x: float) -> float:
    return lib().oracle_silu(float(x))


def decay_gate(a: float, A_log: float, dt_bias: float) -> float:
    return lib().oracle_decay_gate(float(a), float(A_log), float(dt_bias))


def conv_silu(x: np.ndarray, w: np.ndarray, hist: np.ndarray | None = None) -> np.ndarray:
    """Width-4 causal conv + SiLU over one channel: x [T], w [4], hist [3] or None."""
    x = _c64(x)
    out = np.empty_like(x)
    w = _c64(w)
    h = None if hist is None else _c64(hist)
    lib().oracle_conv_silu_channel(_p(x), 1, x.shape[0], _p(w), _p(h), _p(out))
    return out


def l2norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    x = _c64(x).copy()
    lib().oracle_l2norm(_p(x), x.shape[0], eps)
    return x


def gated_rmsnorm(y_raw, z, norm_w, eps: float = 1e-6) -> np.ndarray:
    y_raw, z, norm_w = _c64(y_raw), _c64(z), _c64(norm_w)
    out = np.empty_like(y_raw)
    lib().oracle_gated_rmsnorm(_p(y_raw), _p(z), _p(norm_w), y_raw.shape[0], eps, _p(out))
    return out


def recurrence(qh, kh, v, g, beta, S0, q_scale: float = 1.0, chunk: int = 0):
    """Recurrence core of one (sequence, value head) on convolved, normalised streams.

    qh, kh [T, d_k]; v [T, d_v]; g, beta [T]; S0 [d_v, d_k].  chunk = 0 runs the per-token
    rule; chunk > 0 runs the chunked rewrite.  Returns (y_raw [T, d_v], S_final).
    """
    qh, kh, v, g, beta = map(_c64, (qh, kh, v, g, beta))
    S = _c64(S0).copy()
    T, dk = kh.shape
    dv = v.shape[1]
    y = np.zeros((T, dv), np.float64)
    if chunk:
        lib().oracle_recurrence_chunked(T, dk, dv, chunk, _p(qh), _p(kh), _p(v), _p(g), _p(beta),
                                        q_scale, _p(S), _p(y))
    else:
        lib().oracle_recurrence_token(T, dk, dv, _p(qh), _p(kh), _p(v), _p(g), _p(beta), q_scale,
                                      _p(S), _p(y))
    return y, S


def recurrence_backward(qh, kh, v, g, beta, S0, dy, dS_T):
    """Reverse-mode gradients of the recurrence core of one (sequence, value head), in fp64.

    The forward is field guide §02's per-token rule (column-vector S, d_v x d_k), with
    alpha_t = e^{g_t}:  S'_t = alpha_t S_{t-1};  e_t = v_t - S'_t k_t;
    S_t = S'_t + beta_t e_t k_t^T;  y_t = S_t q_t.  Given dy [T, d_v] (dL/dy_t) and dS_T
    (dL/dS_T), walking the tokens from the last with D = dL/dS_t:
      D += dy_t q_t^T;  dq_t = S_t^T dy_t;  w = D k_t;  de_t = beta_t w;  dbeta_t = e_t . w;
      dv_t = de_t;  dk_t = beta_t D^T e_t - S'_t^T de_t;  dS'_t = D - de_t k_t^T;
      dg_t = alpha_t <dS'_t, S_{t-1}>;  D <- alpha_t dS'_t.
    Returns dict(dq [T, d_k], dk [T, d_k], dv [T, d_v], dg [T], dbeta [T], dS0 [d_v, d_k])."""
    qh, kh, v, g, beta, dy = map(lambda a: np.asarray(a, np.float64), (qh, kh, v, g, beta, dy))
    T = kh.shape[0]
    S = [np.asarray(S0, np.float64).copy()]
    for t in range(T):  # the forward, keeping every state
        Sp = np.exp(g[t]) * S[-1]
        e = v[t] - Sp @ kh[t]
        S.append(Sp + beta[t] * np.outer(e, kh[t]))
    D = np.asarray(dS_T, np.float64).copy()
    out = {"dq": np.zeros_like(qh), "dk": np.zeros_like(kh), "dv": np.zeros_like(v),
           "dg": np.zeros(T), "dbeta": np.zeros(T)}
    for t in range(T - 1, -1, -1):
        a = np.exp(g[t])
        Sp = a * S[t]
        e = v[t] - Sp @ kh[t]
        D = D + np.outer(dy[t], qh[t])
        out["dq"][t] = S[t + 1].T @ dy[t]
        w = D @ kh[t]
        de = beta[t] * w
        out["dbeta"][t] = e @ w
        out["dv"][t] = de
        out["dk"][t] = beta[t] * (D.T @ e) - Sp.T @ de
        dSp = D - np.outer(de, kh[t])
        out["dg"][t] = a * np.sum(dSp * S[t])
        D = a * dSp
    out["dS0"] = D
    return out


# ---- whole mixer ----------------------------------------------------------------------

def _dims(n_seqs, total, h_qk, h_v, d_k, d_v, enc, q_scale, l2_eps, rms_eps, chunk, threads):
    return OracleDims(n_seqs, total, h_qk, h_v, d_k, d_v, enc, q_scale, l2_eps, rms_eps, chunk,
                      threads)


def prefill(inp: dict, heads: tuple[int, int] | None = None, chunk: int = 0, n_threads: int = 0,
            q_scale: float = 1.0, l2_eps: float = 1e-6, rms_eps: float = 1e-6,
            want_state: bool = True, want_y_raw: bool = False):
    """Run the oracle prefill on an input dict (see gated_deltanet_token_b200.inputs).

    Returns dict(y=[T,h_v,d_v] f64, final_state=[N,h_v,d_v,d_k] f64 or None, y_raw=...).
    Only value heads in ``heads`` = (h0, h1) are computed; other entries stay zero.
    """
    q, k, v, z = (np.ascontiguousarray(inp[n]) for n in ("q", "k", "v", "z"))
    enc = _enc(q)
    T, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    cu = inp.get("cu_seqlens")
    n_seqs = 1 if cu is None else len(cu) - 1
    cu32 = None if cu is None else np.ascontiguousarray(cu, dtype=np.int32)
    h0, h1 = heads if heads is not None else (0, h_v)
    f32 = lambda n: np.ascontiguousarray(inp[n], dtype=np.float32)  # noqa: E731
    init = inp.get("init_state")
    init = None if init is None else np.ascontiguousarray(init, dtype=np.float32)
    y = np.zeros((T, h_v, d_v), np.float64)
    y_raw = np.zeros((T, h_v, d_v), np.float64) if want_y_raw else None
    fs = np.zeros((n_seqs, h_v, d_v, d_k), np.float64) if want_state else None
    dims = _dims(n_seqs, T, h_qk, h_v, d_k, d_v, enc, q_scale, l2_eps, rms_eps, chunk, n_threads)
    a, b, A_log, dt_bias, conv_w, norm_w = (f32(n) for n in ("a", "b", "A_log", "dt_bias", "conv_w",
                                                            "norm_w"))
    rc = lib().oracle_prefill(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(z), _p(a), _p(b),
                              _p(A_log), _p(dt_bias), _p(conv_w), _p(norm_w), _p(init), _p(cu32),
                              h0, h1, _p(y), _p(y_raw), _p(fs))
    if rc != 0:
        raise ValueError("oracle_prefill rejected its arguments")
    return {"y": y, "final_state": fs, "y_raw": y_raw}


def decode(inp: dict, n_threads: int = 0, q_scale: float = 1.0, l2_eps: float = 1e-6,
           rms_eps: float = 1e-6, want_state: bool = True):
    """Oracle decode step.  Returns dict(y, y_raw, state, conv_state) in fp64."""
    q, k, v, z = (np.ascontiguousarray(inp[n]) for n in ("q", "k", "v", "z"))
    enc = _enc(q)
    N, h_qk, d_k = q.shape
    h_v, d_v = v.shape[1], v.shape[2]
    f32 = lambda n: np.ascontiguousarray(inp[n], dtype=np.float32)  # noqa: E731
    a, b, A_log, dt_bias, conv_w, norm_w, state = (
        f32(n) for n in ("a", "b", "A_log", "dt_bias", "conv_w", "norm_w", "state"))
    cs = np.ascontiguousarray(inp["conv_state"])
    if _enc(cs) != enc:
        raise TypeError("conv_state must use the same encoding as q, k, v, z")
    y = np.zeros((N, h_v, d_v), np.float64)
    y_raw = np.zeros((N, h_v, d_v), np.float64)
    st = np.zeros((N, h_v, d_v, d_k), np.float64) if want_state else None
    cso = np.zeros(cs.shape, np.float64)
    dims = _dims(N, N, h_qk, h_v, d_k, d_v, enc, q_scale, l2_eps, rms_eps, 0, n_threads)
    rc = lib().oracle_decode(ctypes.byref(dims), _p(q), _p(k), _p(v), _p(z), _p(a), _p(b),
                             _p(A_log), _p(dt_bias), _p(conv_w), _p(norm_w), _p(cs), _p(state),
                             _p(y), _p(y_raw), _p(st), _p(cso))
    if rc != 0:
        raise ValueError("oracle_decode rejected its arguments")
    return {"y": y, "y_raw": y_raw, "state": st, "conv_state": cso}


# ---- the projections around the mixer ---------------------------------------------------------

def _wide(x: np.ndarray) -> np.ndarray:
    """Exact fp64 value of raw bf16 bits (uint16) or of fp32 values."""
    if x.dtype == np.uint16:
        return (np.ascontiguousarray(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def in_proj(x: np.ndarray, w_in: np.ndarray, h_qk: int, h_v: int, d_k: int = 128, d_v: int = 128):
    """Input projection ("Qwen3.8-Flash-Next" technical report, Fig. 2: the query, key and value
    streams -- and the gate inputs a, b and the output gate z -- are projections of the block
    input): every token's feature vector is W_in x_t, in fp64.  w_in [N_in, hidden] with rows
    q | k | v | z | a | b.  Returns dict(q [T,h_qk,d_k], k, v [T,h_v,d_v], z, a [T,h_v], b)."""
    X, W = _wide(x), _wide(w_in)
    F = X @ W.T
    T = X.shape[0]
    nq, nv = h_qk * d_k, h_v * d_v
    cuts = np.cumsum([0, nq, nq, nv, nv, h_v, h_v])
    if cuts[-1] != W.shape[0]:
        raise ValueError("w_in has the wrong number of rows")
    parts = [F[:, cuts[i]:cuts[i + 1]] for i in range(6)]
    return {"q": parts[0].reshape(T, h_qk, d_k), "k": parts[1].reshape(T, h_qk, d_k),
            "v": parts[2].reshape(T, h_v, d_v), "z": parts[3].reshape(T, h_v, d_v),
            "a": parts[4], "b": parts[5]}


def out_proj(y: np.ndarray, w_out: np.ndarray) -> np.ndarray:
    """Output projection (field guide §02: the gated, RMS-normalised output goes through the
    output projection): W_out y_t for every token, in fp64.  y [T, h_v, d_v] or [T, h_v d_v]."""
    Y = _wide(y)
    return Y.reshape(Y.shape[0], -1) @ _wide(w_out).T
