"""Seeded synthetic inputs for the GDN token-mixer workloads.

This module only draws random numbers and lays them out; it holds none of the mixer's
arithmetic.  The same bytes feed the CUDA library and the fp64 oracle.

Recipe (one ``numpy.random.default_rng(seed)`` PCG64 stream per workload, drawn in this
order): sequence lengths (varlen only), conv_w, A_log, dt_bias, q, k, v, z, a, b,
init_state / resident state, conv_state.
  q, k, v, z ~ N(0, 1)           (rounded to bf16, round-to-nearest-even, when bf16)
  a, b       ~ N(0, 1) fp32
  A_log      = log U(1, 16)      [h_v]
  dt_bias    ~ N(0, 0.1^2)       [h_v]
  conv_w     ~ U(-0.5, 0.5)      [C_conv, 4], channel order q | k | v
  norm_w     = 1                 [d_v]   (not drawn)
  states     ~ N(0, 0.02^2) fp32 where the workload has a nonzero state
  conv_state ~ N(0, 1)           [N, 3, C_conv] in the input dtype (decode only)
Normal draws are made in fp32 in blocks of at most ``_BLOCK`` values so that very long
sequences never need an fp64 copy.

bf16 tensors are returned as ``uint16`` arrays of raw bf16 bits.
"""
from __future__ import annotations

import numpy as np

_BLOCK = 1 << 24

# The workloads: the sizes, head shapes, dtypes and distributions of the mixer in the
# pages (16 QK heads shared by 32 value heads, head width 128, width-4 conv).
WORKLOADS = {
    "tiny_prefill_fp32": dict(kind="prefill", n_seqs=1, T=128, h_qk=2, h_v=4, d=128,
                              dtype="f32", init_state=False),
    "prefill_T4096_bf16": dict(kind="prefill", n_seqs=1, T=4096, h_qk=16, h_v=32, d=128,
                               dtype="bf16", init_state=False),
    "varlen8_prefill_bf16": dict(kind="prefill", n_seqs=8, lengths=(512, 8192), h_qk=16, h_v=32,
                                 d=128, dtype="bf16", init_state=True),
    "long_prefill_T262144_bf16": dict(kind="prefill", n_seqs=1, T=262144, h_qk=16, h_v=32, d=128,
                                      dtype="bf16", init_state=False),
    "decode_N256_bf16": dict(kind="decode", n_seqs=256, h_qk=16, h_v=32, d=128, dtype="bf16"),
}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 (round to nearest, ties to even); return the raw bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of raw bf16 bits to fp32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng, shape, dtype: str, scale: float = 1.0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, np.uint16 if dtype == "bf16" else np.float32)
    for s in range(0, n, _BLOCK):
        e = min(n, s + _BLOCK)
        blk = rng.standard_normal(e - s, dtype=np.float32)
        if scale != 1.0:
            blk *= np.float32(scale)
        out[s:e] = to_bf16_bits(blk) if dtype == "bf16" else blk
    return out.reshape(shape)


def make_inputs(name: str, seed: int = 0, **over) -> dict:
    """Generate one workload's inputs.

    ``over`` may replace any field of the workload spec (e.g. T=200 for a short run of
    the same shapes and distributions, or lengths=[3, 0, 70] -- a list -- for explicit
    varlen lengths; a (lo, hi) tuple draws n_seqs lengths uniformly from lo..hi).
    Returns a dict of numpy arrays plus ``spec`` (the effective spec).
    """
    spec = dict(WORKLOADS[name])
    spec.update(over)
    rng = np.random.default_rng(seed)
    hq, hv, d, dt = spec["h_qk"], spec["h_v"], spec["d"], spec["dtype"]
    cconv = 2 * hq * d + hv * d
    out: dict = {"spec": spec}
    if spec["kind"] == "prefill":
        if "lengths" in spec and spec["lengths"] is not None:
            L = spec["lengths"]
            if isinstance(L, tuple):  # (lo, hi): uniform integer lengths, both ends inclusive
                lens = rng.integers(L[0], L[1], size=spec["n_seqs"], endpoint=True)
            else:
                lens = np.asarray(L, dtype=np.int64)
            cu = np.zeros(len(lens) + 1, np.int32)
            cu[1:] = np.cumsum(lens)
            out["cu_seqlens"] = cu
            T = int(cu[-1])
            n_seqs = len(lens)
        else:
            T = spec["T"]
            n_seqs = spec["n_seqs"]
            out["cu_seqlens"] = None
        spec["T"] = T
        spec["n_seqs"] = n_seqs
        rows = T
    else:
        n_seqs = spec["n_seqs"]
        rows = n_seqs
    out["conv_w"] = rng.uniform(-0.5, 0.5, size=(cconv, 4)).astype(np.float32)
    out["A_log"] = np.log(rng.uniform(1.0, 16.0, size=hv)).astype(np.float32)
    out["dt_bias"] = (rng.standard_normal(hv) * 0.1).astype(np.float32)
    out["norm_w"] = np.ones(d, np.float32)
    out["q"] = _normal(rng, (rows, hq, d), dt)
    out["k"] = _normal(rng, (rows, hq, d), dt)
    out["v"] = _normal(rng, (rows, hv, d), dt)
    out["z"] = _normal(rng, (rows, hv, d), dt)
    out["a"] = _normal(rng, (rows, hv), "f32")
    out["b"] = _normal(rng, (rows, hv), "f32")
    if spec["kind"] == "prefill":
        out["init_state"] = (_normal(rng, (n_seqs, hv, d, d), "f32", 0.02)
                             if spec.get("init_state") else None)
    else:
        out["state"] = _normal(rng, (n_seqs, hv, d, d), "f32", 0.02)
        out["conv_state"] = _normal(rng, (n_seqs, 3, cconv), dt)
    return out


def make_proj_inputs(T: int, hidden: int = 2048, h_qk: int = 16, h_v: int = 32, d: int = 128,
                     seed: int = 0) -> dict:
    """Synthetic inputs of the projections around the mixer (the pages print no weights):
    x ~ N(0, 1) [T, hidden], W_in ~ N(0, 1/hidden) [2 h_qk d + 2 h_v d + 2 h_v, hidden],
    W_out ~ N(0, 1/(h_v d)) [hidden, h_v d] and a mixer output y ~ N(0, 1) [T, h_v, d], all bf16
    (raw bits, round to nearest even), drawn in that order from one PCG64 stream."""
    rng = np.random.default_rng(seed)
    n_in = 2 * h_qk * d + 2 * h_v * d + 2 * h_v
    return {"x": _normal(rng, (T, hidden), "bf16"),
            "w_in": _normal(rng, (n_in, hidden), "bf16", float(hidden) ** -0.5),
            "w_out": _normal(rng, (hidden, h_v * d), "bf16", float(h_v * d) ** -0.5),
            "y": _normal(rng, (T, h_v, d), "bf16")}


def make_bwd_inputs(lengths, h_qk: int = 2, h_v: int = 4, d: int = 128, seed: int = 0) -> dict:
    """Synthetic inputs of the recurrence core's backward pass (fp32): unit query and key
    vectors qh, kh [T, h_qk, d]; v ~ N(0, 1) [T, h_v, d]; the decay g = -exp(A_log) softplus(a +
    dt_bias) with the configs' distributions and beta = sigmoid(b), both [T, h_v]; initial states
    ~ N(0, 0.02^2) [N, h_v, d, d]; upstream gradients dy ~ N(0, 1) [T, h_v, d] and dS_T ~ N(0,
    0.02^2).  `lengths` is a list of sequence lengths (packed, cu_seqlens returned)."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(lengths, dtype=np.int64)
    cu = np.zeros(len(lens) + 1, np.int32)
    cu[1:] = np.cumsum(lens)
    T, N = int(cu[-1]), len(lens)
    qh = rng.standard_normal((T, h_qk, d)).astype(np.float32)
    kh = rng.standard_normal((T, h_qk, d)).astype(np.float32)
    qh /= np.maximum(np.linalg.norm(qh, axis=2, keepdims=True), 1e-6)
    kh /= np.maximum(np.linalg.norm(kh, axis=2, keepdims=True), 1e-6)
    v = rng.standard_normal((T, h_v, d)).astype(np.float32)
    A_log = np.log(rng.uniform(1.0, 16.0, size=h_v))
    dt_bias = rng.standard_normal(h_v) * 0.1
    a = rng.standard_normal((T, h_v))
    x = a + dt_bias
    g = (-np.exp(A_log) * (np.maximum(x, 0) + np.log1p(np.exp(-np.abs(x))))).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((T, h_v))))).astype(np.float32)
    return {"qh": qh, "kh": kh, "v": v, "g": g, "beta": beta, "cu_seqlens": cu,
            "init_state": (rng.standard_normal((N, h_v, d, d)) * 0.02).astype(np.float32),
            "dy": rng.standard_normal((T, h_v, d)).astype(np.float32),
            "dS_T": (rng.standard_normal((N, h_v, d, d)) * 0.02).astype(np.float32)}
