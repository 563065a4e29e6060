"""Shared helpers of the GPU tests: move generated inputs to the device, run the library,
run the oracle, and compute the parity metrics (max-abs error on y against RMS(y_ref),
relative Frobenius error of the states)."""
from __future__ import annotations

import contextlib

import numpy as np
import torch


@contextlib.contextmanager
def path_options(flags):
    """Run the body with the library's path options set to `flags` (gdn_set_options), then
    restore the previous word."""
    from gated_deltanet_token_b200 import gdn

    prev = gdn.gdn_set_options(flags)
    try:
        yield
    finally:
        gdn.gdn_set_options(prev)


def to_dev(x, device="cuda"):
    if x is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(x))
    if x.dtype == np.uint16:
        t = t.view(torch.bfloat16)
    return t.to(device)


def run_prefill(inp, out_dtype=torch.float32, init_alias=False, **kw):
    """Run gdn_prefill on generated inputs (numpy) through the binding; returns fp64 numpy
    (y, final_state).  Extra keyword arguments go to gdn_prefill (e.g. workspace, q_scale)."""
    from gated_deltanet_token_b200 import gdn

    d = {n: to_dev(inp.get(n)) for n in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w",
                                         "norm_w", "init_state")}
    cu = inp.get("cu_seqlens")
    cu_t = None if cu is None else to_dev(cu.astype(np.int32))
    final = d["init_state"] if init_alias else None
    y, fs = gdn.gdn_prefill(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                            d["conv_w"], d["norm_w"], d["init_state"], cu_t, out_dtype=out_dtype,
                            final_state=final, **kw)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64), fs.cpu().numpy().astype(np.float64)


def run_decode(inp, out_dtype=torch.float32):
    from gated_deltanet_token_b200 import gdn

    d = {n: to_dev(inp.get(n)) for n in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w",
                                         "norm_w", "conv_state", "state")}
    y = gdn.gdn_decode(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                       d["conv_w"], d["norm_w"], d["conv_state"], d["state"], out_dtype=out_dtype)
    torch.cuda.synchronize()
    cs = d["conv_state"]
    cs_np = cs.view(torch.int16).cpu().numpy().view(np.uint16) if cs.dtype == torch.bfloat16 else cs.cpu().numpy()
    return (y.float().cpu().numpy().astype(np.float64), d["state"].cpu().numpy().astype(np.float64), cs_np)


def e_y(y, y_ref):
    return float(np.abs(y - y_ref).max()) if y.size else 0.0


def rms(x):
    return float(np.sqrt(np.mean(x * x))) if x.size else 0.0


def e_S(S, S_ref):
    den = np.linalg.norm(S_ref)
    return float(np.linalg.norm(S - S_ref) / den) if den > 0 else float(np.linalg.norm(S - S_ref))


def check_fp32(y, y_ref, S, S_ref, tol=1e-4):
    ey, es = e_y(y, y_ref), e_S(S, S_ref)
    assert ey <= tol, f"e_y = {ey:.3e} > {tol}"
    assert es <= tol, f"e_S = {es:.3e} > {tol}"
    return ey, es


def check_bf16(y, y_ref, S, S_ref, y_is_bf16=False):
    """bf16-input runs: e_y <= 2e-2 RMS(y_ref) and e_S <= 1e-2.  A bf16 y additionally gets
    half a bf16 ulp of y_ref per element (2^-8 |y_ref|), the rounding of the final store."""
    r = rms(y_ref)
    err = np.abs(y - y_ref)
    bound = 2e-2 * r + (2.0 ** -8) * np.abs(y_ref) if y_is_bf16 else 2e-2 * r
    worst = float((err - bound).max()) if y.size else -1.0
    es = e_S(S, S_ref)
    assert worst <= 0, f"e_y = {e_y(y, y_ref):.3e} exceeds its bound (RMS(y_ref) = {r:.3f})"
    assert es <= 1e-2, f"e_S = {es:.3e} > 1e-2"
    return e_y(y, y_ref) / max(r, 1e-30), es
