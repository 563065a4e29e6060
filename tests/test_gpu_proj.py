"""GPU parity of the projections around the mixer (gdn_in_proj, gdn_out_proj: tcgen05 GEMMs
with bf16 operands and fp32 accumulation) against the fp64 oracle's matrix products, and of
the whole block path in_proj -> prefill -> out_proj.

Tolerances: a bf16 output is compared with the fp64 product per element within half a bf16 ulp
of the reference (2^-8 |ref|, its rounding) plus 1e-5 RMS(ref) for the fp32 accumulation over
`hidden` terms; an fp32 output (a, b) within 1e-5 RMS(ref) + 1e-6 |ref|."""
import numpy as np
import pytest
import torch

from gated_deltanet_token_b200 import gdn
from gated_deltanet_token_b200.inputs import make_inputs, make_proj_inputs
from tests._helpers import check_bf16, to_dev

pytestmark = pytest.mark.gpu


def _host(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def _check(got, ref, bf16):
    r = float(np.sqrt(np.mean(ref * ref))) if ref.size else 0.0
    bound = (2.0 ** -8 * np.abs(ref) + 1e-5 * r) if bf16 else (1e-6 * np.abs(ref) + 1e-5 * r)
    worst = float((np.abs(got - ref) - bound).max()) if ref.size else -1.0
    assert worst <= 0, f"max |err| = {np.abs(got - ref).max():.3e} (RMS(ref) = {r:.3f})"


@pytest.mark.parametrize("T,hidden,h_qk,h_v", [(1, 2048, 16, 32), (77, 2048, 16, 32), (4096, 2048, 16, 32),
                                               (130, 128, 2, 4), (300, 192, 1, 3)])
def test_in_proj_matches_oracle(oracle_mod, T, hidden, h_qk, h_v):
    p = make_proj_inputs(T, hidden, h_qk, h_v)
    ref = oracle_mod.in_proj(p["x"], p["w_in"], h_qk, h_v)
    outs = gdn.gdn_in_proj(to_dev(p["x"]), to_dev(p["w_in"]), h_qk, h_v)
    torch.cuda.synchronize()
    for name, t in zip(("q", "k", "v", "z", "a", "b"), outs):
        _check(_host(t), ref[name], t.dtype == torch.bfloat16)


@pytest.mark.parametrize("T,hidden,h_v", [(1, 2048, 32), (200, 2048, 32), (4096, 2048, 32), (65, 96, 2)])
def test_out_proj_matches_oracle(oracle_mod, T, hidden, h_v):
    p = make_proj_inputs(T, hidden, max(1, h_v // 2), h_v)
    ref = oracle_mod.out_proj(p["y"], p["w_out"])
    out = gdn.gdn_out_proj(to_dev(p["y"]), to_dev(p["w_out"]), max(1, h_v // 2), h_v)
    torch.cuda.synchronize()
    _check(_host(out), ref, True)


def test_projection_rejects_bad_arguments():
    x = torch.zeros((4, 100), dtype=torch.bfloat16, device="cuda")  # hidden not a multiple of 64
    w = torch.zeros((2 * 128 + 2 * 256 + 4, 100), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(gdn.GdnError) as ei:
        gdn.gdn_in_proj(x, w, 1, 2)
    assert ei.value.code == -2


def _bits(t):
    """Raw bf16 bits of a bf16 device tensor, as the oracle takes them."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_block_path_in_proj_prefill_out_proj(oracle_mod):
    """x -> in_proj -> prefill (bf16 y) -> out_proj, each stage against the oracle on the inputs
    that stage actually received: the bf16 rounding of q, k, v, z (and of y) is a decision taken
    on an fp32 accumulation on the GPU and on an fp64 one in the oracle, so values at a rounding
    tie may differ by one ulp; the stage's own bar then applies to what follows."""
    T, hidden, h_qk, h_v = 300, 2048, 16, 32
    p = make_proj_inputs(T, hidden, h_qk, h_v, seed=4)
    base = make_inputs("prefill_T4096_bf16", T=T)  # conv taps, gate parameters, norm weights
    q, k, v, z, a, b = gdn.gdn_in_proj(to_dev(p["x"]), to_dev(p["w_in"]), h_qk, h_v)
    prm = {nm: to_dev(base[nm]) for nm in ("A_log", "dt_bias", "conv_w", "norm_w")}
    y, S = gdn.gdn_prefill(q, k, v, z, a, b, prm["A_log"], prm["dt_bias"], prm["conv_w"], prm["norm_w"], None, None,
                           out_dtype=torch.bfloat16)
    out = gdn.gdn_out_proj(y, to_dev(p["w_out"]), h_qk, h_v)
    torch.cuda.synchronize()
    ref = oracle_mod.in_proj(p["x"], p["w_in"], h_qk, h_v)
    for name, t in zip(("q", "k", "v", "z", "a", "b"), (q, k, v, z, a, b)):
        _check(_host(t), ref[name], t.dtype == torch.bfloat16)
    inp = dict(base)
    for nm, t in zip(("q", "k", "v", "z"), (q, k, v, z)):
        inp[nm] = _bits(t)
    inp["a"], inp["b"] = a.cpu().numpy(), b.cpu().numpy()
    mix = oracle_mod.prefill(inp)
    check_bf16(_host(y), mix["y"], S.cpu().numpy().astype(np.float64), mix["final_state"], y_is_bf16=True)
    _check(_host(out), oracle_mod.out_proj(_bits(y), p["w_out"]), True)
