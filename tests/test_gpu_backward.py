"""GPU parity of the recurrence core's backward pass (gdn_recurrence_backward, fp32 CUDA cores)
against the fp64 reverse-mode oracle (itself pinned by finite differences), per (sequence,
value head), on packed sequences that cross chunk boundaries.

Bar: every gradient within 1e-4 of the oracle in relative Frobenius norm, and no element off by
more than 1e-3 of that gradient's largest magnitude."""
import numpy as np
import pytest
import torch

from gated_deltanet_token_b200 import gdn
from gated_deltanet_token_b200.inputs import make_bwd_inputs
from tests._helpers import to_dev

pytestmark = pytest.mark.gpu


def _oracle_grads(oracle_mod, inp, h_qk, h_v):
    cu = inp["cu_seqlens"]
    G = h_v // h_qk
    T = cu[-1]
    out = {"dq": np.zeros((T, h_qk, 128)), "dk": np.zeros((T, h_qk, 128)), "dv": np.zeros((T, h_v, 128)),
           "dg": np.zeros((T, h_v)), "dbeta": np.zeros((T, h_v)), "dS0": np.zeros((len(cu) - 1, h_v, 128, 128))}
    for n in range(len(cu) - 1):
        a, b = cu[n], cu[n + 1]
        for h in range(h_v):
            j = h // G
            r = oracle_mod.recurrence_backward(inp["qh"][a:b, j], inp["kh"][a:b, j], inp["v"][a:b, h],
                                               inp["g"][a:b, h], inp["beta"][a:b, h], inp["init_state"][n, h],
                                               inp["dy"][a:b, h], inp["dS_T"][n, h])
            out["dq"][a:b, j] += r["dq"]
            out["dk"][a:b, j] += r["dk"]
            out["dv"][a:b, h] = r["dv"]
            out["dg"][a:b, h] = r["dg"]
            out["dbeta"][a:b, h] = r["dbeta"]
            out["dS0"][n, h] = r["dS0"]
    return out


def _compare(got, ref, name):
    got = got.cpu().numpy().astype(np.float64)
    den = np.linalg.norm(ref)
    if den == 0:
        assert np.abs(got).max() == 0, name
        return
    rel = np.linalg.norm(got - ref) / den
    assert rel <= 1e-4, f"{name}: relative error {rel:.3e}"
    assert np.abs(got - ref).max() <= 1e-3 * np.abs(ref).max(), f"{name}: max error {np.abs(got - ref).max():.3e}"


@pytest.mark.parametrize("lengths,h_qk,h_v", [([1], 2, 4), ([64], 2, 4), ([65, 130], 2, 4), ([200], 1, 2),
                                               ([0, 70, 5, 129], 2, 4), ([256], 16, 32)])
def test_recurrence_backward_matches_oracle(oracle_mod, lengths, h_qk, h_v):
    inp = make_bwd_inputs(lengths, h_qk, h_v, seed=len(lengths) + h_v)
    ref = _oracle_grads(oracle_mod, inp, h_qk, h_v)
    t = {k: to_dev(inp[k]) for k in ("qh", "kh", "v", "g", "beta", "init_state", "dy", "dS_T")}
    cu = to_dev(inp["cu_seqlens"].astype(np.int32))
    dq, dk, dv, dg, dbeta, dS0 = gdn.gdn_recurrence_backward(t["qh"], t["kh"], t["v"], t["g"], t["beta"],
                                                             t["init_state"], cu, t["dy"], t["dS_T"])
    torch.cuda.synchronize()
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dg, "dg"), (dbeta, "dbeta"), (dS0, "dS0")):
        _compare(got, ref[name], name)


def test_recurrence_backward_null_state_and_final_gradient(oracle_mod):
    """init_state = NULL and dS_final = NULL read as zeros."""
    inp = make_bwd_inputs([70, 3], 2, 4, seed=11)
    inp["init_state"] = np.zeros_like(inp["init_state"])
    inp["dS_T"] = np.zeros_like(inp["dS_T"])
    ref = _oracle_grads(oracle_mod, inp, 2, 4)
    t = {k: to_dev(inp[k]) for k in ("qh", "kh", "v", "g", "beta", "dy")}
    cu = to_dev(inp["cu_seqlens"].astype(np.int32))
    dq, dk, dv, dg, dbeta, dS0 = gdn.gdn_recurrence_backward(t["qh"], t["kh"], t["v"], t["g"], t["beta"], None, cu,
                                                             t["dy"], None)
    torch.cuda.synchronize()
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dg, "dg"), (dbeta, "dbeta"), (dS0, "dS0")):
        _compare(got, ref[name], name)


def test_recurrence_backward_full_size_sampled_heads(oracle_mod):
    """The launch the benchmark times (one sequence, T = 4096, 16 QK / 32 value heads), compared
    on QK head 15 and its two value heads 30, 31: every gradient of those heads, dq and dk of
    the QK head (the sum over exactly those two value heads)."""
    T, h_qk, h_v = 4096, 16, 32
    inp = make_bwd_inputs([T], h_qk, h_v, seed=0)
    t = {k: to_dev(inp[k]) for k in ("qh", "kh", "v", "g", "beta", "init_state", "dy", "dS_T")}
    dq, dk, dv, dg, dbeta, dS0 = gdn.gdn_recurrence_backward(t["qh"], t["kh"], t["v"], t["g"], t["beta"],
                                                             t["init_state"], None, t["dy"], t["dS_T"])
    torch.cuda.synchronize()
    j = 15
    rdq = np.zeros((T, 128))
    rdk = np.zeros((T, 128))
    for h in (30, 31):
        r = oracle_mod.recurrence_backward(inp["qh"][:, j], inp["kh"][:, j], inp["v"][:, h], inp["g"][:, h],
                                           inp["beta"][:, h], inp["init_state"][0, h], inp["dy"][:, h],
                                           inp["dS_T"][0, h])
        rdq += r["dq"]
        rdk += r["dk"]
        _compare(dv[:, h], r["dv"], f"dv[{h}]")
        _compare(dg[:, h], r["dg"], f"dg[{h}]")
        _compare(dbeta[:, h], r["dbeta"], f"dbeta[{h}]")
        _compare(dS0[0, h], r["dS0"], f"dS0[{h}]")
    _compare(dq[:, j], rdq, "dq")
    _compare(dk[:, j], rdk, "dk")


def test_recurrence_backward_extreme_gates(oracle_mod):
    """alpha = e^g underflowing to 0 (g = -1000), beta at 0 and at 1, by value head."""
    inp = make_bwd_inputs([70, 130], 2, 4, seed=5)
    g = inp["g"].copy()
    beta = inp["beta"].copy()
    g[:, 0] = -1000.0
    beta[:, 1] = 0.0
    beta[:, 2] = 1.0
    g[::3, 3] = -1000.0
    inp = dict(inp)
    inp["g"], inp["beta"] = g.astype(np.float32), beta.astype(np.float32)
    ref = _oracle_grads(oracle_mod, inp, 2, 4)
    t = {k: to_dev(inp[k]) for k in ("qh", "kh", "v", "g", "beta", "init_state", "dy", "dS_T")}
    cu = to_dev(inp["cu_seqlens"].astype(np.int32))
    dq, dk, dv, dg, dbeta, dS0 = gdn.gdn_recurrence_backward(t["qh"], t["kh"], t["v"], t["g"], t["beta"],
                                                             t["init_state"], cu, t["dy"], t["dS_T"])
    torch.cuda.synchronize()
    for got, name in ((dq, "dq"), (dk, "dk"), (dv, "dv"), (dg, "dg"), (dbeta, "dbeta"), (dS0, "dS0")):
        _compare(got, ref[name], name)
