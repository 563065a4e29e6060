"""GPU parity of gdn_decode against the fp64 oracle (same tolerances as the prefill), plus
the bit-exact conv-history shift and the prefill -> decode hand-off."""
import numpy as np
import pytest
import torch

from gated_deltanet_token_b200.inputs import bf16_bits_to_f32, make_inputs
from tests._helpers import check_bf16, check_fp32, run_decode, run_prefill, to_dev

pytestmark = pytest.mark.gpu


def test_decode_N256_bf16(oracle_mod):
    inp = make_inputs("decode_N256_bf16")
    ref = oracle_mod.decode(inp)
    y, S, cs = run_decode(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["state"])
    assert cs.dtype == np.uint16  # the raw bf16 history, shifted by one token, bit-exact
    assert np.array_equal(bf16_bits_to_f32(cs).astype(np.float64), ref["conv_state"])
    yb, Sb, _ = run_decode(inp, torch.bfloat16)
    check_bf16(yb, ref["y"], Sb, ref["state"], y_is_bf16=True)


def test_decode_fp32_small(oracle_mod):
    inp = make_inputs("decode_N256_bf16", n_seqs=5, h_qk=2, h_v=4, dtype="f32")
    ref = oracle_mod.decode(inp)
    y, S, cs = run_decode(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["state"])
    assert np.array_equal(cs.astype(np.float64), ref["conv_state"])


@pytest.mark.parametrize("ratio", [1, 4, 8])
def test_decode_head_ratios(oracle_mod, ratio):
    inp = make_inputs("decode_N256_bf16", n_seqs=3, h_qk=2, h_v=2 * ratio, dtype="f32")
    ref = oracle_mod.decode(inp)
    y, S, _ = run_decode(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["state"])


def test_prefill_then_decode_matches_longer_prefill(oracle_mod):
    T = 70
    full = make_inputs("tiny_prefill_fp32", T=T + 1)
    head = dict(full)
    for n in ("q", "k", "v", "z", "a", "b"):
        head[n] = full[n][:T]
    _, S_T = run_prefill(head, torch.float32)
    dec = dict(full)
    for n in ("q", "k", "v", "z", "a", "b"):
        dec[n] = full[n][T:T + 1]
    dec["state"] = S_T.astype(np.float32)
    dec["conv_state"] = np.ascontiguousarray(np.concatenate(
        [full["q"][T - 3:T].reshape(3, -1), full["k"][T - 3:T].reshape(3, -1),
         full["v"][T - 3:T].reshape(3, -1)], axis=1)[None])
    y, S, _ = run_decode(dec, torch.float32)
    ref = oracle_mod.prefill(full)
    assert np.abs(y[0] - ref["y"][T]).max() <= 1e-4
    assert np.linalg.norm(S[0] - ref["final_state"][0]) / np.linalg.norm(ref["final_state"][0]) <= 1e-4


def test_decode_norm_weights(oracle_mod):
    """A non-trivial norm_w (every component different) through the decode step's output norm."""
    inp = make_inputs("decode_N256_bf16", n_seqs=7, h_qk=2, h_v=4, dtype="f32")
    inp["norm_w"] = np.random.default_rng(6).uniform(0.5, 1.5, inp["norm_w"].shape).astype(np.float32)
    ref = oracle_mod.decode(inp)
    y, S, _ = run_decode(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["state"])


# ---- prefill -> decode hand-off on resident pools ---------------------------------------

def _raw_history(inp, ts, te):
    """Rows x_{te-3..te-1} of the raw q | k | v channels, zeros before token ts (numpy)."""
    q, k, v = inp["q"], inp["k"], inp["v"]
    width = q.shape[1] * q.shape[2] * 2 + v.shape[1] * v.shape[2]
    rows = np.zeros((3, width), dtype=q.dtype)
    for r in range(3):
        t = te - 3 + r
        if t >= ts:
            rows[r] = np.concatenate([q[t].ravel(), k[t].ravel(), v[t].ravel()])
    return rows


def _as_np(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.cpu().numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_prefill_conv_state_is_the_raw_history(dtype):
    from gated_deltanet_token_b200 import gdn

    lens = [0, 1, 2, 3, 70, 130]
    inp = make_inputs("varlen8_prefill_bf16", lengths=lens, h_qk=2, h_v=4, dtype=dtype)
    cu = inp["cu_seqlens"]
    cs = gdn.gdn_prefill_conv_state(to_dev(inp["q"]), to_dev(inp["k"]), to_dev(inp["v"]),
                                    to_dev(cu.astype(np.int32)))
    torch.cuda.synchronize()
    got = _as_np(cs)
    for n in range(len(lens)):
        assert np.array_equal(got[n], _raw_history(inp, int(cu[n]), int(cu[n + 1])))  # bit-exact


def test_handoff_prefill_to_decode_slots(oracle_mod):
    """Prefill the first L_n tokens of each sequence, hand the final states and conv histories to
    pool slots (scattered, with spare slots), decode token L_n + 1 of each sequence plus one
    padding entry through gdn_decode_slots, and compare with the oracle's prefill over L_n + 1
    tokens: y of the last token and the state.  Spare slots and the padding row stay as they
    were; each used slot's conv history is the raw history shifted by the new token."""
    from gated_deltanet_token_b200 import gdn

    L = [70, 3, 1, 0, 130]
    N = len(L)
    full = make_inputs("varlen8_prefill_bf16", lengths=[n + 1 for n in L], h_qk=2, h_v=4, seed=3)
    cf = full["cu_seqlens"]
    head = dict(full)
    for nm in ("q", "k", "v", "z", "a", "b"):
        head[nm] = np.ascontiguousarray(np.concatenate([full[nm][cf[n]:cf[n] + L[n]] for n in range(N)]))
    ch = np.zeros(N + 1, np.int32)
    ch[1:] = np.cumsum(L)
    head["cu_seqlens"] = ch
    d = {nm: to_dev(head[nm]) for nm in ("q", "k", "v", "z", "a", "b")}
    par = {nm: to_dev(full[nm]) for nm in ("A_log", "dt_bias", "conv_w", "norm_w")}
    cu_d = to_dev(ch)
    _, fs = gdn.gdn_prefill(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], par["A_log"], par["dt_bias"],
                            par["conv_w"], par["norm_w"], to_dev(full["init_state"]), cu_d,
                            out_dtype=torch.float32)
    cs = gdn.gdn_prefill_conv_state(d["q"], d["k"], d["v"], cu_d)

    n_slots, perm = N + 2, [4, 0, 6, 2, 1]
    g = torch.Generator(device="cuda").manual_seed(7)
    state_pool = torch.randn((n_slots,) + tuple(fs.shape[1:]), generator=g, device="cuda")
    conv_pool = torch.randn((n_slots,) + tuple(cs.shape[1:]), generator=g, device="cuda").to(cs.dtype)
    for n, sl in enumerate(perm):
        state_pool[sl].copy_(fs[n])
        conv_pool[sl].copy_(cs[n])
    spare = [s for s in range(n_slots) if s not in perm]
    spare_state, spare_conv = state_pool[spare].clone(), conv_pool[spare].clone()

    last = [int(cf[n + 1]) - 1 for n in range(N)] + [int(cf[1]) - 1]  # + one padding entry
    dec = {nm: to_dev(np.ascontiguousarray(full[nm][last])) for nm in ("q", "k", "v", "z", "a", "b")}
    ids = to_dev(np.array(perm + [-1], np.int32))
    y = torch.full((N + 1, 4, 128), float("nan"), device="cuda")
    gdn.gdn_decode_slots(dec["q"], dec["k"], dec["v"], dec["z"], dec["a"], dec["b"], par["A_log"],
                         par["dt_bias"], par["conv_w"], par["norm_w"], conv_pool, state_pool, ids,
                         out_dtype=torch.float32, y=y)
    torch.cuda.synchronize()
    assert gdn.gdn_read_device_status() == 0

    ref = oracle_mod.prefill(full)
    yy = y.cpu().numpy().astype(np.float64)
    S = state_pool.cpu().numpy().astype(np.float64)
    check_bf16(yy[:N], ref["y"][last[:N]], S[perm], ref["final_state"])
    assert np.isnan(yy[N]).all()  # the padding entry wrote nothing
    assert torch.equal(state_pool[spare], spare_state) and torch.equal(conv_pool[spare], spare_conv)
    got = _as_np(conv_pool)
    for n, sl in enumerate(perm):  # the history now ends with the decoded token, bit-exact
        assert np.array_equal(got[sl], _raw_history(full, int(cf[n]), int(cf[n + 1])))


def test_decode_slot_past_the_pool_sets_the_index_status():
    from gated_deltanet_token_b200 import gdn

    inp = make_inputs("decode_N256_bf16", n_seqs=2, h_qk=2, h_v=4)
    dd = {nm: to_dev(inp[nm]) for nm in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w",
                                          "norm_w", "conv_state", "state")}
    ref_state, ref_conv = dd["state"].clone(), dd["conv_state"].clone()
    y_ref = gdn.gdn_decode(dd["q"], dd["k"], dd["v"], dd["z"], dd["a"], dd["b"], dd["A_log"], dd["dt_bias"],
                           dd["conv_w"], dd["norm_w"], ref_conv, ref_state, out_dtype=torch.float32)
    y = torch.full((2, 4, 128), float("nan"), device="cuda")
    gdn.gdn_decode_slots(dd["q"], dd["k"], dd["v"], dd["z"], dd["a"], dd["b"], dd["A_log"], dd["dt_bias"],
                         dd["conv_w"], dd["norm_w"], dd["conv_state"], dd["state"],
                         to_dev(np.array([0, 2], np.int32)), out_dtype=torch.float32, y=y)
    assert gdn.gdn_read_device_status() == gdn.GDN_ERR_INDEX
    assert gdn.gdn_read_device_status() == 0  # read clears it
    assert torch.equal(y[0], y_ref[0]) and torch.isnan(y[1]).all()
    assert torch.equal(dd["state"][0], ref_state[0])  # entry 0 ran; slot 1 was left alone
    assert torch.equal(dd["state"][1], torch.from_numpy(inp["state"][1]).cuda())


# ---- several decode tokens per sequence in one call ---------------------------------------

def bf16_from_f64(x):
    """Bits of fp64 values that are exact bf16 numbers (raw history rows), as uint16."""
    return (np.ascontiguousarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _multi_inputs(K, N=3, dtype="bf16", seed=11, h_qk=2, h_v=4):
    """K consecutive decode tokens per sequence: the per-token fields of K seeded one-token
    workloads stacked on axis 1; state, conv history and parameters from the first."""
    steps = [make_inputs("decode_N256_bf16", seed=seed + i, n_seqs=N, h_qk=h_qk, h_v=h_v, dtype=dtype)
             for i in range(K)]
    out = dict(steps[0])
    for nm in ("q", "k", "v", "z", "a", "b"):
        out[nm] = np.ascontiguousarray(np.stack([s_[nm] for s_ in steps], axis=1))
    return out


def _run_multi(inp, out_dtype=torch.float32):
    from gated_deltanet_token_b200 import gdn

    d = {nm: to_dev(inp[nm]) for nm in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w", "norm_w",
                                        "conv_state", "state")}
    y = gdn.gdn_decode_multi(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                             d["conv_w"], d["norm_w"], d["conv_state"], d["state"], out_dtype=out_dtype)
    torch.cuda.synchronize()
    return y, d["state"], d["conv_state"]


def test_decode_multi_one_token_equals_decode():
    from gated_deltanet_token_b200 import gdn

    inp = _multi_inputs(1)
    y_m, S_m, cs_m = _run_multi(inp)
    one = dict(inp)
    for nm in ("q", "k", "v", "z", "a", "b"):
        one[nm] = np.ascontiguousarray(inp[nm][:, 0])
    d = {nm: to_dev(one[nm]) for nm in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w", "norm_w",
                                        "conv_state", "state")}
    y_1 = gdn.gdn_decode(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"], d["conv_w"],
                         d["norm_w"], d["conv_state"], d["state"], out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y_m[:, 0], y_1) and torch.equal(S_m, d["state"]) and torch.equal(cs_m, d["conv_state"])


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("K", [2, 3, 4, 5, 8])
def test_decode_multi_equals_successive_steps(oracle_mod, K, dtype):
    _check_multi(oracle_mod, _multi_inputs(K, dtype=dtype), K, dtype)


@pytest.mark.parametrize("h_qk,h_v", [(2, 2), (2, 8), (1, 8), (16, 32)])
def test_decode_multi_head_ratios(oracle_mod, h_qk, h_v):
    """Every value-head ratio the row partition of the multi-token kernel handles (1, 4, 8 and
    the model's 2), four tokens per sequence."""
    _check_multi(oracle_mod, _multi_inputs(4, N=2, h_qk=h_qk, h_v=h_v), 4, "bf16")


def _check_multi(oracle_mod, inp, K, dtype):
    y, S, cs = _run_multi(inp)
    state = inp["state"].astype(np.float32)
    hist = inp["conv_state"]
    ys = []
    for t in range(K):  # the oracle, one token at a time, carrying the state and the history
        step = dict(inp)
        for nm in ("q", "k", "v", "z", "a", "b"):
            step[nm] = np.ascontiguousarray(inp[nm][:, t])
        step["state"], step["conv_state"] = state, hist
        o = oracle_mod.decode(step)
        ys.append(o["y"])
        state = o["state"].astype(np.float32)
        hist = (bf16_from_f64(o["conv_state"]) if dtype == "bf16" else o["conv_state"].astype(np.float32))
    y_ref = np.stack(ys, axis=1)
    yy = y.cpu().numpy().astype(np.float64)
    SS = S.cpu().numpy().astype(np.float64)
    if dtype == "bf16":
        check_bf16(yy, y_ref, SS, o["state"])
    else:
        check_fp32(yy, y_ref, SS, o["state"])
    got = cs.view(torch.int16).cpu().numpy().view(np.uint16) if cs.dtype == torch.bfloat16 else cs.cpu().numpy()
    exp = bf16_from_f64(o["conv_state"]) if dtype == "bf16" else o["conv_state"].astype(np.float32)
    assert np.array_equal(got, exp)  # the raw history, bit-exact



def _extreme_decode_gates(inp):
    """Gates at the ends of their ranges, by value-head group: A_log = log 1e6 (e^g underflows
    to 0), b = +30 (beta = 1), b = -30 (beta ~ 1e-13), and a = +20 on the last group."""
    h_v = inp["A_log"].shape[0]
    q4 = max(1, h_v // 4)
    out = dict(inp)
    A_log = inp["A_log"].copy()
    A_log[:q4] = np.log(1e6)
    a = inp["a"].copy()
    b = inp["b"].copy()
    b[..., q4:2 * q4] = 30.0
    b[..., 2 * q4:3 * q4] = -30.0
    a[..., 3 * q4:] = 20.0
    out["A_log"], out["a"], out["b"] = A_log.astype(np.float32), a.astype(np.float32), b.astype(np.float32)
    return out


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_decode_multi_extreme_gates(oracle_mod, dtype):
    """The multi-token decode with the decay underflowing to zero, beta at 0 and 1 and a strong
    single-token decay, against the oracle's successive steps (the one-token decode is the same
    kernel at K = 1)."""
    _check_multi(oracle_mod, _extreme_decode_gates(_multi_inputs(4, N=3, dtype=dtype, h_qk=2, h_v=8)), 4, dtype)
