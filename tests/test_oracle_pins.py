"""Pins for the fp64 oracle, checked against what the pages and the mathematics fix.

None of these retypes the oracle's own formula: each compares it with a library routine
(numpy.convolve, numpy.logaddexp, scipy.special.expit, numpy.linalg), a closed form the
definitions imply, an invariant, or brute force on tiny inputs.

References: "Qwen3-Next 80B-A3B" field guide, §02 "Gated DeltaNet state update" (the six
update steps, head counts, column-vector convention, RMSNorm * SiLU(z) output);
"Qwen3.8-Flash-Next" technical report, Fig. 2 (conv on q, k, v; L2-normalised q, k;
decay and write gates); "Qwen3.8-Flash-Next" model notes (decay gate; chunk-loop
state update).
"""
import numpy as np
import pytest
from scipy.special import expit

from gated_deltanet_token_b200.inputs import bf16_bits_to_f32, make_inputs

RTOL = 1e-12


def unit_rows(rng, n, d):
    x = rng.standard_normal((n, d))
    return x / np.linalg.norm(x, axis=1, keepdims=True)


def rel(a, b):
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ---- scalar functions and stages against library routines ------------------------------

def test_softplus_sigmoid_silu_match_library(oracle_mod):
    xs = np.concatenate([np.linspace(-60, 60, 241), [-700.0, -30.5, 0.0, 1e-9, 30.5, 700.0]])
    for x in xs:
        assert oracle_mod.softplus(x) == pytest.approx(np.logaddexp(0.0, x), rel=1e-14, abs=1e-300)
        assert oracle_mod.sigmoid(x) == pytest.approx(expit(x), rel=1e-14, abs=1e-300)
        assert oracle_mod.silu(x) == pytest.approx(x * expit(x), rel=1e-14, abs=1e-300)


def test_decay_gate_special_values(oracle_mod):
    # softplus(0) = ln 2, so a + dt_bias = 0 gives g = -exp(A_log) ln 2
    for A_log in (0.0, np.log(3.0), np.log(16.0)):
        assert oracle_mod.decay_gate(0.3, A_log, -0.3) == pytest.approx(-np.exp(A_log) * np.log(2.0),
                                                                      rel=1e-14)
    # very negative pre-activation: softplus(x) -> e^x, so g -> -exp(A_log) e^x
    assert oracle_mod.decay_gate(-40.0, np.log(2.0), 0.0) == pytest.approx(-2.0 * np.exp(-40.0),
                                                                          rel=1e-12)
    # very positive: softplus(x) -> x
    assert oracle_mod.decay_gate(50.0, np.log(5.0), 1.0) == pytest.approx(-5.0 * 51.0, rel=1e-14)
    # g <= 0 and monotone non-increasing in a
    gs = [oracle_mod.decay_gate(a, 0.7, 0.05) for a in np.linspace(-10, 10, 101)]
    assert max(gs) < 0 and np.all(np.diff(gs) <= 0)


def test_conv_silu_matches_numpy_convolve(oracle_mod):
    rng = np.random.default_rng(1)
    for T in (1, 2, 3, 4, 7, 50):
        x = rng.standard_normal(T)
        w = rng.uniform(-0.5, 0.5, 4)
        pre = np.convolve(x, w[::-1])[:T]  # causal cross-correlation, zero history
        assert rel(oracle_mod.conv_silu(x, w), pre * expit(pre)) < RTOL
        hist = rng.standard_normal(3)
        pre_h = np.convolve(np.concatenate([hist, x]), w[::-1])[3:3 + T]
        assert rel(oracle_mod.conv_silu(x, w, hist), pre_h * expit(pre_h)) < RTOL


def test_conv_tap_order(oracle_mod):
    # tap 3 is the current token: a unit impulse at t=0 shows the taps in reverse time order
    x = np.array([1.0, 0.0, 0.0, 0.0, 0.0])
    w = np.array([0.1, 0.2, 0.3, 0.4])
    pre = np.array([0.4, 0.3, 0.2, 0.1, 0.0])
    assert rel(oracle_mod.conv_silu(x, w), pre * expit(pre)) < RTOL


def test_l2norm_matches_numpy_norm(oracle_mod):
    rng = np.random.default_rng(2)
    x = rng.standard_normal(128) * 3.0
    out = oracle_mod.l2norm(x, 1e-6)
    assert rel(out, x / np.sqrt(np.linalg.norm(x) ** 2 + 1e-6)) < RTOL
    assert abs(np.linalg.norm(oracle_mod.l2norm(x * 1e4, 0.0)) - 1.0) < 1e-14


def test_gated_rmsnorm_invariants(oracle_mod):
    rng = np.random.default_rng(3)
    y_raw = rng.standard_normal(128) * 0.05
    z = rng.standard_normal(128)
    w = rng.uniform(0.5, 1.5, 128)
    eps = 1e-6
    y = oracle_mod.gated_rmsnorm(y_raw, z, w, eps)
    ms = np.mean(y_raw ** 2)
    # removing the gate and weight leaves a vector with mean square ms / (ms + eps)
    core = y / (w * z * expit(z))
    assert abs(np.mean(core ** 2) - ms / (ms + eps)) < 1e-12
    # and pointing along y_raw
    assert rel(core / np.linalg.norm(core), y_raw / np.linalg.norm(y_raw)) < 1e-12
    # scale invariance when eps = 0
    assert rel(oracle_mod.gated_rmsnorm(7.0 * y_raw, z, w, 0.0),
               oracle_mod.gated_rmsnorm(y_raw, z, w, 0.0)) < 1e-13


# ---- the recurrence: invariants and closed forms (field guide §02) ---------------------

def _rand_stream(rng, T, dk, dv, unit_k=True):
    q = unit_rows(rng, T, dk)
    k = unit_rows(rng, T, dk) if unit_k else rng.standard_normal((T, dk))
    v = rng.standard_normal((T, dv))
    g = -rng.uniform(0.0, 2.0, T)
    beta = rng.uniform(0.05, 1.0, T)
    return q, k, v, g, beta


def test_I1_full_write_recalls_value(oracle_mod):
    """beta = 1 and unit k: after each write, S'' k = v exactly, for any decay and state."""
    rng = np.random.default_rng(4)
    dk, dv = 16, 12
    S0 = rng.standard_normal((dv, dk))
    q, k, v, g, _ = _rand_stream(rng, 6, dk, dv)
    for T in range(1, 7):
        _, S = oracle_mod.recurrence(q[:T], k[:T], v[:T], g[:T], np.ones(T), S0)
        assert rel(S @ k[T - 1], v[T - 1]) < 1e-12


def test_I2_zero_write_is_pure_decay(oracle_mod):
    rng = np.random.default_rng(5)
    dk, dv, T = 16, 8, 9
    S0 = rng.standard_normal((dv, dk))
    q, k, v, g, _ = _rand_stream(rng, T, dk, dv)
    y, S = oracle_mod.recurrence(q, k, v, g, np.zeros(T), S0)
    gam = np.cumsum(g)
    assert rel(S, np.exp(gam[-1]) * S0) < RTOL
    assert rel(y, np.exp(gam)[:, None] * (q @ S0.T)) < RTOL


def test_I3_orthonormal_keys_accumulate_outer_products(oracle_mod):
    """g = 0, beta = 1, orthonormal keys, S0 = 0: S_t = sum v_i k_i^T, y_t = sum v_i (k_i.q_t)."""
    rng = np.random.default_rng(6)
    d = 32
    Qm, _ = np.linalg.qr(rng.standard_normal((d, d)))
    T = 20
    k = Qm[:T]  # orthonormal rows
    v = rng.standard_normal((T, d))
    q = unit_rows(rng, T, d)
    y, S = oracle_mod.recurrence(q, k, v, np.zeros(T), np.ones(T), np.zeros((d, d)))
    assert rel(S, v.T @ k) < 1e-12
    expect = np.stack([(v[: t + 1] * (k[: t + 1] @ q[t])[:, None]).sum(0) for t in range(T)])
    assert rel(y, expect) < 1e-12


def test_I5_strong_decay_limit(oracle_mod):
    rng = np.random.default_rng(7)
    dk, dv, T = 16, 16, 7
    q, k, v, _, beta = _rand_stream(rng, T, dk, dv)
    S0 = rng.standard_normal((dv, dk))
    g = np.full(T, -1e6)  # exp(g) == 0 exactly: every token sees only its own write
    y, S = oracle_mod.recurrence(q, k, v, g, beta, S0)
    assert rel(S, beta[-1] * np.outer(v[-1], k[-1])) < RTOL
    assert rel(y, (beta * np.einsum("td,td->t", k, q))[:, None] * v) < RTOL


def test_I6_one_token_closed_form(oracle_mod):
    """y = e^g S0 q + beta (v - e^g S0 k)(k.q) and S = e^g S0 + beta (v - e^g S0 k) k^T."""
    rng = np.random.default_rng(8)
    dk, dv = 24, 20
    for _ in range(5):
        S0 = rng.standard_normal((dv, dk))
        q, k, v, g, beta = _rand_stream(rng, 1, dk, dv, unit_k=False)
        y, S = oracle_mod.recurrence(q, k, v, g, beta, S0)
        a = np.exp(g[0])
        err = v[0] - a * S0 @ k[0]
        assert rel(y[0], a * S0 @ q[0] + beta[0] * err * (k[0] @ q[0])) < 1e-12
        assert rel(S, a * S0 + beta[0] * np.outer(err, k[0])) < 1e-12


def test_brute_force_product_form(oracle_mod):
    """S_t = e^{g_t} S_{t-1} (I - beta_t k k^T) + beta_t v k^T, by dense matrix products."""
    rng = np.random.default_rng(9)
    dk, dv, T = 6, 5, 11
    q, k, v, g, beta = _rand_stream(rng, T, dk, dv, unit_k=False)
    S0 = rng.standard_normal((dv, dk))
    y, S = oracle_mod.recurrence(q, k, v, g, beta, S0, q_scale=0.5)
    Sb = S0.copy()
    ys = []
    for t in range(T):
        Sb = np.exp(g[t]) * Sb @ (np.eye(dk) - beta[t] * np.outer(k[t], k[t])) + beta[t] * np.outer(v[t], k[t])
        ys.append(Sb @ (0.5 * q[t]))
    assert rel(S, Sb) < 1e-12
    assert rel(y, np.array(ys)) < 1e-12


@pytest.mark.parametrize("T", [1, 5, 63, 64, 65, 200])
@pytest.mark.parametrize("C", [1, 4, 16, 64, 0])
def test_I4_chunked_equals_token_form(oracle_mod, T, C):
    rng = np.random.default_rng(100 + T)
    dk, dv = 32, 24
    q, k, v, g, beta = _rand_stream(rng, T, dk, dv)
    g = g * 3.0
    S0 = rng.standard_normal((dv, dk)) * 0.3
    y_t, S_t = oracle_mod.recurrence(q, k, v, g, beta, S0)
    y_c, S_c = oracle_mod.recurrence(q, k, v, g, beta, S0, chunk=C if C else T)
    assert rel(y_c, y_t) < 1e-11
    assert rel(S_c, S_t) < 1e-11


def test_I7_resume_equals_one_pass(oracle_mod):
    rng = np.random.default_rng(10)
    dk, dv, T = 16, 16, 40
    q, k, v, g, beta = _rand_stream(rng, T, dk, dv)
    S0 = rng.standard_normal((dv, dk))
    y, S = oracle_mod.recurrence(q, k, v, g, beta, S0)
    for t in (1, 17, 39):
        y1, S1 = oracle_mod.recurrence(q[:t], k[:t], v[:t], g[:t], beta[:t], S0)
        y2, S2 = oracle_mod.recurrence(q[t:], k[t:], v[t:], g[t:], beta[t:], S1)
        assert rel(np.concatenate([y1, y2]), y) < RTOL
        assert rel(S2, S) < RTOL


# ---- the whole mixer: plumbing, packing, symmetry, decode ----------------------------

def _f64(x):
    return bf16_bits_to_f32(x).astype(np.float64) if x.dtype == np.uint16 else x.astype(np.float64)


def test_prefill_composes_the_stages(oracle_mod):
    """Whole prefill == conv (numpy.convolve) -> norms -> gates -> recurrence -> output gate,
    assembled here with the documented layouts and the QK head of value head h = h // 2."""
    inp = make_inputs("tiny_prefill_fp32", T=37)
    out = oracle_mod.prefill(inp)
    hq, hv, d = 2, 4, 128
    q, k, v, z = (_f64(inp[n]) for n in "qkvz")
    cw = inp["conv_w"].astype(np.float64)

    def conv(x, w):
        pre = np.stack([np.convolve(x[:, c], w[c, ::-1])[: x.shape[0]] for c in range(x.shape[1])], 1)
        return pre * expit(pre)

    for h in range(hv):
        j = h // (hv // hq)
        qc = conv(q[:, j], cw[j * d:(j + 1) * d])
        kc = conv(k[:, j], cw[hq * d + j * d: hq * d + (j + 1) * d])
        vc = conv(v[:, h], cw[2 * hq * d + h * d: 2 * hq * d + (h + 1) * d])
        qn = qc / np.sqrt(np.linalg.norm(qc, axis=1, keepdims=True) ** 2 + 1e-6)
        kn = kc / np.sqrt(np.linalg.norm(kc, axis=1, keepdims=True) ** 2 + 1e-6)
        x = inp["a"][:, h].astype(np.float64) + float(inp["dt_bias"][h])
        g = -np.exp(float(inp["A_log"][h])) * np.logaddexp(0.0, x)
        beta = expit(inp["b"][:, h].astype(np.float64))
        y_raw, S = oracle_mod.recurrence(qn, kn, vc, g, beta, np.zeros((d, d)))
        for t in range(y_raw.shape[0]):
            yo = oracle_mod.gated_rmsnorm(y_raw[t], z[t, h], inp["norm_w"], 1e-6)
            assert rel(out["y"][t, h], yo) < 1e-12
        assert rel(out["final_state"][0, h], S) < 1e-12


def test_varlen_packing_equals_separate_sequences(oracle_mod):
    lens = [5, 0, 70, 1, 64]
    inp = make_inputs("varlen8_prefill_bf16", lengths=lens, h_qk=2, h_v=4)
    out = oracle_mod.prefill(inp)
    cu = inp["cu_seqlens"]
    for n, L in enumerate(lens):
        t0, t1 = cu[n], cu[n + 1]
        sub = dict(inp)
        for name in ("q", "k", "v", "z", "a", "b"):
            sub[name] = inp[name][t0:t1]
        sub["cu_seqlens"] = None
        sub["init_state"] = inp["init_state"][n: n + 1]
        if L == 0:
            assert np.array_equal(out["final_state"][n], inp["init_state"][n].astype(np.float64))
            continue
        o = oracle_mod.prefill(sub)
        assert rel(out["y"][t0:t1], o["y"]) < 1e-13
        assert rel(out["final_state"][n], o["final_state"][0]) < 1e-13


def test_I8_head_symmetry(oracle_mod):
    inp = make_inputs("tiny_prefill_fp32", T=21)
    for name in ("v", "z", "a", "b"):
        inp[name][:, 1] = inp[name][:, 0]
    inp["A_log"][1] = inp["A_log"][0]
    inp["dt_bias"][1] = inp["dt_bias"][0]
    d = 128
    base = 2 * 2 * d
    inp["conv_w"][base + d: base + 2 * d] = inp["conv_w"][base: base + d]
    out = oracle_mod.prefill(inp)
    assert np.array_equal(out["y"][:, 0], out["y"][:, 1])
    assert np.array_equal(out["final_state"][0, 0], out["final_state"][0, 1])


def test_I8_value_permutation(oracle_mod):
    """Permuting value components of v, z, norm_w, the v conv taps and the rows of S0
    permutes y and the rows of S (value rows evolve independently)."""
    inp = make_inputs("varlen8_prefill_bf16", lengths=[19], h_qk=1, h_v=2)
    inp["norm_w"] = np.random.default_rng(11).uniform(0.5, 1.5, 128).astype(np.float32)
    out = oracle_mod.prefill(inp)
    perm = np.random.default_rng(12).permutation(128)
    p = dict(inp)
    p["v"] = inp["v"][:, :, perm]
    p["z"] = inp["z"][:, :, perm]
    p["norm_w"] = inp["norm_w"][perm]
    cw = inp["conv_w"].copy()
    base = 2 * 128
    for h in range(2):
        cw[base + h * 128: base + (h + 1) * 128] = inp["conv_w"][base + h * 128 + perm]
    p["conv_w"] = cw
    p["init_state"] = inp["init_state"][:, :, perm, :]
    o2 = oracle_mod.prefill(p)
    assert rel(o2["y"], out["y"][:, :, perm]) < 1e-13
    assert rel(o2["final_state"], out["final_state"][:, :, perm, :]) < 1e-13


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_I9_decode_continues_prefill(oracle_mod, dtype):
    """decode(token T) on prefill(T)'s final state and the raw x_{T-3..T-1} as conv history
    equals the last token of prefill(T+1)."""
    T = 9
    name = "tiny_prefill_fp32"
    full = make_inputs(name, T=T + 1, dtype=dtype)
    head = dict(full)
    for n in ("q", "k", "v", "z", "a", "b"):
        head[n] = full[n][:T]
    pre_T = oracle_mod.prefill(head)
    pre_T1 = oracle_mod.prefill(full)
    cs = np.concatenate([full["q"][T - 3:T].reshape(3, -1), full["k"][T - 3:T].reshape(3, -1),
                         full["v"][T - 3:T].reshape(3, -1)], axis=1)[None]
    dec = dict(full)
    for n in ("q", "k", "v", "z", "a", "b"):
        dec[n] = full[n][T:T + 1]
    dec["state"] = pre_T["final_state"].astype(np.float32)
    dec["conv_state"] = np.ascontiguousarray(cs)
    o = oracle_mod.decode(dec)
    # the state went through fp32 on the way in: compare at fp32 resolution of the state
    assert np.abs(o["y"][0] - pre_T1["y"][T]).max() < 1e-5
    assert rel(o["state"][0], pre_T1["final_state"][0]) < 1e-5
    # conv history shifted by one token, raw values copied exactly
    expect = np.concatenate([full["q"][T - 2:T + 1].reshape(3, -1), full["k"][T - 2:T + 1].reshape(3, -1),
                             full["v"][T - 2:T + 1].reshape(3, -1)], axis=1)
    assert np.array_equal(o["conv_state"][0], _f64(expect))


@pytest.mark.parametrize("T", [2, 9])
def test_decode_steps_continue_prefill(oracle_mod, T):
    """K = 5 decode steps in a row, from prefill(T)'s final state and conv history (zeros
    before the first token when T < 3), equal the last K tokens and the final state of
    prefill(T + K): the decode step composes with itself as the recurrence does."""
    K = 5
    full = make_inputs("tiny_prefill_fp32", T=T + K)
    head = dict(full)
    for n in ("q", "k", "v", "z", "a", "b"):
        head[n] = full[n][:T]
    pre = oracle_mod.prefill(full)
    state = oracle_mod.prefill(head)["final_state"].astype(np.float32)
    width = 2 * full["q"].shape[1] * full["q"].shape[2] + full["v"].shape[1] * full["v"].shape[2]
    hist = np.zeros((1, 3, width), np.float32)
    for r in range(3):
        t = T - 3 + r
        if t >= 0:
            hist[0, r] = np.concatenate([full["q"][t].ravel(), full["k"][t].ravel(), full["v"][t].ravel()])
    for i in range(K):
        dec = dict(full)
        for n in ("q", "k", "v", "z", "a", "b"):
            dec[n] = full[n][T + i:T + i + 1]
        dec["state"], dec["conv_state"] = state, hist
        o = oracle_mod.decode(dec)
        assert np.abs(o["y"][0] - pre["y"][T + i]).max() < 1e-5
        state, hist = o["state"].astype(np.float32), o["conv_state"].astype(np.float32)
    assert rel(o["state"][0], pre["final_state"][0]) < 1e-5


def test_decode_exact_state_roundtrip(oracle_mod):
    """With the state given exactly in fp32, decode equals a one-token prefill whose
    conv history is the same raw values (both in fp64)."""
    inp = make_inputs("decode_N256_bf16", n_seqs=3, h_qk=2, h_v=4)
    o = oracle_mod.decode(inp)
    for n in range(3):
        hist = inp["conv_state"][n]
        pre = {}
        d = 128
        pre["q"] = np.concatenate([hist[:, : 2 * d].reshape(3, 2, d), inp["q"][n:n + 1]])
        pre["k"] = np.concatenate([hist[:, 2 * d: 4 * d].reshape(3, 2, d), inp["k"][n:n + 1]])
        pre["v"] = np.concatenate([hist[:, 4 * d:].reshape(3, 4, d), inp["v"][n:n + 1]])
        # the three history tokens write nothing (beta = 0) and do not decay (g = 0): the
        # state reaches the fourth token unchanged
        pre["z"] = np.concatenate([np.zeros((3, 4, d), np.uint16), inp["z"][n:n + 1]])
        pre["a"] = np.concatenate([np.full((3, 4), -800.0, np.float32), inp["a"][n:n + 1]])
        pre["b"] = np.concatenate([np.full((3, 4), -800.0, np.float32), inp["b"][n:n + 1]])
        for nm in ("A_log", "dt_bias", "conv_w", "norm_w"):
            pre[nm] = inp[nm]
        pre["init_state"] = inp["state"][n:n + 1]
        pre["cu_seqlens"] = None
        r = oracle_mod.prefill(pre)
        assert rel(r["y"][3], o["y"][n]) < 1e-12
        assert rel(r["final_state"][0], o["state"][n]) < 1e-12


# ---- the projections around the mixer (technical report Fig. 2; field guide §02) -----------

def _bits(a):
    return (np.asarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_projections_brute_force_tiny(oracle_mod):
    """A triple loop over (token, feature, input) on values that are exact in bf16."""
    oracle = oracle_mod
    rng = np.random.default_rng(3)
    T, hidden, h_qk, h_v, d = 3, 8, 1, 1, 2
    n_in = 2 * h_qk * d + 2 * h_v * d + 2 * h_v
    x = rng.integers(-4, 5, size=(T, hidden)).astype(np.float32)
    w = rng.integers(-4, 5, size=(n_in, hidden)).astype(np.float32)
    o = oracle.in_proj(_bits(x), _bits(w), h_qk, h_v, d, d)
    flat = np.concatenate([o["q"].reshape(T, -1), o["k"].reshape(T, -1), o["v"].reshape(T, -1),
                           o["z"].reshape(T, -1), o["a"], o["b"]], axis=1)
    for t in range(T):
        for n in range(n_in):
            acc = 0.0
            for i in range(hidden):
                acc += float(x[t, i]) * float(w[n, i])
            assert flat[t, n] == acc
    wo = rng.integers(-4, 5, size=(5, h_v * d)).astype(np.float32)
    y = rng.integers(-4, 5, size=(T, h_v, d)).astype(np.float32)
    out = oracle.out_proj(_bits(y), _bits(wo))
    for t in range(T):
        for n in range(5):
            assert out[t, n] == sum(float(y.reshape(T, -1)[t, i]) * float(wo[n, i]) for i in range(h_v * d))


def test_in_proj_row_order_and_head_layout(oracle_mod):
    """Selector weights: row n of W_in picks input feature n % hidden, scaled by its block's
    number (q 1, k 2, v 3, z 4, a 5, b 6), so every output lands where the mixer reads it."""
    oracle = oracle_mod
    T, hidden, h_qk, h_v, d = 2, 16, 2, 4, 4
    nq, nv = h_qk * d, h_v * d
    sizes = [nq, nq, nv, nv, h_v, h_v]
    w = np.zeros((sum(sizes), hidden), np.float32)
    r = 0
    for blk, sz in enumerate(sizes):
        for i in range(sz):
            w[r, r % hidden] = blk + 1
            r += 1
    x = np.arange(T * hidden, dtype=np.float32).reshape(T, hidden) + 1
    o = oracle.in_proj(_bits(x), _bits(w), h_qk, h_v, d, d)
    r = 0
    for blk, name in enumerate(("q", "k", "v", "z", "a", "b")):
        arr = o[name].reshape(T, -1)
        for i in range(arr.shape[1]):
            assert np.array_equal(arr[:, i], (blk + 1) * x[:, r % hidden])
            r += 1
    assert o["q"].shape == (T, h_qk, d) and o["v"].shape == (T, h_v, d) and o["a"].shape == (T, h_v)


# ---- the backward of the recurrence core (NEXT-4) --------------------------------------------

def test_recurrence_backward_matches_finite_differences(oracle_mod):
    """Every gradient of the reverse-mode oracle against central differences of the forward
    recurrence (the C per-token rule) of L = sum dy . y + <dS_T, S_T>, on a tiny case."""
    rng = np.random.default_rng(7)
    T, d = 5, 4
    qh = rng.standard_normal((T, d)); kh = rng.standard_normal((T, d))
    kh /= np.linalg.norm(kh, axis=1, keepdims=True)
    v = rng.standard_normal((T, d)); g = -rng.uniform(0.05, 1.0, T); beta = rng.uniform(0.1, 0.9, T)
    S0 = rng.standard_normal((d, d)) * 0.3
    dy = rng.standard_normal((T, d)); dST = rng.standard_normal((d, d))

    def loss(qh_, kh_, v_, g_, b_, S0_):
        y, S = oracle_mod.recurrence(qh_, kh_, v_, g_, b_, S0_)
        return float(np.sum(dy * y) + np.sum(dST * S))

    got = oracle_mod.recurrence_backward(qh, kh, v, g, beta, S0, dy, dST)
    args = [qh, kh, v, g, beta, S0]
    names = ["dq", "dk", "dv", "dg", "dbeta", "dS0"]
    h = 1e-6
    for ai, name in enumerate(names):
        base = args[ai]
        fd = np.zeros_like(base)
        it = np.nditer(base, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[ai][idx] += h
            minus[ai][idx] -= h
            fd[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        np.testing.assert_allclose(got[name], fd, rtol=1e-6, atol=1e-7, err_msg=name)


def test_recurrence_backward_zero_write_is_pure_decay(oracle_mod):
    """beta = 0: the state only decays, S_T = e^{sum g} S_0, y_t = e^{gamma_t} S_0 q_t; then
    dv = 0, dS_0 = sum_t e^{gamma_t} dy_t q_t^T + e^{gamma_T} dS_T in closed form."""
    rng = np.random.default_rng(8)
    T, d = 6, 3
    qh = rng.standard_normal((T, d)); kh = rng.standard_normal((T, d)); v = rng.standard_normal((T, d))
    g = -rng.uniform(0.1, 0.5, T); beta = np.zeros(T); S0 = rng.standard_normal((d, d))
    dy = rng.standard_normal((T, d)); dST = rng.standard_normal((d, d))
    got = oracle_mod.recurrence_backward(qh, kh, v, g, beta, S0, dy, dST)
    gam = np.cumsum(g)
    want = sum(np.exp(gam[t]) * np.outer(dy[t], qh[t]) for t in range(T)) + np.exp(gam[-1]) * dST
    np.testing.assert_allclose(got["dS0"], want, rtol=1e-12, atol=1e-12)
    assert np.all(got["dv"] == 0)
