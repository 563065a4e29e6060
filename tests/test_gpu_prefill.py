"""GPU parity of gdn_prefill against the fp64 oracle on the same seeded inputs.

Tolerances (fixed for the mixer): fp32 runs e_y = max|y - y_ref| <= 1e-4 and
e_S = ||S - S_ref||_F / ||S_ref||_F <= 1e-4; bf16-input runs e_y <= 2e-2 RMS(y_ref) and
e_S <= 1e-2, with half a bf16 ulp of y_ref per element added when y itself is bf16."""
import numpy as np
import pytest
import torch

from gated_deltanet_token_b200 import gdn
from gated_deltanet_token_b200.inputs import make_inputs
from tests._helpers import check_bf16, check_fp32, e_S, path_options, rms, run_prefill

pytestmark = pytest.mark.gpu


def _oracle(oracle_mod, inp, heads=None):
    return oracle_mod.prefill(inp, heads=heads)


def test_tiny_prefill_fp32(oracle_mod):
    inp = make_inputs("tiny_prefill_fp32")
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["final_state"])


@pytest.mark.parametrize("T", [1, 2, 3, 4, 63, 64, 65, 130, 200])
def test_short_lengths_fp32(oracle_mod, T):
    inp = make_inputs("tiny_prefill_fp32", T=T)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["final_state"])


@pytest.mark.parametrize("ratio", [1, 2, 4])
def test_head_ratios_fp32(oracle_mod, ratio):
    inp = make_inputs("tiny_prefill_fp32", T=77, h_qk=2, h_v=2 * ratio)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["final_state"])


def test_q_scale_and_init_state_fp32(oracle_mod):
    inp = make_inputs("tiny_prefill_fp32", T=90)
    inp["init_state"] = (np.random.default_rng(5).standard_normal((1, 4, 128, 128)) * 0.02).astype(np.float32)
    ref = oracle_mod.prefill(inp, q_scale=128 ** -0.5)
    y, S = run_prefill(inp, torch.float32, q_scale=128 ** -0.5)
    check_fp32(y, ref["y"], S, ref["final_state"])


def test_model_shape_short_bf16(oracle_mod):
    inp = make_inputs("prefill_T4096_bf16", T=300)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["final_state"])
    yb, Sb = run_prefill(inp, torch.bfloat16)
    check_bf16(yb, ref["y"], Sb, ref["final_state"], y_is_bf16=True)


def test_prefill_T4096_bf16(oracle_mod):
    inp = make_inputs("prefill_T4096_bf16")
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["final_state"])
    yb, Sb = run_prefill(inp, torch.bfloat16)
    check_bf16(yb, ref["y"], Sb, ref["final_state"], y_is_bf16=True)


def test_varlen_with_empty_sequences_and_alias(oracle_mod):
    lens = [0, 5, 64, 0, 65, 1, 130, 0]
    inp = make_inputs("varlen8_prefill_bf16", lengths=lens)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32, init_alias=True)
    check_bf16(y, ref["y"], S, ref["final_state"])
    for n, L in enumerate(lens):  # empty sequences copy their initial state exactly
        if L == 0:
            assert np.array_equal(S[n], inp["init_state"][n].astype(np.float64))


@pytest.mark.parametrize("n_seqs", [1024, 1100])
def test_many_short_sequences_dispatch_order(oracle_mod, n_seqs):
    """Phase B takes the sequences longest first up to 1024 of them (the tile map ranks them)
    and in index order beyond: both orders give every sequence its own result."""
    rng = np.random.default_rng(n_seqs)
    lens = [int(x) for x in rng.integers(0, 70, size=n_seqs)]
    lens[3] = 200  # a long one late in the index order
    inp = make_inputs("varlen8_prefill_bf16", lengths=lens, h_qk=1, h_v=2)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["final_state"])


def test_varlen_equals_separate_calls():
    lens = [37, 100, 64]
    inp = make_inputs("varlen8_prefill_bf16", lengths=lens, h_qk=4, h_v=8)
    y, S = run_prefill(inp, torch.float32)
    cu = inp["cu_seqlens"]
    for n in range(len(lens)):
        sub = dict(inp)
        for nm in ("q", "k", "v", "z", "a", "b"):
            sub[nm] = inp[nm][cu[n]:cu[n + 1]]
        sub["init_state"] = inp["init_state"][n:n + 1]
        sub["cu_seqlens"] = None
        y1, S1 = run_prefill(sub, torch.float32)
        assert np.array_equal(y1, y[cu[n]:cu[n + 1]])
        assert np.array_equal(S1[0], S[n])


def test_zero_tokens_copies_init():
    inp = make_inputs("varlen8_prefill_bf16", lengths=[0, 0], h_qk=2, h_v=4)
    y, S = run_prefill(inp, torch.float32)
    assert y.shape[0] == 0
    assert np.array_equal(S, inp["init_state"].astype(np.float64))


def _check_blocked(y_dev, y_ref, y_is_bf16, block=8192):
    """The bf16-run bound on y, token block by token block (the long workload's fp64 copies
    would not fit in host memory three times over).  Returns (e_y / RMS(y_ref), RMS(y_ref))."""
    T = y_ref.shape[0]
    ss = 0.0
    for t0 in range(0, T, block):
        r = y_ref[t0:t0 + block]
        ss += float(np.sum(r * r))
    r_all = float(np.sqrt(ss / y_ref.size)) if y_ref.size else 0.0
    worst, ey = -1.0, 0.0
    for t0 in range(0, T, block):
        r = y_ref[t0:t0 + block]
        g = y_dev[t0:t0 + block].float().cpu().numpy().astype(np.float64)
        err = np.abs(g - r)
        bound = 2e-2 * r_all + (2.0 ** -8) * np.abs(r) if y_is_bf16 else 2e-2 * r_all
        worst = max(worst, float((err - bound).max()))
        ey = max(ey, float(err.max()))
    assert worst <= 0, f"e_y = {ey:.3e} exceeds its bound (RMS(y_ref) = {r_all:.3f})"
    return ey / max(r_all, 1e-30), r_all


def _full_config_parity(oracle_mod, name):
    """A configuration on all of its value heads: y (fp32, then bf16) under the bf16-run bound,
    e_S <= 1e-2 jointly over every (sequence, head) state, and the worst single head reported."""
    inp = make_inputs(name)
    ref = _oracle(oracle_mod, inp)
    from tests._helpers import to_dev

    d = {n: to_dev(inp.get(n)) for n in ("q", "k", "v", "z", "a", "b", "A_log", "dt_bias", "conv_w",
                                         "norm_w", "init_state")}
    cu = inp.get("cu_seqlens")
    cu_t = None if cu is None else to_dev(cu.astype(np.int32))
    out = {}
    for out_dtype in (torch.float32, torch.bfloat16):
        y, fs = gdn.gdn_prefill(d["q"], d["k"], d["v"], d["z"], d["a"], d["b"], d["A_log"], d["dt_bias"],
                                d["conv_w"], d["norm_w"], d["init_state"], cu_t, out_dtype=out_dtype)
        torch.cuda.synchronize()
        rel, _ = _check_blocked(y, ref["y"], out_dtype == torch.bfloat16)
        S = fs.cpu().numpy().astype(np.float64)
        es = e_S(S, ref["final_state"])
        worst_head = max(e_S(S[n, h], ref["final_state"][n, h])
                         for n in range(S.shape[0]) for h in range(S.shape[1]))
        assert es <= 1e-2, f"e_S = {es:.3e} > 1e-2"
        out[str(out_dtype)] = (rel, es, worst_head)
        del y, fs
    print(name, out)
    return out


def test_varlen8_bf16_all_heads(oracle_mod):
    """Config 2 in full: 8 packed sequences of U{512..8192} tokens, nonzero initial states, all
    32 value heads."""
    _full_config_parity(oracle_mod, "varlen8_prefill_bf16")


@pytest.mark.slow
def test_long_prefill_T262144_all_heads(oracle_mod):
    """Config 3 in full: one sequence of 262,144 tokens (a chain of 4,096 chunks), all 32 value
    heads."""
    _full_config_parity(oracle_mod, "long_prefill_T262144_bf16")


def _extreme_gates(inp):
    """Gates at the ends of their ranges, by head group: A_log = log 1e6 (e^g underflows to 0
    inside a chunk), b = +30 (beta = 1 to fp32 precision), b = -30 (beta ~ 1e-13), and a mix of
    tokens with a = +20 (a decay of about -20 e^{A_log}) among ordinary ones."""
    h_v = inp["A_log"].shape[0]
    q4 = max(1, h_v // 4)
    A_log = inp["A_log"].copy()
    A_log[:q4] = np.log(1e6)
    b = inp["b"].copy()
    b[:, q4:2 * q4] = 30.0
    b[:, 2 * q4:3 * q4] = -30.0
    a = inp["a"].copy()
    a[::7, 3 * q4:] = 20.0
    b[::5, 3 * q4:] = 30.0
    b[2::5, 3 * q4:] = -30.0
    inp = dict(inp)
    inp["A_log"], inp["b"], inp["a"] = A_log.astype(np.float32), b.astype(np.float32), a.astype(np.float32)
    return inp


@pytest.mark.parametrize("opts", [0, gdn.GDN_OPT_SEPARATE_NORM, gdn.GDN_OPT_FORCE_FP32_PATH])
def test_extreme_gates_model_shape(oracle_mod, opts):
    """The decay gate has no clamp: a decay that underflows inside a chunk, beta at 0 and 1,
    and strong single-token decays, at the model head shapes, on the tensor-core path (fused
    and separate output norm) and on the fp32 path."""
    inp = _extreme_gates(make_inputs("varlen8_prefill_bf16", lengths=[300, 64, 129, 1]))
    ref = _oracle(oracle_mod, inp)
    with path_options(opts):
        y, S = run_prefill(inp, torch.float32)
    assert np.isfinite(y).all() and np.isfinite(S).all()
    check_bf16(y, ref["y"], S, ref["final_state"])


def test_extreme_gates_fp32_inputs(oracle_mod):
    inp = _extreme_gates(make_inputs("tiny_prefill_fp32", T=200, h_qk=2, h_v=8))
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    assert np.isfinite(y).all() and np.isfinite(S).all()
    check_fp32(y, ref["y"], S, ref["final_state"])


# ---- the bf16 (tensor-core) path: head ratios, ragged lengths, SIMT cross-check ----------

@pytest.mark.parametrize("ratio", [1, 2, 3, 4, 8])
def test_head_ratios_bf16_tensor_core_path(oracle_mod, ratio):
    inp = make_inputs("varlen8_prefill_bf16", lengths=[77, 3, 130], h_qk=2, h_v=2 * ratio)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["final_state"])


@pytest.mark.parametrize("T", [1, 2, 3, 4, 31, 32, 33, 63, 64, 65, 129])
def test_short_lengths_bf16_tensor_core_path(oracle_mod, T):
    inp = make_inputs("prefill_T4096_bf16", T=T, h_qk=4, h_v=8)
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_bf16(y, ref["y"], S, ref["final_state"])


def test_tensor_core_path_is_insensitive_to_stale_workspace(oracle_mod):
    """The workspace is reused between calls: fill it with NaN bit patterns first and check
    that nothing left in it reaches the results (rows past a chunk's length are rewritten)."""
    from gated_deltanet_token_b200 import gdn

    inp = make_inputs("varlen8_prefill_bf16", lengths=[5, 70, 33], h_qk=2, h_v=4)
    ref = _oracle(oracle_mod, inp)
    T = inp["q"].shape[0]
    dims = gdn.make_dims(3, T, 2, 4, gdn.GDN_DTYPE_BF16, gdn.GDN_DTYPE_F32)
    ws = torch.full((gdn.gdn_prefill_workspace_size(dims),), 0xFF, dtype=torch.uint8, device="cuda")
    y, S = run_prefill(inp, torch.float32, workspace=ws)
    assert np.isfinite(y).all() and np.isfinite(S).all()
    check_bf16(y, ref["y"], S, ref["final_state"])


def test_tensor_core_and_fp32_paths_agree():
    """Both arithmetic paths of the bf16-input prefill (tensor cores with bf16 hi/lo products,
    and fp32 FFMA) against each other, on the model head shapes."""
    inp = make_inputs("varlen8_prefill_bf16", lengths=[200, 64, 1])
    y_tc, S_tc = run_prefill(inp, torch.float32)
    with path_options(gdn.GDN_OPT_FORCE_FP32_PATH):
        y_s, S_s = run_prefill(inp, torch.float32)
    r = float(np.sqrt(np.mean(y_s ** 2)))
    assert np.abs(y_tc - y_s).max() <= 2e-2 * r
    assert np.linalg.norm(S_tc - S_s) / np.linalg.norm(S_s) <= 1e-2


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fused_output_norm_matches_separate_epilogue(oracle_mod, out_dtype):
    """The gated RMS norm fused into the state pass (clusters of the four slices of a head
    exchange their sums of squares) against the same norm in its own kernel, and both
    against the oracle; lengths include empty sequences and partial chunks."""
    inp = make_inputs("varlen8_prefill_bf16", lengths=[0, 130, 1, 64, 0, 77], h_qk=4, h_v=8)
    ref = _oracle(oracle_mod, inp)
    y_f, S_f = run_prefill(inp, out_dtype)
    with path_options(gdn.GDN_OPT_SEPARATE_NORM):
        y_e, S_e = run_prefill(inp, out_dtype)
    is_bf16 = out_dtype == torch.bfloat16
    check_bf16(y_f, ref["y"], S_f, ref["final_state"], y_is_bf16=is_bf16)
    check_bf16(y_e, ref["y"], S_e, ref["final_state"], y_is_bf16=is_bf16)
    assert np.array_equal(S_f, S_e)
    r = float(np.sqrt(np.mean(ref["y"] ** 2)))
    tol = 1e-5 * r if out_dtype == torch.float32 else 2.0 ** -8 * np.abs(ref["y"]).max()
    assert np.abs(y_f - y_e).max() <= tol


def _random_norm_w(inp, seed=5):
    inp["norm_w"] = np.random.default_rng(seed).uniform(0.5, 1.5, inp["norm_w"].shape).astype(np.float32)
    return inp


@pytest.mark.parametrize("fused", [True, False])
@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_norm_weights_bf16_path(oracle_mod, fused, out_dtype):
    """A non-trivial norm_w (every component different) through the fused output norm and
    through the separate epilogue: a wrong component index in either shows up here."""
    inp = _random_norm_w(make_inputs("varlen8_prefill_bf16", lengths=[70, 1, 130], h_qk=4, h_v=8))
    ref = _oracle(oracle_mod, inp)
    with path_options(0 if fused else gdn.GDN_OPT_SEPARATE_NORM):
        y, S = run_prefill(inp, out_dtype)
    check_bf16(y, ref["y"], S, ref["final_state"], y_is_bf16=out_dtype == torch.bfloat16)


def test_norm_weights_fp32_path(oracle_mod):
    inp = _random_norm_w(make_inputs("tiny_prefill_fp32"))
    ref = _oracle(oracle_mod, inp)
    y, S = run_prefill(inp, torch.float32)
    check_fp32(y, ref["y"], S, ref["final_state"])


def test_q_scale_bf16_path(oracle_mod):
    """q_scale on the tensor-core path (the prologue scales the normalised query)."""
    inp = make_inputs("varlen8_prefill_bf16", lengths=[90, 40], h_qk=2, h_v=4)
    ref = oracle_mod.prefill(inp, q_scale=0.7)
    y, S = run_prefill(inp, torch.float32, q_scale=0.7)
    check_bf16(y, ref["y"], S, ref["final_state"])


def test_back_to_back_calls_chain_the_state(oracle_mod):
    """Three prefill calls queued on one stream with no synchronisation between them, sharing one
    workspace, each reading the state the previous one wrote into the same buffer
    (init_state aliases final_state).  The kernels of a call may become resident while the
    previous call's kernels drain, so this checks that every read still follows the write it
    depends on: each segment's y and the final state match the oracle run segment by segment."""
    from gated_deltanet_token_b200 import gdn
    from tests._helpers import to_dev

    lens = [300, 200, 130]
    segs = [make_inputs("prefill_T4096_bf16", seed=10 + i, T=L, h_qk=4, h_v=8, init_state=True)
            for i, L in enumerate(lens)]
    for sg in segs[1:]:  # one layer: the same parameters in every segment
        for nm in ("A_log", "dt_bias", "conv_w", "norm_w"):
            sg[nm] = segs[0][nm]
    par = {nm: to_dev(segs[0][nm]) for nm in ("A_log", "dt_bias", "conv_w", "norm_w")}
    dims = gdn.make_dims(1, max(lens), 4, 8, gdn.GDN_DTYPE_BF16, gdn.GDN_DTYPE_F32)
    ws = torch.empty(gdn.gdn_prefill_workspace_size(dims), dtype=torch.uint8, device="cuda")
    state = to_dev(segs[0]["init_state"]).clone()
    dev_in = [{nm: to_dev(sg[nm]) for nm in ("q", "k", "v", "z", "a", "b")} for sg in segs]
    torch.cuda.synchronize()
    ys = []
    for t in dev_in:  # queued back to back
        y, _ = gdn.gdn_prefill(t["q"], t["k"], t["v"], t["z"], t["a"], t["b"], par["A_log"], par["dt_bias"],
                               par["conv_w"], par["norm_w"], state, None, out_dtype=torch.float32,
                               final_state=state, workspace=ws)
        ys.append(y)
    torch.cuda.synchronize()
    assert gdn.gdn_read_device_status() == 0
    init = segs[0]["init_state"].astype(np.float32)
    for sg, y in zip(segs, ys):  # the oracle, segment by segment, each from the last one's state
        sg = dict(sg)
        sg["init_state"] = init
        ref = _oracle(oracle_mod, sg)
        init = ref["final_state"].astype(np.float32)
        check_bf16(y.float().cpu().numpy().astype(np.float64), ref["y"], ref["final_state"], ref["final_state"])
    check_bf16(ys[-1].float().cpu().numpy().astype(np.float64), ref["y"], state.cpu().numpy().astype(np.float64),
               ref["final_state"])
