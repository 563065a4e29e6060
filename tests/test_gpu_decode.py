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
