"""Fixtures under tests/golden/: the mixer's shape as the pages print it (field guide §02), and
the oracle's own outputs on two tiny seeded workloads (written by tests/golden/make_golden.py,
which calls only the input generator and oracle/), so that any later change to the oracle's
arithmetic shows up here."""
import importlib.util
import json
import os

import numpy as np

from gated_deltanet_token_b200.inputs import WORKLOADS, make_inputs

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def test_model_workloads_have_the_printed_shape(oracle_mod):
    shape = json.load(open(os.path.join(GOLDEN, "gdn_shape.json")))
    for name in ("prefill_T4096_bf16", "varlen8_prefill_bf16", "long_prefill_T262144_bf16", "decode_N256_bf16"):
        spec = WORKLOADS[name]
        assert (spec["h_qk"], spec["h_v"], spec["d"]) == (shape["h_qk"], shape["h_v"], shape["d_k"])
    inp = make_inputs("prefill_T4096_bf16", T=2)
    assert inp["conv_w"].shape == ((2 * shape["h_qk"] + shape["h_v"]) * shape["d_k"], shape["conv_width"])
    out = oracle_mod.prefill(inp)
    assert out["final_state"].shape[1:] == (shape["n_states"], *shape["state_shape"])


def test_oracle_matches_its_regression_fixture(oracle_mod):
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    stored = json.load(open(os.path.join(GOLDEN, "oracle_tiny.json")))
    now = mg.compute()
    for part in ("prefill", "decode"):
        assert stored[part]["workload"] == json.loads(json.dumps(now[part]["workload"]))
        for key, val in stored[part].items():
            if key == "workload":
                continue
            np.testing.assert_allclose(np.asarray(now[part][key]), np.asarray(val), rtol=1e-12, atol=1e-14)
