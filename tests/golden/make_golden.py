"""Writes tests/golden/oracle_tiny.json: the oracle's prefill and decode on two tiny seeded
workloads, a few KB of values kept as a regression fixture for the oracle itself (the pages
print no worked numeric example of this path).  Calls only the seeded input generator and
oracle/; run it after a change to the oracle's arithmetic that a passage of the pages
justifies, and name that passage in the commit.

    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from gated_deltanet_token_b200.inputs import make_inputs  # noqa: E402

PREFILL = dict(name="tiny_prefill_fp32", seed=0, over={"T": 70})
DECODE = dict(name="decode_N256_bf16", seed=0, over={"n_seqs": 2, "h_qk": 2, "h_v": 4, "dtype": "f32"})


def compute():
    p = oracle.prefill(make_inputs(PREFILL["name"], seed=PREFILL["seed"], **PREFILL["over"]))
    d = oracle.decode(make_inputs(DECODE["name"], seed=DECODE["seed"], **DECODE["over"]))
    y, S = p["y"], p["final_state"]
    return {
        "source": "written by tests/golden/make_golden.py from oracle/ (the pages print no worked "
                  "numeric example of this path)",
        "prefill": {"workload": PREFILL,
                    "y[t, 0, :8] for t in 0, 1, 63, 64, 69": [y[t, 0, :8].tolist() for t in (0, 1, 63, 64, 69)],
                    "y sum, sum of squares": [float(y.sum()), float((y * y).sum())],
                    "final_state[0, h, 0, :8] for h in 0..3": [S[0, h, 0, :8].tolist() for h in range(4)],
                    "final_state sum, sum of squares": [float(S.sum()), float((S * S).sum())]},
        "decode": {"workload": DECODE,
                   "y[n, 0, :8] for n in 0, 1": [d["y"][n, 0, :8].tolist() for n in range(2)],
                   "state sum, sum of squares": [float(d["state"].sum()), float((d["state"] ** 2).sum())]},
    }


if __name__ == "__main__":
    oracle.build()
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_tiny.json")
    with open(out, "w") as f:
        json.dump(compute(), f, indent=1)
    print("wrote", out)
