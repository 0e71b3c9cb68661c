"""Writes tests/golden/oracle_small_cases.json from the oracle alone.

The TTT pages print no worked example with values, so there is no page-given golden vector.
These fixtures are small seeded cases whose expected values come only from oracle/ (run this
script after a change to the oracle's arithmetic, and name the passage that justifies the
change in the commit).  tests/test_golden.py checks that the oracle still reproduces them and
that the independent dual-form implementation agrees with them.
"""
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth  # noqa: E402


def cases():
    o = oracle.default()
    out = {}
    # TTT-Linear: d=8, K=4, L=10 (two full mini-batches and a tail of 2), unit LN
    w = synth.workload(0, B=1, H=1, L=10, d=8, K=4, ln="random", x_std=0.5, seed=0x5EED01)
    x = synth.linear_inputs(w)
    x["b0"] = synth.random_bias(w, "B0", (1, 8), 0.1)
    r = o.linear_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"] * 10, x["b0"], x["ln_w"], x["ln_b"],
                         w.K, w.eps)
    out["linear_d8_K4_L10"] = {
        "inputs": {"XQ": x["XQ"][0, 0], "XK": x["XK"][0, 0], "XV": x["XV"][0, 0], "lr": x["lr"][0, 0],
                   "W0": x["W0"][0] * 10, "b0": x["b0"][0], "ln_w": x["ln_w"][0], "ln_b": x["ln_b"][0]},
        "K": w.K, "eps": w.eps,
        "expected": {k: r[k][0] for k in ("out", "W_last", "b_last", "W_grad_tail", "b_grad_tail")},
    }
    # TTT-MLP: d=4, h=8, K=3, L=7
    w = synth.workload(3, B=1, H=1, L=7, d=4, K=3, hidden=8, x_std=0.5, seed=0x5EED02)
    x = synth.linear_inputs(w)
    r = o.mlp_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W1"] * 20, x["b1"], x["W2"] * 20, x["b2"],
                      x["ln_w"], x["ln_b"], w.K, w.eps)
    out["mlp_d4_h8_K3_L7"] = {
        "inputs": {"XQ": x["XQ"][0, 0], "XK": x["XK"][0, 0], "XV": x["XV"][0, 0], "lr": x["lr"][0, 0],
                   "W1": x["W1"][0] * 20, "b1": x["b1"][0], "W2": x["W2"][0] * 20, "b2": x["b2"][0],
                   "ln_w": x["ln_w"][0], "ln_b": x["ln_b"][0]},
        "K": w.K, "eps": w.eps,
        "expected": {k: r[k][0] for k in ("out", "W1_last", "b1_last", "W2_last", "b2_last")},
    }
    return out


def to_json(obj):
    if isinstance(obj, dict):
        return {k: to_json(v) for k, v in obj.items()}
    if isinstance(obj, np.ndarray):
        return np.asarray(obj, np.float64).tolist()
    return obj


if __name__ == "__main__":
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "oracle_small_cases.json")
    with open(path, "w") as f:
        json.dump({"_source": "written by tests/golden/make_golden.py from oracle/ only; the TTT pages "
                              "print no worked example with values",
                   **to_json(cases())}, f, indent=1)
    print("wrote", path)
