"""Stored small cases: the oracle still reproduces them, and the independent dual form agrees."""
import json
import os

import numpy as np

import dual_form as dual

_G = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "oracle_small_cases.json")))


def _rel(a, b):
    return np.linalg.norm(np.asarray(a) - np.asarray(b)) / max(np.linalg.norm(b), 1e-300)


def test_linear_small_case(orc):
    c = _G["linear_d8_K4_L10"]
    x = {k: np.array(v) for k, v in c["inputs"].items()}
    r = orc.linear_chain(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"], x["b0"], x["ln_w"], x["ln_b"],
                         c["K"], c["eps"])
    for k, v in c["expected"].items():
        assert _rel(r[k], v) < 1e-13, k
    ref = dual.linear_dual(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"], x["b0"], x["ln_w"], x["ln_b"],
                           c["K"], c["eps"])
    for k in ("out", "W_last", "b_last"):
        assert _rel(ref[k], c["expected"][k]) < 1e-10, k


def test_mlp_small_case(orc):
    c = _G["mlp_d4_h8_K3_L7"]
    x = {k: np.array(v) for k, v in c["inputs"].items()}
    args = (x["XQ"], x["XK"], x["XV"], x["lr"], x["W1"], x["b1"], x["W2"], x["b2"], x["ln_w"], x["ln_b"],
            c["K"], c["eps"])
    r = orc.mlp_chain(*args)
    for k, v in c["expected"].items():
        assert _rel(r[k], v) < 1e-13, k
    ref = dual.mlp_dual(*args)
    for k in c["expected"]:
        assert _rel(ref[k], c["expected"][k]) < 1e-10, k
