"""Planted mistakes in the oracle must each fail at least one pin.

Each mutant is a copy of oracle/ttt_oracle.c with one plausible mistake (a dropped term, a
wrong sign or index, a transposed operand, a wrong normaliser, a wrong commit rule), built with
gcc into a temporary directory and run through tests/pins.py.  Everything runs on the CPU.
"""
import os

import pytest

import oracle
from pins import PINS

_SRC = open(os.path.join(os.path.dirname(oracle.__file__), "ttt_oracle.c")).read()

# (name, original text, replacement, occurrence index to replace)
MUTANTS = [
    ("drop_bias_grad", "gb[c] += lri * gi[c];", "(void)0;", 0),
    ("update_sign", "Wbar[e] = W[e] - ti * G[e];", "Wbar[e] = W[e] + ti * G[e];", 0),
    ("token_eta_offset", "1.0 / (real)(i + 1)", "1.0 / (real)(i + 2)", 0),
    ("transposed_outer", "G[(size_t)a * d + c] += lri * xki[a] * gi[c];",
     "G[(size_t)c * d + a] += lri * xki[a] * gi[c];", 0),
    ("unbiased_variance", "v /= d;", "v /= (d - 1);", 0),
    ("eps_outside_sqrt", "*sigma = sqrt(v + eps);", "*sigma = sqrt(v) + eps;", 0),
    ("drop_xhat_term", " - xhat[c] * sqx) / (d * sigma)", ") / (d * sigma)", 0),
    ("target_sign", "tgt[c] = xvj[c] - xkj[c];", "tgt[c] = xkj[c] - xvj[c];", 0),
    ("commit_tail_state", "        if (full) {\n            memcpy(W, Wbar", "        if (1) {\n            memcpy(W, Wbar", 0),
    ("drop_residual", "oi[c] = xqi[c] + y[c];", "oi[c] = y[c];", 0),
    ("lr_index_shift", "real lri = lr[t0 + i];", "real lri = lr[t0 + (i + 1) % Km];", 0),
    ("grad_uses_xq", "row_times(xkj, W, b, d, d, z);", "row_times(xq + (size_t)(t0 + j) * d, W, b, d, d, z);", 0),
    ("strict_lower_triangle", "            real ti = token_eta_at(token_eta, i);\n            for (size_t e = 0; e < dd; ++e) Wbar[e] = W[e] - ti * G[e];",
     "            real ti = token_eta_at(token_eta, i);\n            for (size_t e = 0; e < dd; ++e) Wbar[e] = W[e] - ti * (G[e] - lri * xki[e / d] * gi[e % d]);", 0),
    ("ln_missing_bias", "y[c] = ln_w[c] * (u[c] - mu) / sigma + ln_b[c];", "y[c] = ln_w[c] * (u[c] - mu) / sigma;", 0),
    ("decode_commit_rule", "int commit = (p == K - 1);", "int commit = (p == 0);", 0),
    ("decode_position", "int p = (int)(offset % K);", "int p = (int)((offset + 1) % K);", 0),
    ("decode_no_grad_reset", "        memset(W_grad, 0, sizeof(real) * dd);\n        memset(b_grad, 0, sizeof(real) * d);\n    }",
     "    }", 0),
    ("gelu_deriv_factor", "(1.0 + 3.0 * 0.044715 * x * x)", "(1.0 + 0.044715 * x * x)", 0),
    ("mlp_drop_b2_grad", "gb2[c] += lri * g2i[c];", "(void)0;", 0),
    ("mlp_layer2_input", "G2[(size_t)u * d + c] += lri * x2i[u] * g2i[c];",
     "G2[(size_t)u * d + c] += lri * g1i[u] * g2i[c];", 0),
    ("mlp_no_gelu_on_query", "for (int u = 0; u < h; ++u) a1[u] = gelu_tanh(z1[u]);",
     "for (int u = 0; u < h; ++u) a1[u] = z1[u];", 0),
    ("rope_sin_sign", "yr[ia] = xa * c - xb * s;\n            yr[ib] = xa * s + xb * c;",
     "yr[ia] = xa * c + xb * s;\n            yr[ib] = -xa * s + xb * c;", 0),
    ("rope_position_not_mod_K", "const real p = (real)(t % K);", "const real p = (real)t;", 0),
    ("rope_frequency_exponent", "pow(theta, -2.0 * k / d)", "pow(theta, -1.0 * k / d)", 0),
    ("rope_pairs_swapped", "const int ia = half_split ? k : 2 * k, ib = half_split ? k + half : 2 * k + 1;",
     "const int ia = half_split ? 2 * k : k, ib = half_split ? 2 * k + 1 : k + half;", 0),
    ("o_proj_transposed", "const real* wn = Wo + (size_t)n * C;\n            real acc = 0.0;\n            for (int k = 0; k < C; ++k) acc += u[k] * wn[k];",
     "real acc = 0.0;\n            for (int k = 0; k < C && k < N; ++k) acc += u[k] * Wo[(size_t)k * C + n];", 0),
    ("post_norm_skipped", "        ln_forward(x + (size_t)t * C, ln_w, ln_b, C, eps, u);",
     "        for (int k = 0; k < C; ++k) u[k] = x[(size_t)t * C + k];", 0),
    ("post_norm_no_affine", "        ln_forward(x + (size_t)t * C, ln_w, ln_b, C, eps, u);",
     "        ln_forward(x + (size_t)t * C, ln_w, ln_b, C, eps, u);\n        for (int k = 0; k < C; ++k) u[k] = (u[k] - ln_b[k]) / ln_w[k];", 0),
]


def _mutate(src, old, new, occ):
    idx = -1
    for _ in range(occ + 1):
        idx = src.index(old, idx + 1)
    return src[:idx] + new + src[idx + len(old):]


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, occ):
    src = tmp_path / f"{name}.c"
    src.write_text(_mutate(_SRC, old, new, occ))
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / f"lib{name}.so"))
    o = oracle.Oracle(lib)
    for pin in PINS:
        try:
            pin(o)
        except (AssertionError, ValueError):
            return  # caught
    pytest.fail(f"planted mistake '{name}' passed every pin")
