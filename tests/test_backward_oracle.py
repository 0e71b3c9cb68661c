"""Pins of the backward oracle (oracle/ttt_backward.py), all on the CPU.

The backward oracle differentiates its own torch restatement of the scan, so it is pinned to
things outside itself:
  * its forward equals the C oracle's (oracle/ttt_oracle.c) to rounding;
  * its gradients equal central finite differences of the C oracle's forward, along random
    directions of every input and entry by entry at random positions;
  * with lr = 0 the scan reduces to out = XQ + LN(XQ W0 + b0) with the state left alone, whose
    gradients torch's own layer_norm gives, and XK and XV then receive exactly zero.
Planted mistakes in the backward oracle (a detached statistic, a state that stops carrying
gradient, a dropped upstream term, a wrong operand) each fail one of these.
"""
import types

import numpy as np
import pytest
import torch

from oracle import ttt_backward as bw

D = 64
NAMES = ("xq", "xk", "xv", "lr", "W0", "b0", "ln_w", "ln_b")
GRAD = {"xq": "dXQ", "xk": "dXK", "xv": "dXV", "lr": "dlr", "W0": "dW0", "b0": "db0", "ln_w": "dln_w",
        "ln_b": "dln_b"}


def _case(seed, n, L, lr_scale=4.0):
    """Inputs in the range of the workloads, with a larger lr and W0 so that the state path and
    the LayerNorm nonlinearity both carry weight in the gradients."""
    rng = np.random.default_rng(seed)
    x = {k: rng.standard_normal((n, L, D)) / 8 for k in ("xq", "xk", "xv")}
    x["lr"] = lr_scale / (1 + np.exp(-rng.standard_normal((n, L)))) / D
    x["W0"] = rng.standard_normal((n, D, D)) * 0.1
    x["b0"] = rng.standard_normal((n, D)) * 0.1
    x["ln_w"] = 1 + 0.3 * rng.standard_normal((n, D))
    x["ln_b"] = 0.3 * rng.standard_normal((n, D))
    up = {"d_out": rng.standard_normal((n, L, D)), "dW_last": rng.standard_normal((n, D, D)),
          "db_last": rng.standard_normal((n, D))}
    return x, up


def _c_loss(orc, x, up, K, eps, token_eta=None):
    """<d_out, out> + <dW_last, W_last> + <db_last, b_last> from the C oracle's forward."""
    tot = 0.0
    for c in range(x["xq"].shape[0]):
        r = orc.linear_chain(*(x[k][c] for k in NAMES), K=K, eps=eps, token_eta=token_eta)
        tot += float((r["out"] * up["d_out"][c]).sum() + (r["W_last"] * up["dW_last"][c]).sum()
                     + (r["b_last"] * up["db_last"][c]).sum())
    return tot


def _grads(mod, x, up, K, eps, token_eta=None):
    return mod.linear_backward(*(x[k] for k in NAMES), K=K, eps=eps, d_out=up["d_out"], dW_last=up["dW_last"],
                               db_last=up["db_last"], token_eta=token_eta)


CASES = [  # (seed, chains, L, K, token_eta): full mini-batches and a remainder tail in each
    (1, 2, 21, 4, None),
    (2, 1, 37, 16, None),
    (3, 2, 9, 3, [0.9, 0.4, 0.25]),
]


def pin_forward_matches_c_oracle(orc, mod):
    for seed, n, L, K, te in CASES:
        x, up = _case(seed, n, L)
        r = _grads(mod, x, up, K, 1e-6, te)
        for c in range(n):
            ref = orc.linear_chain(*(x[k][c] for k in NAMES), K=K, eps=1e-6, token_eta=te)
            for k in ("out", "W_last", "b_last"):
                err = np.abs(r[k][c] - ref[k]).max() / max(np.abs(ref[k]).max(), 1e-300)
                assert err < 1e-12, (seed, k, err)


def pin_gradients_match_directional_differences(orc, mod):
    for seed, n, L, K, te in CASES:
        x, up = _case(seed, n, L)
        r = _grads(mod, x, up, K, 1e-6, te)
        rng = np.random.default_rng(seed + 100)
        for name in NAMES:
            v = rng.standard_normal(x[name].shape) * (np.sqrt((x[name] ** 2).mean()) or 1.0)

            def cd(h):  # central difference along v
                xp, xm = dict(x), dict(x)
                xp[name], xm[name] = x[name] + h * v, x[name] - h * v
                return (_c_loss(orc, xp, up, K, 1e-6, te) - _c_loss(orc, xm, up, K, 1e-6, te)) / (2 * h)

            fd = (4 * cd(5e-5) - cd(1e-4)) / 3  # Richardson: the h^2 term cancels
            an = float((r[GRAD[name]] * v).sum())
            assert abs(fd - an) <= 1e-7 * max(abs(fd), abs(an)) + 1e-10, (seed, name, fd, an)


def pin_gradients_match_entrywise_differences(orc, mod):
    seed, n, L, K, te = CASES[0]
    x, up = _case(seed, n, L)
    r = _grads(mod, x, up, K, 1e-6, te)
    rng = np.random.default_rng(7)
    for name in NAMES:
        g = r[GRAD[name]]
        scale = np.sqrt((g ** 2).mean())
        for _ in range(3):
            idx = tuple(rng.integers(0, s) for s in x[name].shape)
            h = 1e-5 * max(abs(x[name][idx]), 1e-2)
            xp, xm = dict(x), dict(x)
            xp[name], xm[name] = x[name].copy(), x[name].copy()
            xp[name][idx] += h
            xm[name][idx] -= h
            fd = (_c_loss(orc, xp, up, K, 1e-6, te) - _c_loss(orc, xm, up, K, 1e-6, te)) / (2 * h)
            assert abs(fd - g[idx]) <= 1e-5 * (abs(g[idx]) + scale), (name, idx, fd, g[idx])


def pin_zero_lr_reduces_to_layer_norm(orc, mod):
    x, up = _case(4, 2, 23, lr_scale=0.0)
    eps, K = 1e-5, 4
    r = _grads(mod, x, up, K, eps)
    assert not np.any(r["dXK"]) and not np.any(r["dXV"])
    for c in range(2):
        t = {k: torch.tensor(x[k][c], dtype=torch.float64, requires_grad=True) for k in ("xq", "W0", "b0", "ln_w", "ln_b")}
        u = t["xq"] @ t["W0"] + t["b0"]
        out = t["xq"] + torch.nn.functional.layer_norm(u, (D,), t["ln_w"], t["ln_b"], eps)
        loss = (out * torch.tensor(up["d_out"][c])).sum() + (t["W0"] * torch.tensor(up["dW_last"][c])).sum() \
            + (t["b0"] * torch.tensor(up["db_last"][c])).sum()
        gr = torch.autograd.grad(loss, [t[k] for k in ("xq", "W0", "b0", "ln_w", "ln_b")])
        for k, ref in zip(("dXQ", "dW0", "db0", "dln_w", "dln_b"), gr):
            ref = ref.numpy()
            err = np.abs(r[k][c] - ref).max() / np.abs(ref).max()
            assert err < 1e-12, (k, err)


PINS = [pin_forward_matches_c_oracle, pin_gradients_match_directional_differences,
        pin_gradients_match_entrywise_differences, pin_zero_lr_reduces_to_layer_norm]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_backward_pin(orc, pin):
    pin(orc, bw)


_SRC = open(bw.__file__).read()

# (name, original text, replacement)
MUTANTS = [
    ("detached_sigma", "sigma = torch.sqrt((c * c).mean(dim=-1, keepdim=True) + eps)",
     "sigma = torch.sqrt((c * c).mean(dim=-1, keepdim=True).detach() + eps)"),
    ("state_stops_carrying", "            W, b = Wi, bi", "            W, b = Wi.detach(), bi.detach()"),
    ("dropped_dW_last", "loss = loss + (W_last * _t(dW_last)).sum()", "loss = loss"),
    ("detached_loss_gradient", "g = lnl2_grad(z, xv[:, sl] - xk[:, sl], lw, lb, eps)",
     "g = lnl2_grad(z, xv[:, sl] - xk[:, sl], lw, lb, eps).detach()"),
    ("gradient_at_query", 'z = torch.einsum("njk,nkf->njf", xk[:, sl], W)', 'z = torch.einsum("njk,nkf->njf", xq[:, sl], W)'),
    ("bias_state_not_updated", "            bi = b - ti * gb", "            bi = b - ti * gb.detach()"),
]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_backward_mutant_is_caught(orc, mutant):
    name, old, new = mutant
    assert _SRC.count(old) == 1, name
    mod = types.ModuleType(f"ttt_backward_{name}")
    exec(compile(_SRC.replace(old, new), f"<{name}>", "exec"), mod.__dict__)
    caught = []
    for pin in PINS:
        try:
            pin(orc, mod)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every backward pin"
