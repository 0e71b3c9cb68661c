"""Pins of the CPU oracle against facts that do not come from the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError on a mismatch.  They are run on
the real oracle (test_oracle_pins.py) and on builds of it with planted mistakes
(test_oracle_mutants.py), where at least one pin must fail per mistake.

What pins what:
  * LayerNorm forward, tanh-GELU and its derivative: library routines (torch F.layer_norm,
    F.gelu(approximate="tanh"), autograd).
  * LN-L2 gradient: central finite differences of the loss, and autograd.
  * The whole TTT-Linear / TTT-MLP scan: the dual branch of compute_mini_batch, implemented
    independently in tests/dual_form.py (matrix form, autograd gradients), against the
    oracle's primal branch -- the two are printed side by side on the walkthrough page as
    interchangeable.
  * Closed forms: eta = 0 (no learning) gives out = XQ + LN(XQ W0 + b0); a zero state gives
    g = (q - mean q) / sqrt(eps) for the first mini-batch.
  * Mini-batch size 1 is online gradient descent with autograd gradients w.r.t. W directly.
  * Tiny brute force: the state after each mini-batch equals W minus the eta-weighted sum of
    central-difference gradients of the per-token losses w.r.t. every entry of W and b.
  * Structure: a mini-batch moves W by a matrix of rank <= K; with eta = 0 out ignores XV;
    splitting a sequence at a mini-batch boundary and carrying (W, b) changes nothing;
    decode steps from a carried cache reproduce the prefill.
  * Integers: the partition equals floor division / remainder.
  * Rotary position embedding (applied to XQ, XK before the scan): position 0 is the identity,
    every rotated pair keeps its norm, dot products depend only on the difference of positions,
    and a torch restatement of the rotate-half form (with the pair permutation that permute_qk /
    undo_permute_qk perform, for the interleaved convention) gives the same values.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.nn.functional as F

import dual_form as dual

RTOL_EXACT = 1e-10  # two fp64 formulations of one function


def _rel(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


def _rng(seed):
    return np.random.default_rng(seed)


def _chain(rng, L, d, x_std=0.5, w_std=0.2, bias=True, ln_random=True):
    xq = rng.normal(0, x_std, (L, d))
    xk = rng.normal(0, x_std, (L, d))
    xv = rng.normal(0, x_std, (L, d))
    lr = 1.0 / (1.0 + np.exp(-rng.normal(0, 1, L)))  # positive rates
    W0 = rng.normal(0, w_std, (d, d))
    b0 = rng.normal(0, 0.1, d) if bias else np.zeros(d)
    ln_w = 1.0 + rng.normal(0, 0.2, d) if ln_random else np.ones(d)
    ln_b = rng.normal(0, 0.2, d) if ln_random else np.zeros(d)
    return xq, xk, xv, lr, W0, b0, ln_w, ln_b


# ------------------------------------------------------------------------------------------
def pin_partition(o):
    for K in (1, 2, 3, 16):
        for L in (0, 1, 2, 15, 16, 17, 31, 32, 33, 8192, 8200):
            assert o.partition(L, K) == (L // K, L % K), (L, K)


def pin_ln_forward_library(o):
    rng = _rng(1)
    for d in (4, 64):
        u = rng.normal(0.3, 2.0, d)
        w, b = rng.normal(1, 0.3, d), rng.normal(0, 0.3, d)
        for eps in (1e-6, 1e-5, 0.3):
            ref = F.layer_norm(torch.tensor(u), (d,), torch.tensor(w), torch.tensor(b), eps).numpy()
            assert _rel(o.ln_forward(u, w, b, eps), ref) < 1e-13, (d, eps)


def pin_lnl2_grad_finite_differences(o):
    rng = _rng(2)
    d, eps, h = 64, 1e-5, 1e-5
    z = rng.normal(0.1, 0.7, d)
    tgt, w, b = rng.normal(0, 1, d), rng.normal(1, 0.3, d), rng.normal(0, 0.3, d)

    def loss(zz):  # the loss written from its definition, LN from the library
        y = F.layer_norm(torch.tensor(zz), (d,), torch.tensor(w), torch.tensor(b), eps).numpy()
        return 0.5 * np.sum((y - tgt) ** 2)

    fd = np.array([(loss(z + h * e) - loss(z - h * e)) / (2 * h) for e in np.eye(d)])
    assert _rel(o.lnl2_grad(z, tgt, w, b, eps), fd) < 1e-7


def pin_lnl2_grad_autograd(o):
    rng = _rng(3)
    for d, eps in ((64, 1e-6), (64, 1e-5), (8, 1e-2)):
        z = rng.normal(-0.2, 0.05, d)
        tgt, w, b = rng.normal(0, 1, d), rng.normal(1, 0.3, d), rng.normal(0, 0.3, d)
        ref = dual.lnl2_grad_autograd(z[None], tgt[None], w, b, eps)[0].numpy()
        assert _rel(o.lnl2_grad(z, tgt, w, b, eps), ref) < 1e-11, (d, eps)


def pin_gelu_library(o):
    x = np.linspace(-6, 6, 241)
    y, dy = o.gelu(x)
    xt = torch.tensor(x, requires_grad=True)
    yt = F.gelu(xt, approximate="tanh")
    (gt,) = torch.autograd.grad(yt.sum(), xt)
    assert _rel(y, yt.detach().numpy()) < 1e-14
    assert _rel(dy, gt.numpy()) < 1e-13


def pin_linear_dual_equals_primal(o):
    rng = _rng(4)
    cases = [(64, 64, 16, None), (37, 64, 16, None), (5, 64, 16, None), (48, 16, 4, None),
             (50, 16, 8, "table"), (16, 64, 16, None), (3, 8, 1, None)]
    for L, d, K, te in cases:
        xq, xk, xv, lr, W0, b0, w, b = _chain(rng, L, d, w_std=0.3 / np.sqrt(d) * 4)
        token_eta = rng.uniform(0.05, 1.0, K) if te else None
        got = o.linear_chain(xq, xk, xv, lr, W0, b0, w, b, K, 1e-6, token_eta)
        ref = dual.linear_dual(xq, xk, xv, lr, W0, b0, w, b, K, 1e-6, token_eta)
        for k in ("out", "W_last", "b_last"):
            assert _rel(got[k], ref[k]) < RTOL_EXACT, (L, d, K, te, k, _rel(got[k], ref[k]))


def pin_linear_eta_zero_closed_form(o):
    rng = _rng(5)
    L, d, K = 40, 64, 16
    xq, xk, xv, lr, W0, b0, w, b = _chain(rng, L, d)
    got = o.linear_chain(xq, xk, xv, np.zeros(L), W0, b0, w, b, K, 1e-6)
    ref = xq + F.layer_norm(torch.tensor(xq @ W0 + b0), (d,), torch.tensor(w), torch.tensor(b),
                            1e-6).numpy()
    assert _rel(got["out"], ref) < 1e-13
    assert np.array_equal(got["W_last"], W0) and np.array_equal(got["b_last"], b0)
    # with nothing learned, out cannot depend on the reconstruction target XV
    got2 = o.linear_chain(xq, xk, xv + 3.0, np.zeros(L), W0, b0, w, b, K, 1e-6)
    assert np.array_equal(got["out"], got2["out"])


def pin_linear_zero_state_closed_form(o):
    rng = _rng(6)
    L, d, K, eps = 16, 64, 16, 1e-6
    xq, xk, xv, lr, _, _, w, b = _chain(rng, L, d)
    got = o.linear_chain(xq, xk, xv, lr, np.zeros((d, d)), np.zeros(d), w, b, K, eps)
    # z = 0 -> xhat = 0, sigma = sqrt(eps): g = (q - mean q) / sqrt(eps), q = w * (b - (xv - xk))
    q = w * (b - (xv - xk))
    g = (q - q.mean(axis=1, keepdims=True)) / np.sqrt(eps)
    W_ref = -(1.0 / K) * (lr[:, None] * xk).T @ g
    b_ref = -(1.0 / K) * (lr[:, None] * g).sum(0)
    assert _rel(got["W_last"], W_ref) < 1e-12
    assert _rel(got["b_last"], b_ref) < 1e-12


def pin_linear_online_gd(o):
    """K = 1: W <- W - lr * dl/dW (autograd w.r.t. W), out at the updated W."""
    rng = _rng(7)
    L, d, eps = 12, 16, 1e-6
    xq, xk, xv, lr, W0, b0, w, b = _chain(rng, L, d)
    W, bb = torch.tensor(W0), torch.tensor(b0)
    wt, bt = torch.tensor(w), torch.tensor(b)
    outs = []
    for t in range(L):
        Wv, bv = W.clone().requires_grad_(True), bb.clone().requires_grad_(True)
        z = torch.tensor(xk[t]) @ Wv + bv
        loss = 0.5 * ((F.layer_norm(z, (d,), wt, bt, eps) - torch.tensor(xv[t] - xk[t])) ** 2).sum()
        gW, gb = torch.autograd.grad(loss, (Wv, bv))
        W, bb = W - lr[t] * gW, bb - lr[t] * gb
        zq = torch.tensor(xq[t]) @ W + bb
        outs.append(xq[t] + F.layer_norm(zq, (d,), wt, bt, eps).numpy())
    got = o.linear_chain(xq, xk, xv, lr, W0, b0, w, b, 1, eps)
    assert _rel(got["out"], np.stack(outs)) < 1e-11
    assert _rel(got["W_last"], W.numpy()) < 1e-11
    assert _rel(got["b_last"], bb.numpy()) < 1e-11


def pin_linear_brute_force_tiny(o):
    """d=4, K=2, L=4: state after each mini-batch from central differences w.r.t. W and b."""
    rng = _rng(8)
    L, d, K, eps, h = 4, 4, 2, 1e-3, 1e-6
    xq, xk, xv, lr, W0, b0, w, b = _chain(rng, L, d, w_std=0.5)

    def loss(W, bb, t):
        z = xk[t] @ W + bb
        mu = z.mean()
        y = w * (z - mu) / np.sqrt(((z - mu) ** 2).mean() + eps) + b
        return 0.5 * np.sum((y - (xv[t] - xk[t])) ** 2)

    W, bb = W0.copy(), b0.copy()
    for m in range(L // K):
        dW, db = np.zeros_like(W), np.zeros_like(bb)
        for j in range(K):
            t = m * K + j
            eta_last = lr[t] / K
            for a in range(d):
                for c in range(d):
                    E = np.zeros_like(W)
                    E[a, c] = h
                    dW[a, c] += eta_last * (loss(W + E, bb, t) - loss(W - E, bb, t)) / (2 * h)
                e = np.zeros(d)
                e[a] = h
                db[a] += eta_last * (loss(W, bb + e, t) - loss(W, bb - e, t)) / (2 * h)
        W, bb = W - dW, bb - db
    got = o.linear_chain(xq, xk, xv, lr, W0, b0, w, b, K, eps)
    assert _rel(got["W_last"], W) < 1e-7, _rel(got["W_last"], W)
    assert _rel(got["b_last"], bb) < 1e-7


def pin_linear_update_rank(o):
    rng = _rng(9)
    d, K = 32, 4
    xq, xk, xv, lr, W0, b0, w, b = _chain(rng, 2 * K, d)
    one = o.linear_chain(xq[:K], xk[:K], xv[:K], lr[:K], W0, b0, w, b, K, 1e-6)
    two = o.linear_chain(xq, xk, xv, lr, W0, b0, w, b, K, 1e-6)
    for delta in (one["W_last"] - W0, two["W_last"] - one["W_last"]):
        s = np.linalg.svd(delta, compute_uv=False)
        assert s[K] < 1e-12 * s[0] and s[K - 1] > 1e-6 * s[0], s[: K + 2]


def pin_linear_split_and_carry(o):
    rng = _rng(10)
    d, K = 64, 16
    xq, xk, xv, lr, W0, b0, w, b = _chain(rng, 69, d)
    whole = o.linear_chain(xq, xk, xv, lr, W0, b0, w, b, K, 1e-6)
    # split at a mini-batch boundary, carrying (W, b)
    a = o.linear_chain(xq[:32], xk[:32], xv[:32], lr[:32], W0, b0, w, b, K, 1e-6)
    c = o.linear_chain(xq[32:], xk[32:], xv[32:], lr[32:], a["W_last"], a["b_last"], w, b, K, 1e-6)
    assert _rel(np.concatenate([a["out"], c["out"]]), whole["out"]) < 1e-13
    assert _rel(c["W_last"], whole["W_last"]) < 1e-13
    # full part, then the remainder as its own call with mini-batch size r (TTTBase.forward)
    full = o.linear_chain(xq[:64], xk[:64], xv[:64], lr[:64], W0, b0, w, b, K, 1e-6)
    tail = o.linear_chain(xq[64:], xk[64:], xv[64:], lr[64:], full["W_last"], full["b_last"], w, b,
                          5, 1e-6)
    assert _rel(np.concatenate([full["out"], tail["out"]]), whole["out"]) < 1e-13
    assert np.array_equal(whole["W_last"], full["W_last"])


def pin_decode_equals_prefill(o):
    """Cache continuation: prefill L0 tokens, then one decode step per token, equals one prefill
    over all tokens; W, b match the prefill state at every mini-batch boundary."""
    rng = _rng(11)
    d, K, eps = 16, 4, 1e-6
    L0, L = 6, 17
    xq, xk, xv, lr, W0, b0, w, b = _chain(rng, L, d)
    pre = o.linear_chain(xq[:L0], xk[:L0], xv[:L0], lr[:L0], W0, b0, w, b, K, eps)
    W, bb = pre["W_last"].copy(), pre["b_last"].copy()
    Wg, bg = pre["W_grad_tail"].copy(), pre["b_grad_tail"].copy()
    whole = o.linear_chain(xq, xk, xv, lr, W0, b0, w, b, K, eps)
    for t in range(L0, L):
        out, committed = o.decode_chain(xq[t], xk[t], xv[t], lr[t], w, b, W, bb, Wg, bg, K, t, eps)
        assert committed == ((t + 1) % K == 0)
        assert _rel(out, whole["out"][t]) < 1e-12, t
        if committed:
            ref = o.linear_chain(xq[:t + 1], xk[:t + 1], xv[:t + 1], lr[:t + 1], W0, b0, w, b, K, eps)
            assert _rel(W, ref["W_last"]) < 1e-12 and _rel(bb, ref["b_last"]) < 1e-12
            assert not Wg.any() and not bg.any()


def pin_mlp_gelu_path_dual_equals_primal(o):
    rng = _rng(12)
    for L, d, hdim, K in ((37, 16, 64, 16), (20, 8, 32, 4), (16, 64, 256, 16)):
        xq, xk, xv, lr, _, _, w, b = _chain(rng, L, d)
        W1 = rng.normal(0, 0.5 / np.sqrt(d), (d, hdim))
        W2 = rng.normal(0, 0.5 / np.sqrt(hdim), (hdim, d))
        b1, b2 = rng.normal(0, 0.1, hdim), rng.normal(0, 0.1, d)
        got = o.mlp_chain(xq, xk, xv, lr, W1, b1, W2, b2, w, b, K, 1e-6)
        ref = dual.mlp_dual(xq, xk, xv, lr, W1, b1, W2, b2, w, b, K, 1e-6)
        for k in ("out", "W1_last", "b1_last", "W2_last", "b2_last"):
            assert _rel(got[k], ref[k]) < RTOL_EXACT, (L, d, hdim, K, k, _rel(got[k], ref[k]))


def pin_mlp_eta_zero_closed_form(o):
    rng = _rng(13)
    L, d, hdim, K = 20, 16, 64, 16
    xq, xk, xv, _, _, _, w, b = _chain(rng, L, d)
    W1, W2 = rng.normal(0, 0.2, (d, hdim)), rng.normal(0, 0.2, (hdim, d))
    b1, b2 = rng.normal(0, 0.1, hdim), rng.normal(0, 0.1, d)
    got = o.mlp_chain(xq, xk, xv, np.zeros(L), W1, b1, W2, b2, w, b, K, 1e-6)
    hid = F.gelu(torch.tensor(xq @ W1 + b1), approximate="tanh").numpy()
    ref = xq + F.layer_norm(torch.tensor(hid @ W2 + b2), (d,), torch.tensor(w), torch.tensor(b),
                            1e-6).numpy()
    assert _rel(got["out"], ref) < 1e-13
    assert np.array_equal(got["W1_last"], W1) and np.array_equal(got["W2_last"], W2)


def pin_mlp_online_gd(o):
    rng = _rng(14)
    L, d, hdim, eps = 6, 8, 16, 1e-6
    xq, xk, xv, lr, _, _, w, b = _chain(rng, L, d)
    W1, W2 = rng.normal(0, 0.4, (d, hdim)), rng.normal(0, 0.4, (hdim, d))
    b1, b2 = rng.normal(0, 0.1, hdim), rng.normal(0, 0.1, d)
    P = [torch.tensor(a) for a in (W1, b1, W2, b2)]
    wt, bt = torch.tensor(w), torch.tensor(b)

    def f(params, x):
        A1, c1, A2, c2 = params
        return F.gelu(x @ A1 + c1, approximate="tanh") @ A2 + c2

    outs = []
    for t in range(L):
        Pv = [p.clone().requires_grad_(True) for p in P]
        z = f(Pv, torch.tensor(xk[t]))
        loss = 0.5 * ((F.layer_norm(z, (d,), wt, bt, eps) - torch.tensor(xv[t] - xk[t])) ** 2).sum()
        grads = torch.autograd.grad(loss, Pv)
        P = [p - lr[t] * gp for p, gp in zip(P, grads)]
        outs.append(xq[t] + F.layer_norm(f(P, torch.tensor(xq[t])), (d,), wt, bt, eps).numpy())
    got = o.mlp_chain(xq, xk, xv, lr, W1, b1, W2, b2, w, b, 1, eps)
    assert _rel(got["out"], np.stack(outs)) < 1e-11
    for k, ref in zip(("W1_last", "b1_last", "W2_last", "b2_last"), P):
        assert _rel(got[k], ref.numpy()) < 1e-11, k


def pin_mlp_split_and_carry(o):
    rng = _rng(15)
    L, d, hdim, K = 40, 16, 32, 8
    xq, xk, xv, lr, _, _, w, b = _chain(rng, L, d)
    W1, W2 = rng.normal(0, 0.3, (d, hdim)), rng.normal(0, 0.3, (hdim, d))
    b1, b2 = rng.normal(0, 0.1, hdim), rng.normal(0, 0.1, d)
    whole = o.mlp_chain(xq, xk, xv, lr, W1, b1, W2, b2, w, b, K, 1e-6)
    a = o.mlp_chain(xq[:24], xk[:24], xv[:24], lr[:24], W1, b1, W2, b2, w, b, K, 1e-6)
    c = o.mlp_chain(xq[24:], xk[24:], xv[24:], lr[24:], a["W1_last"], a["b1_last"], a["W2_last"],
                    a["b2_last"], w, b, K, 1e-6)
    assert _rel(np.concatenate([a["out"], c["out"]]), whole["out"]) < 1e-13
    assert _rel(c["W2_last"], whole["W2_last"]) < 1e-13


def _rope_torch(x, K, theta, interleaved):
    """The rotate-half rotary embedding written with torch ops (cos/sin tables over positions
    t mod K, q * cos + rotate_half(q) * sin); for the interleaved convention the features are
    first permuted from adjacent pairs (2k, 2k+1) to halves (k, k + d/2) and back afterwards."""
    x = torch.as_tensor(x, dtype=torch.float64)
    L, d = x.shape[-2], x.shape[-1]
    inv_freq = 1.0 / (theta ** (torch.arange(0, d, 2, dtype=torch.float64) / d))
    pos = torch.arange(L, dtype=torch.float64) % K
    freqs = torch.outer(pos, inv_freq)
    emb = torch.cat([freqs, freqs], dim=-1)
    cos, sin = emb.cos(), emb.sin()
    if interleaved:
        x = x.reshape(*x.shape[:-1], d // 2, 2).transpose(-1, -2).reshape(*x.shape[:-1], d)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    y = x * cos + torch.cat([-x2, x1], dim=-1) * sin
    if interleaved:
        y = y.reshape(*y.shape[:-1], 2, d // 2).transpose(-1, -2).reshape(*y.shape[:-1], d)
    return y.numpy()


def pin_rope_position_zero_and_pair_norms(o):
    rng = _rng(21)
    L, d, K = 37, 16, 8
    x = rng.normal(0, 1, (L, d))
    for half in (False, True):
        y = o.rope(x, K, 500.0, half)
        assert np.array_equal(y[::K], x[::K])  # positions 0 (t = 0, K, 2K, ...) do not move
        a = np.arange(d // 2) if half else 2 * np.arange(d // 2)
        b = a + d // 2 if half else a + 1
        assert np.allclose(np.hypot(y[:, a], y[:, b]), np.hypot(x[:, a], x[:, b]), rtol=1e-13, atol=0)
        assert not np.allclose(y[1], x[1])


def pin_rope_relative_position(o):
    # <R(p1) q, R(p2) k> = <q, R(p2 - p1) k>: rows p1, p2 of one array against row p2 - p1 of another
    rng = _rng(22)
    d, K = 16, 16
    q, k = rng.normal(0, 1, d), rng.normal(0, 1, d)
    for half in (False, True):
        for p1, p2 in ((3, 11), (5, 5), (0, 15)):
            Aq, Ak, B = np.zeros((K, d)), np.zeros((K, d)), np.zeros((K, d))
            Aq[p1], Ak[p2], B[p2 - p1] = q, k, k
            yq, yk, yB = (o.rope(X, K, 10000.0, half) for X in (Aq, Ak, B))
            assert abs(yq[p1] @ yk[p2] - q @ yB[p2 - p1]) < 1e-12 * (1 + abs(q @ k))


def pin_rope_torch_restatement(o):
    rng = _rng(23)
    x = rng.normal(0, 1, (3, 41, 64))
    for half in (False, True):
        for theta in (10000.0, 37.0):
            assert _rel(o.rope(x, 16, theta, half), _rope_torch(x, 16, theta, not half)) < 1e-13


def _post_norm_case(seed, T=9, C=24, N=10):
    rng = _rng(seed)
    x = rng.normal(0.3, 1.5, (T, C))
    return x, 1 + rng.normal(0, 0.2, C), rng.normal(0, 0.2, C), rng.normal(0, 0.3, (N, C))


def pin_post_norm_identity_is_layer_norm(o):
    # o_proj = identity reduces the step to a LayerNorm over the token's C features
    x, w, b, _ = _post_norm_case(31)
    ref = torch.nn.functional.layer_norm(torch.as_tensor(x), (x.shape[1],), torch.as_tensor(w),
                                         torch.as_tensor(b), eps=1e-5).numpy()
    assert _rel(o.post_norm_o_proj(x, w, b, 1e-5, np.eye(x.shape[1])), ref) < 1e-13


def pin_post_norm_single_entry_weight(o):
    # a weight with one nonzero entry Wo[n0][k0] copies feature k0 of the normalised token into
    # output n0 and nothing else (fixes the orientation of Wo)
    x, w, b, _ = _post_norm_case(32)
    C = x.shape[1]
    ln = o.post_norm_o_proj(x, w, b, 1e-5, np.eye(C))
    Wo = np.zeros((7, C))
    Wo[5, 2] = 2.5
    y = o.post_norm_o_proj(x, w, b, 1e-5, Wo)
    assert np.allclose(y[:, 5], 2.5 * ln[:, 2], rtol=1e-13, atol=1e-14)
    assert not np.delete(y, 5, axis=1).any()


def pin_post_norm_invariances(o):
    # linear in Wo; blind to a per-token shift of x; with ln_w = 0 every token maps to Wo ln_b
    x, w, b, W1 = _post_norm_case(33)
    W2 = _rng(34).normal(0, 0.3, W1.shape)
    y1, y2 = o.post_norm_o_proj(x, w, b, 1e-5, W1), o.post_norm_o_proj(x, w, b, 1e-5, W2)
    assert _rel(o.post_norm_o_proj(x, w, b, 1e-5, W1 + 2 * W2), y1 + 2 * y2) < 1e-13
    shift = _rng(35).normal(0, 3, (x.shape[0], 1))
    assert _rel(o.post_norm_o_proj(x + shift, w, b, 1e-5, W1), y1) < 1e-12
    y0 = o.post_norm_o_proj(x, np.zeros_like(w), b, 1e-5, W1)
    assert np.allclose(y0, np.broadcast_to(W1 @ b, y0.shape), rtol=1e-13, atol=1e-14)


PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
