"""Independent CPU implementation of the DUAL form, used only to pin the oracle.

The oracle (oracle/ttt_oracle.c) follows the primal branch of compute_mini_batch token by token
with a hand-derived LayerNorm backward.  This module follows the DUAL branch of the same listing
("代码连连看——TTT", compute_mini_batch, ``use_dual_form``) in matrix form, in torch float64, and
takes every gradient from torch autograd through ``torch.nn.functional.layer_norm`` and
``torch.nn.functional.gelu(approximate="tanh")`` -- no code is shared with the oracle.
"""
from __future__ import annotations

import torch
import torch.nn.functional as F


def _t(a):
    return torch.as_tensor(a, dtype=torch.float64)


def layer_norm(u, ln_w, ln_b, eps):
    return F.layer_norm(u, (u.shape[-1],), ln_w, ln_b, eps)


def lnl2_grad_autograd(Z, tgt, ln_w, ln_b, eps):
    """d/dZ of sum over rows of 1/2 * ||LN(Z_row) - tgt_row||^2, by autograd."""
    Z = _t(Z).clone().requires_grad_(True)
    loss = 0.5 * ((layer_norm(Z, _t(ln_w), _t(ln_b), eps) - _t(tgt)) ** 2).sum()
    (g,) = torch.autograd.grad(loss, Z)
    return g


def eta_matrix(lr_mb, token_eta=None):
    """eta[i, j] = token_eta_i * lr_j (unmasked; callers apply tril)."""
    K = lr_mb.shape[0]
    te = 1.0 / torch.arange(1, K + 1, dtype=torch.float64) if token_eta is None else _t(token_eta)[:K]
    return te[:, None] * lr_mb[None, :]


def linear_dual(xq, xk, xv, lr, W0, b0, ln_w, ln_b, K, eps, token_eta=None):
    """One chain of TTT-Linear: full mini-batches of K, then the remainder with K = r
    from the carried (W, b) (TTTBase.forward); returns out, W_last, b_last (state after the
    full mini-batches, the remainder's params being dropped)."""
    xq, xk, xv, lr = map(_t, (xq, xk, xv, lr))
    W, b = _t(W0).clone(), _t(b0).clone()
    ln_w, ln_b = _t(ln_w), _t(ln_b)
    L = xq.shape[0]
    n_full, r = L // K, L % K
    outs = []
    for m in range(n_full + (1 if r else 0)):
        Km = K if m < n_full else r
        s = slice(m * K, m * K + Km)
        XQ, X1, XV = xq[s], xk[s], xv[s]
        Z1 = X1 @ W + b
        g = lnl2_grad_autograd(Z1, XV - X1, ln_w, ln_b, eps)
        eta = eta_matrix(lr[s], token_eta)
        Attn = torch.tril(XQ @ X1.T)
        b_bar = b - torch.tril(eta) @ g
        Z_bar = XQ @ W - (eta * Attn) @ g + b_bar
        outs.append(XQ + layer_norm(Z_bar, ln_w, ln_b, eps))
        if m < n_full:
            last = eta[-1, :, None]
            W = W - (last * X1).T @ g
            b = b - (last * g).sum(0)
    out = torch.cat(outs) if outs else torch.zeros((0, xq.shape[1]), dtype=torch.float64)
    return {"out": out.numpy(), "W_last": W.numpy(), "b_last": b.numpy()}


def mlp_dual(xq, xk, xv, lr, W1, b1, W2, b2, ln_w, ln_b, K, eps, token_eta=None):
    """One chain of TTT-MLP, layer-wise dual form: each layer of the two-layer state takes the
    TTT-Linear dual update with its own input (XK for layer 1, gelu(Z1) for layer 2) and its own
    gradient, both gradients coming from autograd through the whole MLP."""
    xq, xk, xv, lr = map(_t, (xq, xk, xv, lr))
    W1, b1, W2, b2 = (_t(a).clone() for a in (W1, b1, W2, b2))
    ln_w, ln_b = _t(ln_w), _t(ln_b)
    L = xq.shape[0]
    n_full, r = L // K, L % K
    outs = []
    for m in range(n_full + (1 if r else 0)):
        Km = K if m < n_full else r
        s = slice(m * K, m * K + Km)
        XQ, X1, XV = xq[s], xk[s], xv[s]
        Z1 = (X1 @ W1 + b1).requires_grad_(True)
        X2 = F.gelu(Z1, approximate="tanh")
        Z2 = X2 @ W2 + b2
        loss = 0.5 * ((layer_norm(Z2, ln_w, ln_b, eps) - (XV - X1)) ** 2).sum()
        g1, g2 = torch.autograd.grad(loss, (Z1, Z2))
        X2 = X2.detach()
        eta = eta_matrix(lr[s], token_eta)
        Attn1 = torch.tril(XQ @ X1.T)
        Z1_bar = XQ @ W1 - (eta * Attn1) @ g1 + (b1 - torch.tril(eta) @ g1)
        X2_bar = F.gelu(Z1_bar, approximate="tanh")
        Attn2 = torch.tril(X2_bar @ X2.T)
        Z2_bar = X2_bar @ W2 - (eta * Attn2) @ g2 + (b2 - torch.tril(eta) @ g2)
        outs.append(XQ + layer_norm(Z2_bar, ln_w, ln_b, eps))
        if m < n_full:
            last = eta[-1, :, None]
            W1 = W1 - (last * X1).T @ g1
            b1 = b1 - (last * g1).sum(0)
            W2 = W2 - (last * X2).T @ g2
            b2 = b2 - (last * g2).sum(0)
    out = torch.cat(outs) if outs else torch.zeros((0, xq.shape[1]), dtype=torch.float64)
    return {"out": out.numpy(), "W1_last": W1.detach().numpy(), "b1_last": b1.detach().numpy(),
            "W2_last": W2.detach().numpy(), "b2_last": b2.detach().numpy()}
