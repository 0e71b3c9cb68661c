"""Backward of the TTT-Linear scan: the gradients of the outer inputs, in float64.

TEST INFRASTRUCTURE ONLY: used by ``tests/`` and the bench's CPU legs.  The CUDA library never
imports or calls anything here, and nothing here imports the CUDA library.

What it computes.  The forward is the scan of the walkthrough ("代码连连看——TTT",
``TTTLinear.ttt`` and ``compute_mini_batch``), written here once more in its primal form, token by
token, with plain torch CPU operations: per mini-batch of K tokens every token's loss gradient
g_j is taken at the mini-batch-start state (W, b); token i then sees the state
W - t_i * sum_{j<=i} lr_j xk_j^T g_j (and b alike) and outputs xq_i + LN(xq_i W_i + b_i); a full
mini-batch commits its last state, the remainder tail does not.  The loss gradient is the
LayerNorm-plus-L2 gradient of the walkthrough's ``ln_fused_l2_bwd``, written out in closed
form (so that its own derivative, which the backward needs, is taken through that formula).

The backward is the gradient of the scalar

    <d_out, out> + <dW_last, W_last> + <db_last, b_last>

with respect to XQ, XK, XV, lr, W0, b0, ln_w and ln_b, taken by torch's reverse-mode
differentiation of that forward: the plain definition of the gradient, with no formula of
its own.  The walkthrough trains through the same scan (its ``scan`` call takes
``scan_checkpoint_group_size`` while training); checkpointing changes where the states come
from, not the gradient, so the oracle keeps every state and has no checkpoint parameter.

Pinned by ``tests/test_backward_oracle.py``: its forward against the C oracle, its gradients
against central finite differences of the C oracle's forward, and the eta = 0 case against
torch's own layer_norm.
"""
from __future__ import annotations

import numpy as np
import torch


def _t(a):
    return torch.as_tensor(np.ascontiguousarray(a, dtype=np.float64))


def _stats(x, eps):
    """Mean, sigma = sqrt(biased variance + eps) and x_hat of the rows of x."""
    mu = x.mean(dim=-1, keepdim=True)
    c = x - mu
    sigma = torch.sqrt((c * c).mean(dim=-1, keepdim=True) + eps)
    return mu, sigma, c / sigma


def layer_norm(u, ln_w, ln_b, eps):
    """ln_w * (u - mean) / sigma + ln_b over the last dimension."""
    _, _, xh = _stats(u, eps)
    return ln_w * xh + ln_b


def lnl2_grad(z, tgt, ln_w, ln_b, eps):
    """Gradient over z of 0.5 * ||LN(z) - tgt||^2 (the walkthrough's ln_fused_l2_bwd):
    g = (d q - sum q - x_hat sum(q x_hat)) / (d sigma), q = ln_w (ln_w x_hat + ln_b - tgt)."""
    d = z.shape[-1]
    _, sigma, xh = _stats(z, eps)
    q = ln_w * (ln_w * xh + ln_b - tgt)
    return (d * q - q.sum(dim=-1, keepdim=True) - xh * (q * xh).sum(dim=-1, keepdim=True)) / (d * sigma)


def linear_forward(xq, xk, xv, lr, W0, b0, ln_w, ln_b, K, eps, token_eta=None):
    """The scan over n chains at once: xq/xk/xv [n, L, d], lr [n, L], W0 [n, d, d], b0 [n, d],
    ln_w/ln_b [n, d] (torch float64).  Returns (out [n, L, d], W_last [n, d, d], b_last [n, d])."""
    n, L, d = xq.shape
    W, b = W0, b0
    lw, lb = ln_w[:, None, :], ln_b[:, None, :]
    outs = []
    t0 = 0
    while t0 < L:
        Km = min(K, L - t0)
        full = Km == K
        sl = slice(t0, t0 + Km)
        # every token's gradient at the mini-batch-start state
        z = torch.einsum("njk,nkf->njf", xk[:, sl], W) + b[:, None, :]
        g = lnl2_grad(z, xv[:, sl] - xk[:, sl], lw, lb, eps)
        G = torch.zeros_like(W)
        gb = torch.zeros_like(b)
        for i in range(Km):
            ti = float(token_eta[i]) if token_eta is not None else 1.0 / (i + 1)
            li = lr[:, t0 + i]
            G = G + li[:, None, None] * xk[:, t0 + i, :, None] * g[:, i, None, :]
            gb = gb + li[:, None] * g[:, i]
            Wi = W - ti * G
            bi = b - ti * gb
            u = torch.einsum("nk,nkf->nf", xq[:, t0 + i], Wi) + bi
            outs.append(xq[:, t0 + i] + layer_norm(u, ln_w, ln_b, eps))
        if full:
            W, b = Wi, bi
        t0 += Km
    out = torch.stack(outs, dim=1) if outs else xq.new_zeros((n, 0, d))
    return out, W, b


def linear_backward(xq, xk, xv, lr, W0, b0, ln_w, ln_b, K, eps, d_out, dW_last=None, db_last=None,
                    token_eta=None):
    """Per-chain gradients (numpy float64) of <d_out, out> + <dW_last, W_last> + <db_last, b_last>.

    Inputs are per chain, stacked: xq/xk/xv/d_out [n, L, d], lr [n, L], W0 [n, d, d], b0 [n, d],
    ln_w/ln_b [n, d]; dW_last [n, d, d] and db_last [n, d] may be None (zero).  Returns a dict
    with dXQ, dXK, dXV, dlr, dW0, db0, dln_w, dln_b (each chain's own share; a head's shared
    parameters take the sum over the chains of that head).  Also returns the forward's out,
    W_last and b_last.
    """
    leaves = [_t(a).requires_grad_(True) for a in (xq, xk, xv, lr, W0, b0, ln_w, ln_b)]
    out, W_last, b_last = linear_forward(*leaves, K=K, eps=eps, token_eta=token_eta)
    loss = (out * _t(d_out)).sum()
    if dW_last is not None:
        loss = loss + (W_last * _t(dW_last)).sum()
    if db_last is not None:
        loss = loss + (b_last * _t(db_last)).sum()
    grads = torch.autograd.grad(loss, leaves, allow_unused=True)
    names = ("dXQ", "dXK", "dXV", "dlr", "dW0", "db0", "dln_w", "dln_b")
    res = {k: (torch.zeros_like(x) if gr is None else gr).detach().numpy() for k, gr, x in zip(names, grads, leaves)}
    res.update(out=out.detach().numpy(), W_last=W_last.detach().numpy(), b_last=b_last.detach().numpy())
    return res
