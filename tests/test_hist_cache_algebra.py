"""The history-format decode cache's algebra on the CPU (no GPU): a float64 numpy step that keeps
the rows (a_j = lr_j xk_j, g_j) of the current mini-batch instead of the dense gradient sum,
written from the primal identity of TTTLinear.ttt ("代码连连看——TTT", primal branch) --

    xq W_bar = xq W - t (sum_{j<p} (xq . a_j) g_j + lr (xq . xk) g),
    b_bar    = b - t (b_grad + lr g),
    commit at p = K - 1:  W -= t sum_{j<=p} a_j^T g_j,  b = b_bar,

-- must reproduce the oracle's dense-cache decode (and hence the prefill) token for token,
across mini-batch commits.  This is the reformulation the history decode kernel computes."""
import numpy as np
import pytest


def _hist_step(o, xq, xk, xv, lr, ln_w, ln_b, W, b, rows, b_grad, K, offset, eps, te=None):
    p = offset % K
    t = te[p] if te is not None else 1.0 / (p + 1)
    g = o.lnl2_grad(xk @ W + b, xv - xk, ln_w, ln_b, eps)
    c = np.array([xq @ a for a, _ in rows])                    # xq . a_j, j < p
    xqWg = sum((cj * gj for cj, (_, gj) in zip(c, rows)), np.zeros_like(g)) + lr * (xq @ xk) * g
    gb = b_grad + lr * g
    b_bar = b - t * gb
    out = xq + o.ln_forward(xq @ W - t * xqWg + b_bar, ln_w, ln_b, eps)
    rows = rows + [(lr * xk, g)]
    if p == K - 1:
        W = W - t * sum(np.outer(a, gj) for a, gj in rows)
        return out, W, b_bar, [], np.zeros_like(b)
    return out, W, b, rows, gb


@pytest.mark.parametrize("K,L0,steps,with_te", [(16, 32, 40, False), (4, 6, 23, False), (5, 10, 17, True)])
def test_history_cache_equals_dense_cache_decode(orc, K, L0, steps, with_te):
    rng = np.random.default_rng(1000 + K)
    d, eps = 16, 1e-6
    L = L0 + steps
    xq, xk, xv = (rng.normal(0, 0.5, (L, d)) for _ in range(3))
    lr = 1.0 / (1.0 + np.exp(-rng.normal(0, 1, L)))
    W0, b0 = rng.normal(0, 0.2, (d, d)), rng.normal(0, 0.1, d)
    ln_w, ln_b = 1.0 + rng.normal(0, 0.2, d), rng.normal(0, 0.2, d)
    te = np.linspace(1.0, 0.3, K) if with_te else None
    # start both caches at a mini-batch boundary (the history cache holds no rows there)
    L0 -= L0 % K
    pre = orc.linear_chain(xq[:L0], xk[:L0], xv[:L0], lr[:L0], W0, b0, ln_w, ln_b, K, eps, token_eta=te)
    Wd, bd = pre["W_last"].copy(), pre["b_last"].copy()
    Wg, bg = np.zeros((d, d)), np.zeros(d)
    Wh, bh, rows, gbh = pre["W_last"].copy(), pre["b_last"].copy(), [], np.zeros(d)
    for tok in range(L0, L):
        od, _ = orc.decode_chain(xq[tok], xk[tok], xv[tok], lr[tok], ln_w, ln_b, Wd, bd, Wg, bg, K, tok, eps,
                                 token_eta=te)
        oh, Wh, bh, rows, gbh = _hist_step(orc, xq[tok], xk[tok], xv[tok], lr[tok], ln_w, ln_b, Wh, bh, rows,
                                           gbh, K, tok, eps, te)
        assert np.linalg.norm(oh - od) <= 1e-12 * np.linalg.norm(od), tok
        assert len(rows) == (tok + 1) % K
        if (tok + 1) % K == 0:
            assert np.linalg.norm(Wh - Wd) <= 1e-12 * np.linalg.norm(Wd)
            assert np.linalg.norm(bh - bd) <= 1e-12 * max(np.linalg.norm(bd), 1e-300)
        assert np.linalg.norm(gbh - bg) <= 1e-12 * max(np.linalg.norm(bg), 1e-12)
        # the dense gradient sum is the rows' sum of outer products
        dense = sum((np.outer(a, gj) for a, gj in rows), np.zeros((d, d)))
        assert np.linalg.norm(dense - Wg) <= 1e-12 * max(np.linalg.norm(Wg), 1e-12)
