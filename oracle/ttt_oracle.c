/*
 * ttt_oracle.c -- plain, slow, single-threaded CPU oracle of the TTT scan, in double.
 *
 * The scalar type is `real`: double unless ORACLE_REAL says otherwise.  The parity build is
 * the double one; a float build of the same source (-DORACLE_REAL=float) is only timed, as
 * the CPU baseline's single-precision figure.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or load this file:
 * only the tests, the smoke check and the bench's CPU-baseline leg use it.  It shares no
 * code, header, table or helper with the CUDA library.
 *
 * Sources (cited by page title and section):
 *   [walkthrough]  "代码连连看——TTT" (jiafeimiao.top): TTTBase.forward listing, TTTLinear.ttt
 *                  listing, compute_mini_batch listing (dual branch and primal branch).
 *   [explainer]    "测试时学习（TTT）原理解析" (nanhubrain.csdn.net): TTTLinear.__init__,
 *                  TTTCache ("TTT缓存机制").
 *   [readme]       the ttt-lm-pytorch README (downcodes.com mirror): TTT-Linear / TTT-MLP,
 *                  hidden state = a linear model / a two-layer MLP.
 *
 * The oracle takes the PRIMAL form of compute_mini_batch ([walkthrough], primal branch), token
 * by token: for token i of a mini-batch, the state it is evaluated at is
 *     W_bar_i = W - t_i * sum_{j<=i} lr_j * xk_j^T g_j,   b_bar_i = b - t_i * sum_{j<=i} lr_j g_j
 * with every g_j taken at the mini-batch-start state (Z1 = X1 @ W1_init + b1_init), and the
 * state carried to the next mini-batch is W_bar_{K-1}, b_bar_{K-1}.  The dual branch on the
 * same page computes the same quantity in matrix form; the tests check the two agree.
 *
 * Readings where the pages are silent (each one is a parameter or stated choice):
 *   - eta[i][j] = t_i * lr_j on j <= i, t_i = 1/(i+1) unless a token_eta table is passed.
 *   - ln_fused_l2_bwd: gradient w.r.t. Z of l = 1/2 * || LN(Z) - target ||^2 per token, the
 *     sum running over the d features (no 1/d, no 1/K), LN with biased variance and eps inside
 *     the square root.
 *   - tail (L % K = r > 0): the tail runs with mini-batch size r from the state after the full
 *     mini-batches; the returned state is the one after the full mini-batches (the tail's
 *     params are dropped in TTTBase.forward: "output_reminder, _ = self.ttt(...)"); the tail's
 *     un-scaled grad sums are reported separately for cache continuation.
 *   - TTTCache commit: W, b commit (and grads reset) after the token at position p = K-1 of a
 *     mini-batch; otherwise only the grad sums are stored.
 *   - TTT-MLP: the state is x -> gelu_tanh(x W1 + b1) W2 + b2; both layers take the same eta,
 *     the gradient of the same LN-L2 loss, and the same per-token primal rule.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_REAL
#define ORACLE_REAL double
#endif
typedef ORACLE_REAL real;

#define ORACLE_OK 0
#define ORACLE_ERR_ARG -1

/* ---------------------------------------------------------------------------------------- */
/* Mini-batch partition ([walkthrough], TTTBase.forward: num_mini_batch = L // K,            */
/* reminder_len = L % K), counted with a plain loop rather than division.                    */
/* ---------------------------------------------------------------------------------------- */
int oracle_partition(long long L, int K, long long* n_full, long long* rem) {
    if (L < 0 || K < 1 || !n_full || !rem) return ORACLE_ERR_ARG;
    long long n = 0, pos = 0;
    while (pos + K <= L) {
        pos += K;
        n += 1;
    }
    *n_full = n;
    *rem = L - pos;
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------------------- */
/* Rotary position embedding of XQ and XK before the scan ([walkthrough], TTTBase.forward:    */
/* cos, sin = rotary_emb(XV, position_ids % mini_batch_size); permute_qk; apply_rotary_pos_emb; */
/* undo_permute_qk -- the bodies are not on the pages).  Token t of a chain takes position     */
/* p = t mod K; feature pair k (k < d/2) turns by the angle p * theta^(-2k/d) (RoFormer):       */
/*     (x_a, x_b) -> (x_a cos - x_b sin, x_a sin + x_b cos)                                   */
/* with (a, b) = (2k, 2k+1) -- adjacent features, the reading of permute_qk, the rotate-half  */
/* form and undo_permute_qk composed -- or (a, b) = (k, k + d/2) when half_split is set (the   */
/* rotate-half form alone).  x, y: [L][d]; y may equal x.                                      */
/* ---------------------------------------------------------------------------------------- */
int oracle_rope(const real* x, long long L, int d, int K, real theta, int half_split, real* y) {
    if (!x || !y || L < 0 || d < 2 || (d % 2) != 0 || K < 1 || !(theta > 0)) return ORACLE_ERR_ARG;
    const int half = d / 2;
    for (long long t = 0; t < L; ++t) {
        const real p = (real)(t % K);
        const real* xr = x + (size_t)t * d;
        real* yr = y + (size_t)t * d;
        for (int k = 0; k < half; ++k) {
            const real ang = p * pow(theta, -2.0 * k / d);
            const real c = cos(ang), s = sin(ang);
            const int ia = half_split ? k : 2 * k, ib = half_split ? k + half : 2 * k + 1;
            const real xa = xr[ia], xb = xr[ib];
            yr[ia] = xa * c - xb * s;
            yr[ib] = xa * s + xb * c;
        }
    }
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------------------- */
/* LayerNorm pieces ([walkthrough], compute_mini_batch: ln_fused_l2_bwd and ln_fwd).          */
/* ---------------------------------------------------------------------------------------- */

/* mean and sigma = sqrt(biased variance + eps) of one row of d values */
static void ln_stats(const real* z, int d, real eps, real* mu, real* sigma) {
    real s = 0.0;
    for (int c = 0; c < d; ++c) s += z[c];
    real m = s / d;
    real v = 0.0;
    for (int c = 0; c < d; ++c) v += (z[c] - m) * (z[c] - m);
    v /= d;
    *mu = m;
    *sigma = sqrt(v + eps);
}

/* y = ln_w * (u - mu) / sigma + ln_b */
static void ln_forward(const real* u, const real* ln_w, const real* ln_b, int d, real eps,
                       real* y) {
    real mu, sigma;
    ln_stats(u, d, eps, &mu, &sigma);
    for (int c = 0; c < d; ++c) y[c] = ln_w[c] * (u[c] - mu) / sigma + ln_b[c];
}

/* g = d/dz of 1/2 * || ln_w * xhat + ln_b - tgt ||^2, xhat = (z - mu) / sigma.
 * With q = ln_w * (ln_w * xhat + ln_b - tgt) (the gradient w.r.t. xhat), the LayerNorm
 * backward gives g_c = (d q_c - sum q - xhat_c * sum(q * xhat)) / (d sigma). */
static void lnl2_grad(const real* z, const real* tgt, const real* ln_w, const real* ln_b,
                      int d, real eps, real* xhat, real* q, real* g) {
    real mu, sigma;
    ln_stats(z, d, eps, &mu, &sigma);
    real sq = 0.0, sqx = 0.0;
    for (int c = 0; c < d; ++c) {
        xhat[c] = (z[c] - mu) / sigma;
        real r = ln_w[c] * xhat[c] + ln_b[c] - tgt[c];
        q[c] = ln_w[c] * r;
        sq += q[c];
        sqx += q[c] * xhat[c];
    }
    for (int c = 0; c < d; ++c) g[c] = (d * q[c] - sq - xhat[c] * sqx) / (d * sigma);
}

/* Exported for the gradient pins (finite differences, autograd). */
int oracle_lnl2_grad(const real* z, const real* tgt, const real* ln_w, const real* ln_b,
                     int d, real eps, real* g) {
    if (d < 1 || !z || !tgt || !ln_w || !ln_b || !g) return ORACLE_ERR_ARG;
    real* tmp = (real*)malloc(sizeof(real) * 2 * d);
    if (!tmp) return ORACLE_ERR_ARG;
    lnl2_grad(z, tgt, ln_w, ln_b, d, eps, tmp, tmp + d, g);
    free(tmp);
    return ORACLE_OK;
}

int oracle_ln_forward(const real* u, const real* ln_w, const real* ln_b, int d, real eps,
                      real* y) {
    if (d < 1 || !u || !ln_w || !ln_b || !y) return ORACLE_ERR_ARG;
    ln_forward(u, ln_w, ln_b, d, eps, y);
    return ORACLE_OK;
}

/* token_eta_i: the per-position scale of the accumulated grad (default 1/(i+1)). */
static real token_eta_at(const real* token_eta, int i) {
    return token_eta ? token_eta[i] : 1.0 / (real)(i + 1);
}

/* y[c] = sum_a x[a] * M[a][c] + bias[c], M is rows x cols row-major */
static void row_times(const real* x, const real* M, const real* bias, int rows, int cols,
                      real* y) {
    for (int c = 0; c < cols; ++c) y[c] = bias ? bias[c] : 0.0;
    for (int a = 0; a < rows; ++a) {
        real xa = x[a];
        const real* Ma = M + (size_t)a * cols;
        for (int c = 0; c < cols; ++c) y[c] += xa * Ma[c];
    }
}

/* ---------------------------------------------------------------------------------------- */
/* TTT-Linear, one (batch, head) chain.                                                       */
/* [walkthrough] TTTBase.forward (full mini-batches, then the remainder with K = r starting   */
/* from the carried params), TTTLinear.ttt (initial params W1, b1 tiled over the batch;       */
/* scan over mini-batches), compute_mini_batch primal branch.                                 */
/* ---------------------------------------------------------------------------------------- */
int oracle_ttt_linear_chain(const real* xq, const real* xk, const real* xv, /* [L][d] */
                            const real* lr,                                     /* [L] */
                            const real* token_eta,                              /* [K] or NULL */
                            const real* W0, const real* b0,                   /* [d][d], [d] */
                            const real* ln_w, const real* ln_b,               /* [d] */
                            long long L, int d, int K, real eps,
                            real* out,                                          /* [L][d] */
                            real* W_last, real* b_last,                       /* [d][d], [d] */
                            real* W_grad_tail, real* b_grad_tail)             /* nullable */
{
    if (L < 0 || d < 1 || K < 1 || !W0 || !b0 || !ln_w || !ln_b || !W_last || !b_last)
        return ORACLE_ERR_ARG;
    if (L > 0 && (!xq || !xk || !xv || !lr || !out)) return ORACLE_ERR_ARG;
    long long n_full, rem;
    oracle_partition(L, K, &n_full, &rem);

    size_t dd = (size_t)d * d;
    real* W = (real*)malloc(sizeof(real) * dd);
    real* b = (real*)malloc(sizeof(real) * d);
    real* G = (real*)malloc(sizeof(real) * dd);   /* sum_{j<=i} lr_j xk_j^T g_j */
    real* gb = (real*)malloc(sizeof(real) * d);   /* sum_{j<=i} lr_j g_j */
    real* Wbar = (real*)malloc(sizeof(real) * dd);
    real* bbar = (real*)malloc(sizeof(real) * d);
    real* g = (real*)malloc(sizeof(real) * (size_t)K * d); /* grads of the mini-batch */
    real* z = (real*)malloc(sizeof(real) * d);
    real* tgt = (real*)malloc(sizeof(real) * d);
    real* xhat = (real*)malloc(sizeof(real) * d);
    real* q = (real*)malloc(sizeof(real) * d);
    real* y = (real*)malloc(sizeof(real) * d);
    if (!W || !b || !G || !gb || !Wbar || !bbar || !g || !z || !tgt || !xhat || !q || !y) {
        free(W); free(b); free(G); free(gb); free(Wbar); free(bbar); free(g);
        free(z); free(tgt); free(xhat); free(q); free(y);
        return ORACLE_ERR_ARG;
    }
    memcpy(W, W0, sizeof(real) * dd);
    memcpy(b, b0, sizeof(real) * d);
    memset(G, 0, sizeof(real) * dd);
    memset(gb, 0, sizeof(real) * d);

    long long n_mb = n_full + (rem > 0 ? 1 : 0);
    for (long long m = 0; m < n_mb; ++m) {
        int full = m < n_full;
        int Km = full ? K : (int)rem;
        long long t0 = m * (long long)K;

        /* g_j = ln_fused_l2_bwd(xk_j W + b, xv_j - xk_j), all at the mini-batch-start state */
        for (int j = 0; j < Km; ++j) {
            const real* xkj = xk + (size_t)(t0 + j) * d;
            const real* xvj = xv + (size_t)(t0 + j) * d;
            row_times(xkj, W, b, d, d, z);
            for (int c = 0; c < d; ++c) tgt[c] = xvj[c] - xkj[c];
            lnl2_grad(z, tgt, ln_w, ln_b, d, eps, xhat, q, g + (size_t)j * d);
        }

        /* primal: accumulate lr-weighted grads token by token and evaluate at W_bar_i */
        memset(G, 0, sizeof(real) * dd);
        memset(gb, 0, sizeof(real) * d);
        for (int i = 0; i < Km; ++i) {
            const real* xki = xk + (size_t)(t0 + i) * d;
            const real* xqi = xq + (size_t)(t0 + i) * d;
            const real* gi = g + (size_t)i * d;
            real lri = lr[t0 + i];
            for (int a = 0; a < d; ++a)
                for (int c = 0; c < d; ++c) G[(size_t)a * d + c] += lri * xki[a] * gi[c];
            for (int c = 0; c < d; ++c) gb[c] += lri * gi[c];

            real ti = token_eta_at(token_eta, i);
            for (size_t e = 0; e < dd; ++e) Wbar[e] = W[e] - ti * G[e];
            for (int c = 0; c < d; ++c) bbar[c] = b[c] - ti * gb[c];

            /* out_i = xq_i + LN(xq_i W_bar_i + b_bar_i) */
            row_times(xqi, Wbar, bbar, d, d, z);
            ln_forward(z, ln_w, ln_b, d, eps, y);
            real* oi = out + (size_t)(t0 + i) * d;
            for (int c = 0; c < d; ++c) oi[c] = xqi[c] + y[c];
        }
        if (full) {
            memcpy(W, Wbar, sizeof(real) * dd);
            memcpy(b, bbar, sizeof(real) * d);
        }
    }

    memcpy(W_last, W, sizeof(real) * dd);
    memcpy(b_last, b, sizeof(real) * d);
    if (W_grad_tail) {
        if (rem > 0) memcpy(W_grad_tail, G, sizeof(real) * dd);
        else memset(W_grad_tail, 0, sizeof(real) * dd);
    }
    if (b_grad_tail) {
        if (rem > 0) memcpy(b_grad_tail, gb, sizeof(real) * d);
        else memset(b_grad_tail, 0, sizeof(real) * d);
    }
    free(W); free(b); free(G); free(gb); free(Wbar); free(bbar); free(g);
    free(z); free(tgt); free(xhat); free(q); free(y);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------------------- */
/* TTT-Linear decode: one token of one chain through the cached state.                      */
/* [walkthrough] TTTLinear.ttt (decoding reads the params from the cache, and a mini-batch   */
/* size that is not a multiple of K takes the primal branch so the grads can be stored) and   */
/* [explainer] TTTCache (last states + grads, seqlen_offset, mini_batch_size).                */
/* The token sits at position p = offset % K of its mini-batch; W, b are the state committed  */
/* at the last mini-batch boundary; W_grad, b_grad hold sum_{j<p} lr_j xk_j^T g_j, ...        */
/* ---------------------------------------------------------------------------------------- */
int oracle_ttt_linear_decode_chain(const real* xq, const real* xk, const real* xv, /* [d] */
                                   real lr, const real* token_eta, /* [K] or NULL */
                                   const real* ln_w, const real* ln_b,
                                   real* W, real* b, real* W_grad, real* b_grad,
                                   int d, int K, long long offset, real eps, real* out,
                                   int* committed) {
    if (d < 1 || K < 1 || offset < 0 || !xq || !xk || !xv || !ln_w || !ln_b || !W || !b ||
        !W_grad || !b_grad || !out)
        return ORACLE_ERR_ARG;
    int p = (int)(offset % K);
    size_t dd = (size_t)d * d;
    real* z = (real*)malloc(sizeof(real) * d);
    real* tgt = (real*)malloc(sizeof(real) * d);
    real* xhat = (real*)malloc(sizeof(real) * d);
    real* q = (real*)malloc(sizeof(real) * d);
    real* g = (real*)malloc(sizeof(real) * d);
    real* y = (real*)malloc(sizeof(real) * d);
    real* Wbar = (real*)malloc(sizeof(real) * dd);
    real* bbar = (real*)malloc(sizeof(real) * d);
    if (!z || !tgt || !xhat || !q || !g || !y || !Wbar || !bbar) {
        free(z); free(tgt); free(xhat); free(q); free(g); free(y); free(Wbar); free(bbar);
        return ORACLE_ERR_ARG;
    }
    row_times(xk, W, b, d, d, z);
    for (int c = 0; c < d; ++c) tgt[c] = xv[c] - xk[c];
    lnl2_grad(z, tgt, ln_w, ln_b, d, eps, xhat, q, g);
    for (int a = 0; a < d; ++a)
        for (int c = 0; c < d; ++c) W_grad[(size_t)a * d + c] += lr * xk[a] * g[c];
    for (int c = 0; c < d; ++c) b_grad[c] += lr * g[c];
    real tp = token_eta_at(token_eta, p);
    for (size_t e = 0; e < dd; ++e) Wbar[e] = W[e] - tp * W_grad[e];
    for (int c = 0; c < d; ++c) bbar[c] = b[c] - tp * b_grad[c];
    row_times(xq, Wbar, bbar, d, d, z);
    ln_forward(z, ln_w, ln_b, d, eps, y);
    for (int c = 0; c < d; ++c) out[c] = xq[c] + y[c];
    int commit = (p == K - 1);
    if (commit) {
        memcpy(W, Wbar, sizeof(real) * dd);
        memcpy(b, bbar, sizeof(real) * d);
        memset(W_grad, 0, sizeof(real) * dd);
        memset(b_grad, 0, sizeof(real) * d);
    }
    if (committed) *committed = commit;
    free(z); free(tgt); free(xhat); free(q); free(g); free(y); free(Wbar); free(bbar);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------------------- */
/* TTT-MLP ([readme]: the hidden state is a two-layer MLP; [walkthrough]: "TTTMLP is two     */
/* TTTLinear stacked").  f(x) = gelu(x W1 + b1) W2 + b2 with the tanh form of GELU.           */
/* ---------------------------------------------------------------------------------------- */
static real gelu_tanh(real x) {
    const real k = 0.79788456080286535588; /* sqrt(2/pi) */
    real u = k * (x + 0.044715 * x * x * x);
    return 0.5 * x * (1.0 + tanh(u));
}

static real gelu_tanh_deriv(real x) {
    const real k = 0.79788456080286535588;
    real u = k * (x + 0.044715 * x * x * x);
    real th = tanh(u);
    return 0.5 * (1.0 + th) + 0.5 * x * (1.0 - th * th) * k * (1.0 + 3.0 * 0.044715 * x * x);
}

int oracle_gelu_tanh(const real* x, long long n, real* y, real* dy) {
    if (n < 0 || !x) return ORACLE_ERR_ARG;
    for (long long i = 0; i < n; ++i) {
        if (y) y[i] = gelu_tanh(x[i]);
        if (dy) dy[i] = gelu_tanh_deriv(x[i]);
    }
    return ORACLE_OK;
}

int oracle_ttt_mlp_chain(const real* xq, const real* xk, const real* xv, /* [L][d] */
                         const real* lr, const real* token_eta,
                         const real* W1_0, const real* b1_0, /* [d][h], [h] */
                         const real* W2_0, const real* b2_0, /* [h][d], [d] */
                         const real* ln_w, const real* ln_b,
                         long long L, int d, int h, int K, real eps,
                         real* out,
                         real* W1_last, real* b1_last, real* W2_last, real* b2_last) {
    if (L < 0 || d < 1 || h < 1 || K < 1 || !W1_0 || !b1_0 || !W2_0 || !b2_0 || !ln_w || !ln_b ||
        !W1_last || !b1_last || !W2_last || !b2_last)
        return ORACLE_ERR_ARG;
    if (L > 0 && (!xq || !xk || !xv || !lr || !out)) return ORACLE_ERR_ARG;
    long long n_full, rem;
    oracle_partition(L, K, &n_full, &rem);
    size_t dh = (size_t)d * h;

    real* W1 = (real*)malloc(sizeof(real) * dh);
    real* b1 = (real*)malloc(sizeof(real) * h);
    real* W2 = (real*)malloc(sizeof(real) * dh);
    real* b2 = (real*)malloc(sizeof(real) * d);
    real* G1 = (real*)malloc(sizeof(real) * dh);
    real* gb1 = (real*)malloc(sizeof(real) * h);
    real* G2 = (real*)malloc(sizeof(real) * dh);
    real* gb2 = (real*)malloc(sizeof(real) * d);
    real* W1b = (real*)malloc(sizeof(real) * dh);
    real* b1b = (real*)malloc(sizeof(real) * h);
    real* W2b = (real*)malloc(sizeof(real) * dh);
    real* b2b = (real*)malloc(sizeof(real) * d);
    real* x2 = (real*)malloc(sizeof(real) * (size_t)K * h);  /* gelu(Z1_j) */
    real* g1 = (real*)malloc(sizeof(real) * (size_t)K * h);  /* dl/dZ1_j */
    real* g2 = (real*)malloc(sizeof(real) * (size_t)K * d);  /* dl/dZ2_j */
    real* z1 = (real*)malloc(sizeof(real) * h);
    real* a1 = (real*)malloc(sizeof(real) * h);
    real* z2 = (real*)malloc(sizeof(real) * d);
    real* tgt = (real*)malloc(sizeof(real) * d);
    real* xhat = (real*)malloc(sizeof(real) * d);
    real* q = (real*)malloc(sizeof(real) * d);
    real* y = (real*)malloc(sizeof(real) * d);
    void* all[] = {W1, b1, W2, b2, G1, gb1, G2, gb2, W1b, b1b, W2b, b2b, x2, g1, g2,
                   z1, a1, z2, tgt, xhat, q, y};
    int nall = (int)(sizeof(all) / sizeof(all[0]));
    for (int i = 0; i < nall; ++i)
        if (!all[i]) {
            for (int k = 0; k < nall; ++k) free(all[k]);
            return ORACLE_ERR_ARG;
        }
    memcpy(W1, W1_0, sizeof(real) * dh);
    memcpy(b1, b1_0, sizeof(real) * h);
    memcpy(W2, W2_0, sizeof(real) * dh);
    memcpy(b2, b2_0, sizeof(real) * d);

    long long n_mb = n_full + (rem > 0 ? 1 : 0);
    for (long long m = 0; m < n_mb; ++m) {
        int full = m < n_full;
        int Km = full ? K : (int)rem;
        long long t0 = m * (long long)K;

        /* forward and backward of the reconstruction loss at the mini-batch-start state */
        for (int j = 0; j < Km; ++j) {
            const real* xkj = xk + (size_t)(t0 + j) * d;
            const real* xvj = xv + (size_t)(t0 + j) * d;
            row_times(xkj, W1, b1, d, h, z1);
            real* x2j = x2 + (size_t)j * h;
            for (int u = 0; u < h; ++u) x2j[u] = gelu_tanh(z1[u]);
            row_times(x2j, W2, b2, h, d, z2);
            for (int c = 0; c < d; ++c) tgt[c] = xvj[c] - xkj[c];
            real* g2j = g2 + (size_t)j * d;
            lnl2_grad(z2, tgt, ln_w, ln_b, d, eps, xhat, q, g2j);
            /* dl/dZ1 = (dl/dZ2 W2^T) * gelu'(Z1) */
            real* g1j = g1 + (size_t)j * h;
            for (int u = 0; u < h; ++u) {
                real s = 0.0;
                const real* W2u = W2 + (size_t)u * d;
                for (int c = 0; c < d; ++c) s += g2j[c] * W2u[c];
                g1j[u] = s * gelu_tanh_deriv(z1[u]);
            }
        }

        memset(G1, 0, sizeof(real) * dh);
        memset(gb1, 0, sizeof(real) * h);
        memset(G2, 0, sizeof(real) * dh);
        memset(gb2, 0, sizeof(real) * d);
        for (int i = 0; i < Km; ++i) {
            const real* xki = xk + (size_t)(t0 + i) * d;
            const real* xqi = xq + (size_t)(t0 + i) * d;
            const real* x2i = x2 + (size_t)i * h;
            const real* g1i = g1 + (size_t)i * h;
            const real* g2i = g2 + (size_t)i * d;
            real lri = lr[t0 + i];
            for (int a = 0; a < d; ++a)
                for (int u = 0; u < h; ++u) G1[(size_t)a * h + u] += lri * xki[a] * g1i[u];
            for (int u = 0; u < h; ++u) gb1[u] += lri * g1i[u];
            for (int u = 0; u < h; ++u)
                for (int c = 0; c < d; ++c) G2[(size_t)u * d + c] += lri * x2i[u] * g2i[c];
            for (int c = 0; c < d; ++c) gb2[c] += lri * g2i[c];

            real ti = token_eta_at(token_eta, i);
            for (size_t e = 0; e < dh; ++e) W1b[e] = W1[e] - ti * G1[e];
            for (int u = 0; u < h; ++u) b1b[u] = b1[u] - ti * gb1[u];
            for (size_t e = 0; e < dh; ++e) W2b[e] = W2[e] - ti * G2[e];
            for (int c = 0; c < d; ++c) b2b[c] = b2[c] - ti * gb2[c];

            row_times(xqi, W1b, b1b, d, h, z1);
            for (int u = 0; u < h; ++u) a1[u] = gelu_tanh(z1[u]);
            row_times(a1, W2b, b2b, h, d, z2);
            ln_forward(z2, ln_w, ln_b, d, eps, y);
            real* oi = out + (size_t)(t0 + i) * d;
            for (int c = 0; c < d; ++c) oi[c] = xqi[c] + y[c];
        }
        if (full) {
            memcpy(W1, W1b, sizeof(real) * dh);
            memcpy(b1, b1b, sizeof(real) * h);
            memcpy(W2, W2b, sizeof(real) * dh);
            memcpy(b2, b2b, sizeof(real) * d);
        }
    }
    memcpy(W1_last, W1, sizeof(real) * dh);
    memcpy(b1_last, b1, sizeof(real) * h);
    memcpy(W2_last, W2, sizeof(real) * dh);
    memcpy(b2_last, b2, sizeof(real) * d);
    for (int k = 0; k < nall; ++k) free(all[k]);
    return ORACLE_OK;
}

/* ---------------------------------------------------------------------------------------- */
/* The output side of the layer ([walkthrough] TTTBase.forward, after the concatenation of    */
/* the mini-batch outputs): y = o_proj(post_norm(x)) per token.  post_norm is a LayerNorm over  */
/* the C = num_heads * head_dim features of the token (affine ln_w, ln_b; biased variance, eps  */
/* inside the square root, as every LayerNorm here), o_proj a linear map without bias,          */
/* y[n] = sum_k LN(x)[k] * Wo[n][k], with Wo stored [N][C] (out x in).  The page names both     */
/* modules and shows neither body; apply_gate ("Mamba only" on the page) is not applied.        */
/* x: [T][C], y: [T][N].                                                                        */
int oracle_post_norm_o_proj(const real* x, long long T, int C, const real* ln_w, const real* ln_b,
                            real eps, const real* Wo, int N, real* y) {
    if (T < 0 || C < 1 || N < 1 || !ln_w || !ln_b || !Wo || (T > 0 && (!x || !y))) return ORACLE_ERR_ARG;
    real* u = (real*)malloc(sizeof(real) * (size_t)C);
    if (!u) return ORACLE_ERR_ARG;
    for (long long t = 0; t < T; ++t) {
        ln_forward(x + (size_t)t * C, ln_w, ln_b, C, eps, u);
        real* yt = y + (size_t)t * N;
        for (int n = 0; n < N; ++n) {
            const real* wn = Wo + (size_t)n * C;
            real acc = 0.0;
            for (int k = 0; k < C; ++k) acc += u[k] * wn[k];
            yt[n] = acc;
        }
    }
    free(u);
    return ORACLE_OK;
}
