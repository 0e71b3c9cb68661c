// linear_bwd.cu -- backward of the TTT-Linear scan: the gradients of the outer inputs.
//
// The walkthrough ("代码连连看——TTT", TTTLinear.ttt) trains through the same scan as the forward,
// passing scan_checkpoint_group_size to its scan while training: the carried state is kept every
// G mini-batches and rebuilt inside a group when the backward reaches it.  This file is that
// backward, per chain (b, h), for the dual form of compute_mini_batch.  Per full mini-batch of
// K tokens at state (W, b), with t_i the token eta, e_j = t_{K-1} lr_j, tau = XV - XK:
//   Z = XK W + b;  g = ln_fused_l2_bwd(Z, tau)   (x_hat, sigma: Z's LayerNorm statistics)
//   M = eta * tril(XQ XK^T + 1), eta[i][j] = t_i lr_j;  Zbar = XQ W + b - M g
//   out = XQ + LN(Zbar);  W' = W - XK^T diag(e) g;  b' = b - e^T g
// Given dout and the adjoints (dW', db') of the state after the mini-batch:
//   dZbar = LN backward of dout;  dXQ = dout + dZbar W^T + dA XK
//   dM = -dZbar g^T (lower triangle);  dA = dM * eta;  dlr_j += sum_i t_i (A_ij + 1) dM_ij
//   U = XK dW' + db';  dg = -M^T dZbar - diag(e) U;  dlr_j += -t_{K-1} sum_f g_jf U_jf
//   dXK = -diag(e) g dW'^T + dA^T XQ - dtau + dZ W^T;  dXV = dtau
//   (dZ, dtau, d ln_w, d ln_b) = the vector-Jacobian product of ln_fused_l2_bwd with dg
//   dW = dW' + XQ^T dZbar + XK^T dZ;  db = db' + sum_rows (dZbar + dZ)
// The remainder tail (K = r) has no update: its terms in dW', db' and e are absent, and it
// starts from the state after the full mini-batches, whose adjoint is the caller's dW_last.
//
// Design (one CTA of 256 threads per chain; two kernels that share this structure):
//  * Phase 1 runs the forward state recursion over the full mini-batches from (W0, b0) and
//    writes every G-th state to the workspace.  Phase 2 walks the groups from the last: it
//    rebuilds the group's states from its checkpoint into a per-chain slab, then runs the
//    backward step for each mini-batch of the group in reverse.  Both phases run the same
//    forward-step code, so a rebuilt state has the bits of the first.
//  * The LayerNorm work uses a row layout: thread (r, c0) = (tid / 16, 4 (tid % 16)) owns four
//    consecutive features of one row of a 16 x 64 tile, so a row's sums are half-warp shuffles.
//  * linear_bwd_tc_kernel (bf16 activations): the 16 x 64 x 64 products, the 16 x 16 products
//    XQ XK^T and dZbar g^T, and the rank-16 state updates are TF32 warp MMAs (m16n8k8, fp32
//    accumulation); the state and its adjoint live as accumulators (the layouts are described
//    at the kernel), the LayerNorm statistics are taken in one pass, and each step's input tiles
//    are copied in one step ahead by cp.async.
//  * linear_bwd_kernel (fp32 activations): every product is one row of a tile times a 64-wide
//    matrix read as float4 rows, fp32 throughout, the 16 x 16 products per-thread dot products
//    and the LayerNorm statistics two-pass; the state and its adjoint live in shared memory as
//    [k][f] and transposed, each thread owning a 4 x 4 block of both in registers.
//  * No waits: nothing in either kernel can hang.
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kT = 256;                          // threads per CTA
constexpr int kS = TTT_D + 4;                    // row stride of the 64-wide arrays (floats)
constexpr int kS16 = TTT_KMAX + 4;               // row stride of the 16 x 16 arrays
constexpr int kState = TTT_D * TTT_D + TTT_D;    // floats of one saved state (W, then b)
constexpr int kPart = TTT_D * TTT_D + 3 * TTT_D; // floats of one chain's shares (dW0, db0, dln_w, dln_b)

struct __align__(16) BwdSmem {
    float W[TTT_D][kS];     // the state at the current mini-batch's start, [k][f]
    float WT[TTT_D][kS];    // its transpose, [f][k]
    float dW[TTT_D][kS];    // the adjoint of the state after the mini-batch, [k][f]
    float dWT[TTT_D][kS];
    float xq[TTT_KMAX][kS];
    float xk[TTT_KMAX][kS];
    float g[TTT_KMAX][kS];   // the loss gradient of each token
    float dzb[TTT_KMAX][kS]; // dZbar
    float dz[TTT_KMAX][kS];  // dZ
    float A[TTT_KMAX][kS16];
    float M[TTT_KMAX][kS16];
    float MT[TTT_KMAX][kS16];
    float dA[TTT_KMAX][kS16];
    float dAT[TTT_KMAX][kS16];
    float dlr_eta[TTT_KMAX][kS16];  // t_i (A_ij + 1) dM_ij: the eta path's share of dlr_j
    float b[TTT_D];
    float db[TTT_D];
    float lr[TTT_KMAX];
    float te[TTT_KMAX];
    float dlr_row[TTT_KMAX];        // the update path's share of dlr_j
};

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ void st4(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
__device__ __forceinline__ void st4(__nv_bfloat16* p, float4 v) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v.x, v.y), pack_bf16x2(v.z, v.w));
}

__device__ __forceinline__ float4 f4(float a) { return make_float4(a, a, a, a); }
__device__ __forceinline__ float4 operator+(float4 a, float4 b) { return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w); }
__device__ __forceinline__ float4 operator-(float4 a, float4 b) { return make_float4(a.x - b.x, a.y - b.y, a.z - b.z, a.w - b.w); }
__device__ __forceinline__ float4 operator*(float4 a, float4 b) { return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w); }
__device__ __forceinline__ float4 operator*(float4 a, float s) { return make_float4(a.x * s, a.y * s, a.z * s, a.w * s); }
__device__ __forceinline__ float hsum4(float4 a) { return (a.x + a.y) + (a.z + a.w); }

// Sum over the 16 lanes of a half-warp (the 16 threads of one tile row).
__device__ __forceinline__ float row_sum(float v) {
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// sum_{k < N} x[k] Y[k][c0 .. c0 + 3]: one row x (16-byte aligned) times the rows of Y.
template <int N, int kStride>
__device__ __forceinline__ float4 row_times(const float* x, const float (*Y)[kStride], int c0) {
    float4 acc = f4(0.f);
#pragma unroll 2  // (full unrolling spills at 2 CTAs per SM)
    for (int k = 0; k < N; k += 4) {
        const float4 xv = ld4(x + k);
        const float xs[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 y = ld4(&Y[k + j][c0]);
            acc.x = fmaf(xs[j], y.x, acc.x);
            acc.y = fmaf(xs[j], y.y, acc.y);
            acc.z = fmaf(xs[j], y.z, acc.z);
            acc.w = fmaf(xs[j], y.w, acc.w);
        }
    }
    return acc;
}

// sum_f p[f] q[f] over 64 features (rows of stride kS), in two interleaved partial sums (half
// the dependent FMA chain).
__device__ __forceinline__ float dot64(const float* p, const float* q) {
    float a0 = 0.f, a1 = 0.f;
#pragma unroll 4
    for (int f = 0; f < TTT_D; f += 4) {
        const float4 a = ld4(p + f), b = ld4(q + f);
        a0 = fmaf(a.x, b.x, a0);
        a1 = fmaf(a.y, b.y, a1);
        a0 = fmaf(a.z, b.z, a0);
        a1 = fmaf(a.w, b.w, a1);
    }
    return a0 + a1;
}

// LayerNorm statistics of a row whose four features z this thread holds, in two passes: x_hat
// and sigma.
__device__ __forceinline__ void row_norm(float4 z, float eps, float4& xh, float& sigma) {
    const float mu = row_sum(hsum4(z)) * (1.0f / TTT_D);
    const float4 c = z - f4(mu);
    const float v = row_sum(hsum4(c * c)) * (1.0f / TTT_D);
    sigma = sqrtf(v + eps);
    xh = c * (1.0f / sigma);
}

template <typename T>
__global__ void __launch_bounds__(kT, 2) linear_bwd_kernel(const LinearBwdArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    BwdSmem& s = *reinterpret_cast<BwdSmem*>(smem_raw);
    const int tid = threadIdx.x;
    const int r = tid >> 4, c0 = 4 * (tid & 15);  // this thread's tile row and four features
    const int kb = 4 * (tid >> 4);                 // its 4 x 4 block of a state: rows kb.., columns c0..
    const long long chain = blockIdx.x;
    const int h = static_cast<int>(chain % a.H);
    const int K = a.K;
    const int G = a.G;
    const long long L = a.L;
    const float eps = a.eps;
    const long long base = (chain / a.H) * a.act_b + h * a.act_h;  // this chain's token 0
    const long long ts = a.act_t;                                     // elements between its tokens
    const T* XQ = static_cast<const T*>(a.XQ) + base;
    const T* XK = static_cast<const T*>(a.XK) + base;
    const T* XV = static_cast<const T*>(a.XV) + base;
    const T* DO = static_cast<const T*>(a.d_out) + base;
    T* dXQ = static_cast<T*>(a.dXQ) + base;
    T* dXK = static_cast<T*>(a.dXK) + base;
    T* dXV = static_cast<T*>(a.dXV) + base;
    const float* lr = a.lr + chain * L;
    float* dlr = a.d_lr + chain * L;
    const float* lwp = a.ln_w + h * TTT_D + c0;
    const float* lbp = a.ln_b + h * TTT_D + c0;
    const float4 lw = make_float4(lwp[0], lwp[1], lwp[2], lwp[3]);
    const float4 lb = make_float4(lbp[0], lbp[1], lbp[2], lbp[3]);

    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    const float* W0 = a.W0 + (a.w0_chain_stride ? chain * a.w0_chain_stride : static_cast<long long>(h) * TTT_D * TTT_D);
    const float* b0 = a.b0 + (a.w0_chain_stride ? chain * TTT_D : static_cast<long long>(h) * TTT_D);
    float Wb[4][4];   // W[kb + i][c0 + j]
    float dWb[4][4];  // the adjoint, same block
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 v = ld4(W0 + (kb + i) * TTT_D + c0);
        Wb[i][0] = v.x; Wb[i][1] = v.y; Wb[i][2] = v.z; Wb[i][3] = v.w;
    }
    if (tid < TTT_D) s.b[tid] = b0[tid];

    auto put_state = [&](bool transposed) {
#pragma unroll
        for (int i = 0; i < 4; ++i) st4(&s.W[kb + i][c0], make_float4(Wb[i][0], Wb[i][1], Wb[i][2], Wb[i][3]));
        if (transposed) {
#pragma unroll
            for (int j = 0; j < 4; ++j) st4(&s.WT[c0 + j][kb], make_float4(Wb[0][j], Wb[1][j], Wb[2][j], Wb[3][j]));
        }
    };
    auto put_adjoint = [&]() {
#pragma unroll
        for (int i = 0; i < 4; ++i) st4(&s.dW[kb + i][c0], make_float4(dWb[i][0], dWb[i][1], dWb[i][2], dWb[i][3]));
#pragma unroll
        for (int j = 0; j < 4; ++j) st4(&s.dWT[c0 + j][kb], make_float4(dWb[0][j], dWb[1][j], dWb[2][j], dWb[3][j]));
    };
    // a state in the workspace: this thread's block, and b from the threads tid < 64
    auto save_state = [&](float* dst) {
#pragma unroll
        for (int i = 0; i < 4; ++i) st4(dst + (kb + i) * TTT_D + c0, make_float4(Wb[i][0], Wb[i][1], Wb[i][2], Wb[i][3]));
        if (tid < TTT_D) dst[TTT_D * TTT_D + tid] = s.b[tid];
    };
    auto load_state = [&](const float* src) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float4 v = ld4(src + (kb + i) * TTT_D + c0);
            Wb[i][0] = v.x; Wb[i][1] = v.y; Wb[i][2] = v.z; Wb[i][3] = v.w;
        }
        if (tid < TTT_D) s.b[tid] = src[TTT_D * TTT_D + tid];
    };

    // One full mini-batch of the forward state recursion: (W, b) in Wb / s.b (W also published in
    // s.W) becomes W - XK^T diag(e) g, b - e^T g.
    auto fwd_step = [&](long long t0) {
        const bool live = r < K;
        const long long row = (t0 + r) * ts + c0;
        const float4 k4 = live ? ld4(XK + row) : f4(0.f);
        const float4 v4 = live ? ld4(XV + row) : f4(0.f);
        st4(&s.xk[r][c0], k4);
        if (tid < TTT_KMAX) s.lr[tid] = tid < K ? lr[t0 + tid] : 0.f;
        __syncthreads();
        const float4 z = row_times<TTT_D>(s.xk[r], s.W, c0) + ld4(&s.b[c0]);
        float4 xh;
        float sig;
        row_norm(z, eps, xh, sig);
        const float4 q = lw * (lw * xh + lb - (v4 - k4));
        const float mq = row_sum(hsum4(q)) * (1.0f / TTT_D), mqx = row_sum(hsum4(q * xh)) * (1.0f / TTT_D);
        const float4 g = live ? (q - f4(mq) - xh * mqx) * (1.0f / sig) : f4(0.f);
        st4(&s.g[r][c0], g);
        __syncthreads();
        const float tl = s.te[K - 1];
        for (int i = 0; i < K; ++i) {
            const float4 x = ld4(&s.xk[i][kb]);
            const float4 ge = ld4(&s.g[i][c0]) * (tl * s.lr[i]);
            const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                Wb[u][0] = fmaf(-xs[u], ge.x, Wb[u][0]);
                Wb[u][1] = fmaf(-xs[u], ge.y, Wb[u][1]);
                Wb[u][2] = fmaf(-xs[u], ge.z, Wb[u][2]);
                Wb[u][3] = fmaf(-xs[u], ge.w, Wb[u][3]);
            }
        }
        if (tid < TTT_D) {
            float acc = 0.f;
            for (int i = 0; i < K; ++i) acc = fmaf(tl * s.lr[i], s.g[i][tid], acc);
            s.b[tid] -= acc;
        }
        __syncthreads();  // every read of this step's tiles and of s.W is done
        put_state(false);
    };

    float4 dgam = f4(0.f), dbet = f4(0.f);  // this thread's shares of d ln_w, d ln_b

    // The backward step of the mini-batch at t0 (Km tokens; full: it updated the state), with its
    // start state in Wb / s.W / s.WT / s.b and the adjoint of the state after it in dWb / s.dW /
    // s.dWT / s.db.  Leaves the adjoint of its start state there.
    auto bwd_step = [&](long long t0, int Km, bool full) {
        const bool live = r < Km;
        const long long row = (t0 + r) * ts + c0;
        const float4 q4 = live ? ld4(XQ + row) : f4(0.f);
        const float4 k4 = live ? ld4(XK + row) : f4(0.f);
        const float4 v4 = live ? ld4(XV + row) : f4(0.f);
        const float4 o4 = live ? ld4(DO + row) : f4(0.f);
        st4(&s.xq[r][c0], q4);
        st4(&s.xk[r][c0], k4);
        if (tid < TTT_KMAX) s.lr[tid] = tid < Km ? lr[t0 + tid] : 0.f;
        __syncthreads();  // (1)
        // the mini-batch's forward once more: Z, its statistics, g
        const float4 z = row_times<TTT_D>(s.xk[r], s.W, c0) + ld4(&s.b[c0]);
        float4 xh;
        float sig;
        row_norm(z, eps, xh, sig);
        const float4 res = lw * xh + lb - (v4 - k4);  // LN(Z) - (XV - XK)
        const float4 q = lw * res;
        const float mq = row_sum(hsum4(q)) * (1.0f / TTT_D), mqx = row_sum(hsum4(q * xh)) * (1.0f / TTT_D);
        const float4 g = live ? (q - f4(mq) - xh * mqx) * (1.0f / sig) : f4(0.f);
        st4(&s.g[r][c0], g);
        {  // A = XQ XK^T and M = eta * tril(A + 1) at (i, j) = (r, tid % 16)
            const int i = r, j = tid & 15;
            const float av = dot64(s.xq[i], s.xk[j]);
            const float m = (j <= i && i < Km) ? s.te[i] * s.lr[j] * (av + 1.0f) : 0.f;
            s.A[i][j] = av;
            s.M[i][j] = m;
            s.MT[j][i] = m;
        }
        __syncthreads();  // (2)
        // Zbar, and the backward of out = XQ + LN(Zbar)
        const float4 zb = row_times<TTT_D>(s.xq[r], s.W, c0) + ld4(&s.b[c0]) - row_times<TTT_KMAX>(s.M[r], s.g, c0);
        float4 xhb;
        float sigb;
        row_norm(zb, eps, xhb, sigb);
        const float4 p = lw * o4;
        const float mp = row_sum(hsum4(p)) * (1.0f / TTT_D), mpx = row_sum(hsum4(p * xhb)) * (1.0f / TTT_D);
        const float4 dzb = (p - f4(mp) - xhb * mpx) * (1.0f / sigb);
        dgam = dgam + o4 * xhb;
        dbet = dbet + o4;
        st4(&s.dzb[r][c0], dzb);
        // the update's terms, read from the adjoint after the mini-batch before this step adds to it
        float4 U = f4(0.f), V = f4(0.f);
        if (full) {
            U = row_times<TTT_D>(s.xk[r], s.dW, c0) + ld4(&s.db[c0]);  // XK dW' + db'
            V = row_times<TTT_D>(s.g[r], s.dWT, c0);                   // g dW'^T
        }
        __syncthreads();  // (3)
        float4 dg = f4(0.f) - row_times<TTT_KMAX>(s.MT[r], s.dzb, c0);  // -M^T dZbar
        float4 dxk = f4(0.f);
        float dlr_upd = 0.f;
        if (full) {
            const float tl = s.te[K - 1], e = tl * s.lr[r];
            dg = dg - U * e;
            dlr_upd = -tl * row_sum(hsum4(g * U));
            dxk = f4(0.f) - V * e;
        }
        if ((tid & 15) == 0) s.dlr_row[r] = dlr_upd;
        {  // dM = -dZbar g^T on the lower triangle: its shares of dA and of dlr
            const int i = r, j = tid & 15;
            const float dm = (j <= i && i < Km) ? -dot64(s.dzb[i], s.g[j]) : 0.f;
            s.dlr_eta[i][j] = s.te[i] * (s.A[i][j] + 1.0f) * dm;
            const float da = dm * s.te[i] * s.lr[j];
            s.dA[i][j] = da;
            s.dAT[j][i] = da;
        }
        {  // the vector-Jacobian product of g = ln_fused_l2_bwd(Z, tau) with dg
            const float rs = 1.0f / sig;
            const float mu = row_sum(hsum4(dg)) * (1.0f / TTT_D), mux = row_sum(hsum4(dg * xh)) * (1.0f / TTT_D);
            const float4 w = (dg - f4(mu) - xh * mux) * rs;             // through q
            const float4 hx = lw * lw * w - (dg * mqx + q * mux) * rs;  // through x_hat
            const float ds = -row_sum(hsum4(dg * g)) * rs;              // through sigma's own factor
            const float mh = row_sum(hsum4(hx)) * (1.0f / TTT_D), mhx = row_sum(hsum4(hx * xh)) * (1.0f / TTT_D);
            const float4 dz = (hx - f4(mh) - xh * mhx) * rs + xh * (ds * (1.0f / TTT_D));
            dgam = dgam + w * (res + lw * xh);
            dbet = dbet + w * lw;
            const float4 dtau = f4(0.f) - w * lw;
            dxk = dxk - dtau;
            if (live) st4(dXV + row, dtau);
            st4(&s.dz[r][c0], live ? dz : f4(0.f));
        }
        __syncthreads();  // (4)
        const float4 dxq = o4 + row_times<TTT_D>(s.dzb[r], s.WT, c0) + row_times<TTT_KMAX>(s.dA[r], s.xk, c0);
        dxk = dxk + row_times<TTT_KMAX>(s.dAT[r], s.xq, c0) + row_times<TTT_D>(s.dz[r], s.WT, c0);
        if (live) {
            st4(dXQ + row, dxq);
            st4(dXK + row, dxk);
        }
        if (tid < Km) {
            float acc = s.dlr_row[tid];
            for (int i = 0; i < TTT_KMAX; ++i) acc += s.dlr_eta[i][tid];
            dlr[t0 + tid] = acc;
        }
        // the adjoint of the start state: dW' + XQ^T dZbar + XK^T dZ, db' + sum of the rows
        for (int i = 0; i < Km; ++i) {
            const float4 xa = ld4(&s.xq[i][kb]), xb = ld4(&s.xk[i][kb]);
            const float4 ua = ld4(&s.dzb[i][c0]), ub = ld4(&s.dz[i][c0]);
            const float as[4] = {xa.x, xa.y, xa.z, xa.w}, bs[4] = {xb.x, xb.y, xb.z, xb.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                dWb[u][0] = fmaf(as[u], ua.x, fmaf(bs[u], ub.x, dWb[u][0]));
                dWb[u][1] = fmaf(as[u], ua.y, fmaf(bs[u], ub.y, dWb[u][1]));
                dWb[u][2] = fmaf(as[u], ua.z, fmaf(bs[u], ub.z, dWb[u][2]));
                dWb[u][3] = fmaf(as[u], ua.w, fmaf(bs[u], ub.w, dWb[u][3]));
            }
        }
        if (tid < TTT_D) {
            float acc = 0.f;
            for (int i = 0; i < Km; ++i) acc += s.dzb[i][tid] + s.dz[i][tid];
            s.db[tid] += acc;
        }
        __syncthreads();  // (5) every read of this step's tiles and adjoint copies is done
        put_adjoint();
    };

    // ---- phase 1: the forward state recursion, a checkpoint every G full mini-batches --------
    // (with the caller's checkpoints, only the state after the full mini-batches: the last entry)
    if (a.ckpt_given) {
        load_state(a.ckpt + (chain * a.ckpt_stride + a.n_ckpt) * kState);
    } else {
        put_state(false);
        __syncthreads();
        for (long long m = 0; m < a.n_full; ++m) {
            if (m % G == 0) save_state(a.ckpt + (chain * a.ckpt_stride + m / G) * kState);
            fwd_step(m * K);
        }
    }

    // ---- the remainder tail, from the state after the full mini-batches -----------------------
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float4 v = a.dW_last ? ld4(a.dW_last + chain * TTT_D * TTT_D + (kb + i) * TTT_D + c0) : f4(0.f);
        dWb[i][0] = v.x; dWb[i][1] = v.y; dWb[i][2] = v.z; dWb[i][3] = v.w;
    }
    if (tid < TTT_D) s.db[tid] = a.db_last ? a.db_last[chain * TTT_D + tid] : 0.f;
    put_adjoint();
    if (a.rem > 0) {
        put_state(true);
        __syncthreads();
        bwd_step(a.n_full * K, static_cast<int>(a.rem), false);
    }

    // ---- phase 2: the groups from the last; rebuild each one's states, then step back ----------
    float* const slab = a.slab + chain * G * kState;
    for (long long c = a.n_ckpt - 1; c >= 0; --c) {
        const long long m0 = c * G, m1 = m0 + G < a.n_full ? m0 + G : a.n_full;
        __syncthreads();
        load_state(a.ckpt + (chain * a.ckpt_stride + c) * kState);
        put_state(false);
        __syncthreads();
        for (long long m = m0; m < m1; ++m) {
            save_state(slab + (m - m0) * kState);
            if (m + 1 < m1) fwd_step(m * K);
        }
        for (long long m = m1 - 1; m >= m0; --m) {
            __syncthreads();
            load_state(slab + (m - m0) * kState);
            put_state(true);
            __syncthreads();
            bwd_step(m * K, K, true);
        }
    }

    // ---- this chain's shares of the shared parameters' gradients -----------------------------
    float* part = a.part + chain * kPart;
#pragma unroll
    for (int i = 0; i < 4; ++i) st4(part + (kb + i) * TTT_D + c0, make_float4(dWb[i][0], dWb[i][1], dWb[i][2], dWb[i][3]));
    __syncthreads();
    st4(&s.g[r][c0], dgam);
    st4(&s.dzb[r][c0], dbet);
    __syncthreads();
    if (tid < TTT_D) {
        float sg = 0.f, sb = 0.f;
        for (int i = 0; i < TTT_KMAX; ++i) {
            sg += s.g[i][tid];
            sb += s.dzb[i][tid];
        }
        part[TTT_D * TTT_D + tid] = s.db[tid];
        part[TTT_D * TTT_D + TTT_D + tid] = sg;
        part[TTT_D * TTT_D + 2 * TTT_D + tid] = sb;
    }
}

// The batch sums of the chains' shares: d ln_w, d ln_b per head, and dW0, db0 per head when the
// initial state is one per head (w0_per_chain = 0).  Fixed summation order over b.
__global__ void linear_bwd_reduce_kernel(const float* part, int B, int H, int w0_per_chain, float* dW0, float* db0,
                                         float* dlnw, float* dlnb) {
    const long long n = static_cast<long long>(H) * kPart;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int h = static_cast<int>(idx / kPart), e = static_cast<int>(idx % kPart);
        if (w0_per_chain && e < TTT_D * TTT_D + TTT_D) continue;
        float acc = 0.f;
        for (int b = 0; b < B; ++b) acc += part[(static_cast<long long>(b) * H + h) * kPart + e];
        if (e < TTT_D * TTT_D) dW0[static_cast<long long>(h) * TTT_D * TTT_D + e] = acc;
        else if (e < TTT_D * TTT_D + TTT_D) db0[h * TTT_D + e - TTT_D * TTT_D] = acc;
        else if (e < TTT_D * TTT_D + 2 * TTT_D) dlnw[h * TTT_D + e - TTT_D * TTT_D - TTT_D] = acc;
        else dlnb[h * TTT_D + e - TTT_D * TTT_D - 2 * TTT_D] = acc;
    }
}

// dW0, db0 of each chain when every chain started from its own state.
__global__ void linear_bwd_copy_kernel(const float* part, long long chains, float* dW0, float* db0) {
    constexpr int kN = TTT_D * TTT_D + TTT_D;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < chains * kN;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const long long c = idx / kN;
        const int e = static_cast<int>(idx % kN);
        const float v = part[c * kPart + e];
        if (e < TTT_D * TTT_D) dW0[c * TTT_D * TTT_D + e] = v;
        else db0[c * TTT_D + e - TTT_D * TTT_D] = v;
    }
}

// ---------------------------------------------------------------------------------------------
// Tensor-core form (bf16 activations).  The 16 x 64 x 64 products and the rank-16 state updates
// run as TF32 warp MMAs (m16n8k8, fp32 accumulation).
//  * The state W lives as accumulators of W^T: warp w holds output features 16 (w % 4) .. +15
//    (rows of W^T) and inputs 32 (w / 4) .. +31 (columns), four 16 x 8 tiles.  Read with the k
//    slots t and t + 4 of an MMA step standing for the inputs k0 + 2t and k0 + 2t + 1, that
//    accumulator layout is the B operand of Z = XK W, so a forward step multiplies by W straight
//    from registers (each warp half of Z's inner dimension; the halves meet in shared memory with
//    the LayerNorm's row exchange) and takes XK as bf16 pairs, one 32-bit load for two operands.
//    The update W^T += (-t lr g)^T XK accumulates into the same registers, XK arriving by
//    transposing ldmatrix loads.  W^T is written to shared memory only for the backward steps.
//  * The adjoint dW lives in the same layout (dW^T accumulators); its updates dW^T += dZbar^T XQ
//    + dZ^T XK take XQ and XK by transposing ldmatrix loads as well, and its shared copy (dW^T)
//    is a B operand of the next step's products.
//  * A 16 x 64 product of a backward step lands in a shared result tile, warp w computing columns
//    8w .. 8w + 7, and the row-layout threads read it back.  The LayerNorm work and the 16 x 16
//    products are as above.
//  * A step's inputs are copied in (cp.async) during the step before it, into a ring of three
//    buffers, so that a forward step needs no barrier at its top: the copy it reads was waited
//    for before the last barrier of the step before, and the buffer it refills was last read two
//    steps ago.
// ---------------------------------------------------------------------------------------------
constexpr int kSB = TTT_D + 8;  // row stride (bf16 elements) of the staged input tiles: 144 bytes
constexpr int kSW = TTT_D + 8;  // row stride (floats) of W^T in shared memory
constexpr int kStages = 3;      // staged steps in flight

struct __align__(16) BwdTcSmem {
    float WT[TTT_D][kSW];  // W^T, [output feature][input feature], for the backward steps
    float dWT[TTT_D][kSW];  // dW^T, likewise
    float g[TTT_KMAX][kS];
    float dzb[TTT_KMAX][kS];
    float dz[TTT_KMAX][kS];
    float P0[TTT_KMAX][kS];  // product results
    float P1[TTT_KMAX][kS];
    float P2[TTT_KMAX][kS];
    float Zp[TTT_KMAX][kS];  // a forward step's Z over inputs 32..63 (P2 holds it over 0..31)
    float A[TTT_KMAX][kS16];
    float M[TTT_KMAX][kS16];
    float MT[TTT_KMAX][kS16];
    float dA[TTT_KMAX][kS16];
    float dAT[TTT_KMAX][kS16];
    float dlr_eta[TTT_KMAX][kS16];
    float b[TTT_D];
    float db[TTT_D];
    float te[TTT_KMAX];
    float dlr_row[TTT_KMAX];
    // each step's inputs, copied in while the step before runs: [buffer][XQ, XK, XV, d_out]; the
    // MMAs and dot products read XQ and XK from here (bf16 values are exact TF32 operands)
    __nv_bfloat16 stage[kStages][4][TTT_KMAX][kSB];
    float stage_lr[kStages][TTT_KMAX];
};

// 16- and 4-byte cp.async with zero fill: src_bytes = size copies, 0 writes zeros without reading.
__device__ __forceinline__ void cp_async_16z(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_4z(void* dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ uint32_t tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

// D += A B for one m16n8k8 tile, TF32 operands, fp32 accumulators in place.
__device__ __forceinline__ void mma_tf32(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 "
                 "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// A TF32 operand from fp32 (rounded to nearest) or from bf16 (exact: the bits moved up).
__device__ __forceinline__ uint32_t op32(float x) { return tf32(x); }
__device__ __forceinline__ uint32_t op32(__nv_bfloat16 x) { return static_cast<uint32_t>(__bfloat16_as_ushort(x)) << 16; }
// The two TF32 operands in a pair of bf16 values (low half: the first element).
__device__ __forceinline__ uint32_t bf_lo(uint32_t p) { return p << 16; }
__device__ __forceinline__ uint32_t bf_hi(uint32_t p) { return p & 0xffff0000u; }
__device__ __forceinline__ uint32_t ld_pair(const __nv_bfloat16* p) { return *reinterpret_cast<const uint32_t*>(p); }

// acc += sum_{k < K} X[m][k] Y(k, n0 + n) for the 16 x 8 tile at columns n0: X rows of stride kSX;
// Y(k, n) = Ymat[k][n], or Ymat[n][k] when kTrans (rows of stride kSY).  Even and odd k-steps
// accumulate apart (half the dependent MMA latency) and meet at the end.
template <int K, bool kTrans, typename TX, int kSX, typename TY, int kSY>
__device__ __forceinline__ void tc_tile(float (&acc)[4], const TX (*X)[kSX], const TY (*Y)[kSY], int n0, int g,
                                        int t) {
    float odd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < K; k0 += 8) {
        const uint32_t a0 = op32(X[g][k0 + t]), a1 = op32(X[g + 8][k0 + t]);
        const uint32_t a2 = op32(X[g][k0 + t + 4]), a3 = op32(X[g + 8][k0 + t + 4]);
        const uint32_t b0 = op32(kTrans ? Y[n0 + g][k0 + t] : Y[k0 + t][n0 + g]);
        const uint32_t b1 = op32(kTrans ? Y[n0 + g][k0 + t + 4] : Y[k0 + t + 4][n0 + g]);
        if ((k0 >> 3) & 1) mma_tf32(odd, a0, a1, a2, a3, b0, b1);
        else mma_tf32(acc, a0, a1, a2, a3, b0, b1);
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[e] += odd[e];
}

// c0 += X0 Y and c1 += X1 Y over K = 64 for the tile at columns n0, sharing Y's fragments.
template <bool kTrans, typename TX, int kSX, int kSY>
__device__ __forceinline__ void tc_tile2(float (&c0)[4], float (&c1)[4], const TX (*X0)[kSX], const TX (*X1)[kSX],
                                         const float (*Y)[kSY], int n0, int g, int t) {
#pragma unroll
    for (int k0 = 0; k0 < TTT_D; k0 += 8) {
        const uint32_t b0 = tf32(kTrans ? Y[n0 + g][k0 + t] : Y[k0 + t][n0 + g]);
        const uint32_t b1 = tf32(kTrans ? Y[n0 + g][k0 + t + 4] : Y[k0 + t + 4][n0 + g]);
        mma_tf32(c0, op32(X0[g][k0 + t]), op32(X0[g + 8][k0 + t]), op32(X0[g][k0 + t + 4]), op32(X0[g + 8][k0 + t + 4]),
                 b0, b1);
        mma_tf32(c1, op32(X1[g][k0 + t]), op32(X1[g + 8][k0 + t]), op32(X1[g][k0 + t + 4]), op32(X1[g + 8][k0 + t + 4]),
                 b0, b1);
    }
}

// c0 += X0 W and c1 += X1 W over K = 64 for the tile at columns n0, X0 and X1 bf16 tiles and W
// given as W^T: the k slots t and t + 4 of each MMA step stand for the inputs k0 + 2t and
// k0 + 2t + 1, so each operand pair is one 32-bit load of X and one 64-bit load of W^T.
__device__ __forceinline__ void tc_tile2_wt(float (&c0)[4], float (&c1)[4], const __nv_bfloat16 (*X0)[kSB],
                                            const __nv_bfloat16 (*X1)[kSB], const float (*WT)[kSW], int n0, int g,
                                            int t) {
#pragma unroll
    for (int k0 = 0; k0 < TTT_D; k0 += 8) {
        const float2 w2 = *reinterpret_cast<const float2*>(&WT[n0 + g][k0 + 2 * t]);
        const uint32_t b0 = tf32(w2.x), b1 = tf32(w2.y);
        const uint32_t p0 = ld_pair(&X0[g][k0 + 2 * t]), p1 = ld_pair(&X0[g + 8][k0 + 2 * t]);
        const uint32_t q0 = ld_pair(&X1[g][k0 + 2 * t]), q1 = ld_pair(&X1[g + 8][k0 + 2 * t]);
        mma_tf32(c0, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), b0, b1);
        mma_tf32(c1, bf_lo(q0), bf_lo(q1), bf_hi(q0), bf_hi(q1), b0, b1);
    }
}

// c += X W over K = 64 for the tile at columns n0, as tc_tile2_wt with one operand.
__device__ __forceinline__ void tc_tile_wt(float (&c)[4], const __nv_bfloat16 (*X)[kSB], const float (*WT)[kSW], int n0,
                                           int g, int t) {
    float odd[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < TTT_D; k0 += 8) {
        const float2 w2 = *reinterpret_cast<const float2*>(&WT[n0 + g][k0 + 2 * t]);
        const uint32_t p0 = ld_pair(&X[g][k0 + 2 * t]), p1 = ld_pair(&X[g + 8][k0 + 2 * t]);
        if ((k0 >> 3) & 1) mma_tf32(odd, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), tf32(w2.x), tf32(w2.y));
        else mma_tf32(c, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), tf32(w2.x), tf32(w2.y));
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) c[e] += odd[e];
}

// acc (a matrix's transpose in the W^T accumulator layout: tile j at rows ni .. ni + 15, columns
// kh + 8j .. + 7) += sum over the 16 tokens j of s_j Gm[j][n] X[j][k], s_j = scale * lr[j] (lr
// non-null) or 1: the rank-16 update of a state or its adjoint by a mini-batch.  The token pairs
// 2t, 2t + 1 fill the k slots t, t + 4; X (bf16) arrives by transposing ldmatrix loads.
__device__ __forceinline__ void tc_rank16_t(float (&acc)[4][4], const float (*Gm)[kS], const float* lr, float scale,
                                            const __nv_bfloat16 (*X)[kSB], int ni, int kh, int lane, int g, int t) {
    uint32_t xb[2][4];
    ldmatrix_x4_trans(smem_u32(&X[lane & 7][kh + 8 * (lane >> 3)]), xb[0][0], xb[0][1], xb[0][2], xb[0][3]);
    ldmatrix_x4_trans(smem_u32(&X[8 + (lane & 7)][kh + 8 * (lane >> 3)]), xb[1][0], xb[1][1], xb[1][2], xb[1][3]);
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        const int j0 = 8 * hf + 2 * t;
        const float se = lr ? scale * lr[j0] : 1.f, so = lr ? scale * lr[j0 + 1] : 1.f;
        const uint32_t a0 = tf32(se * Gm[j0][ni + g]), a1 = tf32(se * Gm[j0][ni + g + 8]);
        const uint32_t a2 = tf32(so * Gm[j0 + 1][ni + g]), a3 = tf32(so * Gm[j0 + 1][ni + g + 8]);
#pragma unroll
        for (int j = 0; j < 4; ++j) mma_tf32(acc[j], a0, a1, a2, a3, bf_lo(xb[hf][j]), bf_hi(xb[hf][j]));
    }
}

// A 16 x 8 accumulator tile into rows 0..15, columns n0..n0+7 of a result tile.
__device__ __forceinline__ void put_tile(float (*P)[kS], const float (&c)[4], int n0, int g, int t) {
    *reinterpret_cast<float2*>(&P[g][n0 + 2 * t]) = make_float2(c[0], c[1]);
    *reinterpret_cast<float2*>(&P[g + 8][n0 + 2 * t]) = make_float2(c[2], c[3]);
}

// row_norm with one-pass statistics: the sum and the sum of squares in one shuffle tree, the
// variance as E[z^2] - mean^2 (its rounding grows with (mean / std)^2 of the row).
__device__ __forceinline__ void row_norm1(float4 z, float eps, float4& xh, float& sigma) {
    float s1 = hsum4(z), s2 = hsum4(z * z);
#pragma unroll
    for (int o = 1; o < 16; o <<= 1) {
        s1 += __shfl_xor_sync(0xffffffffu, s1, o);
        s2 += __shfl_xor_sync(0xffffffffu, s2, o);
    }
    const float mu = s1 * (1.0f / TTT_D);
    const float v = fmaxf(s2 * (1.0f / TTT_D) - mu * mu, 0.f);
    sigma = sqrtf(v + eps);
    xh = (z - f4(mu)) * (1.0f / sigma);
}

template <typename T>
__global__ void __launch_bounds__(kT, 2) linear_bwd_tc_kernel(const LinearBwdArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    BwdTcSmem& s = *reinterpret_cast<BwdTcSmem*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int r = tid >> 4, c0 = 4 * (tid & 15);       // row layout: this thread's row and four features
    const int ni = 16 * (w & 3), kh = 32 * (w >> 2);    // this warp's block of W^T and dW^T (outputs, inputs)
    const int nt = 8 * w;                               // this warp's columns of a 16 x 64 product
    const long long chain = blockIdx.x;
    const int h = static_cast<int>(chain % a.H);
    const int K = a.K;
    const int G = a.G;
    const long long L = a.L;
    const float eps = a.eps;
    const long long base = (chain / a.H) * a.act_b + h * a.act_h;  // this chain's token 0
    const long long ts = a.act_t;                                     // elements between its tokens
    const T* XQ = static_cast<const T*>(a.XQ) + base;
    const T* XK = static_cast<const T*>(a.XK) + base;
    const T* XV = static_cast<const T*>(a.XV) + base;
    const T* DO = static_cast<const T*>(a.d_out) + base;
    T* dXQ = static_cast<T*>(a.dXQ) + base;
    T* dXK = static_cast<T*>(a.dXK) + base;
    T* dXV = static_cast<T*>(a.dXV) + base;
    const float* lr = a.lr + chain * L;
    float* dlr = a.d_lr + chain * L;
    const float* lwp = a.ln_w + h * TTT_D + c0;
    const float* lbp = a.ln_b + h * TTT_D + c0;
    const float4 lw = make_float4(lwp[0], lwp[1], lwp[2], lwp[3]);
    const float4 lb = make_float4(lbp[0], lbp[1], lbp[2], lbp[3]);

    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    const float* W0 = a.W0 + (a.w0_chain_stride ? chain * a.w0_chain_stride : static_cast<long long>(h) * TTT_D * TTT_D);
    const float* b0 = a.b0 + (a.w0_chain_stride ? chain * TTT_D : static_cast<long long>(h) * TTT_D);

    // A [k][n] matrix in memory <-> accumulators in the W^T layout: tile j holds entry (k, n) for
    // inputs k = kh + 8j + 2t (elements 0, 2) and k + 1 (1, 3), outputs n = ni + g (0, 1) and
    // ni + g + 8 (2, 3).
    auto load_acc = [&](float (&acc)[4][4], const float* src) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float* p = src + (kh + 8 * j + 2 * t) * TTT_D + ni + g;
            acc[j][0] = p[0];
            acc[j][1] = p[TTT_D];
            acc[j][2] = p[8];
            acc[j][3] = p[TTT_D + 8];
        }
    };
    auto store_acc = [&](float* dst, const float (&acc)[4][4]) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            float* p = dst + (kh + 8 * j + 2 * t) * TTT_D + ni + g;
            p[0] = acc[j][0];
            p[TTT_D] = acc[j][1];
            p[8] = acc[j][2];
            p[TTT_D + 8] = acc[j][3];
        }
    };
    // the transpose into shared memory ([n][k]), each thread its own elements
    auto put_t = [&](float (*dst)[kSW], const float (&acc)[4][4]) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            *reinterpret_cast<float2*>(&dst[ni + g][kh + 8 * j + 2 * t]) = make_float2(acc[j][0], acc[j][1]);
            *reinterpret_cast<float2*>(&dst[ni + g + 8][kh + 8 * j + 2 * t]) = make_float2(acc[j][2], acc[j][3]);
        }
    };
    // the state W and the adjoint dW, as W^T and dW^T
    float Wacc[4][4], dWacc[4][4];
    load_acc(Wacc, W0);
    if (tid < TTT_D) s.b[tid] = b0[tid];
    auto publish_w = [&]() { put_t(s.WT, Wacc); };  // for a backward step
    // a state in the workspace: each thread's sixteen accumulators (its own layout), b from tid < 64
    auto save_state = [&](float* dst) {
#pragma unroll
        for (int q = 0; q < 4; ++q) st4(dst + tid * 16 + 4 * q, make_float4(Wacc[q][0], Wacc[q][1], Wacc[q][2], Wacc[q][3]));
        if (tid < TTT_D) dst[TTT_D * TTT_D + tid] = s.b[tid];
    };
    // a checkpoint (W as [k][n], then b), the format the forward kernels write
    auto save_ckpt = [&](float* dst) {
        store_acc(dst, Wacc);
        if (tid < TTT_D) dst[TTT_D * TTT_D + tid] = s.b[tid];
    };
    auto load_ckpt = [&](const float* src) {
        load_acc(Wacc, src);
        if (tid < TTT_D) s.b[tid] = src[TTT_D * TTT_D + tid];
    };
    auto load_regs = [&](const float* src) {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 v = ld4(src + tid * 16 + 4 * q);
            Wacc[q][0] = v.x; Wacc[q][1] = v.y; Wacc[q][2] = v.z; Wacc[q][3] = v.w;
        }
    };

    // The inputs of the step at t0 (Km tokens) into staging buffer buf, asynchronously: XK and XV
    // (a forward step) or XQ, XK, XV and d_out (a backward step), rows past Km zero, and lr.
    auto prefetch = [&](int buf, long long t0, int Km, bool bwd) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int cidx = tid + i * kT, ti = cidx >> 7;
            if (!bwd && (ti == 0 || ti == 3)) continue;
            const int rowc = (cidx & 127) >> 3, part = cidx & 7;
            const bool in = rowc < Km;
            const T* src = ti == 0 ? XQ : ti == 1 ? XK : ti == 2 ? XV : DO;
            cp_async_16z(&s.stage[buf][ti][rowc][part * 8], in ? src + (t0 + rowc) * ts + part * 8 : src,
                         in ? 16u : 0u);
        }
        if (tid < TTT_KMAX) cp_async_4z(&s.stage_lr[buf][tid], tid < Km ? lr + t0 + tid : lr, tid < Km ? 4u : 0u);
        cp_async_commit();
    };
    auto staged = [&](int buf, int ti) {
        const uint2 u = *reinterpret_cast<const uint2*>(&s.stage[buf][ti][r][c0]);
        const float2 lo = unpack_bf16x2(u.x), hi = unpack_bf16x2(u.y);
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    };
    // What a step prefetches for its successor: nothing (kind 0), a forward step (1) or a
    // backward step (2) at token t0 with Km tokens.
    struct Next {
        int kind;
        long long t0;
        int Km;
    };
    auto next_buf = [](int b) { return b == kStages - 1 ? 0 : b + 1; };
    auto start_next = [&](int buf, const Next& nx) {
        if (nx.kind) prefetch(next_buf(buf), nx.t0, nx.Km, nx.kind == 2);
    };

    // One full mini-batch of the forward state recursion (W^T in Wacc, b in s.b), its inputs in
    // staging buffer buf (copied and waited for during the step before).
    auto fwd_step = [&](long long t0, int buf, const Next& nx) {
        const bool live = r < K;
        const float4 k4 = staged(buf, 1), v4 = staged(buf, 2);
        const __nv_bfloat16 (*xk)[kSB] = s.stage[buf][1];
        const float* lrs = s.stage_lr[buf];
        start_next(buf, nx);
        {  // Z over this warp's inputs kh .. kh + 31, at outputs ni .. ni + 15
            float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int k0 = kh + 8 * j;
                const uint32_t p0 = ld_pair(&xk[g][k0 + 2 * t]), p1 = ld_pair(&xk[g + 8][k0 + 2 * t]);
                mma_tf32(z0, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), tf32(Wacc[j][0]), tf32(Wacc[j][1]));
                mma_tf32(z1, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), tf32(Wacc[j][2]), tf32(Wacc[j][3]));
            }
            float (*Pz)[kS] = kh ? s.Zp : s.P2;
            put_tile(Pz, z0, ni, g, t);
            put_tile(Pz, z1, ni + 8, g, t);
        }
        __syncthreads();
        const float4 z = ld4(&s.P2[r][c0]) + ld4(&s.Zp[r][c0]) + ld4(&s.b[c0]);
        float4 xh;
        float sig;
        row_norm1(z, eps, xh, sig);
        const float4 q = lw * (lw * xh + lb - (v4 - k4));
        const float mq = row_sum(hsum4(q)) * (1.0f / TTT_D), mqx = row_sum(hsum4(q * xh)) * (1.0f / TTT_D);
        const float4 gv = live ? (q - f4(mq) - xh * mqx) * (1.0f / sig) : f4(0.f);
        st4(&s.g[r][c0], gv);
        cp_async_wait_all();  // the next step's inputs, copied since this step began
        __syncthreads();
        const float tl = s.te[K - 1];
        tc_rank16_t(Wacc, s.g, lrs, -tl, xk, ni, kh, lane, g, t);  // W^T += (-tl lr g)^T XK
        if (tid < TTT_D) {  // rows past K hold zeros (g and the zero-filled lr): the fixed bound adds nothing
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < TTT_KMAX; ++i) acc = fmaf(tl * lrs[i], s.g[i][tid], acc);
            s.b[tid] -= acc;
        }
    };

    float4 dgam = f4(0.f), dbet = f4(0.f);

    // The backward step of the mini-batch at t0 (as in linear_bwd_kernel), with its start state in
    // s.WT / s.b, the adjoint after it in dWacc / s.dWT / s.db, its inputs in staging buffer buf;
    // next_state (or null): the saved start state of the step after, loaded into the W registers
    // early and written to s.WT and s.b once this step has no more use for them.
    auto bwd_step = [&](long long t0, int Km, bool full, int buf, const Next& nx, const float* next_state) {
        const bool live = r < Km;
        const long long row = (t0 + r) * ts + c0;
        cp_async_wait_all();
        __syncthreads();  // (0) the staged inputs have landed; the step reads XQ, XK and lr from them
        const float4 k4 = staged(buf, 1), v4 = staged(buf, 2), o4 = staged(buf, 3);
        const __nv_bfloat16 (*xq)[kSB] = s.stage[buf][0];
        const __nv_bfloat16 (*xk)[kSB] = s.stage[buf][1];
        const float* lrs = s.stage_lr[buf];
        start_next(buf, nx);
        float b_next = 0.f;
        if (next_state) {  // the next step's start state into the idle W registers, a step ahead of its use
            load_regs(next_state);
            if (tid < TTT_D) b_next = next_state[TTT_D * TTT_D + tid];
        }
        {  // XK W and XQ W, sharing W's fragments
            float cz[4] = {0.f, 0.f, 0.f, 0.f}, cb[4] = {0.f, 0.f, 0.f, 0.f};
            tc_tile2_wt(cz, cb, xk, xq, s.WT, nt, g, t);
            put_tile(s.P0, cz, nt, g, t);
            put_tile(s.P1, cb, nt, g, t);
        }
        if (w < 2) {  // A = XQ XK^T at columns 8w .. 8w + 7 (bf16 products are exact), and M = eta * tril(A + 1)
            float ca[4] = {0.f, 0.f, 0.f, 0.f}, odd[4] = {0.f, 0.f, 0.f, 0.f};
            const int j0 = 8 * w;
#pragma unroll
            for (int k0 = 0; k0 < TTT_D; k0 += 8) {
                const uint32_t p0 = ld_pair(&xq[g][k0 + 2 * t]), p1 = ld_pair(&xq[g + 8][k0 + 2 * t]);
                const uint32_t kb = ld_pair(&xk[j0 + g][k0 + 2 * t]);
                if ((k0 >> 3) & 1) mma_tf32(odd, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), bf_lo(kb), bf_hi(kb));
                else mma_tf32(ca, bf_lo(p0), bf_lo(p1), bf_hi(p0), bf_hi(p1), bf_lo(kb), bf_hi(kb));
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // element (i, j): i = g (+ 8), j = j0 + 2t (+ 1)
                const int i = g + 8 * (e >> 1), j = j0 + 2 * t + (e & 1);
                const float av = ca[e] + odd[e];
                const float m = (j <= i && i < Km) ? s.te[i] * lrs[j] * (av + 1.0f) : 0.f;
                s.A[i][j] = av;
                s.M[i][j] = m;
                s.MT[j][i] = m;
            }
        }
        __syncthreads();  // (2)
        const float4 bb = ld4(&s.b[c0]);
        const float4 z = ld4(&s.P0[r][c0]) + bb;
        float4 xh;
        float sig;
        row_norm1(z, eps, xh, sig);
        const float4 res = lw * xh + lb - (v4 - k4);
        const float4 q = lw * res;
        const float mq = row_sum(hsum4(q)) * (1.0f / TTT_D), mqx = row_sum(hsum4(q * xh)) * (1.0f / TTT_D);
        const float4 gv = live ? (q - f4(mq) - xh * mqx) * (1.0f / sig) : f4(0.f);
        st4(&s.g[r][c0], gv);
        const float4 zb0 = ld4(&s.P1[r][c0]) + bb;
        __syncthreads();  // (3)
        {  // M g; and the update's XK dW' and g dW'^T from the adjoint after the mini-batch
            float cm[4] = {0.f, 0.f, 0.f, 0.f};
            tc_tile<TTT_KMAX, false>(cm, s.M, s.g, nt, g, t);
            put_tile(s.P0, cm, nt, g, t);
            if (full) {
                float cu[4] = {0.f, 0.f, 0.f, 0.f}, cv[4] = {0.f, 0.f, 0.f, 0.f};
                tc_tile_wt(cu, xk, s.dWT, nt, g, t);
                tc_tile<TTT_D, false>(cv, s.g, s.dWT, nt, g, t);
                put_tile(s.P1, cu, nt, g, t);
                put_tile(s.P2, cv, nt, g, t);
            }
        }
        __syncthreads();  // (4)
        const float4 zb = zb0 - ld4(&s.P0[r][c0]);
        float4 xhb;
        float sigb;
        row_norm1(zb, eps, xhb, sigb);
        const float4 p = lw * o4;
        const float mp = row_sum(hsum4(p)) * (1.0f / TTT_D), mpx = row_sum(hsum4(p * xhb)) * (1.0f / TTT_D);
        st4(&s.dzb[r][c0], (p - f4(mp) - xhb * mpx) * (1.0f / sigb));
        dgam = dgam + o4 * xhb;
        dbet = dbet + o4;
        const float4 U = full ? ld4(&s.P1[r][c0]) + ld4(&s.db[c0]) : f4(0.f);
        const float4 V = full ? ld4(&s.P2[r][c0]) : f4(0.f);
        __syncthreads();  // (5)
        {  // M^T dZbar
            float cg[4] = {0.f, 0.f, 0.f, 0.f};
            tc_tile<TTT_KMAX, false>(cg, s.MT, s.dzb, nt, g, t);
            put_tile(s.P0, cg, nt, g, t);
        }
        if (w < 2) {  // dM = -dZbar g^T at columns 8w .. 8w + 7, lower triangle: its shares of dA and of dlr
            // three TF32 products per step (hi hi + hi lo + lo hi, each operand split in two TF32
            // parts), close to fp32 products
            float ch[4] = {0.f, 0.f, 0.f, 0.f}, cl[4] = {0.f, 0.f, 0.f, 0.f};
            const int j0 = 8 * w;
            auto split = [](float x, uint32_t& hi, uint32_t& lo) {
                hi = tf32(x);
                lo = tf32(x - __uint_as_float(hi));
            };
#pragma unroll
            for (int k0 = 0; k0 < TTT_D; k0 += 8) {
                uint32_t ah[4], al[4], bh[2], bl[2];
                split(s.dzb[g][k0 + t], ah[0], al[0]);
                split(s.dzb[g + 8][k0 + t], ah[1], al[1]);
                split(s.dzb[g][k0 + t + 4], ah[2], al[2]);
                split(s.dzb[g + 8][k0 + t + 4], ah[3], al[3]);
                split(s.g[j0 + g][k0 + t], bh[0], bl[0]);
                split(s.g[j0 + g][k0 + t + 4], bh[1], bl[1]);
                mma_tf32(ch, ah[0], ah[1], ah[2], ah[3], bh[0], bh[1]);
                mma_tf32(cl, ah[0], ah[1], ah[2], ah[3], bl[0], bl[1]);
                mma_tf32(cl, al[0], al[1], al[2], al[3], bh[0], bh[1]);
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {  // element (i, j): i = g (+ 8), j = j0 + 2t (+ 1)
                const int i = g + 8 * (e >> 1), j = j0 + 2 * t + (e & 1);
                const float dm = (j <= i && i < Km) ? -(ch[e] + cl[e]) : 0.f;
                s.dlr_eta[i][j] = s.te[i] * (s.A[i][j] + 1.0f) * dm;
                const float da = dm * s.te[i] * lrs[j];
                s.dA[i][j] = da;
                s.dAT[j][i] = da;
            }
        }
        __syncthreads();  // (6)
        float4 dg = f4(0.f) - ld4(&s.P0[r][c0]);
        float4 dxk = f4(0.f);
        float dlr_upd = 0.f;
        if (full) {
            const float tl = s.te[K - 1], e = tl * lrs[r];
            dg = dg - U * e;
            dlr_upd = -tl * row_sum(hsum4(gv * U));
            dxk = f4(0.f) - V * e;
        }
        if ((tid & 15) == 0) s.dlr_row[r] = dlr_upd;
        {  // the vector-Jacobian product of g = ln_fused_l2_bwd(Z, tau) with dg
            const float rs = 1.0f / sig;
            const float mu = row_sum(hsum4(dg)) * (1.0f / TTT_D), mux = row_sum(hsum4(dg * xh)) * (1.0f / TTT_D);
            const float4 wq = (dg - f4(mu) - xh * mux) * rs;
            const float4 hx = lw * lw * wq - (dg * mqx + q * mux) * rs;
            const float ds = -row_sum(hsum4(dg * gv)) * rs;
            const float mh = row_sum(hsum4(hx)) * (1.0f / TTT_D), mhx = row_sum(hsum4(hx * xh)) * (1.0f / TTT_D);
            const float4 dz = (hx - f4(mh) - xh * mhx) * rs + xh * (ds * (1.0f / TTT_D));
            dgam = dgam + wq * (res + lw * xh);
            dbet = dbet + wq * lw;
            const float4 dtau = f4(0.f) - wq * lw;
            dxk = dxk - dtau;
            if (live) st4(dXV + row, dtau);
            st4(&s.dz[r][c0], live ? dz : f4(0.f));
        }
        __syncthreads();  // (7)
        {  // dZbar W^T + dA XK and dZ W^T + dA^T XQ; the adjoint of the start state
            float cq[4] = {0.f, 0.f, 0.f, 0.f}, ck[4] = {0.f, 0.f, 0.f, 0.f};
            tc_tile2<false>(cq, ck, s.dzb, s.dz, s.WT, nt, g, t);
            tc_tile<TTT_KMAX, false>(cq, s.dA, xk, nt, g, t);
            tc_tile<TTT_KMAX, false>(ck, s.dAT, xq, nt, g, t);
            put_tile(s.P0, cq, nt, g, t);
            put_tile(s.P1, ck, nt, g, t);
            tc_rank16_t(dWacc, s.dzb, nullptr, 1.f, xq, ni, kh, lane, g, t);
            tc_rank16_t(dWacc, s.dz, nullptr, 1.f, xk, ni, kh, lane, g, t);
        }
        cp_async_wait_all();  // the next step's inputs (a forward step after this one has no barrier at its top)
        __syncthreads();      // (8)
        if (next_state) {  // s.WT's and s.b's readers are done
            publish_w();
            if (tid < TTT_D) s.b[tid] = b_next;
        }
        if (live) {
            st4(dXQ + row, o4 + ld4(&s.P0[r][c0]));
            st4(dXK + row, dxk + ld4(&s.P1[r][c0]));
        }
        if (tid < Km) {
            float acc = s.dlr_row[tid];
            for (int i = 0; i < TTT_KMAX; ++i) acc += s.dlr_eta[i][tid];
            dlr[t0 + tid] = acc;
        }
        if (tid >= TTT_D && tid < 2 * TTT_D) {  // db, on the third and fourth warps
            const int f = tid - TTT_D;
            float acc = 0.f;
#pragma unroll
            for (int i = 0; i < TTT_KMAX; ++i)
                if (i < Km) acc += s.dzb[i][f] + s.dz[i][f];
            s.db[f] += acc;
        }
        put_t(s.dWT, dWacc);  // s.dWT's readers (the update's products) finished before barrier (4)
    };

    // ---- the order of the steps, for the prefetch of each one's successor ----------------------
    const long long n_full = a.n_full;
    const int rem = static_cast<int>(a.rem);
    auto group_first = [&](long long c) -> Next {  // the first step of group c in phase 2
        const long long m0g = c * G, m1g = m0g + G < n_full ? m0g + G : n_full;
        return m1g - m0g > 1 ? Next{1, m0g * K, K} : Next{2, m0g * K, K};
    };
    const Next after_tail = a.n_ckpt > 0 ? group_first(a.n_ckpt - 1) : Next{0, 0, 0};
    const Next after_phase1 = rem > 0 ? Next{2, n_full * K, rem} : after_tail;
    int buf = 0;

    // ---- phase 1: the forward state recursion, a checkpoint every G full mini-batches --------
    // (with the caller's checkpoints, only the state after the full mini-batches: the last entry)
    if (a.ckpt_given) {
        if (after_phase1.kind) prefetch(0, after_phase1.t0, after_phase1.Km, after_phase1.kind == 2);
        load_ckpt(a.ckpt + (chain * a.ckpt_stride + a.n_ckpt) * kState);
    } else if (n_full > 0) {
        prefetch(0, 0, K, false);
    } else if (after_phase1.kind) {
        prefetch(0, after_phase1.t0, after_phase1.Km, after_phase1.kind == 2);
    }
    cp_async_wait_all();
    __syncthreads();  // the first step's inputs, b and the step coefficients in place for every thread
    for (long long m = 0; m < (a.ckpt_given ? 0 : n_full); ++m) {
        if (m % G == 0) save_ckpt(a.ckpt + (chain * a.ckpt_stride + m / G) * kState);
        fwd_step(m * K, buf, m + 1 < n_full ? Next{1, (m + 1) * K, K} : after_phase1);
        buf = next_buf(buf);
    }

    // ---- the remainder tail, from the state after the full mini-batches -----------------------
    if (a.dW_last) {
        load_acc(dWacc, a.dW_last + chain * TTT_D * TTT_D);
    } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) dWacc[q][0] = dWacc[q][1] = dWacc[q][2] = dWacc[q][3] = 0.f;
    }
    if (tid < TTT_D) s.db[tid] = a.db_last ? a.db_last[chain * TTT_D + tid] : 0.f;
    put_t(s.dWT, dWacc);
    if (rem > 0) {
        publish_w();  // s.WT's last readers passed barriers long ago; the step's first barrier orders the rest
        bwd_step(n_full * K, rem, false, buf, after_tail, nullptr);
        buf = next_buf(buf);
    }

    // ---- phase 2: the groups from the last; rebuild each one's states, then step back ----------
    float* const slab = a.slab + chain * G * kState;
    for (long long c = a.n_ckpt - 1; c >= 0; --c) {
        const long long m0g = c * G, m1g = m0g + G < n_full ? m0g + G : n_full;
        // no barrier: s.b's readers of the last step passed its later barriers, and each thread
        // rewrites only its own elements
        load_ckpt(a.ckpt + (chain * a.ckpt_stride + c) * kState);
        for (long long m = m0g; m + 1 < m1g; ++m) {  // the group's states but its last, kept in the slab
            save_state(slab + (m - m0g) * kState);
            fwd_step(m * K, buf, m + 2 < m1g ? Next{1, (m + 1) * K, K} : Next{2, (m1g - 1) * K, K});
            buf = next_buf(buf);
        }
        publish_w();  // the last state of the group is the first one its backward steps need
        for (long long m = m1g - 1; m >= m0g; --m) {
            bwd_step(m * K, K, true, buf, m > m0g ? Next{2, (m - 1) * K, K} : (c > 0 ? group_first(c - 1) : Next{0, 0, 0}),
                     m > m0g ? slab + (m - 1 - m0g) * kState : nullptr);
            buf = next_buf(buf);
        }
    }

    // ---- this chain's shares of the shared parameters' gradients -----------------------------
    float* part = a.part + chain * kPart;
    store_acc(part, dWacc);
    __syncthreads();
    st4(&s.g[r][c0], dgam);
    st4(&s.dzb[r][c0], dbet);
    __syncthreads();
    if (tid < TTT_D) {
        float sg = 0.f, sb = 0.f;
        for (int i = 0; i < TTT_KMAX; ++i) {
            sg += s.g[i][tid];
            sb += s.dzb[i][tid];
        }
        part[TTT_D * TTT_D + tid] = s.db[tid];
        part[TTT_D * TTT_D + TTT_D + tid] = sg;
        part[TTT_D * TTT_D + 2 * TTT_D + tid] = sb;
    }
}

}  // namespace

cudaError_t launch_linear_bwd(const LinearBwdArgs& a, int dtype, cudaStream_t st) {
    // fp32 activations: the FFMA kernel (float32 products); bf16: the tensor-core kernel
    const size_t smem = dtype == 0 ? sizeof(BwdSmem) : sizeof(BwdTcSmem);
    auto kernel = dtype == 0 ? linear_bwd_kernel<float> : linear_bwd_tc_kernel<__nv_bfloat16>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    kernel<<<static_cast<unsigned>(a.B * a.H), kT, smem, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_linear_bwd_reduce(const float* part, int B, int H, int w0_per_chain, float* dW0, float* db0,
                                     float* d_ln_w, float* d_ln_b, cudaStream_t st) {
    const long long n = static_cast<long long>(H) * kPart;
    const unsigned blocks = static_cast<unsigned>((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
    linear_bwd_reduce_kernel<<<blocks, 256, 0, st>>>(part, B, H, w0_per_chain, dW0, db0, d_ln_w, d_ln_b);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || !w0_per_chain) return e;
    const long long chains = static_cast<long long>(B) * H;
    const long long m = chains * (TTT_D * TTT_D + TTT_D);
    const unsigned cb = static_cast<unsigned>((m + 255) / 256 < 8192 ? (m + 255) / 256 : 8192);
    linear_bwd_copy_kernel<<<cb, 256, 0, st>>>(part, chains, dW0, db0);
    return cudaGetLastError();
}

}  // namespace ttt
