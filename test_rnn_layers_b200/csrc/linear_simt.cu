// linear_simt.cu -- TTT-Linear prefill on the FFMA pipes, fp32 compute (the fp32 debug build).
//
// One CTA of 256 threads per (batch, head) chain; the state W (64x64 fp32) and b stay in shared
// memory for the whole sequence.  Each mini-batch follows the dual branch of compute_mini_batch
// ("代码连连看——TTT", compute_mini_batch, dual branch):
//   Z = XK W + b, g = ln_fused_l2_bwd(Z, XV - XK),
//   Zbar = XQ W + b - (eta * tril(XQ XK^T + 1)) g        (the tril(eta) g term folded in),
//   out = XQ + LN(Zbar), and for a full mini-batch W -= (eta[K-1,:] XK)^T g, b -= eta[K-1,:] g.
// The remainder (L % K tokens) runs last with K = r from the carried state (TTTBase.forward);
// its params are dropped, its un-scaled grad sums are optionally stored.
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;

struct SimtSmem {
    float W[TTT_D * TTT_D];
    float b[TTT_D];
    float xq[TTT_KMAX][TTT_D];
    float xk[TTT_KMAX][TTT_D];
    float xv[TTT_KMAX][TTT_D];
    float Z[TTT_KMAX][TTT_D];   // Z, then Zbar
    float G[TTT_KMAX][TTT_D];   // g = dl/dZ
    float M[TTT_KMAX][TTT_KMAX];
    float lr[TTT_KMAX];
    float te[TTT_KMAX];
    float lnw[TTT_D];
    float lnb[TTT_D];
};

// Row statistics of a 64-wide row held two values per lane: mean and 1/sqrt(var + eps).
__device__ __forceinline__ void row_stats(float v0, float v1, float eps, float& mu, float& rstd) {
    mu = warp_sum(v0 + v1) * (1.0f / TTT_D);
    float c0 = v0 - mu, c1 = v1 - mu;
    float var = warp_sum(c0 * c0 + c1 * c1) * (1.0f / TTT_D);
    rstd = 1.0f / sqrtf(var + eps);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) linear_simt_kernel(LinearArgs a) {
    __shared__ SimtSmem s;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long chain = blockIdx.x;
    const int h = static_cast<int>(chain % a.H);
    const long long aoff = (chain / a.H) * a.act_b + (chain % a.H) * a.act_h;  // token 0 of this chain
    const long long ts = a.act_t;                                               // elements per token step
    const T* XQ = static_cast<const T*>(a.XQ) + aoff;
    const T* XK = static_cast<const T*>(a.XK) + aoff;
    const T* XV = static_cast<const T*>(a.XV) + aoff;
    const float* lr = a.lr + chain * a.L;
    T* out = static_cast<T*>(a.out) + aoff;

    const float* W0 = a.W0 + (a.w0_chain_stride ? chain * a.w0_chain_stride
                                                 : static_cast<long long>(h) * TTT_D * TTT_D);
    const float* b0 = a.b0 + (a.w0_chain_stride ? chain * TTT_D : static_cast<long long>(h) * TTT_D);
    for (int i = tid; i < TTT_D * TTT_D; i += kThreads) s.W[i] = W0[i];
    if (tid < TTT_D) {
        s.b[tid] = b0[tid];
        s.lnw[tid] = a.ln_w[h * TTT_D + tid];
        s.lnb[tid] = a.ln_b[h * TTT_D + tid];
    }
    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < a.K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    __syncthreads();

    const long long n_mb = a.n_full + (a.rem > 0 ? 1 : 0);
    for (long long m = 0; m < n_mb; ++m) {
        const bool full = m < a.n_full;
        const int Km = full ? a.K : static_cast<int>(a.rem);
        const long long t0 = m * a.K;
        if (a.ckpt && full && m % a.ckpt_G == 0) {  // a checkpoint for the backward: the state before m
            float* d = a.ckpt + (chain * a.ckpt_stride + m / a.ckpt_G) * (TTT_D * TTT_D + TTT_D);
            for (int i = tid; i < TTT_D * TTT_D; i += kThreads) d[i] = s.W[i];
            if (tid < TTT_D) d[TTT_D * TTT_D + tid] = s.b[tid];
        }

        for (int i = tid; i < TTT_KMAX * TTT_D; i += kThreads) {
            int r = i / TTT_D, c = i % TTT_D;
            bool v = r < Km;
            long long off = (t0 + r) * ts + c;
            s.xq[r][c] = v ? to_f32(XQ[off]) : 0.f;
            s.xk[r][c] = v ? to_f32(XK[off]) : 0.f;
            s.xv[r][c] = v ? to_f32(XV[off]) : 0.f;
        }
        if (tid < TTT_KMAX) s.lr[tid] = tid < Km ? lr[t0 + tid] : 0.f;
        __syncthreads();

        // Z = XK W + b
        for (int i = tid; i < TTT_KMAX * TTT_D; i += kThreads) {
            int r = i / TTT_D, c = i % TTT_D;
            float acc = s.b[c];
#pragma unroll 16
            for (int k = 0; k < TTT_D; ++k) acc = fmaf(s.xk[r][k], s.W[k * TTT_D + c], acc);
            s.Z[r][c] = acc;
        }
        // M = eta * tril(XQ XK^T + 1), eta[i][j] = te_i lr_j
        {
            int i = tid >> 4, j = tid & 15;
            float acc = 0.f;
#pragma unroll 16
            for (int k = 0; k < TTT_D; ++k) acc = fmaf(s.xq[i][k], s.xk[j][k], acc);
            s.M[i][j] = (j <= i && i < Km) ? s.te[i] * s.lr[j] * (acc + 1.0f) : 0.f;
        }
        __syncthreads();

        // g = ln_fused_l2_bwd(Z, XV - XK): 2 rows per warp, 2 features per lane
        for (int rr = 0; rr < 2; ++rr) {
            int r = warp * 2 + rr;
            float z0 = s.Z[r][lane], z1 = s.Z[r][lane + 32];
            float mu, rstd;
            row_stats(z0, z1, a.eps, mu, rstd);
            float xh0 = (z0 - mu) * rstd, xh1 = (z1 - mu) * rstd;
            float t0v = s.xv[r][lane] - s.xk[r][lane], t1v = s.xv[r][lane + 32] - s.xk[r][lane + 32];
            float q0 = s.lnw[lane] * (s.lnw[lane] * xh0 + s.lnb[lane] - t0v);
            float q1 = s.lnw[lane + 32] * (s.lnw[lane + 32] * xh1 + s.lnb[lane + 32] - t1v);
            float sq = warp_sum(q0 + q1), sqx = warp_sum(q0 * xh0 + q1 * xh1);
            float scale = rstd * (1.0f / TTT_D);
            bool v = r < Km;
            s.G[r][lane] = v ? (TTT_D * q0 - sq - xh0 * sqx) * scale : 0.f;
            s.G[r][lane + 32] = v ? (TTT_D * q1 - sq - xh1 * sqx) * scale : 0.f;
        }
        __syncthreads();

        // Zbar = XQ W + b - M g  (overwrites Z)
        for (int i = tid; i < TTT_KMAX * TTT_D; i += kThreads) {
            int r = i / TTT_D, c = i % TTT_D;
            float acc = s.b[c];
#pragma unroll 16
            for (int k = 0; k < TTT_D; ++k) acc = fmaf(s.xq[r][k], s.W[k * TTT_D + c], acc);
#pragma unroll
            for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(-s.M[r][j], s.G[j][c], acc);
            s.Z[r][c] = acc;
        }
        __syncthreads();

        // out = XQ + LN(Zbar)
        for (int rr = 0; rr < 2; ++rr) {
            int r = warp * 2 + rr;
            float z0 = s.Z[r][lane], z1 = s.Z[r][lane + 32];
            float mu, rstd;
            row_stats(z0, z1, a.eps, mu, rstd);
            if (r < Km) {
                out[(t0 + r) * ts + lane] =
                    from_f32<T>(s.xq[r][lane] + s.lnw[lane] * (z0 - mu) * rstd + s.lnb[lane]);
                out[(t0 + r) * ts + lane + 32] = from_f32<T>(
                    s.xq[r][lane + 32] + s.lnw[lane + 32] * (z1 - mu) * rstd + s.lnb[lane + 32]);
            }
        }

        if (full) {
            // W -= (eta[K-1,:] * XK)^T g ; b -= sum_j eta[K-1,j] g_j
            const float tl = s.te[a.K - 1];
            for (int i = tid; i < TTT_D * TTT_D; i += kThreads) {
                int r = i / TTT_D, c = i % TTT_D;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j] * s.xk[j][r], s.G[j][c], acc);
                s.W[i] -= tl * acc;
            }
            if (tid < TTT_D) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j], s.G[j][tid], acc);
                s.b[tid] -= tl * acc;
            }
        } else if (a.W_grad_tail) {
            float* Wg = a.W_grad_tail + chain * TTT_D * TTT_D;
            for (int i = tid; i < TTT_D * TTT_D; i += kThreads) {
                int r = i / TTT_D, c = i % TTT_D;
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j] * s.xk[j][r], s.G[j][c], acc);
                Wg[i] = acc;
            }
        }
        if (!full && a.b_grad_tail && tid < TTT_D) {
            float acc = 0.f;
#pragma unroll
            for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j], s.G[j][tid], acc);
            a.b_grad_tail[chain * TTT_D + tid] = acc;
        }
        __syncthreads();
    }

    float* Wl = a.W_last + chain * TTT_D * TTT_D;
    for (int i = tid; i < TTT_D * TTT_D; i += kThreads) Wl[i] = s.W[i];
    if (tid < TTT_D) a.b_last[chain * TTT_D + tid] = s.b[tid];
    if (a.ckpt) {  // the state after the last full mini-batch, the last checkpoint entry
        float* d = a.ckpt + (chain * a.ckpt_stride + a.ckpt_stride - 1) * (TTT_D * TTT_D + TTT_D);
        for (int i = tid; i < TTT_D * TTT_D; i += kThreads) d[i] = s.W[i];
        if (tid < TTT_D) d[TTT_D * TTT_D + tid] = s.b[tid];
    }
    if (a.rem == 0) {
        if (a.W_grad_tail)
            for (int i = tid; i < TTT_D * TTT_D; i += kThreads) a.W_grad_tail[chain * TTT_D * TTT_D + i] = 0.f;
        if (a.b_grad_tail && tid < TTT_D) a.b_grad_tail[chain * TTT_D + tid] = 0.f;
    }
}

// L == 0: the state passes through unchanged, tail grads are zero.
__global__ void linear_state_copy_kernel(LinearArgs a) {
    const long long chain = blockIdx.x;
    const int h = static_cast<int>(chain % a.H);
    const float* W0 = a.W0 + (a.w0_chain_stride ? chain * a.w0_chain_stride
                                                 : static_cast<long long>(h) * TTT_D * TTT_D);
    const float* b0 = a.b0 + (a.w0_chain_stride ? chain * TTT_D : static_cast<long long>(h) * TTT_D);
    float* Wl = a.W_last + chain * TTT_D * TTT_D;
    // (no full mini-batch: the only checkpoint entry is the state after none, W0 and b0)
    float* ck = a.ckpt ? a.ckpt + (chain * a.ckpt_stride + a.ckpt_stride - 1) * (TTT_D * TTT_D + TTT_D) : nullptr;
    for (int i = threadIdx.x; i < TTT_D * TTT_D; i += blockDim.x) {
        float w = W0[i];
        Wl[i] = w;
        if (ck) ck[i] = w;
        if (a.W_grad_tail) a.W_grad_tail[chain * TTT_D * TTT_D + i] = 0.f;
    }
    if (threadIdx.x < TTT_D) {
        a.b_last[chain * TTT_D + threadIdx.x] = b0[threadIdx.x];
        if (ck) ck[TTT_D * TTT_D + threadIdx.x] = b0[threadIdx.x];
        if (a.b_grad_tail) a.b_grad_tail[chain * TTT_D + threadIdx.x] = 0.f;
    }
}

}  // namespace

cudaError_t launch_linear_simt(const LinearArgs& a, int dtype, cudaStream_t st) {
    dim3 grid(static_cast<unsigned>(a.B * a.H));
    if (dtype == 0)
        linear_simt_kernel<float><<<grid, kThreads, 0, st>>>(a);
    else
        linear_simt_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_linear_state_copy(const LinearArgs& a, cudaStream_t st) {
    linear_state_copy_kernel<<<static_cast<unsigned>(a.B * a.H), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ttt
