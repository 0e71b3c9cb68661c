// mlp_simt.cu -- TTT-MLP prefill on the FFMA pipes, fp32 compute (the fp32 debug build).
//
// The hidden state is the two-layer MLP f(x) = gelu(x W1 + b1) W2 + b2 (ttt-lm-pytorch README:
// "TTT-MLP ... a two-layer MLP"; "代码连连看——TTT": "TTTMLP is two TTTLinear stacked"), and
// each mini-batch takes the layer-wise dual update of TTT-Linear:
//   Z1 = XK W1 + b1, X2 = gelu(Z1), Z2 = X2 W2 + b2, g2 = ln_fused_l2_bwd(Z2, XV - XK),
//   g1 = (g2 W2^T) * gelu'(Z1),
//   Zbar1 = XQ W1 + b1 - (eta * tril(XQ XK^T + 1)) g1, Xbar2 = gelu(Zbar1),
//   Zbar2 = Xbar2 W2 + b2 - (eta * tril(Xbar2 X2^T + 1)) g2, out = XQ + LN(Zbar2),
//   full mini-batch: W1 -= (eta[K-1,:] XK)^T g1, W2 -= (eta[K-1,:] X2)^T g2, biases alike.
// One CTA of 256 threads per chain, W1 (64x256) and W2 (256x64, rows padded to 65 floats) in
// shared memory for the whole sequence.
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;
constexpr int kHid = TTT_HIDDEN;
constexpr int kW2Pitch = TTT_D + 1;

struct MlpSmem {
    float W1[TTT_D * kHid];
    float W2[kHid * kW2Pitch];
    float b1[kHid];
    float b2[TTT_D];
    float lnw[TTT_D];
    float lnb[TTT_D];
    float xq[TTT_KMAX][TTT_D];
    float xk[TTT_KMAX][TTT_D];
    float xv[TTT_KMAX][TTT_D];
    float Z1[TTT_KMAX][kHid];    // Z1, then g1
    float X2[TTT_KMAX][kHid];    // gelu(Z1)
    float Xb2[TTT_KMAX][kHid];   // gelu(Zbar1)
    float Z2[TTT_KMAX][TTT_D];   // Z2, then Zbar2
    float G2[TTT_KMAX][TTT_D];
    float M1[TTT_KMAX][TTT_KMAX];
    float M2[TTT_KMAX][TTT_KMAX];
    float lr[TTT_KMAX];
    float te[TTT_KMAX];
};

__device__ __forceinline__ float gelu_tanh(float x) {
    const float k = 0.7978845608028654f;  // sqrt(2/pi)
    float u = k * (x + 0.044715f * x * x * x);
    return 0.5f * x * (1.0f + tanhf(u));
}

__device__ __forceinline__ float gelu_tanh_grad(float x) {
    const float k = 0.7978845608028654f;
    float u = k * (x + 0.044715f * x * x * x);
    float th = tanhf(u);
    return 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * k * (1.0f + 3.0f * 0.044715f * x * x);
}

__device__ __forceinline__ void row_stats(float v0, float v1, float eps, float& mu, float& rstd) {
    mu = warp_sum(v0 + v1) * (1.0f / TTT_D);
    float c0 = v0 - mu, c1 = v1 - mu;
    rstd = 1.0f / sqrtf(warp_sum(c0 * c0 + c1 * c1) * (1.0f / TTT_D) + eps);
}

template <typename T>
__global__ void __launch_bounds__(kThreads) mlp_simt_kernel(MlpArgs a) {
    extern __shared__ __align__(16) unsigned char smem_raw[];
    MlpSmem& s = *reinterpret_cast<MlpSmem*>(smem_raw);
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

    const long long wofs = a.w0_chain_stride ? chain * a.w0_chain_stride
                                             : static_cast<long long>(h) * TTT_D * kHid;
    const float* W1_0 = a.W1_0 + wofs;
    const float* W2_0 = a.W2_0 + wofs;
    const float* b1_0 = a.b1_0 + (a.w0_chain_stride ? chain * kHid : static_cast<long long>(h) * kHid);
    const float* b2_0 = a.b2_0 + (a.w0_chain_stride ? chain * TTT_D : static_cast<long long>(h) * TTT_D);
    for (int i = tid; i < TTT_D * kHid; i += kThreads) {
        s.W1[i] = W1_0[i];
        s.W2[(i / TTT_D) * kW2Pitch + i % TTT_D] = W2_0[i];
    }
    s.b1[tid] = b1_0[tid];
    if (tid < TTT_D) {
        s.b2[tid] = b2_0[tid];
        s.lnw[tid] = a.ln_w[h * TTT_D + tid];
        s.lnb[tid] = a.ln_b[h * TTT_D + tid];
    }
    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < a.K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    __syncthreads();

    const int u = tid;  // hidden unit owned by this thread
    const long long n_mb = a.n_full + (a.rem > 0 ? 1 : 0);
    for (long long m = 0; m < n_mb; ++m) {
        const bool full = m < a.n_full;
        const int Km = full ? a.K : static_cast<int>(a.rem);
        const long long t0 = m * a.K;

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

        // Z1 = XK W1 + b1, X2 = gelu(Z1)            (thread = hidden unit u)
        {
            float acc[TTT_KMAX];
#pragma unroll
            for (int r = 0; r < TTT_KMAX; ++r) acc[r] = s.b1[u];
            for (int k = 0; k < TTT_D; ++k) {
                float w = s.W1[k * kHid + u];
#pragma unroll
                for (int r = 0; r < TTT_KMAX; ++r) acc[r] = fmaf(s.xk[r][k], w, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < TTT_KMAX; ++r) {
                s.Z1[r][u] = acc[r];
                s.X2[r][u] = gelu_tanh(acc[r]);
            }
        }
        // M1 = eta * tril(XQ XK^T + 1)
        {
            int i = tid >> 4, j = tid & 15;
            float acc = 0.f;
            for (int k = 0; k < TTT_D; ++k) acc = fmaf(s.xq[i][k], s.xk[j][k], acc);
            s.M1[i][j] = (j <= i && i < Km) ? s.te[i] * s.lr[j] * (acc + 1.0f) : 0.f;
        }
        __syncthreads();

        // Z2 = X2 W2 + b2                           (thread = column c, 4 rows)
        {
            int c = tid & 63, r0 = (tid >> 6) * 4;
            float acc[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r] = s.b2[c];
            for (int k = 0; k < kHid; ++k) {
                float w = s.W2[k * kW2Pitch + c];
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r] = fmaf(s.X2[r0 + r][k], w, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) s.Z2[r0 + r][c] = acc[r];
        }
        __syncthreads();

        // g2 = ln_fused_l2_bwd(Z2, XV - XK)
        for (int rr = 0; rr < 2; ++rr) {
            int r = warp * 2 + rr;
            float z0 = s.Z2[r][lane], z1 = s.Z2[r][lane + 32];
            float mu, rstd;
            row_stats(z0, z1, a.eps, mu, rstd);
            float xh0 = (z0 - mu) * rstd, xh1 = (z1 - mu) * rstd;
            float q0 = s.lnw[lane] * (s.lnw[lane] * xh0 + s.lnb[lane] - (s.xv[r][lane] - s.xk[r][lane]));
            float q1 = s.lnw[lane + 32] *
                       (s.lnw[lane + 32] * xh1 + s.lnb[lane + 32] - (s.xv[r][lane + 32] - s.xk[r][lane + 32]));
            float sq = warp_sum(q0 + q1), sqx = warp_sum(q0 * xh0 + q1 * xh1);
            float scale = rstd * (1.0f / TTT_D);
            bool v = r < Km;
            s.G2[r][lane] = v ? (TTT_D * q0 - sq - xh0 * sqx) * scale : 0.f;
            s.G2[r][lane + 32] = v ? (TTT_D * q1 - sq - xh1 * sqx) * scale : 0.f;
        }
        __syncthreads();

        // g1 = (g2 W2^T) * gelu'(Z1)                (in place over Z1)
        {
            float acc[TTT_KMAX];
#pragma unroll
            for (int r = 0; r < TTT_KMAX; ++r) acc[r] = 0.f;
            for (int c = 0; c < TTT_D; ++c) {
                float w = s.W2[u * kW2Pitch + c];
#pragma unroll
                for (int r = 0; r < TTT_KMAX; ++r) acc[r] = fmaf(s.G2[r][c], w, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < TTT_KMAX; ++r) s.Z1[r][u] = acc[r] * gelu_tanh_grad(s.Z1[r][u]);
        }
        __syncthreads();

        // Zbar1 = XQ W1 + b1 - M1 g1, Xbar2 = gelu(Zbar1)
        {
            float acc[TTT_KMAX];
#pragma unroll
            for (int r = 0; r < TTT_KMAX; ++r) acc[r] = s.b1[u];
            for (int k = 0; k < TTT_D; ++k) {
                float w = s.W1[k * kHid + u];
#pragma unroll
                for (int r = 0; r < TTT_KMAX; ++r) acc[r] = fmaf(s.xq[r][k], w, acc[r]);
            }
            for (int j = 0; j < TTT_KMAX; ++j) {
                float gj = s.Z1[j][u];
#pragma unroll
                for (int r = 0; r < TTT_KMAX; ++r) acc[r] = fmaf(-s.M1[r][j], gj, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < TTT_KMAX; ++r) s.Xb2[r][u] = gelu_tanh(acc[r]);
        }
        __syncthreads();

        // M2 = eta * tril(Xbar2 X2^T + 1): each warp two rows i, lanes split the hidden units
        for (int rr = 0; rr < 2; ++rr) {
            int i = warp * 2 + rr;
            for (int j = 0; j < TTT_KMAX; ++j) {
                float acc = 0.f;
                for (int k = lane; k < kHid; k += 32) acc = fmaf(s.Xb2[i][k], s.X2[j][k], acc);
                acc = warp_sum(acc);
                if (lane == 0) s.M2[i][j] = (j <= i && i < Km) ? s.te[i] * s.lr[j] * (acc + 1.0f) : 0.f;
            }
        }
        __syncthreads();

        // Zbar2 = Xbar2 W2 + b2 - M2 g2              (over Z2)
        {
            int c = tid & 63, r0 = (tid >> 6) * 4;
            float acc[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[r] = s.b2[c];
            for (int k = 0; k < kHid; ++k) {
                float w = s.W2[k * kW2Pitch + c];
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r] = fmaf(s.Xb2[r0 + r][k], w, acc[r]);
            }
            for (int j = 0; j < TTT_KMAX; ++j) {
                float gj = s.G2[j][c];
#pragma unroll
                for (int r = 0; r < 4; ++r) acc[r] = fmaf(-s.M2[r0 + r][j], gj, acc[r]);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) s.Z2[r0 + r][c] = acc[r];
        }
        __syncthreads();

        // out = XQ + LN(Zbar2)
        for (int rr = 0; rr < 2; ++rr) {
            int r = warp * 2 + rr;
            float z0 = s.Z2[r][lane], z1 = s.Z2[r][lane + 32];
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
            const float tl = s.te[a.K - 1];
            float g1r[TTT_KMAX], x2r[TTT_KMAX];
#pragma unroll
            for (int j = 0; j < TTT_KMAX; ++j) {
                g1r[j] = s.Z1[j][u];
                x2r[j] = s.lr[j] * s.X2[j][u];
            }
            // W1[:, u] -= tl * sum_j lr_j xk_j^T g1_j[u]
            for (int k = 0; k < TTT_D; ++k) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j] * s.xk[j][k], g1r[j], acc);
                s.W1[k * kHid + u] -= tl * acc;
            }
            {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j], g1r[j], acc);
                s.b1[u] -= tl * acc;
            }
            // W2[u, :] -= tl * sum_j lr_j X2_j[u] g2_j
            for (int c = 0; c < TTT_D; ++c) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(x2r[j], s.G2[j][c], acc);
                s.W2[u * kW2Pitch + c] -= tl * acc;
            }
            if (tid < TTT_D) {
                float acc = 0.f;
#pragma unroll
                for (int j = 0; j < TTT_KMAX; ++j) acc = fmaf(s.lr[j], s.G2[j][tid], acc);
                s.b2[tid] -= tl * acc;
            }
        }
        __syncthreads();
    }

    float* W1l = a.W1_last + chain * TTT_D * kHid;
    float* W2l = a.W2_last + chain * TTT_D * kHid;
    for (int i = tid; i < TTT_D * kHid; i += kThreads) {
        W1l[i] = s.W1[i];
        W2l[i] = s.W2[(i / TTT_D) * kW2Pitch + i % TTT_D];
    }
    a.b1_last[chain * kHid + tid] = s.b1[tid];
    if (tid < TTT_D) a.b2_last[chain * TTT_D + tid] = s.b2[tid];
}

__global__ void mlp_state_copy_kernel(MlpArgs a) {
    const long long chain = blockIdx.x;
    const int h = static_cast<int>(chain % a.H);
    const long long wofs = a.w0_chain_stride ? chain * a.w0_chain_stride
                                             : static_cast<long long>(h) * TTT_D * kHid;
    for (int i = threadIdx.x; i < TTT_D * kHid; i += blockDim.x) {
        a.W1_last[chain * TTT_D * kHid + i] = a.W1_0[wofs + i];
        a.W2_last[chain * TTT_D * kHid + i] = a.W2_0[wofs + i];
    }
    const long long b1o = a.w0_chain_stride ? chain * kHid : static_cast<long long>(h) * kHid;
    const long long b2o = a.w0_chain_stride ? chain * TTT_D : static_cast<long long>(h) * TTT_D;
    for (int i = threadIdx.x; i < kHid; i += blockDim.x) a.b1_last[chain * kHid + i] = a.b1_0[b1o + i];
    for (int i = threadIdx.x; i < TTT_D; i += blockDim.x) a.b2_last[chain * TTT_D + i] = a.b2_0[b2o + i];
}

}  // namespace

cudaError_t launch_mlp_simt(const MlpArgs& a, int dtype, cudaStream_t st) {
    const size_t smem = sizeof(MlpSmem);
    cudaError_t e;
    dim3 grid(static_cast<unsigned>(a.B * a.H));
    if (dtype == 0) {
        e = cudaFuncSetAttribute(mlp_simt_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mlp_simt_kernel<float><<<grid, kThreads, smem, st>>>(a);
    } else {
        e = cudaFuncSetAttribute(mlp_simt_kernel<__nv_bfloat16>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        mlp_simt_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_mlp_state_copy(const MlpArgs& a, cudaStream_t st) {
    mlp_state_copy_kernel<<<static_cast<unsigned>(a.B * a.H), 256, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ttt
