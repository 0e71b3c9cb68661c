// mlp_tc.cu -- TTT-MLP prefill on the 5th-generation tensor cores (tcgen05 + tensor memory).
//
// The hidden state is the two-layer MLP f(x) = gelu(x W1 + b1) W2 + b2, d = 64 -> 256 -> 64
// (ttt-lm-pytorch README: "TTT-MLP ... a two-layer MLP"; "代码连连看——TTT": "TTTMLP is two
// TTTLinear stacked").  Each mini-batch takes the layer-wise dual update of TTT-Linear:
//   Z1 = XK W1 + b1, X2 = gelu(Z1), Z2 = X2 W2 + b2, g2 = ln_fused_l2_bwd(Z2, XV - XK),
//   g1 = (g2 W2^T) * gelu'(Z1),
//   Zbar1 = XQ W1 + b1 - M1 g1, Xbar2 = gelu(Zbar1), Zbar2 = Xbar2 W2 + b2 - M2 g2,
//   M1 = eta * tril(XQ XK^T + 1), M2 = eta * tril(Xbar2 X2^T + 1), out = XQ + LN(Zbar2),
//   full mini-batch: W1 -= (eta[K-1,:] XK)^T g1, W2 -= (eta[K-1,:] X2)^T g2, biases alike.
//
// Design (one CTA of 8 warps per (batch, head) chain, the whole sequence on chip):
//  * The fp32 masters W1^T (256 x 64) and W2 (256 x 64) live in tensor memory (hidden unit =
//    lane, two 128-lane tiles each) and are updated by accumulating tcgen05 MMAs.  Each
//    mini-batch refreshes their bf16 shadows in shared memory (128-byte swizzle), which are the
//    operands of the forward MMAs: W1^T as K-major A of Z1^T | (XQ W1)^T, the W2 shadow as
//    K-major A of (g2 W2^T)^T and, read MN-major, as the A operand W2^T of Z2^T and Zbar2^T.
//  * Thread u of the CTA owns hidden unit u (its tensor-memory lane): GELU, GELU', the g1
//    product and b1 are per-thread register work, written back in bf16 straight into the
//    operand layouts of the next MMAs (X2 as K-major B and MN-major A, g1 and lr-scaled g1 as
//    MN-major A).
//  * The two LayerNorms (loss gradient on Z2, output on Zbar2) run on token rows, 16 lanes per
//    row (all 8 warps), after a transpose of the 64 x 16 accumulator through shared memory.
//  * W1's update takes its lr scaling on the small operand: W1^T += g1^T (-t_{K-1} lr XK).
//  * The 16 x 16 token-pair products XQ XK^T and Xbar2 X2^T are too small for tcgen05
//    (M >= 64) and run as mma.sync m16n8k16 on the same shared-memory tiles.
//  * One thread issues every tcgen05.mma and commits to one mbarrier; all waits are bounded.
//    XQ, XK, XV tiles arrive by TMA (box {64, K}, 128-byte swizzle, no multicast) into a ring.
#include "tc5.cuh"
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;
constexpr int kHid = TTT_HIDDEN;
constexpr int kStages = 3;
constexpr int kTile = TTT_KMAX * 128;  // [16 rows x 128 bytes] bf16 tile
constexpr uint32_t kTmemCols = 512;
constexpr long long kDrainPolls = 1ll << 24;
// tensor-memory columns
constexpr uint32_t cW1 = 0;     // + 64 mt: W1^T tile mt (rows = hidden 128mt.., cols = input dim)
constexpr uint32_t cW2 = 128;   // + 64 mt: W2 tile mt (rows = hidden, cols = output dim)
constexpr uint32_t cZQ = 256;   // + 32 mt: Z1^T (cols 0..15) | (XQ W1)^T -> Zbar1^T (cols 16..31)
constexpr uint32_t cG1 = 320;   // + 16 mt: (g2 W2^T)^T
constexpr uint32_t cZ2 = 352;   // M = 64: Z2^T
constexpr uint32_t cZB2 = 368;  // M = 64: Zbar2^T

struct __align__(1024) MlpSmem {
    uint8_t stage[kStages][3 * kTile];  // XK | XQ | XV (XK, XQ adjacent: the N = 32 B operand)
    uint8_t W1s[2][128 * 128];          // bf16 W1^T shadow, K-major [tile][128 hidden rows x 128 B]
    uint8_t W2s[kHid * 128];            // bf16 W2 shadow [256 hidden rows x 128 B (64 outputs)]
    uint8_t X2s[4 * kTile];             // bf16 X2     [4 hidden blocks][16 token rows x 128 B]
    uint8_t XB2s[4 * kTile];            // bf16 Xbar2
    uint8_t G1s[4 * kTile];             // bf16 g1
    uint8_t XKL[kTile];                 // bf16 -t_{K-1} lr XK [16 token rows x 128 B]
    uint8_t G2s[kTile];                 // bf16 g2 [16 token rows x 128 B (64 outputs)]
    uint8_t G2Ls[kTile];                // bf16 -t_{K-1} lr g2
    uint8_t M1s[kTile];                 // bf16 -M1, row i, cols j < 16
    uint8_t M2s[kTile];                 // bf16 -M2
    float Zt[TTT_KMAX][TTT_D];          // Z2, then Zbar2, as token rows
    float A2p[4][TTT_KMAX][TTT_KMAX];   // Xbar2 X2^T partial sums over the 4 hidden blocks
    float b2[TTT_D];
    float b2part[8][TTT_D];
    float lr[kStages][TTT_KMAX];
    float te[TTT_KMAX];
    uint64_t full[kStages];
    uint64_t mma_bar;
    uint64_t drain_bar;
    uint32_t tmem_base;
    int fail;
};

// byte offset of bf16 element (row r, col c < 64) in a [rows x 128 B] tile, 128-byte swizzle
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return static_cast<uint32_t>(r * 128 + ((((c >> 3) ^ (r & 7))) << 4) + ((c & 7) << 1));
}

__device__ __forceinline__ void st_bf16(uint8_t* base, uint32_t off, float v) {
    *reinterpret_cast<__nv_bfloat16*>(base + off) = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float tanh_fast(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// tanh form of GELU and its derivative
__device__ __forceinline__ void gelu2(float x, float& y, float& dy) {
    const float k = 0.7978845608028654f, c = 0.044715f;
    const float th = tanh_fast(k * fmaf(c * x, x * x, x));
    y = 0.5f * x * (1.0f + th);
    dy = 0.5f * (1.0f + th) + 0.5f * x * (1.0f - th * th) * k * fmaf(3.0f * c, x * x, 1.0f);
}
__device__ __forceinline__ float gelu(float x) {
    const float k = 0.7978845608028654f, c = 0.044715f;
    return 0.5f * x * (1.0f + tanh_fast(k * fmaf(c * x, x * x, x)));
}

// Mean and 1/sqrt(var + eps) of a 64-value row held 4 per lane by 16 lanes (Chan merges).
__device__ __forceinline__ void row_stats16(const float (&v)[4], float eps, float& mu, float& rstd) {
    float m = 0.25f * ((v[0] + v[1]) + (v[2] + v[3]));
    float M2 = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) M2 = fmaf(v[i] - m, v[i] - m, M2);
#pragma unroll
    for (int off = 1; off < 16; off <<= 1) {
        const float mo = __shfl_xor_sync(0xffffffffu, m, off);
        const float M2o = __shfl_xor_sync(0xffffffffu, M2, off);
        const float dm = mo - m;
        M2 = M2 + M2o + dm * dm * (2.0f * off);
        m = 0.5f * (m + mo);
    }
    mu = m;
    rstd = rsqrtf(M2 * (1.0f / TTT_D) + eps);
}

__device__ __forceinline__ float sum16(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    v += __shfl_xor_sync(0xffffffffu, v, 4);
    v += __shfl_xor_sync(0xffffffffu, v, 8);
    return v;
}


// 4 consecutive bf16 of row r starting at column c (c % 4 == 0) -> floats
__device__ __forceinline__ void ld4_bf16(const uint8_t* tile, int r, int c, float* out) {
    const uint2 v = *reinterpret_cast<const uint2*>(tile + swz(r, c));
    const float2 a = unpack_bf16x2(v.x), b = unpack_bf16x2(v.y);
    out[0] = a.x; out[1] = a.y; out[2] = b.x; out[3] = b.y;
}
__device__ __forceinline__ void st4_bf16(uint8_t* tile, int r, int c, float a, float b, float d, float e) {
    *reinterpret_cast<uint2*>(tile + swz(r, c)) = make_uint2(pack_bf16x2(a, b), pack_bf16x2(d, e));
}

__global__ void __launch_bounds__(kThreads, 1)
mlp_tc_kernel(const MlpArgs a, const __grid_constant__ LinearMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    MlpSmem& s = *reinterpret_cast<MlpSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int q = w & 3, mt = w >> 2;            // tensor-memory lane quarter and 128-lane tile
    const int u = 128 * mt + 32 * q + lane;      // the hidden unit this thread owns
    const int g = lane >> 2, t4 = lane & 3;
    const int chain = blockIdx.x;
    const int h = chain % a.H;
    const int K = a.K;
    const int n_full = static_cast<int>(a.n_full);
    const int n_mb = n_full + (a.rem > 0 ? 1 : 0);
    const float eps = a.eps;
    const long long wait_limit = a.wait_limit;
    const float* lr_g = a.lr + static_cast<long long>(chain) * a.L;
    const uint32_t tile_tx = static_cast<uint32_t>(K) * TTT_D * 2;

    // ---- set-up --------------------------------------------------------------------------------
    if (w == 0) tc5::alloc(&s.tmem_base, kTmemCols);
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&s.full[i], 1 + TTT_KMAX);
        mbar_init(&s.mma_bar, 1);
        mbar_init(&s.drain_bar, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&maps.xq);
        tma_prefetch_desc(&maps.xk);
        tma_prefetch_desc(&maps.xv);
        s.fail = 0;
    }
    for (int i = tid; i < kStages * 3 * kTile / 16; i += kThreads)
        reinterpret_cast<uint4*>(&s.stage[0][0])[i] = make_uint4(0, 0, 0, 0);  // rows >= K stay zero
    for (int i = tid; i < 2 * kTile / 16; i += kThreads)
        reinterpret_cast<uint4*>(&s.M1s[0])[i] = make_uint4(0, 0, 0, 0);
    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    const long long w0off = a.w0_chain_stride ? static_cast<long long>(chain) * a.w0_chain_stride
                                              : static_cast<long long>(h) * TTT_D * kHid;
    const long long b1off = a.w0_chain_stride ? static_cast<long long>(chain) * kHid : static_cast<long long>(h) * kHid;
    const long long b2off = a.w0_chain_stride ? static_cast<long long>(chain) * TTT_D : static_cast<long long>(h) * TTT_D;
    if (tid < TTT_D) s.b2[tid] = a.b2_0[b2off + tid];
    float b1r = a.b1_0[b1off + u];
    fence_proxy_async_smem();
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem_base;
    const uint32_t my_lane = static_cast<uint32_t>(32 * q);  // base lane of this warp's quarter

    // masters into tensor memory, bf16 shadows into shared memory
    {
        const float* W1 = a.W1_0 + w0off;  // [64 in][256 hid]
        const float* W2 = a.W2_0 + w0off;  // [256 hid][64 out]
        const int r = u & 127;             // row of this thread in its 128-row tile
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float v1[16], v2[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                v1[i] = W1[(16 * c + i) * kHid + u];
                v2[i] = W2[u * TTT_D + 16 * c + i];
            }
            tc5::st16(tc5::taddr(tm, my_lane, cW1 + 64 * mt + 16 * c), v1);
            tc5::st16(tc5::taddr(tm, my_lane, cW2 + 64 * mt + 16 * c), v2);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int cc = 16 * c + 8 * half;  // 8 columns = one 16-byte chunk
                uint4 p1, p2;
                p1.x = pack_bf16x2(v1[8 * half + 0], v1[8 * half + 1]); p1.y = pack_bf16x2(v1[8 * half + 2], v1[8 * half + 3]);
                p1.z = pack_bf16x2(v1[8 * half + 4], v1[8 * half + 5]); p1.w = pack_bf16x2(v1[8 * half + 6], v1[8 * half + 7]);
                p2.x = pack_bf16x2(v2[8 * half + 0], v2[8 * half + 1]); p2.y = pack_bf16x2(v2[8 * half + 2], v2[8 * half + 3]);
                p2.z = pack_bf16x2(v2[8 * half + 4], v2[8 * half + 5]); p2.w = pack_bf16x2(v2[8 * half + 6], v2[8 * half + 7]);
                *reinterpret_cast<uint4*>(&s.W1s[mt][0] + swz(r, cc)) = p1;
                *reinterpret_cast<uint4*>(&s.W2s[0] + swz(u, cc)) = p2;
            }
        }
        tc5::wait_st();
    }
    fence_proxy_async_smem();
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();

    // producer (warp 0): mini-batch mm into stage st
    auto issue = [&](int mm, int st) {
        const int Kmm = mm < n_full ? K : static_cast<int>(a.rem);
        const int row0 = mm * K;
        if (lane == 0) {
            mbar_arrive_expect_tx(&s.full[st], 3 * tile_tx);
            tma_load_3d(&s.stage[st][0], &maps.xk, 0, row0, chain, &s.full[st]);
            tma_load_3d(&s.stage[st][kTile], &maps.xq, 0, row0, chain, &s.full[st]);
            tma_load_3d(&s.stage[st][2 * kTile], &maps.xv, 0, row0, chain, &s.full[st]);
        }
        if (lane < TTT_KMAX) {
            if (lane < Kmm) {
                cp_async_4(&s.lr[st][lane], lr_g + row0 + lane);
                cp_async_mbar_arrive_noinc(&s.full[st]);
            } else {
                s.lr[st][lane] = 0.f;
                mbar_arrive(&s.full[st]);
            }
        }
    };
    if (w == 0)
        for (int mm = 0; mm < kStages - 1 && mm < n_mb; ++mm) issue(mm, mm);

    // row-phase geometry (all 8 warps): token row rr, features f4..f4+3 (16 lanes per row)
    const int rr = tid >> 4, f4 = 4 * (tid & 15);
    float lw[4], lb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lw[i] = a.ln_w[h * TTT_D + f4 + i];
        lb[i] = a.ln_b[h * TTT_D + f4 + i];
    }
    const float tl = s.te[K - 1];
    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row supplied by this lane
    const int lchunk = lane >> 4;
    const uint32_t idZQ = tc5::idesc_bf16(128, 32, 0, 0);
    const uint32_t idM64 = tc5::idesc_bf16(64, 16, 1, 0);
    const uint32_t idG1 = tc5::idesc_bf16(128, 16, 0, 0);
    const uint32_t idC1 = tc5::idesc_bf16(128, 16, 1, 0);
    const uint32_t idUp = tc5::idesc_bf16(128, 64, 1, 1);

    // Operand descriptors, built once: per MMA only a constant offset is added (the single
    // issuing thread is otherwise the bottleneck of these small-N MMAs).
    const uint64_t dW1k = tc5::sdesc(smem_u32(&s.W1s[0][0]), 16, 1024);     // W1^T, K-major A
    const uint64_t dW2k = tc5::sdesc(smem_u32(&s.W2s[0]), 16, 1024);        // W2, K-major A
    const uint64_t dW2m = tc5::sdesc(smem_u32(&s.W2s[0]), 2048, 1024);      // W2^T, MN-major A (M = 64)
    const uint64_t dX2k = tc5::sdesc(smem_u32(&s.X2s[0]), 16, 1024);        // X2, K-major B
    const uint64_t dX2m = tc5::sdesc(smem_u32(&s.X2s[0]), kTile, 1024);     // X2^T, MN-major A
    const uint64_t dXB2k = tc5::sdesc(smem_u32(&s.XB2s[0]), 16, 1024);      // Xbar2, K-major B
    const uint64_t dG1m = tc5::sdesc(smem_u32(&s.G1s[0]), kTile, 1024);     // g1^T, MN-major A
    const uint64_t dXKLm = tc5::sdesc(smem_u32(&s.XKL[0]), kTile, 1024);    // -t lr XK, MN-major B
    const uint64_t dG2k = tc5::sdesc(smem_u32(&s.G2s[0]), 16, 1024);        // g2, K-major B
    const uint64_t dG2m = tc5::sdesc(smem_u32(&s.G2s[0]), 2048, 1024);      // g2^T, MN-major A (M = 64)
    const uint64_t dG2Lm = tc5::sdesc(smem_u32(&s.G2Ls[0]), kTile, 1024);   // -t lr g2, MN-major B
    const uint64_t dM1k = tc5::sdesc(smem_u32(&s.M1s[0]), 16, 1024);        // -M1, K-major B
    const uint64_t dM2k = tc5::sdesc(smem_u32(&s.M2s[0]), 16, 1024);        // -M2, K-major B
    const uint64_t dSk = tc5::sdesc(smem_u32(&s.stage[0][0]), 16, 1024);    // [XK; XQ] of stage 0, K-major B
    const uint64_t dSm = tc5::sdesc(smem_u32(&s.stage[0][0]), kTile, 1024); // XK of stage 0, MN-major B

    uint32_t mpar = 0;  // phase parity of mma_bar
    auto mma_wait = [&]() {
        if (!mbar_wait_bounded(&s.mma_bar, mpar, wait_limit, a.status)) s.fail = 1;
        mpar ^= 1;
        tc5::fence_after();
    };
    auto sync_operands = [&]() {  // generic-proxy smem writes -> visible to the tensor cores
        fence_proxy_async_smem();
        tc5::fence_before();
        __syncthreads();
        tc5::fence_after();
    };

    int st = 0;
    uint32_t par = 0;
    int m_stop = n_mb;  // first mini-batch whose loads may still be in flight (failure path)
    for (int m = 0; m < n_mb; ++m, st = (st + 1 == kStages ? 0 : st + 1), par ^= (st == 0)) {
        const bool full_mb = m < n_full;
        const int Km = full_mb ? K : static_cast<int>(a.rem);
        if (w == 0 && m + kStages - 1 < n_mb) issue(m + kStages - 1, (m + kStages - 1) % kStages);
        if (!mbar_wait_bounded(&s.full[st], par, wait_limit, a.status)) s.fail = 1;
        uint8_t* xk_t = &s.stage[st][0];
        uint8_t* xq_t = &s.stage[st][kTile];
        const uint8_t* xv_t = &s.stage[st][2 * kTile];
        const float* lr_s = s.lr[st];

        // (1) Z1^T | (XQ W1)^T = W1^T [XK; XQ]^T
        if (tid == 0) {
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc5::mma_ss(tm + cZQ + 32 * t2, tc5::sdesc_add(dW1k, t2 * 16384 + 32 * ks),
                                tc5::sdesc_add(dSk, st * 3 * kTile + 32 * ks), idZQ, ks > 0);
            tc5::commit(&s.mma_bar);
        }
        // meanwhile: -M1 = -(eta * tril(XQ XK^T + 1)) into M1s (warp 4, mma.sync)
        if (w == 4) {
            float at[2][4] = {};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t k0, k1, k2, k3, q0, q1, q2, q3;
                ldmatrix_x4(smem_u32(xk_t) + swz128(lrow, 2 * kk + lchunk), k0, k1, k2, k3);
                ldmatrix_x4(smem_u32(xq_t) + swz128(lrow, 2 * kk + lchunk), q0, q1, q2, q3);
                mma_bf16_16816(at[0], q0, q1, q2, q3, k0, k2);
                mma_bf16_16816(at[1], q0, q1, q2, q3, k1, k3);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int i = g + 8 * (e >> 1), j = 8 * nt + 2 * t4 + (e & 1);
                    const float mv = (j <= i) ? s.te[i] * lr_s[j] * (at[nt][e] + 1.0f) : 0.f;
                    st_bf16(&s.M1s[0], swz(i, j), -mv);
                }
        }
        mma_wait();

        // (2) X2 = gelu(Z1 + b1), by hidden unit; keep gelu'(Z1 + b1)
        float dg[16];
        {
            float z1[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cZQ + 32 * mt), z1);
            tc5::wait_ld();
            uint8_t* xb = &s.X2s[(u >> 6) * kTile];
#pragma unroll
            for (int tt = 0; tt < 16; ++tt) {
                float y;
                gelu2(z1[tt] + b1r, y, dg[tt]);
                st_bf16(xb, swz(tt, u & 63), y);
            }
        }
        sync_operands();

        // (3) Z2^T = W2^T X2^T (M = 64 outputs, K = 256 hidden)
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 16; ++ks)
                tc5::mma_ss(tm + cZ2, tc5::sdesc_add(dW2m, 2048 * ks),
                            tc5::sdesc_add(dX2k, (ks >> 2) * kTile + 32 * (ks & 3)), idM64,
                            ks > 0);
            tc5::commit(&s.mma_bar);
        }
        mma_wait();
        if (w < 4) {  // rows 16q..16q+15 of the M = 64 accumulator sit in lanes 32q..32q+15
            float v[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cZ2), v);
            tc5::wait_ld();
            if (lane < 16)
#pragma unroll
                for (int tt = 0; tt < 16; ++tt) s.Zt[tt][16 * q + lane] = v[tt];
        }
        __syncthreads();

        // (4) g2 = ln_fused_l2_bwd(Z2 + b2, XV - XK) on token rows; also -t lr XK for W1's update
        {
            float z[4], xk[4], xv[4];
            const float4 zz = *reinterpret_cast<const float4*>(&s.Zt[rr][f4]);
            const float4 bb = *reinterpret_cast<const float4*>(&s.b2[f4]);
            z[0] = zz.x + bb.x; z[1] = zz.y + bb.y; z[2] = zz.z + bb.z; z[3] = zz.w + bb.w;
            ld4_bf16(xk_t, rr, f4, xk);
            ld4_bf16(xv_t, rr, f4, xv);
            float mu, rs;
            row_stats16(z, eps, mu, rs);
            float xh[4], qv[4], sq = 0.f, sqx = 0.f;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                xh[i] = (z[i] - mu) * rs;
                qv[i] = lw[i] * (fmaf(lw[i], xh[i], lb[i]) - (xv[i] - xk[i]));
                sq += qv[i];
                sqx = fmaf(qv[i], xh[i], sqx);
            }
            sq = sum16(sq);
            sqx = sum16(sqx);
            const float sc = (rr < Km) ? rs * (1.0f / TTT_D) : 0.f;
            float g2[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) g2[i] = fmaf(-xh[i], sqx, fmaf(static_cast<float>(TTT_D), qv[i], -sq)) * sc;
            st4_bf16(&s.G2s[0], rr, f4, g2[0], g2[1], g2[2], g2[3]);
            const float ls = -tl * lr_s[rr];
            st4_bf16(&s.G2Ls[0], rr, f4, ls * g2[0], ls * g2[1], ls * g2[2], ls * g2[3]);
            st4_bf16(&s.XKL[0], rr, f4, ls * xk[0], ls * xk[1], ls * xk[2], ls * xk[3]);
            // b2: sum over this warp's 2 token rows of lr g2
            float bs[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                bs[i] = lr_s[rr] * g2[i];
                bs[i] += __shfl_xor_sync(0xffffffffu, bs[i], 16);
            }
            if (lane < 16) *reinterpret_cast<float4*>(&s.b2part[w][f4]) = make_float4(bs[0], bs[1], bs[2], bs[3]);
        }
        sync_operands();

        // (5) (g2 W2^T)^T = W2 g2^T (M = 256 hidden in two tiles, K = 64 outputs)
        if (tid == 0) {
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    tc5::mma_ss(tm + cG1 + 16 * t2, tc5::sdesc_add(dW2k, t2 * 16384 + 32 * ks),
                                tc5::sdesc_add(dG2k, 32 * ks), idG1, ks > 0);
            tc5::commit(&s.mma_bar);
        }
        mma_wait();

        // (6) g1 = (g2 W2^T) * gelu'(Z1 + b1), by hidden unit
        float b1sum = 0.f;
        {
            float gr[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cG1 + 16 * mt), gr);
            tc5::wait_ld();
            uint8_t* gb = &s.G1s[(u >> 6) * kTile];
#pragma unroll
            for (int tt = 0; tt < 16; ++tt) {
                const float gv = gr[tt] * dg[tt];
                st_bf16(gb, swz(tt, u & 63), gv);
                b1sum = fmaf(lr_s[tt], gv, b1sum);
            }
        }
        sync_operands();

        // (7) Zbar1^T = (XQ W1)^T - g1^T M1^T; (11) the state update on a full mini-batch
        if (tid == 0) {
#pragma unroll
            for (int t2 = 0; t2 < 2; ++t2)
                tc5::mma_ss(tm + cZQ + 32 * t2 + 16, tc5::sdesc_add(dG1m, t2 * 2 * kTile), dM1k, idC1, 1);
            if (full_mb) {
#pragma unroll
                for (int t2 = 0; t2 < 2; ++t2) {
                    // W1^T += g1^T (-t lr XK) ;  W2 += X2^T (-t lr g2)
                    tc5::mma_ss(tm + cW1 + 64 * t2, tc5::sdesc_add(dG1m, t2 * 2 * kTile), dXKLm, idUp, 1);
                    tc5::mma_ss(tm + cW2 + 64 * t2, tc5::sdesc_add(dX2m, t2 * 2 * kTile), dG2Lm, idUp, 1);
                }
            }
            tc5::commit(&s.mma_bar);
        }
        mma_wait();

        // (8) Xbar2 = gelu(Zbar1 + b1), by hidden unit; then b1's update
        {
            float zb[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cZQ + 32 * mt + 16), zb);
            tc5::wait_ld();
            uint8_t* xb = &s.XB2s[(u >> 6) * kTile];
#pragma unroll
            for (int tt = 0; tt < 16; ++tt) st_bf16(xb, swz(tt, u & 63), gelu(zb[tt] + b1r));
            if (full_mb) b1r -= tl * b1sum;
        }
        __syncthreads();
        // Xbar2 X2^T partial sums over hidden block w (warps 0..3, mma.sync)
        if (w < 4) {
            float at[2][4] = {};
            const uint32_t xa = smem_u32(&s.XB2s[w * kTile]), xb = smem_u32(&s.X2s[w * kTile]);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t a0, a1, a2, a3, b0, b1, b2, b3;
                ldmatrix_x4(xa + swz128(lrow, 2 * kk + lchunk), a0, a1, a2, a3);
                ldmatrix_x4(xb + swz128(lrow, 2 * kk + lchunk), b0, b1, b2, b3);
                mma_bf16_16816(at[0], a0, a1, a2, a3, b0, b2);
                mma_bf16_16816(at[1], a0, a1, a2, a3, b1, b3);
            }
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                s.A2p[w][g][8 * nt + 2 * t4] = at[nt][0];
                s.A2p[w][g][8 * nt + 2 * t4 + 1] = at[nt][1];
                s.A2p[w][g + 8][8 * nt + 2 * t4] = at[nt][2];
                s.A2p[w][g + 8][8 * nt + 2 * t4 + 1] = at[nt][3];
            }
        }
        __syncthreads();
        {  // -M2 = -(eta * tril(Xbar2 X2^T + 1)), one element per thread
            const int i = tid >> 4, j = tid & 15;
            const float a2 = s.A2p[0][i][j] + s.A2p[1][i][j] + s.A2p[2][i][j] + s.A2p[3][i][j];
            const float mv = (j <= i) ? s.te[i] * lr_s[j] * (a2 + 1.0f) : 0.f;
            st_bf16(&s.M2s[0], swz(i, j), -mv);
        }
        sync_operands();

        // (9) Zbar2^T = W2^T Xbar2^T - g2^T M2^T (M = 64)
        if (tid == 0) {
#pragma unroll
            for (int ks = 0; ks < 16; ++ks)
                tc5::mma_ss(tm + cZB2, tc5::sdesc_add(dW2m, 2048 * ks),
                            tc5::sdesc_add(dXB2k, (ks >> 2) * kTile + 32 * (ks & 3)), idM64,
                            ks > 0);
            tc5::mma_ss(tm + cZB2, dG2m, dM2k,
                        idM64, 1);
            tc5::commit(&s.mma_bar);
        }
        mma_wait();
        if (w < 4) {
            float v[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cZB2), v);
            tc5::wait_ld();
            if (lane < 16)
#pragma unroll
                for (int tt = 0; tt < 16; ++tt) s.Zt[tt][16 * q + lane] = v[tt];
        }
        __syncthreads();

        // (10) out = XQ + LN(Zbar2 + b2) on token rows
        {
            float z[4], xq[4];
            const float4 zz = *reinterpret_cast<const float4*>(&s.Zt[rr][f4]);
            const float4 bb = *reinterpret_cast<const float4*>(&s.b2[f4]);
            z[0] = zz.x + bb.x; z[1] = zz.y + bb.y; z[2] = zz.z + bb.z; z[3] = zz.w + bb.w;
            ld4_bf16(xq_t, rr, f4, xq);
            float mu, rs;
            row_stats16(z, eps, mu, rs);
            if (rr < Km) {
                float o[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) o[i] = xq[i] + fmaf(lw[i], (z[i] - mu) * rs, lb[i]);
                __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) +
                                     (static_cast<long long>(chain) * a.L + static_cast<long long>(m) * K + rr) * TTT_D;
                *reinterpret_cast<uint2*>(out + f4) = make_uint2(pack_bf16x2(o[0], o[1]), pack_bf16x2(o[2], o[3]));
            }
        }
        __syncthreads();

        // (12) new state: b2, and the bf16 shadows of the updated masters
        if (full_mb) {
            if (tid < TTT_D)
                s.b2[tid] -= tl * (((s.b2part[0][tid] + s.b2part[1][tid]) + (s.b2part[2][tid] + s.b2part[3][tid])) +
                                   ((s.b2part[4][tid] + s.b2part[5][tid]) + (s.b2part[6][tid] + s.b2part[7][tid])));
            const int r = u & 127;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                float v1[16], v2[16];
                tc5::ld16(tc5::taddr(tm, my_lane, cW1 + 64 * mt + 16 * c), v1);
                tc5::ld16(tc5::taddr(tm, my_lane, cW2 + 64 * mt + 16 * c), v2);
                tc5::wait_ld();
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int cc = 16 * c + 8 * half;
                    uint4 p1, p2;
                    p1.x = pack_bf16x2(v1[8 * half + 0], v1[8 * half + 1]); p1.y = pack_bf16x2(v1[8 * half + 2], v1[8 * half + 3]);
                    p1.z = pack_bf16x2(v1[8 * half + 4], v1[8 * half + 5]); p1.w = pack_bf16x2(v1[8 * half + 6], v1[8 * half + 7]);
                    p2.x = pack_bf16x2(v2[8 * half + 0], v2[8 * half + 1]); p2.y = pack_bf16x2(v2[8 * half + 2], v2[8 * half + 3]);
                    p2.z = pack_bf16x2(v2[8 * half + 4], v2[8 * half + 5]); p2.w = pack_bf16x2(v2[8 * half + 6], v2[8 * half + 7]);
                    *reinterpret_cast<uint4*>(&s.W1s[mt][0] + swz(r, cc)) = p1;
                    *reinterpret_cast<uint4*>(&s.W2s[0] + swz(u, cc)) = p2;
                }
            }
        }
        sync_operands();
        if (s.fail) {
            m_stop = m;
            break;
        }
    }

    // ---- final state (the masters) ----------------------------------------------------------------
    if (!s.fail) {
        float* W1l = a.W1_last + static_cast<long long>(chain) * TTT_D * kHid;
        float* W2l = a.W2_last + static_cast<long long>(chain) * TTT_D * kHid;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            float v1[16], v2[16];
            tc5::ld16(tc5::taddr(tm, my_lane, cW1 + 64 * mt + 16 * c), v1);
            tc5::ld16(tc5::taddr(tm, my_lane, cW2 + 64 * mt + 16 * c), v2);
            tc5::wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                W1l[(16 * c + i) * kHid + u] = v1[i];
                W2l[u * TTT_D + 16 * c + i] = v2[i];
            }
        }
        a.b1_last[static_cast<long long>(chain) * kHid + u] = b1r;
        if (tid < TTT_D) a.b2_last[static_cast<long long>(chain) * TTT_D + tid] = s.b2[tid];
    } else if (tid == 0) {
        // A wait gave up: let the MMAs and the loads still in flight land (bounded) before the
        // tensor memory is freed and the CTA exits.  Mini-batches m_stop .. issued-1 were loaded
        // but not consumed; the drain commit arrives once every MMA issued so far has finished.
        tc5::commit(&s.drain_bar);
        mbar_wait_bounded(&s.drain_bar, 0, kDrainPolls, nullptr);
        const int issued = min(n_mb, m_stop + kStages);
        for (int mm = m_stop; mm < issued; ++mm)
            mbar_wait_bounded(&s.full[mm % kStages], static_cast<uint32_t>((mm / kStages) & 1), kDrainPolls, nullptr);
    }
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    if (w == 0) tc5::dealloc(tm, kTmemCols);
}

}  // namespace

cudaError_t launch_mlp_tc(const MlpArgs& a, const LinearMaps& maps, cudaStream_t st) {
    const size_t smem = sizeof(MlpSmem) + 1024;  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(mlp_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    mlp_tc_kernel<<<static_cast<unsigned>(a.B * a.H), kThreads, smem, st>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace ttt
