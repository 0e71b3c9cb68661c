// linear_tc.cu -- TTT-Linear prefill, bf16 tensor-core kernel (fp32 accumulation, fp32 state).
//
// The method ("代码连连看——TTT", compute_mini_batch, dual branch), per chain and mini-batch of
// K <= 16 tokens, state (W, b):
//   Z = XK W + b;  g = ln_fused_l2_bwd(Z, XV - XK)
//   Zbar = XQ W + b - M g,  M = eta * tril(XQ XK^T + 1),  eta[i][j] = t_i lr_j
//   out = XQ + LN(Zbar);  full mini-batch: W -= (eta[K-1,:] * XK)^T g,  b -= sum_j eta[K-1,j] g_j
//
// Design (one persistent CTA of 4 warps per (batch, head) chain, the whole sequence on chip):
//  * The fp32 master state W^T (64x64) lives in mma.sync accumulator registers: warp w owns
//    output features 16w..16w+15, i.e. rows 16w.. of W^T, as eight m16n8 fragments.  The
//    accumulator layout of W^T is exactly the B-operand layout of W for Z = XK W, so each
//    mini-batch only rounds the accumulators to bf16 pairs; the rank-K update of W is an MMA
//    that accumulates straight into the same registers.  W never leaves the SM.
//  * The dense contractions are m16n8k16 bf16 MMAs: Z and XQ W (16x64x64), XQ XK^T (16x16x64),
//    M g (16x16x64) and the update (64x16x64).  g enters the B and A operands through
//    movmatrix (register transposes), with no shared-memory round trip.
//  * LayerNorm statistics: each thread holds 2 rows x 4 features, quads reduce with shuffles,
//    the 4 warps merge (sum, centred sum of squares) pairs through shared memory (Chan's
//    formula), so the loss gradient costs two 128-thread barriers per mini-batch.  The output
//    LayerNorm of mini-batch m is finished during mini-batch m+1 and shares those barriers.
//  * A TMA ring of kStages mini-batches (XQ, XK, XV tiles with 128-byte swizzle, box {64, K})
//    plus cp.async for lr, tracked by one mbarrier per stage, prefetches ahead of the scan; the
//    output tile is staged in shared memory and written back by a TMA store.  All mbarrier
//    waits are bounded; on expiry the kernel raises the status word, drains its in-flight
//    copies (again bounded) and returns.
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kWarps = 4;
constexpr int kThreads = 32 * kWarps;
constexpr int kStages = 4;
constexpr int kTileBytes = TTT_KMAX * TTT_D * 2;  // 16 rows x 128 bytes
constexpr long long kDrainPolls = 1ll << 24;

struct __align__(1024) TcSmem {
    uint8_t xq[kStages][kTileBytes];
    uint8_t xk[kStages][kTileBytes];
    uint8_t xv[kStages][kTileBytes];
    uint8_t outb[2][kTileBytes];
    float gtail[TTT_KMAX][TTT_D];      // tail grads (fp32), only on the remainder mini-batch
    float lr[kStages][TTT_KMAX];
    float te[TTT_KMAX];
    float2 red1[kWarps][TTT_KMAX];     // Z rows: (sum, centred sum of squares) per warp
    float2 red2[kWarps][TTT_KMAX];     // (sum q, sum q * xhat) per warp
    float2 red3[kWarps][TTT_KMAX];     // Zbar rows of the previous mini-batch
    uint64_t full[kStages];
    int fail;
};

// Sum over the 4 lanes of a quad (lanes sharing rows g, g+8).
__device__ __forceinline__ float quad_sum(float v) {
    v += __shfl_xor_sync(0xffffffffu, v, 1);
    v += __shfl_xor_sync(0xffffffffu, v, 2);
    return v;
}

// Per-warp row partials of a [16 x 16-feature] slice held as v[nt][0..3] (rows g and g+8):
// returns (sum, centred sum of squares) over this warp's 16 features for each of the 2 rows.
__device__ __forceinline__ void warp_row_partials(const float (&v)[2][4], float2& r0, float2& r1) {
    float s0 = quad_sum(v[0][0] + v[0][1] + v[1][0] + v[1][1]);
    float s1 = quad_sum(v[0][2] + v[0][3] + v[1][2] + v[1][3]);
    float m0 = s0 * (1.0f / 16), m1 = s1 * (1.0f / 16);
    float c0 = 0.f, c1 = 0.f;
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
        float a = v[nt][0] - m0, b = v[nt][1] - m0, c = v[nt][2] - m1, d = v[nt][3] - m1;
        c0 += a * a + b * b;
        c1 += c * c + d * d;
    }
    r0 = make_float2(s0, quad_sum(c0));
    r1 = make_float2(s1, quad_sum(c1));
}

// Merge the 4 warps' partials of one row into mean and 1/sqrt(var + eps).
__device__ __forceinline__ void merge_row(const float2 (*red)[TTT_KMAX], int row, float eps,
                                          float& mu, float& rstd) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) s += red[w][row].x;
    mu = s * (1.0f / TTT_D);
    float m2 = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        float dm = red[w][row].x * (1.0f / 16) - mu;
        m2 += red[w][row].y + 16.0f * dm * dm;
    }
    rstd = rsqrtf(m2 * (1.0f / TTT_D) + eps);
}

__global__ void __launch_bounds__(kThreads, 2)
linear_tc_kernel(const LinearArgs a, const __grid_constant__ LinearMaps maps) {
    extern __shared__ uint8_t smem_raw[];
    TcSmem& s = *reinterpret_cast<TcSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

    const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int chain = blockIdx.x;
    const int h = chain % a.H;
    const int K = a.K;
    const long long n_mb = a.n_full + (a.rem > 0 ? 1 : 0);
    const float* lr_g = a.lr + static_cast<long long>(chain) * a.L;
    const uint32_t tile_tx = static_cast<uint32_t>(K) * TTT_D * 2;

    // ---- set-up ------------------------------------------------------------------------------
    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) mbar_init(&s.full[i], 1 + TTT_KMAX);
        fence_mbarrier_init();
        tma_prefetch_desc(&maps.xq);
        tma_prefetch_desc(&maps.xk);
        tma_prefetch_desc(&maps.xv);
        tma_prefetch_desc(&maps.out);
        s.fail = 0;
    }
    // rows K..15 of every tile stay zero for the whole run (TMA writes rows < K only)
    for (int i = tid; i < kStages * kTileBytes / 16; i += kThreads) {
        reinterpret_cast<uint4*>(&s.xq[0][0])[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(&s.xk[0][0])[i] = make_uint4(0, 0, 0, 0);
        reinterpret_cast<uint4*>(&s.xv[0][0])[i] = make_uint4(0, 0, 0, 0);
    }
    if (tid < TTT_KMAX) s.te[tid] = a.token_eta ? (tid < K ? a.token_eta[tid] : 0.f) : 1.0f / (tid + 1);
    fence_proxy_async_smem();
    __syncthreads();

    // producer: warp 0 loads mini-batch mm into stage mm % kStages
    auto issue = [&](long long mm) {
        const int st = static_cast<int>(mm % kStages);
        const int Kmm = mm < a.n_full ? K : static_cast<int>(a.rem);
        const int row0 = static_cast<int>(mm * K);
        if (lane == 0) {
            mbar_arrive_expect_tx(&s.full[st], 3 * tile_tx);
            tma_load_3d(&s.xq[st][0], &maps.xq, 0, row0, chain, &s.full[st]);
            tma_load_3d(&s.xk[st][0], &maps.xk, 0, row0, chain, &s.full[st]);
            tma_load_3d(&s.xv[st][0], &maps.xv, 0, row0, chain, &s.full[st]);
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
    long long issued = 0;
    if (w == 0)
        for (; issued < kStages - 1 && issued < n_mb; ++issued) issue(issued);

    // ---- state: W^T accumulators, b, LayerNorm affine --------------------------------------
    const long long w0off = a.w0_chain_stride ? static_cast<long long>(chain) * a.w0_chain_stride
                                              : static_cast<long long>(h) * TTT_D * TTT_D;
    const long long b0off = a.w0_chain_stride ? static_cast<long long>(chain) * TTT_D
                                              : static_cast<long long>(h) * TTT_D;
    float Wt[8][4];  // Wt[jt][e]: W^T[16w + g + 8(e>>1)][8jt + 2t + (e&1)]
#pragma unroll
    for (int jt = 0; jt < 8; ++jt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int j = 8 * jt + 2 * t + (e & 1), f = 16 * w + g + 8 * (e >> 1);
            Wt[jt][e] = a.W0[w0off + j * TTT_D + f];
        }
    float bc[2][2], lw[2][2], lb[2][2];  // per n-tile nt, feature 16w + 8nt + 2t + e
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            int f = 16 * w + 8 * nt + 2 * t + e;
            bc[nt][e] = a.b0[b0off + f];
            lw[nt][e] = a.ln_w[h * TTT_D + f];
            lb[nt][e] = a.ln_b[h * TTT_D + f];
        }

    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;  // ldmatrix row supplied by this lane
    const int lchunk = lane >> 4;
    float zbar_prev[2][4];
    uint32_t xq_prev[2][2];  // bf16 pairs of XQ at this thread's output positions
    bool failed = false;
    long long m = 0;

    for (; m < n_mb; ++m) {
        const int st = static_cast<int>(m % kStages);
        const uint32_t par = static_cast<uint32_t>((m / kStages) & 1);
        const bool full_mb = m < a.n_full;
        const int Km = full_mb ? K : static_cast<int>(a.rem);
        if (!mbar_wait_bounded(&s.full[st], par, a.wait_limit, a.status)) s.fail = 1;

        const uint32_t xq_s = smem_u32(&s.xq[st][0]);
        const uint32_t xk_s = smem_u32(&s.xk[st][0]);
        const uint32_t xv_s = smem_u32(&s.xv[st][0]);

        // ---- Z = XK W + b, XQW = XQ W + b, Attn = XQ XK^T -----------------------------------
        float z[2][4], xqw[2][4], at[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            z[nt][0] = z[nt][2] = xqw[nt][0] = xqw[nt][2] = bc[nt][0];
            z[nt][1] = z[nt][3] = xqw[nt][1] = xqw[nt][3] = bc[nt][1];
            at[nt][0] = at[nt][1] = at[nt][2] = at[nt][3] = 0.f;
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t k0, k1, k2, k3, q0, q1, q2, q3;
            ldmatrix_x4(xk_s + swz128(lrow, 2 * kk + lchunk), k0, k1, k2, k3);
            ldmatrix_x4(xq_s + swz128(lrow, 2 * kk + lchunk), q0, q1, q2, q3);
            const uint32_t w00 = pack_bf16x2(Wt[2 * kk][0], Wt[2 * kk][1]);
            const uint32_t w01 = pack_bf16x2(Wt[2 * kk + 1][0], Wt[2 * kk + 1][1]);
            const uint32_t w10 = pack_bf16x2(Wt[2 * kk][2], Wt[2 * kk][3]);
            const uint32_t w11 = pack_bf16x2(Wt[2 * kk + 1][2], Wt[2 * kk + 1][3]);
            mma_bf16_16816(z[0], k0, k1, k2, k3, w00, w01);
            mma_bf16_16816(z[1], k0, k1, k2, k3, w10, w11);
            mma_bf16_16816(xqw[0], q0, q1, q2, q3, w00, w01);
            mma_bf16_16816(xqw[1], q0, q1, q2, q3, w10, w11);
            mma_bf16_16816(at[0], q0, q1, q2, q3, k0, k2);
            mma_bf16_16816(at[1], q0, q1, q2, q3, k1, k3);
        }

        // ---- LayerNorm statistics of Z (and of Zbar of the previous mini-batch) -------------
        {
            float2 r0, r1;
            warp_row_partials(z, r0, r1);
            if (t == 0) {
                s.red1[w][g] = r0;
                s.red1[w][g + 8] = r1;
            }
        }
        if (tid == 0 && m >= 2) bulk_wait_group_read<1>();  // out buffer (m-1)&1 is free again
        named_barrier_sync(1, kThreads);  // ---------------------------------------- B1
        if (s.fail) {
            failed = true;
            break;
        }
        if (w == 0 && issued < n_mb) issue(issued++);  // stage (m-1) % kStages is free

        // finish out of the previous mini-batch into the staging buffer
        if (m > 0) {
            float mu0, rs0, mu1, rs1;
            merge_row(s.red3, g, a.eps, mu0, rs0);
            merge_row(s.red3, g + 8, a.eps, mu1, rs1);
            uint8_t* ob = &s.outb[(m - 1) & 1][0];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                float2 x0 = unpack_bf16x2(xq_prev[nt][0]), x1 = unpack_bf16x2(xq_prev[nt][1]);
                float o00 = x0.x + lw[nt][0] * (zbar_prev[nt][0] - mu0) * rs0 + lb[nt][0];
                float o01 = x0.y + lw[nt][1] * (zbar_prev[nt][1] - mu0) * rs0 + lb[nt][1];
                float o10 = x1.x + lw[nt][0] * (zbar_prev[nt][2] - mu1) * rs1 + lb[nt][0];
                float o11 = x1.y + lw[nt][1] * (zbar_prev[nt][3] - mu1) * rs1 + lb[nt][1];
                *reinterpret_cast<uint32_t*>(ob + swz128(g, 2 * w + nt) + 4 * t) = pack_bf16x2(o00, o01);
                *reinterpret_cast<uint32_t*>(ob + swz128(g + 8, 2 * w + nt) + 4 * t) = pack_bf16x2(o10, o11);
            }
            fence_proxy_async_smem();
        }

        // ---- g = ln_fused_l2_bwd(Z, XV - XK) -------------------------------------------------
        float mu[2], rs[2];
        merge_row(s.red1, g, a.eps, mu[0], rs[0]);
        merge_row(s.red1, g + 8, a.eps, mu[1], rs[1]);
        float xh[2][4], q[2][4];
        float sq[2] = {0.f, 0.f}, sqx[2] = {0.f, 0.f};
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int hr = 0; hr < 2; ++hr) {  // row g (hr=0) or g+8 (hr=1)
                const int row = g + 8 * hr;
                float2 kv = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(
                    &s.xk[st][0] + swz128(row, 2 * w + nt) + 4 * t));
                float2 vv = unpack_bf16x2(*reinterpret_cast<const uint32_t*>(
                    &s.xv[st][0] + swz128(row, 2 * w + nt) + 4 * t));
                float tg[2] = {vv.x - kv.x, vv.y - kv.y};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float x = (z[nt][2 * hr + e] - mu[hr]) * rs[hr];
                    float qq = lw[nt][e] * (lw[nt][e] * x + lb[nt][e] - tg[e]);
                    xh[nt][2 * hr + e] = x;
                    q[nt][2 * hr + e] = qq;
                    sq[hr] += qq;
                    sqx[hr] += qq * x;
                }
            }
        }
        sq[0] = quad_sum(sq[0]); sq[1] = quad_sum(sq[1]);
        sqx[0] = quad_sum(sqx[0]); sqx[1] = quad_sum(sqx[1]);
        if (t == 0) {
            s.red2[w][g] = make_float2(sq[0], sqx[0]);
            s.red2[w][g + 8] = make_float2(sq[1], sqx[1]);
        }
        named_barrier_sync(1, kThreads);  // ---------------------------------------- B2
        if (m > 0 && tid == 0) {
            tma_store_3d(&maps.out, 0, static_cast<int>((m - 1) * K), chain, &s.outb[(m - 1) & 1][0]);
            bulk_commit_group();
        }
        float gg[2][4];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
            const int row = g + 8 * hr;
            float Sq = 0.f, Sqx = 0.f;
#pragma unroll
            for (int ww = 0; ww < kWarps; ++ww) {
                Sq += s.red2[ww][row].x;
                Sqx += s.red2[ww][row].y;
            }
            const bool valid = row < Km;
            const float sc = rs[hr] * (1.0f / TTT_D);
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = (TTT_D * q[nt][2 * hr + e] - Sq - xh[nt][2 * hr + e] * Sqx) * sc;
                    gg[nt][2 * hr + e] = valid ? v : 0.f;
                }
        }

        // ---- Zbar = XQ W + b - M g ------------------------------------------------------------
        const float* lr_s = s.lr[st];
        const float tg0 = s.te[g], tg8 = s.te[g + 8];
        const float l0 = lr_s[2 * t], l1 = lr_s[2 * t + 1], l8 = lr_s[2 * t + 8], l9 = lr_s[2 * t + 9];
        auto Mv = [&](float attn, float te_i, float lr_j, int i, int j) {
            return (j <= i) ? -(te_i * lr_j * (attn + 1.0f)) : 0.f;
        };
        const uint32_t ma0 = pack_bf16x2(Mv(at[0][0], tg0, l0, g, 2 * t), Mv(at[0][1], tg0, l1, g, 2 * t + 1));
        const uint32_t ma1 = pack_bf16x2(Mv(at[0][2], tg8, l0, g + 8, 2 * t), Mv(at[0][3], tg8, l1, g + 8, 2 * t + 1));
        const uint32_t ma2 = pack_bf16x2(Mv(at[1][0], tg0, l8, g, 2 * t + 8), Mv(at[1][1], tg0, l9, g, 2 * t + 9));
        const uint32_t ma3 = pack_bf16x2(Mv(at[1][2], tg8, l8, g + 8, 2 * t + 8), Mv(at[1][3], tg8, l9, g + 8, 2 * t + 9));
        uint32_t gb[2][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            gb[nt][0] = movmatrix_trans(pack_bf16x2(gg[nt][0], gg[nt][1]));  // tokens 0-7
            gb[nt][1] = movmatrix_trans(pack_bf16x2(gg[nt][2], gg[nt][3]));  // tokens 8-15
        }
        mma_bf16_16816(xqw[0], ma0, ma1, ma2, ma3, gb[0][0], gb[0][1]);
        mma_bf16_16816(xqw[1], ma0, ma1, ma2, ma3, gb[1][0], gb[1][1]);
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 4; ++e) zbar_prev[nt][e] = xqw[nt][e];
            xq_prev[nt][0] = *reinterpret_cast<const uint32_t*>(&s.xq[st][0] + swz128(g, 2 * w + nt) + 4 * t);
            xq_prev[nt][1] = *reinterpret_cast<const uint32_t*>(&s.xq[st][0] + swz128(g + 8, 2 * w + nt) + 4 * t);
        }
        {
            float2 r0, r1;
            warp_row_partials(zbar_prev, r0, r1);
            if (t == 0) {
                s.red3[w][g] = r0;
                s.red3[w][g + 8] = r1;
            }
        }

        // ---- state update -----------------------------------------------------------------------
        const float lg0 = lr_s[g], lg8 = lr_s[g + 8];
        if (full_mb) {
            const float tl = s.te[K - 1];
            // A = (-t_{K-1} lr_tok g)^T: features x tokens, via register transposes
            uint32_t ua[2][2];
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) {
                ua[nt][0] = movmatrix_trans(pack_bf16x2(-tl * lg0 * gg[nt][0], -tl * lg0 * gg[nt][1]));
                ua[nt][1] = movmatrix_trans(pack_bf16x2(-tl * lg8 * gg[nt][2], -tl * lg8 * gg[nt][3]));
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                uint32_t r0, r1, r2, r3;  // XK as B: tokens x input dims, j-tiles 2kk and 2kk+1
                ldmatrix_x4_trans(xk_s + swz128(lrow, 2 * kk + lchunk), r0, r1, r2, r3);
                mma_bf16_16816(Wt[2 * kk], ua[0][0], ua[1][0], ua[0][1], ua[1][1], r0, r1);
                mma_bf16_16816(Wt[2 * kk + 1], ua[0][0], ua[1][0], ua[0][1], ua[1][1], r2, r3);
            }
            // b -= t_{K-1} sum_tok lr_tok g_tok
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    float v = lg0 * gg[nt][e] + lg8 * gg[nt][2 + e];
                    v += __shfl_xor_sync(0xffffffffu, v, 4);
                    v += __shfl_xor_sync(0xffffffffu, v, 8);
                    v += __shfl_xor_sync(0xffffffffu, v, 16);
                    bc[nt][e] -= tl * v;
                }
        } else if (a.W_grad_tail || a.b_grad_tail) {
            // remainder: report the un-scaled grad sums in fp32
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    s.gtail[g][16 * w + 8 * nt + 2 * t + e] = gg[nt][e];
                    s.gtail[g + 8][16 * w + 8 * nt + 2 * t + e] = gg[nt][2 + e];
                }
            named_barrier_sync(2, kThreads);
            if (a.W_grad_tail) {
                float* Wg = a.W_grad_tail + static_cast<long long>(chain) * TTT_D * TTT_D;
                for (int i = tid; i < TTT_D * TTT_D; i += kThreads) {
                    const int r = i / TTT_D, c = i % TTT_D;
                    float acc = 0.f;
                    for (int j = 0; j < Km; ++j) {
                        const float xkv = __bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(
                            &s.xk[st][0] + swz128(j, r >> 3) + (r & 7) * 2));
                        acc = fmaf(lr_s[j] * xkv, s.gtail[j][c], acc);
                    }
                    Wg[i] = acc;
                }
            }
            if (a.b_grad_tail && tid < TTT_D) {
                float acc = 0.f;
                for (int j = 0; j < Km; ++j) acc = fmaf(lr_s[j], s.gtail[j][tid], acc);
                a.b_grad_tail[static_cast<long long>(chain) * TTT_D + tid] = acc;
            }
        }
    }

    if (failed) {
        // drain the loads still in flight (bounded), then leave
        if (tid == 0) {
            for (long long mm = m; mm < issued; ++mm)
                mbar_wait_bounded(&s.full[mm % kStages], static_cast<uint32_t>((mm / kStages) & 1),
                                  kDrainPolls, nullptr);
            bulk_wait_group<0>();
        }
        __syncthreads();
        return;
    }

    // ---- the last mini-batch's output ---------------------------------------------------------
    if (n_mb > 0) {
        if (tid == 0 && n_mb >= 2) bulk_wait_group_read<1>();
        named_barrier_sync(1, kThreads);
        float mu0, rs0, mu1, rs1;
        merge_row(s.red3, g, a.eps, mu0, rs0);
        merge_row(s.red3, g + 8, a.eps, mu1, rs1);
        uint8_t* ob = &s.outb[(n_mb - 1) & 1][0];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            float2 x0 = unpack_bf16x2(xq_prev[nt][0]), x1 = unpack_bf16x2(xq_prev[nt][1]);
            float o00 = x0.x + lw[nt][0] * (zbar_prev[nt][0] - mu0) * rs0 + lb[nt][0];
            float o01 = x0.y + lw[nt][1] * (zbar_prev[nt][1] - mu0) * rs0 + lb[nt][1];
            float o10 = x1.x + lw[nt][0] * (zbar_prev[nt][2] - mu1) * rs1 + lb[nt][0];
            float o11 = x1.y + lw[nt][1] * (zbar_prev[nt][3] - mu1) * rs1 + lb[nt][1];
            *reinterpret_cast<uint32_t*>(ob + swz128(g, 2 * w + nt) + 4 * t) = pack_bf16x2(o00, o01);
            *reinterpret_cast<uint32_t*>(ob + swz128(g + 8, 2 * w + nt) + 4 * t) = pack_bf16x2(o10, o11);
        }
        fence_proxy_async_smem();
        named_barrier_sync(1, kThreads);
        if (tid == 0) {
            tma_store_3d(&maps.out, 0, static_cast<int>((n_mb - 1) * K), chain, ob);
            bulk_commit_group();
        }
    }

    // ---- final state ------------------------------------------------------------------------
    float* Wl = a.W_last + static_cast<long long>(chain) * TTT_D * TTT_D;
#pragma unroll
    for (int jt = 0; jt < 8; ++jt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            int j = 8 * jt + 2 * t + (e & 1), f = 16 * w + g + 8 * (e >> 1);
            Wl[j * TTT_D + f] = Wt[jt][e];
        }
    if (g == 0)  // every lane group g holds the same b; lanes 0..3 of each warp write it
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 2; ++e)
                a.b_last[static_cast<long long>(chain) * TTT_D + 16 * w + 8 * nt + 2 * t + e] = bc[nt][e];
    if (a.rem == 0) {
        if (a.W_grad_tail)
            for (int i = tid; i < TTT_D * TTT_D; i += kThreads)
                a.W_grad_tail[static_cast<long long>(chain) * TTT_D * TTT_D + i] = 0.f;
        if (a.b_grad_tail && tid < TTT_D) a.b_grad_tail[static_cast<long long>(chain) * TTT_D + tid] = 0.f;
    }
    if (tid == 0) bulk_wait_group<0>();
}

}  // namespace

cudaError_t launch_linear_tc(const LinearArgs& a, const LinearMaps& maps, cudaStream_t st) {
    const size_t smem = sizeof(TcSmem) + 1024;  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(linear_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    linear_tc_kernel<<<static_cast<unsigned>(a.B * a.H), kThreads, smem, st>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace ttt
