// o_proj.cu -- the layer's output side, Y = o_proj(post_norm(X)), as one tcgen05 GEMM.
//
// The walkthrough ("代码连连看——TTT", TTTBase.forward) ends the layer with post_norm (a LayerNorm
// over the token's C = num_heads * head_dim features) and o_proj (a linear map, weight Wo [N][C])
// applied to the concatenated scan output.  Both are per token, and the LayerNorm folds into the
// GEMM: with mu, rstd the token's statistics, gamma = ln_w, beta = ln_b,
//   y[n] = sum_k (gamma_k (x_k - mu) rstd + beta_k) Wo[n][k]
//        = rstd (sum_k x_k Wp[n][k] - mu u[n]) + v[n],
//   Wp[n][k] = gamma_k Wo[n][k] (bf16),  u[n] = sum_k Wp[n][k],  v[n] = sum_k beta_k Wo[n][k],
// so the tensor cores multiply the raw X by a once-packed weight (oproj_prepare_kernel; u sums
// the rounded Wp, so the correction matches what the MMAs multiply), and the statistics are
// taken from the same X tiles while they stream through shared memory for the MMAs.
//
// Design (one CTA per 128 x 256 output tile; grid x = output tile, y = token tile, so the 8
// CTAs of a token tile run side by side and share its X tiles through L2):
//  * warp 0 streams X [128 tokens x 64 features] and Wp [256 outputs x 64 features] tiles by TMA
//    (128-byte swizzle, no multicast) into a ring of kStages stages with full / empty mbarriers;
//  * warp 1 allocates 256 tensor-memory columns and issues, from one thread, four
//    tcgen05.mma (kind::f16, bf16 operands, M = 128, N = 256, K = 16, fp32 accumulator in
//    tensor memory) per stage, committing each stage's MMAs to its empty barrier;
//  * warps 2-5 (the epilogue warps) take token row r = 32 (warp % 4) + lane of every X tile as it
//    lands and fold its 64 values into the row's (mean, centred sum of squares) with Chan's
//    formula, then, once the last MMA has committed, read their accumulator lane back in
//    16-column pieces (tcgen05.ld 32x32b), apply rstd (acc - mu u) + v and store bf16.
// Every mbarrier wait is bounded; on expiry the status word is raised, the stores are skipped,
// the tensor core and the loads in flight are drained (bounded) and tensor memory is freed.
#include "tc5.cuh"
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kBM = 128, kBN = 256, kBK = 64;
constexpr int kStages = 4;
constexpr int kThreads = 192;                       // producer, MMA, 4 epilogue warps
constexpr uint32_t kTileA = kBM * kBK * 2;          // 16 KB
constexpr uint32_t kTileB = kBN * kBK * 2;          // 32 KB
constexpr uint32_t kTmemCols = 256;
constexpr long long kDrainPolls = 1ll << 24;

struct __align__(1024) OpSmem {
    uint8_t a[kStages][kTileA];
    uint8_t b[kStages][kTileB];
    float u[kBN], v[kBN];
    uint64_t full[kStages];
    uint64_t empty[kStages];   // the MMA commit + one arrival per epilogue warp
    uint64_t acc_full;         // every MMA of the tile has completed
    uint32_t tmem_base;
    int fail;
};

// ---- weight packing: one CTA of 256 threads per output n -----------------------------------
__global__ void __launch_bounds__(256) oproj_prepare_kernel(const __nv_bfloat16* __restrict__ Wo,
                                                            const float* __restrict__ ln_w,
                                                            const float* __restrict__ ln_b, int C,
                                                            __nv_bfloat16* __restrict__ Wp, float* __restrict__ u,
                                                            float* __restrict__ v) {
    const long long n = blockIdx.x;
    float su = 0.f, sv = 0.f;
    for (int k = threadIdx.x; k < C; k += blockDim.x) {
        const float wo = __bfloat162float(Wo[n * C + k]);
        const __nv_bfloat16 wp = __float2bfloat16_rn(ln_w[k] * wo);
        Wp[n * C + k] = wp;
        su += __bfloat162float(wp);
        sv = fmaf(ln_b[k], wo, sv);
    }
    __shared__ float red[2][8];
    su = warp_sum(su);
    sv = warp_sum(sv);
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = su;
        red[1][threadIdx.x >> 5] = sv;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        float a = 0.f, b = 0.f;
        for (int i = 0; i < 8; ++i) {
            a += red[0][i];
            b += red[1][i];
        }
        u[n] = a;
        v[n] = b;
    }
}

// ---- the fused GEMM ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
post_norm_oproj_kernel(const OprojArgs a, const __grid_constant__ OprojMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    OpSmem& s = *reinterpret_cast<OpSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * kBN;
    const long long m0 = static_cast<long long>(blockIdx.y) * kBM;
    const int KT = a.C / kBK;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1 + 4);
        }
        mbar_init(&s.acc_full, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&maps.x);
        tma_prefetch_desc(&maps.w);
        s.fail = 0;
    }
    if (warp == 1) tc5::alloc(&s.tmem_base, kTmemCols);
    for (int i = tid; i < kBN; i += kThreads) {
        s.u[i] = a.u[n0 + i];
        s.v[i] = a.v[n0 + i];
    }
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem_base;
    volatile int* const vfail = &s.fail;

    if (warp == 0) {
        // ---- producer: X and Wp tiles of k-chunk kc into stage kc % kStages ----------------------
        if (lane == 0) {
            int kc = 0;
            for (; kc < KT; ++kc) {
                const int st = kc % kStages;
                if (kc >= kStages &&
                    !mbar_wait_bounded_sleep(&s.empty[st], static_cast<uint32_t>((kc / kStages - 1) & 1), a.wait_limit,
                                             64, a.status)) {
                    *vfail = 1;
                    break;
                }
                if (*vfail) break;
                mbar_arrive_expect_tx(&s.full[st], kTileA + kTileB);
                tma_load_2d(&s.a[st][0], &maps.x, kc * kBK, static_cast<int>(m0), &s.full[st]);
                tma_load_2d(&s.b[st][0], &maps.w, kc * kBK, n0, &s.full[st]);
            }
            if (*vfail)  // wait (bounded) until the loads issued and perhaps not consumed have landed
                for (int k = kc > kStages ? kc - kStages : 0; k < kc; ++k)
                    mbar_wait_bounded(&s.full[k % kStages], static_cast<uint32_t>((k / kStages) & 1), kDrainPolls,
                                      nullptr);
        }
    } else if (warp == 1) {
        // ---- MMA issue: D[128 x 256] += X[128 x 64] Wp[256 x 64]^T per stage, 4 steps of K = 16 ----
        if (lane == 0) {
            const uint32_t idesc = tc5::idesc_bf16(kBM, kBN, 0, 0);
            for (int kc = 0; kc < KT; ++kc) {
                const int st = kc % kStages;
                if (!mbar_wait_bounded(&s.full[st], static_cast<uint32_t>((kc / kStages) & 1), a.wait_limit,
                                       a.status)) {
                    *vfail = 1;
                    break;
                }
                tc5::fence_after();
                const uint64_t ad = tc5::sdesc(smem_u32(&s.a[st][0]), 16, 1024);
                const uint64_t bd = tc5::sdesc(smem_u32(&s.b[st][0]), 16, 1024);
#pragma unroll
                for (int k = 0; k < kBK / 16; ++k)
                    tc5::mma_ss(tm, tc5::sdesc_add(ad, 32 * k), tc5::sdesc_add(bd, 32 * k), idesc,
                                (kc | k) != 0 ? 1u : 0u);
                tc5::commit(&s.empty[st]);
            }
            tc5::commit(&s.acc_full);  // once every MMA issued above has completed
        }
        __syncwarp();
    } else {
        // ---- epilogue warps: row statistics while the tiles stream, then the output tile -------
        const int q = warp & 3;            // tensor-memory lane quarter of this warp
        const int row = 32 * q + lane;     // tile row: token m0 + row, accumulator lane row
        float mean = 0.f, m2 = 0.f;
        int kc = 0;
        for (; kc < KT; ++kc) {
            const int st = kc % kStages;
            if (!mbar_wait_bounded(&s.full[st], static_cast<uint32_t>((kc / kStages) & 1), a.wait_limit, a.status)) {
                *vfail = 1;
                break;
            }
            // this row's 64 features of the chunk (8 swizzled 16-byte pieces), centred on their mean
            const uint8_t* rp = &s.a[st][0] + row * 128;
            float x[64];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 pv = *reinterpret_cast<const uint4*>(rp + ((c ^ (row & 7)) << 4));
                const uint32_t wv[4] = {pv.x, pv.y, pv.z, pv.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const float2 f = unpack_bf16x2(wv[j]);
                    x[8 * c + 2 * j] = f.x;
                    x[8 * c + 2 * j + 1] = f.y;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.empty[st]);  // this warp is done with the stage
            float sum = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) sum += x[i];
            const float cm = sum * (1.0f / kBK);
            float cs = 0.f;
#pragma unroll
            for (int i = 0; i < 64; ++i) cs = fmaf(x[i] - cm, x[i] - cm, cs);
            // Chan's merge of (64 kc values, mean, m2) with (64 values, cm, cs)
            const float delta = cm - mean, inv = 1.0f / static_cast<float>(kc + 1);
            mean = fmaf(delta, inv, mean);
            m2 += cs + delta * delta * (static_cast<float>(kBK * kc) * inv);
        }
        bool ok = kc == KT && mbar_wait_bounded(&s.acc_full, 0, a.wait_limit, a.status);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) *vfail = 1;
        tc5::fence_after();
        if (ok) {
            const float rstd = rsqrtf(m2 * (1.0f / static_cast<float>(a.C)) + a.eps);
            const float nmr = -mean * rstd;
            const long long grow = m0 + row;
            __nv_bfloat16* const yrow = static_cast<__nv_bfloat16*>(a.Y) + grow * a.N + n0;
#pragma unroll 1
            for (int c16 = 0; c16 < kBN / 16; ++c16) {
                float acc[16];
                tc5::ld16(tc5::taddr(tm, 32 * q, 16 * c16), acc);
                tc5::wait_ld();
                uint32_t pk[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int n = 16 * c16 + 2 * j;
                    // rstd (acc - mu u) + v
                    const float y0 = fmaf(rstd, acc[2 * j], fmaf(nmr, s.u[n], s.v[n]));
                    const float y1 = fmaf(rstd, acc[2 * j + 1], fmaf(nmr, s.u[n + 1], s.v[n + 1]));
                    pk[j] = pack_bf16x2(y0, y1);
                }
                if (grow < a.T) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + 16 * c16);
                    dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                    dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
                }
            }
        }
    }

    // ---- teardown: every MMA has completed before tensor memory is freed ------------------------
    if (warp == 1 && lane == 0 && *vfail) mbar_wait_bounded(&s.acc_full, 0, kDrainPolls, nullptr);
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    if (warp == 1) tc5::dealloc(tm, kTmemCols);
}

}  // namespace

cudaError_t launch_oproj_prepare(const void* Wo, const float* ln_w, const float* ln_b, int C, int N, void* Wp,
                                 float* u, float* v, cudaStream_t st) {
    oproj_prepare_kernel<<<static_cast<unsigned>(N), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(Wo), ln_w, ln_b, C,
                                                                  static_cast<__nv_bfloat16*>(Wp), u, v);
    return cudaGetLastError();
}

cudaError_t launch_post_norm_oproj(const OprojArgs& a, const OprojMaps& maps, cudaStream_t st) {
    const size_t smem = sizeof(OpSmem) + 1024;  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(post_norm_oproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const dim3 grid(static_cast<unsigned>(a.N / kBN), static_cast<unsigned>((a.T + kBM - 1) / kBM));
    post_norm_oproj_kernel<<<grid, kThreads, smem, st>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace ttt
