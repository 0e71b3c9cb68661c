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
// the rounded Wp, so the correction matches what the MMAs multiply).  The token statistics come
// from a one-warp-per-token pass over X just before (oproj_stats_kernel: Chan's merge of the
// lanes' two-pass moments); taking them from the GEMM's own X tiles in shared memory instead cost
// shared-memory bandwidth that the tensor core's operand reads need (0.547 against 0.44 ms).
//
// Design: a persistent kernel, one CTA per SM, walking 128 x 256 output tiles (output tile
// fastest, so the CTAs at work at any moment share their X tiles through L2), four roles:
//  * warp 0 streams X [128 tokens x 64 features] and Wp [256 outputs x 64 features] tiles by TMA
//    (128-byte swizzle, no multicast) into a ring of kStages stages with full / empty mbarriers,
//    across tile boundaries;
//  * warp 1 allocates all 512 tensor-memory columns -- two fp32 accumulators of 128 x 256 -- and
//    issues, from one thread, four tcgen05.mma (kind::f16, bf16 operands, M = 128, N = 256,
//    K = 16) per stage into the tile's accumulator, committing each stage to its empty barrier
//    and each finished tile to its accumulator's full barrier;
//  * warps 2-5 (epilogue) read their accumulator lane back (tcgen05.ld 32x32b, 64 columns per
//    wait), apply rstd (acc - mean u) + v with the row's statistics and store bf16, then free the
//    accumulator -- while the MMAs of the next tile already run into the other one.
// Every mbarrier wait is bounded; on expiry the status word is raised, every role stops, the
// tensor core and the loads in flight are drained (bounded) and tensor memory is freed.
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
constexpr uint32_t kTmemCols = 512;                 // two 256-column accumulators
constexpr long long kDrainPolls = 1ll << 24;

struct __align__(1024) OpSmem {
    uint8_t a[kStages][kTileA];
    uint8_t b[kStages][kTileB];
    float uv[4][2][kBN];       // the tile's u and v, one copy per epilogue warp
    uint64_t full[kStages];
    uint64_t empty[kStages];   // the MMA commit
    uint64_t acc_full[2];      // the tile's MMAs have completed (MMA commit)
    uint64_t acc_empty[2];     // the epilogue has read the accumulator (4 epilogue warps)
    uint64_t drain;            // teardown: every MMA issued has completed
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


// ---- token statistics: one warp per token, (mean, rstd) over its C features -----------------
// Each lane takes the 16-byte pieces lane, lane + 32, ... of the row, forms their mean and centred
// sum of squares, and the warp merges the lanes' moments pairwise by Chan's formula.
__global__ void __launch_bounds__(256) oproj_stats_kernel(const __nv_bfloat16* __restrict__ X, long long T, int C,
                                                          float eps, float2* __restrict__ stats) {
    const int lane = threadIdx.x & 31;
    const long long w0 = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const long long nw = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const int pieces = C / 8;
    for (long long t = w0; t < T; t += nw) {
        const uint4* row = reinterpret_cast<const uint4*>(X + t * C);
        // the first 8 pieces of this lane (all of them for C <= 2048), held in registers
        uint4 pv[8];
        int np = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const bool in = lane + 32 * i < pieces;
            pv[i] = in ? __ldg(row + lane + 32 * i) : make_uint4(0, 0, 0, 0);
            np += in ? 1 : 0;
        }
        float sum = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t wv[4] = {pv[i].x, pv[i].y, pv[i].z, pv[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = unpack_bf16x2(wv[j]);
                sum += f.x + f.y;
            }
        }
        int n = 8 * np;
        float mean = n ? sum / n : 0.f, m2 = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            if (i >= np) break;
            const uint32_t wv[4] = {pv[i].x, pv[i].y, pv[i].z, pv[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const float2 f = unpack_bf16x2(wv[j]);
                m2 = fmaf(f.x - mean, f.x - mean, m2);
                m2 = fmaf(f.y - mean, f.y - mean, m2);
            }
        }
        for (int p = lane + 32 * 8; p < pieces; p += 32) {  // rows wider than 2048 features
            const uint4 q = __ldg(row + p);
            const uint32_t wv[4] = {q.x, q.y, q.z, q.w};
            for (int j = 0; j < 4; ++j) {
                const float2 f = unpack_bf16x2(wv[j]);
                const float d0 = f.x - mean;
                mean += d0 / static_cast<float>(n + 1);
                m2 = fmaf(d0, f.x - mean, m2);
                ++n;
                const float d1 = f.y - mean;
                mean += d1 / static_cast<float>(n + 1);
                m2 = fmaf(d1, f.y - mean, m2);
                ++n;
            }
        }
        // Chan's merge across the lanes: (n, mean, m2) pairs, xor butterfly
        float fn = static_cast<float>(n);
        for (int o = 16; o > 0; o >>= 1) {
            const float on = __shfl_xor_sync(0xffffffffu, fn, o);
            const float om = __shfl_xor_sync(0xffffffffu, mean, o);
            const float oq = __shfl_xor_sync(0xffffffffu, m2, o);
            const float tn = fn + on;
            if (tn > 0.f) {
                const float delta = om - mean;
                mean = fmaf(delta, on / tn, mean);
                m2 += oq + delta * delta * (fn * on / tn);
            }
            fn = tn;
        }
        if (lane == 0) stats[t] = make_float2(mean, rsqrtf(m2 / static_cast<float>(C) + eps));
    }
}

// tcgen05.ld results are defined only after tcgen05.wait::ld; tie the registers to a point after it
__device__ __forceinline__ void after_wait(float (&v)[16]) {
    asm volatile("" : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]),
                 "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]));
}

// ---- the fused GEMM (persistent) ---------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
post_norm_oproj_kernel(const OprojArgs a, const __grid_constant__ OprojMaps maps) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    OpSmem& s = *reinterpret_cast<OpSmem*>(smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int KT = a.C / kBK;
    const int n_tiles = a.N / kBN;
    const long long tiles = ((a.T + kBM - 1) / kBM) * n_tiles;

    if (tid == 0) {
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&s.full[i], 1);
            mbar_init(&s.empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&s.acc_full[i], 1);
            mbar_init(&s.acc_empty[i], 4);
        }
        mbar_init(&s.drain, 1);
        fence_mbarrier_init();
        tma_prefetch_desc(&maps.x);
        tma_prefetch_desc(&maps.w);
        s.fail = 0;
    }
    if (warp == 1) tc5::alloc(&s.tmem_base, kTmemCols);
    tc5::fence_before();
    __syncthreads();
    tc5::fence_after();
    const uint32_t tm = s.tmem_base;
    volatile int* const vfail = &s.fail;
    const long long wl = a.wait_limit;

    if (warp == 0) {
        // ---- producer: the X and Wp tiles of every k-chunk of every tile, through the ring -------
        if (lane == 0) {
            long long g = 0;  // chunks issued
            for (long long tile = blockIdx.x; tile < tiles && !*vfail; tile += gridDim.x) {
                const int m0 = static_cast<int>((tile / n_tiles) * kBM), n0 = static_cast<int>((tile % n_tiles) * kBN);
                for (int kc = 0; kc < KT; ++kc, ++g) {
                    const int st = static_cast<int>(g % kStages);
                    if (g >= kStages &&
                        !mbar_wait_bounded_sleep(&s.empty[st], static_cast<uint32_t>((g / kStages - 1) & 1), wl, 64,
                                                 a.status)) {
                        *vfail = 1;
                        break;
                    }
                    if (*vfail) break;
                    mbar_arrive_expect_tx(&s.full[st], kTileA + kTileB);
                    tma_load_2d(&s.a[st][0], &maps.x, kc * kBK, m0, &s.full[st]);
                    tma_load_2d(&s.b[st][0], &maps.w, kc * kBK, n0, &s.full[st]);
                }
            }
            if (*vfail)  // wait (bounded) until the loads issued and perhaps not consumed have landed
                for (long long k = g > kStages ? g - kStages : 0; k < g; ++k)
                    mbar_wait_bounded(&s.full[k % kStages], static_cast<uint32_t>((k / kStages) & 1), kDrainPolls,
                                      nullptr);
        }
    } else if (warp == 1) {
        // ---- MMA issue into accumulator j % 2 of the j-th tile ---------------------------------------
        if (lane == 0) {
            const uint32_t idesc = tc5::idesc_bf16(kBM, kBN, 0, 0);
            long long g = 0;
            int j = 0;
            for (long long tile = blockIdx.x; tile < tiles && !*vfail; tile += gridDim.x, ++j) {
                const int buf = j & 1;
                if (j >= 2 && !mbar_wait_bounded(&s.acc_empty[buf], static_cast<uint32_t>(((j >> 1) - 1) & 1), wl,
                                                 a.status)) {
                    *vfail = 1;
                    break;
                }
                tc5::fence_after();
                const uint32_t acc = tm + static_cast<uint32_t>(buf) * kBN;
                for (int kc = 0; kc < KT; ++kc, ++g) {
                    const int st = static_cast<int>(g % kStages);
                    if (!mbar_wait_bounded(&s.full[st], static_cast<uint32_t>((g / kStages) & 1), wl, a.status)) {
                        *vfail = 1;
                        break;
                    }
                    tc5::fence_after();
                    const uint64_t ad = tc5::sdesc(smem_u32(&s.a[st][0]), 16, 1024);
                    const uint64_t bd = tc5::sdesc(smem_u32(&s.b[st][0]), 16, 1024);
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        tc5::mma_ss(acc, tc5::sdesc_add(ad, 32 * k), tc5::sdesc_add(bd, 32 * k), idesc,
                                    (kc | k) != 0 ? 1u : 0u);
                    tc5::commit(&s.empty[st]);
                }
                if (*vfail) break;
                tc5::commit(&s.acc_full[buf]);
            }
            tc5::commit(&s.drain);  // once every MMA issued above has completed
            mbar_wait_bounded(&s.drain, 0, kDrainPolls, nullptr);
        }
        __syncwarp();
    } else {
        // ---- epilogue: rstd (acc - mean u) + v of every tile, from tensor memory to bf16 rows -----
        const int q = warp & 3;              // tensor-memory lane quarter of this warp
        const int row = 32 * q + lane;
        int j = 0;
        for (long long tile = blockIdx.x; tile < tiles && !*vfail; tile += gridDim.x, ++j) {
            const int buf = j & 1;
            const uint32_t par = static_cast<uint32_t>((j >> 1) & 1);
            const long long m0 = (tile / n_tiles) * kBM;
            const int n0 = static_cast<int>((tile % n_tiles) * kBN);
            // this warp's copy of the tile's u and v (no barrier across the epilogue warps, so that
            // a warp that gives up on a wait cannot leave the others waiting on it)
            __syncwarp();
            for (int i = lane; i < kBN; i += 32) {
                s.uv[q][0][i] = a.u[n0 + i];
                s.uv[q][1][i] = a.v[n0 + i];
            }
            __syncwarp();
            const float2 st = row < a.T - m0 ? a.stats[m0 + row] : make_float2(0.f, 0.f);
            const bool ok = mbar_wait_bounded(&s.acc_full[buf], par, wl, a.status);
            if (!__all_sync(0xffffffffu, ok)) {
                *vfail = 1;
                break;
            }
            tc5::fence_after();
            const float rstd = st.y, nmr = -st.x * st.y;
            const long long grow = m0 + row;
            __nv_bfloat16* const yrow = static_cast<__nv_bfloat16*>(a.Y) + grow * a.N + n0;
            const float* const uu = s.uv[q][0];
            const float* const vv = s.uv[q][1];
#pragma unroll 1
            for (int c64 = 0; c64 < kBN / 64; ++c64) {
                float acc[4][16];
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    tc5::ld16(tc5::taddr(tm, 32 * q, static_cast<uint32_t>(buf) * kBN + 64 * c64 + 16 * i), acc[i]);
                tc5::wait_ld();
#pragma unroll
                for (int i = 0; i < 4; ++i) after_wait(acc[i]);
                uint32_t pk[32];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) {
                        const int n = 64 * c64 + 16 * i + 2 * jj;
                        const float y0 = fmaf(rstd, acc[i][2 * jj], fmaf(nmr, uu[n], vv[n]));
                        const float y1 = fmaf(rstd, acc[i][2 * jj + 1], fmaf(nmr, uu[n + 1], vv[n + 1]));
                        pk[8 * i + jj] = pack_bf16x2(y0, y1);
                    }
                if (grow < a.T) {
                    uint4* dst = reinterpret_cast<uint4*>(yrow + 64 * c64);
#pragma unroll
                    for (int i = 0; i < 8; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
                }
            }
            tc5::fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&s.acc_empty[buf]);
        }
    }

    // ---- teardown: the MMA thread has seen every MMA complete; free tensor memory -----------------
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
    int dev0 = 0, sms0 = 148;
    if (cudaGetDevice(&dev0) == cudaSuccess) cudaDeviceGetAttribute(&sms0, cudaDevAttrMultiProcessorCount, dev0);
    const long long warps_needed = a.T;
    const long long blocks = (warps_needed + 7) / 8;
    const unsigned sgrid = static_cast<unsigned>(blocks < 16ll * sms0 ? blocks : 16ll * sms0);
    oproj_stats_kernel<<<sgrid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a.X), a.T, a.C, a.eps, a.stats);
    cudaError_t e0 = cudaGetLastError();
    if (e0 != cudaSuccess) return e0;
    const size_t smem = sizeof(OpSmem) + 1024;  // + alignment slack
    cudaError_t e = cudaFuncSetAttribute(post_norm_oproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long tiles = ((a.T + kBM - 1) / kBM) * (a.N / kBN);
    const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
    post_norm_oproj_kernel<<<grid, kThreads, smem, st>>>(a, maps);
    return cudaGetLastError();
}

}  // namespace ttt
