// decode.cu -- TTT-Linear decode: one token per chain through the TTTCache state.
//
// ("代码连连看——TTT", TTTLinear.ttt: decoding takes the params from the cache and the primal
// branch of compute_mini_batch; "测试时学习（TTT）原理解析", TTTCache: last states + grads.)
// With p = seqlen_offset % K and t = token_eta[p]:
//   z = xk W + b, g = ln_fused_l2_bwd(z, xv - xk), W_grad += lr xk^T g, b_grad += lr g,
//   out = xq + LN(xq (W - t W_grad) + b - t b_grad), and at p = K-1 the state commits.
//
// The step is a few matrix-vector products per chain, bound by the state traffic (read W and
// W_grad, write W_grad, and W on a commit).  xq W_bar is formed without materialising W_bar:
//   xq W_bar = xq W - t (xq W_grad_old + lr (xq . xk) g).
// Persistent CTAs walk the chains with a stride; each CTA streams the next chain's W, W_grad,
// b, b_grad and tokens into one of two shared-memory buffers with bulk async copies (an
// mbarrier per buffer, bounded waits) while it computes the current chain from the other, so
// HBM stays busy through the serial LayerNorm part.  The new W_grad (and W) leave by coalesced
// 16-byte stores straight from registers.
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;           // 16 column groups of 4 x 16 row groups of 4
constexpr int kRowGroups = kThreads / 16;
constexpr int kCtasPerSm = 3;  // 3 x ~71 KB of shared memory, 80 registers
constexpr int kBufs = 2;

template <typename T>
struct __align__(16) DecSmem {
    float W[kBufs][TTT_D * TTT_D];
    float G[kBufs][TTT_D * TTT_D];
    float b[kBufs][TTT_D];
    float gb[kBufs][TTT_D];
    T x[kBufs][3][TTT_D];                 // xq, xk, xv
    float lr[kBufs][4];
    float4 part[3][kRowGroups / 2][TTT_D / 4];  // partial xk W, xq W, xq W_grad of each warp (two row groups)
    float sz[TTT_D], sqw[TTT_D], sqg[TTT_D], sg[TTT_D];
    float sqk;
    uint64_t full[kBufs];
    int fail;
};

template <typename T>
__device__ __forceinline__ void issue_chain(DecSmem<T>& s, const DecodeArgs& a, long long c, int bi) {
    const uint32_t bytes = 2u * TTT_D * TTT_D * 4 + 2u * TTT_D * 4 + 3u * TTT_D * sizeof(T);
    mbar_arrive_expect_tx(&s.full[bi], bytes);
    bulk_load(s.W[bi], a.W + c * TTT_D * TTT_D, TTT_D * TTT_D * 4, &s.full[bi]);
    bulk_load(s.G[bi], a.W_grad + c * TTT_D * TTT_D, TTT_D * TTT_D * 4, &s.full[bi]);
    bulk_load(s.b[bi], a.b + c * TTT_D, TTT_D * 4, &s.full[bi]);
    bulk_load(s.gb[bi], a.b_grad + c * TTT_D, TTT_D * 4, &s.full[bi]);
    bulk_load(s.x[bi][0], static_cast<const T*>(a.xq) + c * TTT_D, TTT_D * sizeof(T), &s.full[bi]);
    bulk_load(s.x[bi][1], static_cast<const T*>(a.xk) + c * TTT_D, TTT_D * sizeof(T), &s.full[bi]);
    bulk_load(s.x[bi][2], static_cast<const T*>(a.xv) + c * TTT_D, TTT_D * sizeof(T), &s.full[bi]);
    cp_async_4(&s.lr[bi][0], a.lr + c);
    cp_async_mbar_arrive_noinc(&s.full[bi]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_kernel(DecodeArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    DecSmem<T>& s = *reinterpret_cast<DecSmem<T>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid & 15;        // columns 4cg .. 4cg+3
    const int rg = tid >> 4;        // rows rg, rg+16, rg+32, rg+48
    const long long chains = static_cast<long long>(a.B) * a.H;
    const long long stride = gridDim.x;
    const bool commit = (a.p == a.K - 1);

    if (tid == 0) {
        for (int i = 0; i < kBufs; ++i) mbar_init(&s.full[i], 2);  // expect-tx arrival + lr cp.async
        fence_mbarrier_init();
        s.fail = 0;
    }
    __syncthreads();
    int issued = 0;  // loads issued by thread 0 (the i-th goes to buffer i % 2, phase (i / 2) & 1)
    if (tid == 0)
        for (int i = 0; i < kBufs; ++i)
            if (blockIdx.x + i * stride < chains) {
                issue_chain(s, a, blockIdx.x + i * stride, i);
                ++issued;
            }

    int bi = 0, it = 0;
    uint32_t par = 0;
    for (long long c = blockIdx.x; c < chains; c += stride, ++it, bi ^= 1, par ^= (bi == 0)) {
        const int h = static_cast<int>(c % a.H);
        if (!mbar_wait_bounded(&s.full[bi], par, a.wait_limit, a.status)) s.fail = 1;

        // state of this chain into registers; partial matrix-vector products
        float4 w[4], G[4];
        float4 pk = make_float4(0, 0, 0, 0), pq = pk, pg = pk;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int row = rg + 16 * k;
            w[k] = *reinterpret_cast<const float4*>(&s.W[bi][row * TTT_D + 4 * cg]);
            G[k] = *reinterpret_cast<const float4*>(&s.G[bi][row * TTT_D + 4 * cg]);
            const float xk = to_f32(s.x[bi][1][row]), xq = to_f32(s.x[bi][0][row]);
            pk.x = fmaf(xk, w[k].x, pk.x); pk.y = fmaf(xk, w[k].y, pk.y);
            pk.z = fmaf(xk, w[k].z, pk.z); pk.w = fmaf(xk, w[k].w, pk.w);
            pq.x = fmaf(xq, w[k].x, pq.x); pq.y = fmaf(xq, w[k].y, pq.y);
            pq.z = fmaf(xq, w[k].z, pq.z); pq.w = fmaf(xq, w[k].w, pq.w);
            pg.x = fmaf(xq, G[k].x, pg.x); pg.y = fmaf(xq, G[k].y, pg.y);
            pg.z = fmaf(xq, G[k].z, pg.z); pg.w = fmaf(xq, G[k].w, pg.w);
        }
        // the warp's two row groups (lanes l and l + 16 share columns) summed before the exchange
#pragma unroll
        for (int o = 0; o < 3; ++o) {
            float4& v = o == 0 ? pk : o == 1 ? pq : pg;
            v.x += __shfl_xor_sync(0xffffffffu, v.x, 16);
            v.y += __shfl_xor_sync(0xffffffffu, v.y, 16);
            v.z += __shfl_xor_sync(0xffffffffu, v.z, 16);
            v.w += __shfl_xor_sync(0xffffffffu, v.w, 16);
        }
        if (lane < 16) {
            s.part[0][warp][cg] = pk;
            s.part[1][warp][cg] = pq;
            s.part[2][warp][cg] = pg;
        }
        __syncthreads();
        if (s.fail) break;

        const float lr = s.lr[bi][0];
        const float t = a.token_eta ? a.token_eta[a.p] : 1.0f / (a.p + 1);
        if (tid < 3 * TTT_D) {
            const int which = tid / TTT_D, col = tid % TTT_D;
            const float* pp = reinterpret_cast<const float*>(&s.part[which][0][0]);
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kRowGroups / 2; ++r) acc += pp[r * TTT_D + col];
            if (which == 0) s.sz[col] = acc + s.b[bi][col];
            else if (which == 1) s.sqw[col] = acc;
            else s.sqg[col] = acc;
        }
        if (warp == 7) {
            const float v = to_f32(s.x[bi][0][lane]) * to_f32(s.x[bi][1][lane]) +
                            to_f32(s.x[bi][0][lane + 32]) * to_f32(s.x[bi][1][lane + 32]);
            const float r = warp_sum(v);
            if (lane == 0) s.sqk = r;
        }
        __syncthreads();

        const float* lnw = a.ln_w + h * TTT_D;
        const float* lnb = a.ln_b + h * TTT_D;
        if (warp == 0) {
            // g = ln_fused_l2_bwd(z, xv - xk)
            const float z0 = s.sz[lane], z1 = s.sz[lane + 32];
            float mu, rstd;
            warp_row_stats(z0, z1, a.eps, mu, rstd);
            const float xh0 = (z0 - mu) * rstd, xh1 = (z1 - mu) * rstd;
            const float w0 = lnw[lane], w1 = lnw[lane + 32];
            const float xk0 = to_f32(s.x[bi][1][lane]), xk1 = to_f32(s.x[bi][1][lane + 32]);
            const float xq0 = to_f32(s.x[bi][0][lane]), xq1 = to_f32(s.x[bi][0][lane + 32]);
            const float q0 = w0 * (w0 * xh0 + lnb[lane] - (to_f32(s.x[bi][2][lane]) - xk0));
            const float q1 = w1 * (w1 * xh1 + lnb[lane + 32] - (to_f32(s.x[bi][2][lane + 32]) - xk1));
            float sq = q0 + q1, sqx = fmaf(q0, xh0, q1 * xh1);
            warp_sum2(sq, sqx);
            const float g0 = (TTT_D * q0 - sq - xh0 * sqx) * rstd * (1.0f / TTT_D);
            const float g1 = (TTT_D * q1 - sq - xh1 * sqx) * rstd * (1.0f / TTT_D);
            s.sg[lane] = g0;
            s.sg[lane + 32] = g1;

            // bias grads and the bar state
            const float gb0 = s.gb[bi][lane] + lr * g0, gb1 = s.gb[bi][lane + 32] + lr * g1;
            const float bb0 = s.b[bi][lane] - t * gb0, bb1 = s.b[bi][lane + 32] - t * gb1;
            // xq W_bar + b_bar
            const float u0 = s.sqw[lane] - t * (s.sqg[lane] + lr * s.sqk * g0) + bb0;
            const float u1 = s.sqw[lane + 32] - t * (s.sqg[lane + 32] + lr * s.sqk * g1) + bb1;
            float m2, r2;
            warp_row_stats(u0, u1, a.eps, m2, r2);
            const float d0 = u0 - m2, d1 = u1 - m2;
            T* out = static_cast<T*>(a.out) + c * TTT_D;
            out[lane] = from_f32<T>(xq0 + w0 * d0 * r2 + lnb[lane]);
            out[lane + 32] = from_f32<T>(xq1 + w1 * d1 * r2 + lnb[lane + 32]);

            float* bsw = a.b + c * TTT_D;
            float* bgw = a.b_grad + c * TTT_D;
            if (commit) {
                bsw[lane] = bb0;
                bsw[lane + 32] = bb1;
                bgw[lane] = 0.f;
                bgw[lane + 32] = 0.f;
            } else {
                bgw[lane] = gb0;
                bgw[lane + 32] = gb1;
            }
        }
        __syncthreads();

        // W_grad += lr xk^T g ; on commit W -= t W_grad and W_grad = 0
        float* Wc = a.W + c * TTT_D * TTT_D;
        float* Gc = a.W_grad + c * TTT_D * TTT_D;
        const float4 gv = *reinterpret_cast<const float4*>(&s.sg[4 * cg]);
        float xkr[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) xkr[k] = lr * to_f32(s.x[bi][1][rg + 16 * k]);
        __syncthreads();  // buffer bi fully read: refill it with the chain after next
        if (tid == 0 && c + kBufs * stride < chains) {
            issue_chain(s, a, c + kBufs * stride, bi);
            ++issued;
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int row = rg + 16 * k;
            float4 n;
            n.x = fmaf(xkr[k], gv.x, G[k].x); n.y = fmaf(xkr[k], gv.y, G[k].y);
            n.z = fmaf(xkr[k], gv.z, G[k].z); n.w = fmaf(xkr[k], gv.w, G[k].w);
            if (commit) {
                float4 nw;
                nw.x = w[k].x - t * n.x; nw.y = w[k].y - t * n.y;
                nw.z = w[k].z - t * n.z; nw.w = w[k].w - t * n.w;
                *reinterpret_cast<float4*>(Wc + row * TTT_D + 4 * cg) = nw;
                *reinterpret_cast<float4*>(Gc + row * TTT_D + 4 * cg) = make_float4(0, 0, 0, 0);
            } else {
                *reinterpret_cast<float4*>(Gc + row * TTT_D + 4 * cg) = n;
            }
        }
    }
    // after a failed wait, leave only once this CTA's issued copies have landed (bounded)
    if (s.fail && tid == 0)
        for (int j = it; j < issued; ++j)
            mbar_wait_bounded(&s.full[j % kBufs], static_cast<uint32_t>((j / kBufs) & 1), 1ll << 24, nullptr);
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int dtype, cudaStream_t st) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long chains = static_cast<long long>(a.B) * a.H;
    const unsigned grid = static_cast<unsigned>(chains < kCtasPerSm * static_cast<long long>(sms)
                                                    ? chains : kCtasPerSm * static_cast<long long>(sms));
    cudaError_t e;
    if (dtype == 0) {
        const size_t smem = sizeof(DecSmem<float>);
        e = cudaFuncSetAttribute(decode_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        decode_kernel<float><<<grid, kThreads, smem, st>>>(a);
    } else {
        const size_t smem = sizeof(DecSmem<__nv_bfloat16>);
        e = cudaFuncSetAttribute(decode_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        decode_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace ttt
