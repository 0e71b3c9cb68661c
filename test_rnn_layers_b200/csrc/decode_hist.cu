// decode_hist.cu -- TTT-Linear decode with a history-format cache.
//
// The decode step ("代码连连看——TTT", TTTLinear.ttt primal branch; "测试时学习（TTT）原理解析",
// TTTCache) needs, at position p = seqlen_offset % K inside the mini-batch, the gradient sums of
// the tokens j <= p so far: W_grad = sum_j lr_j xk_j^T g_j and b_grad = sum_j lr_j g_j.  The
// reference cache keeps W_grad as a dense d x d matrix.  This cache keeps the rows that make it
// up instead, (a_j = lr_j xk_j, g_j) for j < p (at most K - 1 of them), plus the dense b_grad.
// With t = token_eta[p]:
//   z = xk W + b, g = ln_fused_l2_bwd(z, xv - xk),
//   xq W_bar = xq W - t (sum_{j<p} (xq . a_j) g_j + lr (xq . xk) g),
//   b_bar = b - t (b_grad + lr g),  out = xq + LN(xq W_bar + b_bar),
//   row p = (lr xk, g); at p = K-1 the state commits: W -= t sum_{j<=p} a_j^T g_j, b = b_bar.
// The same numbers as the dense cache, with far less state traffic: per step and chain it reads
// W, b, b_grad and p rows of 512 bytes and writes one row and b_grad (the dense cache reads W and
// W_grad and writes W_grad back, 3 x 16 KB).
//
// Persistent CTAs walk the chains; each CTA streams the next chain's W, b, b_grad, rows and
// tokens into one of two shared-memory buffers by bulk async copies (an mbarrier per buffer,
// bounded waits) while it computes the current chain.
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;           // 16 column groups of 4 x 16 row groups of 4
constexpr int kRowGroups = kThreads / 16;
constexpr int kBufs = 2;
constexpr int kRow = 2 * TTT_D;         // floats per history row: a_j then g_j
constexpr int kCtasPerSm = 4;           // 4 x ~55 KB of shared memory, 64 registers: more chains in flight

template <typename T>
struct __align__(16) HistSmem {
    float W[kBufs][TTT_D * TTT_D];
    float hist[kBufs][TTT_KMAX][kRow];
    float b[kBufs][TTT_D];
    float gb[kBufs][TTT_D];
    T x[kBufs][3][TTT_D];                 // xq, xk, xv
    float lr[kBufs][4];
    float4 part[2][kRowGroups / 2][TTT_D / 4];  // partial xk W, xq W of each warp (two row groups)
    float sz[TTT_D], sqw[TTT_D], sg[TTT_D];
    float scr[TTT_D];                     // sum_{j<p} (xq . a_j) g_j
    float c[TTT_KMAX];                    // xq . a_j
    float sqk;
    uint64_t full[kBufs];
    int fail;
};

template <typename T>
__device__ __forceinline__ void issue_chain(HistSmem<T>& s, const DecodeHistArgs& a, long long c, int bi) {
    const uint32_t rows = static_cast<uint32_t>(a.p) * kRow * 4;
    const uint32_t bytes = TTT_D * TTT_D * 4 + 2u * TTT_D * 4 + 3u * TTT_D * sizeof(T) + rows;
    mbar_arrive_expect_tx(&s.full[bi], bytes);
    bulk_load(s.W[bi], a.W + c * TTT_D * TTT_D, TTT_D * TTT_D * 4, &s.full[bi]);
    if (rows) bulk_load(s.hist[bi], a.hist + c * a.K * kRow, rows, &s.full[bi]);
    bulk_load(s.b[bi], a.b + c * TTT_D, TTT_D * 4, &s.full[bi]);
    bulk_load(s.gb[bi], a.b_grad + c * TTT_D, TTT_D * 4, &s.full[bi]);
    bulk_load(s.x[bi][0], static_cast<const T*>(a.xq) + c * TTT_D, TTT_D * sizeof(T), &s.full[bi]);
    bulk_load(s.x[bi][1], static_cast<const T*>(a.xk) + c * TTT_D, TTT_D * sizeof(T), &s.full[bi]);
    bulk_load(s.x[bi][2], static_cast<const T*>(a.xv) + c * TTT_D, TTT_D * sizeof(T), &s.full[bi]);
    cp_async_4(&s.lr[bi][0], a.lr + c);
    cp_async_mbar_arrive_noinc(&s.full[bi]);
}

template <typename T>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_hist_kernel(DecodeHistArgs a) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    HistSmem<T>& s = *reinterpret_cast<HistSmem<T>*>(smem_raw);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cg = tid & 15;        // columns 4cg .. 4cg+3
    const int rg = tid >> 4;        // rows rg, rg+16, rg+32, rg+48
    const long long chains = static_cast<long long>(a.B) * a.H;
    const long long stride = gridDim.x;
    const int p = a.p;
    const bool commit = (p == a.K - 1);

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

    const float t = a.token_eta ? a.token_eta[p] : 1.0f / (p + 1);
    int bi = 0, it = 0;
    uint32_t par = 0;
    for (long long c = blockIdx.x; c < chains; c += stride, ++it, bi ^= 1, par ^= (bi == 0)) {
        const int h = static_cast<int>(c % a.H);
        if (!mbar_wait_bounded(&s.full[bi], par, a.wait_limit, a.status)) s.fail = 1;

        // partial xk W, xq W over this thread's rows; xq . a_j for the rows so far
        float4 w[4];
        float4 pk = make_float4(0, 0, 0, 0), pq = pk;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int row = rg + 16 * k;
            w[k] = *reinterpret_cast<const float4*>(&s.W[bi][row * TTT_D + 4 * cg]);
            const float xk = to_f32(s.x[bi][1][row]), xq = to_f32(s.x[bi][0][row]);
            pk.x = fmaf(xk, w[k].x, pk.x); pk.y = fmaf(xk, w[k].y, pk.y);
            pk.z = fmaf(xk, w[k].z, pk.z); pk.w = fmaf(xk, w[k].w, pk.w);
            pq.x = fmaf(xq, w[k].x, pq.x); pq.y = fmaf(xq, w[k].y, pq.y);
            pq.z = fmaf(xq, w[k].z, pq.z); pq.w = fmaf(xq, w[k].w, pq.w);
        }
        // the warp's two row groups (lanes l and l + 16 share columns) summed before the exchange
        pk.x += __shfl_xor_sync(0xffffffffu, pk.x, 16); pk.y += __shfl_xor_sync(0xffffffffu, pk.y, 16);
        pk.z += __shfl_xor_sync(0xffffffffu, pk.z, 16); pk.w += __shfl_xor_sync(0xffffffffu, pk.w, 16);
        pq.x += __shfl_xor_sync(0xffffffffu, pq.x, 16); pq.y += __shfl_xor_sync(0xffffffffu, pq.y, 16);
        pq.z += __shfl_xor_sync(0xffffffffu, pq.z, 16); pq.w += __shfl_xor_sync(0xffffffffu, pq.w, 16);
        if (lane < 16) {
            s.part[0][warp][cg] = pk;
            s.part[1][warp][cg] = pq;
        }
        {
            const float xq0 = to_f32(s.x[bi][0][lane]), xq1 = to_f32(s.x[bi][0][lane + 32]);
            for (int j = warp; j < p; j += kThreads / 32) {
                const float v = xq0 * s.hist[bi][j][lane] + xq1 * s.hist[bi][j][lane + 32];
                const float r = warp_sum(v);
                if (lane == 0) s.c[j] = r;
            }
        }
        __syncthreads();
        if (s.fail) break;

        const float lr = s.lr[bi][0];
        if (tid < 2 * TTT_D) {
            const int which = tid / TTT_D, col = tid % TTT_D;
            const float* pp = reinterpret_cast<const float*>(&s.part[which][0][0]);
            float acc = 0.f;
#pragma unroll
            for (int r = 0; r < kRowGroups / 2; ++r) acc += pp[r * TTT_D + col];
            if (which == 0) s.sz[col] = acc + s.b[bi][col];
            else s.sqw[col] = acc;
        }
        if (tid >= 2 * TTT_D && tid < 3 * TTT_D) {  // the rows' part of xq W_grad, off warp 0's path
            const int col = tid - 2 * TTT_D;
            float acc = 0.f;
            for (int j = 0; j < p; ++j) acc = fmaf(s.c[j], s.hist[bi][j][TTT_D + col], acc);
            s.scr[col] = acc;
        }
        if (warp == 7) {
            const float v = to_f32(s.x[bi][0][lane]) * to_f32(s.x[bi][1][lane]) +
                            to_f32(s.x[bi][0][lane + 32]) * to_f32(s.x[bi][1][lane + 32]);
            const float r = warp_sum(v);
            if (lane == 0) s.sqk = r;
        }
        __syncthreads();

        T* const outp = static_cast<T*>(a.out) + c * TTT_D;
        float* const rowp = a.hist + (c * a.K + p) * kRow;  // this token's history row
        if (warp == 0) {
            const float* lnw = a.ln_w + h * TTT_D;
            const float* lnb = a.ln_b + h * TTT_D;
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

            // xq W_grad = sum_{j<p} (xq . a_j) g_j + lr (xq . xk) g
            const float cr0 = fmaf(lr * s.sqk, g0, s.scr[lane]), cr1 = fmaf(lr * s.sqk, g1, s.scr[lane + 32]);
            const float gb0 = s.gb[bi][lane] + lr * g0, gb1 = s.gb[bi][lane + 32] + lr * g1;
            const float bb0 = s.b[bi][lane] - t * gb0, bb1 = s.b[bi][lane + 32] - t * gb1;
            const float u0 = s.sqw[lane] - t * cr0 + bb0, u1 = s.sqw[lane + 32] - t * cr1 + bb1;
            float m2, r2;
            warp_row_stats(u0, u1, a.eps, m2, r2);
            const float d0 = u0 - m2, d1 = u1 - m2;
            outp[lane] = from_f32<T>(xq0 + w0 * d0 * r2 + lnb[lane]);
            outp[lane + 32] = from_f32<T>(xq1 + w1 * d1 * r2 + lnb[lane + 32]);

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
                rowp[lane] = lr * xk0;  // row p = (lr xk, g)
                rowp[lane + 32] = lr * xk1;
                rowp[TTT_D + lane] = g0;
                rowp[TTT_D + lane + 32] = g1;
            }
        }
        __syncthreads();

        // on a commit: W -= t sum_{j<=p} a_j^T g_j (row p from this step's lr xk and g)
        if (commit) {
            float4 acc[4] = {make_float4(0, 0, 0, 0), make_float4(0, 0, 0, 0), make_float4(0, 0, 0, 0),
                             make_float4(0, 0, 0, 0)};
            for (int j = 0; j < p; ++j) {
                const float4 gj = *reinterpret_cast<const float4*>(&s.hist[bi][j][TTT_D + 4 * cg]);
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float aj = s.hist[bi][j][rg + 16 * k];
                    acc[k].x = fmaf(aj, gj.x, acc[k].x); acc[k].y = fmaf(aj, gj.y, acc[k].y);
                    acc[k].z = fmaf(aj, gj.z, acc[k].z); acc[k].w = fmaf(aj, gj.w, acc[k].w);
                }
            }
            const float4 gp = *reinterpret_cast<const float4*>(&s.sg[4 * cg]);
            float* Wc = a.W + c * TTT_D * TTT_D;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int row = rg + 16 * k;
                const float ap = lr * to_f32(s.x[bi][1][row]);
                float4 n;
                n.x = w[k].x - t * fmaf(ap, gp.x, acc[k].x); n.y = w[k].y - t * fmaf(ap, gp.y, acc[k].y);
                n.z = w[k].z - t * fmaf(ap, gp.z, acc[k].z); n.w = w[k].w - t * fmaf(ap, gp.w, acc[k].w);
                *reinterpret_cast<float4*>(Wc + row * TTT_D + 4 * cg) = n;
            }
        }
        __syncthreads();  // buffer bi fully read: refill it with the chain after next
        if (tid == 0 && c + kBufs * stride < chains) {
            issue_chain(s, a, c + kBufs * stride, bi);
            ++issued;
        }
    }
    // after a failed wait, leave only once this CTA's issued copies have landed (bounded)
    if (s.fail && tid == 0)
        for (int j = it; j < issued; ++j)
            mbar_wait_bounded(&s.full[j % kBufs], static_cast<uint32_t>((j / kBufs) & 1), 1ll << 24, nullptr);
}

}  // namespace

cudaError_t launch_decode_hist(const DecodeHistArgs& a, int dtype, cudaStream_t st) {
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const long long chains = static_cast<long long>(a.B) * a.H;
    const unsigned grid = static_cast<unsigned>(chains < kCtasPerSm * static_cast<long long>(sms) ? chains : kCtasPerSm * static_cast<long long>(sms));
    cudaError_t e;
    if (dtype == 0) {
        const size_t smem = sizeof(HistSmem<float>);
        e = cudaFuncSetAttribute(decode_hist_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        decode_hist_kernel<float><<<grid, kThreads, smem, st>>>(a);
    } else {
        const size_t smem = sizeof(HistSmem<__nv_bfloat16>);
        e = cudaFuncSetAttribute(decode_hist_kernel<__nv_bfloat16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(smem));
        if (e != cudaSuccess) return e;
        decode_hist_kernel<__nv_bfloat16><<<grid, kThreads, smem, st>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace ttt
