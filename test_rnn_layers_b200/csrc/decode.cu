// decode.cu -- TTT-Linear decode: one token per chain through the TTTCache state.
//
// ("代码连连看——TTT", TTTLinear.ttt: decoding takes the params from the cache and the primal
// branch of compute_mini_batch; "测试时学习（TTT）原理解析", TTTCache: last states + grads.)
// With p = seqlen_offset % K and t = token_eta[p]:
//   z = xk W + b, g = ln_fused_l2_bwd(z, xv - xk), W_grad += lr xk^T g, b_grad += lr g,
//   out = xq + LN(xq (W - t W_grad) + b - t b_grad), and at p = K-1 the state commits.
//
// The step is a few matrix-vector products per chain: it is bound by the state traffic
// (read W and W_grad, write W_grad, and W on a commit), so it runs on the FFMA pipes with
// 16-byte coalesced loads.  xq W_bar is formed without materialising W_bar:
//   xq W_bar = xq W - t (xq W_grad_old + lr (xq . xk) g).
#include "ttt_common.cuh"
#include "ttt_internal.h"

namespace ttt {
namespace {

constexpr int kThreads = 256;          // 16 column groups of 4 x 16 row groups of 4
constexpr int kRowGroups = kThreads / 16;

template <typename T>
__global__ void __launch_bounds__(kThreads) decode_kernel(DecodeArgs a) {
    __shared__ float sx[3][TTT_D];                      // xq, xk, xv
    __shared__ float4 part[3][kRowGroups][TTT_D / 4];   // partial xk W, xq W, xq W_grad
    __shared__ float sz[TTT_D], sqw[TTT_D], sqg[TTT_D], sg[TTT_D];
    __shared__ float sqk;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const long long chain = blockIdx.x;
    const int h = static_cast<int>(chain % a.H);
    const int cg = tid & 15;        // columns 4cg .. 4cg+3
    const int rg = tid >> 4;        // rows rg, rg+16, rg+32, rg+48

    float* W = a.W + chain * TTT_D * TTT_D;
    float* Wg = a.W_grad + chain * TTT_D * TTT_D;
    float4 w[4], G[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        int row = rg + 16 * k;
        w[k] = *reinterpret_cast<const float4*>(W + row * TTT_D + 4 * cg);
        G[k] = *reinterpret_cast<const float4*>(Wg + row * TTT_D + 4 * cg);
    }
    if (tid < 3 * TTT_D) {
        int which = tid / TTT_D, c = tid % TTT_D;
        const T* src = static_cast<const T*>(which == 0 ? a.xq : which == 1 ? a.xk : a.xv);
        sx[which][c] = to_f32(src[chain * TTT_D + c]);
    }
    __syncthreads();

    float4 pk = make_float4(0, 0, 0, 0), pq = pk, pg = pk;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        int row = rg + 16 * k;
        float xk = sx[1][row], xq = sx[0][row];
        pk.x = fmaf(xk, w[k].x, pk.x); pk.y = fmaf(xk, w[k].y, pk.y);
        pk.z = fmaf(xk, w[k].z, pk.z); pk.w = fmaf(xk, w[k].w, pk.w);
        pq.x = fmaf(xq, w[k].x, pq.x); pq.y = fmaf(xq, w[k].y, pq.y);
        pq.z = fmaf(xq, w[k].z, pq.z); pq.w = fmaf(xq, w[k].w, pq.w);
        pg.x = fmaf(xq, G[k].x, pg.x); pg.y = fmaf(xq, G[k].y, pg.y);
        pg.z = fmaf(xq, G[k].z, pg.z); pg.w = fmaf(xq, G[k].w, pg.w);
    }
    part[0][rg][cg] = pk;
    part[1][rg][cg] = pq;
    part[2][rg][cg] = pg;
    __syncthreads();

    const float* bst = a.b + chain * TTT_D;
    const float* bg = a.b_grad + chain * TTT_D;
    const float lr = a.lr[chain];
    const float t = a.token_eta ? a.token_eta[a.p] : 1.0f / (a.p + 1);
    if (tid < 3 * TTT_D) {
        int which = tid / TTT_D, c = tid % TTT_D;
        const float* pp = reinterpret_cast<const float*>(&part[which][0][0]);
        float acc = 0.f;
#pragma unroll
        for (int r = 0; r < kRowGroups; ++r) acc += pp[r * TTT_D + c];
        if (which == 0) sz[c] = acc + bst[c];
        else if (which == 1) sqw[c] = acc;
        else sqg[c] = acc;
    }
    if (warp == 7) {
        float v = sx[0][lane] * sx[1][lane] + sx[0][lane + 32] * sx[1][lane + 32];
        v = warp_sum(v);
        if (lane == 0) sqk = v;
    }
    __syncthreads();

    const float* lnw = a.ln_w + h * TTT_D;
    const float* lnb = a.ln_b + h * TTT_D;
    if (warp == 0) {
        // g = ln_fused_l2_bwd(z, xv - xk)
        float z0 = sz[lane], z1 = sz[lane + 32];
        float mu = warp_sum(z0 + z1) * (1.0f / TTT_D);
        float c0 = z0 - mu, c1 = z1 - mu;
        float rstd = 1.0f / sqrtf(warp_sum(c0 * c0 + c1 * c1) * (1.0f / TTT_D) + a.eps);
        float xh0 = c0 * rstd, xh1 = c1 * rstd;
        float w0 = lnw[lane], w1 = lnw[lane + 32];
        float q0 = w0 * (w0 * xh0 + lnb[lane] - (sx[2][lane] - sx[1][lane]));
        float q1 = w1 * (w1 * xh1 + lnb[lane + 32] - (sx[2][lane + 32] - sx[1][lane + 32]));
        float sq = warp_sum(q0 + q1), sqx = warp_sum(q0 * xh0 + q1 * xh1);
        float g0 = (TTT_D * q0 - sq - xh0 * sqx) * rstd * (1.0f / TTT_D);
        float g1 = (TTT_D * q1 - sq - xh1 * sqx) * rstd * (1.0f / TTT_D);
        sg[lane] = g0;
        sg[lane + 32] = g1;

        // bias grads and the bar state
        float gb0 = bg[lane] + lr * g0, gb1 = bg[lane + 32] + lr * g1;
        float bb0 = bst[lane] - t * gb0, bb1 = bst[lane + 32] - t * gb1;
        // xq W_bar + b_bar
        float u0 = sqw[lane] - t * (sqg[lane] + lr * sqk * g0) + bb0;
        float u1 = sqw[lane + 32] - t * (sqg[lane + 32] + lr * sqk * g1) + bb1;
        float m2 = warp_sum(u0 + u1) * (1.0f / TTT_D);
        float d0 = u0 - m2, d1 = u1 - m2;
        float r2 = 1.0f / sqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.0f / TTT_D) + a.eps);
        T* out = static_cast<T*>(a.out) + chain * TTT_D;
        out[lane] = from_f32<T>(sx[0][lane] + w0 * d0 * r2 + lnb[lane]);
        out[lane + 32] = from_f32<T>(sx[0][lane + 32] + w1 * d1 * r2 + lnb[lane + 32]);

        const bool commit = (a.p == a.K - 1);
        float* bsw = a.b + chain * TTT_D;
        float* bgw = a.b_grad + chain * TTT_D;
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
    const bool commit = (a.p == a.K - 1);
    float4 gv = *reinterpret_cast<const float4*>(&sg[4 * cg]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        int row = rg + 16 * k;
        float s = lr * sx[1][row];
        float4 n;
        n.x = fmaf(s, gv.x, G[k].x); n.y = fmaf(s, gv.y, G[k].y);
        n.z = fmaf(s, gv.z, G[k].z); n.w = fmaf(s, gv.w, G[k].w);
        if (commit) {
            float4 nw;
            nw.x = w[k].x - t * n.x; nw.y = w[k].y - t * n.y;
            nw.z = w[k].z - t * n.z; nw.w = w[k].w - t * n.w;
            *reinterpret_cast<float4*>(W + row * TTT_D + 4 * cg) = nw;
            *reinterpret_cast<float4*>(Wg + row * TTT_D + 4 * cg) = make_float4(0, 0, 0, 0);
        } else {
            *reinterpret_cast<float4*>(Wg + row * TTT_D + 4 * cg) = n;
        }
    }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, int dtype, cudaStream_t st) {
    dim3 grid(static_cast<unsigned>(a.B * a.H));
    if (dtype == 0)
        decode_kernel<float><<<grid, kThreads, 0, st>>>(a);
    else
        decode_kernel<__nv_bfloat16><<<grid, kThreads, 0, st>>>(a);
    return cudaGetLastError();
}

}  // namespace ttt
