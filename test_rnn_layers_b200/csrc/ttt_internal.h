// ttt_internal.h -- launch arguments and launcher prototypes shared between the C-ABI layer
// (ttt_api.cu) and the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ttt {

// Arguments of one TTT-Linear prefill launch (all pointers device pointers).
struct LinearArgs {
    const void* XQ;
    const void* XK;
    const void* XV;
    const float* lr;
    const float* token_eta;   // [K] or nullptr -> 1/(i+1)
    const float* W0;
    const float* b0;
    long long w0_chain_stride;  // elements between consecutive chains' W0 (0: per head only)
    const float* ln_w;
    const float* ln_b;
    int B, H;
    long long L;
    int K;
    long long n_full, rem;
    float eps;
    // element strides of XQ, XK, XV and out between batch rows, heads and tokens:
    // [B, H, L, d] (head-major): H*L*d, L*d, d;  [B, L, H, d] (token-major): L*H*d, d, H*d
    long long act_b, act_h, act_t;
    int tok_major;            // 1: token-major, the order of the tensor maps' coordinates
    // rotary embedding of XQ and XK at position (token index mod K), tensor-core kernel only:
    // 0 none, 1 pairs (2k, 2k+1), 2 pairs (k, k + d/2); angle of pair k = position * theta^(-2k/d)
    int rope;
    float rope_theta;
    void* out;
    float* W_last;
    float* b_last;
    float* W_grad_tail;
    float* b_grad_tail;
    unsigned int* status;     // device status word
    long long wait_limit;     // polls per bounded wait
    // checkpoints for the backward (or nullptr): the state (W as [k][n], then b) before every
    // ckpt_G-th full mini-batch, then the state after the last full one, ckpt_stride per chain
    float* ckpt;
    int ckpt_G;
    long long ckpt_stride;
};

struct MlpArgs {
    const void* XQ;
    const void* XK;
    const void* XV;
    const float* lr;
    const float* token_eta;
    const float* W1_0;
    const float* b1_0;
    const float* W2_0;
    const float* b2_0;
    long long w0_chain_stride;  // elements between chains' W1_0 / W2_0 (0: per head only)
    const float* ln_w;
    const float* ln_b;
    int B, H;
    long long L;
    int K;
    long long n_full, rem;
    float eps;
    long long act_b, act_h, act_t;  // as in LinearArgs
    int tok_major;
    void* out;
    float* W1_last;
    float* b1_last;
    float* W2_last;
    float* b2_last;
    unsigned int* status;
    long long wait_limit;
};

struct DecodeArgs {
    const void* xq;
    const void* xk;
    const void* xv;
    const float* lr;
    const float* token_eta;
    const float* ln_w;
    const float* ln_b;
    float* W;
    float* b;
    float* W_grad;
    float* b_grad;
    int B, H, K;
    int p;          // position inside the mini-batch: seqlen_offset % K
    float eps;
    void* out;
    unsigned int* status;
    long long wait_limit;
};

// The decode step with a history-format cache (rows (lr_j xk_j, g_j) of the current mini-batch
// instead of the dense gradient sum).
struct DecodeHistArgs {
    const void* xq;
    const void* xk;
    const void* xv;
    const float* lr;
    const float* token_eta;
    const float* ln_w;
    const float* ln_b;
    float* W;
    float* b;
    float* hist;    // [B*H][K][2][d]
    float* b_grad;
    int B, H, K;
    int p;
    float eps;
    void* out;
    unsigned int* status;
    long long wait_limit;
};

// Tensor maps of XQ, XK, XV for the bf16 tensor-core prefill kernels, 128-byte swizzle:
// head-major 4-D dims {64, L, H, B}, box {64, K, 1, 1}, coordinates (0, token, h, b) -- or, for
// the TTT-Linear kernel, 3-D dims {64, L, B*H}, box {64, K, 1}, coordinates (0, token, chain);
// token-major dims {64, H, L, B}, box {64, 1, K, 1}, coordinates (0, h, token, b).
// Either way a box lands in shared memory as K rows of 128 bytes; rows past L read zero.
struct LinearMaps {
    CUtensorMap xq, xk, xv;
};

// launchers (return cudaSuccess or the launch error)
// The layer's output side, Y = o_proj(post_norm(X)) (see ttt_post_norm_o_proj).
struct OprojArgs {
    long long T;              // tokens (rows of X and Y)
    int C;                    // features of X (the post-norm width), a multiple of 64
    int N;                    // outputs (rows of the packed weight), a multiple of 256
    float eps;
    const float* u;           // [N] sum_k Wp[n][k]
    const float* v;           // [N] sum_k ln_b[k] Wo[n][k]
    const void* X;            // [T][C] bf16 (the statistics pass reads it directly)
    float2* stats;            // [T] (mean, rstd), written by the statistics pass
    void* Y;                  // [T][N] bf16
    unsigned int* status;
    long long wait_limit;
};
struct OprojMaps {
    CUtensorMap x, w;         // X [T][C] box {64, 128}; Wp [N][C] box {64, 256}; bf16, 128-byte swizzle
};
// The backward of the TTT-Linear scan (see ttt_linear_backward): one CTA per chain; fp32
// throughout.  The workspace holds, per chain, the states kept every G mini-batches, one group's
// rebuilt states, and the chain's shares of the gradients of the shared parameters.
struct LinearBwdArgs {
    const void* XQ;
    const void* XK;
    const void* XV;
    const void* d_out;          // upstream gradient of out, the activations' dtype and layout
    const float* lr;
    const float* token_eta;     // [K] or nullptr -> 1/(i+1)
    const float* W0;
    const float* b0;
    long long w0_chain_stride;  // elements between chains' W0 (0: one per head)
    const float* ln_w;
    const float* ln_b;
    const float* dW_last;       // [B*H][d][d] or nullptr (zero)
    const float* db_last;       // [B*H][d] or nullptr (zero)
    int B, H, K;
    long long L, n_full, rem;
    // element strides of XQ, XK, XV, d_out and their gradients between batch rows, heads and
    // tokens: head-major [B, H, L, d] or token-major [B, L, H, d] (as in LinearArgs)
    long long act_b, act_h, act_t;
    float eps;
    int G;                      // checkpoint group: a state is kept every G full mini-batches
    long long n_ckpt;           // ceil(n_full / G)
    void* dXQ;
    void* dXK;
    void* dXV;
    float* d_lr;
    float* ckpt;                // [B*H][ckpt_stride][d*d + d]: W ([k][n]) and b before every G-th full mini-batch
    long long ckpt_stride;      // states per chain in ckpt
    int ckpt_given;             // 1: ckpt holds the caller's checkpoints, the state after the last full
                                //    mini-batch at index n_ckpt; phase 1 is skipped
    float* slab;                // [B*H][G][d*d + d]
    float* part;                // [B*H][d*d + 3d]: dW0, db0, d ln_w, d ln_b of each chain
};
cudaError_t launch_linear_bwd(const LinearBwdArgs& a, int dtype, cudaStream_t s);
// Sum the per-chain shares over the batch: dW0/db0 per head (w0_per_chain = 0) or copied per chain,
// d ln_w / d ln_b per head.
cudaError_t launch_linear_bwd_reduce(const float* part, int B, int H, int w0_per_chain, float* dW0, float* db0,
                                     float* d_ln_w, float* d_ln_b, cudaStream_t s);
cudaError_t launch_oproj_prepare(const void* Wo, const float* ln_w, const float* ln_b, int C, int N, void* Wp,
                                 float* u, float* v, cudaStream_t s);
cudaError_t launch_post_norm_oproj(const OprojArgs& a, const OprojMaps& maps, cudaStream_t s);
cudaError_t launch_linear_simt(const LinearArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_linear_tc(const LinearArgs& a, const LinearMaps& maps, cudaStream_t s);
cudaError_t launch_linear_state_copy(const LinearArgs& a, cudaStream_t s);
cudaError_t launch_mlp_simt(const MlpArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_mlp_tc(const MlpArgs& a, const LinearMaps& maps, cudaStream_t s);
cudaError_t launch_mlp_state_copy(const MlpArgs& a, cudaStream_t s);
cudaError_t launch_decode(const DecodeArgs& a, int dtype, cudaStream_t s);
cudaError_t launch_decode_hist(const DecodeHistArgs& a, int dtype, cudaStream_t s);

}  // namespace ttt
