/*
 * ttt.h -- C ABI of libttt.so: the TTT-Linear / TTT-MLP mini-batch test-time-training scan
 * and the TTT-Linear cache decode step, for NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [walkthrough] "代码连连看——TTT" (jiafeimiao.top): TTTBase.forward, TTTLinear.ttt and
 *                 compute_mini_batch (dual branch, primal branch) listings.
 *   [explainer]   "测试时学习（TTT）原理解析：ttt-lm-pytorch如何让模型在推理时持续学习"
 *                 (nanhubrain.csdn.net): TTTLinear.__init__ and the TTTCache section.
 *   [readme]      the ttt-lm-pytorch README (downcodes.com mirror): TTT-Linear and TTT-MLP.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensor pointers are DEVICE pointers into memory the caller owns (allocated by the
 *    caller, e.g. PyTorch) -- except in ttt_linear_forward_host, whose tensors are HOST
 *    buffers.  The library allocates no device memory and keeps no state across calls except
 *    a thread-local last-error message and one device status word per device.
 *  - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL = the legacy
 *    default stream).  No call synchronises the stream, except ttt_device_status().
 *  - A "chain" is one (batch b, head h) pair; chain index = b * H + h.
 *  - Activations are [B, H, L, d] contiguous (the layout TTTLinear.ttt receives after the head
 *    split), so one chain's mini-batch is one contiguous block of K * d elements -- or, for the
 *    prefill calls with TTT_FLAG_TOKEN_MAJOR, [B, L, H, d] (the [B, L, C] of the projections).
 *  - dtype selects the element type of XQ, XK, XV and out: TTT_F32 or TTT_BF16.  The output
 *    takes the input dtype (the walkthrough allocates XQW_batch with the input dtype).  The
 *    hidden state (W, b, grads), lr, token_eta, ln_w and ln_b are always float32.
 *  - Only head dimension d = 64 is supported; mini_batch K in [1, 16].
 *  - Return value: TTT_OK (0) or a negative TTT_ERR_* code, and ttt_last_error_message()
 *    describes the cause.  After an argument error (every code but TTT_ERR_CUDA) nothing has been
 *    enqueued.  TTT_ERR_CUDA from the single-launch calls also means nothing ran; only
 *    ttt_linear_forward_host, which enqueues many copies and launches, can fail with TTT_ERR_CUDA
 *    after part of its work is enqueued (see there).  No C++ exception crosses the ABI.
 *  - Argument errors are found on the host before any CUDA call, so they can be tested
 *    without a GPU.
 */
#ifndef TTT_H_
#define TTT_H_

#ifdef __cplusplus
extern "C" {
#endif

#define TTT_OK 0
#define TTT_ERR_ARG (-1)         /* null required pointer, bad size, bad dtype or flag */
#define TTT_ERR_ALIGN (-2)       /* a pointer is not aligned as documented */
#define TTT_ERR_ALIAS (-3)       /* an output overlaps an input or another output */
#define TTT_ERR_CUDA (-4)        /* a CUDA runtime/driver call or a launch failed */
#define TTT_ERR_TIMEOUT (-5)     /* a bounded device-side wait expired (see ttt_device_status) */
#define TTT_ERR_UNSUPPORTED (-6) /* valid but not implemented here (e.g. d != 64) */

#define TTT_F32 0
#define TTT_BF16 1

/* flags for the forward calls */
#define TTT_FLAG_FP32_COMPUTE 1u /* run bf16 inputs through the FFMA (fp32-compute) kernel */
/* XQ, XK, XV and out are token-major [B,L,H,d] -- the [B,L,C] (C = H*d) layout of the QKV
 * projections and of the scan's return value in TTTBase.forward / TTTLinear.ttt -- instead of
 * the head-major [B,H,L,d].  lr stays [B,H,L].  The arithmetic and the results are the same. */
#define TTT_FLAG_TOKEN_MAJOR 2u
/* ttt_linear_forward_rope only: rotate the feature pairs (k, k + d/2) (the half-split rotation
 * applied directly, without permute_qk / undo_permute_qk) instead of (2k, 2k+1). */
#define TTT_FLAG_ROPE_HALF_SPLIT 4u

/* Bits of the device status word */
#define TTT_STATUS_TIMEOUT 1u /* a kernel gave up on a bounded wait and returned early */

/*
 * ttt_partition -- split a sequence of L tokens into mini-batches of K.
 * [walkthrough] TTTBase.forward: num_mini_batch = L // K full mini-batches run first, then
 * reminder_len = L % K remaining tokens run as one mini-batch of size r.
 *   L >= 0, mini_batch >= 1; n_full, rem: host pointers receiving L / K and L % K.
 * Host-only, exact integer arithmetic.  Returns TTT_ERR_ARG on a bad argument.
 */
int ttt_partition(long long L, int mini_batch, long long* n_full, long long* rem);

/* Static description of an error code; never NULL. */
const char* ttt_error_string(int code);

/* Message of the last failing call on this host thread ("" if none); valid until the next call. */
const char* ttt_last_error_message(void);

/*
 * ttt_device_status -- read (and optionally clear) the status word that kernels on the CURRENT
 * device set when a bounded wait expires.  Synchronises `stream`.  *status receives the
 * TTT_STATUS_* bits (0 = healthy).  With clear != 0 the word is read and zeroed in one atomic
 * step on the device (a one-thread kernel on `stream`), so a bit that a kernel on another
 * stream raises meanwhile is reported by this call or the next, never lost.  Returns
 * TTT_ERR_TIMEOUT if the timeout bit was set, TTT_ERR_CUDA on a CUDA error, else TTT_OK.
 */
int ttt_device_status(void* stream, unsigned int* status, int clear);

/*
 * ttt_set_wait_limit -- test hook: cap on the polls of every bounded device-side wait issued
 * by later launches from this process.  polls > 0: that cap; 0: the default (2^24 polls,
 * far above any healthy wait); < 0: zero polls, so every bounded wait gives up at once.  This
 * exercises the TTT_ERR_TIMEOUT path without faulting or hanging the GPU: the kernel raises
 * the status bit, waits (with the default bound) for its own copies in flight and returns.
 * The tensor-core TTT-Linear and TTT-MLP prefill kernels and the decode kernel have such waits.
 * Host-only; returns TTT_OK.
 */
int ttt_set_wait_limit(long long polls);

/*
 * ttt_linear_forward -- TTT-Linear prefill: the mini-batch TTT scan over L tokens of every
 * chain ([walkthrough] TTTBase.forward, TTTLinear.ttt, compute_mini_batch).
 *
 * Per chain (b, h), with K = mini_batch, state (W, b) starting at (W0, b0):
 *   for each mini-batch X of K tokens (then one tail mini-batch of r = L % K tokens):
 *     Z = XK W + b;  g = d/dZ 1/2 ||LN(Z) - (XV - XK)||^2          (ln_fused_l2_bwd)
 *     eta[i][j] = token_eta[i] * lr[j] for j <= i, else 0
 *     Zbar = XQ W - (eta * tril(XQ XK^T)) g + b - tril(eta) g      (dual branch)
 *     out  = XQ + LN(Zbar)                                         (ln_fwd, residual)
 *     full mini-batch only: W -= (eta[K-1,:] * XK)^T g;  b -= sum_j eta[K-1,j] g_j
 *   LN(u) = ln_w * (u - mean(u)) / sqrt(var(u) + eps) + ln_b, biased variance over d.
 *
 * Arguments:
 *   XQ, XK, XV   [B,H,L,d] dtype, 16-byte aligned.  May be NULL only when L == 0.
 *   lr           [B,H,L] float32, 4-byte aligned: the per-token learning rate (ttt_lr_eta).
 *   token_eta    [K] float32 or NULL (= 1/(i+1), i = position inside the mini-batch).
 *   W0, b0       float32, 16-byte aligned: [H,d,d] and [H,d] shared over the batch when
 *                w0_batch_stride == 0 (the walkthrough tiles W1, b1 over B), or [B,H,d,d] and
 *                [B,H,d] per chain when w0_batch_stride == H*d*d (a continuation).
 *                W is indexed W[a][c]: Z[c] = sum_a XK[a] W[a][c] + b[c].
 *   ln_w, ln_b   [H,d] float32: the per-head LayerNorm affine parameters (ttt_norm_*).
 *   B, H, L, d   sizes: B, H >= 1; L >= 0; d == 64.  L == 0 copies the state only.
 *   mini_batch   K in [1, 16].
 *   eps          LayerNorm epsilon, > 0.
 *   dtype        TTT_F32 or TTT_BF16.
 *   flags        TTT_FLAG_FP32_COMPUTE and/or TTT_FLAG_TOKEN_MAJOR, or 0.  bf16 inputs run on
 *                the tensor-core kernel (fp16 operands, fp32 accumulation and fp32 state) unless
 *                FP32_COMPUTE asks for the FFMA kernel; fp32 inputs always run on the FFMA
 *                kernel.  The tensor-core kernel takes each LayerNorm variance in one pass,
 *                E[x^2] - mean^2 in fp32, which holds 1e-2 relative accuracy while every row of
 *                Z = XK W + b has |mean over features| below about 50x its spread; the scan never
 *                raises that ratio above what W0 and b0 give (the LayerNorm gradient's features
 *                sum to zero, so the updates keep the feature means of W and b), and it is about
 *                1/8 for the walkthrough's initialisation.  FP32_COMPUTE (two-pass statistics)
 *                serves states beyond that.  TOKEN_MAJOR: XQ, XK, XV and out are [B,L,H,d] instead of [B,H,L,d]
 *                (the walkthrough's [B,L,C] before its reshape/transpose and after the scan's
 *                permute/reshape, so neither permute is needed); lr stays [B,H,L].
 * Outputs (device, caller-allocated):
 *   out          [B,H,L,d] dtype, 16-byte aligned (may be NULL when L == 0).
 *   W_last, b_last  [B,H,d,d], [B,H,d] float32: the state after the last FULL mini-batch (the
 *                tail's params are dropped, as TTTBase.forward does).  W_last may be the same
 *                pointer as W0 (and b_last as b0) for an in-place update when the state is
 *                per chain; no other overlap is allowed.
 *   W_grad_tail, b_grad_tail  NULL, or [B,H,d,d], [B,H,d] float32 receiving the tail's
 *                un-scaled grad sums sum_{j<r} lr_j XK_j^T g_j and sum_{j<r} lr_j g_j (zeros when
 *                r == 0): with W_last/b_last they form the TTTCache state for decoding on.
 */
int ttt_linear_forward(const void* XQ, const void* XK, const void* XV, const float* lr,
                       const float* token_eta, const float* W0, const float* b0,
                       long long w0_batch_stride, const float* ln_w, const float* ln_b, int B,
                       int H, long long L, int d, int mini_batch, float eps, int dtype,
                       unsigned int flags, void* out, float* W_last, float* b_last,
                       float* W_grad_tail, float* b_grad_tail, void* stream);

/*
 * ttt_linear_forward_rope -- ttt_linear_forward with the rotary position embedding of XQ and XK
 * fused into the scan's load path ([walkthrough] TTTBase.forward: cos, sin = rotary_emb(XV,
 * position_ids % mini_batch_size); permute_qk; apply_rotary_pos_emb; undo_permute_qk -- the
 * rotation of RoFormer).  The scan sees, in place of XQ and XK (both for the contractions and
 * for the reconstruction target XV - XK and the residual XQ + LN(Zbar)),
 *   X'[t, 2k]   = X[t, 2k] cos(a) - X[t, 2k+1] sin(a)
 *   X'[t, 2k+1] = X[t, 2k] sin(a) + X[t, 2k+1] cos(a),   a = (t mod K) * rope_theta^(-2k/d),
 * for k = 0 .. d/2 - 1: the position restarts at 0 in every mini-batch (the tail mini-batch
 * included), and the pairs (2k, 2k+1) are the net effect of permute_qk, the half-split rotation
 * and undo_permute_qk.  With TTT_FLAG_ROPE_HALF_SPLIT the pairs are (k, k + d/2) instead.  The
 * rotated activations exist only on chip (in fp16, the tensor-core operand type); XQ and XK in
 * memory are not changed.  The angle is evaluated in fp32.
 * Arguments and results are those of ttt_linear_forward, plus
 *   rope_theta   the rotary base theta, finite and > 0 (the walkthrough does not print its value;
 *                RoFormer's is 10000);
 *   flags        TTT_FLAG_TOKEN_MAJOR and/or TTT_FLAG_ROPE_HALF_SPLIT, or 0;
 * and the restrictions: dtype must be TTT_BF16 and TTT_FLAG_FP32_COMPUTE is not accepted (both
 * TTT_ERR_UNSUPPORTED: the rotation lives in the tensor-core kernel only).  Errors otherwise as
 * ttt_linear_forward, plus TTT_ERR_ARG for a bad rope_theta.
 */
int ttt_linear_forward_rope(const void* XQ, const void* XK, const void* XV, const float* lr,
                            const float* token_eta, const float* W0, const float* b0,
                            long long w0_batch_stride, const float* ln_w, const float* ln_b, int B,
                            int H, long long L, int d, int mini_batch, float eps, float rope_theta,
                            int dtype, unsigned int flags, void* out, float* W_last, float* b_last,
                            float* W_grad_tail, float* b_grad_tail, void* stream);

/*
 * ttt_linear_host_workspace_bytes -- size in bytes of the device workspace that
 * ttt_linear_forward_host needs for these sizes: the per-head parameters plus two staging sets
 * (inputs and outputs of `chunk_batches` batch rows each, tail-grad room included).
 * Same size rules as ttt_linear_forward; 1 <= chunk_batches <= B; w0_batch_stride 0 or H*d*d.
 * Host-only.  Returns the byte count (> 0) or a negative TTT_ERR_* code.
 * (No counterpart on the pages: the walkthrough's tensors are already on the device.)
 */
long long ttt_linear_host_workspace_bytes(int B, int H, long long L, int d, int mini_batch, int dtype,
                                          int chunk_batches, long long w0_batch_stride);

/*
 * ttt_linear_forward_host -- ttt_linear_forward on HOST buffers: the same scan, the same
 * arguments and results, except that
 *   - every tensor argument (XQ, XK, XV, lr, token_eta, W0, b0, ln_w, ln_b and the outputs out,
 *     W_last, b_last, W_grad_tail, b_grad_tail) is a HOST pointer; page-locked (pinned) memory
 *     lets the copies run asynchronously and overlap;
 *   - workspace is a caller-owned DEVICE buffer of at least ttt_linear_host_workspace_bytes()
 *     bytes (same B, H, L, d, mini_batch, dtype, chunk_batches, w0_batch_stride), 256-byte
 *     aligned; its contents on entry are irrelevant and on return undefined.
 * The batch runs in chunks of chunk_batches batch rows (the last may be shorter): the
 * host-to-device copies of a chunk run on a copy stream owned by the library while the chunk
 * before it computes and its results return on `stream`, so both copy directions and the
 * kernels overlap.  The results equal ttt_linear_forward's on the same values, bit for bit.
 * Asynchronous on `stream`: on return everything is enqueued; the host buffers must stay valid
 * and unchanged, and the workspace unused by anyone else, until `stream` passes this point.
 * The library creates, once per device, one non-blocking copy stream and five events (never
 * freed) and allocates no device memory; concurrent calls are serialised while they enqueue.
 * (No counterpart on the pages: the walkthrough's tensors are already on the device.)
 * Errors as ttt_linear_forward, plus TTT_ERR_ARG for a missing or too small workspace or a bad
 * chunk_batches, TTT_ERR_ALIGN for a misaligned workspace.  All of these are found before
 * anything is enqueued.  A TTT_ERR_CUDA, however, can come after the copies and scans of earlier
 * chunks are already enqueued on `stream` and on the copy stream: after such a failure,
 * synchronise `stream` before reusing the workspace or the host buffers, and treat the outputs
 * as undefined.
 */
int ttt_linear_forward_host(const void* XQ, const void* XK, const void* XV, const float* lr,
                            const float* token_eta, const float* W0, const float* b0,
                            long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                            long long L, int d, int mini_batch, float eps, int dtype, unsigned int flags,
                            void* out, float* W_last, float* b_last, float* W_grad_tail,
                            float* b_grad_tail, void* workspace, long long workspace_bytes,
                            int chunk_batches, void* stream);

/*
 * ttt_linear_forward_host_static -- ttt_linear_forward_host for callers that cannot allocate
 * device memory, using scratch built into the library instead of a caller's workspace.
 * (No counterpart on the pages: it is a deployment variant of the host-buffer entry.)
 *
 * Who needs it: a caller whose device memory is all handed out in advance by another owner (a
 * serving framework's caching pool, a fixed per-process budget), so that a cudaMalloc would fail
 * or break that owner's accounting; a plain C host program with no device allocator of its own;
 * a latency-sensitive caller that must not take the device-wide synchronisation that cudaMalloc
 * and cudaFree can imply.  It allocates nothing: no cudaMalloc, no cudaFree, no library
 * allocation, no stream or event creation.
 *
 * The scratch is one static device array of TTT_STATIC_SCRATCH_BYTES (32 MiB) per device that
 * loads the library, held until the process exits.  The batch runs in chunks of as many batch
 * rows as fit in it (the per-head parameters plus one set of staged inputs and outputs); sizes
 * whose single batch row does not fit are rejected with TTT_ERR_ARG and a message giving the
 * bytes needed (use ttt_linear_forward_host with a workspace for those).  Copies and kernels run
 * one after another on `stream` (no overlap between chunks).
 *
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 * that device current); make that first call before any stream capture.  Every call on a device
 * shares the one array: calls that can overlap on the GPU (on different streams, or from
 * several threads without ordering) race and corrupt each other's results -- order them on one
 * stream.  The array keeps the last call's contents; nothing in it needs to start at zero, since
 * each call writes every byte it reads.
 *
 * Arguments, results and errors as ttt_linear_forward_host, without workspace, workspace_bytes
 * and chunk_batches.  Asynchronous on `stream`; the host buffers must stay valid and unchanged
 * until `stream` passes this point.  A TTT_ERR_CUDA can come after earlier chunks are enqueued;
 * synchronise `stream` before reusing the buffers after one.
 */
#define TTT_STATIC_SCRATCH_BYTES 33554432
int ttt_linear_forward_host_static(const void* XQ, const void* XK, const void* XV, const float* lr,
                                   const float* token_eta, const float* W0, const float* b0,
                                   long long w0_batch_stride, const float* ln_w, const float* ln_b, int B,
                                   int H, long long L, int d, int mini_batch, float eps, int dtype,
                                   unsigned int flags, void* out, float* W_last, float* b_last,
                                   float* W_grad_tail, float* b_grad_tail, void* stream);

/*
 * ttt_mlp_forward -- TTT-MLP prefill ([readme]: the hidden state is a two-layer MLP;
 * [walkthrough]: "TTTMLP is two TTTLinear stacked").  The state is
 *   f(x) = gelu(x W1 + b1) W2 + b2,  gelu = tanh form, W1 [d,hid], W2 [hid,d],
 * and each mini-batch takes the layer-wise dual update of ttt_linear_forward:
 *   Z1 = XK W1 + b1, X2 = gelu(Z1), Z2 = X2 W2 + b2, g2 = d/dZ2 1/2||LN(Z2) - (XV - XK)||^2,
 *   g1 = (g2 W2^T) * gelu'(Z1);
 *   Zbar1 = XQ W1 - (eta * tril(XQ XK^T)) g1 + b1 - tril(eta) g1;  Xbar2 = gelu(Zbar1);
 *   Zbar2 = Xbar2 W2 - (eta * tril(Xbar2 X2^T)) g2 + b2 - tril(eta) g2;  out = XQ + LN(Zbar2);
 *   full mini-batch: W1 -= (eta[K-1,:] * XK)^T g1, W2 -= (eta[K-1,:] * X2)^T g2, biases alike.
 * Arguments as ttt_linear_forward, with hidden == 256 (= 4 d), states W1_0 [H,d,hid],
 * b1_0 [H,hid], W2_0 [H,hid,d], b2_0 [H,d] (w0_batch_stride 0), or per chain [B,H,...]
 * (w0_batch_stride == H*d*hid), and outputs W1_last, b1_last, W2_last, b2_last per chain.
 * The tail's params are dropped as in TTT-Linear; no tail grads are reported.
 */
int ttt_mlp_forward(const void* XQ, const void* XK, const void* XV, const float* lr,
                    const float* token_eta, const float* W1_0, const float* b1_0,
                    const float* W2_0, const float* b2_0, long long w0_batch_stride,
                    const float* ln_w, const float* ln_b, int B, int H, long long L, int d,
                    int hidden, int mini_batch, float eps, int dtype, unsigned int flags,
                    void* out, float* W1_last, float* b1_last, float* W2_last, float* b2_last,
                    void* stream);

/*
 * ttt_linear_decode_step -- one new token per chain through the TTTCache state
 * ([walkthrough] TTTLinear.ttt: decoding reads the params from the cache and, the mini-batch
 * not being a multiple of K, takes the primal branch so the grads can be stored;
 * [explainer] TTTCache: last states + grads, seqlen_offset, mini_batch_size).
 * With p = seqlen_offset % K (every chain shares one offset) and t = token_eta[p] (default
 * 1/(p+1)):
 *   z = xk W + b;  g = d/dz 1/2||LN(z) - (xv - xk)||^2;
 *   W_grad += lr xk^T g;  b_grad += lr g;
 *   out = xq + LN(xq (W - t W_grad) + (b - t b_grad));
 *   if p == K-1: W -= t W_grad; b -= t b_grad; W_grad = 0; b_grad = 0   (commit)
 * W, b hold the state committed at the last mini-batch boundary; W_grad, b_grad the
 * lr-weighted grad sums of the tokens since.  After ttt_linear_forward over L tokens, the
 * cache is (W_last, b_last, W_grad_tail, b_grad_tail) with seqlen_offset = L.
 * Arguments:
 *   xq, xk, xv  [B,H,d] dtype, 16-byte aligned;  lr [B,H] float32;  token_eta [K] or NULL.
 *   ln_w, ln_b  [H,d] float32.
 *   W, b, W_grad, b_grad  [B,H,d,d], [B,H,d], [B,H,d,d], [B,H,d] float32, 16-byte aligned,
 *               read and written in place (the caller's cache).
 *   seqlen_offset >= 0: absolute position of this token.  The caller advances it by one.
 *   out         [B,H,d] dtype.
 */
int ttt_linear_decode_step(const void* xq, const void* xk, const void* xv, const float* lr,
                           const float* token_eta, const float* ln_w, const float* ln_b,
                           float* W, float* b, float* W_grad, float* b_grad, int B, int H,
                           int d, int mini_batch, long long seqlen_offset, float eps, int dtype,
                           void* out, void* stream);

/*
 * ttt_linear_decode_step_hist -- the decode step of ttt_linear_decode_step with a history-format
 * cache.  The dense cache keeps W_grad = sum_{j<p} lr_j xk_j^T g_j (d x d per chain); this one
 * keeps the rows that make it up, (lr_j * xk_j, g_j) for the tokens j < p of the current
 * mini-batch, and forms xq W_grad as sum_j (xq . lr_j xk_j) g_j.  The results are those of the
 * dense cache (up to fp32 rounding order); the state traffic per step is W, b, b_grad and p rows
 * read, one row and b_grad written (and W, b on the commit step) instead of W and W_grad read
 * and W_grad written.
 * Arguments as ttt_linear_decode_step, except
 *   hist    [B,H,K,2,d] float32 in/out (K = mini_batch), 16-byte aligned: row j of a chain holds
 *           lr_j * xk_j (d floats) then g_j (d floats).  Rows j < p = seqlen_offset mod K are
 *           read; row p is written (except on the commit step p = K-1, which folds the rows into
 *           W); rows past p are neither read nor written.
 *   b_grad  [B,H,d] float32 in/out: sum_{j<p} lr_j g_j, zeroed on the commit step.
 * A history cache starts at a mini-batch boundary (seqlen_offset mod K == 0) with b_grad = 0;
 * there the dense and history caches coincide (both are just W, b).
 * Rows are read only while the p read for this call says so: all chains share seqlen_offset.
 * (No counterpart on the pages beyond the identity W_grad = sum_j lr_j xk_j^T g_j of the primal
 * branch in "代码连连看——TTT", compute_mini_batch.)
 * Errors as ttt_linear_decode_step.
 */
int ttt_linear_decode_step_hist(const void* xq, const void* xk, const void* xv, const float* lr,
                                const float* token_eta, const float* ln_w, const float* ln_b, float* W, float* b,
                                float* hist, float* b_grad, int B, int H, int d, int mini_batch,
                                long long seqlen_offset, float eps, int dtype, void* out, void* stream);

/*
 * The layer's output side: Y = o_proj(post_norm(X)) per token ([walkthrough] TTTBase.forward,
 * after torch.cat of the mini-batch outputs: post_norm, then o_proj; apply_gate is "Mamba only"
 * on the page and is not part of this path).  Readings, as in the oracle: post_norm is a
 * LayerNorm over the token's C = num_heads * head_dim features (affine ln_w, ln_b; biased
 * variance; eps inside the square root), o_proj a linear map without bias whose weight Wo is
 * stored [N][C] (out x in, the layout of torch's nn.Linear.weight).  X is the scan's output
 * taken token-major: [B, L, num_heads * 64] = [T, C] (ttt_linear_forward with
 * TTT_FLAG_TOKEN_MAJOR writes exactly that), T = B * L.
 *
 * The LayerNorm folds into the product: y[n] = rstd (sum_k x_k Wp[n][k] - mean u[n]) + v[n],
 * with Wp[n][k] = ln_w[k] Wo[n][k], u[n] = sum_k Wp[n][k], v[n] = sum_k ln_b[k] Wo[n][k].
 * ttt_o_proj_prepare packs those once per weight; ttt_post_norm_o_proj then runs one
 * tensor-core GEMM (tcgen05, fp32 accumulation in tensor memory) whose epilogue applies the
 * token statistics, which a one-warp-per-token pass over X (Chan's merge of the lanes' moments)
 * writes just before.  Y is rounded to bf16.  The correction subtracts mean * u[n] from the product in
 * fp32, so its accuracy falls as a token's |mean| / std grows (the scan's output has mean near
 * zero next to its spread).
 *
 * Sizes: C a positive multiple of 64, N a positive multiple of 256 (both hold for the 125M and
 * 1B layers, C = N = 768 and 2048); T >= 0, at most 65535 * 128 tokens.
 */

/*
 * ttt_o_proj_prepare -- pack o_proj's weight for ttt_post_norm_o_proj.
 *   Wo           [N][C] bf16 (device), 16-byte aligned: the o_proj weight (out x in).
 *   ln_w, ln_b   [C] float32 (device): post_norm's affine parameters.
 *   Wp           [N][C] bf16 (device, caller-allocated), 16-byte aligned: receives ln_w[k] * Wo[n][k].
 *   u, v         [N] float32 (device, caller-allocated): receive sum_k Wp[n][k] (of the rounded
 *                Wp) and sum_k ln_b[k] Wo[n][k].
 * Asynchronous on `stream`.  Errors: TTT_ERR_UNSUPPORTED for C or N outside the sizes above,
 * TTT_ERR_ARG for a null pointer, TTT_ERR_ALIGN, TTT_ERR_ALIAS if an output overlaps an input
 * or another output, TTT_ERR_CUDA if the launch fails.  (No counterpart on the pages: it is the
 * one-time weight transform of the fused form above.)
 */
int ttt_o_proj_prepare(const void* Wo, const float* ln_w, const float* ln_b, int C, int N, void* Wp, float* u,
                       float* v, void* stream);

/*
 * ttt_post_norm_o_proj -- Y = o_proj(post_norm(X)) for T tokens.
 *   X            [T][C] bf16 (device), 16-byte aligned (NULL allowed when T == 0).
 *   Wp, u, v     from ttt_o_proj_prepare for this weight and these post_norm parameters.
 *   eps          post_norm's epsilon, finite and > 0.
 *   Y            [T][N] bf16 (device, caller-allocated), 16-byte aligned; must not overlap the
 *                inputs.
 *   row_stats    [T][2] float32 (device, caller-allocated), 8-byte aligned: receives each token's
 *                (mean, 1/sqrt(var + eps)) of post_norm (written by the first of the call's two
 *                launches, read by the second); must not overlap the inputs or Y.
 * Asynchronous on `stream`; allocates nothing.  T == 0 does nothing.  Errors as
 * ttt_o_proj_prepare, plus TTT_ERR_ARG for a bad eps or T < 0, TTT_ERR_UNSUPPORTED for T above
 * 65535 * 128.  The kernel's waits are bounded (see ttt_device_status).
 */
int ttt_post_norm_o_proj(const void* X, long long T, int C, const void* Wp, const float* u, const float* v, int N,
                         float eps, void* Y, float* row_stats, void* stream);

/* ---- training: the backward of the TTT-Linear scan ----------------------------------------
 * [walkthrough] TTTLinear.ttt hands scan_checkpoint_group_size to its scan while training, so
 * the outer parameters learn through the scan; [readme] says training with the pure-PyTorch
 * code is slow.  The backward below runs through the same scan on the device. */

/*
 * ttt_linear_backward_workspace_bytes -- bytes of device workspace ttt_linear_backward needs:
 * per chain, ceil(n_full / ckpt_group) kept states and ckpt_group rebuilt states of
 * (d*d + d) float32 each, plus (d*d + 3d) float32 of per-chain gradient shares; n_full = L / K.
 * Host-only.  Returns the byte count (> 0) or a negative TTT_ERR_* code.
 */
long long ttt_linear_backward_workspace_bytes(int B, int H, long long L, int d, int mini_batch, int ckpt_group);

/*
 * ttt_linear_backward -- gradients of the outer inputs of ttt_linear_forward.
 *
 * For the forward described at ttt_linear_forward (same inputs, same tail rule), and caller
 * gradients d_out of out, dW_last of W_last and db_last of b_last, it returns the gradients of
 *   <d_out, out> + <dW_last, W_last> + <db_last, b_last>
 * with respect to XQ, XK, XV, lr, W0, b0, ln_w and ln_b -- the reverse-mode derivative of the
 * scan, through every mini-batch's loss gradient (the derivative of ln_fused_l2_bwd itself),
 * the dual form's attention-like terms and the state updates.  token_eta and eps are constants.
 *
 * Scan checkpoint groups: the forward state recursion runs once over the full mini-batches and
 * keeps every ckpt_group-th state; the backward then takes the groups from the last, rebuilds a
 * group's states from its kept state, and steps back through the group.  ckpt_group trades
 * workspace (above) for nothing else: the results do not depend on it.
 *
 * Arguments:
 *   XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride, ln_w, ln_b, B, H, L, d, mini_batch,
 *   eps, dtype   as ttt_linear_forward.
 *   flags        0 or TTT_FLAG_TOKEN_MAJOR: XQ, XK, XV, d_out, dXQ, dXK and dXV are [B,L,H,d] instead
 *                of [B,H,L,d] (lr and d_lr stay [B,H,L]); TTT_FLAG_FP32_COMPUTE is
 *                TTT_ERR_UNSUPPORTED (fp32 activations already run in fp32).
 *   ckpt_group   >= 1: mini-batches per checkpoint group.
 *   d_out        [B,H,L,d] (or token-major) dtype, 16-byte aligned: the gradient of out (NULL
 *                allowed if L == 0).
 *   dW_last, db_last  [B,H,d,d], [B,H,d] float32, 16-byte aligned, or NULL (zero).
 * Outputs (device, caller-allocated, none overlapping an input, another output or the workspace):
 *   dXQ, dXK, dXV  [B,H,L,d] (or token-major) dtype, 16-byte aligned (NULL allowed if L == 0).
 *   d_lr         [B,H,L] float32.
 *   dW0, db0     float32: [H,d,d] and [H,d] summed over the batch when w0_batch_stride == 0 (one
 *                initial state per head), else [B,H,d,d] and [B,H,d] per chain.
 *   d_ln_w, d_ln_b  [H,d] float32, summed over the batch.
 *   workspace    device buffer of at least ttt_linear_backward_workspace_bytes, 256-byte aligned;
 *                its contents on entry do not matter and are overwritten.
 * One CTA per chain.  fp32 activations compute in float32 throughout (two-pass LayerNorm
 * statistics); bf16 activations run the products and state updates on the tensor cores with TF32
 * operands (11-bit significands, like the forward's fp16 operands) and fp32 accumulation, state
 * and adjoint, and take each LayerNorm variance in one pass, with the forward kernel's bound (rows
 * of Z with |mean over features| below about 50x their spread; see ttt_linear_forward).  fp32
 * activations serve states beyond it.  The batch sums run in
 * a fixed order, so results are reproducible bit for bit.  Asynchronous on `stream`; allocates nothing; has no
 * device-side waits.  Errors as ttt_linear_forward (flags aside), plus TTT_ERR_ARG for
 * ckpt_group < 1 or a workspace smaller than needed.  The call makes two launches (the scan's
 * backward, then the batch sums); a TTT_ERR_CUDA from the second comes after the first is
 * enqueued, so synchronise `stream` before reusing the workspace or the outputs after it.
 */
int ttt_linear_backward(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                        const float* W0, const float* b0, long long w0_batch_stride, const float* ln_w,
                        const float* ln_b, int B, int H, long long L, int d, int mini_batch, float eps, int dtype,
                        unsigned int flags, int ckpt_group, const void* d_out, const float* dW_last,
                        const float* db_last, void* dXQ, void* dXK, void* dXV, float* d_lr, float* dW0, float* db0,
                        float* d_ln_w, float* d_ln_b, void* workspace, long long workspace_bytes, void* stream);

/* ---- checkpoints from the forward ------------------------------------------------------------
 * [walkthrough] TTTLinear.ttt's scan keeps the carried state at the start of every checkpoint
 * group during the forward pass and rebuilds the states inside a group during the backward.  The
 * three calls below give training that split: the forward writes the group-boundary states, and
 * the backward starts from them instead of running the state recursion once more (its phase 1). */

/*
 * ttt_linear_ckpt_bytes -- bytes of the checkpoint buffer of ttt_linear_forward_ckpt and
 * ttt_linear_backward_ckpt: per chain, ceil(n_full / ckpt_group) + 1 states of (d*d + d) float32,
 * n_full = L / K.  Host-only.  Returns the byte count (> 0) or a negative TTT_ERR_* code.
 */
long long ttt_linear_ckpt_bytes(int B, int H, long long L, int d, int mini_batch, int ckpt_group);

/*
 * ttt_linear_forward_ckpt -- ttt_linear_forward that also writes checkpoints for the backward.
 * Arguments and results as ttt_linear_forward, plus
 *   ckpt_group   G >= 1: a state is kept before every G-th full mini-batch (mini-batches 0, G, 2G, ...).
 *   ckpt         device buffer of ttt_linear_ckpt_bytes, 16-byte aligned, written: chain c's entry i
 *                (c * (n_ckpt + 1) + i, each d*d + d float32) is W as [k][n] then b before full
 *                mini-batch i*G for i < n_ckpt, and the state after the last full mini-batch (equal
 *                to W_last, b_last) at i = n_ckpt.  The states are the kernel's own fp32 state.
 * Errors as ttt_linear_forward, plus TTT_ERR_ARG for a null ckpt or ckpt_group < 1, TTT_ERR_ALIGN,
 * and TTT_ERR_ALIAS when ckpt overlaps another argument.
 */
int ttt_linear_forward_ckpt(const void* XQ, const void* XK, const void* XV, const float* lr,
                            const float* token_eta, const float* W0, const float* b0,
                            long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                            long long L, int d, int mini_batch, float eps, int dtype, unsigned int flags,
                            void* out, float* W_last, float* b_last, float* W_grad_tail,
                            float* b_grad_tail, int ckpt_group, float* ckpt, void* stream);

/*
 * ttt_linear_backward_ckpt -- ttt_linear_backward from the checkpoints of ttt_linear_forward_ckpt
 * (the same inputs and ckpt_group): the backward skips its own pass of the state recursion over
 * the full mini-batches and rebuilds each group from the caller's state at its start.
 * Arguments and results as ttt_linear_backward, plus
 *   ckpt         the checkpoint buffer (read only), 16-byte aligned; the workspace keeps its size.
 * The gradients are those of ttt_linear_backward up to rounding: the forward's fp16-operand
 * state recursion and the backward's TF32 one differ in the last bits (bf16 activations), so
 * unlike ttt_linear_backward the results depend on ckpt_group in those bits.
 * Errors as ttt_linear_backward, plus TTT_ERR_ARG for a null ckpt, TTT_ERR_ALIGN, TTT_ERR_ALIAS.
 */
int ttt_linear_backward_ckpt(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                             const float* W0, const float* b0, long long w0_batch_stride, const float* ln_w,
                             const float* ln_b, int B, int H, long long L, int d, int mini_batch, float eps,
                             int dtype, unsigned int flags, int ckpt_group, const float* ckpt, const void* d_out,
                             const float* dW_last, const float* db_last, void* dXQ, void* dXK, void* dXV,
                             float* d_lr, float* dW0, float* db0, float* d_ln_w, float* d_ln_b, void* workspace,
                             long long workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* TTT_H_ */
