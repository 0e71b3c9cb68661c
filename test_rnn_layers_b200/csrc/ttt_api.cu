// ttt_api.cu -- the extern "C" boundary of libttt.so (declared in include/ttt.h).
//
// Argument checks run on the host before any CUDA call; each entry point then picks a kernel
// and enqueues it on the caller's stream.  No device memory is allocated here.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/ttt.h"
#include "ttt_internal.h"

namespace {

thread_local std::string g_last_error;
std::atomic<long long> g_wait_limit{0};
constexpr long long kDefaultWaitPolls = 1ll << 24;
constexpr int kD = 64;
constexpr int kHidden = 256;

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int ok() {
    g_last_error.clear();
    return TTT_OK;
}

bool aligned(const void* p, size_t n) { return (reinterpret_cast<uintptr_t>(p) % n) == 0; }

// A byte range [p, p + n) of one argument, for the overlap checks.
struct Span {
    const char* name;
    const void* p;
    size_t n;
};

bool overlaps(const Span& x, const Span& y) {
    if (!x.p || !y.p || x.n == 0 || y.n == 0) return false;
    auto a = reinterpret_cast<uintptr_t>(x.p), b = reinterpret_cast<uintptr_t>(y.p);
    return a < b + y.n && b < a + x.n;
}

// outputs must not overlap inputs or each other; `same_ok` lists (output, input) index pairs
// allowed to be the SAME buffer (identical pointer and size: an in-place state update).
int check_aliasing(const Span* in, int nin, const Span* out, int nout,
                   const int (*same_ok)[2] = nullptr, int nsame = 0) {
    for (int o = 0; o < nout; ++o) {
        for (int i = 0; i < nin; ++i) {
            if (!overlaps(out[o], in[i])) continue;
            bool allowed = false;
            for (int k = 0; k < nsame; ++k)
                if (same_ok[k][0] == o && same_ok[k][1] == i && out[o].p == in[i].p && out[o].n == in[i].n)
                    allowed = true;
            if (!allowed)
                return fail(TTT_ERR_ALIAS, "output %s overlaps input %s", out[o].name, in[i].name);
        }
        for (int p = o + 1; p < nout; ++p)
            if (overlaps(out[o], out[p]))
                return fail(TTT_ERR_ALIAS, "outputs %s and %s overlap", out[o].name, out[p].name);
    }
    return TTT_OK;
}

unsigned int* status_word();  // device address of the status word of the current device

// polls per bounded device wait: the default, a caller's cap, or 0 polls (give up at once)
long long wait_limit() {
    long long v = g_wait_limit.load();
    return v == 0 ? kDefaultWaitPolls : (v < 0 ? 0 : v);
}

// ---- driver entry point for tensor-map encoding (no link-time libcuda dependency) ----------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// XQ / XK / XV (bf16) as a tensor map with 128-byte swizzle; out-of-range rows read 0.
// Head-major [B, H, L, 64]: 4-D dims {64, L, H, B}, box {64, K, 1, 1}, or (three_d) 3-D dims
// {64, L, B*H}, box {64, K, 1}.  Token-major [B, L, H, 64]: 4-D dims {64, H, L, B}, box {64, 1, K, 1}.
int encode_act_map(CUtensorMap* map, const void* base, int B, int H, long long L, int K, bool tok_major,
                   const char* name, bool three_d = false) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return fail(TTT_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    const cuuint64_t row = static_cast<cuuint64_t>(kD) * 2;  // bytes of one token of one head
    const cuuint64_t d1 = tok_major ? H : L, d2 = tok_major ? L : H;
    cuuint64_t dims[4] = {static_cast<cuuint64_t>(kD), d1, d2, static_cast<cuuint64_t>(B)};
    cuuint64_t strides[3] = {row, row * d1, row * d1 * d2};
    cuuint32_t box[4] = {static_cast<cuuint32_t>(kD), tok_major ? 1u : static_cast<cuuint32_t>(K),
                         tok_major ? static_cast<cuuint32_t>(K) : 1u, 1};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    cuuint32_t rank = 4;
    if (three_d && !tok_major) {  // chains (b, h) flattened: b * H + h
        rank = 3;
        dims[2] = static_cast<cuuint64_t>(B) * static_cast<cuuint64_t>(H);
    }
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TTT_ERR_CUDA, "tensor map for %s: cuTensorMapEncodeTiled error %d", name, (int)r);
    return TTT_OK;
}

// Element strides of the activations between batch rows, heads and tokens.
template <class Args>
void set_act_strides(Args& a, int H, long long L, bool tok_major) {
    const long long hd = static_cast<long long>(H) * kD;
    a.act_b = L * hd;
    a.act_h = tok_major ? kD : L * kD;
    a.act_t = tok_major ? hd : kD;
    a.tok_major = tok_major ? 1 : 0;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(TTT_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// Common checks of the prefill entry points.
int check_common(int B, int H, long long L, int d, int K, float eps, int dtype, unsigned int flags) {
    if (B < 1 || H < 1) return fail(TTT_ERR_ARG, "B and H must be >= 1 (got %d, %d)", B, H);
    if (static_cast<long long>(B) * H > (1ll << 31) - 1) return fail(TTT_ERR_ARG, "B*H too large");
    if (L < 0) return fail(TTT_ERR_ARG, "L must be >= 0 (got %lld)", L);
    if (L > (1ll << 31) - 1) return fail(TTT_ERR_ARG, "L too large (%lld)", L);
    if (d != kD) return fail(TTT_ERR_UNSUPPORTED, "only head dim d = 64 is supported (got %d)", d);
    if (K < 1 || K > 16) return fail(TTT_ERR_ARG, "mini_batch must be in [1, 16] (got %d)", K);
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(TTT_ERR_ARG, "eps must be finite and > 0");
    if (dtype != TTT_F32 && dtype != TTT_BF16) return fail(TTT_ERR_ARG, "dtype must be TTT_F32 or TTT_BF16");
    if (flags & ~(TTT_FLAG_FP32_COMPUTE | TTT_FLAG_TOKEN_MAJOR)) return fail(TTT_ERR_ARG, "unknown flags 0x%x", flags);
    return TTT_OK;
}

}  // namespace

// The status word.  Kernels OR TTT_STATUS_* bits into it; ttt_device_status reads it.  A read
// that clears takes the word with one atomic exchange into g_ttt_status_taken and copies that,
// so a bit raised by a kernel still running on another stream is never lost between the read
// and the clear.
__device__ unsigned int g_ttt_status;
__device__ unsigned int g_ttt_status_taken;

namespace {
__global__ void status_take_kernel(unsigned int* word, unsigned int* taken) { *taken = atomicExch(word, 0u); }

// Device address of a __device__ word on the current device (looked up once per device).
template <unsigned int& kSym>
unsigned int* device_word() {
    static std::mutex mu;
    static unsigned int* ptrs[256] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 256) return nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, kSym) != cudaSuccess) return nullptr;
        ptrs[dev] = static_cast<unsigned int*>(p);
    }
    return ptrs[dev];
}

unsigned int* status_word() { return device_word<g_ttt_status>(); }

// The launch part of ttt_linear_forward, on validated device pointers: pick the kernel, build
// its arguments (and tensor maps) and enqueue it on `st`.
int enqueue_linear(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                   const float* W0, const float* b0, long long w0_chain_stride, const float* ln_w, const float* ln_b,
                   int B, int H, long long L, int mini_batch, float eps, int dtype, unsigned int flags, void* out,
                   float* W_last, float* b_last, float* W_grad_tail, float* b_grad_tail, cudaStream_t st,
                   int rope = 0, float rope_theta = 0.f, float* ckpt = nullptr, int ckpt_group = 0) {
    int rc;
    ttt::LinearArgs a{};
    a.XQ = XQ; a.XK = XK; a.XV = XV; a.lr = lr; a.token_eta = token_eta;
    a.W0 = W0; a.b0 = b0; a.w0_chain_stride = w0_chain_stride;
    a.ln_w = ln_w; a.ln_b = ln_b; a.B = B; a.H = H; a.L = L; a.K = mini_batch;
    a.n_full = L / mini_batch; a.rem = L % mini_batch; a.eps = eps;
    a.out = out; a.W_last = W_last; a.b_last = b_last; a.W_grad_tail = W_grad_tail; a.b_grad_tail = b_grad_tail;
    a.status = status_word();
    a.wait_limit = wait_limit();
    a.rope = rope;
    a.rope_theta = rope_theta;
    a.ckpt = ckpt;
    a.ckpt_G = ckpt_group;
    a.ckpt_stride = ckpt ? (a.n_full + ckpt_group - 1) / ckpt_group + 1 : 0;
    const bool tm = (flags & TTT_FLAG_TOKEN_MAJOR) != 0;
    set_act_strides(a, H, L, tm);

    cudaError_t e;
    if (L == 0) {
        e = ttt::launch_linear_state_copy(a, st);
    } else if (dtype == TTT_F32 || (flags & TTT_FLAG_FP32_COMPUTE)) {
        e = ttt::launch_linear_simt(a, dtype, st);
    } else {
        ttt::LinearMaps maps;
        if ((rc = encode_act_map(&maps.xq, XQ, B, H, L, mini_batch, tm, "XQ", true))) return rc;
        if ((rc = encode_act_map(&maps.xk, XK, B, H, L, mini_batch, tm, "XK", true))) return rc;
        if ((rc = encode_act_map(&maps.xv, XV, B, H, L, mini_batch, tm, "XV", true))) return rc;
        e = ttt::launch_linear_tc(a, maps, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward launch");
    return ok();
}

// ---- host-buffer entry: one copy stream and a few events per device, created on first use ----
struct HostCtx {
    cudaStream_t copy = nullptr;
    cudaEvent_t start = nullptr, in[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
};
std::mutex g_host_mu;  // held while a host-buffer call enqueues (its events are shared per device)
HostCtx g_host_ctx[256];

int host_ctx(HostCtx** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 256) return fail(TTT_ERR_CUDA, "device index %d out of range", dev);
    HostCtx& c = g_host_ctx[dev];
    if (!c.copy) {
        if ((e = cudaStreamCreateWithFlags(&c.copy, cudaStreamNonBlocking)) != cudaSuccess)
            return cuda_fail(e, "creating the copy stream");
        cudaEvent_t* evs[5] = {&c.start, &c.in[0], &c.in[1], &c.freed[0], &c.freed[1]};
        for (cudaEvent_t* ev : evs)
            if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess)
                return cuda_fail(e, "creating an event");
    }
    *out = &c;
    return TTT_OK;
}

size_t up256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// Byte offsets inside the workspace of ttt_linear_forward_host.
struct HostLayout {
    size_t lnw, lnb, te, w0, b0;               // shared parameters (w0, b0: per head, when shared)
    size_t set;                                // offset of staging set 0; set 1 follows at set + set_bytes
    size_t set_bytes;
    size_t xq, xk, xv, lr, w0c, b0c, out, wl, bl, wg, bg;  // offsets inside a staging set
    size_t total;
};

HostLayout host_layout(int H, long long L, int K, int dtype, int chunk_batches, bool per_chain) {
    HostLayout y{};
    const size_t cc = static_cast<size_t>(chunk_batches) * H;  // chains per chunk
    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t act = cc * static_cast<size_t>(L) * kD * esz;
    const size_t st = static_cast<size_t>(kD) * kD * 4, sb = static_cast<size_t>(kD) * 4;
    size_t o = 0;
    y.lnw = o; o += up256(static_cast<size_t>(H) * sb);
    y.lnb = o; o += up256(static_cast<size_t>(H) * sb);
    y.te = o; o += up256(static_cast<size_t>(K) * 4);
    y.w0 = o; o += per_chain ? 0 : up256(static_cast<size_t>(H) * st);
    y.b0 = o; o += per_chain ? 0 : up256(static_cast<size_t>(H) * sb);
    y.set = o;
    size_t q = 0;
    y.xq = q; q += up256(act);
    y.xk = q; q += up256(act);
    y.xv = q; q += up256(act);
    y.lr = q; q += up256(cc * static_cast<size_t>(L) * 4);
    y.w0c = q; q += per_chain ? up256(cc * st) : 0;
    y.b0c = q; q += per_chain ? up256(cc * sb) : 0;
    y.out = q; q += up256(act);
    y.wl = q; q += up256(cc * st);
    y.bl = q; q += up256(cc * sb);
    y.wg = q; q += up256(cc * st);
    y.bg = q; q += up256(cc * sb);
    y.set_bytes = q;
    y.total = o + 2 * q;
    return y;
}
}  // namespace

extern "C" {

int ttt_partition(long long L, int mini_batch, long long* n_full, long long* rem) {
    if (!n_full || !rem) return fail(TTT_ERR_ARG, "n_full and rem must be non-null");
    if (L < 0) return fail(TTT_ERR_ARG, "L must be >= 0 (got %lld)", L);
    if (mini_batch < 1) return fail(TTT_ERR_ARG, "mini_batch must be >= 1 (got %d)", mini_batch);
    *n_full = L / mini_batch;
    *rem = L % mini_batch;
    return ok();
}

const char* ttt_error_string(int code) {
    switch (code) {
        case TTT_OK: return "ok";
        case TTT_ERR_ARG: return "invalid argument";
        case TTT_ERR_ALIGN: return "misaligned pointer";
        case TTT_ERR_ALIAS: return "output overlaps another buffer";
        case TTT_ERR_CUDA: return "CUDA error";
        case TTT_ERR_TIMEOUT: return "device-side wait timed out";
        case TTT_ERR_UNSUPPORTED: return "unsupported configuration";
        default: return "unknown error code";
    }
}

const char* ttt_last_error_message(void) { return g_last_error.c_str(); }

int ttt_set_wait_limit(long long polls) {
    g_wait_limit.store(polls);
    return ok();
}

int ttt_device_status(void* stream, unsigned int* status, int clear) {
    if (!status) return fail(TTT_ERR_ARG, "status must be non-null");
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    unsigned int* word = status_word();
    if (!word) return fail(TTT_ERR_CUDA, "no device status word on the current device");
    const unsigned int* src = word;
    cudaError_t e = cudaSuccess;
    if (clear) {  // read and clear in one atomic step on the device
        unsigned int* taken = device_word<g_ttt_status_taken>();
        if (!taken) return fail(TTT_ERR_CUDA, "no device status word on the current device");
        status_take_kernel<<<1, 1, 0, st>>>(word, taken);
        e = cudaGetLastError();
        src = taken;
    }
    unsigned int v = 0;
    if (e == cudaSuccess) e = cudaMemcpyAsync(&v, src, sizeof(v), cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    *status = v;
    if (v & TTT_STATUS_TIMEOUT) return fail(TTT_ERR_TIMEOUT, "a kernel gave up on a bounded wait");
    return ok();
}

// ttt_linear_forward and ttt_linear_forward_rope: checks on the device pointers, then the launch.
// rope: 0 none, 1 pairs (2k, 2k+1), 2 pairs (k, k + d/2); flags hold no rope bit here.
static int linear_forward_checked(const void* XQ, const void* XK, const void* XV, const float* lr,
                                  const float* token_eta, const float* W0, const float* b0,
                                  long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                                  long long L, int d, int mini_batch, float eps, int dtype, unsigned int flags,
                                  int rope, float rope_theta, void* out, float* W_last, float* b_last,
                                  float* W_grad_tail, float* b_grad_tail, void* stream, float* ckpt = nullptr,
                                  int ckpt_group = 0) {
    int rc = check_common(B, H, L, d, mini_batch, eps, dtype, flags);
    if (rc) return rc;
    if (ckpt && ckpt_group < 1) return fail(TTT_ERR_ARG, "ckpt_group must be >= 1 (got %d)", ckpt_group);
    if (ckpt && !aligned(ckpt, 16)) return fail(TTT_ERR_ALIGN, "ckpt must be 16-byte aligned");
    const long long chains = static_cast<long long>(B) * H;
    const long long per_head = static_cast<long long>(kD) * kD;
    if (w0_batch_stride != 0 && w0_batch_stride != H * per_head)
        return fail(TTT_ERR_ARG, "w0_batch_stride must be 0 or H*d*d (got %lld)", w0_batch_stride);
    if (!W0 || !b0 || !ln_w || !ln_b || !W_last || !b_last)
        return fail(TTT_ERR_ARG, "W0, b0, ln_w, ln_b, W_last and b_last must be non-null");
    if (L > 0 && (!XQ || !XK || !XV || !lr || !out))
        return fail(TTT_ERR_ARG, "XQ, XK, XV, lr and out must be non-null when L > 0");
    const void* a16[] = {XQ, XK, XV, out, W0, b0, W_last, b_last, W_grad_tail, b_grad_tail};
    const char* n16[] = {"XQ", "XK", "XV", "out", "W0", "b0", "W_last", "b_last", "W_grad_tail", "b_grad_tail"};
    for (int i = 0; i < 10; ++i)
        if (a16[i] && !aligned(a16[i], 16)) return fail(TTT_ERR_ALIGN, "%s must be 16-byte aligned", n16[i]);
    const void* a4[] = {lr, token_eta, ln_w, ln_b};
    const char* n4[] = {"lr", "token_eta", "ln_w", "ln_b"};
    for (int i = 0; i < 4; ++i)
        if (a4[i] && !aligned(a4[i], 4)) return fail(TTT_ERR_ALIGN, "%s must be 4-byte aligned", n4[i]);

    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t act = static_cast<size_t>(chains) * L * kD * esz;
    const long long wrows = w0_batch_stride ? chains : H;
    Span in[] = {{"XQ", XQ, act}, {"XK", XK, act}, {"XV", XV, act}, {"lr", lr, static_cast<size_t>(chains * L) * 4},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4},
                 {"W0", W0, static_cast<size_t>(wrows * per_head) * 4}, {"b0", b0, static_cast<size_t>(wrows * kD) * 4},
                 {"ln_w", ln_w, static_cast<size_t>(H) * kD * 4}, {"ln_b", ln_b, static_cast<size_t>(H) * kD * 4}};
    const size_t ckpt_bytes = ckpt ? static_cast<size_t>(chains) * ((L / mini_batch + ckpt_group - 1) / ckpt_group + 1) *
                                         (per_head + kD) * 4 : 0;
    Span outs[] = {{"out", out, act}, {"W_last", W_last, static_cast<size_t>(chains * per_head) * 4},
                   {"b_last", b_last, static_cast<size_t>(chains * kD) * 4},
                   {"W_grad_tail", W_grad_tail, static_cast<size_t>(chains * per_head) * 4},
                   {"b_grad_tail", b_grad_tail, static_cast<size_t>(chains * kD) * 4}, {"ckpt", ckpt, ckpt_bytes}};
    const int same_ok[2][2] = {{1, 5}, {2, 6}};  // W_last == W0, b_last == b0 (per-chain state)
    rc = check_aliasing(in, 9, outs, 6, same_ok, 2);
    if (rc) return rc;

    return enqueue_linear(XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride ? per_head : 0, ln_w, ln_b, B, H, L,
                          mini_batch, eps, dtype, flags, out, W_last, b_last, W_grad_tail, b_grad_tail,
                          static_cast<cudaStream_t>(stream), rope, rope_theta, ckpt, ckpt_group);
}

int ttt_linear_forward(const void* XQ, const void* XK, const void* XV, const float* lr,
                       const float* token_eta, const float* W0, const float* b0,
                       long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                       long long L, int d, int mini_batch, float eps, int dtype, unsigned int flags,
                       void* out, float* W_last, float* b_last, float* W_grad_tail,
                       float* b_grad_tail, void* stream) {
    return linear_forward_checked(XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride, ln_w, ln_b, B, H, L, d,
                                  mini_batch, eps, dtype, flags, 0, 0.f, out, W_last, b_last, W_grad_tail,
                                  b_grad_tail, stream);
}

long long ttt_linear_ckpt_bytes(int B, int H, long long L, int d, int mini_batch, int ckpt_group) {
    int rc = check_common(B, H, L, d, mini_batch, 1.0f, TTT_F32, 0);
    if (rc) return rc;
    if (ckpt_group < 1) return fail(TTT_ERR_ARG, "ckpt_group must be >= 1 (got %d)", ckpt_group);
    ok();
    const long long n_ckpt = (L / mini_batch + ckpt_group - 1) / ckpt_group;
    return static_cast<long long>(B) * H * (n_ckpt + 1) * (kD * kD + kD) * 4;
}

int ttt_linear_forward_ckpt(const void* XQ, const void* XK, const void* XV, const float* lr,
                            const float* token_eta, const float* W0, const float* b0,
                            long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                            long long L, int d, int mini_batch, float eps, int dtype, unsigned int flags,
                            void* out, float* W_last, float* b_last, float* W_grad_tail,
                            float* b_grad_tail, int ckpt_group, float* ckpt, void* stream) {
    if (!ckpt) return fail(TTT_ERR_ARG, "ckpt must be non-null");
    return linear_forward_checked(XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride, ln_w, ln_b, B, H, L, d,
                                  mini_batch, eps, dtype, flags, 0, 0.f, out, W_last, b_last, W_grad_tail,
                                  b_grad_tail, stream, ckpt, ckpt_group);
}

int ttt_linear_forward_rope(const void* XQ, const void* XK, const void* XV, const float* lr,
                            const float* token_eta, const float* W0, const float* b0,
                            long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                            long long L, int d, int mini_batch, float eps, float rope_theta, int dtype,
                            unsigned int flags, void* out, float* W_last, float* b_last, float* W_grad_tail,
                            float* b_grad_tail, void* stream) {
    if (!(rope_theta > 0.f) || !std::isfinite(rope_theta))
        return fail(TTT_ERR_ARG, "rope_theta must be finite and > 0");
    if (flags & TTT_FLAG_FP32_COMPUTE)
        return fail(TTT_ERR_UNSUPPORTED, "the rotary embedding runs on the tensor-core kernel only (no FP32_COMPUTE)");
    const unsigned int rest = flags & ~TTT_FLAG_ROPE_HALF_SPLIT;
    int rc = check_common(B, H, L, d, mini_batch, eps, dtype, rest);
    if (rc) return rc;
    if (dtype != TTT_BF16) return fail(TTT_ERR_UNSUPPORTED, "the rotary embedding takes bf16 activations only");
    return linear_forward_checked(XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride, ln_w, ln_b, B, H, L, d,
                                  mini_batch, eps, dtype, rest, (flags & TTT_FLAG_ROPE_HALF_SPLIT) ? 2 : 1,
                                  rope_theta, out, W_last, b_last, W_grad_tail, b_grad_tail, stream);
}

long long ttt_linear_host_workspace_bytes(int B, int H, long long L, int d, int mini_batch, int dtype,
                                          int chunk_batches, long long w0_batch_stride) {
    int rc = check_common(B, H, L, d, mini_batch, 1e-6f, dtype, 0);
    if (rc) return rc;
    if (chunk_batches < 1 || chunk_batches > B)
        return fail(TTT_ERR_ARG, "chunk_batches must be in [1, B] (got %d, B = %d)", chunk_batches, B);
    if (w0_batch_stride != 0 && w0_batch_stride != static_cast<long long>(H) * kD * kD)
        return fail(TTT_ERR_ARG, "w0_batch_stride must be 0 or H*d*d (got %lld)", w0_batch_stride);
    ok();
    return static_cast<long long>(host_layout(H, L, mini_batch, dtype, chunk_batches, w0_batch_stride != 0).total);
}

int ttt_linear_forward_host(const void* XQ, const void* XK, const void* XV, const float* lr,
                            const float* token_eta, const float* W0, const float* b0,
                            long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H,
                            long long L, int d, int mini_batch, float eps, int dtype, unsigned int flags,
                            void* out, float* W_last, float* b_last, float* W_grad_tail,
                            float* b_grad_tail, void* workspace, long long workspace_bytes,
                            int chunk_batches, void* stream) {
    int rc = check_common(B, H, L, d, mini_batch, eps, dtype, flags);
    if (rc) return rc;
    const long long per_head = static_cast<long long>(kD) * kD;
    const bool per_chain = w0_batch_stride != 0;
    if (per_chain && w0_batch_stride != H * per_head)
        return fail(TTT_ERR_ARG, "w0_batch_stride must be 0 or H*d*d (got %lld)", w0_batch_stride);
    if (!W0 || !b0 || !ln_w || !ln_b || !W_last || !b_last)
        return fail(TTT_ERR_ARG, "W0, b0, ln_w, ln_b, W_last and b_last must be non-null");
    if (L > 0 && (!XQ || !XK || !XV || !lr || !out))
        return fail(TTT_ERR_ARG, "XQ, XK, XV, lr and out must be non-null when L > 0");
    if (chunk_batches < 1 || chunk_batches > B)
        return fail(TTT_ERR_ARG, "chunk_batches must be in [1, B] (got %d, B = %d)", chunk_batches, B);
    if (!workspace) return fail(TTT_ERR_ARG, "workspace must be non-null");
    if (!aligned(workspace, 256)) return fail(TTT_ERR_ALIGN, "workspace must be 256-byte aligned");
    const HostLayout y = host_layout(H, L, mini_batch, dtype, chunk_batches, per_chain);
    if (workspace_bytes < static_cast<long long>(y.total))
        return fail(TTT_ERR_ARG, "workspace too small: %lld bytes, %lld needed", workspace_bytes,
                    static_cast<long long>(y.total));
    const long long chains = static_cast<long long>(B) * H;
    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t act = static_cast<size_t>(chains) * L * kD * esz;
    const long long wrows = per_chain ? chains : H;
    Span in[] = {{"XQ", XQ, act}, {"XK", XK, act}, {"XV", XV, act}, {"lr", lr, static_cast<size_t>(chains * L) * 4},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4},
                 {"W0", W0, static_cast<size_t>(wrows * per_head) * 4}, {"b0", b0, static_cast<size_t>(wrows * kD) * 4},
                 {"ln_w", ln_w, static_cast<size_t>(H) * kD * 4}, {"ln_b", ln_b, static_cast<size_t>(H) * kD * 4}};
    Span outs[] = {{"out", out, act}, {"W_last", W_last, static_cast<size_t>(chains * per_head) * 4},
                   {"b_last", b_last, static_cast<size_t>(chains * kD) * 4},
                   {"W_grad_tail", W_grad_tail, static_cast<size_t>(chains * per_head) * 4},
                   {"b_grad_tail", b_grad_tail, static_cast<size_t>(chains * kD) * 4}};
    const int same_ok[2][2] = {{1, 5}, {2, 6}};
    rc = check_aliasing(in, 9, outs, 5, same_ok, 2);
    if (rc) return rc;

    std::lock_guard<std::mutex> lock(g_host_mu);
    HostCtx* c = nullptr;
    if ((rc = host_ctx(&c))) return rc;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    char* ws = static_cast<char*>(workspace);
    const auto H2D = cudaMemcpyHostToDevice;
    const auto D2H = cudaMemcpyDeviceToHost;
    cudaError_t e = cudaEventRecord(c->start, st);  // the workspace is free once earlier work on st is done
    if (e == cudaSuccess) e = cudaStreamWaitEvent(c->copy, c->start, 0);
    // shared parameters
    const size_t hb = static_cast<size_t>(H) * kD * 4;
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + y.lnw, ln_w, hb, H2D, c->copy);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + y.lnb, ln_b, hb, H2D, c->copy);
    if (e == cudaSuccess && token_eta) e = cudaMemcpyAsync(ws + y.te, token_eta, static_cast<size_t>(mini_batch) * 4, H2D, c->copy);
    if (e == cudaSuccess && !per_chain) e = cudaMemcpyAsync(ws + y.w0, W0, static_cast<size_t>(H) * per_head * 4, H2D, c->copy);
    if (e == cudaSuccess && !per_chain) e = cudaMemcpyAsync(ws + y.b0, b0, hb, H2D, c->copy);
    if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward_host: parameters");

    const int n_chunks = (B + chunk_batches - 1) / chunk_batches;
    for (int ci = 0; ci < n_chunks; ++ci) {
        const int slot = ci & 1;
        const int bfirst = ci * chunk_batches;
        const int bc = (B - bfirst < chunk_batches) ? B - bfirst : chunk_batches;
        const size_t cc = static_cast<size_t>(bc) * H;                       // chains in this chunk
        const size_t c0 = static_cast<size_t>(bfirst) * H;                   // first chain
        const size_t a_off = c0 * static_cast<size_t>(L) * kD * esz, a_n = cc * static_cast<size_t>(L) * kD * esz;
        const size_t l_off = c0 * static_cast<size_t>(L) * 4, l_n = cc * static_cast<size_t>(L) * 4;
        const size_t s_off = c0 * per_head * 4, s_n = cc * per_head * 4;
        const size_t v_off = c0 * kD * 4, v_n = cc * kD * 4;
        char* set = ws + y.set + slot * y.set_bytes;
        // inputs of this chunk (once the kernel two chunks back has finished reading the set)
        if (ci >= 2) e = cudaStreamWaitEvent(c->copy, c->freed[slot], 0);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.xq, static_cast<const char*>(XQ) + a_off, a_n, H2D, c->copy);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.xk, static_cast<const char*>(XK) + a_off, a_n, H2D, c->copy);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.xv, static_cast<const char*>(XV) + a_off, a_n, H2D, c->copy);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.lr, reinterpret_cast<const char*>(lr) + l_off, l_n, H2D, c->copy);
        if (e == cudaSuccess && per_chain) e = cudaMemcpyAsync(set + y.w0c, reinterpret_cast<const char*>(W0) + s_off, s_n, H2D, c->copy);
        if (e == cudaSuccess && per_chain) e = cudaMemcpyAsync(set + y.b0c, reinterpret_cast<const char*>(b0) + v_off, v_n, H2D, c->copy);
        if (e == cudaSuccess) e = cudaEventRecord(c->in[slot], c->copy);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, c->in[slot], 0);
        if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward_host: inputs");
        // the scan of this chunk
        rc = enqueue_linear(set + y.xq, set + y.xk, set + y.xv, reinterpret_cast<const float*>(set + y.lr),
                            token_eta ? reinterpret_cast<const float*>(ws + y.te) : nullptr,
                            reinterpret_cast<const float*>(per_chain ? set + y.w0c : ws + y.w0),
                            reinterpret_cast<const float*>(per_chain ? set + y.b0c : ws + y.b0), per_chain ? per_head : 0,
                            reinterpret_cast<const float*>(ws + y.lnw), reinterpret_cast<const float*>(ws + y.lnb), bc, H,
                            L, mini_batch, eps, dtype, flags, set + y.out, reinterpret_cast<float*>(set + y.wl),
                            reinterpret_cast<float*>(set + y.bl), W_grad_tail ? reinterpret_cast<float*>(set + y.wg) : nullptr,
                            b_grad_tail ? reinterpret_cast<float*>(set + y.bg) : nullptr, st);
        if (rc) return rc;
        e = cudaEventRecord(c->freed[slot], st);
        // results of this chunk
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(static_cast<char*>(out) + a_off, set + y.out, a_n, D2H, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(reinterpret_cast<char*>(W_last) + s_off, set + y.wl, s_n, D2H, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(reinterpret_cast<char*>(b_last) + v_off, set + y.bl, v_n, D2H, st);
        if (e == cudaSuccess && W_grad_tail) e = cudaMemcpyAsync(reinterpret_cast<char*>(W_grad_tail) + s_off, set + y.wg, s_n, D2H, st);
        if (e == cudaSuccess && b_grad_tail) e = cudaMemcpyAsync(reinterpret_cast<char*>(b_grad_tail) + v_off, set + y.bg, v_n, D2H, st);
        if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward_host: outputs");
    }
    return ok();
}

int ttt_mlp_forward(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                    const float* W1_0, const float* b1_0, const float* W2_0, const float* b2_0,
                    long long w0_batch_stride, const float* ln_w, const float* ln_b, int B, int H, long long L,
                    int d, int hidden, int mini_batch, float eps, int dtype, unsigned int flags, void* out,
                    float* W1_last, float* b1_last, float* W2_last, float* b2_last, void* stream) {
    int rc = check_common(B, H, L, d, mini_batch, eps, dtype, flags);
    if (rc) return rc;
    if (hidden != kHidden) return fail(TTT_ERR_UNSUPPORTED, "only hidden = 256 is supported (got %d)", hidden);
    const long long chains = static_cast<long long>(B) * H;
    const long long per_head = static_cast<long long>(kD) * kHidden;
    if (w0_batch_stride != 0 && w0_batch_stride != H * per_head)
        return fail(TTT_ERR_ARG, "w0_batch_stride must be 0 or H*d*hidden (got %lld)", w0_batch_stride);
    if (!W1_0 || !b1_0 || !W2_0 || !b2_0 || !ln_w || !ln_b || !W1_last || !b1_last || !W2_last || !b2_last)
        return fail(TTT_ERR_ARG, "state, LayerNorm and state-output pointers must be non-null");
    if (L > 0 && (!XQ || !XK || !XV || !lr || !out))
        return fail(TTT_ERR_ARG, "XQ, XK, XV, lr and out must be non-null when L > 0");
    const void* a16[] = {XQ, XK, XV, out, W1_0, b1_0, W2_0, b2_0, W1_last, b1_last, W2_last, b2_last};
    for (int i = 0; i < 12; ++i)
        if (a16[i] && !aligned(a16[i], 16)) return fail(TTT_ERR_ALIGN, "tensor argument %d must be 16-byte aligned", i);
    const void* a4[] = {lr, token_eta, ln_w, ln_b};
    for (int i = 0; i < 4; ++i)
        if (a4[i] && !aligned(a4[i], 4)) return fail(TTT_ERR_ALIGN, "lr/token_eta/ln_w/ln_b must be 4-byte aligned");

    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t act = static_cast<size_t>(chains) * L * kD * esz;
    const long long rows = w0_batch_stride ? chains : H;
    Span in[] = {{"XQ", XQ, act}, {"XK", XK, act}, {"XV", XV, act}, {"lr", lr, static_cast<size_t>(chains * L) * 4},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4},
                 {"W1_0", W1_0, static_cast<size_t>(rows * per_head) * 4}, {"b1_0", b1_0, static_cast<size_t>(rows * kHidden) * 4},
                 {"W2_0", W2_0, static_cast<size_t>(rows * per_head) * 4}, {"b2_0", b2_0, static_cast<size_t>(rows * kD) * 4},
                 {"ln_w", ln_w, static_cast<size_t>(H) * kD * 4}, {"ln_b", ln_b, static_cast<size_t>(H) * kD * 4}};
    Span outs[] = {{"out", out, act}, {"W1_last", W1_last, static_cast<size_t>(chains * per_head) * 4},
                   {"b1_last", b1_last, static_cast<size_t>(chains * kHidden) * 4},
                   {"W2_last", W2_last, static_cast<size_t>(chains * per_head) * 4},
                   {"b2_last", b2_last, static_cast<size_t>(chains * kD) * 4}};
    const int same_ok[4][2] = {{1, 5}, {2, 6}, {3, 7}, {4, 8}};
    rc = check_aliasing(in, 11, outs, 5, same_ok, 4);
    if (rc) return rc;

    ttt::MlpArgs a{};
    a.XQ = XQ; a.XK = XK; a.XV = XV; a.lr = lr; a.token_eta = token_eta;
    a.W1_0 = W1_0; a.b1_0 = b1_0; a.W2_0 = W2_0; a.b2_0 = b2_0;
    a.w0_chain_stride = w0_batch_stride ? per_head : 0;
    a.ln_w = ln_w; a.ln_b = ln_b; a.B = B; a.H = H; a.L = L; a.K = mini_batch;
    a.n_full = L / mini_batch; a.rem = L % mini_batch; a.eps = eps; a.out = out;
    a.W1_last = W1_last; a.b1_last = b1_last; a.W2_last = W2_last; a.b2_last = b2_last;
    a.status = status_word();
    a.wait_limit = wait_limit();
    const bool tm = (flags & TTT_FLAG_TOKEN_MAJOR) != 0;
    set_act_strides(a, H, L, tm);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (L == 0) {
        e = ttt::launch_mlp_state_copy(a, st);
    } else if (dtype == TTT_F32 || (flags & TTT_FLAG_FP32_COMPUTE)) {
        e = ttt::launch_mlp_simt(a, dtype, st);
    } else {
        ttt::LinearMaps maps;
        if ((rc = encode_act_map(&maps.xq, XQ, B, H, L, mini_batch, tm, "XQ"))) return rc;
        if ((rc = encode_act_map(&maps.xk, XK, B, H, L, mini_batch, tm, "XK"))) return rc;
        if ((rc = encode_act_map(&maps.xv, XV, B, H, L, mini_batch, tm, "XV"))) return rc;
        e = ttt::launch_mlp_tc(a, maps, st);
    }
    if (e != cudaSuccess) return cuda_fail(e, "ttt_mlp_forward launch");
    return ok();
}

int ttt_linear_decode_step(const void* xq, const void* xk, const void* xv, const float* lr,
                           const float* token_eta, const float* ln_w, const float* ln_b, float* W, float* b,
                           float* W_grad, float* b_grad, int B, int H, int d, int mini_batch,
                           long long seqlen_offset, float eps, int dtype, void* out, void* stream) {
    int rc = check_common(B, H, 1, d, mini_batch, eps, dtype, 0);
    if (rc) return rc;
    if (seqlen_offset < 0) return fail(TTT_ERR_ARG, "seqlen_offset must be >= 0");
    if (!xq || !xk || !xv || !lr || !ln_w || !ln_b || !W || !b || !W_grad || !b_grad || !out)
        return fail(TTT_ERR_ARG, "all tensor arguments except token_eta must be non-null");
    const void* a16[] = {xq, xk, xv, out, W, b, W_grad, b_grad};
    for (int i = 0; i < 8; ++i)
        if (!aligned(a16[i], 16)) return fail(TTT_ERR_ALIGN, "tensor argument %d must be 16-byte aligned", i);
    const void* a4[] = {lr, token_eta, ln_w, ln_b};
    for (int i = 0; i < 4; ++i)
        if (a4[i] && !aligned(a4[i], 4)) return fail(TTT_ERR_ALIGN, "lr/token_eta/ln_w/ln_b must be 4-byte aligned");
    const long long chains = static_cast<long long>(B) * H;
    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t vec = static_cast<size_t>(chains) * kD * esz;
    const size_t mat = static_cast<size_t>(chains) * kD * kD * 4, bv = static_cast<size_t>(chains) * kD * 4;
    Span in[] = {{"xq", xq, vec}, {"xk", xk, vec}, {"xv", xv, vec}, {"lr", lr, static_cast<size_t>(chains) * 4},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4},
                 {"ln_w", ln_w, static_cast<size_t>(H) * kD * 4}, {"ln_b", ln_b, static_cast<size_t>(H) * kD * 4}};
    Span outs[] = {{"out", out, vec}, {"W", W, mat}, {"b", b, bv}, {"W_grad", W_grad, mat}, {"b_grad", b_grad, bv}};
    rc = check_aliasing(in, 7, outs, 5);
    if (rc) return rc;

    ttt::DecodeArgs a{};
    a.xq = xq; a.xk = xk; a.xv = xv; a.lr = lr; a.token_eta = token_eta; a.ln_w = ln_w; a.ln_b = ln_b;
    a.W = W; a.b = b; a.W_grad = W_grad; a.b_grad = b_grad; a.B = B; a.H = H; a.K = mini_batch;
    a.p = static_cast<int>(seqlen_offset % mini_batch); a.eps = eps; a.out = out;
    a.status = status_word();
    a.wait_limit = wait_limit();
    cudaError_t e = ttt::launch_decode(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_decode_step launch");
    return ok();
}

int ttt_linear_decode_step_hist(const void* xq, const void* xk, const void* xv, const float* lr,
                                const float* token_eta, const float* ln_w, const float* ln_b, float* W, float* b,
                                float* hist, float* b_grad, int B, int H, int d, int mini_batch,
                                long long seqlen_offset, float eps, int dtype, void* out, void* stream) {
    int rc = check_common(B, H, 1, d, mini_batch, eps, dtype, 0);
    if (rc) return rc;
    if (seqlen_offset < 0) return fail(TTT_ERR_ARG, "seqlen_offset must be >= 0");
    if (!xq || !xk || !xv || !lr || !ln_w || !ln_b || !W || !b || !hist || !b_grad || !out)
        return fail(TTT_ERR_ARG, "all tensor arguments except token_eta must be non-null");
    const void* a16[] = {xq, xk, xv, out, W, b, hist, b_grad};
    for (int i = 0; i < 8; ++i)
        if (!aligned(a16[i], 16)) return fail(TTT_ERR_ALIGN, "tensor argument %d must be 16-byte aligned", i);
    const void* a4[] = {lr, token_eta, ln_w, ln_b};
    for (int i = 0; i < 4; ++i)
        if (a4[i] && !aligned(a4[i], 4)) return fail(TTT_ERR_ALIGN, "lr/token_eta/ln_w/ln_b must be 4-byte aligned");
    const long long chains = static_cast<long long>(B) * H;
    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t vec = static_cast<size_t>(chains) * kD * esz;
    const size_t mat = static_cast<size_t>(chains) * kD * kD * 4, bv = static_cast<size_t>(chains) * kD * 4;
    const size_t hv = static_cast<size_t>(chains) * mini_batch * 2 * kD * 4;
    Span in[] = {{"xq", xq, vec}, {"xk", xk, vec}, {"xv", xv, vec}, {"lr", lr, static_cast<size_t>(chains) * 4},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4},
                 {"ln_w", ln_w, static_cast<size_t>(H) * kD * 4}, {"ln_b", ln_b, static_cast<size_t>(H) * kD * 4}};
    Span outs[] = {{"out", out, vec}, {"W", W, mat}, {"b", b, bv}, {"hist", hist, hv}, {"b_grad", b_grad, bv}};
    rc = check_aliasing(in, 7, outs, 5);
    if (rc) return rc;

    ttt::DecodeHistArgs a{};
    a.xq = xq; a.xk = xk; a.xv = xv; a.lr = lr; a.token_eta = token_eta; a.ln_w = ln_w; a.ln_b = ln_b;
    a.W = W; a.b = b; a.hist = hist; a.b_grad = b_grad; a.B = B; a.H = H; a.K = mini_batch;
    a.p = static_cast<int>(seqlen_offset % mini_batch); a.eps = eps; a.out = out;
    a.status = status_word();
    a.wait_limit = wait_limit();
    cudaError_t e = ttt::launch_decode_hist(a, dtype, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_decode_step_hist launch");
    return ok();
}

// ---- the layer's output side: post_norm + o_proj ---------------------------------------------
static int check_oproj_sizes(int C, int N) {
    if (C < 64 || C % 64 != 0) return fail(TTT_ERR_UNSUPPORTED, "C must be a positive multiple of 64 (got %d)", C);
    if (N < 256 || N % 256 != 0) return fail(TTT_ERR_UNSUPPORTED, "N must be a positive multiple of 256 (got %d)", N);
    if (static_cast<long long>(C) * N > (1ll << 31) - 1) return fail(TTT_ERR_ARG, "C*N too large");
    return TTT_OK;
}

int ttt_o_proj_prepare(const void* Wo, const float* ln_w, const float* ln_b, int C, int N, void* Wp, float* u,
                       float* v, void* stream) {
    int rc = check_oproj_sizes(C, N);
    if (rc) return rc;
    if (!Wo || !ln_w || !ln_b || !Wp || !u || !v) return fail(TTT_ERR_ARG, "every pointer must be non-null");
    if (!aligned(Wo, 16) || !aligned(Wp, 16)) return fail(TTT_ERR_ALIGN, "Wo and Wp must be 16-byte aligned");
    const void* a4[] = {ln_w, ln_b, u, v};
    const char* n4[] = {"ln_w", "ln_b", "u", "v"};
    for (int i = 0; i < 4; ++i)
        if (!aligned(a4[i], 4)) return fail(TTT_ERR_ALIGN, "%s must be 4-byte aligned", n4[i]);
    const size_t w = static_cast<size_t>(C) * N * 2;
    Span in[] = {{"Wo", Wo, w}, {"ln_w", ln_w, static_cast<size_t>(C) * 4}, {"ln_b", ln_b, static_cast<size_t>(C) * 4}};
    Span outs[] = {{"Wp", Wp, w}, {"u", u, static_cast<size_t>(N) * 4}, {"v", v, static_cast<size_t>(N) * 4}};
    if ((rc = check_aliasing(in, 3, outs, 3))) return rc;
    cudaError_t e = ttt::launch_oproj_prepare(Wo, ln_w, ln_b, C, N, Wp, u, v, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ttt_o_proj_prepare launch");
    return ok();
}

// A [rows][cols] bf16 matrix as a 2-D tensor map with 128-byte swizzle and a {64, box_rows} box.
static int encode_rows_map(CUtensorMap* map, const void* base, long long rows, int cols, int box_rows,
                           const char* name) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return fail(TTT_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(TTT_ERR_CUDA, "tensor map for %s: cuTensorMapEncodeTiled error %d", name, (int)r);
    return TTT_OK;
}

int ttt_post_norm_o_proj(const void* X, long long T, int C, const void* Wp, const float* u, const float* v, int N,
                         float eps, void* Y, float* row_stats, void* stream) {
    int rc = check_oproj_sizes(C, N);
    if (rc) return rc;
    if (T < 0) return fail(TTT_ERR_ARG, "T must be >= 0 (got %lld)", T);
    if (T > 65535ll * 128) return fail(TTT_ERR_UNSUPPORTED, "T above 65535 * 128 tokens (got %lld)", T);
    if (!(eps > 0.f) || !std::isfinite(eps)) return fail(TTT_ERR_ARG, "eps must be finite and > 0");
    if (!Wp || !u || !v) return fail(TTT_ERR_ARG, "Wp, u and v must be non-null");
    if (T > 0 && (!X || !Y || !row_stats)) return fail(TTT_ERR_ARG, "X, Y and row_stats must be non-null when T > 0");
    const void* a16[] = {X, Wp, Y};
    const char* n16[] = {"X", "Wp", "Y"};
    for (int i = 0; i < 3; ++i)
        if (a16[i] && !aligned(a16[i], 16)) return fail(TTT_ERR_ALIGN, "%s must be 16-byte aligned", n16[i]);
    if (!aligned(u, 4) || !aligned(v, 4)) return fail(TTT_ERR_ALIGN, "u and v must be 4-byte aligned");
    if (row_stats && !aligned(row_stats, 8)) return fail(TTT_ERR_ALIGN, "row_stats must be 8-byte aligned");
    Span in[] = {{"X", X, static_cast<size_t>(T) * C * 2}, {"Wp", Wp, static_cast<size_t>(C) * N * 2},
                 {"u", u, static_cast<size_t>(N) * 4}, {"v", v, static_cast<size_t>(N) * 4}};
    Span outs[] = {{"Y", Y, static_cast<size_t>(T) * N * 2}, {"row_stats", row_stats, static_cast<size_t>(T) * 8}};
    if ((rc = check_aliasing(in, 4, outs, 2))) return rc;
    if (T == 0) return ok();
    ttt::OprojMaps maps;
    if ((rc = encode_rows_map(&maps.x, X, T, C, 128, "X"))) return rc;
    if ((rc = encode_rows_map(&maps.w, Wp, N, C, 256, "Wp"))) return rc;
    ttt::OprojArgs a{};
    a.T = T; a.C = C; a.N = N; a.eps = eps; a.u = u; a.v = v; a.X = X; a.stats = reinterpret_cast<float2*>(row_stats);
    a.Y = Y;
    a.status = status_word();
    a.wait_limit = wait_limit();
    cudaError_t e = ttt::launch_post_norm_oproj(a, maps, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "ttt_post_norm_o_proj launch");
    return ok();
}

// ---- the backward of the TTT-Linear scan -------------------------------------------------------
// Workspace: [chains][n_ckpt] kept states, [chains][G] rebuilt states, [chains] gradient shares.
struct BwdLayout {
    long long n_ckpt;
    size_t slab, part, total;
};

static BwdLayout bwd_layout(int B, int H, long long L, int K, int G) {
    const long long chains = static_cast<long long>(B) * H;
    const long long n_full = L / K;
    const size_t state = static_cast<size_t>(kD * kD + kD) * 4;
    BwdLayout y;
    y.n_ckpt = (n_full + G - 1) / G;
    y.slab = up256(static_cast<size_t>(chains * y.n_ckpt) * state);
    y.part = y.slab + up256(static_cast<size_t>(chains) * G * state);
    y.total = y.part + up256(static_cast<size_t>(chains) * (kD * kD + 3 * kD) * 4);
    return y;
}

long long ttt_linear_backward_workspace_bytes(int B, int H, long long L, int d, int mini_batch, int ckpt_group) {
    int rc = check_common(B, H, L, d, mini_batch, 1.0f, TTT_F32, 0);
    if (rc) return rc;
    if (ckpt_group < 1) return fail(TTT_ERR_ARG, "ckpt_group must be >= 1 (got %d)", ckpt_group);
    ok();
    return static_cast<long long>(bwd_layout(B, H, L, mini_batch, ckpt_group).total);
}

// ttt_linear_backward and ttt_linear_backward_ckpt (ckpt_in: the forward's checkpoints, or null).
static int linear_backward_impl(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                                const float* W0, const float* b0, long long w0_batch_stride, const float* ln_w,
                                const float* ln_b, int B, int H, long long L, int d, int mini_batch, float eps,
                                int dtype, unsigned int flags, int ckpt_group, const float* ckpt_in,
                                const void* d_out, const float* dW_last, const float* db_last, void* dXQ, void* dXK,
                                void* dXV, float* d_lr, float* dW0, float* db0, float* d_ln_w, float* d_ln_b,
                                void* workspace, long long workspace_bytes, void* stream) {
    int rc = check_common(B, H, L, d, mini_batch, eps, dtype, flags);
    if (rc) return rc;
    if (flags & TTT_FLAG_FP32_COMPUTE)
        return fail(TTT_ERR_UNSUPPORTED, "the backward takes no TTT_FLAG_FP32_COMPUTE (fp32 activations run in fp32)");
    if (ckpt_group < 1) return fail(TTT_ERR_ARG, "ckpt_group must be >= 1 (got %d)", ckpt_group);
    const long long chains = static_cast<long long>(B) * H;
    const long long per_head = static_cast<long long>(kD) * kD;
    if (w0_batch_stride != 0 && w0_batch_stride != H * per_head)
        return fail(TTT_ERR_ARG, "w0_batch_stride must be 0 or H*d*d (got %lld)", w0_batch_stride);
    if (!W0 || !b0 || !ln_w || !ln_b || !dW0 || !db0 || !d_ln_w || !d_ln_b || !workspace)
        return fail(TTT_ERR_ARG, "W0, b0, ln_w, ln_b, dW0, db0, d_ln_w, d_ln_b and workspace must be non-null");
    if (L > 0 && (!XQ || !XK || !XV || !lr || !d_out || !dXQ || !dXK || !dXV || !d_lr))
        return fail(TTT_ERR_ARG, "XQ, XK, XV, lr, d_out, dXQ, dXK, dXV and d_lr must be non-null when L > 0");
    const void* a16[] = {XQ, XK, XV, d_out, dXQ, dXK, dXV, W0, b0, dW_last, db_last, dW0, db0, ckpt_in};
    const char* n16[] = {"XQ", "XK", "XV", "d_out", "dXQ", "dXK", "dXV", "W0", "b0", "dW_last", "db_last", "dW0", "db0",
                         "ckpt"};
    for (int i = 0; i < 14; ++i)
        if (a16[i] && !aligned(a16[i], 16)) return fail(TTT_ERR_ALIGN, "%s must be 16-byte aligned", n16[i]);
    const void* a4[] = {lr, token_eta, ln_w, ln_b, d_lr, d_ln_w, d_ln_b};
    const char* n4[] = {"lr", "token_eta", "ln_w", "ln_b", "d_lr", "d_ln_w", "d_ln_b"};
    for (int i = 0; i < 7; ++i)
        if (a4[i] && !aligned(a4[i], 4)) return fail(TTT_ERR_ALIGN, "%s must be 4-byte aligned", n4[i]);
    if (!aligned(workspace, 256)) return fail(TTT_ERR_ALIGN, "workspace must be 256-byte aligned");
    const BwdLayout lay = bwd_layout(B, H, L, mini_batch, ckpt_group);
    if (workspace_bytes < 0 || static_cast<size_t>(workspace_bytes) < lay.total)
        return fail(TTT_ERR_ARG, "workspace_bytes %lld below the %zu bytes needed", workspace_bytes, lay.total);

    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t act = static_cast<size_t>(chains) * L * kD * esz;
    const size_t tok = static_cast<size_t>(chains * L) * 4;
    const long long wrows = w0_batch_stride ? chains : H;
    const size_t wbytes = static_cast<size_t>(wrows * per_head) * 4, bbytes = static_cast<size_t>(wrows * kD) * 4;
    const size_t hbytes = static_cast<size_t>(H) * kD * 4;
    Span in[] = {{"XQ", XQ, act}, {"XK", XK, act}, {"XV", XV, act}, {"lr", lr, tok},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4}, {"W0", W0, wbytes}, {"b0", b0, bbytes},
                 {"ln_w", ln_w, hbytes}, {"ln_b", ln_b, hbytes}, {"d_out", d_out, act},
                 {"dW_last", dW_last, static_cast<size_t>(chains * per_head) * 4},
                 {"db_last", db_last, static_cast<size_t>(chains * kD) * 4},
                 {"ckpt", ckpt_in, ckpt_in ? static_cast<size_t>(chains) * (lay.n_ckpt + 1) * (per_head + kD) * 4 : 0}};
    Span outs[] = {{"dXQ", dXQ, act}, {"dXK", dXK, act}, {"dXV", dXV, act}, {"d_lr", d_lr, tok},
                   {"dW0", dW0, wbytes}, {"db0", db0, bbytes}, {"d_ln_w", d_ln_w, hbytes}, {"d_ln_b", d_ln_b, hbytes},
                   {"workspace", workspace, lay.total}};
    rc = check_aliasing(in, 13, outs, 9);
    if (rc) return rc;

    ttt::LinearBwdArgs a{};
    a.XQ = XQ; a.XK = XK; a.XV = XV; a.d_out = d_out;
    a.lr = lr; a.token_eta = token_eta; a.W0 = W0; a.b0 = b0;
    a.w0_chain_stride = w0_batch_stride ? per_head : 0;
    a.ln_w = ln_w; a.ln_b = ln_b; a.dW_last = dW_last; a.db_last = db_last;
    a.B = B; a.H = H; a.K = mini_batch;
    a.L = L; a.n_full = L / mini_batch; a.rem = L % mini_batch;
    const bool tok_major = (flags & TTT_FLAG_TOKEN_MAJOR) != 0;
    a.act_b = static_cast<long long>(H) * L * kD;
    a.act_h = tok_major ? kD : L * kD;
    a.act_t = tok_major ? static_cast<long long>(H) * kD : kD;
    a.eps = eps; a.G = ckpt_group; a.n_ckpt = lay.n_ckpt;
    a.dXQ = dXQ; a.dXK = dXK; a.dXV = dXV; a.d_lr = d_lr;
    char* ws = static_cast<char*>(workspace);
    a.ckpt = ckpt_in ? const_cast<float*>(ckpt_in) : reinterpret_cast<float*>(ws);  // (read only when given)
    a.ckpt_stride = ckpt_in ? lay.n_ckpt + 1 : lay.n_ckpt;
    a.ckpt_given = ckpt_in ? 1 : 0;
    a.slab = reinterpret_cast<float*>(ws + lay.slab);
    a.part = reinterpret_cast<float*>(ws + lay.part);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    cudaError_t e = ttt::launch_linear_bwd(a, dtype, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward launch");
    e = ttt::launch_linear_bwd_reduce(a.part, B, H, w0_batch_stride ? 1 : 0, dW0, db0, d_ln_w, d_ln_b, st);
    if (e != cudaSuccess) return cuda_fail(e, "backward reduction launch");
    return ok();
}

int ttt_linear_backward(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                        const float* W0, const float* b0, long long w0_batch_stride, const float* ln_w,
                        const float* ln_b, int B, int H, long long L, int d, int mini_batch, float eps, int dtype,
                        unsigned int flags, int ckpt_group, const void* d_out, const float* dW_last,
                        const float* db_last, void* dXQ, void* dXK, void* dXV, float* d_lr, float* dW0, float* db0,
                        float* d_ln_w, float* d_ln_b, void* workspace, long long workspace_bytes, void* stream) {
    return linear_backward_impl(XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride, ln_w, ln_b, B, H, L, d,
                                mini_batch, eps, dtype, flags, ckpt_group, nullptr, d_out, dW_last, db_last, dXQ, dXK,
                                dXV, d_lr, dW0, db0, d_ln_w, d_ln_b, workspace, workspace_bytes, stream);
}

int ttt_linear_backward_ckpt(const void* XQ, const void* XK, const void* XV, const float* lr, const float* token_eta,
                             const float* W0, const float* b0, long long w0_batch_stride, const float* ln_w,
                             const float* ln_b, int B, int H, long long L, int d, int mini_batch, float eps,
                             int dtype, unsigned int flags, int ckpt_group, const float* ckpt, const void* d_out,
                             const float* dW_last, const float* db_last, void* dXQ, void* dXK, void* dXV,
                             float* d_lr, float* dW0, float* db0, float* d_ln_w, float* d_ln_b, void* workspace,
                             long long workspace_bytes, void* stream) {
    if (!ckpt) return fail(TTT_ERR_ARG, "ckpt must be non-null");
    return linear_backward_impl(XQ, XK, XV, lr, token_eta, W0, b0, w0_batch_stride, ln_w, ln_b, B, H, L, d,
                                mini_batch, eps, dtype, flags, ckpt_group, ckpt, d_out, dW_last, db_last, dXQ, dXK,
                                dXV, d_lr, dW0, db0, d_ln_w, d_ln_b, workspace, workspace_bytes, stream);
}

}  // extern "C"

// ---- host-buffer entry that allocates nothing ---------------------------------------------------
// The device scratch of ttt_linear_forward_host_static: one array per device that loads this
// library, held until the process exits.  In host code its name is only a host-side stand-in;
// the device address comes from cudaGetSymbolAddress, looked up once per device with that
// device current.
static __device__ __align__(256) unsigned char g_static_scratch[TTT_STATIC_SCRATCH_BYTES];

namespace {
int static_scratch(char** out) {
    static std::mutex mu;
    static char* ptrs[256] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 256) return fail(TTT_ERR_CUDA, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (!ptrs[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress of the built-in scratch");
        ptrs[dev] = static_cast<char*>(p);
    }
    *out = ptrs[dev];
    return TTT_OK;
}

// Bytes of scratch for chunks of `cb` batch rows: the shared parameters and one staging set.
size_t static_need(int H, long long L, int K, int dtype, int cb, bool per_chain) {
    const HostLayout y = host_layout(H, L, K, dtype, cb, per_chain);
    return y.set + y.set_bytes;
}
}  // namespace

extern "C" int ttt_linear_forward_host_static(const void* XQ, const void* XK, const void* XV, const float* lr,
                                              const float* token_eta, const float* W0, const float* b0,
                                              long long w0_batch_stride, const float* ln_w, const float* ln_b, int B,
                                              int H, long long L, int d, int mini_batch, float eps, int dtype,
                                              unsigned int flags, void* out, float* W_last, float* b_last,
                                              float* W_grad_tail, float* b_grad_tail, void* stream) {
    int rc = check_common(B, H, L, d, mini_batch, eps, dtype, flags);
    if (rc) return rc;
    const long long per_head = static_cast<long long>(kD) * kD;
    const bool per_chain = w0_batch_stride != 0;
    if (per_chain && w0_batch_stride != H * per_head)
        return fail(TTT_ERR_ARG, "w0_batch_stride must be 0 or H*d*d (got %lld)", w0_batch_stride);
    if (!W0 || !b0 || !ln_w || !ln_b || !W_last || !b_last)
        return fail(TTT_ERR_ARG, "W0, b0, ln_w, ln_b, W_last and b_last must be non-null");
    if (L > 0 && (!XQ || !XK || !XV || !lr || !out))
        return fail(TTT_ERR_ARG, "XQ, XK, XV, lr and out must be non-null when L > 0");
    // the largest chunk of batch rows whose staging fits the built-in scratch
    const size_t cap = static_cast<size_t>(TTT_STATIC_SCRATCH_BYTES);
    if (static_need(H, L, mini_batch, dtype, 1, per_chain) > cap)
        return fail(TTT_ERR_ARG,
                    "one batch row needs %zu bytes of staging; the built-in scratch holds %zu "
                    "(use ttt_linear_forward_host with a workspace of your own)",
                    static_need(H, L, mini_batch, dtype, 1, per_chain), cap);
    int lo = 1, hi = B;
    while (lo < hi) {
        const int mid = lo + (hi - lo + 1) / 2;
        if (static_need(H, L, mini_batch, dtype, mid, per_chain) <= cap) lo = mid; else hi = mid - 1;
    }
    const int cb = lo;
    const long long chains = static_cast<long long>(B) * H;
    const size_t esz = dtype == TTT_F32 ? 4 : 2;
    const size_t act = static_cast<size_t>(chains) * L * kD * esz;
    const long long wrows = per_chain ? chains : H;
    Span in[] = {{"XQ", XQ, act}, {"XK", XK, act}, {"XV", XV, act}, {"lr", lr, static_cast<size_t>(chains * L) * 4},
                 {"token_eta", token_eta, static_cast<size_t>(mini_batch) * 4},
                 {"W0", W0, static_cast<size_t>(wrows * per_head) * 4}, {"b0", b0, static_cast<size_t>(wrows * kD) * 4},
                 {"ln_w", ln_w, static_cast<size_t>(H) * kD * 4}, {"ln_b", ln_b, static_cast<size_t>(H) * kD * 4}};
    Span outs[] = {{"out", out, act}, {"W_last", W_last, static_cast<size_t>(chains * per_head) * 4},
                   {"b_last", b_last, static_cast<size_t>(chains * kD) * 4},
                   {"W_grad_tail", W_grad_tail, static_cast<size_t>(chains * per_head) * 4},
                   {"b_grad_tail", b_grad_tail, static_cast<size_t>(chains * kD) * 4}};
    const int same_ok[2][2] = {{1, 5}, {2, 6}};
    rc = check_aliasing(in, 9, outs, 5, same_ok, 2);
    if (rc) return rc;

    char* ws = nullptr;
    if ((rc = static_scratch(&ws))) return rc;
    const HostLayout y = host_layout(H, L, mini_batch, dtype, cb, per_chain);
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const auto H2D = cudaMemcpyHostToDevice;
    const auto D2H = cudaMemcpyDeviceToHost;
    // Every byte a call reads from the scratch was written earlier in the same call (parameters,
    // then per chunk the inputs by copies and the outputs by the kernels), so nothing needs
    // clearing.  Everything runs on `stream`, in order.
    const size_t hb = static_cast<size_t>(H) * kD * 4;
    cudaError_t e = cudaMemcpyAsync(ws + y.lnw, ln_w, hb, H2D, st);
    if (e == cudaSuccess) e = cudaMemcpyAsync(ws + y.lnb, ln_b, hb, H2D, st);
    if (e == cudaSuccess && token_eta) e = cudaMemcpyAsync(ws + y.te, token_eta, static_cast<size_t>(mini_batch) * 4, H2D, st);
    if (e == cudaSuccess && !per_chain) e = cudaMemcpyAsync(ws + y.w0, W0, static_cast<size_t>(H) * per_head * 4, H2D, st);
    if (e == cudaSuccess && !per_chain) e = cudaMemcpyAsync(ws + y.b0, b0, hb, H2D, st);
    if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward_host_static: parameters");
    char* set = ws + y.set;
    for (int bfirst = 0; bfirst < B; bfirst += cb) {
        const int bc = (B - bfirst < cb) ? B - bfirst : cb;
        const size_t cc = static_cast<size_t>(bc) * H, c0 = static_cast<size_t>(bfirst) * H;
        const size_t a_off = c0 * static_cast<size_t>(L) * kD * esz, a_n = cc * static_cast<size_t>(L) * kD * esz;
        const size_t l_off = c0 * static_cast<size_t>(L) * 4, l_n = cc * static_cast<size_t>(L) * 4;
        const size_t s_off = c0 * per_head * 4, s_n = cc * per_head * 4;
        const size_t v_off = c0 * kD * 4, v_n = cc * kD * 4;
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.xq, static_cast<const char*>(XQ) + a_off, a_n, H2D, st);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.xk, static_cast<const char*>(XK) + a_off, a_n, H2D, st);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.xv, static_cast<const char*>(XV) + a_off, a_n, H2D, st);
        if (e == cudaSuccess && L > 0) e = cudaMemcpyAsync(set + y.lr, reinterpret_cast<const char*>(lr) + l_off, l_n, H2D, st);
        if (e == cudaSuccess && per_chain) e = cudaMemcpyAsync(set + y.w0c, reinterpret_cast<const char*>(W0) + s_off, s_n, H2D, st);
        if (e == cudaSuccess && per_chain) e = cudaMemcpyAsync(set + y.b0c, reinterpret_cast<const char*>(b0) + v_off, v_n, H2D, st);
        if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward_host_static: inputs");
        rc = enqueue_linear(set + y.xq, set + y.xk, set + y.xv, reinterpret_cast<const float*>(set + y.lr),
                            token_eta ? reinterpret_cast<const float*>(ws + y.te) : nullptr,
                            reinterpret_cast<const float*>(per_chain ? set + y.w0c : ws + y.w0),
                            reinterpret_cast<const float*>(per_chain ? set + y.b0c : ws + y.b0), per_chain ? per_head : 0,
                            reinterpret_cast<const float*>(ws + y.lnw), reinterpret_cast<const float*>(ws + y.lnb), bc, H,
                            L, mini_batch, eps, dtype, flags, set + y.out, reinterpret_cast<float*>(set + y.wl),
                            reinterpret_cast<float*>(set + y.bl), W_grad_tail ? reinterpret_cast<float*>(set + y.wg) : nullptr,
                            b_grad_tail ? reinterpret_cast<float*>(set + y.bg) : nullptr, st);
        if (rc) return rc;
        if (L > 0) e = cudaMemcpyAsync(static_cast<char*>(out) + a_off, set + y.out, a_n, D2H, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(reinterpret_cast<char*>(W_last) + s_off, set + y.wl, s_n, D2H, st);
        if (e == cudaSuccess) e = cudaMemcpyAsync(reinterpret_cast<char*>(b_last) + v_off, set + y.bl, v_n, D2H, st);
        if (e == cudaSuccess && W_grad_tail) e = cudaMemcpyAsync(reinterpret_cast<char*>(W_grad_tail) + s_off, set + y.wg, s_n, D2H, st);
        if (e == cudaSuccess && b_grad_tail) e = cudaMemcpyAsync(reinterpret_cast<char*>(b_grad_tail) + v_off, set + y.bg, v_n, D2H, st);
        if (e != cudaSuccess) return cuda_fail(e, "ttt_linear_forward_host_static: outputs");
    }
    return ok();
}
