/* Plain C99 client of include/ttt.h: the ABI is usable from C (no C++ or torch types), and the
 * host-only calls behave as documented.  Built and run by tests/test_c_abi.py; needs no GPU
 * (argument errors are reported before any CUDA call).  Prints one line per check; exit 0 iff
 * every check passed. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "ttt.h"

static int failures = 0;

static void check(int ok, const char* what) {
    printf("%s %s\n", ok ? "ok" : "FAIL", what);
    if (!ok) ++failures;
}

int main(void) {
    long long n = -1, r = -1;
    check(ttt_partition(8200, 16, &n, &r) == TTT_OK && n == 512 && r == 8, "partition 8200 / 16");
    check(ttt_partition(0, 16, &n, &r) == TTT_OK && n == 0 && r == 0, "partition 0 / 16");
    check(ttt_partition(-1, 16, &n, &r) == TTT_ERR_ARG, "partition rejects L < 0");
    check(ttt_partition(10, 0, &n, &r) == TTT_ERR_ARG, "partition rejects K < 1");
    check(strlen(ttt_last_error_message()) > 0, "a failed call leaves a message");
    check(strcmp(ttt_error_string(TTT_ERR_ALIGN), "misaligned pointer") == 0, "error string");

    /* fake, 16-byte aligned device addresses: validation never dereferences them */
    const uintptr_t A = (uintptr_t)1 << 20;
    const void* XQ = (const void*)(1 * A);
    const void* XK = (const void*)(2 * A);
    const void* XV = (const void*)(3 * A);
    const float* lr = (const float*)(4 * A);
    const float* W0 = (const float*)(5 * A);
    const float* b0 = (const float*)(6 * A);
    const float* lnw = (const float*)(7 * A);
    const float* lnb = (const float*)(8 * A);
    void* out = (void*)(9 * A);
    float* Wl = (float*)(10 * A);
    float* bl = (float*)(11 * A);
    check(ttt_linear_forward(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 17, 1e-6f, TTT_BF16, 0,
                             out, Wl, bl, NULL, NULL, NULL) == TTT_ERR_ARG, "forward rejects K = 17");
    check(ttt_linear_forward(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 32, 16, 1e-6f, TTT_BF16, 0,
                             out, Wl, bl, NULL, NULL, NULL) == TTT_ERR_UNSUPPORTED, "forward rejects d = 32");
    check(ttt_linear_forward(XQ, (const char*)XK + 2, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f,
                             TTT_BF16, TTT_FLAG_TOKEN_MAJOR, out, Wl, bl, NULL, NULL, NULL) == TTT_ERR_ALIGN,
          "forward rejects a misaligned XK (token-major flag accepted)");
    check(ttt_linear_forward(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, TTT_BF16, 0,
                             (void*)XQ, Wl, bl, NULL, NULL, NULL) == TTT_ERR_ALIAS, "forward rejects out == XQ");
    check(ttt_linear_forward(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, TTT_BF16, 8,
                             out, Wl, bl, NULL, NULL, NULL) == TTT_ERR_ARG, "forward rejects unknown flags");

    check(ttt_linear_forward_rope(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, 0.0f, TTT_BF16,
                                  0, out, Wl, bl, NULL, NULL, NULL) == TTT_ERR_ARG, "rope forward rejects theta = 0");
    check(ttt_linear_forward_rope(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, 1e4f, TTT_F32,
                                  0, out, Wl, bl, NULL, NULL, NULL) == TTT_ERR_UNSUPPORTED,
          "rope forward rejects fp32 activations");
    check(ttt_linear_forward_rope(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, 1e4f, TTT_BF16,
                                  TTT_FLAG_ROPE_HALF_SPLIT | TTT_FLAG_TOKEN_MAJOR, (void*)XK, Wl, bl, NULL, NULL,
                                  NULL) == TTT_ERR_ALIAS, "rope forward accepts its flags, rejects out == XK");

    check(ttt_o_proj_prepare(XQ, W0, b0, 2048, 100, out, Wl, bl, NULL) == TTT_ERR_UNSUPPORTED,
          "o_proj prepare rejects N = 100");
    check(ttt_post_norm_o_proj(XQ, 65600, 2048, XK, W0, b0, 2048, 0.0f, out, Wl, NULL) == TTT_ERR_ARG,
          "post_norm o_proj rejects eps = 0");
    check(ttt_post_norm_o_proj(NULL, 0, 2048, XK, W0, b0, 2048, 1e-6f, NULL, NULL, NULL) == TTT_OK,
          "post_norm o_proj with T = 0 is a no-op");

    const long long ws = ttt_linear_host_workspace_bytes(8, 32, 8200, 64, 16, TTT_BF16, 1, 0);
    check(ws > 0 && ws % 256 == 0, "host workspace size");
    check(ttt_linear_host_workspace_bytes(8, 32, 8200, 64, 16, TTT_BF16, 9, 0) == TTT_ERR_ARG,
          "host workspace rejects chunk_batches > B");
    const long long bws = ttt_linear_backward_workspace_bytes(8, 32, 8200, 64, 16, 16);
    check(bws > 0 && bws % 256 == 0, "backward workspace size");
    check(ttt_linear_backward_workspace_bytes(8, 32, 8200, 64, 16, 0) == TTT_ERR_ARG,
          "backward workspace rejects ckpt_group = 0");
    float* g[8];
    for (int i = 0; i < 8; ++i) g[i] = (float*)((uintptr_t)(12 + i) * A);  /* fake gradient outputs */
    check(ttt_linear_backward(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, TTT_BF16, 0u, 0, out,
                              NULL, NULL, g[0], g[1], g[2], g[3], g[4], g[5], g[6], g[7], NULL, 0, NULL) == TTT_ERR_ARG,
          "backward rejects ckpt_group = 0");
    const long long cks = ttt_linear_ckpt_bytes(8, 32, 8200, 64, 16, 16);
    check(cks == 8LL * 32 * 33 * (64 * 64 + 64) * 4, "checkpoint buffer size");
    check(ttt_linear_ckpt_bytes(8, 32, 8200, 64, 16, 0) == TTT_ERR_ARG, "checkpoint size rejects ckpt_group = 0");
    float* ck = (float*)((uintptr_t)20 * A);  /* fake checkpoint buffer */
    check(ttt_linear_forward_ckpt(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, TTT_BF16, 0u,
                                  out, Wl, bl, NULL, NULL, 4, NULL, NULL) == TTT_ERR_ARG,
          "forward with checkpoints rejects a null buffer");
    check(ttt_linear_forward_ckpt(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, TTT_BF16, 0u,
                                  out, Wl, bl, NULL, NULL, 0, ck, NULL) == TTT_ERR_ARG,
          "forward with checkpoints rejects ckpt_group = 0");
    check(ttt_linear_backward_ckpt(XQ, XK, XV, lr, NULL, W0, b0, 0, lnw, lnb, 2, 3, 64, 64, 16, 1e-6f, TTT_BF16, 0u, 4,
                                   NULL, out, NULL, NULL, g[0], g[1], g[2], g[3], g[4], g[5], g[6], g[7], NULL, 0,
                                   NULL) == TTT_ERR_ARG,
          "backward from checkpoints rejects a null buffer");
    return failures == 0 ? 0 : 1;
}
