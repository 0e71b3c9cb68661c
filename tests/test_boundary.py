"""The C-ABI boundary on the host: the library loads, exports what include/ttt.h declares, and
rejects bad arguments with the documented codes before any CUDA call (no GPU needed)."""
import ctypes
import os
import re

import pytest

import oracle

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "ttt.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ttt_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for f in ("ttt_linear_forward", "ttt_linear_forward_host", "ttt_linear_host_workspace_bytes",
              "ttt_mlp_forward", "ttt_linear_decode_step", "ttt_partition", "ttt_error_string",
              "ttt_last_error_message", "ttt_device_status", "ttt_set_wait_limit"):
        assert f in names


def test_binding_constants_match_the_header(libttt):
    defines = dict(re.findall(r"#define\s+(TTT_\w+)\s+\(?(-?\d+)u?\)?", open(HEADER).read()))
    shared = [n for n in defines if hasattr(libttt, n)]
    assert "TTT_FLAG_TOKEN_MAJOR" in shared and "TTT_ERR_ALIAS" in shared
    for n in shared:
        assert getattr(libttt, n) == int(defines[n]), n


def test_library_exports_every_declared_symbol(libttt):
    lib = ctypes.CDLL(libttt.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name
    assert set(libttt.EXPORTS) <= set(declared_functions())


@pytest.mark.parametrize("K", [1, 2, 3, 16])
@pytest.mark.parametrize("L", [0, 1, 15, 16, 17, 31, 8192, 8200])
def test_partition_bit_exact_against_oracle(libttt, orc, L, K):
    assert libttt.ttt_partition(L, K) == orc.partition(L, K)


def test_partition_rejects_bad_arguments(libttt):
    for L, K in ((-1, 16), (10, 0), (10, -3)):
        with pytest.raises(libttt.TTTError) as e:
            libttt.ttt_partition(L, K)
        assert e.value.code == libttt.TTT_ERR_ARG


def test_error_strings(libttt):
    lib = libttt.lib()
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert lib.ttt_error_string(code)
    assert lib.ttt_error_string(-99) == b"unknown error code"


# --- host-side argument validation of the compute entry points (nothing is launched) ----------
A = 1 << 20  # fake, 16-byte aligned "device addresses": validation never dereferences them


def _fwd(lib, **kw):
    args = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W0=5 * A, b0=6 * A, stride=0, lnw=7 * A,
                lnb=8 * A, B=2, H=3, L=64, d=64, K=16, eps=1e-6, dtype=1, flags=0, out=9 * A,
                Wl=10 * A, bl=11 * A, Wg=None, bg=None)
    args.update(kw)
    return lib.ttt_linear_forward(args["XQ"], args["XK"], args["XV"], args["lr"], args["te"], args["W0"],
                                  args["b0"], args["stride"], args["lnw"], args["lnb"], args["B"], args["H"],
                                  args["L"], args["d"], args["K"], args["eps"], args["dtype"], args["flags"],
                                  args["out"], args["Wl"], args["bl"], args["Wg"], args["bg"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), -1), (dict(H=-1), -1), (dict(L=-5), -1), (dict(K=0), -1), (dict(K=17), -1),
    (dict(eps=0.0), -1), (dict(eps=float("nan")), -1), (dict(dtype=7), -1), (dict(flags=8), -1),
    (dict(d=32), -6), (dict(XQ=None), -1), (dict(W0=None), -1), (dict(out=None), -1),
    (dict(stride=5), -1), (dict(XK=2 * A + 2), -2), (dict(out=9 * A + 8), -2), (dict(lr=4 * A + 1), -2),
    (dict(out=A), -3), (dict(Wl=5 * A), -3), (dict(bl=10 * A + 64), -3), (dict(Wg=10 * A), -3),
    (dict(flags=4), -1), (dict(flags=2 | 4), -1),
    # TTT_FLAG_TOKEN_MAJOR (2) alone or with FP32_COMPUTE passes the flag check; the later checks still apply
    (dict(flags=2, out=A), -3), (dict(flags=3, XK=2 * A + 2), -2), (dict(flags=2, K=0), -1),
])
def test_linear_forward_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _fwd(lib, **kw) == code
    assert lib.ttt_last_error_message()


def _fwd_rope(lib, theta=10000.0, **kw):
    args = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W0=5 * A, b0=6 * A, stride=0, lnw=7 * A,
                lnb=8 * A, B=2, H=3, L=64, d=64, K=16, eps=1e-6, dtype=1, flags=0, out=9 * A,
                Wl=10 * A, bl=11 * A, Wg=None, bg=None)
    args.update(kw)
    return lib.ttt_linear_forward_rope(args["XQ"], args["XK"], args["XV"], args["lr"], args["te"], args["W0"],
                                       args["b0"], args["stride"], args["lnw"], args["lnb"], args["B"], args["H"],
                                       args["L"], args["d"], args["K"], args["eps"], theta, args["dtype"],
                                       args["flags"], args["out"], args["Wl"], args["bl"], args["Wg"], args["bg"],
                                       None)


@pytest.mark.parametrize("kw,code", [
    (dict(theta=0.0), -1), (dict(theta=-1.0), -1), (dict(theta=float("nan")), -1), (dict(theta=float("inf")), -1),
    (dict(dtype=0), -6), (dict(flags=1), -6), (dict(flags=8), -1), (dict(flags=4 | 8), -1),
    (dict(K=0), -1), (dict(d=32), -6), (dict(eps=0.0), -1), (dict(XQ=None), -1),
    # the pair flag (4) and token-major (2) pass the flag check; the later checks still apply
    (dict(flags=4, out=A), -3), (dict(flags=2 | 4, XK=2 * A + 2), -2), (dict(flags=2, Wl=5 * A), -3),
])
def test_linear_forward_rope_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _fwd_rope(lib, **kw) == code
    assert lib.ttt_last_error_message()


def test_linear_forward_L0_allows_null_activations_but_checks_state(libttt):
    lib = libttt.lib()
    assert _fwd(lib, L=0, XQ=None, XK=None, XV=None, lr=None, out=None, W0=None) == -1


def test_decode_rejects(libttt):
    lib = libttt.lib()

    def call(**kw):
        a = dict(xq=A, xk=2 * A, xv=3 * A, lr=4 * A, te=None, lnw=5 * A, lnb=6 * A, W=7 * A, b=8 * A,
                 Wg=9 * A, bg=10 * A, B=2, H=2, d=64, K=16, off=3, eps=1e-6, dtype=1, out=11 * A)
        a.update(kw)
        return lib.ttt_linear_decode_step(a["xq"], a["xk"], a["xv"], a["lr"], a["te"], a["lnw"], a["lnb"],
                                          a["W"], a["b"], a["Wg"], a["bg"], a["B"], a["H"], a["d"], a["K"],
                                          a["off"], a["eps"], a["dtype"], a["out"], None)
    assert call(off=-1) == -1
    assert call(W=None) == -1
    assert call(d=48) == -6
    assert call(W=7 * A + 4) == -2
    assert call(out=A) == -3
    assert call(Wg=7 * A) == -3


def test_mlp_rejects(libttt):
    lib = libttt.lib()

    def call(**kw):
        a = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W1=5 * A, b1=6 * A, W2=7 * A, b2=8 * A,
                 stride=0, lnw=9 * A, lnb=10 * A, B=1, H=2, L=32, d=64, hid=256, K=16, eps=1e-6, dtype=1,
                 flags=0, out=11 * A, W1l=12 * A, b1l=13 * A, W2l=14 * A, b2l=15 * A)
        a.update(kw)
        return lib.ttt_mlp_forward(a["XQ"], a["XK"], a["XV"], a["lr"], a["te"], a["W1"], a["b1"], a["W2"],
                                   a["b2"], a["stride"], a["lnw"], a["lnb"], a["B"], a["H"], a["L"], a["d"],
                                   a["hid"], a["K"], a["eps"], a["dtype"], a["flags"], a["out"], a["W1l"],
                                   a["b1l"], a["W2l"], a["b2l"], None)
    assert call(hid=128) == -6
    assert call(W2=None) == -1
    assert call(out=3 * A) == -3
    assert call(b2l=15 * A + 4) == -2
    assert call(flags=4) == -1
    assert call(flags=2, out=3 * A) == -3  # token-major accepted; the overlap check still applies


def test_binding_refuses_cpu_tensors(libttt):
    import torch
    x = torch.zeros(1, 1, 16, 64)
    with pytest.raises(ValueError, match="CUDA"):
        libttt.ttt_linear_forward(x, x, x, torch.zeros(1, 1, 16), torch.zeros(1, 64, 64), torch.zeros(1, 64),
                                  torch.ones(1, 64), torch.zeros(1, 64))


# --- the host-buffer entry point: sizing and rejections (host-only; nothing is copied) ---------
def _host(lib, **kw):
    args = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W0=5 * A, b0=6 * A, stride=0, lnw=7 * A,
                lnb=8 * A, B=2, H=3, L=64, d=64, K=16, eps=1e-6, dtype=1, flags=0, out=9 * A,
                Wl=10 * A, bl=11 * A, Wg=None, bg=None, ws=64 * A, wsb=1 << 40, chunk=1)
    args.update(kw)
    return lib.ttt_linear_forward_host(args["XQ"], args["XK"], args["XV"], args["lr"], args["te"], args["W0"],
                                       args["b0"], args["stride"], args["lnw"], args["lnb"], args["B"], args["H"],
                                       args["L"], args["d"], args["K"], args["eps"], args["dtype"], args["flags"],
                                       args["out"], args["Wl"], args["bl"], args["Wg"], args["bg"], args["ws"],
                                       args["wsb"], args["chunk"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(ws=None), -1), (dict(ws=64 * A + 16), -2), (dict(wsb=1000), -1), (dict(chunk=0), -1),
    (dict(chunk=3), -1), (dict(B=0), -1), (dict(XQ=None), -1), (dict(W0=None), -1), (dict(out=A), -3),
    (dict(Wl=5 * A), -3), (dict(stride=5), -1), (dict(d=32), -6), (dict(K=17), -1), (dict(dtype=5), -1),
])
def test_linear_forward_host_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _host(lib, **kw) == code
    assert lib.ttt_last_error_message()


def test_host_workspace_bytes(libttt):
    lib = libttt.lib()
    n1 = lib.ttt_linear_host_workspace_bytes(8, 32, 8200, 64, 16, 1, 1, 0)
    n2 = lib.ttt_linear_host_workspace_bytes(8, 32, 8200, 64, 16, 1, 2, 0)
    n1f = lib.ttt_linear_host_workspace_bytes(8, 32, 8200, 64, 16, 0, 1, 0)
    npc = lib.ttt_linear_host_workspace_bytes(8, 32, 8200, 64, 16, 1, 1, 32 * 64 * 64)
    act = 32 * 8200 * 64 * 2  # one chunk's bf16 activations
    assert 2 * 4 * act <= n1 < n2 < 2 * n1 + (1 << 20)
    assert n1f > n1 and npc > n1
    assert n1 % 256 == 0
    # the binding reports the same number
    import torch
    assert libttt.ttt_linear_host_workspace_bytes(8, 32, 8200, 16, torch.bfloat16, 1) == n1
    for args, code in (((8, 32, 8200, 64, 16, 1, 0, 0), -1), ((8, 32, 8200, 64, 16, 1, 9, 0), -1),
                       ((8, 32, 8200, 32, 16, 1, 1, 0), -6), ((8, 32, 8200, 64, 16, 1, 1, 5), -1),
                       ((8, 32, -1, 64, 16, 1, 1, 0), -1)):
        assert lib.ttt_linear_host_workspace_bytes(*args) == code


def test_decode_hist_rejects(libttt):
    lib = libttt.lib()

    def call(**kw):
        args = dict(xq=A, xk=2 * A, xv=3 * A, lr=4 * A, te=None, lnw=5 * A, lnb=6 * A, W=7 * A, b=8 * A,
                    hist=9 * A, bg=10 * A, B=2, H=3, d=64, K=16, off=5, eps=1e-6, dtype=1, out=11 * A)
        args.update(kw)
        return lib.ttt_linear_decode_step_hist(args["xq"], args["xk"], args["xv"], args["lr"], args["te"],
                                               args["lnw"], args["lnb"], args["W"], args["b"], args["hist"],
                                               args["bg"], args["B"], args["H"], args["d"], args["K"], args["off"],
                                               args["eps"], args["dtype"], args["out"], None)

    for kw, code in ((dict(hist=None), -1), (dict(off=-1), -1), (dict(hist=9 * A + 4), -2), (dict(K=0), -1),
                     (dict(d=48), -6), (dict(hist=7 * A), -3), (dict(out=A), -3), (dict(bg=None), -1)):
        assert call(**kw) == code, kw
        assert lib.ttt_last_error_message()


def test_token_major_sizes_in_the_binding(libttt):
    """The binding reads (B, H, L, d) from [B,H,L,d], or from [B,L,H,d] with token_major (host only)."""
    import torch
    x = torch.empty(2, 5, 3, 64)
    assert libttt._act_sizes(x, False) == (2, 5, 3, 64)
    assert libttt._act_sizes(x, True) == (2, 3, 5, 64)
    with pytest.raises(ValueError):
        libttt._act_sizes(torch.empty(2, 5, 64), False)
    assert libttt.TTT_FLAG_TOKEN_MAJOR == 2


def test_last_error_message_is_per_host_thread(libttt):
    """Two host threads failing in different ways each read back their own message."""
    import threading
    lib = libttt.lib()
    got = {}
    barrier = threading.Barrier(2)

    def worker(name, kw):
        rc = _fwd(lib, **kw)
        barrier.wait()  # both calls have failed before either reads its message
        got[name] = (rc, lib.ttt_last_error_message())

    threads = [threading.Thread(target=worker, args=("K", dict(K=0))),
               threading.Thread(target=worker, args=("align", dict(XK=2 * A + 2)))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert got["K"][0] == -1 and b"mini_batch" in got["K"][1]
    assert got["align"][0] == -2 and b"aligned" in got["align"][1]


def _prep(lib, **kw):
    a = dict(Wo=A, lnw=2 * A, lnb=3 * A, C=2048, N=2048, Wp=4 * A, u=5 * A, v=6 * A)
    a.update(kw)
    return lib.ttt_o_proj_prepare(a["Wo"], a["lnw"], a["lnb"], a["C"], a["N"], a["Wp"], a["u"], a["v"], None)


def _onorm(lib, **kw):
    a = dict(X=A, T=65600, C=2048, Wp=8 * A, u=9 * A, v=10 * A, N=2048, eps=1e-6, Y=1 << 30, st=1 << 31)
    a.update(kw)
    return lib.ttt_post_norm_o_proj(a["X"], a["T"], a["C"], a["Wp"], a["u"], a["v"], a["N"], a["eps"], a["Y"], a["st"],
                                    None)


@pytest.mark.parametrize("kw,code", [
    (dict(C=32), -6), (dict(C=100), -6), (dict(N=128), -6), (dict(N=300), -6), (dict(Wo=None), -1),
    (dict(v=None), -1), (dict(Wo=A + 8), -2), (dict(Wp=4 * A + 4), -2), (dict(u=5 * A + 2), -2),
    (dict(Wp=A + 64), -3), (dict(u=4 * A + 16), -3), (dict(v=5 * A), -3),
])
def test_o_proj_prepare_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _prep(lib, **kw) == code
    assert lib.ttt_last_error_message()


@pytest.mark.parametrize("kw,code", [
    (dict(T=-1), -1), (dict(T=65535 * 128 + 1), -6), (dict(C=96), -6), (dict(N=512 + 64), -6),
    (dict(eps=0.0), -1), (dict(eps=float("inf")), -1), (dict(X=None), -1), (dict(Wp=None), -1),
    (dict(X=A + 2), -2), (dict(Y=(1 << 30) + 8), -2), (dict(u=9 * A + 1), -2),
    (dict(Y=A), -3), (dict(Y=8 * A - 64), -3), (dict(st=None), -1), (dict(st=(1 << 31) + 4), -2),
    (dict(st=A), -3), (dict(st=(1 << 30) + 64), -3),
])
def test_post_norm_o_proj_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _onorm(lib, **kw) == code
    assert lib.ttt_last_error_message()


def test_post_norm_o_proj_T0_is_a_no_op(libttt):
    lib = libttt.lib()
    assert _onorm(lib, T=0, X=None, Y=None, st=None) == 0


def _bwd(lib, **kw):
    a = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W0=5 * A, b0=6 * A, stride=0, lnw=7 * A, lnb=8 * A, B=2,
             H=3, L=64, d=64, K=16, eps=1e-6, dtype=1, flags=0, G=4, dout=9 * A, dWl=None, dbl=None, dXQ=10 * A, dXK=11 * A,
             dXV=12 * A, dlr=13 * A, dW0=14 * A, db0=15 * A, dlnw=16 * A, dlnb=17 * A, ws=1 << 32, wsb=1 << 30)
    a.update(kw)
    return lib.ttt_linear_backward(a["XQ"], a["XK"], a["XV"], a["lr"], a["te"], a["W0"], a["b0"], a["stride"],
                                   a["lnw"], a["lnb"], a["B"], a["H"], a["L"], a["d"], a["K"], a["eps"], a["dtype"],
                                   a["flags"], a["G"], a["dout"], a["dWl"], a["dbl"], a["dXQ"], a["dXK"], a["dXV"], a["dlr"],
                                   a["dW0"], a["db0"], a["dlnw"], a["dlnb"], a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), -1), (dict(K=17), -1), (dict(d=32), -6), (dict(dtype=7), -1), (dict(eps=0.0), -1), (dict(G=0), -1),
    (dict(stride=5), -1), (dict(XQ=None), -1), (dict(dout=None), -1), (dict(dW0=None), -1), (dict(ws=None), -1),
    (dict(wsb=100), -1), (dict(ws=(1 << 32) + 16), -2), (dict(XK=2 * A + 2), -2), (dict(dXQ=10 * A + 8), -2),
    (dict(dlr=13 * A + 1), -2), (dict(dWl=18 * A + 4), -2), (dict(dXQ=A), -3), (dict(dXK=10 * A), -3),
    (dict(ws=5 * A), -3), (dict(dW0=9 * A), -3), (dict(dlnb=16 * A + 64), -3),
    (dict(flags=1), -6), (dict(flags=4), -1), (dict(flags=2, dXQ=A), -3), (dict(flags=2, XK=2 * A + 2), -2),
])
def test_linear_backward_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _bwd(lib, **kw) == code
    assert lib.ttt_last_error_message()


def test_linear_backward_workspace_bytes(libttt):
    # per chain: ceil(n_full / G) kept states + G rebuilt states of (64*64 + 64) floats, and the shares
    n = libttt.ttt_linear_backward_workspace_bytes(2, 3, 8200, 16, 16)
    state = (64 * 64 + 64) * 4
    up = lambda x: (x + 255) // 256 * 256
    assert n == up(6 * 32 * state) + up(6 * 16 * state) + up(6 * (64 * 64 + 3 * 64) * 4)
    assert libttt.ttt_linear_backward_workspace_bytes(2, 3, 0, 16, 16) == up(6 * 16 * state) + up(6 * (64 * 64 + 192) * 4)
    with pytest.raises(libttt.TTTError):
        libttt.ttt_linear_backward_workspace_bytes(2, 3, 100, 16, 0)


def _fwd_ckpt(lib, G=4, ck=19 * A, **kw):
    args = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W0=5 * A, b0=6 * A, stride=0, lnw=7 * A,
                lnb=8 * A, B=2, H=3, L=64, d=64, K=16, eps=1e-6, dtype=1, flags=0, out=9 * A,
                Wl=10 * A, bl=11 * A, Wg=None, bg=None)
    args.update(kw)
    return lib.ttt_linear_forward_ckpt(args["XQ"], args["XK"], args["XV"], args["lr"], args["te"], args["W0"],
                                       args["b0"], args["stride"], args["lnw"], args["lnb"], args["B"], args["H"],
                                       args["L"], args["d"], args["K"], args["eps"], args["dtype"], args["flags"],
                                       args["out"], args["Wl"], args["bl"], args["Wg"], args["bg"], G, ck, None)


@pytest.mark.parametrize("kw,code", [
    (dict(ck=None), -1), (dict(G=0), -1), (dict(ck=19 * A + 8), -2), (dict(ck=9 * A), -3),
    (dict(ck=10 * A + 64), -3), (dict(ck=A), -3), (dict(K=0), -1), (dict(d=32), -6),
])
def test_linear_forward_ckpt_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _fwd_ckpt(lib, **kw) == code
    assert lib.ttt_last_error_message()


def _bwd_ckpt(lib, ck=19 * A, **kw):
    a = dict(XQ=A, XK=2 * A, XV=3 * A, lr=4 * A, te=None, W0=5 * A, b0=6 * A, stride=0, lnw=7 * A, lnb=8 * A, B=2,
             H=3, L=64, d=64, K=16, eps=1e-6, dtype=1, flags=0, G=4, dout=9 * A, dWl=None, dbl=None, dXQ=10 * A,
             dXK=11 * A, dXV=12 * A, dlr=13 * A, dW0=14 * A, db0=15 * A, dlnw=16 * A, dlnb=17 * A, ws=1 << 32,
             wsb=1 << 30)
    a.update(kw)
    return lib.ttt_linear_backward_ckpt(a["XQ"], a["XK"], a["XV"], a["lr"], a["te"], a["W0"], a["b0"], a["stride"],
                                        a["lnw"], a["lnb"], a["B"], a["H"], a["L"], a["d"], a["K"], a["eps"],
                                        a["dtype"], a["flags"], a["G"], ck, a["dout"], a["dWl"], a["dbl"], a["dXQ"],
                                        a["dXK"], a["dXV"], a["dlr"], a["dW0"], a["db0"], a["dlnw"], a["dlnb"],
                                        a["ws"], a["wsb"], None)


@pytest.mark.parametrize("kw,code", [
    (dict(ck=None), -1), (dict(G=0), -1), (dict(ck=19 * A + 4), -2), (dict(ck=10 * A), -3),
    (dict(ck=(1 << 32) + 4096), -3), (dict(flags=1), -6), (dict(wsb=100), -1),
])
def test_linear_backward_ckpt_rejects(libttt, kw, code):
    lib = libttt.lib()
    assert _bwd_ckpt(lib, **kw) == code
    assert lib.ttt_last_error_message()


def test_linear_ckpt_bytes(libttt):
    # per chain: ceil(n_full / G) group starts + the state after the last full mini-batch
    state = (64 * 64 + 64) * 4
    assert libttt.ttt_linear_ckpt_bytes(2, 3, 8200, 16, 16) == 6 * (32 + 1) * state
    assert libttt.ttt_linear_ckpt_bytes(2, 3, 8200, 16, 5) == 6 * (103 + 1) * state
    assert libttt.ttt_linear_ckpt_bytes(2, 3, 15, 16, 4) == 6 * 1 * state
    assert libttt.ttt_linear_ckpt_bytes(2, 3, 0, 16, 4) == 6 * 1 * state
    with pytest.raises(libttt.TTTError):
        libttt.ttt_linear_ckpt_bytes(2, 3, 100, 16, 0)
