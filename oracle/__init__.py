"""CPU oracle of the TTT scan (ctypes wrapper over ``ttt_oracle.c``), in float64.

TEST INFRASTRUCTURE ONLY: used by ``tests/``, ``__graft_entry__.smoke()`` and the bench's
CPU-baseline leg.  The CUDA library never imports, links or calls anything here, and nothing
here imports the CUDA library.  Every array handed in is widened to float64 exactly
(fp32 values and bf16-valued fp32 are exact in double).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ttt_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libttt_oracle.so")


_LIB_F32_PATH = os.path.join(_HERE, "libttt_oracle_f32.so")


def build(force: bool = False, src: str = _SRC, out: str = _LIB_PATH, real: str = "double") -> str:
    """Compile the oracle with gcc: plain -O2, no fast-math, no FMA contraction.  real="float"
    builds the same source in single precision (timed as a CPU baseline, never a parity
    reference)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-std=c99",
                               f"-DORACLE_REAL={real}", "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def build_f32(force: bool = False) -> str:
    return build(force, _SRC, _LIB_F32_PATH, "float")


_D = ctypes.POINTER(ctypes.c_double)
_LL = ctypes.c_longlong


def load(path: str | None = None):
    """Load (building if needed) an oracle shared library and declare its signatures."""
    lib = ctypes.CDLL(path or build())
    i, dbl = ctypes.c_int, ctypes.c_double
    lib.oracle_partition.argtypes = [_LL, i, ctypes.POINTER(_LL), ctypes.POINTER(_LL)]
    lib.oracle_lnl2_grad.argtypes = [_D, _D, _D, _D, i, dbl, _D]
    lib.oracle_ln_forward.argtypes = [_D, _D, _D, i, dbl, _D]
    lib.oracle_gelu_tanh.argtypes = [_D, _LL, _D, _D]
    lib.oracle_ttt_linear_chain.argtypes = [_D, _D, _D, _D, _D, _D, _D, _D, _D, _LL, i, i, dbl,
                                            _D, _D, _D, _D, _D]
    lib.oracle_ttt_linear_decode_chain.argtypes = [_D, _D, _D, dbl, _D, _D, _D, _D, _D, _D, _D,
                                                   i, i, _LL, dbl, _D, ctypes.POINTER(i)]
    lib.oracle_rope.argtypes = [_D, _LL, i, i, dbl, i, _D]
    lib.oracle_post_norm_o_proj.argtypes = [_D, _LL, i, _D, _D, dbl, _D, i, _D]
    lib.oracle_ttt_mlp_chain.argtypes = [_D, _D, _D, _D, _D, _D, _D, _D, _D, _D, _D, _LL, i, i, i,
                                         dbl, _D, _D, _D, _D, _D]
    for f in ("oracle_partition", "oracle_lnl2_grad", "oracle_ln_forward", "oracle_gelu_tanh",
              "oracle_ttt_linear_chain", "oracle_ttt_linear_decode_chain", "oracle_ttt_mlp_chain",
              "oracle_rope", "oracle_post_norm_o_proj"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


class Oracle:
    """Python face of one oracle build (the default one, or a test-made variant)."""

    def __init__(self, path: str | None = None):
        self.lib = load(path)

    # ---- helpers ---------------------------------------------------------------------------
    @staticmethod
    def _f64(a):
        return None if a is None else np.ascontiguousarray(a, dtype=np.float64)

    @staticmethod
    def _p(a):
        return None if a is None else a.ctypes.data_as(_D)

    def _check(self, rc, what):
        if rc != 0:
            raise ValueError(f"{what}: oracle rejected its arguments (rc={rc})")

    # ---- pieces ----------------------------------------------------------------------------
    def partition(self, L: int, K: int):
        n, r = _LL(), _LL()
        self._check(self.lib.oracle_partition(L, K, ctypes.byref(n), ctypes.byref(r)), "partition")
        return n.value, r.value

    def lnl2_grad(self, z, tgt, ln_w, ln_b, eps):
        z, tgt, ln_w, ln_b = map(self._f64, (z, tgt, ln_w, ln_b))
        g = np.empty_like(z)
        self._check(self.lib.oracle_lnl2_grad(self._p(z), self._p(tgt), self._p(ln_w), self._p(ln_b),
                                              z.size, eps, self._p(g)), "lnl2_grad")
        return g

    def ln_forward(self, u, ln_w, ln_b, eps):
        u, ln_w, ln_b = map(self._f64, (u, ln_w, ln_b))
        y = np.empty_like(u)
        self._check(self.lib.oracle_ln_forward(self._p(u), self._p(ln_w), self._p(ln_b), u.size, eps,
                                               self._p(y)), "ln_forward")
        return y

    def gelu(self, x):
        x = self._f64(x)
        y, dy = np.empty_like(x), np.empty_like(x)
        self._check(self.lib.oracle_gelu_tanh(self._p(x), x.size, self._p(y), self._p(dy)), "gelu")
        return y, dy

    def rope(self, x, K, theta, half_split=False):
        """Rotary embedding of [..., L, d] rows (position = token index mod K), float64."""
        x = self._f64(x)
        y = np.empty_like(x)
        L, d = x.shape[-2], x.shape[-1]
        flat_x, flat_y = x.reshape(-1, L, d), y.reshape(-1, L, d)
        for c in range(flat_x.shape[0]):
            xc = np.ascontiguousarray(flat_x[c])
            yc = np.empty_like(xc)
            self._check(self.lib.oracle_rope(self._p(xc), L, d, K, float(theta), 1 if half_split else 0,
                                             self._p(yc)), "rope")
            flat_y[c] = yc
        return y

    def post_norm_o_proj(self, x, ln_w, ln_b, eps, Wo):
        """y = o_proj(post_norm(x)) per token: x [T, C], ln_w / ln_b [C], Wo [N, C] (out x in)."""
        x, ln_w, ln_b, Wo = map(self._f64, (x, ln_w, ln_b, Wo))
        T, C = x.shape
        N = Wo.shape[0]
        y = np.empty((T, N))
        self._check(self.lib.oracle_post_norm_o_proj(self._p(x), T, C, self._p(ln_w), self._p(ln_b), float(eps),
                                                     self._p(Wo), N, self._p(y)), "post_norm_o_proj")
        return y

    # ---- TTT-Linear ------------------------------------------------------------------------
    def linear_chain(self, xq, xk, xv, lr, W0, b0, ln_w, ln_b, K, eps, token_eta=None):
        """One chain: xq/xk/xv [L,d], lr [L], W0 [d,d], b0 [d], ln_w/ln_b [d]."""
        xq, xk, xv, lr, W0, b0, ln_w, ln_b, te = map(self._f64, (xq, xk, xv, lr, W0, b0, ln_w, ln_b,
                                                                 token_eta))
        L, d = xq.shape
        out = np.empty((L, d))
        W_last, b_last = np.empty((d, d)), np.empty(d)
        Wg, bg = np.empty((d, d)), np.empty(d)
        rc = self.lib.oracle_ttt_linear_chain(self._p(xq), self._p(xk), self._p(xv), self._p(lr),
                                              self._p(te), self._p(W0), self._p(b0), self._p(ln_w),
                                              self._p(ln_b), L, d, K, eps, self._p(out),
                                              self._p(W_last), self._p(b_last), self._p(Wg), self._p(bg))
        self._check(rc, "ttt_linear_chain")
        return {"out": out, "W_last": W_last, "b_last": b_last, "W_grad_tail": Wg, "b_grad_tail": bg}

    def linear_forward(self, XQ, XK, XV, lr, W0, b0, ln_w, ln_b, K, eps, token_eta=None,
                       chains=None, state_per_chain=False):
        """Batched over chains.  W0/b0 are [H,d,d]/[H,d] shared over the batch, or
        [B,H,d,d]/[B,H,d] when state_per_chain is set (a continuation from an earlier call).

        chains: optional list of flat chain ids (b*H + h).  XQ/XK/XV/lr are then [n,L,d]/[n,L]
        stacks holding those chains in order; otherwise full [B,H,L,d]/[B,H,L] tensors.
        Returns stacked per-chain results ([n, ...]).
        """
        return self._batched(self.linear_chain, XQ, XK, XV, lr, (W0, b0), ln_w, ln_b,
                             dict(K=K, eps=eps, token_eta=token_eta), chains, state_per_chain)

    def mlp_forward(self, XQ, XK, XV, lr, W1, b1, W2, b2, ln_w, ln_b, K, eps, token_eta=None,
                    chains=None, state_per_chain=False):
        """TTT-MLP counterpart of linear_forward (states W1 [H,d,h], b1 [H,h], W2 [H,h,d], b2 [H,d])."""
        return self._batched(self.mlp_chain, XQ, XK, XV, lr, (W1, b1, W2, b2), ln_w, ln_b,
                             dict(K=K, eps=eps, token_eta=token_eta), chains, state_per_chain)

    def _batched(self, fn, XQ, XK, XV, lr, states, ln_w, ln_b, kw, chains, state_per_chain):
        H = ln_w.shape[0]
        if chains is None:
            B = XQ.shape[0]
            ids = list(range(B * H))
            acts = lambda a, n, c: a[c // H, c % H]
        else:
            ids = list(chains)
            acts = lambda a, n, c: a[n]
        results = []
        for n, c in enumerate(ids):
            b, h = divmod(c, H)
            st = [np.asarray(s)[b, h] if state_per_chain else np.asarray(s)[h] for s in states]
            results.append(fn(acts(XQ, n, c), acts(XK, n, c), acts(XV, n, c), acts(lr, n, c),
                              *st, ln_w[h], ln_b[h], **kw))
        keys = results[0].keys() if results else []
        return {k: np.stack([r[k] for r in results]) for k in keys}

    # ---- decode ----------------------------------------------------------------------------
    def decode_chain(self, xq, xk, xv, lr, ln_w, ln_b, W, b, W_grad, b_grad, K, offset, eps,
                     token_eta=None):
        """One token of one chain.  W, b, W_grad, b_grad are updated IN PLACE (float64)."""
        xq, xk, xv, ln_w, ln_b, te = map(self._f64, (xq, xk, xv, ln_w, ln_b, token_eta))
        for s in (W, b, W_grad, b_grad):
            assert s.dtype == np.float64 and s.flags.c_contiguous
        d = xq.size
        out = np.empty(d)
        committed = ctypes.c_int()
        rc = self.lib.oracle_ttt_linear_decode_chain(self._p(xq), self._p(xk), self._p(xv), float(lr),
                                                     self._p(te), self._p(ln_w), self._p(ln_b),
                                                     self._p(W), self._p(b), self._p(W_grad),
                                                     self._p(b_grad), d, K, offset, eps, self._p(out),
                                                     ctypes.byref(committed))
        self._check(rc, "decode_chain")
        return out, bool(committed.value)

    # ---- TTT-MLP ---------------------------------------------------------------------------
    def mlp_chain(self, xq, xk, xv, lr, W1, b1, W2, b2, ln_w, ln_b, K, eps, token_eta=None):
        xq, xk, xv, lr, W1, b1, W2, b2, ln_w, ln_b, te = map(
            self._f64, (xq, xk, xv, lr, W1, b1, W2, b2, ln_w, ln_b, token_eta))
        L, d = xq.shape
        h = W1.shape[1]
        out = np.empty((L, d))
        W1l, b1l, W2l, b2l = np.empty((d, h)), np.empty(h), np.empty((h, d)), np.empty(d)
        rc = self.lib.oracle_ttt_mlp_chain(self._p(xq), self._p(xk), self._p(xv), self._p(lr),
                                           self._p(te), self._p(W1), self._p(b1), self._p(W2),
                                           self._p(b2), self._p(ln_w), self._p(ln_b), L, d, h, K, eps,
                                           self._p(out), self._p(W1l), self._p(b1l), self._p(W2l),
                                           self._p(b2l))
        self._check(rc, "ttt_mlp_chain")
        return {"out": out, "W1_last": W1l, "b1_last": b1l, "W2_last": W2l, "b2_last": b2l}


class OracleF32:
    """The float build of the same oracle source: TTT-Linear chains only, for timing (the CPU
    baseline's single-precision figure).  Not a parity reference."""

    def __init__(self):
        lib = ctypes.CDLL(build_f32())
        F = ctypes.POINTER(ctypes.c_float)
        lib.oracle_ttt_linear_chain.argtypes = [F, F, F, F, F, F, F, F, F, _LL, ctypes.c_int, ctypes.c_int,
                                                ctypes.c_float, F, F, F, F, F]
        lib.oracle_ttt_linear_chain.restype = ctypes.c_int
        self.lib = lib

    def linear_chain(self, xq, xk, xv, lr, W0, b0, ln_w, ln_b, K, eps):
        f = lambda a: np.ascontiguousarray(a, dtype=np.float32)
        xq, xk, xv, lr, W0, b0, ln_w, ln_b = map(f, (xq, xk, xv, lr, W0, b0, ln_w, ln_b))
        L, d = xq.shape
        out, W_last, b_last = np.empty((L, d), np.float32), np.empty((d, d), np.float32), np.empty(d, np.float32)
        Wg, bg = np.empty((d, d), np.float32), np.empty(d, np.float32)
        p = lambda a: a.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
        rc = self.lib.oracle_ttt_linear_chain(p(xq), p(xk), p(xv), p(lr), None, p(W0), p(b0), p(ln_w), p(ln_b),
                                              L, d, K, eps, p(out), p(W_last), p(b_last), p(Wg), p(bg))
        if rc != 0:
            raise ValueError(f"float oracle rejected its arguments (rc={rc})")
        return {"out": out, "W_last": W_last, "b_last": b_last}


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle()
    return _default
