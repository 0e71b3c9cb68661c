"""Seeded synthetic inputs for the TTT scan (shared by the oracle tests, the CUDA tests and the bench).

This module holds no arithmetic of the TTT method.  It draws the tensors the method takes as
inputs, with the shapes and value distributions of the workloads on the TTT pages (the
``TTTLinear.__init__`` listing on the nanhubrain/jiafeimiao pages for W0 ~ N(0, 0.02) and
b0 = 0; the 125M / 1B layer shapes from ``TTT_STANDARD_CONFIGS``), and hands out the exact
bits: fp32 arrays, or bf16 bit patterns (uint16) rounded to nearest-even from fp32 draws.

Every element depends only on (seed, tensor tag, flat element index), so any chain's slice
can be regenerated without drawing the whole tensor (see ``synth.c``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")

# Tensor tags: one independent stream per tensor.
TAG = {
    "XQ": 1, "XK": 2, "XV": 3, "LR": 4, "W0": 5, "LNW": 6, "LNB": 7,
    "W1": 8, "W2": 9, "B0": 10, "B1": 11, "B2": 12,
    "ONX": 13, "ONW": 14, "ONLW": 15, "ONLB": 16,
    "DO": 17, "DWL": 18, "DBL": 19,
}

SEED_BASE = 0x77170000


def build(force: bool = False) -> str:
    """Compile the generator (gcc, OpenMP).  Returns the shared-library path."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def _get_lib():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, dbl = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
        fptr = ctypes.POINTER(ctypes.c_float)
        lib.synth_stream_key.argtypes = [u64, u64]
        lib.synth_stream_key.restype = u64
        lib.synth_draw_u64.argtypes = [u64, u64]
        lib.synth_draw_u64.restype = u64
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, dbl, fptr]
        lib.synth_normal_f32.restype = None
        lib.synth_logistic_normal_f32.argtypes = [u64, u64, i64, dbl, fptr]
        lib.synth_logistic_normal_f32.restype = None
        _lib = lib
    return _lib


def stream_key(seed: int, tag: int) -> int:
    return int(_get_lib().synth_stream_key(seed, tag))


def normal(seed: int, tag: int, n: int, first: int = 0, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """n fp32 values mean + std*N(0,1), elements [first, first+n) of stream (seed, tag)."""
    out = np.empty(n, dtype=np.float32)
    if n:
        _get_lib().synth_normal_f32(stream_key(seed, tag), first, n, mean, std,
                                    out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return out


def logistic_normal(seed: int, tag: int, n: int, first: int = 0, denom: float = 1.0) -> np.ndarray:
    """n fp32 values sigmoid(N(0,1)) / denom."""
    out = np.empty(n, dtype=np.float32)
    if n:
        _get_lib().synth_logistic_normal_f32(stream_key(seed, tag), first, n, denom,
                                             out.ctypes.data_as(ctypes.POINTER(ctypes.c_float)))
    return out


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = (b + np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Workload:
    """Shapes and distributions of one synthetic workload.

    kind: "linear" (TTT-Linear prefill), "mlp" (TTT-MLP prefill) or "decode".
    dtype: "f32" or "bf16" for XQ/XK/XV (and out); state and lr are always fp32.
    x_std: std of XQ/XK/XV; ln: "unit" (ln_w=1, ln_b=0) or "random" (1+N(0,ln_w_std),
    N(0,ln_b_std)); w_std: std of the initial weights (W0, or W1 and W2 for TTT-MLP).
    """
    name: str
    kind: str
    B: int
    H: int
    L: int
    d: int = 64
    K: int = 16
    dtype: str = "bf16"
    x_std: float = 0.125
    ln: str = "random"
    w_std: float = 0.02
    ln_w_std: float = 0.1
    ln_b_std: float = 0.1
    hidden: int = 256
    seed: int = SEED_BASE
    eps: float = 1e-6
    decode_steps: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def chains(self) -> int:
        return self.B * self.H


def workload(index: int, **overrides) -> Workload:
    """The five workloads of the TTT scan (layer shapes from TTT_STANDARD_CONFIGS)."""
    seed = SEED_BASE + index
    presets = {
        0: Workload("ttt_linear_fp32_B1_H2_L64", "linear", B=1, H=2, L=64, dtype="f32",
                    x_std=1.0 / 8.0, ln="unit", seed=seed),
        1: Workload("ttt_linear_125m_B16_H12_L2048", "linear", B=16, H=12, L=2048, seed=seed),
        2: Workload("ttt_linear_1b_B8_H32_L8192", "linear", B=8, H=32, L=8192, seed=seed),
        3: Workload("ttt_mlp_B8_H32_L2048_h256", "mlp", B=8, H=32, L=2048, seed=seed),
        4: Workload("ttt_linear_decode_B128_H32_prefill2048", "decode", B=128, H=32, L=2048,
                    decode_steps=1024, seed=seed),
    }
    w = presets[index]
    for k, v in overrides.items():
        setattr(w, k, v)
    return w


def stream_length(w: Workload) -> int:
    """Tokens per chain in the workload's stream: the prefill, then the decode tokens."""
    return w.L + w.decode_steps


def _window(w: Workload, tag: str, per_token: int, t0: int, t1: int, chains, draw) -> np.ndarray:
    """Tokens [t0, t1) of every listed chain of a [chains, stream_length, per_token] stream."""
    Ltot = stream_length(w)
    ids = range(w.chains) if chains is None else chains
    if chains is None and t0 == 0 and t1 == Ltot:
        return draw(w.seed, TAG[tag], w.chains * Ltot * per_token, 0).reshape(w.chains, Ltot, per_token)
    n = (t1 - t0) * per_token
    out = np.empty((len(ids), t1 - t0, per_token), np.float32)
    for i, c in enumerate(ids):
        out[i] = draw(w.seed, TAG[tag], n, (c * Ltot + t0) * per_token).reshape(t1 - t0, per_token)
    return out


def _x_tensor(w: Workload, tag: str, t0: int, t1: int, chains=None, values: bool = True):
    """Activations of tokens [t0, t1): fp32 values (None when values is False and the workload
    is bf16) and bf16 bit patterns (None for fp32 workloads); [B,H,T,d] or [n,T,d]."""
    vals = _window(w, tag, w.d, t0, t1, chains,
                   lambda seed, tag_, n, first: normal(seed, tag_, n, first, 0.0, w.x_std))
    shape = (w.B, w.H, t1 - t0, w.d) if chains is None else (len(chains), t1 - t0, w.d)
    vals = vals.reshape(shape)
    if w.dtype == "bf16":
        bits = f32_to_bf16_bits(vals).reshape(shape)
        del vals
        return (bf16_bits_to_f32(bits).reshape(shape) if values else None), bits
    return vals, None


def linear_inputs(w: Workload, chains=None, values: bool = True, t0: int = 0, t1: int | None = None) -> dict:
    """Inputs of ttt_linear_forward / ttt_mlp_forward / the decode steps, for tokens [t0, t1) of
    each chain's stream of stream_length(w) tokens (default: the whole stream).

    Returns a dict of numpy arrays: XQ, XK, XV as fp32 values ([B,H,T,d], or [n,T,d] for a
    chain subset; omitted for bf16 workloads when values is False, to save host memory),
    XQ_bits/XK_bits/XV_bits (uint16 bf16 patterns, bf16 workloads only),
    lr [B,H,T] fp32 = sigmoid(N(0,1))/d, and the per-head state and LayerNorm parameters
    (state_inputs).  A chain's values are identical whether drawn alone, in a window or in full.
    """
    t1 = stream_length(w) if t1 is None else t1
    out = {}
    for t in ("XQ", "XK", "XV"):
        vals, bits = _x_tensor(w, t, t0, t1, chains, values)
        if vals is not None:
            out[t] = vals
        if bits is not None:
            out[t + "_bits"] = bits
    lr = _window(w, "LR", 1, t0, t1, chains,
                 lambda seed, tag_, n, first: logistic_normal(seed, tag_, n, first, float(w.d)))
    out["lr"] = lr.reshape((w.B, w.H, t1 - t0) if chains is None else (len(chains), t1 - t0))
    out.update(state_inputs(w))
    return out


def upstream_grads(w: Workload, chains=None, values: bool = True, std: float = 1.0) -> dict:
    """Seeded gradients arriving at the scan's outputs, for its backward: d_out shaped and typed
    like the activations (fp32 values and, for bf16 workloads, bf16 bit patterns in d_out_bits;
    values omitted for bf16 when values is False), dW_last [B,H,d,d] and db_last [B,H,d] fp32
    ([n,...] for a chain subset); every entry N(0, std^2).  A chain's draws do not depend on
    which other chains are drawn."""
    d = w.d
    draw = lambda seed, tag_, n, first: normal(seed, tag_, n, first, 0.0, std)
    vals = _window(w, "DO", d, 0, w.L, chains, draw)
    shape = (w.B, w.H, w.L, d) if chains is None else (len(chains), w.L, d)
    vals = vals.reshape(shape)
    out = {}
    if w.dtype == "bf16":
        out["d_out_bits"] = f32_to_bf16_bits(vals).reshape(shape)
        if values:
            out["d_out"] = bf16_bits_to_f32(out["d_out_bits"]).reshape(shape)
    else:
        out["d_out"] = vals
    ids = range(w.chains) if chains is None else chains
    lead = (w.B, w.H) if chains is None else (len(chains),)
    out["dW_last"] = np.stack([normal(w.seed, TAG["DWL"], d * d, c * d * d, 0.0, std) for c in ids]).reshape(*lead, d, d)
    out["db_last"] = np.stack([normal(w.seed, TAG["DBL"], d, c * d, 0.0, std) for c in ids]).reshape(*lead, d)
    return out


def state_inputs(w: Workload) -> dict:
    """Per-head initial state and LayerNorm parameters."""
    H, d = w.H, w.d
    out = {}
    if w.kind == "mlp":
        h = w.hidden
        out["W1"] = normal(w.seed, TAG["W1"], H * d * h, 0, 0.0, w.w_std).reshape(H, d, h)
        out["b1"] = np.zeros((H, h), np.float32)
        out["W2"] = normal(w.seed, TAG["W2"], H * h * d, 0, 0.0, w.w_std).reshape(H, h, d)
        out["b2"] = np.zeros((H, d), np.float32)
    else:
        out["W0"] = normal(w.seed, TAG["W0"], H * d * d, 0, 0.0, w.w_std).reshape(H, d, d)
        out["b0"] = np.zeros((H, d), np.float32)
    if w.ln == "unit":
        out["ln_w"] = np.ones((H, d), np.float32)
        out["ln_b"] = np.zeros((H, d), np.float32)
    else:
        out["ln_w"] = normal(w.seed, TAG["LNW"], H * d, 0, 1.0, w.ln_w_std).reshape(H, d)
        out["ln_b"] = normal(w.seed, TAG["LNB"], H * d, 0, 0.0, w.ln_b_std).reshape(H, d)
    return out


def random_bias(w: Workload, tag: str, shape, std: float = 0.02) -> np.ndarray:
    """A non-zero bias draw, for tests that must exercise the bias path."""
    n = int(np.prod(shape))
    return normal(w.seed, TAG[tag], n, 0, 0.0, std).reshape(shape)


def chain_index(b: int, h: int, H: int) -> int:
    return b * H + h


def oproj_inputs(seed: int, T: int, C: int, N: int, x_std: float = 1.0, w_std: float = 0.02,
                 ln_w_std: float = 0.1, ln_b_std: float = 0.1, values: bool = True) -> dict:
    """Inputs of the layer's output side (post_norm, then o_proj): X [T, C] bf16 shaped like the
    scan's output (XQ + LN(Zbar): about unit spread per feature), the o_proj weight Wo [N, C] bf16
    ~ N(0, w_std), post_norm's ln_w ~ 1 + N(0, ln_w_std) and ln_b ~ N(0, ln_b_std) [C] fp32.
    Returns X_bits / Wo_bits (uint16 bf16 patterns), and X / Wo as their fp32 values when asked."""
    x = normal(seed, TAG["ONX"], T * C, 0, 0.0, x_std).reshape(T, C)
    wo = normal(seed, TAG["ONW"], N * C, 0, 0.0, w_std).reshape(N, C)
    out = {"X_bits": f32_to_bf16_bits(x), "Wo_bits": f32_to_bf16_bits(wo),
           "ln_w": normal(seed, TAG["ONLW"], C, 0, 1.0, ln_w_std),
           "ln_b": normal(seed, TAG["ONLB"], C, 0, 0.0, ln_b_std)}
    if values:
        out["X"] = bf16_bits_to_f32(out["X_bits"])
        out["Wo"] = bf16_bits_to_f32(out["Wo_bits"])
    return out
