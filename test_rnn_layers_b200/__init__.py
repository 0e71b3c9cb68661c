"""Python binding of libttt.so: the TTT-Linear / TTT-MLP scan and the decode step on B200.

Argument marshalling only -- every step of the computation runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  The functions carry the C-ABI names
(include/ttt.h); each checks the tensors it is handed, allocates missing outputs with torch,
calls the library and raises TTTError on a non-zero return code.

If libttt.so is missing this module raises on first use: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libttt.so")

TTT_OK = 0
TTT_ERR_ARG = -1
TTT_ERR_ALIGN = -2
TTT_ERR_ALIAS = -3
TTT_ERR_CUDA = -4
TTT_ERR_TIMEOUT = -5
TTT_ERR_UNSUPPORTED = -6
TTT_F32 = 0
TTT_BF16 = 1
TTT_FLAG_FP32_COMPUTE = 1
TTT_FLAG_TOKEN_MAJOR = 2
TTT_FLAG_ROPE_HALF_SPLIT = 4
TTT_STATUS_TIMEOUT = 1
TTT_STATIC_SCRATCH_BYTES = 33554432

EXPORTS = ("ttt_partition", "ttt_error_string", "ttt_last_error_message", "ttt_device_status",
           "ttt_set_wait_limit", "ttt_linear_forward", "ttt_linear_forward_rope", "ttt_linear_host_workspace_bytes",
           "ttt_linear_forward_host", "ttt_linear_forward_host_static", "ttt_mlp_forward",
           "ttt_linear_decode_step", "ttt_linear_decode_step_hist", "ttt_o_proj_prepare", "ttt_post_norm_o_proj",
           "ttt_linear_backward_workspace_bytes", "ttt_linear_backward", "ttt_linear_ckpt_bytes",
           "ttt_linear_forward_ckpt", "ttt_linear_backward_ckpt")


class TTTError(RuntimeError):
    def __init__(self, code: int, message: str):
        super().__init__(f"[{code}] {message}")
        self.code = code


_lib = None


def lib():
    """The loaded libttt.so with its signatures declared (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m test_rnn_layers_b200.build` "
                               "(there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        vp, fp, ll, i, u, f = (ctypes.c_void_p, ctypes.c_void_p, ctypes.c_longlong, ctypes.c_int,
                               ctypes.c_uint, ctypes.c_float)
        L.ttt_partition.argtypes = [ll, i, ctypes.POINTER(ll), ctypes.POINTER(ll)]
        L.ttt_error_string.argtypes = [i]
        L.ttt_error_string.restype = ctypes.c_char_p
        L.ttt_last_error_message.argtypes = []
        L.ttt_last_error_message.restype = ctypes.c_char_p
        L.ttt_device_status.argtypes = [vp, ctypes.POINTER(u), i]
        L.ttt_set_wait_limit.argtypes = [ll]
        L.ttt_linear_forward.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, i, u,
                                         vp, fp, fp, fp, fp, vp]
        L.ttt_linear_forward_rope.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, f, i, u,
                                              vp, fp, fp, fp, fp, vp]
        L.ttt_linear_host_workspace_bytes.argtypes = [i, i, ll, i, i, i, i, ll]
        L.ttt_linear_host_workspace_bytes.restype = ll
        L.ttt_linear_forward_host.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, i, u,
                                              vp, fp, fp, fp, fp, vp, ll, i, vp]
        L.ttt_linear_forward_host_static.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, i,
                                                     u, vp, fp, fp, fp, fp, vp]
        L.ttt_mlp_forward.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, i, f, i,
                                      u, vp, fp, fp, fp, fp, vp]
        L.ttt_linear_decode_step.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, i, i, i, i, ll, f, i,
                                             vp, vp]
        L.ttt_linear_decode_step_hist.argtypes = [vp, vp, vp, fp, fp, fp, fp, fp, fp, fp, fp, i, i, i, i, ll, f,
                                                  i, vp, vp]
        L.ttt_o_proj_prepare.argtypes = [vp, fp, fp, i, i, vp, fp, fp, vp]
        L.ttt_post_norm_o_proj.argtypes = [vp, ll, i, vp, fp, fp, i, f, vp, fp, vp]
        L.ttt_linear_backward_workspace_bytes.argtypes = [i, i, ll, i, i, i]
        L.ttt_linear_backward_workspace_bytes.restype = ll
        L.ttt_linear_backward.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, i, u, i, vp, fp,
                                          fp, vp, vp, vp, fp, fp, fp, fp, fp, vp, ll, vp]
        L.ttt_linear_ckpt_bytes.argtypes = [i, i, ll, i, i, i]
        L.ttt_linear_ckpt_bytes.restype = ll
        L.ttt_linear_forward_ckpt.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, i, u,
                                              vp, fp, fp, fp, fp, i, fp, vp]
        L.ttt_linear_backward_ckpt.argtypes = [vp, vp, vp, fp, fp, fp, fp, ll, fp, fp, i, i, ll, i, i, f, i, u, i, fp,
                                               vp, fp, fp, vp, vp, vp, fp, fp, fp, fp, fp, vp, ll, vp]
        for name in ("ttt_partition", "ttt_device_status", "ttt_set_wait_limit", "ttt_linear_forward",
                     "ttt_o_proj_prepare", "ttt_post_norm_o_proj",
                     "ttt_linear_forward_rope",
                     "ttt_linear_forward_host", "ttt_linear_forward_host_static", "ttt_mlp_forward", "ttt_linear_decode_step",
                     "ttt_linear_decode_step_hist", "ttt_linear_backward", "ttt_linear_forward_ckpt",
                     "ttt_linear_backward_ckpt"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(rc: int):
    if rc != TTT_OK:
        raise TTTError(rc, lib().ttt_last_error_message().decode() or lib().ttt_error_string(rc).decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TTT_F32
    if t.dtype == torch.bfloat16:
        return TTT_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _need(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def _act_sizes(XQ, token_major: bool):
    """(B, H, L, d) of activations laid out [B,H,L,d], or [B,L,H,d] when token_major."""
    if XQ.dim() != 4:
        raise ValueError(f"XQ must be 4-D, got shape {tuple(XQ.shape)}")
    if token_major:
        B, L, H, d = XQ.shape
    else:
        B, H, L, d = XQ.shape
    return B, H, L, d


def ttt_partition(L: int, mini_batch: int):
    """(n_full, rem) = (L // K, L % K), computed by the library (host-only)."""
    n, r = ctypes.c_longlong(), ctypes.c_longlong()
    _check(lib().ttt_partition(L, mini_batch, ctypes.byref(n), ctypes.byref(r)))
    return n.value, r.value


def ttt_set_wait_limit(polls: int = 0):
    """Cap the polls of bounded device waits of later launches (0 = default).  A test hook."""
    _check(lib().ttt_set_wait_limit(polls))


def ttt_device_status(clear: bool = True, stream=None) -> int:
    """Synchronise the stream and return the device status bits; raises TTTError on a timeout."""
    v = ctypes.c_uint()
    _check(lib().ttt_device_status(_stream(stream), ctypes.byref(v), 1 if clear else 0))
    return v.value


def ttt_linear_forward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch: int = 16, eps: float = 1e-6,
                       token_eta=None, out=None, W_last=None, b_last=None, W_grad_tail=None,
                       b_grad_tail=None, tail_grads: bool = False, flags: int = 0, token_major: bool = False,
                       stream=None, ckpt=None, ckpt_group: int = 16):
    """TTT-Linear prefill over [B,H,L,64] activations, or [B,L,H,64] with token_major (see include/ttt.h).

    W0/b0: [H,64,64]/[H,64] shared over the batch, or [B,H,64,64]/[B,H,64] per chain.
    ckpt: a float32 CUDA tensor of ttt_linear_ckpt_bytes(...) bytes to receive the checkpoints of
    ttt_linear_backward (ttt_linear_forward_ckpt: the state before every ckpt_group-th full
    mini-batch, then the state after the last), or None.
    Returns (out, W_last, b_last) or, with tail_grads, (out, W_last, b_last, W_grad_tail, b_grad_tail).
    """
    return _linear_forward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch, eps, token_eta, out, W_last, b_last,
                           W_grad_tail, b_grad_tail, tail_grads, flags, token_major, stream, None, ckpt, ckpt_group)


def ttt_linear_forward_rope(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch: int = 16, eps: float = 1e-6,
                            rope_theta: float = 10000.0, half_split: bool = False, token_eta=None, out=None,
                            W_last=None, b_last=None, W_grad_tail=None, b_grad_tail=None,
                            tail_grads: bool = False, flags: int = 0, token_major: bool = False, stream=None):
    """ttt_linear_forward with the rotary embedding of XQ and XK (positions t mod K) fused into the scan.

    Pairs (2k, 2k+1), or (k, k+32) with half_split; bf16 activations only (see include/ttt.h).
    """
    flags |= TTT_FLAG_ROPE_HALF_SPLIT if half_split else 0
    return _linear_forward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch, eps, token_eta, out, W_last, b_last,
                           W_grad_tail, b_grad_tail, tail_grads, flags, token_major, stream, rope_theta)


def ttt_linear_ckpt_bytes(B: int, H: int, L: int, mini_batch: int = 16, ckpt_group: int = 16, d: int = 64) -> int:
    """Bytes of the checkpoint buffer of ttt_linear_forward(..., ckpt=) and ttt_linear_backward(..., ckpt=)."""
    n = lib().ttt_linear_ckpt_bytes(B, H, L, d, mini_batch, ckpt_group)
    if n < 0:
        _check(int(n))
    return int(n)


def _linear_forward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch, eps, token_eta, out, W_last, b_last,
                    W_grad_tail, b_grad_tail, tail_grads, flags, token_major, stream, rope_theta, ckpt=None,
                    ckpt_group=16):
    _need(XQ, "XQ")
    B, H, L, d = _act_sizes(XQ, token_major)
    flags |= TTT_FLAG_TOKEN_MAJOR if token_major else 0
    dt = XQ.dtype
    for n, t in (("XK", XK), ("XV", XV)):
        _need(t, n, dt, XQ.shape)
    _need(lr, "lr", torch.float32, (B, H, L))
    per_chain = W0.dim() == 4
    _need(W0, "W0", torch.float32, (B, H, d, d) if per_chain else (H, d, d))
    _need(b0, "b0", torch.float32, (B, H, d) if per_chain else (H, d))
    _need(ln_w, "ln_w", torch.float32, (H, d))
    _need(ln_b, "ln_b", torch.float32, (H, d))
    if token_eta is not None:
        _need(token_eta, "token_eta", torch.float32, (mini_batch,))
    dev = XQ.device
    out = torch.empty_like(XQ) if out is None else _need(out, "out", dt, XQ.shape)
    W_last = torch.empty((B, H, d, d), device=dev) if W_last is None else _need(W_last, "W_last", torch.float32, (B, H, d, d))
    b_last = torch.empty((B, H, d), device=dev) if b_last is None else _need(b_last, "b_last", torch.float32, (B, H, d))
    if tail_grads:
        W_grad_tail = torch.empty((B, H, d, d), device=dev) if W_grad_tail is None else W_grad_tail
        b_grad_tail = torch.empty((B, H, d), device=dev) if b_grad_tail is None else b_grad_tail
    head = (_ptr(XQ), _ptr(XK), _ptr(XV), _ptr(lr), _ptr(token_eta), _ptr(W0), _ptr(b0),
            H * d * d if per_chain else 0, _ptr(ln_w), _ptr(ln_b), B, H, L, d, mini_batch, eps)
    tail = (_dtype_code(XQ), flags, _ptr(out), _ptr(W_last), _ptr(b_last), _ptr(W_grad_tail), _ptr(b_grad_tail),
            _stream(stream))
    if ckpt is not None:
        _need(ckpt, "ckpt", torch.float32)
        if ckpt.numel() * 4 < ttt_linear_ckpt_bytes(B, H, L, mini_batch, ckpt_group, d):
            raise ValueError("ckpt is smaller than ttt_linear_ckpt_bytes(...)")
        rc = lib().ttt_linear_forward_ckpt(*head, *tail[:-1], ckpt_group, _ptr(ckpt), tail[-1])
    elif rope_theta is None:
        rc = lib().ttt_linear_forward(*head, *tail)
    else:
        rc = lib().ttt_linear_forward_rope(*head, rope_theta, *tail)
    _check(rc)
    if tail_grads:
        return out, W_last, b_last, W_grad_tail, b_grad_tail
    return out, W_last, b_last


def _need_host(t, name, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor for the host-buffer entry point")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t


def ttt_linear_host_workspace_bytes(B: int, H: int, L: int, mini_batch: int = 16, dtype=torch.bfloat16,
                                    chunk_batches: int = 1, per_chain_state: bool = False, d: int = 64) -> int:
    """Bytes of device workspace that ttt_linear_forward_host needs (host-only)."""
    code = TTT_BF16 if dtype == torch.bfloat16 else TTT_F32
    n = lib().ttt_linear_host_workspace_bytes(B, H, L, d, mini_batch, code, chunk_batches,
                                              H * d * d if per_chain_state else 0)
    if n < 0:
        _check(int(n))
    return int(n)


def ttt_linear_forward_host(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch: int = 16, eps: float = 1e-6,
                            token_eta=None, out=None, W_last=None, b_last=None, W_grad_tail=None,
                            b_grad_tail=None, tail_grads: bool = False, flags: int = 0, chunk_batches: int = 1,
                            workspace=None, token_major: bool = False, stream=None):
    """ttt_linear_forward on HOST tensors (pin them for overlap): the batch streams through the
    GPU in chunks of `chunk_batches` batch rows, copies in both directions overlapping the scan.
    `workspace`: a CUDA uint8 tensor of at least ttt_linear_host_workspace_bytes(...) bytes, or
    None (allocated here).  Outputs are host tensors (pinned when allocated here).
    Asynchronous on `stream`: synchronise before reading the outputs.
    Returns (out, W_last, b_last) or, with tail_grads, (out, W_last, b_last, W_grad_tail, b_grad_tail)."""
    _need_host(XQ, "XQ")
    B, H, L, d = _act_sizes(XQ, token_major)
    flags |= TTT_FLAG_TOKEN_MAJOR if token_major else 0
    dt = XQ.dtype
    for n, t in (("XK", XK), ("XV", XV)):
        _need_host(t, n, dt, XQ.shape)
    _need_host(lr, "lr", torch.float32, (B, H, L))
    per_chain = W0.dim() == 4
    _need_host(W0, "W0", torch.float32, (B, H, d, d) if per_chain else (H, d, d))
    _need_host(b0, "b0", torch.float32, (B, H, d) if per_chain else (H, d))
    _need_host(ln_w, "ln_w", torch.float32, (H, d))
    _need_host(ln_b, "ln_b", torch.float32, (H, d))
    if token_eta is not None:
        _need_host(token_eta, "token_eta", torch.float32, (mini_batch,))

    def host(shape, dtype):
        return torch.empty(shape, dtype=dtype, pin_memory=True)

    out = host(XQ.shape, dt) if out is None else _need_host(out, "out", dt, XQ.shape)
    W_last = host((B, H, d, d), torch.float32) if W_last is None else _need_host(W_last, "W_last", torch.float32, (B, H, d, d))
    b_last = host((B, H, d), torch.float32) if b_last is None else _need_host(b_last, "b_last", torch.float32, (B, H, d))
    if tail_grads:
        W_grad_tail = host((B, H, d, d), torch.float32) if W_grad_tail is None else W_grad_tail
        b_grad_tail = host((B, H, d), torch.float32) if b_grad_tail is None else b_grad_tail
    need = ttt_linear_host_workspace_bytes(B, H, L, mini_batch, dt, chunk_batches, per_chain, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    _need(workspace, "workspace", torch.uint8)
    rc = lib().ttt_linear_forward_host(_ptr(XQ), _ptr(XK), _ptr(XV), _ptr(lr), _ptr(token_eta), _ptr(W0), _ptr(b0),
                                       H * d * d if per_chain else 0, _ptr(ln_w), _ptr(ln_b), B, H, L, d, mini_batch,
                                       eps, _dtype_code(XQ), flags, _ptr(out), _ptr(W_last), _ptr(b_last),
                                       _ptr(W_grad_tail), _ptr(b_grad_tail), _ptr(workspace), workspace.numel(),
                                       chunk_batches, _stream(stream))
    _check(rc)
    if tail_grads:
        return out, W_last, b_last, W_grad_tail, b_grad_tail
    return out, W_last, b_last


def ttt_linear_forward_host_static(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch: int = 16, eps: float = 1e-6,
                                   token_eta=None, out=None, W_last=None, b_last=None, W_grad_tail=None,
                                   b_grad_tail=None, tail_grads: bool = False, flags: int = 0,
                                   token_major: bool = False, stream=None):
    """ttt_linear_forward_host without a workspace: the library stages the batch through its
    built-in device scratch (TTT_STATIC_SCRATCH_BYTES per device) and allocates nothing, for
    callers that cannot allocate device memory.  Calls that overlap on the GPU race on that
    scratch; order them on one stream.  Host tensors in and out (pin them for faster copies);
    asynchronous on `stream`: synchronise before reading the outputs.
    Returns (out, W_last, b_last) or, with tail_grads, (out, W_last, b_last, W_grad_tail, b_grad_tail)."""
    _need_host(XQ, "XQ")
    B, H, L, d = _act_sizes(XQ, token_major)
    flags |= TTT_FLAG_TOKEN_MAJOR if token_major else 0
    dt = XQ.dtype
    for n, t in (("XK", XK), ("XV", XV)):
        _need_host(t, n, dt, XQ.shape)
    _need_host(lr, "lr", torch.float32, (B, H, L))
    per_chain = W0.dim() == 4
    _need_host(W0, "W0", torch.float32, (B, H, d, d) if per_chain else (H, d, d))
    _need_host(b0, "b0", torch.float32, (B, H, d) if per_chain else (H, d))
    _need_host(ln_w, "ln_w", torch.float32, (H, d))
    _need_host(ln_b, "ln_b", torch.float32, (H, d))
    if token_eta is not None:
        _need_host(token_eta, "token_eta", torch.float32, (mini_batch,))

    def host(shape, dtype):
        return torch.empty(shape, dtype=dtype, pin_memory=True)

    out = host(XQ.shape, dt) if out is None else _need_host(out, "out", dt, XQ.shape)
    W_last = host((B, H, d, d), torch.float32) if W_last is None else _need_host(W_last, "W_last", torch.float32, (B, H, d, d))
    b_last = host((B, H, d), torch.float32) if b_last is None else _need_host(b_last, "b_last", torch.float32, (B, H, d))
    if tail_grads:
        W_grad_tail = host((B, H, d, d), torch.float32) if W_grad_tail is None else W_grad_tail
        b_grad_tail = host((B, H, d), torch.float32) if b_grad_tail is None else b_grad_tail
    rc = lib().ttt_linear_forward_host_static(_ptr(XQ), _ptr(XK), _ptr(XV), _ptr(lr), _ptr(token_eta), _ptr(W0),
                                              _ptr(b0), H * d * d if per_chain else 0, _ptr(ln_w), _ptr(ln_b), B, H,
                                              L, d, mini_batch, eps, _dtype_code(XQ), flags, _ptr(out), _ptr(W_last),
                                              _ptr(b_last), _ptr(W_grad_tail), _ptr(b_grad_tail), _stream(stream))
    _check(rc)
    if tail_grads:
        return out, W_last, b_last, W_grad_tail, b_grad_tail
    return out, W_last, b_last


def ttt_mlp_forward(XQ, XK, XV, lr, W1, b1, W2, b2, ln_w, ln_b, mini_batch: int = 16, eps: float = 1e-6,
                    token_eta=None, out=None, flags: int = 0, token_major: bool = False, stream=None):
    """TTT-MLP prefill; states W1 [H,64,256], b1 [H,256], W2 [H,256,64], b2 [H,64] (or per chain).
    Activations [B,H,L,64], or [B,L,H,64] with token_major.

    Returns (out, W1_last, b1_last, W2_last, b2_last).
    """
    _need(XQ, "XQ")
    B, H, L, d = _act_sizes(XQ, token_major)
    flags |= TTT_FLAG_TOKEN_MAJOR if token_major else 0
    dt = XQ.dtype
    for n, t in (("XK", XK), ("XV", XV)):
        _need(t, n, dt, XQ.shape)
    _need(lr, "lr", torch.float32, (B, H, L))
    hid = W1.shape[-1]
    per_chain = W1.dim() == 4
    pre = (B, H) if per_chain else (H,)
    _need(W1, "W1", torch.float32, pre + (d, hid))
    _need(b1, "b1", torch.float32, pre + (hid,))
    _need(W2, "W2", torch.float32, pre + (hid, d))
    _need(b2, "b2", torch.float32, pre + (d,))
    _need(ln_w, "ln_w", torch.float32, (H, d))
    _need(ln_b, "ln_b", torch.float32, (H, d))
    if token_eta is not None:
        _need(token_eta, "token_eta", torch.float32, (mini_batch,))
    dev = XQ.device
    out = torch.empty_like(XQ) if out is None else _need(out, "out", dt, XQ.shape)
    W1l = torch.empty((B, H, d, hid), device=dev)
    b1l = torch.empty((B, H, hid), device=dev)
    W2l = torch.empty((B, H, hid, d), device=dev)
    b2l = torch.empty((B, H, d), device=dev)
    rc = lib().ttt_mlp_forward(_ptr(XQ), _ptr(XK), _ptr(XV), _ptr(lr), _ptr(token_eta), _ptr(W1), _ptr(b1),
                               _ptr(W2), _ptr(b2), H * d * hid if per_chain else 0, _ptr(ln_w), _ptr(ln_b),
                               B, H, L, d, hid, mini_batch, eps, _dtype_code(XQ), flags, _ptr(out), _ptr(W1l),
                               _ptr(b1l), _ptr(W2l), _ptr(b2l), _stream(stream))
    _check(rc)
    return out, W1l, b1l, W2l, b2l


def ttt_linear_decode_step(xq, xk, xv, lr, ln_w, ln_b, W, b, W_grad, b_grad, seqlen_offset: int,
                           mini_batch: int = 16, eps: float = 1e-6, token_eta=None, out=None, stream=None):
    """One decode token per chain ([B,H,64] inputs) through the cache state (W, b, W_grad, b_grad),
    which is updated in place.  Returns out [B,H,64]."""
    _need(xq, "xq")
    B, H, d = xq.shape
    dt = xq.dtype
    for n, t in (("xk", xk), ("xv", xv)):
        _need(t, n, dt, xq.shape)
    _need(lr, "lr", torch.float32, (B, H))
    _need(ln_w, "ln_w", torch.float32, (H, d))
    _need(ln_b, "ln_b", torch.float32, (H, d))
    _need(W, "W", torch.float32, (B, H, d, d))
    _need(b, "b", torch.float32, (B, H, d))
    _need(W_grad, "W_grad", torch.float32, (B, H, d, d))
    _need(b_grad, "b_grad", torch.float32, (B, H, d))
    if token_eta is not None:
        _need(token_eta, "token_eta", torch.float32, (mini_batch,))
    out = torch.empty_like(xq) if out is None else _need(out, "out", dt, xq.shape)
    rc = lib().ttt_linear_decode_step(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(lr), _ptr(token_eta), _ptr(ln_w),
                                      _ptr(ln_b), _ptr(W), _ptr(b), _ptr(W_grad), _ptr(b_grad), B, H, d,
                                      mini_batch, seqlen_offset, eps, _dtype_code(xq), _ptr(out), _stream(stream))
    _check(rc)
    return out


def ttt_linear_decode_step_hist(xq, xk, xv, lr, ln_w, ln_b, W, b, hist, b_grad, seqlen_offset: int,
                                mini_batch: int = 16, eps: float = 1e-6, token_eta=None, out=None, stream=None):
    """One decode token per chain ([B,H,64] inputs) through a history-format cache: W [B,H,64,64],
    b [B,H,64], hist [B,H,K,2,64] (rows (lr_j xk_j, g_j) of the current mini-batch), b_grad
    [B,H,64], all updated in place.  Start it at a mini-batch boundary with b_grad = 0.
    Returns out [B,H,64]."""
    _need(xq, "xq")
    B, H, d = xq.shape
    dt = xq.dtype
    for n, t in (("xk", xk), ("xv", xv)):
        _need(t, n, dt, xq.shape)
    _need(lr, "lr", torch.float32, (B, H))
    _need(ln_w, "ln_w", torch.float32, (H, d))
    _need(ln_b, "ln_b", torch.float32, (H, d))
    _need(W, "W", torch.float32, (B, H, d, d))
    _need(b, "b", torch.float32, (B, H, d))
    _need(hist, "hist", torch.float32, (B, H, mini_batch, 2, d))
    _need(b_grad, "b_grad", torch.float32, (B, H, d))
    if token_eta is not None:
        _need(token_eta, "token_eta", torch.float32, (mini_batch,))
    out = torch.empty_like(xq) if out is None else _need(out, "out", dt, xq.shape)
    rc = lib().ttt_linear_decode_step_hist(_ptr(xq), _ptr(xk), _ptr(xv), _ptr(lr), _ptr(token_eta), _ptr(ln_w),
                                           _ptr(ln_b), _ptr(W), _ptr(b), _ptr(hist), _ptr(b_grad), B, H, d,
                                           mini_batch, seqlen_offset, eps, _dtype_code(xq), _ptr(out), _stream(stream))
    _check(rc)
    return out


def ttt_o_proj_prepare(Wo, ln_w, ln_b, Wp=None, u=None, v=None, stream=None):
    """Pack o_proj's weight Wo [N, C] (bf16, nn.Linear layout) with post_norm's ln_w, ln_b [C]:
    returns (Wp, u, v) for ttt_post_norm_o_proj (see include/ttt.h)."""
    _need(Wo, "Wo", torch.bfloat16)
    if Wo.dim() != 2:
        raise ValueError("Wo must be [N, C]")
    N, C = Wo.shape
    _need(ln_w, "ln_w", torch.float32, (C,))
    _need(ln_b, "ln_b", torch.float32, (C,))
    dev = Wo.device
    Wp = torch.empty_like(Wo) if Wp is None else _need(Wp, "Wp", torch.bfloat16, (N, C))
    u = torch.empty(N, device=dev) if u is None else _need(u, "u", torch.float32, (N,))
    v = torch.empty(N, device=dev) if v is None else _need(v, "v", torch.float32, (N,))
    _check(lib().ttt_o_proj_prepare(_ptr(Wo), _ptr(ln_w), _ptr(ln_b), C, N, _ptr(Wp), _ptr(u), _ptr(v),
                                    _stream(stream)))
    return Wp, u, v


def ttt_post_norm_o_proj(X, Wp, u, v, eps: float = 1e-6, Y=None, row_stats=None, stream=None):
    """Y = o_proj(post_norm(X)) for X [..., C] bf16 (the token-major scan output), with (Wp, u, v)
    from ttt_o_proj_prepare; returns Y [..., N] bf16 (row_stats, [T, 2] fp32, receives each token's
    post_norm mean and 1/sqrt(var + eps))."""
    _need(X, "X", torch.bfloat16)
    _need(Wp, "Wp", torch.bfloat16)
    N, C = Wp.shape
    if X.shape[-1] != C:
        raise ValueError(f"X's last dimension must be C = {C}, got {tuple(X.shape)}")
    _need(u, "u", torch.float32, (N,))
    _need(v, "v", torch.float32, (N,))
    T = X.numel() // C
    Y = torch.empty((*X.shape[:-1], N), dtype=torch.bfloat16, device=X.device) if Y is None else \
        _need(Y, "Y", torch.bfloat16, (*X.shape[:-1], N))
    row_stats = torch.empty((T, 2), device=X.device) if row_stats is None else _need(row_stats, "row_stats", torch.float32, (T, 2))
    _check(lib().ttt_post_norm_o_proj(_ptr(X), T, C, _ptr(Wp), _ptr(u), _ptr(v), N, eps, _ptr(Y), _ptr(row_stats),
                                      _stream(stream)))
    return Y


def ttt_linear_backward_workspace_bytes(B: int, H: int, L: int, mini_batch: int = 16, ckpt_group: int = 16,
                                        d: int = 64) -> int:
    """Bytes of device workspace that ttt_linear_backward needs (host-only)."""
    n = lib().ttt_linear_backward_workspace_bytes(B, H, L, d, mini_batch, ckpt_group)
    if n < 0:
        _check(int(n))
    return int(n)


def ttt_linear_backward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, d_out, dW_last=None, db_last=None,
                        mini_batch: int = 16, eps: float = 1e-6, token_eta=None, ckpt_group: int = 16,
                        token_major: bool = False, workspace=None, stream=None, ckpt=None):
    """Gradients of <d_out, out> + <dW_last, W_last> + <db_last, b_last> for ttt_linear_forward's
    inputs ([B,H,L,64], or [B,L,H,64] with token_major; see include/ttt.h).
    ckpt: the checkpoints ttt_linear_forward(..., ckpt=, ckpt_group=) wrote for the same inputs and
    ckpt_group (ttt_linear_backward_ckpt: the backward then skips its own pass of the state
    recursion), or None.

    Returns a dict: dXQ, dXK, dXV (the activations' dtype), dlr [B,H,L], dW0/db0 (per head when W0
    is [H,64,64], per chain when it is [B,H,64,64]), dln_w/dln_b [H,64].
    """
    _need(XQ, "XQ")
    B, H, L, d = _act_sizes(XQ, token_major)
    dt = XQ.dtype
    for n, t in (("XK", XK), ("XV", XV), ("d_out", d_out)):
        _need(t, n, dt, XQ.shape)
    _need(lr, "lr", torch.float32, (B, H, L))
    per_chain = W0.dim() == 4
    _need(W0, "W0", torch.float32, (B, H, d, d) if per_chain else (H, d, d))
    _need(b0, "b0", torch.float32, (B, H, d) if per_chain else (H, d))
    _need(ln_w, "ln_w", torch.float32, (H, d))
    _need(ln_b, "ln_b", torch.float32, (H, d))
    if dW_last is not None:
        _need(dW_last, "dW_last", torch.float32, (B, H, d, d))
    if db_last is not None:
        _need(db_last, "db_last", torch.float32, (B, H, d))
    if token_eta is not None:
        _need(token_eta, "token_eta", torch.float32, (mini_batch,))
    dev = XQ.device
    ws_bytes = ttt_linear_backward_workspace_bytes(B, H, L, mini_batch, ckpt_group, d)
    if workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    else:
        _need(workspace, "workspace", torch.uint8)
    g = {"dXQ": torch.empty_like(XQ), "dXK": torch.empty_like(XQ), "dXV": torch.empty_like(XQ),
         "dlr": torch.empty((B, H, L), device=dev),
         "dW0": torch.empty(W0.shape, device=dev), "db0": torch.empty(b0.shape, device=dev),
         "dln_w": torch.empty((H, d), device=dev), "dln_b": torch.empty((H, d), device=dev)}
    head = (_ptr(XQ), _ptr(XK), _ptr(XV), _ptr(lr), _ptr(token_eta), _ptr(W0), _ptr(b0),
            H * d * d if per_chain else 0, _ptr(ln_w), _ptr(ln_b), B, H, L, d, mini_batch, eps, _dtype_code(XQ),
            TTT_FLAG_TOKEN_MAJOR if token_major else 0, ckpt_group)
    tail = (_ptr(d_out), _ptr(dW_last), _ptr(db_last), _ptr(g["dXQ"]), _ptr(g["dXK"]), _ptr(g["dXV"]), _ptr(g["dlr"]),
            _ptr(g["dW0"]), _ptr(g["db0"]), _ptr(g["dln_w"]), _ptr(g["dln_b"]), _ptr(workspace), workspace.numel(),
            _stream(stream))
    if ckpt is None:
        _check(lib().ttt_linear_backward(*head, *tail))
    else:
        _need(ckpt, "ckpt", torch.float32)
        if ckpt.numel() * 4 < ttt_linear_ckpt_bytes(B, H, L, mini_batch, ckpt_group, d):
            raise ValueError("ckpt is smaller than ttt_linear_ckpt_bytes(...)")
        _check(lib().ttt_linear_backward_ckpt(*head, _ptr(ckpt), *tail))
    return g
