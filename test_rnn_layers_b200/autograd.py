"""torch.autograd face of the TTT-Linear scan, for training through it.

`ttt_linear(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, ...)` returns (out, W_last, b_last) like
`ttt_linear_forward`, recording the call so that `.backward()` reaches XQ, XK, XV, lr, W0, b0, ln_w
and ln_b through `ttt_linear_backward` (the scan's backward with checkpoint groups, the
walkthrough's training path through `scan`).  As in that path, the forward keeps the state at the
start of every checkpoint group (ttt_linear_forward_ckpt) and the backward rebuilds each group
from it (ttt_linear_backward_ckpt), instead of running the state recursion a second time.  Both
directions run in libttt.so's kernels; this module only passes tensors between autograd and the
C ABI.  token_eta, eps and the mini-batch size are constants.
"""
from __future__ import annotations

import torch

from . import _act_sizes, ttt_linear_backward, ttt_linear_ckpt_bytes, ttt_linear_forward


class _TTTLinear(torch.autograd.Function):
    @staticmethod
    def forward(ctx, XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch, eps, token_eta, ckpt_group, token_major):
        B, H, L, _ = _act_sizes(XQ, token_major)
        ckpt = torch.empty(ttt_linear_ckpt_bytes(B, H, L, mini_batch, ckpt_group) // 4, device=XQ.device)
        out, W_last, b_last = ttt_linear_forward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch=mini_batch, eps=eps,
                                                 token_eta=token_eta, token_major=token_major, ckpt=ckpt,
                                                 ckpt_group=ckpt_group)
        ctx.save_for_backward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, ckpt)
        ctx.cfg = (mini_batch, eps, token_eta, ckpt_group, token_major)
        return out, W_last, b_last

    @staticmethod
    def backward(ctx, d_out, dW_last, db_last):
        XQ, XK, XV, lr, W0, b0, ln_w, ln_b, ckpt = ctx.saved_tensors
        mini_batch, eps, token_eta, ckpt_group, token_major = ctx.cfg
        if d_out is None:
            d_out = torch.zeros_like(XQ)
        g = ttt_linear_backward(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, d_out.contiguous(),
                                None if dW_last is None else dW_last.contiguous(),
                                None if db_last is None else db_last.contiguous(),
                                mini_batch=mini_batch, eps=eps, token_eta=token_eta, ckpt_group=ckpt_group,
                                token_major=token_major, ckpt=ckpt)
        return (g["dXQ"], g["dXK"], g["dXV"], g["dlr"], g["dW0"], g["db0"], g["dln_w"], g["dln_b"],
                None, None, None, None, None)


def ttt_linear(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch: int = 16, eps: float = 1e-6, token_eta=None,
               ckpt_group: int = 16, token_major: bool = False):
    """(out, W_last, b_last) of the TTT-Linear scan over [B,H,L,64] activations ([B,L,H,64] with
    token_major), with gradients for every input (see ttt_linear_forward and ttt_linear_backward
    in include/ttt.h)."""
    return _TTTLinear.apply(XQ, XK, XV, lr, W0, b0, ln_w, ln_b, mini_batch, eps, token_eta, ckpt_group, token_major)
