"""Training through the scan with torch.autograd (test_rnn_layers_b200.autograd.ttt_linear), and the
two backward kernels against each other.

* `.backward()` through ttt_linear gives the backward oracle's gradients for every input.
* The same values run as fp32 activations (the FFMA backward) and as bf16 activations (the
  tensor-core backward) give the same gradients within the bf16 bar.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ttt_backward as bw
from parity_util import dev_act, dev_f32, rel_l2, to_np

pytestmark = pytest.mark.gpu


def test_autograd_backward_matches_the_oracle(libttt):
    from test_rnn_layers_b200.autograd import ttt_linear
    w = synth.workload(1, B=2, H=2, L=16 * 3 + 7, seed=0xA6)
    ids = list(range(w.chains))
    x, up = synth.linear_inputs(w), synth.upstream_grads(w)
    leaves = [dev_act(x, n).requires_grad_() for n in ("XQ", "XK", "XV")]
    leaves += [dev_f32(x[k]).requires_grad_() for k in ("lr", "W0", "b0", "ln_w", "ln_b")]
    out, W_last, b_last = ttt_linear(*leaves, mini_batch=w.K, eps=w.eps, ckpt_group=2)
    R = dev_act(up, "d_out")  # bf16-exact, so the gradient reaching out is exactly these values
    loss = (out.float() * R.float()).sum() + (W_last * dev_f32(up["dW_last"])).sum() + (b_last * dev_f32(up["db_last"])).sum()
    loss.backward()
    torch.cuda.synchronize()
    xs, us = synth.linear_inputs(w, chains=ids), synth.upstream_grads(w, chains=ids)
    st = lambda a: np.stack([a[c % w.H] for c in ids])
    ref = bw.linear_backward(xs["XQ"], xs["XK"], xs["XV"], xs["lr"], st(xs["W0"]), st(xs["b0"]), st(xs["ln_w"]),
                             st(xs["ln_b"]), w.K, w.eps, us["d_out"], us["dW_last"], us["db_last"])
    n = w.chains
    head_sum = lambda a: np.asarray(a).reshape(w.B, w.H, *np.asarray(a).shape[1:]).sum(axis=0)
    errs = {}
    for name, leaf in zip(("dXQ", "dXK", "dXV", "dlr"), leaves[:4]):
        errs[name] = rel_l2(to_np(leaf.grad).reshape(n, -1), ref[name].reshape(n, -1))
    for name, leaf in zip(("dW0", "db0", "dln_w", "dln_b"), leaves[4:]):
        errs[name] = rel_l2(to_np(leaf.grad), head_sum(ref[name]))
    print("[autograd]", {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= 1e-2, (k, v)


def test_ffma_and_tensor_core_backwards_agree(libttt):
    w = synth.workload(1, B=2, H=3, L=16 * 4 + 5, seed=0xA7)
    x, up = synth.linear_inputs(w), synth.upstream_grads(w)
    common = [dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b")]
    act16 = [dev_act(x, n) for n in ("XQ", "XK", "XV")]
    act32 = [a.float() for a in act16]  # the same (bf16) values as fp32 activations
    d16 = dev_act(up, "d_out")
    last = (dev_f32(up["dW_last"]), dev_f32(up["db_last"]))
    g16 = libttt.ttt_linear_backward(*act16, *common, d16, *last, mini_batch=w.K, eps=w.eps, ckpt_group=3)
    g32 = libttt.ttt_linear_backward(*act32, *common, d16.float(), *last, mini_batch=w.K, eps=w.eps, ckpt_group=3)
    torch.cuda.synchronize()
    for k in g16:
        a, b = to_np(g16[k]), to_np(g32[k])
        lead = a.shape[0] * (a.shape[1] if a.ndim > 2 else 1)
        e = rel_l2(a.reshape(lead, -1), b.reshape(lead, -1))
        print(f"[ffma vs tensor cores] {k}: {e:.2e}")
        assert e <= 1e-2, (k, e)
