"""Parity of the TTT-Linear backward (ttt_linear_backward, through the C ABI) with the backward
oracle (oracle/ttt_backward.py, float64 reverse mode of the primal-form scan), chain by chain,
on seeded workloads: full mini-batches and ragged tails, token_eta tables, both dtypes, per-head
and per-chain initial states, several checkpoint groups, and the 1B layer's shapes on sampled
chains.

Tolerances (max over chains of the relative L2 error): float32 activations 1e-5 for every result
(the scan's fp32 bar; the FFMA kernel computes in float32 throughout, and the state's adjoint
sums a few hundred rank-16 terms per entry at these lengths); bfloat16 activations 1e-2 for every
result (the scan's bf16 bar): the tensor-core kernel takes its products with TF32 operands
(11-bit significands, like the forward's fp16 operands) and dXQ, dXK, dXV are rounded to bf16.
"""
import numpy as np
import pytest
import torch

import synth
from oracle import ttt_backward as bw
from parity_util import dev_act, dev_f32, rel_l2, sample_chains, to_np

pytestmark = pytest.mark.gpu

TOL32, TOL16 = 1e-5, 1e-2


def _tol(dt, k):
    return TOL16 if dt == "bf16" else TOL32


def _oracle(w, x, up, chains, per_chain_w0=False, token_eta=None, with_last=True):
    """Per-chain oracle gradients for the listed chains (x, up drawn for exactly those chains)."""
    H = w.H
    st = lambda a, c: a[c // H, c % H] if per_chain_w0 else a[c % H]
    W0 = np.stack([st(x["W0"], c) for c in chains])
    b0 = np.stack([st(x["b0"], c) for c in chains])
    lw = np.stack([x["ln_w"][c % H] for c in chains])
    lb = np.stack([x["ln_b"][c % H] for c in chains])
    return bw.linear_backward(x["XQ"], x["XK"], x["XV"], x["lr"], W0, b0, lw, lb, w.K, w.eps, up["d_out"],
                              up["dW_last"] if with_last else None, up["db_last"] if with_last else None,
                              token_eta=token_eta)


def _gpu(libttt, w, x, up, G, per_chain_w0=False, token_eta=None, with_last=True):
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    dout = dev_act(up, "d_out")
    W0, b0 = dev_f32(x["W0"]), dev_f32(x["b0"])
    if per_chain_w0:
        W0 = W0.unsqueeze(0).repeat(w.B, 1, 1, 1).contiguous() if W0.dim() == 3 else W0
        b0 = b0.unsqueeze(0).repeat(w.B, 1, 1).contiguous() if b0.dim() == 2 else b0
    te = None if token_eta is None else dev_f32(np.asarray(token_eta, np.float32))
    g = libttt.ttt_linear_backward(XQ, XK, XV, dev_f32(x["lr"]), W0, b0, dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), dout,
                                   dev_f32(up["dW_last"]) if with_last else None,
                                   dev_f32(up["db_last"]) if with_last else None,
                                   mini_batch=w.K, eps=w.eps, token_eta=te, ckpt_group=G)
    torch.cuda.synchronize()
    return g


def _head_sum(a, H):
    """[n_chains, ...] per-chain shares -> [H, ...] sums over the batch (chain c is head c % H)."""
    a = np.asarray(a)
    return a.reshape(-1, H, *a.shape[1:]).sum(axis=0)


def _compare(w, g, ref, per_chain_w0=False, tag=""):
    n = w.chains
    errs = {
        "dXQ": rel_l2(to_np(g["dXQ"]).reshape(n, -1), ref["dXQ"].reshape(n, -1)),
        "dXK": rel_l2(to_np(g["dXK"]).reshape(n, -1), ref["dXK"].reshape(n, -1)),
        "dXV": rel_l2(to_np(g["dXV"]).reshape(n, -1), ref["dXV"].reshape(n, -1)),
        "dlr": rel_l2(to_np(g["dlr"]).reshape(n, -1), ref["dlr"].reshape(n, -1)),
        "dln_w": rel_l2(to_np(g["dln_w"]), _head_sum(ref["dln_w"], w.H)),
        "dln_b": rel_l2(to_np(g["dln_b"]), _head_sum(ref["dln_b"], w.H)),
    }
    if per_chain_w0:
        errs["dW0"] = rel_l2(to_np(g["dW0"]).reshape(n, -1), ref["dW0"].reshape(n, -1))
        errs["db0"] = rel_l2(to_np(g["db0"]).reshape(n, -1), ref["db0"].reshape(n, -1))
    else:
        errs["dW0"] = rel_l2(to_np(g["dW0"]), _head_sum(ref["dW0"], w.H))
        errs["db0"] = rel_l2(to_np(g["db0"]), _head_sum(ref["db0"], w.H))
    print(f"[backward {tag}]", {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= _tol(w.dtype, k), (tag, k, v)


CASES = [  # (name, dtype, B, H, L, K, G, token_eta)
    ("f32_tail_groups", "f32", 2, 3, 16 * 3 + 5, 16, 2, None),
    ("f32_K4_eta_table", "f32", 1, 2, 37, 4, 3, [0.9, 0.5, 0.3, 0.2]),
    ("f32_tail_only", "f32", 2, 2, 10, 16, 4, None),
    ("f32_no_tail_G1", "f32", 1, 3, 64, 16, 1, None),
    ("f32_K1_online", "f32", 1, 2, 9, 1, 4, None),
    ("bf16_tail", "bf16", 2, 2, 16 * 8 + 7, 16, 4, None),
    ("bf16_no_tail", "bf16", 1, 4, 16 * 6, 16, 6, None),
    ("bf16_K8_tail", "bf16", 1, 3, 8 * 5 + 3, 8, 2, None),
    ("bf16_K4_eta_table", "bf16", 2, 1, 37, 4, 3, [0.9, 0.5, 0.3, 0.2]),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_backward_matches_oracle(libttt, case):
    name, dt, B, H, L, K, G, te = case
    w = synth.workload(1, B=B, H=H, L=L, K=K, dtype=dt, seed=0xB0 + L)
    x = synth.linear_inputs(w, chains=list(range(w.chains)))
    up = synth.upstream_grads(w, chains=list(range(w.chains)))
    ref = _oracle(w, x, up, range(w.chains), token_eta=te)
    xf = synth.linear_inputs(w)
    upf = synth.upstream_grads(w)
    g = _gpu(libttt, w, xf, upf, G, token_eta=te)
    _compare(w, g, ref, tag=name)


def test_backward_per_chain_state_and_no_upstream_state_grads(libttt):
    w = synth.workload(1, B=2, H=2, L=16 * 4 + 3, dtype="f32", seed=0xB1)
    ids = list(range(w.chains))
    x, up = synth.linear_inputs(w, chains=ids), synth.upstream_grads(w, chains=ids)
    # a per-chain initial state: each batch row gets the head's state scaled differently
    scale = np.array([1.0, 1.7], np.float32)
    xs = dict(x)
    xs["W0"] = np.stack([x["W0"] * s for s in scale])
    xs["b0"] = np.stack([x["b0"] + 0.05 * s for s in scale])
    ref = _oracle(w, xs, up, ids, per_chain_w0=True, with_last=False)
    xf, upf = synth.linear_inputs(w), synth.upstream_grads(w)
    xf["W0"], xf["b0"] = xs["W0"], xs["b0"]
    g = _gpu(libttt, w, xf, upf, 3, per_chain_w0=True, with_last=False)
    assert tuple(g["dW0"].shape) == (w.B, w.H, 64, 64)
    _compare(w, g, ref, per_chain_w0=True, tag="per-chain state, no dW_last")


def test_backward_results_do_not_depend_on_the_checkpoint_group(libttt):
    w = synth.workload(1, B=2, H=2, L=16 * 11 + 9, dtype="bf16", seed=0xB2)
    x, up = synth.linear_inputs(w), synth.upstream_grads(w)
    runs = [_gpu(libttt, w, x, up, G) for G in (1, 2, 4, 5, 11, 64)]
    for r in runs[1:]:
        for k in runs[0]:
            assert torch.equal(r[k], runs[0][k]), k


def test_backward_batch_sum_of_per_chain_state_grads(libttt):
    """dW0/db0 for a per-head state equal the batch sums of the per-chain gradients."""
    w = synth.workload(1, B=3, H=2, L=16 * 5 + 2, dtype="f32", seed=0xB3)
    x, up = synth.linear_inputs(w), synth.upstream_grads(w)
    shared = _gpu(libttt, w, x, up, 2)
    per = _gpu(libttt, w, x, up, 2, per_chain_w0=True)
    for k in ("dXQ", "dXK", "dXV", "dlr", "dln_w", "dln_b"):
        assert torch.equal(shared[k], per[k]), k
    torch.testing.assert_close(per["dW0"].sum(0), shared["dW0"], rtol=1e-5, atol=1e-6)
    torch.testing.assert_close(per["db0"].sum(0), shared["db0"], rtol=1e-5, atol=1e-6)


def test_backward_empty_sequence(libttt):
    w = synth.workload(1, B=2, H=3, L=0, dtype="bf16", seed=0xB4)
    up = synth.upstream_grads(w)
    x = synth.linear_inputs(w)
    e = torch.empty((w.B, w.H, 0, 64), dtype=torch.bfloat16, device="cuda")
    g = libttt.ttt_linear_backward(e, e, e, torch.empty((w.B, w.H, 0), device="cuda"), dev_f32(x["W0"]),
                                   dev_f32(x["b0"]), dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), e,
                                   dev_f32(up["dW_last"]), dev_f32(up["db_last"]), ckpt_group=4)
    torch.cuda.synchronize()
    np.testing.assert_allclose(to_np(g["dW0"]), up["dW_last"].sum(0), rtol=1e-6, atol=1e-6)
    np.testing.assert_allclose(to_np(g["db0"]), up["db_last"].sum(0), rtol=1e-6, atol=1e-6)
    assert not g["dln_w"].any() and not g["dln_b"].any()


def test_backward_long_sequence(libttt):
    """1027 tokens (64 full mini-batches and a tail of 3), float32: the adjoint through 64 updates."""
    w = synth.workload(1, B=1, H=2, L=16 * 64 + 3, dtype="f32", seed=0xB5)
    ids = list(range(w.chains))
    ref = _oracle(w, synth.linear_inputs(w, chains=ids), synth.upstream_grads(w, chains=ids), ids)
    g = _gpu(libttt, w, synth.linear_inputs(w), synth.upstream_grads(w), 8)
    _compare(w, g, ref, tag="L=1027")


def test_backward_1b_layer_sampled_chains(libttt):
    """The 1B layer's shapes (B=8, H=32, L=8192, bf16), the launch the bench times (ckpt_group 16),
    every output of sampled chains against the oracle; per-chain W0 tiles the per-head one so that
    dW0 and db0 come per chain."""
    w = synth.workload(2)
    x, up = synth.linear_inputs(w, values=False), synth.upstream_grads(w, values=False)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    W0 = dev_f32(x["W0"]).unsqueeze(0).repeat(w.B, 1, 1, 1).contiguous()
    b0 = dev_f32(x["b0"]).unsqueeze(0).repeat(w.B, 1, 1).contiguous()
    g = libttt.ttt_linear_backward(XQ, XK, XV, dev_f32(x["lr"]), W0, b0, dev_f32(x["ln_w"]), dev_f32(x["ln_b"]),
                                   dev_act(up, "d_out"), dev_f32(up["dW_last"]), dev_f32(up["db_last"]),
                                   mini_batch=w.K, eps=w.eps, ckpt_group=16)
    torch.cuda.synchronize()
    del XQ, XK, XV, x, up
    chains = sample_chains(w.chains, 3)
    xs, us = synth.linear_inputs(w, chains=chains), synth.upstream_grads(w, chains=chains)
    ref = _oracle(w, xs, us, chains)
    errs = {}
    for k in ("dXQ", "dXK", "dXV", "dlr", "dW0", "db0"):
        gk = to_np(g[k].reshape(w.chains, -1)[chains])
        errs[k] = rel_l2(gk, ref[k].reshape(len(chains), -1))
    print("[backward 1b sampled]", chains, {k: f"{v:.2e}" for k, v in errs.items()})
    for k, v in errs.items():
        assert v <= _tol("bf16", k), (k, v)


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_backward_token_major_gives_the_head_major_bits(libttt, dt):
    """[B,L,H,64] activations and gradients (TTT_FLAG_TOKEN_MAJOR): the same arithmetic as the
    head-major call, so the same bits."""
    w = synth.workload(1, B=2, H=3, L=16 * 4 + 5, dtype=dt, seed=0xB6)
    x, up = synth.linear_inputs(w), synth.upstream_grads(w)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    dout = dev_act(up, "d_out")
    common = [dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b")]
    last = (dev_f32(up["dW_last"]), dev_f32(up["db_last"]))
    gh = libttt.ttt_linear_backward(XQ, XK, XV, *common, dout, *last, mini_batch=w.K, eps=w.eps, ckpt_group=3)
    tm = lambda t: t.transpose(1, 2).contiguous()
    gt = libttt.ttt_linear_backward(tm(XQ), tm(XK), tm(XV), *common, tm(dout), *last, mini_batch=w.K, eps=w.eps,
                                    ckpt_group=3, token_major=True)
    torch.cuda.synchronize()
    for k in ("dXQ", "dXK", "dXV"):
        assert torch.equal(gt[k].transpose(1, 2), gh[k]), k
    for k in ("dlr", "dW0", "db0", "dln_w", "dln_b"):
        assert torch.equal(gt[k], gh[k]), k
