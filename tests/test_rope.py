"""Rotary position embedding fused into the TTT-Linear prefill (ttt_linear_forward_rope), through
the C ABI on the GPU, against the oracle.

The expected values are the oracle's RoPE step (the walkthrough, "代码连连看——TTT",
TTTBase.forward: rotary_emb at position_ids % mini_batch_size, apply_rotary_pos_emb between
permute_qk and undo_permute_qk) applied to XQ and XK, then the oracle's scan on the rotated
values -- both in float64.  The kernel rotates in fp32 and rounds the rotated activations to fp16,
its tensor-core operand type, so the bar is the bf16 build's: 1e-2 max relative L2 per chain, on
out, W_last, b_last and the tail grads.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import chain_slice, dev_act, dev_f32, rel_l2, sample_chains, to_np

pytestmark = pytest.mark.gpu

TOL = 1e-2
NAMES = ("out", "W_last", "b_last", "W_grad_tail", "b_grad_tail")


def _gpu(ttt, x, w, theta, half, token_major=False, te=None):
    acts = [dev_act(x, n) for n in ("XQ", "XK", "XV")]
    if token_major:
        acts = [a.transpose(1, 2).contiguous() for a in acts]
    res = ttt.ttt_linear_forward_rope(*acts, dev_f32(x["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]),
                                      dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps,
                                      rope_theta=theta, half_split=half, tail_grads=True,
                                      token_major=token_major, token_eta=None if te is None else dev_f32(te))
    torch.cuda.synchronize()
    return res


def _oracle(x, w, theta, half, chains=None, te=None):
    orc = oracle.default()
    if chains is None:
        XQ, XK, XV, lr = x["XQ"], x["XK"], x["XV"], x["lr"]
    else:
        XQ, XK, XV, lr = (x[k].reshape(w.chains, *x[k].shape[2:])[chains] for k in ("XQ", "XK", "XV", "lr"))
    rq, rk = orc.rope(XQ, w.K, theta, half), orc.rope(XK, w.K, theta, half)
    return orc.linear_forward(rq, rk, XV, lr, x["W0"], x["b0"], x["ln_w"], x["ln_b"], w.K, w.eps,
                              None if te is None else te.astype(np.float64), chains=chains)


def _errs(res, ref, chains=None):
    n = len(chains) if chains is not None else None
    e = {}
    for name, t in zip(NAMES, res):
        got = chain_slice(t, chains, t.shape[1]) if chains is not None else to_np(t).reshape(-1, *t.shape[2:])
        e[name] = rel_l2(got.reshape(n or got.shape[0], -1), ref[name].reshape(ref[name].shape[0], -1))
    return e


@pytest.mark.parametrize("half", [False, True], ids=["pairs_2k_2k1", "half_split"])
@pytest.mark.parametrize("theta", [10000.0, 100.0])
@pytest.mark.parametrize("K,L", [(16, 16 * 19 + 7), (16, 16), (16, 5), (8, 8 * 5 + 3), (3, 20), (1, 9)])
def test_rope_against_oracle(libttt, half, theta, K, L):
    """Several tiles and a ragged tail, one exact mini-batch, a sequence shorter than K, small K
    (positions wrap every K tokens), K = 1 (every position 0: the rotation is the identity)."""
    w = synth.workload(1, B=2, H=3, L=L, K=K, seed=0x2075 + 31 * L + K)
    x = synth.linear_inputs(w)
    e = _errs(_gpu(libttt, x, w, theta, half), _oracle(x, w, theta, half))
    print(f"\n[rope] half={half} theta={theta} K={K} L={L}:", {k: f"{v:.2e}" for k, v in e.items()})
    assert max(e.values()) <= TOL, e


def test_rope_with_token_eta_and_token_major(libttt):
    """Token-major activations give the bits of the head-major call; with a token_eta table."""
    w = synth.workload(1, B=3, H=5, L=16 * 6 + 11, seed=0x2076)
    x = synth.linear_inputs(w)
    te = np.linspace(1.0, 0.3, 16).astype(np.float32)
    hm = _gpu(libttt, x, w, 10000.0, False, te=te)
    tm = _gpu(libttt, x, w, 10000.0, False, token_major=True, te=te)
    assert torch.equal(tm[0].transpose(1, 2), hm[0])
    for a, b in zip(hm[1:], tm[1:]):
        assert torch.equal(a, b)
    e = _errs(hm, _oracle(x, w, 10000.0, False, te=te))
    assert max(e.values()) <= TOL, e


def test_rope_is_applied(libttt):
    """The rotated scan is far from the unrotated oracle and from the other pair convention, so a
    kernel that skipped the rotation or swapped the pairs would fail the parity tests above."""
    w = synth.workload(1, B=1, H=2, L=16 * 8 + 3, seed=0x2077)
    x = synth.linear_inputs(w)
    res = _gpu(libttt, x, w, 100.0, False)
    plain = oracle.default().linear_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"], x["b0"], x["ln_w"],
                                            x["ln_b"], w.K, w.eps)
    assert _errs(res, plain)["out"] > 20 * TOL
    assert _errs(res, _oracle(x, w, 100.0, True))["out"] > 20 * TOL


def test_rope_fused_equals_unfused(libttt):
    """The fused call against an unfused one: XQ and XK rotated on the device by a plain torch
    restatement (stored back in bf16), then ttt_linear_forward."""
    w = synth.workload(1, B=2, H=4, L=16 * 12 + 5, seed=0x2078)
    x = synth.linear_inputs(w)
    theta = 10000.0
    fused = _gpu(libttt, x, w, theta, False)
    pos = (torch.arange(w.L, device="cuda") % w.K).double()
    inv = 1.0 / theta ** (torch.arange(0, 64, 2, device="cuda").double() / 64)
    ang = pos[:, None] * inv[None, :]
    cos, sin = ang.cos(), ang.sin()

    def rot(t):
        p = t.double().reshape(*t.shape[:-1], 32, 2)
        a, b = p[..., 0], p[..., 1]
        return torch.stack((a * cos - b * sin, a * sin + b * cos), -1).reshape(t.shape).to(t.dtype)

    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    unfused = libttt.ttt_linear_forward(rot(XQ), rot(XK), XV, dev_f32(x["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]),
                                        dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps,
                                        tail_grads=True)
    torch.cuda.synchronize()
    for name, a, b in zip(NAMES, fused, unfused):
        e = rel_l2(to_np(a).reshape(w.chains, -1), to_np(b).reshape(w.chains, -1))
        assert e <= TOL, (name, e)


@pytest.mark.parametrize("half", [False, True], ids=["pairs_2k_2k1", "half_split"])
def test_rope_full_size_sampled(libttt, half):
    """The 1B layer's workload (B = 8, H = 32, L = 8200: 512 full mini-batches and a tail of 8) in
    the launch configuration the benchmark times, on four sampled chains."""
    w = synth.workload(2, L=8200, seed=0x2079 + half)
    x = synth.linear_inputs(w)
    res = _gpu(libttt, x, w, 10000.0, half)
    chains = sample_chains(w.chains, 4)
    e = _errs(res, _oracle(x, w, 10000.0, half, chains=chains), chains)
    print(f"\n[rope] full size half={half}:", {k: f"{v:.2e}" for k, v in e.items()})
    assert max(e.values()) <= TOL, e
    assert libttt.ttt_device_status() == 0
