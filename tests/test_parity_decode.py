"""TTT-Linear decode steps through the C-ABI on the GPU against the oracle.

The cache state after a prefill of L0 tokens is (W_last, b_last, W_grad_tail, b_grad_tail) with
seqlen_offset = L0; each decode step takes one token per chain.  Tolerances as the prefill:
1e-5 for fp32 inputs, 1e-2 for bf16 inputs (max relative L2 per chain and tensor).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import chain_slice, dev_act, dev_f32, rel_l2, sample_chains, to_np

pytestmark = pytest.mark.gpu


def _tok(x, name, t):
    """[B,H,d] device tensor of token t of a [B,H,T,d] input dict (bf16 from exact bits)."""
    key = name + "_bits" if name + "_bits" in x else name
    sub = {name if key == name else name + "_bits": np.ascontiguousarray(x[key][:, :, t])}
    return dev_act(sub, name)


def _oracle_cache(x, w, L0, chains=None):
    """Oracle prefill over [0, L0) of the listed chains, then its cache as float64 arrays."""
    o = oracle.default()
    r = o.linear_forward(x["XQ"][..., :L0, :], x["XK"][..., :L0, :], x["XV"][..., :L0, :], x["lr"][..., :L0],
                         x["W0"], x["b0"], x["ln_w"], x["ln_b"], w.K, w.eps, chains=chains)
    return [r[k].copy() for k in ("W_last", "b_last", "W_grad_tail", "b_grad_tail")]


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 1e-2)])
def test_decode_steps_follow_the_oracle(libttt, dtype, tol):
    L0, steps = 37, 40
    w = synth.workload(4, B=2, H=3, L=L0, decode_steps=steps, dtype=dtype, seed=0x4D0C)
    x = synth.linear_inputs(w)
    H = w.H
    # GPU prefill gives the cache
    pre = {k: (v[:, :, :L0] if k in ("XQ", "XK", "XV", "XQ_bits", "XK_bits", "XV_bits", "lr") else v)
           for k, v in x.items()}
    pre = {k: np.ascontiguousarray(v) for k, v in pre.items()}
    _, W, b, Wg, bg = libttt.ttt_linear_forward(dev_act(pre, "XQ"), dev_act(pre, "XK"), dev_act(pre, "XV"),
                                                dev_f32(pre["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]),
                                                dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), eps=w.eps,
                                                tail_grads=True)
    # oracle cache per chain
    oW, ob, oWg, obg = _oracle_cache(x, w, L0)
    o = oracle.default()
    lnw, lnb = dev_f32(x["ln_w"]), dev_f32(x["ln_b"])
    for t in range(L0, L0 + steps):
        out = libttt.ttt_linear_decode_step(_tok(x, "XQ", t), _tok(x, "XK", t), _tok(x, "XV", t),
                                            dev_f32(np.ascontiguousarray(x["lr"][:, :, t])), lnw, lnb, W, b, Wg, bg,
                                            seqlen_offset=t, mini_batch=w.K, eps=w.eps)
        ref = np.empty((w.chains, 64))
        for c in range(w.chains):
            bb, hh = divmod(c, H)
            ref[c], committed = o.decode_chain(x["XQ"][bb, hh, t], x["XK"][bb, hh, t], x["XV"][bb, hh, t],
                                               x["lr"][bb, hh, t], x["ln_w"][hh], x["ln_b"][hh], oW[c], ob[c],
                                               oWg[c], obg[c], w.K, t, w.eps)
        torch.cuda.synchronize()
        assert rel_l2(to_np(out).reshape(-1, 64), ref) <= tol, t
        commit = (t + 1) % w.K == 0
        assert committed == commit
        if commit:  # integer/commit logic: the grads are exactly zero after a commit
            assert not to_np(Wg).any() and not to_np(bg).any()
        else:
            assert to_np(Wg).any()
    assert rel_l2(to_np(W).reshape(-1, 64, 64), oW) <= tol
    assert rel_l2(to_np(b).reshape(-1, 64), ob) <= tol
    assert rel_l2(to_np(Wg).reshape(-1, 64, 64), oWg) <= tol


@pytest.mark.parametrize("p", [0, 5, 15])
def test_decode_kernel_alone_from_the_oracle_state(libttt, p):
    """One step from an fp32 copy of the oracle's cache at position p (fp32 inputs): isolates the
    decode kernel from the prefill kernel's rounding."""
    L0 = 32 + p
    w = synth.workload(4, B=2, H=2, L=L0, decode_steps=1, dtype="f32", seed=0x4D0D + p)
    x = synth.linear_inputs(w)
    oW, ob, oWg, obg = _oracle_cache(x, w, L0)
    f32 = lambda a: np.asarray(a, np.float32)
    W, b = dev_f32(f32(oW).reshape(2, 2, 64, 64)), dev_f32(f32(ob).reshape(2, 2, 64))
    Wg, bg = dev_f32(f32(oWg).reshape(2, 2, 64, 64)), dev_f32(f32(obg).reshape(2, 2, 64))
    state = [f32(a).astype(np.float64) for a in (oW, ob, oWg, obg)]
    out = libttt.ttt_linear_decode_step(_tok(x, "XQ", L0), _tok(x, "XK", L0), _tok(x, "XV", L0),
                                        dev_f32(np.ascontiguousarray(x["lr"][:, :, L0])), dev_f32(x["ln_w"]),
                                        dev_f32(x["ln_b"]), W, b, Wg, bg, seqlen_offset=L0, eps=w.eps)
    o = oracle.default()
    ref = np.empty((4, 64))
    for c in range(4):
        bb, hh = divmod(c, 2)
        ref[c], _ = o.decode_chain(x["XQ"][bb, hh, L0], x["XK"][bb, hh, L0], x["XV"][bb, hh, L0],
                                   x["lr"][bb, hh, L0], x["ln_w"][hh], x["ln_b"][hh], state[0][c], state[1][c],
                                   state[2][c], state[3][c], w.K, L0, w.eps)
    torch.cuda.synchronize()
    assert rel_l2(to_np(out).reshape(-1, 64), ref) <= 1e-5
    for got, want in zip((W, b, Wg, bg), state):
        assert rel_l2(to_np(got).reshape(want.shape), want) <= 1e-5


def test_decode_full_size_sampled(libttt):
    """B=128, H=32 from a 2048-token prefill (GPU tensor-core kernel), 20 decode steps; the
    oracle follows a sample of chains through the same prefill and steps."""
    steps = 20
    w = synth.workload(4, decode_steps=steps)
    L0 = w.L
    x = synth.linear_inputs(w, values=False, t1=L0)
    _, W, b, Wg, bg = libttt.ttt_linear_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"),
                                                dev_f32(x["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]),
                                                dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), eps=w.eps,
                                                tail_grads=True)
    del x
    chains = sample_chains(w.chains, 3)
    xs = synth.linear_inputs(w, chains=chains)
    o = oracle.default()
    r = o.linear_forward(xs["XQ"][:, :L0], xs["XK"][:, :L0], xs["XV"][:, :L0], xs["lr"][:, :L0], xs["W0"],
                         xs["b0"], xs["ln_w"], xs["ln_b"], w.K, w.eps, chains=chains)
    st = [r[k].copy() for k in ("W_last", "b_last", "W_grad_tail", "b_grad_tail")]
    lnw, lnb = dev_f32(xs["ln_w"]), dev_f32(xs["ln_b"])
    for t in range(L0, L0 + steps):
        xt = synth.linear_inputs(w, values=False, t0=t, t1=t + 1)
        out = libttt.ttt_linear_decode_step(*(dev_act({k + "_bits": np.ascontiguousarray(xt[k + "_bits"][:, :, 0])}, k)
                                              for k in ("XQ", "XK", "XV")),
                                            dev_f32(np.ascontiguousarray(xt["lr"][:, :, 0])), lnw, lnb, W, b, Wg, bg,
                                            seqlen_offset=t, eps=w.eps)
        ref = np.empty((len(chains), 64))
        for i, c in enumerate(chains):
            hh = c % w.H
            ref[i], _ = o.decode_chain(xs["XQ"][i, t], xs["XK"][i, t], xs["XV"][i, t], xs["lr"][i, t],
                                       xs["ln_w"][hh], xs["ln_b"][hh], st[0][i], st[1][i], st[2][i], st[3][i],
                                       w.K, t, w.eps)
        torch.cuda.synchronize()
        assert rel_l2(chain_slice(out, chains, w.H), ref) <= 1e-2, t
    assert rel_l2(chain_slice(W, chains, w.H), st[0]) <= 1e-2
    assert rel_l2(chain_slice(Wg, chains, w.H), st[2]) <= 1e-2


def test_decode_bounded_wait_timeout_reports_and_recovers(libttt):
    """Every bounded wait of the decode kernel gives up at once: the status word reports it, the
    context stays usable and the next step (on a fresh copy of the cache) is correct."""
    L0 = 40
    w = synth.workload(4, B=2, H=2, L=L0, decode_steps=1, dtype="f32", seed=0x4D0E)
    x = synth.linear_inputs(w)
    oW, ob, oWg, obg = _oracle_cache(x, w, L0)
    f32 = lambda a: np.asarray(a, np.float32)

    def cache():
        return (dev_f32(f32(oW).reshape(2, 2, 64, 64)), dev_f32(f32(ob).reshape(2, 2, 64)),
                dev_f32(f32(oWg).reshape(2, 2, 64, 64)), dev_f32(f32(obg).reshape(2, 2, 64)))

    args = (_tok(x, "XQ", L0), _tok(x, "XK", L0), _tok(x, "XV", L0), dev_f32(np.ascontiguousarray(x["lr"][:, :, L0])),
            dev_f32(x["ln_w"]), dev_f32(x["ln_b"]))
    libttt.ttt_device_status(clear=True)
    libttt.ttt_set_wait_limit(-1)
    try:
        libttt.ttt_linear_decode_step(*args, *cache(), seqlen_offset=L0, eps=w.eps)
        torch.cuda.synchronize()
        with pytest.raises(libttt.TTTError) as e:
            libttt.ttt_device_status(clear=True)
        assert e.value.code == libttt.TTT_ERR_TIMEOUT
    finally:
        libttt.ttt_set_wait_limit(0)
    assert libttt.ttt_device_status(clear=True) == 0
    state = [f32(a).astype(np.float64) for a in (oW, ob, oWg, obg)]
    out = libttt.ttt_linear_decode_step(*args, *cache(), seqlen_offset=L0, eps=w.eps)
    o = oracle.default()
    ref = np.empty((4, 64))
    for c in range(4):
        bb, hh = divmod(c, 2)
        ref[c], _ = o.decode_chain(x["XQ"][bb, hh, L0], x["XK"][bb, hh, L0], x["XV"][bb, hh, L0],
                                   x["lr"][bb, hh, L0], x["ln_w"][hh], x["ln_b"][hh], state[0][c], state[1][c],
                                   state[2][c], state[3][c], w.K, L0, w.eps)
    torch.cuda.synchronize()
    assert rel_l2(to_np(out).reshape(-1, 64), ref) <= 1e-5
    assert libttt.ttt_device_status() == 0
