"""TTT-Linear decode through the history-format cache (ttt_linear_decode_step_hist) on the GPU:
against the oracle's decode steps (which keep the dense gradient sum), and against the dense-cache
kernel.  Tolerances as the other decode tests: 1e-5 for fp32 inputs, 1e-2 for bf16."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import dev_act, dev_f32, rel_l2, sample_chains, to_np
from test_parity_decode import _oracle_cache, _tok

pytestmark = pytest.mark.gpu


def _prefill(libttt, x, w, L0):
    pre = {k: (v[:, :, :L0] if k in ("XQ", "XK", "XV", "XQ_bits", "XK_bits", "XV_bits", "lr") else v)
           for k, v in x.items()}
    pre = {k: np.ascontiguousarray(v) for k, v in pre.items()}
    _, W, b = libttt.ttt_linear_forward(dev_act(pre, "XQ"), dev_act(pre, "XK"), dev_act(pre, "XV"),
                                        dev_f32(pre["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]), dev_f32(x["ln_w"]),
                                        dev_f32(x["ln_b"]), eps=w.eps)
    return W, b


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 1e-2)])
def test_hist_decode_follows_the_oracle(libttt, dtype, tol):
    L0, steps = 32, 40  # starts at a mini-batch boundary; crosses two commits
    w = synth.workload(4, B=2, H=3, L=L0, decode_steps=steps, dtype=dtype, seed=0x4E0C)
    x = synth.linear_inputs(w)
    H = w.H
    W, b = _prefill(libttt, x, w, L0)
    hist = torch.zeros(w.B, H, w.K, 2, 64, device="cuda")
    gb = torch.zeros(w.B, H, 64, device="cuda")
    oW, ob, oWg, obg = _oracle_cache(x, w, L0)
    o = oracle.default()
    lnw, lnb = dev_f32(x["ln_w"]), dev_f32(x["ln_b"])
    for t in range(L0, L0 + steps):
        out = libttt.ttt_linear_decode_step_hist(_tok(x, "XQ", t), _tok(x, "XK", t), _tok(x, "XV", t),
                                                 dev_f32(np.ascontiguousarray(x["lr"][:, :, t])), lnw, lnb, W, b,
                                                 hist, gb, seqlen_offset=t, mini_batch=w.K, eps=w.eps)
        ref = np.empty((w.chains, 64))
        for c in range(w.chains):
            bb, hh = divmod(c, H)
            ref[c], _ = o.decode_chain(x["XQ"][bb, hh, t], x["XK"][bb, hh, t], x["XV"][bb, hh, t], x["lr"][bb, hh, t],
                                       x["ln_w"][hh], x["ln_b"][hh], oW[c], ob[c], oWg[c], obg[c], w.K, t, w.eps)
        torch.cuda.synchronize()
        assert rel_l2(to_np(out).reshape(-1, 64), ref) <= tol, t
    assert rel_l2(to_np(W).reshape(-1, 64, 64), oW) <= tol
    assert rel_l2(to_np(b).reshape(-1, 64), ob) <= tol
    assert rel_l2(to_np(gb).reshape(-1, 64), obg) <= tol


def test_hist_decode_equals_dense_decode(libttt):
    """The two caches hold the same state in different forms: fp32 runs agree to rounding."""
    L0, steps = 48, 37
    w = synth.workload(4, B=2, H=2, L=L0, decode_steps=steps, dtype="f32", seed=0x4E0D)
    x = synth.linear_inputs(w)
    W, b = _prefill(libttt, x, w, L0)
    Wd, bd = W.clone(), b.clone()
    Wg, bg = torch.zeros_like(W), torch.zeros_like(b)
    hist = torch.zeros(w.B, w.H, w.K, 2, 64, device="cuda")
    gb = torch.zeros_like(b)
    lnw, lnb = dev_f32(x["ln_w"]), dev_f32(x["ln_b"])
    for t in range(L0, L0 + steps):
        args = (_tok(x, "XQ", t), _tok(x, "XK", t), _tok(x, "XV", t), dev_f32(np.ascontiguousarray(x["lr"][:, :, t])),
                lnw, lnb)
        o1 = libttt.ttt_linear_decode_step_hist(*args, W, b, hist, gb, seqlen_offset=t, eps=w.eps)
        o2 = libttt.ttt_linear_decode_step(*args, Wd, bd, Wg, bg, seqlen_offset=t, eps=w.eps)
        torch.cuda.synchronize()
        assert rel_l2(to_np(o1), to_np(o2)) <= 1e-5, t
    assert rel_l2(to_np(W), to_np(Wd)) <= 1e-5 and rel_l2(to_np(b), to_np(bd)) <= 1e-5
    assert rel_l2(to_np(gb), to_np(bg)) <= 1e-5


def test_hist_decode_full_size_sampled(libttt):
    """B=128, H=32 from a 2048-token prefill (tensor-core kernel), 20 steps; the oracle follows a
    sample of chains through the same prefill and steps."""
    steps = 20
    w = synth.workload(4, decode_steps=steps)
    L0 = w.L
    x = synth.linear_inputs(w, values=False, t1=L0)
    _, W, b = libttt.ttt_linear_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"), dev_f32(x["lr"]),
                                        dev_f32(x["W0"]), dev_f32(x["b0"]), dev_f32(x["ln_w"]), dev_f32(x["ln_b"]),
                                        eps=w.eps)
    del x
    hist = torch.zeros(w.B, w.H, w.K, 2, 64, device="cuda")
    gb = torch.zeros(w.B, w.H, 64, device="cuda")
    toks = synth.linear_inputs(w, values=False, t0=L0, t1=L0 + steps)
    XQ, XK, XV = (dev_act(toks, n) for n in ("XQ", "XK", "XV"))
    lr = dev_f32(toks["lr"])
    lnw, lnb = dev_f32(toks["ln_w"]), dev_f32(toks["ln_b"])
    outs = []
    for i in range(steps):
        outs.append(libttt.ttt_linear_decode_step_hist(XQ[:, :, i].contiguous(), XK[:, :, i].contiguous(),
                                                       XV[:, :, i].contiguous(), lr[:, :, i].contiguous(), lnw, lnb,
                                                       W, b, hist, gb, seqlen_offset=L0 + i, eps=w.eps))
    torch.cuda.synchronize()
    chains = sample_chains(w.chains, 3)
    xs = synth.linear_inputs(w, chains=chains, t1=L0 + steps)
    o = oracle.default()
    r = o.linear_forward(xs["XQ"][..., :L0, :], xs["XK"][..., :L0, :], xs["XV"][..., :L0, :], xs["lr"][..., :L0],
                         xs["W0"], xs["b0"], xs["ln_w"], xs["ln_b"], w.K, w.eps, chains=chains)
    for n, c in enumerate(chains):
        hh = c % w.H
        st = [r[k][n].copy() for k in ("W_last", "b_last", "W_grad_tail", "b_grad_tail")]
        got = np.stack([to_np(outs[i]).reshape(-1, 64)[c] for i in range(steps)])
        want = np.stack([o.decode_chain(xs["XQ"][n, L0 + i], xs["XK"][n, L0 + i], xs["XV"][n, L0 + i],
                                        xs["lr"][n, L0 + i], xs["ln_w"][hh], xs["ln_b"][hh], *st, w.K, L0 + i,
                                        w.eps)[0] for i in range(steps)])
        assert rel_l2(got, want) <= 1e-2, c


def test_hist_decode_bounded_wait_timeout_reports_and_recovers(libttt):
    w = synth.workload(4, B=2, H=2, L=16, decode_steps=1, dtype="f32", seed=0x4E0E)
    x = synth.linear_inputs(w)
    W, b = _prefill(libttt, x, w, 16)
    args = (_tok(x, "XQ", 16), _tok(x, "XK", 16), _tok(x, "XV", 16), dev_f32(np.ascontiguousarray(x["lr"][:, :, 16])),
            dev_f32(x["ln_w"]), dev_f32(x["ln_b"]))
    hist = torch.zeros(2, 2, 16, 2, 64, device="cuda")
    gb = torch.zeros(2, 2, 64, device="cuda")
    libttt.ttt_device_status(clear=True)
    libttt.ttt_set_wait_limit(-1)
    try:
        libttt.ttt_linear_decode_step_hist(*args, W.clone(), b.clone(), hist.clone(), gb.clone(), seqlen_offset=16,
                                           eps=w.eps)
        torch.cuda.synchronize()
        with pytest.raises(libttt.TTTError) as e:
            libttt.ttt_device_status(clear=True)
        assert e.value.code == libttt.TTT_ERR_TIMEOUT
    finally:
        libttt.ttt_set_wait_limit(0)
    assert libttt.ttt_device_status(clear=True) == 0
    Wd, bd = W.clone(), b.clone()
    o1 = libttt.ttt_linear_decode_step_hist(*args, W, b, hist, gb, seqlen_offset=16, eps=w.eps)
    o2 = libttt.ttt_linear_decode_step(*args, Wd, bd, torch.zeros_like(Wd), torch.zeros_like(bd), seqlen_offset=16,
                                       eps=w.eps)
    torch.cuda.synchronize()
    assert rel_l2(to_np(o1), to_np(o2)) <= 1e-5
    assert libttt.ttt_device_status() == 0
