"""The decode workload at its full length: B=128, H=32, a 2048-token prefill on the GPU, then
1024 single-token decode steps (64 commits of W, b) with fresh tokens at every step, through
both cache formats ([explainer] TTTCache section; [walkthrough] TTTLinear.ttt, the cache path).

The oracle follows sampled chains (the first, a middle one and the last) through the same
prefill and all 1024 steps.  Checked at every step: out of those chains (max relative L2 per
chain <= 1e-2); at every commit (every 16th step): W and b; at the end: W, b and the grads.
The largest error seen and the error at step 1024 are printed (pytest -s shows them), so the
growth of the bf16-input / fp32-state error over 64 commits is on record.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import chain_slice, dev_act, dev_f32, rel_l2, sample_chains

pytestmark = pytest.mark.gpu

TOL = 1e-2
BLOCK = 64  # decode tokens drawn per block (host memory stays small)


def test_decode_1024_steps_dense_and_history_cache(libttt):
    w = synth.workload(4)  # B=128, H=32, L=2048 prefill, 1024 decode steps
    L0, steps, K, H = w.L, w.decode_steps, w.K, w.H
    assert L0 % K == 0  # the history cache starts at a mini-batch boundary

    # GPU prefill of every chain -> the dense cache (W, b, W_grad, b_grad) at offset L0
    x = synth.linear_inputs(w, values=False, t1=L0)
    _, W, b, Wg, bg = libttt.ttt_linear_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"),
                                                dev_f32(x["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]),
                                                dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), eps=w.eps,
                                                tail_grads=True)
    lnw, lnb = dev_f32(x["ln_w"]), dev_f32(x["ln_b"])
    del x
    # the history cache starts from the same committed state
    Wh, bh = W.clone(), b.clone()
    hist = torch.zeros((w.B, H, K, 2, 64), device="cuda")
    bgh = torch.zeros((w.B, H, 64), device="cuda")

    chains = sample_chains(w.chains, 3)
    assert chains[0] == 0 and chains[-1] == w.chains - 1
    xs = synth.linear_inputs(w, chains=chains)  # the sampled chains' whole stream, fp64-exact values
    o = oracle.default()
    r = o.linear_forward(xs["XQ"][:, :L0], xs["XK"][:, :L0], xs["XV"][:, :L0], xs["lr"][:, :L0], xs["W0"],
                         xs["b0"], xs["ln_w"], xs["ln_b"], K, w.eps, chains=chains)
    st = [r[k].copy() for k in ("W_last", "b_last", "W_grad_tail", "b_grad_tail")]

    worst = {"dense out": 0.0, "hist out": 0.0, "dense W": 0.0, "hist W": 0.0, "dense b": 0.0, "hist b": 0.0}
    last = {}
    idx = torch.tensor(chains, device="cuda")
    for blk0 in range(L0, L0 + steps, BLOCK):
        blk1 = min(blk0 + BLOCK, L0 + steps)
        xt = synth.linear_inputs(w, values=False, t0=blk0, t1=blk1)  # fresh tokens for every step
        tok = {k: dev_act({k + "_bits": xt[k + "_bits"]}, k) for k in ("XQ", "XK", "XV")}
        lr_blk = dev_f32(xt["lr"])
        for t in range(blk0, blk1):
            j = t - blk0
            args = [tok[k][:, :, j].contiguous() for k in ("XQ", "XK", "XV")]
            lr_t = lr_blk[:, :, j].contiguous()
            out_d = libttt.ttt_linear_decode_step(*args, lr_t, lnw, lnb, W, b, Wg, bg, seqlen_offset=t, eps=w.eps)
            out_h = libttt.ttt_linear_decode_step_hist(*args, lr_t, lnw, lnb, Wh, bh, hist, bgh, seqlen_offset=t,
                                                       eps=w.eps)
            ref = np.empty((len(chains), 64))
            for i, c in enumerate(chains):
                hh = c % H
                ref[i], committed = o.decode_chain(xs["XQ"][i, t], xs["XK"][i, t], xs["XV"][i, t], xs["lr"][i, t],
                                                   xs["ln_w"][hh], xs["ln_b"][hh], st[0][i], st[1][i], st[2][i],
                                                   st[3][i], K, t, w.eps)
            assert committed == ((t + 1) % K == 0)
            got_d = out_d.reshape(-1, 64)[idx].float().cpu().numpy()
            got_h = out_h.reshape(-1, 64)[idx].float().cpu().numpy()
            ed, eh = rel_l2(got_d, ref), rel_l2(got_h, ref)
            worst["dense out"] = max(worst["dense out"], ed)
            worst["hist out"] = max(worst["hist out"], eh)
            assert ed <= TOL, (t, ed)
            assert eh <= TOL, (t, eh)
            if committed:
                e = {"dense W": rel_l2(chain_slice(W, chains, H), st[0]),
                     "hist W": rel_l2(chain_slice(Wh, chains, H), st[0]),
                     "dense b": rel_l2(chain_slice(b, chains, H), st[1]),
                     "hist b": rel_l2(chain_slice(bh, chains, H), st[1])}
                for k, v in e.items():
                    worst[k] = max(worst[k], v)
                    assert v <= TOL, (t, k, v)
                last = dict(e, **{"dense out": ed, "hist out": eh, "step": t - L0 + 1})
    torch.cuda.synchronize()
    # after step 1024 (a commit: 2048 + 1024 is a multiple of 16) the grads are zero again
    assert (L0 + steps) % K == 0
    assert not Wg.any().item() and not bg.any().item() and not bgh.any().item()
    assert rel_l2(chain_slice(W, chains, H), chain_slice(Wh, chains, H)) <= 1e-4
    assert last["step"] == steps
    print("\ndecode over 1024 steps (64 commits), max relative L2 over sampled chains:")
    print("  worst over all steps:", {k: f"{v:.3e}" for k, v in worst.items()})
    print("  at step 1024:", {k: (f"{v:.3e}" if isinstance(v, float) else v) for k, v in last.items()})
