"""Sharding through the library itself: the batch slices that batch_shard hands to the ranks of a
data-parallel job, each run through the C ABI as its own call, give the bits of one call over the
whole batch.  Every chain is independent (no exchange at any mini-batch), so a rank's result must
not depend on which other rows share its launch.  One GPU runs the ranks' calls one after the
other; the multi-process host path itself is covered on CPU by tests/test_multi_rank.py.
"""
import numpy as np
import pytest
import torch

import synth
from parity_util import dev_act, dev_f32
from test_rnn_layers_b200.shard import batch_shard

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("world", [2, 3, 5])
def test_linear_prefill_shards_give_the_unsharded_bits(libttt, world):
    w = synth.workload(1, B=5, H=4, L=16 * 11 + 6, seed=0x5A5 + world)
    x = synth.linear_inputs(w)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    lr, W0, b0, lnw, lnb = (dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b"))
    whole = libttt.ttt_linear_forward(XQ, XK, XV, lr, W0, b0, lnw, lnb, eps=w.eps, tail_grads=True)
    parts = []
    for r in range(world):
        s, e = batch_shard(w.B, world, r)
        if e > s:
            parts.append(libttt.ttt_linear_forward(XQ[s:e].contiguous(), XK[s:e].contiguous(), XV[s:e].contiguous(),
                                                   lr[s:e].contiguous(), W0, b0, lnw, lnb, eps=w.eps,
                                                   tail_grads=True))
    torch.cuda.synchronize()
    for i, t in enumerate(whole):
        assert torch.equal(torch.cat([p[i] for p in parts]), t), i


def test_mlp_prefill_shards_give_the_unsharded_bits(libttt):
    w = synth.workload(3, B=3, H=2, L=16 * 5 + 3, seed=0x5A6)
    x = synth.linear_inputs(w)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    p = [dev_f32(x[k]) for k in ("W1", "b1", "W2", "b2", "ln_w", "ln_b")]
    lr = dev_f32(x["lr"])
    whole = libttt.ttt_mlp_forward(XQ, XK, XV, lr, *p, mini_batch=w.K, eps=w.eps)
    parts = [libttt.ttt_mlp_forward(XQ[s:e].contiguous(), XK[s:e].contiguous(), XV[s:e].contiguous(),
                                    lr[s:e].contiguous(), *p, mini_batch=w.K, eps=w.eps)
             for s, e in (batch_shard(w.B, 2, r) for r in range(2))]
    torch.cuda.synchronize()
    for i, t in enumerate(whole):
        assert torch.equal(torch.cat([q[i] for q in parts]), t), i


def test_output_side_token_shards_give_the_unsharded_bits(libttt):
    T, C, N = 1000, 768, 768
    d = synth.oproj_inputs(0x5A7, T, C, N, values=False)
    X = torch.from_numpy(np.ascontiguousarray(d["X_bits"]).view(np.int16)).cuda().view(torch.bfloat16)
    Wo = torch.from_numpy(np.ascontiguousarray(d["Wo_bits"]).view(np.int16)).cuda().view(torch.bfloat16)
    Wp, u, v = libttt.ttt_o_proj_prepare(Wo, dev_f32(d["ln_w"]), dev_f32(d["ln_b"]))
    whole = libttt.ttt_post_norm_o_proj(X, Wp, u, v)
    parts = [libttt.ttt_post_norm_o_proj(X[s:e].contiguous(), Wp, u, v) for s, e in (batch_shard(T, 3, r) for r in range(3))]
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts), whole)
