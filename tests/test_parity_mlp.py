"""TTT-MLP prefill through the C-ABI on the GPU against the oracle (max relative L2 per chain and
tensor: 1e-5 for fp32 inputs, 1e-2 for bf16 inputs)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import chain_slice, dev_act, dev_f32, rel_l2, sample_chains, to_np

pytestmark = pytest.mark.gpu

KEYS = ("out", "W1_last", "b1_last", "W2_last", "b2_last")


def gpu_mlp(ttt, x, w, flags=0):
    res = ttt.ttt_mlp_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"), dev_f32(x["lr"]),
                              dev_f32(x["W1"]), dev_f32(x["b1"]), dev_f32(x["W2"]), dev_f32(x["b2"]),
                              dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps, flags=flags)
    torch.cuda.synchronize()
    return res


def oracle_mlp(x, w, chains=None):
    return oracle.default().mlp_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W1"], x["b1"], x["W2"], x["b2"],
                                        x["ln_w"], x["ln_b"], w.K, w.eps, chains=chains)


def _check(res, ref, tol, chains=None, H=None):
    for k, t in zip(KEYS, res):
        got = chain_slice(t, chains, H) if chains is not None else to_np(t).reshape(ref[k].shape)
        e = rel_l2(got.reshape(ref[k].shape), ref[k])
        assert e <= tol, f"{k}: {e:.3e}"


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 1e-2)])
@pytest.mark.parametrize("L,K", [(16 * 3 + 5, 16), (1, 16), (16, 16), (21, 4)])
def test_mlp_small(libttt, dtype, tol, L, K):
    w = synth.workload(3, B=1, H=2, L=L, K=K, dtype=dtype, seed=0x3A1 + L + K)
    x = synth.linear_inputs(w)
    x["b1"] = synth.random_bias(w, "B1", x["b1"].shape)
    x["b2"] = synth.random_bias(w, "B2", x["b2"].shape)
    _check(gpu_mlp(libttt, x, w), oracle_mlp(x, w), tol)


def test_mlp_full_size_sampled(libttt):
    """B=8, H=32, L=2048: GPU on all chains, oracle on a sample."""
    w = synth.workload(3)
    x = synth.linear_inputs(w, values=False)
    res = gpu_mlp(libttt, x, w)
    chains = sample_chains(w.chains, 3)
    ref = oracle_mlp(synth.linear_inputs(w, chains=chains), w, chains=chains)
    _check(res, ref, 1e-2, chains, w.H)


def test_mlp_L0(libttt):
    w = synth.workload(3, B=1, H=2, L=0)
    x = synth.linear_inputs(w)
    out, W1, b1, W2, b2 = gpu_mlp(libttt, x, w)
    assert out.numel() == 0 and np.array_equal(to_np(W2)[0], x["W2"])
