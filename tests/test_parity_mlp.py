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


def test_mlp_full_size_every_chain(libttt):
    """Every one of the 256 chains (B=8, H=32, L=2048) against the oracle.  With bf16 operands
    one chain of this workload ends at 1.18e-2 on b2_last; the kernel takes fp16 operands."""
    from concurrent.futures import ThreadPoolExecutor
    import os

    w = synth.workload(3)
    x = synth.linear_inputs(w, values=False)
    res = gpu_mlp(libttt, x, w)
    o = oracle.default()

    def one(c):
        xs = synth.linear_inputs(w, chains=[c])
        h = c % w.H
        return o.mlp_chain(xs["XQ"][0], xs["XK"][0], xs["XV"][0], xs["lr"][0], xs["W1"][h], xs["b1"][h], xs["W2"][h],
                           xs["b2"][h], xs["ln_w"][h], xs["ln_b"][h], w.K, w.eps)

    with ThreadPoolExecutor(max(1, len(os.sched_getaffinity(0)))) as ex:
        refs = list(ex.map(one, range(w.chains)))
    errs = {k: rel_l2(to_np(t).reshape(w.chains, -1), np.stack([r[k].reshape(-1) for r in refs]))
            for k, t in zip(KEYS, res)}
    print("[parity] mlp every chain:", ", ".join(f"{k}={e:.2e}" for k, e in errs.items()))
    for k, e in errs.items():
        assert e <= 1e-2, (k, e, errs)


def test_mlp_L0(libttt):
    w = synth.workload(3, B=1, H=2, L=0)
    x = synth.linear_inputs(w)
    out, W1, b1, W2, b2 = gpu_mlp(libttt, x, w)
    assert out.numel() == 0 and np.array_equal(to_np(W2)[0], x["W2"])


def _mlp_inputs(w):
    x = synth.linear_inputs(w)
    x["b1"] = synth.random_bias(w, "B1", x["b1"].shape)
    x["b2"] = synth.random_bias(w, "B2", x["b2"].shape)
    return x


@pytest.mark.parametrize("L,K", [(16 * 9 + 3, 16), (8 * 7 + 5, 8), (13 * 4, 13), (3, 1), (16 * 40, 16)])
def test_mlp_tensor_core_ragged(libttt, L, K):
    """bf16 inputs take the tensor-core kernel: several mini-batches, a ragged tail, K < 16."""
    w = synth.workload(3, B=2, H=2, L=L, K=K, dtype="bf16", seed=0x3B00 + L * 17 + K)
    x = _mlp_inputs(w)
    _check(gpu_mlp(libttt, x, w), oracle_mlp(x, w), 1e-2)


def test_mlp_token_eta_table(libttt):
    w = synth.workload(3, B=1, H=2, L=16 * 5 + 7, dtype="bf16")
    x = _mlp_inputs(w)
    te = np.linspace(1.0, 0.3, 16).astype(np.float32)
    res = libttt.ttt_mlp_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"), dev_f32(x["lr"]),
                                 dev_f32(x["W1"]), dev_f32(x["b1"]), dev_f32(x["W2"]), dev_f32(x["b2"]),
                                 dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps,
                                 token_eta=dev_f32(te))
    torch.cuda.synchronize()
    ref = oracle.default().mlp_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W1"], x["b1"], x["W2"], x["b2"],
                                       x["ln_w"], x["ln_b"], w.K, w.eps, token_eta=te.astype(np.float64))
    _check(res, ref, 1e-2)


def test_mlp_per_chain_state(libttt):
    """A continuation: per-chain initial states of shape [B,H,...]."""
    w = synth.workload(3, B=2, H=2, L=16 * 4 + 9, dtype="bf16")
    x = _mlp_inputs(w)
    rng = np.random.default_rng(11)
    st = {}
    for k in ("W1", "b1", "W2", "b2"):
        base = np.broadcast_to(x[k], (2,) + x[k].shape)
        st[k] = (base + rng.normal(0, 0.01, base.shape)).astype(np.float32)
    res = libttt.ttt_mlp_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"), dev_f32(x["lr"]),
                                 dev_f32(st["W1"]), dev_f32(st["b1"]), dev_f32(st["W2"]), dev_f32(st["b2"]),
                                 dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps)
    torch.cuda.synchronize()
    ref = oracle.default().mlp_forward(x["XQ"], x["XK"], x["XV"], x["lr"], st["W1"], st["b1"], st["W2"],
                                       st["b2"], x["ln_w"], x["ln_b"], w.K, w.eps, state_per_chain=True)
    _check(res, ref, 1e-2)


def test_mlp_fp32_compute_flag(libttt):
    """bf16 inputs with TTT_FLAG_FP32_COMPUTE take the fp32 kernel; its bf16 output is compared at
    bf16 resolution, its fp32 states at fp32 accuracy."""
    w = synth.workload(3, B=1, H=2, L=16 * 3 + 5, dtype="bf16")
    x = _mlp_inputs(w)
    res = gpu_mlp(libttt, x, w, flags=libttt.TTT_FLAG_FP32_COMPUTE)
    ref = oracle_mlp(x, w)
    for k, t in zip(KEYS, res):
        e = rel_l2(to_np(t).reshape(ref[k].shape), ref[k])
        assert e <= (4e-3 if k == "out" else 1e-5), f"{k}: {e:.3e}"


def test_mlp_bounded_wait_timeout_reports_and_recovers(libttt):
    """Every bounded wait of the tensor-core kernel gives up at once: the status word reports it,
    the context stays usable and the next call is correct."""
    w = synth.workload(3, B=1, H=2, L=16 * 6 + 3, dtype="bf16")
    x = _mlp_inputs(w)
    libttt.ttt_device_status(clear=True)
    libttt.ttt_set_wait_limit(-1)
    try:
        gpu_mlp(libttt, x, w)
        with pytest.raises(libttt.TTTError) as e:
            libttt.ttt_device_status(clear=True)
        assert e.value.code == libttt.TTT_ERR_TIMEOUT
    finally:
        libttt.ttt_set_wait_limit(0)
    assert libttt.ttt_device_status(clear=True) == 0
    _check(gpu_mlp(libttt, x, w), oracle_mlp(x, w), 1e-2)
    assert libttt.ttt_device_status() == 0


def test_mlp_odd_chain_count(libttt):
    """Chains are paired per CTA; with an odd count the last pair has one chain."""
    w = synth.workload(3, B=1, H=3, L=16 * 3 + 5, dtype="bf16", seed=0x3C01)
    x = _mlp_inputs(w)
    _check(gpu_mlp(libttt, x, w), oracle_mlp(x, w), 1e-2)
