"""Token-major activations (TTT_FLAG_TOKEN_MAJOR): XQ, XK, XV and out as [B,L,H,d], the [B,L,C]
layout of the QKV projections and of the scan's return value in TTTBase.forward / TTTLinear.ttt.

Only the addressing changes, so every kernel must give the same bits as on the head-major
[B,H,L,d] copy of the same values (which the parity tests hold to the oracle); one case per
kernel is also compared with the oracle directly."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import dev_act, dev_f32, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _tm(t):
    """[B,H,L,d] -> a contiguous [B,L,H,d] copy."""
    return t.transpose(1, 2).contiguous()


def _linear(ttt, x, w, token_major, flags=0, te=None):
    acts = [dev_act(x, n) for n in ("XQ", "XK", "XV")]
    if token_major:
        acts = [_tm(a) for a in acts]
    res = ttt.ttt_linear_forward(*acts, dev_f32(x["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]), dev_f32(x["ln_w"]),
                                 dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps, tail_grads=True, flags=flags,
                                 token_major=token_major, token_eta=None if te is None else dev_f32(te))
    torch.cuda.synchronize()
    return res


def _mlp(ttt, x, w, token_major, flags=0):
    acts = [dev_act(x, n) for n in ("XQ", "XK", "XV")]
    if token_major:
        acts = [_tm(a) for a in acts]
    res = ttt.ttt_mlp_forward(*acts, dev_f32(x["lr"]), dev_f32(x["W1"]), dev_f32(x["b1"]), dev_f32(x["W2"]),
                              dev_f32(x["b2"]), dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps,
                              flags=flags, token_major=token_major)
    torch.cuda.synchronize()
    return res


def _same(head_major, token_major):
    out_h, *state_h = head_major
    out_t, *state_t = token_major
    assert out_t.shape == (out_h.shape[0], out_h.shape[2], out_h.shape[1], out_h.shape[3])
    assert torch.equal(out_t.transpose(1, 2), out_h)
    for a, b in zip(state_h, state_t):
        assert torch.equal(a, b)


@pytest.mark.parametrize("dtype,flags", [("bf16", 0), ("bf16", 1), ("f32", 0)])
@pytest.mark.parametrize("L,K", [(16 * 6 + 5, 16), (16 * 4, 16), (7 * 5 + 3, 7), (9, 16)])
def test_linear_token_major_equals_head_major(libttt, dtype, flags, L, K):
    """Tensor-core kernel (bf16), FFMA kernel (bf16 with FP32_COMPUTE, and f32): ragged tails, K < 16,
    a sequence shorter than one mini-batch; B and H both > 1 so the two layouts differ."""
    w = synth.workload(1, B=3, H=5, L=L, K=K, dtype=dtype, seed=0x70C0 + L * 31 + K + 7 * flags)
    x = synth.linear_inputs(w)
    _same(_linear(libttt, x, w, False, flags), _linear(libttt, x, w, True, flags))


def test_linear_token_major_against_oracle(libttt):
    w = synth.workload(1, B=2, H=3, L=16 * 5 + 9, dtype="bf16", seed=0x70C9)
    x = synth.linear_inputs(w)
    te = np.linspace(1.0, 0.3, 16).astype(np.float32)
    out, Wl, bl, Wg, bg = _linear(libttt, x, w, True, te=te)
    ref = oracle.default().linear_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"], x["b0"], x["ln_w"],
                                          x["ln_b"], w.K, w.eps, token_eta=te)
    got = to_np(out.transpose(1, 2))  # back to [B,H,L,d]
    assert rel_l2(got.reshape(ref["out"].shape), ref["out"]) <= 1e-2
    assert rel_l2(to_np(Wl).reshape(ref["W_last"].shape), ref["W_last"]) <= 1e-2
    assert rel_l2(to_np(bl).reshape(ref["b_last"].shape), ref["b_last"]) <= 1e-2


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("L,K", [(16 * 3 + 5, 16), (8 * 4 + 3, 8)])
def test_mlp_token_major_equals_head_major(libttt, dtype, L, K):
    w = synth.workload(3, B=2, H=3, L=L, K=K, dtype=dtype, seed=0x70D0 + L + K)
    x = synth.linear_inputs(w)
    x["b1"] = synth.random_bias(w, "B1", x["b1"].shape)
    x["b2"] = synth.random_bias(w, "B2", x["b2"].shape)
    _same(_mlp(libttt, x, w, False), _mlp(libttt, x, w, True))


def test_mlp_token_major_against_oracle(libttt):
    w = synth.workload(3, B=2, H=2, L=16 * 4 + 6, dtype="bf16", seed=0x70D9)
    x = synth.linear_inputs(w)
    out, W1, b1, W2, b2 = _mlp(libttt, x, w, True)
    ref = oracle.default().mlp_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W1"], x["b1"], x["W2"], x["b2"],
                                       x["ln_w"], x["ln_b"], w.K, w.eps)
    got = to_np(out.transpose(1, 2))
    assert rel_l2(got.reshape(ref["out"].shape), ref["out"]) <= 1e-2
    assert rel_l2(to_np(W2).reshape(ref["W2_last"].shape), ref["W2_last"]) <= 1e-2


@pytest.mark.parametrize("chunk", [1, 2])
def test_host_entry_token_major(libttt, chunk):
    """The host-buffer entry chunks by batch rows, which are contiguous in both layouts."""
    w = synth.workload(1, B=3, H=4, L=16 * 3 + 11, seed=0x70E0 + chunk)
    x = synth.linear_inputs(w)
    dev = _linear(libttt, x, w, True)

    def host_tm(name):
        return _tm(dev_act(x, name)).cpu().pin_memory()

    def host_f32(a):
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).pin_memory()

    host = libttt.ttt_linear_forward_host(host_tm("XQ"), host_tm("XK"), host_tm("XV"), host_f32(x["lr"]),
                                          host_f32(x["W0"]), host_f32(x["b0"]), host_f32(x["ln_w"]),
                                          host_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps, tail_grads=True,
                                          chunk_batches=chunk, token_major=True)
    torch.cuda.synchronize()
    for d, h in zip(dev, host):
        assert torch.equal(d.cpu(), h)
