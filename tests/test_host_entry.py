"""The host-buffer entry point (ttt_linear_forward_host) against the device entry point on the
same values: chunking by batch rows changes nothing inside a chain, so the results must be the
same bits; plus the oracle on the bf16 case."""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import dev_act, dev_f32, rel_l2, to_np

pytestmark = pytest.mark.gpu


def _host_act(x, name):
    key = name + "_bits"
    if key in x:
        return torch.from_numpy(np.ascontiguousarray(x[key]).view(np.int16)).view(torch.bfloat16).pin_memory()
    return torch.from_numpy(np.ascontiguousarray(x[name], np.float32)).pin_memory()


def _host_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).pin_memory()


def _run_both(ttt, x, w, chunk, per_chain=None, te=None, flags=0):
    W0 = x["W0"] if per_chain is None else per_chain[0]
    b0 = x["b0"] if per_chain is None else per_chain[1]
    dev = ttt.ttt_linear_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"), dev_f32(x["lr"]), dev_f32(W0),
                                 dev_f32(b0), dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps,
                                 token_eta=None if te is None else dev_f32(te), tail_grads=True, flags=flags)
    host = ttt.ttt_linear_forward_host(_host_act(x, "XQ"), _host_act(x, "XK"), _host_act(x, "XV"), _host_f32(x["lr"]),
                                       _host_f32(W0), _host_f32(b0), _host_f32(x["ln_w"]), _host_f32(x["ln_b"]),
                                       mini_batch=w.K, eps=w.eps, token_eta=None if te is None else _host_f32(te),
                                       tail_grads=True, flags=flags, chunk_batches=chunk)
    torch.cuda.synchronize()
    return dev, host


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("chunk", [1, 2, 3])
def test_host_entry_equals_device_entry(libttt, dtype, chunk):
    w = synth.workload(1, B=3, H=2, L=16 * 5 + 7, dtype=dtype, seed=0x4057 + chunk)
    x = synth.linear_inputs(w)
    dev, host = _run_both(libttt, x, w, chunk)
    for d, h in zip(dev, host):
        assert torch.equal(d.cpu(), h)
    if dtype == "bf16":
        ref = oracle.default().linear_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"], x["b0"], x["ln_w"],
                                              x["ln_b"], w.K, w.eps)
        assert rel_l2(to_np(host[0]).reshape(ref["out"].shape), ref["out"]) <= 1e-2


def test_host_entry_per_chain_state_in_place_and_token_eta(libttt):
    w = synth.workload(1, B=4, H=2, L=16 * 3 + 2, seed=0x4058)
    x = synth.linear_inputs(w)
    rng = np.random.default_rng(5)
    W0 = (np.broadcast_to(x["W0"], (4, 2, 64, 64)) + rng.normal(0, 0.01, (4, 2, 64, 64))).astype(np.float32)
    b0 = rng.normal(0, 0.05, (4, 2, 64)).astype(np.float32)
    te = np.linspace(1.0, 0.4, 16).astype(np.float32)
    dev = libttt.ttt_linear_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"), dev_f32(x["lr"]), dev_f32(W0),
                                    dev_f32(b0), dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), eps=w.eps,
                                    token_eta=dev_f32(te))
    Wh, bh = _host_f32(W0), _host_f32(b0)
    host = libttt.ttt_linear_forward_host(_host_act(x, "XQ"), _host_act(x, "XK"), _host_act(x, "XV"),
                                          _host_f32(x["lr"]), Wh, bh, _host_f32(x["ln_w"]), _host_f32(x["ln_b"]),
                                          eps=w.eps, token_eta=_host_f32(te), W_last=Wh, b_last=bh, chunk_batches=3)
    torch.cuda.synchronize()
    assert host[1].data_ptr() == Wh.data_ptr()
    for d, h in zip(dev, host):
        assert torch.equal(d.cpu(), h)


def test_host_entry_L0_and_shared_workspace(libttt):
    w = synth.workload(1, B=2, H=3, L=0)
    x = synth.linear_inputs(w)
    out, Wl, bl = libttt.ttt_linear_forward_host(
        torch.empty(2, 3, 0, 64, dtype=torch.bfloat16), torch.empty(2, 3, 0, 64, dtype=torch.bfloat16),
        torch.empty(2, 3, 0, 64, dtype=torch.bfloat16), torch.empty(2, 3, 0), _host_f32(x["W0"]), _host_f32(x["b0"]),
        _host_f32(x["ln_w"]), _host_f32(x["ln_b"]), chunk_batches=2)
    torch.cuda.synchronize()
    assert np.array_equal(Wl.numpy(), np.broadcast_to(x["W0"], (2, 3, 64, 64)))
    # two calls in a row on one workspace (ordered on the same stream) give the same results
    w = synth.workload(1, B=2, H=2, L=16 * 4 + 1, seed=0x4059)
    x = synth.linear_inputs(w)
    need = libttt.ttt_linear_host_workspace_bytes(2, 2, w.L, 16, torch.bfloat16, 1)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    args = (_host_act(x, "XQ"), _host_act(x, "XK"), _host_act(x, "XV"), _host_f32(x["lr"]), _host_f32(x["W0"]),
            _host_f32(x["b0"]), _host_f32(x["ln_w"]), _host_f32(x["ln_b"]))
    r1 = libttt.ttt_linear_forward_host(*args, eps=w.eps, workspace=ws)
    r2 = libttt.ttt_linear_forward_host(*args, eps=w.eps, workspace=ws)
    torch.cuda.synchronize()
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)


@pytest.mark.parametrize("token_major", [False, True], ids=["head_major", "token_major"])
@pytest.mark.parametrize("chunk", [1, 2])
def test_host_entry_odd_heads_both_layouts(libttt, token_major, chunk):
    """Five heads and three batch rows in chunks of 1 or 2 rows (a ragged last chunk), head-major
    and token-major activations: the same bits as the device entry point."""
    w = synth.workload(1, B=3, H=5, L=16 * 3 + 4, seed=0x405A + chunk)
    x = synth.linear_inputs(w)
    tm = (lambda t: t.transpose(1, 2).contiguous()) if token_major else (lambda t: t)
    acts = [n for n in ("XQ", "XK", "XV")]
    dev = libttt.ttt_linear_forward(*[tm(dev_act(x, n)) for n in acts], dev_f32(x["lr"]), dev_f32(x["W0"]),
                                    dev_f32(x["b0"]), dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), mini_batch=w.K,
                                    eps=w.eps, tail_grads=True, token_major=token_major)
    host = libttt.ttt_linear_forward_host(*[tm(_host_act(x, n)).pin_memory() for n in acts], _host_f32(x["lr"]),
                                          _host_f32(x["W0"]), _host_f32(x["b0"]), _host_f32(x["ln_w"]),
                                          _host_f32(x["ln_b"]), mini_batch=w.K, eps=w.eps, tail_grads=True,
                                          chunk_batches=chunk, token_major=token_major)
    torch.cuda.synchronize()
    for d, h in zip(dev, host):
        assert torch.equal(d.cpu(), h)
