"""Checkpoints from the forward (ttt_linear_forward_ckpt) and the backward that starts from them
(ttt_linear_backward_ckpt), the split of the walkthrough's checkpointed scan: the forward keeps
the state at the start of every checkpoint group, the backward rebuilds each group from it.

* The forward with checkpoints gives the same bits as without; entry 0 is (W0, b0) and the last
  entry is (W_last, b_last), bit for bit; a middle entry is the oracle's state after that prefix
  of the sequence, within the dtype's bar (bf16 1e-2, fp32 1e-5).
* The backward from the checkpoints gives the backward oracle's gradients within the same bars
  (test_backward's comparison: every output of every chain).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import dev_act, dev_f32, rel_l2, to_np
from test_backward import _compare, _oracle

pytestmark = pytest.mark.gpu

CASES = [  # (name, dtype, B, H, L, K, G, token_major)
    ("bf16_tail_G4", "bf16", 2, 2, 16 * 9 + 5, 16, 4, False),
    ("bf16_G1", "bf16", 1, 3, 16 * 5, 16, 1, False),
    ("bf16_token_major_G3", "bf16", 2, 2, 16 * 7 + 3, 16, 3, True),
    ("bf16_K8_G2", "bf16", 1, 2, 8 * 6 + 2, 8, 2, False),
    ("bf16_shorter_than_K", "bf16", 1, 2, 10, 16, 4, False),
    ("f32_tail_G3", "f32", 2, 2, 16 * 7 + 4, 16, 3, False),
]
IDS = [c[0] for c in CASES]


def _setup(libttt, case):
    name, dt, B, H, L, K, G, tm = case
    w = synth.workload(1, B=B, H=H, L=L, K=K, dtype=dt, seed=0xC4 + L + G)
    x, up = synth.linear_inputs(w), synth.upstream_grads(w)
    lay = (lambda t: t.transpose(1, 2).contiguous()) if tm else (lambda t: t)
    acts = [lay(dev_act(x, n)) for n in ("XQ", "XK", "XV")]
    rest = [dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b")]
    n_ckpt = (L // K + G - 1) // G
    ckpt = torch.full((libttt.ttt_linear_ckpt_bytes(B, H, L, K, G) // 4,), float("nan"), device="cuda")
    return w, x, up, lay, acts, rest, ckpt, n_ckpt


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_forward_checkpoints(libttt, case):
    _, dt, B, H, L, K, G, tm = case
    w, x, up, lay, acts, rest, ckpt, n_ckpt = _setup(libttt, case)
    plain = libttt.ttt_linear_forward(*acts, *rest, mini_batch=K, eps=w.eps, token_major=tm)
    with_ck = libttt.ttt_linear_forward(*acts, *rest, mini_batch=K, eps=w.eps, token_major=tm, ckpt=ckpt, ckpt_group=G)
    torch.cuda.synchronize()
    for a, b in zip(plain, with_ck):
        assert torch.equal(a, b)
    ck = ckpt.view(B * H, n_ckpt + 1, 64 * 64 + 64)
    Wl, bl = with_ck[1].reshape(B * H, -1), with_ck[2].reshape(B * H, -1)
    assert torch.equal(ck[:, n_ckpt, :4096], Wl) and torch.equal(ck[:, n_ckpt, 4096:], bl)
    heads = torch.arange(B * H, device="cuda") % H
    if n_ckpt > 0:
        assert torch.equal(ck[:, 0, :4096], rest[1].reshape(H, -1)[heads])
        assert torch.equal(ck[:, 0, 4096:], rest[2][heads])
    if n_ckpt > 1:  # the state before mini-batch i*G: the oracle's W_last on that prefix
        i = n_ckpt - 1
        n = i * G * K
        pre = lambda a: np.ascontiguousarray(a[:, :, :n])
        ref = oracle.default().linear_forward(pre(x["XQ"]), pre(x["XK"]), pre(x["XV"]), pre(x["lr"]), x["W0"],
                                              x["b0"], x["ln_w"], x["ln_b"], K, w.eps)
        tol = 1e-2 if dt == "bf16" else 1e-5
        eW = rel_l2(to_np(ck[:, i, :4096]), np.asarray(ref["W_last"]).reshape(w.chains, -1))
        eb = rel_l2(to_np(ck[:, i, 4096:]), np.asarray(ref["b_last"]).reshape(w.chains, -1))
        print(f"[checkpoint {i} of {case[0]}] W {eW:.2e} b {eb:.2e}")
        assert eW <= tol and eb <= tol


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_backward_from_forward_checkpoints(libttt, case):
    name, dt, B, H, L, K, G, tm = case
    w, x, up, lay, acts, rest, ckpt, n_ckpt = _setup(libttt, case)
    libttt.ttt_linear_forward(*acts, *rest, mini_batch=K, eps=w.eps, token_major=tm, ckpt=ckpt, ckpt_group=G)
    g = libttt.ttt_linear_backward(*acts, *rest, lay(dev_act(up, "d_out")), dev_f32(up["dW_last"]),
                                   dev_f32(up["db_last"]), mini_batch=K, eps=w.eps, ckpt_group=G, token_major=tm,
                                   ckpt=ckpt)
    torch.cuda.synchronize()
    if tm:
        for k in ("dXQ", "dXK", "dXV"):
            g[k] = g[k].transpose(1, 2).contiguous()
    ids = list(range(w.chains))
    ref = _oracle(w, synth.linear_inputs(w, chains=ids), synth.upstream_grads(w, chains=ids), ids)
    _compare(w, g, ref, tag=f"from checkpoints {name}")
