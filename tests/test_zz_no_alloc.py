"""The allocation-free host-buffer entry point (ttt_linear_forward_host_static).

Some callers cannot allocate device memory: their memory belongs to another owner that handed
it all out in advance (a serving framework's pool, a fixed budget), or they are plain host
programs without a device allocator, or they cannot afford the synchronisation an allocation
may cause.  For them the library stages the batch through a static device array of its own.
This test calls that entry point through the C ABI twice in a row and checks both results
against the workspace-based entry point (ttt_linear_forward_host) on the same values, at the
bf16 tolerance of the other parity tests; and that a size whose one batch row does not fit the
built-in scratch is refused with a clear error.  It lives in its own file, named to be collected
last, and passes both alone in a fresh process and after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import synth
from parity_util import rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _host_act(x, name):
    return torch.from_numpy(np.ascontiguousarray(x[name + "_bits"]).view(np.int16)).view(torch.bfloat16).pin_memory()


def _host_f32(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).pin_memory()


def test_static_scratch_entry_matches_the_workspace_entry_twice(libttt):
    # (3, 4, 327): the whole batch in one chunk of the scratch, a tail of 7 tokens;
    # (4, 16, 1033): about 8.5 MB of staging per batch row, so the 32 MiB scratch takes the batch
    # in two chunks (3 rows, then 1), a tail of 9 tokens
    for B, H, L in ((3, 4, 16 * 20 + 7), (4, 16, 16 * 64 + 9)):
        w = synth.workload(1, B=B, H=H, L=L, seed=0x57A7 + L)
        x = synth.linear_inputs(w, values=False)
        args = (_host_act(x, "XQ"), _host_act(x, "XK"), _host_act(x, "XV"), _host_f32(x["lr"]), _host_f32(x["W0"]),
                _host_f32(x["b0"]), _host_f32(x["ln_w"]), _host_f32(x["ln_b"]))
        ref = libttt.ttt_linear_forward_host(*args, mini_batch=w.K, eps=w.eps, tail_grads=True, chunk_batches=B)
        torch.cuda.synchronize()
        for call in range(2):
            got = libttt.ttt_linear_forward_host_static(*args, mini_batch=w.K, eps=w.eps, tail_grads=True)
            torch.cuda.synchronize()
            for name, g, r in zip(("out", "W_last", "b_last", "W_grad_tail", "b_grad_tail"), got, ref):
                e = rel_l2(g.float().numpy().reshape(B * H, -1), r.float().numpy().reshape(B * H, -1))
                assert e <= TOL, (B, H, L, call, name, e)
    assert libttt.ttt_device_status() == 0


def test_static_scratch_entry_refuses_sizes_past_its_scratch(libttt):
    # one batch row of 32 heads x 8200 tokens stages about 134 MB, past the 32 MiB scratch
    B, H, L = 1, 32, 8200
    z = torch.zeros((B, H, L, 64), dtype=torch.bfloat16)
    lr = torch.zeros((B, H, L))
    W0, b0, lw, lb = torch.zeros((H, 64, 64)), torch.zeros((H, 64)), torch.ones((H, 64)), torch.zeros((H, 64))
    with pytest.raises(libttt.TTTError) as e:
        libttt.ttt_linear_forward_host_static(z, z, z, lr, W0, b0, lw, lb)
    assert e.value.code == libttt.TTT_ERR_ARG
    assert "built-in scratch" in str(e.value)
