"""The layer's output side, Y = o_proj(post_norm(X)) (the walkthrough, "代码连连看——TTT",
TTTBase.forward after the concatenation), through the C ABI on the GPU, against the oracle.

The kernel multiplies the raw bf16 X by the bf16 weight ln_w[k] Wo[n][k] in one tcgen05 GEMM and
applies the token's LayerNorm statistics in the epilogue; the oracle normalises each token in
float64 and multiplies by Wo.  Both round nothing else, and Y is stored in bf16 (2^-9 relative
per element), so the bar is 1e-2 max relative L2 error per token (row of Y), like the other bf16
outputs.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from parity_util import rel_l2

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _dev_bits(bits, shape):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).reshape(shape)).cuda().view(torch.bfloat16)


def _run(ttt, d, T, C, N, eps=1e-6):
    X = _dev_bits(d["X_bits"], (T, C))
    Wo = _dev_bits(d["Wo_bits"], (N, C))
    ln_w, ln_b = torch.from_numpy(d["ln_w"]).cuda(), torch.from_numpy(d["ln_b"]).cuda()
    Wp, u, v = ttt.ttt_o_proj_prepare(Wo, ln_w, ln_b)
    Y = ttt.ttt_post_norm_o_proj(X, Wp, u, v, eps=eps)
    torch.cuda.synchronize()
    return Y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("T,C,N", [(300, 768, 768), (1, 64, 256), (128, 192, 512), (129, 2048, 2048),
                                   (1000, 2048, 256), (257, 64, 768), (130, 2304, 256)])
def test_post_norm_o_proj_against_oracle(libttt, T, C, N):
    """A ragged last token tile (T not a multiple of 128), a single token, N != C, the smallest C
    (one k-chunk), the model widths of the 125M (768) and 1B (2048) layers, and a row wider than
    the statistics pass keeps in registers (2304 features)."""
    d = synth.oproj_inputs(0x0F0 + T + C + N, T, C, N)
    got = _run(libttt, d, T, C, N)
    ref = oracle.default().post_norm_o_proj(d["X"], d["ln_w"], d["ln_b"], 1e-6, d["Wo"])
    e = rel_l2(got, ref)
    print(f"\n[post_norm o_proj] T={T} C={C} N={N}: max rel L2 per token {e:.2e}")
    assert e <= TOL


def test_post_norm_o_proj_token_offsets_and_eps(libttt):
    """Tokens with a common offset (mean / std up to 3) and another eps."""
    T, C, N = 200, 768, 768
    d = synth.oproj_inputs(0x0F7, T, C, N)
    shift = np.linspace(-3, 3, T, dtype=np.float32)[:, None]
    x = (d["X"] + shift).astype(np.float32)
    d["X_bits"] = synth.f32_to_bf16_bits(x)
    d["X"] = synth.bf16_bits_to_f32(d["X_bits"])
    got = _run(libttt, d, T, C, N, eps=1e-3)
    ref = oracle.default().post_norm_o_proj(d["X"], d["ln_w"], d["ln_b"], 1e-3, d["Wo"])
    assert rel_l2(got, ref) <= TOL


def test_post_norm_o_proj_full_size_sampled(libttt):
    """The 1B layer's output side in the benchmark's launch: T = 8 x 8200 = 65 600 tokens (512 full
    token tiles and one of 64), C = N = 2048; 300 sampled tokens, the last ones included."""
    T, C, N = 8 * 8200, 2048, 2048
    d = synth.oproj_inputs(0x0F8, T, C, N, values=False)
    got = _run(libttt, d, T, C, N)
    rows = np.unique(np.concatenate([np.linspace(0, T - 1, 256).astype(int), np.arange(T - 44, T)]))
    x = synth.bf16_bits_to_f32(d["X_bits"][rows])
    wo = synth.bf16_bits_to_f32(d["Wo_bits"])
    ref = oracle.default().post_norm_o_proj(x, d["ln_w"], d["ln_b"], 1e-6, wo)
    e = rel_l2(got[rows], ref)
    print(f"\n[post_norm o_proj] full size, {len(rows)} tokens: max rel L2 per token {e:.2e}")
    assert e <= TOL
    assert libttt.ttt_device_status() == 0


def test_scan_then_output_side(libttt):
    """The layer's tail as a user chains it: the scan with token-major output feeds the output
    side directly (no permute); checked against the oracle on the scan's own output."""
    w = synth.workload(1, B=2, H=12, L=16 * 9 + 5, seed=0x0F9)
    x = synth.linear_inputs(w)
    acts = [torch.from_numpy(np.ascontiguousarray(x[n + "_bits"]).view(np.int16)).cuda().view(torch.bfloat16)
            .transpose(1, 2).contiguous() for n in ("XQ", "XK", "XV")]
    f32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    out, _, _ = libttt.ttt_linear_forward(*acts, f32(x["lr"]), f32(x["W0"]), f32(x["b0"]), f32(x["ln_w"]),
                                          f32(x["ln_b"]), eps=w.eps, token_major=True)
    C = w.H * 64
    d = synth.oproj_inputs(0x0FA, 1, C, C)
    Wo = _dev_bits(d["Wo_bits"], (C, C))
    Wp, u, v = libttt.ttt_o_proj_prepare(Wo, f32(d["ln_w"]), f32(d["ln_b"]))
    Y = libttt.ttt_post_norm_o_proj(out.reshape(w.B, w.L, C), Wp, u, v, eps=1e-6)  # [B, L, H*64], no copy
    torch.cuda.synchronize()
    assert Y.shape == (w.B, w.L, C)
    xs = out.reshape(-1, C).float().cpu().numpy()
    ref = oracle.default().post_norm_o_proj(xs, d["ln_w"], d["ln_b"], 1e-6, d["Wo"])
    assert rel_l2(Y.reshape(-1, C).float().cpu().numpy(), ref) <= TOL


def test_post_norm_o_proj_bounded_wait_timeout(libttt):
    """Every bounded wait gives up at once: every role of the persistent kernel stops, the tensor
    core and the loads in flight drain, tensor memory is freed, the status word says so, and the
    next call is correct."""
    T, C, N = 700, 512, 512
    d = synth.oproj_inputs(0x0FB, T, C, N)
    libttt.ttt_device_status(clear=True)
    libttt.ttt_set_wait_limit(-1)
    try:
        _run(libttt, d, T, C, N)
        with pytest.raises(libttt.TTTError) as e:
            libttt.ttt_device_status(clear=True)
        assert e.value.code == libttt.TTT_ERR_TIMEOUT
    finally:
        libttt.ttt_set_wait_limit(0)
    assert libttt.ttt_device_status(clear=True) == 0
    ref = oracle.default().post_norm_o_proj(d["X"], d["ln_w"], d["ln_b"], 1e-6, d["Wo"])
    assert rel_l2(_run(libttt, d, T, C, N), ref) <= TOL
    assert libttt.ttt_device_status() == 0
