"""Benchmark of the TTT scan on B200: TTT layer tokens/s and the fraction of the per-layer roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--rows linear,linear_tm,linear_rope,oproj,backward,mlp,decode,decode_hist]
                    [--no-cpu-baseline] [--no-headline] [--seq-len L]

One step = one ttt_linear_forward over the 1B-layer workload (B=8, H=32, L=8200, d=64, K=16,
bf16 activations, fp32 state): every row of the path at once -- the partition, 512 full
mini-batches, the 8-token remainder, the tail grads.  Tokens per step = B * L.  Inputs come from
the seeded generator (synth/), resident in HBM before timing; they are 806 MB per step, larger
than the 126 MB L2, so no flush is needed between steps.

Multi-GPU (torchrun, one rank per GPU): every rank runs the same workload on its own GPU (the
chains are independent; there is no exchange), `value` counts all ranks' tokens over the
slowest rank's device time ("scaling": "weak").

The JSON line also carries: `e2e` (the same scan through the host-buffer entry point
ttt_linear_forward_host from pinned HOST buffers, every input copied in and every result copied
out inside the timed region, the batch pipelined in chunks),
`roofline` (the scan kernel's algorithmic bytes / its CUDA-event time vs the measured HBM copy
bandwidth), `cpu_baseline` (the CPU oracle on a bounded sample, rank 0 at N=1), `clocks`
(NVML samples taken during the timed region) and `rows` (the same scan on token-major
[B,L,H,d] activations beside the time of the permutes that layout saves, the scan with the
rotary embedding fused into its load path, the layer's output side post_norm + o_proj, the
scan's backward with checkpoint groups, the TTT-MLP prefill, the decode step with the dense
cache and with the history-format cache, each timed the same way).  `--impl reference` times the oracle instead, as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402
from test_rnn_layers_b200.shard import aggregate_tokens_per_s  # noqa: E402

D = 64
HBM_FALLBACK_GBS = 6650.0
BF16_FALLBACK_TFLOPS = 1590.0


# ---------------------------------------------------------------------------------------------
# algorithmic work (bytes that must cross HBM, tensor FLOPs) of one call
# ---------------------------------------------------------------------------------------------
def linear_bytes(B, H, L, tail_grads=True):
    """Reads: XQ, XK, XV (bf16), lr (fp32), W0/b0 and ln_w/ln_b per head.  Writes: out (bf16),
    W_last/b_last per chain, and the tail grads when requested."""
    chains = B * H
    per_token = 3 * D * 2 + 4 + D * 2
    state = (D * D + D) * 4
    return chains * L * per_token + H * state + H * 2 * D * 4 + chains * state * (2 if tail_grads else 1)


def linear_flops(B, H, L, K=16):
    """Dense Z = XK W, XQ W and the rank-K update (3 x 2 K d^2 per mini-batch) plus the
    lower-triangular XQ XK^T, (eta*A) g and tril(eta) g (3 x 2 d K(K+1)/2)."""
    n_mb = L // K + (1 if L % K else 0)
    return B * H * n_mb * (3 * 2 * K * D * D + 3 * 2 * D * K * (K + 1) // 2)


def mlp_bytes(B, H, L, hid=256):
    chains = B * H
    state = (2 * D * hid + hid + D) * 4
    return chains * L * (3 * D * 2 + 4 + D * 2) + H * state + H * 2 * D * 4 + chains * state


def mlp_flops(B, H, L, hid=256, K=16):
    n_mb = L // K + (1 if L % K else 0)
    dense = 7 * 2 * K * D * hid                  # Z1, XQ W1, Z2, Xbar2 W2, g2 W2^T, two updates
    tri = 2 * (K * (K + 1) // 2) * (2 * D + 2 * hid)  # Attn1, Attn2, M1 g1, M2 g2
    return B * H * n_mb * (dense + tri)


def linear_bwd_bytes(B, H, L):
    """The backward, once through: reads XQ, XK, XV, d_out (bf16) and lr per token, W0/b0 and
    ln_w/ln_b per head, dW_last/db_last per chain; writes dXQ, dXK, dXV (bf16) and d_lr per token,
    dW0/db0 and d ln_w / d ln_b per head."""
    chains = B * H
    state = (D * D + D) * 4
    per_token = 4 * D * 2 + 4 + 3 * D * 2 + 4
    return chains * L * per_token + 2 * H * state + chains * state + 2 * H * 2 * D * 4


def linear_bwd_flops(B, H, L, K=16):
    """The products the chain rule needs per mini-batch once its Z, g and Zbar are known:
    XK dW', g dW'^T, dZbar W^T, dZ W^T, XQ^T dZbar, XK^T dZ (6 x 2 K d^2) and the lower-triangular
    M^T dZbar, dZbar g^T, dA XK, dA^T XQ (4 x 2 d K(K+1)/2).  Rebuilding the states and the
    forward quantities (Z, XQ W, XQ XK^T, M g, the state updates) is not counted."""
    n_mb = L // K + (1 if L % K else 0)
    return B * H * n_mb * (6 * 2 * K * D * D + 4 * 2 * D * K * (K + 1) // 2)


# dense TF32 tensor peak as the nominal ratio to bf16 (1.1 / 2.25 PFLOP/s) times the bf16 peak in use
TF32_PER_BF16 = 1.1 / 2.25


def decode_hist_bytes(B, H, p, K=16):
    """One step of the history-format cache at position p, per chain: read W, b, b_grad and p
    rows of (lr xk, g); write one row and b_grad, or W, b and b_grad on the commit step; tokens
    xq, xk, xv, lr in, out out (bf16)."""
    state = (D * D + D) * 4
    rows = p * 2 * D * 4
    write = state + D * 4 if p == K - 1 else 2 * D * 4 + D * 4
    return B * H * (state + D * 4 + rows + write + 3 * D * 2 + 4 + D * 2)


def decode_bytes(B, H, commit_fraction=1.0 / 16):
    """Per step and chain: read W, b, W_grad, b_grad; write W_grad, b_grad (and W, b on the
    commit step, once per K steps); tokens xq, xk, xv, lr in, out out (bf16)."""
    state = (D * D + D) * 4
    return B * H * (3 * state + commit_fraction * state + 3 * D * 2 + 4 + D * 2)


# ---------------------------------------------------------------------------------------------
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    return HBM_FALLBACK_GBS, BF16_FALLBACK_TFLOPS, 1400.0, "fallback"


def kernel_traffic(kernel_src: str, key: str):
    """dram bytes per launch from the committed ncu summary, if the kernel source is unchanged
    since the counters were taken (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    src = os.path.join(ROOT, "test_rnn_layers_b200", "csrc", kernel_src)
    if not os.path.exists(path) or not os.path.exists(src):
        return None
    with open(path) as f:
        rec = json.load(f).get(key)
    if not rec:
        return None
    digest = hashlib.sha256(open(src, "rb").read()).hexdigest()
    return rec.get("dram_bytes_per_launch") if rec.get("source_sha256") == digest else None


class ClockSampler:
    """NVML samples of SM clock and clock-event reasons on one GPU, in a thread (read-only)."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples = []
        self.period = period_s
        self.index = device_index
        self._stop = threading.Event()
        self._thread = None
        self.active = False

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            self.max_mhz = None
            return self
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.samples.append((time.perf_counter(), mhz, reasons, self.active))
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()
        return False

    def summary(self):
        busy = [s for s in self.samples if s[3]]
        if not busy:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mask = 0
        for s in busy:
            mask |= s[2]
        reasons = sorted(n for bit, n in self.REASONS.items() if mask & bit and n != "gpu_idle")
        return {"sm_mhz": statistics.median(s[1] for s in busy), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(busy)}


# ---------------------------------------------------------------------------------------------
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v):
    from test_rnn_layers_b200.shard import max_over_ranks as _max
    return _max(v) if world > 1 else v


def time_steps(step, K, W, world, sampler=None):
    """W untimed steps, then exactly K steps between CUDA events on the current stream, with a
    barrier and a device synchronise on both sides; returns ms per step (max over ranks)."""
    import torch
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.active = True
    e0.record(s)
    for _ in range(K):
        step()
    e1.record(s)
    torch.cuda.synchronize()
    if sampler:
        sampler.active = False
    barrier(world)
    torch.cuda.synchronize()
    return max_over_ranks(world, e0.elapsed_time(e1) / K)


def dev_act(x, name):
    import torch
    bits = np.ascontiguousarray(x[name + "_bits"]).view(np.int16)
    return torch.from_numpy(bits).cuda().view(torch.bfloat16)


def dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


# ---------------------------------------------------------------------------------------------
def bench_linear(args, world, rank, local, peaks):
    import torch

    import test_rnn_layers_b200 as ttt
    w = synth.workload(2, L=args.seq_len)
    x = synth.linear_inputs(w, values=False)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    lr, W0, b0, lnw, lnb = (dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b"))
    B, H, L = w.B, w.H, w.L
    out = torch.empty_like(XQ)
    Wl, bl = torch.empty(B, H, D, D, device="cuda"), torch.empty(B, H, D, device="cuda")
    Wg, bg = torch.empty(B, H, D, D, device="cuda"), torch.empty(B, H, D, device="cuda")

    def step():
        ttt.ttt_linear_forward(XQ, XK, XV, lr, W0, b0, lnw, lnb, mini_batch=w.K, eps=w.eps, out=out,
                               W_last=Wl, b_last=bl, W_grad_tail=Wg, b_grad_tail=bg, tail_grads=True)

    with ClockSampler(local) as clk:
        ms = time_steps(step, args.steps, args.warmup, world, clk)
    ttt.ttt_device_status()  # raises if a kernel gave up on a bounded wait
    tokens = B * L
    value = aggregate_tokens_per_s(tokens, world, ms)
    hbm, tf_burst, _, which = peaks
    nbytes = linear_bytes(B, H, L)
    achieved = nbytes / (ms / 1e3) / 1e9
    traffic = kernel_traffic("linear_tc.cu", "linear_tc_kernel@1b_B8_H32_L8200") if L == 8200 else None

    # end to end through the public host-buffer call (ttt_linear_forward_host) from pinned host
    # buffers: every step copies all inputs in and all results out, inside the timed region
    pin = lambda t: t.cpu().pin_memory()  # noqa: E731
    host_in = {"XQ": pin(XQ), "XK": pin(XK), "XV": pin(XV), "lr": pin(lr), "W0": pin(W0), "b0": pin(b0),
               "ln_w": pin(lnw), "ln_b": pin(lnb)}
    host_out = {"out": torch.empty(XQ.shape, dtype=XQ.dtype, pin_memory=True),
                "W_last": torch.empty(Wl.shape, pin_memory=True), "b_last": torch.empty(bl.shape, pin_memory=True),
                "W_grad_tail": torch.empty(Wg.shape, pin_memory=True),
                "b_grad_tail": torch.empty(bg.shape, pin_memory=True)}
    ws = torch.empty(ttt.ttt_linear_host_workspace_bytes(B, H, L, w.K, XQ.dtype, args.e2e_chunk),
                     dtype=torch.uint8, device="cuda")

    def e2e_step():
        ttt.ttt_linear_forward_host(host_in["XQ"], host_in["XK"], host_in["XV"], host_in["lr"], host_in["W0"],
                                    host_in["b0"], host_in["ln_w"], host_in["ln_b"], mini_batch=w.K, eps=w.eps,
                                    out=host_out["out"], W_last=host_out["W_last"], b_last=host_out["b_last"],
                                    W_grad_tail=host_out["W_grad_tail"], b_grad_tail=host_out["b_grad_tail"],
                                    tail_grads=True, chunk_batches=args.e2e_chunk, workspace=ws)

    e2e_K = max(3, min(args.steps, 10))
    e2e_ms = time_steps(e2e_step, e2e_K, 2, world)
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())
    del ws

    line = {
        "metric": "TTT layer tokens/sec (1B shapes, B200) and % of per-layer roofline",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded generator, synth/)",
        "config": {"workload": "ttt_linear_prefill_1b_layer", "B": B, "H": H, "L": L, "d": D,
                   "mini_batch": w.K, "chains_per_gpu": B * H, "global_batch": B * world,
                   "activations": "bf16 [B,H,L,d]", "state": "fp32",
                   "l2": f"inputs larger than L2 ({3 * B * H * L * D * 2 / 1e6:.0f} MB read per step), no flush",
                   "parallelism": f"independent chains, {world} GPU(s), no collective"},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "kernel": "linear_tc_kernel", "achieved": round(achieved, 1),
                     "peak": hbm, "peak_source": f"{which} hbm_gbs", "unit": "GB/s",
                     "frac": round(achieved / hbm, 4), "algorithmic_bytes": nbytes,
                     "traffic": traffic,
                     "tensor_tflops": round(linear_flops(B, H, L) / (ms / 1e3) / 1e12, 2),
                     "tensor_frac_of_bf16_peak": round(linear_flops(B, H, L) / (ms / 1e3) / 1e12 / tf_burst, 4)},
        "e2e": {"value": round(world * tokens / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "call": "ttt_linear_forward_host", "chunk_batches": args.e2e_chunk},
        "clocks": clk.summary(),
    }
    return line


def bench_linear_token_major(args, world, peaks):
    """The headline scan on token-major [B,L,H,d] activations (TTT_FLAG_TOKEN_MAJOR: the layout
    the QKV projections produce and the layer returns), and beside it the time of the four
    [B,H,L,d] <-> [B,L,H,d] copies (XQ, XK, XV in, out back) that the flag makes unnecessary."""
    import torch

    import test_rnn_layers_b200 as ttt
    w = synth.workload(2, L=args.seq_len)
    x = synth.linear_inputs(w, values=False)
    XQ, XK, XV = (dev_act(x, n).transpose(1, 2).contiguous() for n in ("XQ", "XK", "XV"))
    lr, W0, b0, lnw, lnb = (dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b"))
    B, H, L = w.B, w.H, w.L
    out = torch.empty_like(XQ)
    Wl, bl = torch.empty(B, H, D, D, device="cuda"), torch.empty(B, H, D, device="cuda")
    Wg, bg = torch.empty(B, H, D, D, device="cuda"), torch.empty(B, H, D, device="cuda")

    def step():
        ttt.ttt_linear_forward(XQ, XK, XV, lr, W0, b0, lnw, lnb, mini_batch=w.K, eps=w.eps, out=out,
                               W_last=Wl, b_last=bl, W_grad_tail=Wg, b_grad_tail=bg, tail_grads=True,
                               token_major=True)

    K = max(3, min(args.steps, 10))
    ms = time_steps(step, K, 3, world)
    ttt.ttt_device_status()
    hm = [torch.empty(B, H, L, D, dtype=XQ.dtype, device="cuda") for _ in range(4)]

    def permutes():  # what a head-major scan needs around it: 3 inputs in, the output back
        for src, dst in zip((XQ, XK, XV), hm[:3]):
            dst.copy_(src.transpose(1, 2))
        out.copy_(hm[3].transpose(1, 2))

    perm_ms = time_steps(permutes, K, 3, world)
    hbm = peaks[0]
    nbytes = linear_bytes(B, H, L)
    achieved = nbytes / (ms / 1e3) / 1e9
    return {"workload": f"ttt_linear_prefill_1b_layer_token_major_B{B}_H{H}_L{L}", "activations": "bf16 [B,L,H,d]",
            "value": round(world * B * L / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "steps": K, "gpu_launches": K,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(achieved / hbm, 4), "algorithmic_bytes": nbytes},
            "replaced_permutes_ms": round(perm_ms, 4)}


def bench_linear_rope(args, world, peaks, theta=10000.0):
    """The headline scan with the rotary embedding of XQ and XK fused into its load path
    (ttt_linear_forward_rope, pairs (2k, 2k+1), positions t mod K), and beside it the unfused way:
    XQ and XK rotated by torch and written back in bf16 (the walkthrough's apply_rotary_pos_emb on
    [B,H,L,d]), then the plain scan.  Also the HBM floor of any unfused pass: reading and writing
    XQ and XK once at the measured copy bandwidth."""
    import torch

    import test_rnn_layers_b200 as ttt
    w = synth.workload(2, L=args.seq_len)
    x = synth.linear_inputs(w, values=False)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    lr, W0, b0, lnw, lnb = (dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b"))
    B, H, L = w.B, w.H, w.L
    out = torch.empty_like(XQ)
    Wl, bl = torch.empty(B, H, D, D, device="cuda"), torch.empty(B, H, D, device="cuda")
    Wg, bg = torch.empty(B, H, D, D, device="cuda"), torch.empty(B, H, D, device="cuda")

    def fused():
        ttt.ttt_linear_forward_rope(XQ, XK, XV, lr, W0, b0, lnw, lnb, mini_batch=w.K, eps=w.eps, rope_theta=theta,
                                    out=out, W_last=Wl, b_last=bl, W_grad_tail=Wg, b_grad_tail=bg, tail_grads=True)

    K = max(3, min(args.steps, 10))
    ms = time_steps(fused, K, 3, world)
    ttt.ttt_device_status()
    pos = (torch.arange(L, device="cuda") % w.K).float()
    inv = 1.0 / theta ** (torch.arange(0, D, 2, device="cuda").float() / D)
    cos, sin = torch.cos(pos[:, None] * inv), torch.sin(pos[:, None] * inv)  # [L, d/2], outside the timing
    rq, rk = torch.empty_like(XQ), torch.empty_like(XK)

    def rope_pass():
        for src, dst in ((XQ, rq), (XK, rk)):
            p = src.float().view(B, H, L, D // 2, 2)
            a, b = p[..., 0], p[..., 1]
            dst.copy_(torch.stack((a * cos - b * sin, a * sin + b * cos), -1).view(B, H, L, D))

    def unfused():
        rope_pass()
        ttt.ttt_linear_forward(rq, rk, XV, lr, W0, b0, lnw, lnb, mini_batch=w.K, eps=w.eps, out=out, W_last=Wl,
                               b_last=bl, W_grad_tail=Wg, b_grad_tail=bg, tail_grads=True)

    rope_ms = time_steps(rope_pass, K, 3, world)
    unfused_ms = time_steps(unfused, K, 3, world)
    hbm = peaks[0]
    nbytes = linear_bytes(B, H, L)
    achieved = nbytes / (ms / 1e3) / 1e9
    pass_bytes = 4 * B * H * L * D * 2  # XQ, XK read and written once in bf16
    return {"workload": f"ttt_linear_prefill_1b_layer_rope_B{B}_H{H}_L{L}", "rope": f"theta {theta:g}, pairs (2k, 2k+1)",
            "value": round(world * B * L / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "steps": K, "gpu_launches": K,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                         "frac": round(achieved / hbm, 4), "algorithmic_bytes": nbytes},
            "unfused_ms": round(unfused_ms, 4), "unfused_rope_pass_ms": round(rope_ms, 4),
            "unfused_rope_pass_hbm_floor_ms": round(pass_bytes / (hbm * 1e9) * 1e3, 4)}


def bench_post_norm_oproj(args, world, peaks):
    """The layer's output side at the 1B layer, Y = o_proj(post_norm(X)) for the scan's
    token-major output ([B*L, 2048] bf16): a token-statistics pass and one tcgen05 GEMM with the
    LayerNorm folded into its epilogue (ttt_post_norm_o_proj, two launches; the weight packed once
    beforehand, outside the timing), and beside it the unfused torch way (layer_norm, then a cuBLAS
    matmul)."""
    import torch

    import test_rnn_layers_b200 as ttt
    B, L, C = 8, args.seq_len, 2048
    T = B * L
    d = synth.oproj_inputs(0x0B5, T, C, C, values=False)
    bits = lambda b, shape: torch.from_numpy(np.ascontiguousarray(b).view(np.int16).reshape(shape)).cuda().view(
        torch.bfloat16)
    X, Wo = bits(d["X_bits"], (T, C)), bits(d["Wo_bits"], (C, C))
    ln_w, ln_b = torch.from_numpy(d["ln_w"]).cuda(), torch.from_numpy(d["ln_b"]).cuda()
    Wp, u, v = ttt.ttt_o_proj_prepare(Wo, ln_w, ln_b)
    Y = torch.empty_like(X)
    stats = torch.empty((T, 2), device="cuda")

    def fused():
        ttt.ttt_post_norm_o_proj(X, Wp, u, v, eps=1e-6, Y=Y, row_stats=stats)

    K = max(3, min(args.steps, 20))
    ms = time_steps(fused, K, 3, world)
    ttt.ttt_device_status()

    def unfused():
        torch.matmul(torch.nn.functional.layer_norm(X, (C,), ln_w.bfloat16(), ln_b.bfloat16(), 1e-6), Wo.t(), out=Y)

    torch_ms = time_steps(unfused, K, 3, world)
    flops = 2.0 * T * C * C
    peak = peaks[1]
    tf = flops / (ms / 1e3) / 1e12
    return {"workload": f"ttt_post_norm_o_proj_1b_layer_T{T}_C{C}", "value": round(world * T / (ms / 1e3), 1),
            "unit": "tokens/s", "ms_per_step": round(ms, 4), "steps": K, "gpu_launches": 2 * K,
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak,
                         "peak_source": ("measured" if peaks[3] == "measured" else "fallback") + " bf16_tflops",
                         "unit": "TFLOP/s", "frac": round(tf / peak, 4), "algorithmic_flops": int(flops)},
            "unfused_torch_ms": round(torch_ms, 4)}


def bench_linear_backward(args, world, peaks, G=16):
    """The backward of the TTT-Linear scan at the 1B layer (ttt_linear_backward, checkpoint group
    16): the gradients of XQ, XK, XV, lr, W0, b0, ln_w and ln_b from d_out, dW_last and db_last,
    the inputs and upstream gradients resident in HBM (each larger than L2).  bf16 activations run
    the tensor-core kernel (TF32 products), whose roofline is the larger of the HBM time of its
    algorithmic bytes and the TF32 time of its algorithmic FLOPs: the HBM one.  Under torchrun
    each rank runs its own batch (weak scaling) and the step ends with the one exchange data-
    parallel training needs: the all-reduce of the shared-parameter gradients (dW0, db0, d ln_w,
    d ln_b), NCCL."""
    import torch

    import test_rnn_layers_b200 as ttt
    w = synth.workload(2, L=args.seq_len)
    x, up = synth.linear_inputs(w, values=False), synth.upstream_grads(w, values=False)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    dout = dev_act(up, "d_out")
    t = {k: dev_f32(x[k]) for k in ("lr", "W0", "b0", "ln_w", "ln_b")}
    dWl, dbl = dev_f32(up["dW_last"]), dev_f32(up["db_last"])
    del x, up
    ws = torch.empty(ttt.ttt_linear_backward_workspace_bytes(w.B, w.H, w.L, w.K, G), dtype=torch.uint8, device="cuda")

    from test_rnn_layers_b200.shard import allreduce_shared_grads

    def step():
        g = ttt.ttt_linear_backward(XQ, XK, XV, t["lr"], t["W0"], t["b0"], t["ln_w"], t["ln_b"], dout, dWl, dbl,
                                    mini_batch=w.K, eps=w.eps, ckpt_group=G, workspace=ws)
        if world > 1:
            allreduce_shared_grads(g)

    K = max(3, min(args.steps, 10))
    ms = time_steps(step, K, 3, world)
    # the same with every state kept (checkpoint group 1: 2.2 GB of workspace, no rebuild)
    del ws
    ws = torch.empty(ttt.ttt_linear_backward_workspace_bytes(w.B, w.H, w.L, w.K, 1), dtype=torch.uint8, device="cuda")

    def step_all_states():
        g = ttt.ttt_linear_backward(XQ, XK, XV, t["lr"], t["W0"], t["b0"], t["ln_w"], t["ln_b"], dout, dWl, dbl,
                                    mini_batch=w.K, eps=w.eps, ckpt_group=1, workspace=ws)
        if world > 1:
            allreduce_shared_grads(g)

    ms_all = time_steps(step_all_states, K, 3, world)
    ws_all = ws.numel()
    del ws
    # the training split: the forward's checkpoints (ttt_linear_forward_ckpt, written once before
    # the timed region) and the backward from them (ttt_linear_backward_ckpt), which skips its own
    # pass of the state recursion
    ws = torch.empty(ttt.ttt_linear_backward_workspace_bytes(w.B, w.H, w.L, w.K, G), dtype=torch.uint8, device="cuda")
    ckpt = torch.empty(ttt.ttt_linear_ckpt_bytes(w.B, w.H, w.L, w.K, G) // 4, device="cuda")
    ttt.ttt_linear_forward(XQ, XK, XV, t["lr"], t["W0"], t["b0"], t["ln_w"], t["ln_b"], mini_batch=w.K, eps=w.eps,
                           ckpt=ckpt, ckpt_group=G)

    def step_from_ckpt():
        g = ttt.ttt_linear_backward(XQ, XK, XV, t["lr"], t["W0"], t["b0"], t["ln_w"], t["ln_b"], dout, dWl, dbl,
                                    mini_batch=w.K, eps=w.eps, ckpt_group=G, workspace=ws, ckpt=ckpt)
        if world > 1:
            allreduce_shared_grads(g)

    ms_ck = time_steps(step_from_ckpt, K, 3, world)
    del ws, ckpt
    # a whole training step of the layer's scan at checkpoint groups G and 1 (every state kept):
    # the forward with checkpoints, then the backward from them
    train = {}
    for Gt in (G, 1):
        ws = torch.empty(ttt.ttt_linear_backward_workspace_bytes(w.B, w.H, w.L, w.K, Gt), dtype=torch.uint8,
                         device="cuda")
        ckpt = torch.empty(ttt.ttt_linear_ckpt_bytes(w.B, w.H, w.L, w.K, Gt) // 4, device="cuda")

        def train_step(Gt=Gt, ws=ws, ckpt=ckpt):
            ttt.ttt_linear_forward(XQ, XK, XV, t["lr"], t["W0"], t["b0"], t["ln_w"], t["ln_b"], mini_batch=w.K,
                                   eps=w.eps, ckpt=ckpt, ckpt_group=Gt)
            g = ttt.ttt_linear_backward(XQ, XK, XV, t["lr"], t["W0"], t["b0"], t["ln_w"], t["ln_b"], dout, dWl, dbl,
                                        mini_batch=w.K, eps=w.eps, ckpt_group=Gt, workspace=ws, ckpt=ckpt)
            if world > 1:
                allreduce_shared_grads(g)

        ms_t = time_steps(train_step, K, 3, world)
        train[f"ckpt_group_{Gt}"] = {"ms_per_step": round(ms_t, 4), "value": round(world * w.B * w.L / (ms_t / 1e3), 1),
                                     "checkpoint_bytes": ckpt.numel() * 4}
        del ws, ckpt
    flops, nbytes = linear_bwd_flops(w.B, w.H, w.L), linear_bwd_bytes(w.B, w.H, w.L)
    tfl = flops / (ms / 1e3) / 1e12
    gbs = nbytes / (ms / 1e3) / 1e9
    hbm, bf16_peak, _, which = peaks
    tf32_peak = bf16_peak * TF32_PER_BF16
    return {"workload": f"ttt_linear_backward_1b_layer_B{w.B}_H{w.H}_L{w.L}_ckpt{G}",
            "value": round(world * w.B * w.L / (ms / 1e3), 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
            "steps": K, "gpu_launches": 2 * K, "dtype": "bf16 in/out, tf32 products, f32 accumulation and state",
            "collective": (f"all_reduce (sum, NCCL) of the shared-parameter gradients, {(w.H * (D * D + 3 * D)) * 4} "
                           "bytes per step" if world > 1 else "none (one GPU)"),
            "every_state_kept": {"ckpt_group": 1, "ms_per_step": round(ms_all, 4),
                                 "value": round(world * w.B * w.L / (ms_all / 1e3), 1), "workspace_bytes": ws_all},
            "from_forward_checkpoints": {"ckpt_group": G, "call": "ttt_linear_backward_ckpt",
                                         "ms_per_step": round(ms_ck, 4),
                                         "value": round(world * w.B * w.L / (ms_ck / 1e3), 1)},
            "training_step": dict(train, calls="ttt_linear_forward_ckpt then ttt_linear_backward_ckpt"),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm, "peak_source": f"{which} hbm_gbs",
                         "unit": "GB/s", "frac": round(gbs / hbm, 4), "algorithmic_bytes": nbytes,
                         "floor_ms": round(nbytes / hbm / 1e6, 4), "algorithmic_flops": flops,
                         "tensor_tflops": round(tfl, 2),
                         "tensor_frac_tf32": round(tfl / tf32_peak, 4),
                         "tf32_peak": round(tf32_peak, 1)}}


def bench_mlp(args, world, peaks):
    import torch

    import test_rnn_layers_b200 as ttt
    w = synth.workload(3)
    x = synth.linear_inputs(w, values=False)
    XQ, XK, XV = (dev_act(x, n) for n in ("XQ", "XK", "XV"))
    t = {k: dev_f32(x[k]) for k in ("lr", "W1", "b1", "W2", "b2", "ln_w", "ln_b")}
    out = torch.empty_like(XQ)

    def step():
        ttt.ttt_mlp_forward(XQ, XK, XV, t["lr"], t["W1"], t["b1"], t["W2"], t["b2"], t["ln_w"], t["ln_b"],
                            mini_batch=w.K, eps=w.eps, out=out)

    K = max(3, min(args.steps, 10))
    ms = time_steps(step, K, 3, world)
    flops = mlp_flops(w.B, w.H, w.L)
    hbm, tf_burst, _, which = peaks
    tfl = flops / (ms / 1e3) / 1e12
    return {"workload": "ttt_mlp_prefill_B8_H32_L2048_h256", "value": round(world * w.B * w.L / (ms / 1e3), 1),
            "unit": "tokens/s", "ms_per_step": round(ms, 4), "steps": K, "gpu_launches": K,
            "roofline": {"bound": "tensor", "achieved": round(tfl, 2), "peak": tf_burst,
                         "peak_source": f"{which} bf16_tflops", "unit": "TFLOP/s",
                         "frac": round(tfl / tf_burst, 4), "algorithmic_flops": flops,
                         "hbm_frac": round(mlp_bytes(w.B, w.H, w.L) / (ms / 1e3) / 1e9 / hbm, 4)}}


def bench_decode(args, world, peaks, hist=False):
    """The decode step, dense cache (ttt_linear_decode_step) or history-format cache
    (ttt_linear_decode_step_hist), from the state of a 2048-token prefill."""
    import torch

    import test_rnn_layers_b200 as ttt
    w = synth.workload(4, decode_steps=64)
    x = synth.linear_inputs(w, values=False, t1=w.L)
    _, W, b, Wg, bg = ttt.ttt_linear_forward(dev_act(x, "XQ"), dev_act(x, "XK"), dev_act(x, "XV"),
                                             dev_f32(x["lr"]), dev_f32(x["W0"]), dev_f32(x["b0"]),
                                             dev_f32(x["ln_w"]), dev_f32(x["ln_b"]), eps=w.eps, tail_grads=True)
    lnw, lnb = dev_f32(x["ln_w"]), dev_f32(x["ln_b"])
    del x
    if hist:  # 2048 is a mini-batch boundary: the history cache starts empty
        del Wg
        rows = torch.zeros(w.B, w.H, w.K, 2, D, device="cuda")
    toks = synth.linear_inputs(w, values=False, t0=w.L, t1=w.L + w.decode_steps)
    XQ, XK, XV = (dev_act(toks, n) for n in ("XQ", "XK", "XV"))
    lr = dev_f32(toks["lr"])
    out = torch.empty(w.B, w.H, D, dtype=torch.bfloat16, device="cuda")
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device="cuda")
    xs = [(XQ[:, :, i].contiguous(), XK[:, :, i].contiguous(), XV[:, :, i].contiguous(), lr[:, :, i].contiguous())
          for i in range(w.decode_steps)]
    pos = [w.L]

    def one(i):
        q, k, v, l = xs[i % w.decode_steps]
        if hist:
            ttt.ttt_linear_decode_step_hist(q, k, v, l, lnw, lnb, W, b, rows, bg, seqlen_offset=pos[0], eps=w.eps,
                                            out=out)
        else:
            ttt.ttt_linear_decode_step(q, k, v, l, lnw, lnb, W, b, Wg, bg, seqlen_offset=pos[0], eps=w.eps, out=out)
        pos[0] += 1

    # each timed step starts with a cold L2 (the 133 MB state is about the L2 size): a 256 MB read
    # evicts it, and the dirty lines of the step before are written back during that read, not
    # during the timed step
    K = max(16, args.steps)
    for i in range(3):
        one(i)
    flush.fill_(1.0)
    s = torch.cuda.current_stream()
    total = 0.0
    nbytes_total = 0
    for i in range(K):
        flush.sum()
        p = pos[0] % w.K
        nbytes_total += decode_hist_bytes(w.B, w.H, p, w.K) if hist else decode_bytes(w.B, w.H)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        one(i)
        e1.record(s)
        e1.synchronize()
        total += e0.elapsed_time(e1)
    ttt.ttt_device_status()
    ms = max_over_ranks(world, total / K)
    hbm = peaks[0]
    nbytes = nbytes_total / K
    name = "ttt_linear_decode_hist_cache_B128_H32_after_prefill2048" if hist else "ttt_linear_decode_B128_H32_after_prefill2048"
    return {"workload": name, "value": round(world * w.B / (ms / 1e3), 1),
            "unit": "tokens/s", "ms_per_step": round(ms, 5), "steps": K, "gpu_launches": K,
            "l2": "evicted by a 256 MB read before every timed step",
            "roofline": {"bound": "hbm", "achieved": round(nbytes / (ms / 1e3) / 1e9, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(nbytes / (ms / 1e3) / 1e9 / hbm, 4),
                         "algorithmic_bytes": int(nbytes)}}


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    """Cores this process may run on (its CPU affinity set)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_chains(w, ids):
    """Inputs of the listed chains of a workload as float64 arrays (so the oracle's wrapper makes
    no copies while it is timed), generated before any timing."""
    out = []
    for c in ids:
        xs = synth.linear_inputs(w, chains=[c])
        h = c % w.H
        out.append(tuple(np.ascontiguousarray(a, np.float64) for a in
                         (xs["XQ"][0], xs["XK"][0], xs["XV"][0], xs["lr"][0], xs["W0"][h], xs["b0"][h],
                          xs["ln_w"][h], xs["ln_b"][h])))
    return out


def _time_oracle(fn, samples, threads, seconds, K, eps):
    """Run fn(*sample, K, eps) over the samples round-robin on `threads` host threads (each call
    single-threaded; ctypes releases the GIL) until `seconds` have passed; returns (chains done,
    wall seconds)."""
    done = [0] * threads
    start = threading.Barrier(threads + 1)
    deadline = [0.0]

    def worker(i):
        start.wait()
        j = i
        while True:
            fn(*samples[j % len(samples)], K, eps)
            done[i] += 1
            j += threads
            if time.perf_counter() >= deadline[0]:
                return

    ts = [threading.Thread(target=worker, args=(i,)) for i in range(threads)]
    for t in ts:
        t.start()
    t0 = time.perf_counter()
    deadline[0] = t0 + seconds
    start.wait()
    for t in ts:
        t.join()
    return sum(done), time.perf_counter() - t0


def cpu_baseline(seconds_each=3.5):
    """The oracle as it stands, timed on the host on a bounded sample of the 1B workload
    (chains of L = 8200): the fp64 parity build and the float build of the same source, each on
    one core and with the chains spread over every core this process may use (one
    single-threaded oracle call per thread, no change to the oracle)."""
    import oracle
    w = synth.workload(2, L=8200)
    n = host_cores()
    samples = _oracle_chains(w, [(i * 37) % w.chains for i in range(8)])
    o64, o32 = oracle.default(), oracle.OracleF32()
    res = {}
    for name, fn in (("f64", o64.linear_chain), ("f32", o32.linear_chain)):
        for cores in sorted({1, n}):
            chains, wall = _time_oracle(fn, samples, cores, seconds_each, w.K, w.eps)
            res[f"{name}_{cores}core"] = {"value": round(chains * w.L / wall, 1), "chains": chains,
                                          "seconds": round(wall, 2)}
    top = res[f"f64_{n}core"]
    return {"value": top["value"], "unit": "tokens/s", "cores": n, "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"chains of the 1B workload (L={w.L} each) on {n} host threads for ~{seconds_each} s, "
                      f"fp64 oracle ({top['chains']} chains); also the float build and 1 core",
            "runs": res}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on the same workload and metric.  Each
    step runs one chain (L = 8200) per host core, one single-threaded oracle call per thread."""
    if rank != 0:
        return
    import oracle
    w = synth.workload(2, L=8200)
    n = host_cores()
    o = oracle.default()
    samples = _oracle_chains(w, [(i * 53) % w.chains for i in range(min(n, 16))])

    def step():
        ts = [threading.Thread(target=o.linear_chain, args=(*samples[i % len(samples)], w.K, w.eps))
              for i in range(n)]
        for t in ts:
            t.start()
        for t in ts:
            t.join()

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / args.steps
    value = n * w.L / dt
    print(json.dumps({
        "impl": "reference", "metric": "TTT layer tokens/sec (1B shapes, B200) and % of per-layer roofline",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(dt * 1e3, 2), "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded generator, synth/)",
        "config": {"workload": "ttt_linear_prefill_1b_layer", "B": w.B, "H": w.H, "L": w.L, "d": D,
                   "mini_batch": w.K, "sample_per_step": f"{n} chains, one per host core"},
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": n, "kind": "oracle",
                         "cpu_model": cpu_model(),
                         "sample": f"{n} chains of L={w.L} per step, one single-threaded fp64 oracle call per "
                                   f"host thread"},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--rows", default="linear,linear_tm,linear_rope,oproj,backward,mlp,decode,decode_hist",
                    help="comma list: linear (the headline) plus mlp and decode rows in the same line")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-chunk", type=int, default=1,
                    help="batch rows per chunk of the host-buffer (e2e) call")
    ap.add_argument("--seq-len", type=int, default=8200,
                    help="profiling aid: sequence length of the TTT-Linear workload (the headline is 8200)")
    ap.add_argument("--no-headline", action="store_true",
                    help="profiling aid: run only the --rows rows and print them (no headline line)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        run_reference(args, world, int(os.environ.get("RANK", "0")))
        return

    import torch
    world, rank, local = dist_setup(args.gpus)
    torch.cuda.set_device(local)
    peaks = measured_peaks()
    rows = [r.strip() for r in args.rows.split(",") if r.strip()]
    if args.no_headline:
        extra = {}
        if "linear_tm" in rows:
            extra["ttt_linear_prefill_token_major"] = bench_linear_token_major(args, world, peaks)
        if "linear_rope" in rows:
            extra["ttt_linear_prefill_rope"] = bench_linear_rope(args, world, peaks)
        if "oproj" in rows:
            extra["ttt_post_norm_o_proj"] = bench_post_norm_oproj(args, world, peaks)
        if "backward" in rows:
            extra["ttt_linear_backward"] = bench_linear_backward(args, world, peaks)
        if "mlp" in rows:
            extra["ttt_mlp_prefill"] = bench_mlp(args, world, peaks)
        if "decode" in rows:
            extra["ttt_linear_decode"] = bench_decode(args, world, peaks)
        if "decode_hist" in rows:
            extra["ttt_linear_decode_hist"] = bench_decode(args, world, peaks, hist=True)
        if rank == 0:
            print(json.dumps({"rows": extra}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    line = bench_linear(args, world, rank, local, peaks)
    extra = {}
    if "linear_tm" in rows:
        extra["ttt_linear_prefill_token_major"] = bench_linear_token_major(args, world, peaks)
    if "linear_rope" in rows:
        extra["ttt_linear_prefill_rope"] = bench_linear_rope(args, world, peaks)
    if "oproj" in rows:
        extra["ttt_post_norm_o_proj"] = bench_post_norm_oproj(args, world, peaks)
    if "backward" in rows:
        extra["ttt_linear_backward"] = bench_linear_backward(args, world, peaks)
    if "mlp" in rows:
        extra["ttt_mlp_prefill"] = bench_mlp(args, world, peaks)
    if "decode" in rows:
        extra["ttt_linear_decode"] = bench_decode(args, world, peaks)
    if "decode_hist" in rows:
        extra["ttt_linear_decode_hist"] = bench_decode(args, world, peaks, hist=True)
    if extra:
        line["rows"] = extra
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
