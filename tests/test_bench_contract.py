"""The benchmark's accounting and its reference arm, on the CPU.

* The roofline numerators (algorithmic bytes / FLOPs per launch) equal the per-unit figures times
  the units: 516 B per (chain, token) for the TTT-Linear scan (XQ, XK, XV bf16 in, lr fp32 in,
  out bf16 back) plus the state written per chain and the parameters read per head; 27 840 FLOP
  per (chain, token) at K = 16 (three dense 16x64x64 products and three triangular 16x16x64 ones
  per mini-batch of 16 tokens).
* `bench.py --impl reference` (the oracle on the host cores; no GPU) prints one JSON line with the
  contract's keys.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_linear_bytes_per_unit():
    B, H, L, d = 8, 32, 8200, 64
    per_token_chain = 3 * d * 2 + 4 + d * 2
    assert per_token_chain == 516
    state = (d * d + d) * 4                      # 16 640 B: W and b in fp32
    written_per_chain = 2 * state                # W_last, b_last and the tail grads
    read_per_head = state + 2 * d * 4            # W0, b0 and ln_w, ln_b
    expect = B * H * L * per_token_chain + B * H * written_per_chain + H * read_per_head
    assert bench.linear_bytes(B, H, L) == expect == 1_092_255_744


def test_linear_flops_per_unit():
    B, H, L = 8, 32, 8192
    per_token_chain = (3 * 2 * 16 * 64 * 64 + 3 * 2 * 64 * (16 * 17 // 2)) // 16
    assert per_token_chain == 27_840
    assert bench.linear_flops(B, H, L) == B * H * L * per_token_chain
    # a tail mini-batch is counted as a whole one (its products run at full tile size)
    assert bench.linear_flops(1, 1, 17) == bench.linear_flops(1, 1, 32)


def test_decode_hist_bytes_grow_with_the_rows():
    b0, b5 = bench.decode_hist_bytes(1, 1, 0), bench.decode_hist_bytes(1, 1, 5)
    assert b5 - b0 == 5 * 2 * 64 * 4             # five rows of (lr xk, g) read
    commit = bench.decode_hist_bytes(1, 1, 15)
    assert commit > bench.decode_hist_bytes(1, 1, 14)  # W and b written back on the commit step


@pytest.mark.timeout(600)
def test_reference_arm_prints_the_contract_line():
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, cwd=ROOT, timeout=600)
    assert res.returncode == 0, res.stderr
    lines = [ln for ln in res.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3 and d["value"] > 0
    assert d["config"]["workload"] == "ttt_linear_prefill_1b_layer"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["cpu_baseline"]["cpu_model"] and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["e2e"]["value"] == d["value"]


def test_cpu_baseline_reports_both_precisions_and_the_cores():
    """The bench's CPU baseline: the fp64 oracle and its float build, on 1 core and on every core
    of the affinity set, with the CPU model (a short run)."""
    cb = bench.cpu_baseline(seconds_each=0.3)
    n = bench.host_cores()
    assert cb["cores"] == n and cb["kind"] == "oracle" and cb["cpu_model"]
    assert set(cb["runs"]) == {f"{p}_{c}core" for p in ("f64", "f32") for c in {1, n}}
    assert cb["value"] == cb["runs"][f"f64_{n}core"]["value"] > 0


def test_backward_work_counts():
    import bench
    per_mb = 6 * 2 * 16 * 64 * 64 + 4 * 2 * 64 * 16 * 17 // 2
    assert per_mb == 856064
    assert bench.linear_bwd_flops(1, 1, 16 * 3 + 1) == 4 * per_mb     # the tail counts as a mini-batch
    per_token = 4 * 128 + 4 + 3 * 128 + 4                             # 4 bf16 rows + lr in, 3 rows + d lr out
    state = (64 * 64 + 64) * 4
    assert bench.linear_bwd_bytes(2, 3, 10) == 6 * 10 * per_token + 2 * 3 * state + 6 * state + 2 * 3 * 2 * 64 * 4
