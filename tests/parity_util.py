"""Helpers of the GPU parity tests: move synthetic inputs to the device, compare with the oracle."""
from __future__ import annotations

import numpy as np
import torch

import synth


def rel_l2(gpu, ref, floor=1e-6):
    """max over leading (chain) index of ||gpu - ref||_2 / max(||ref||_2, floor * sqrt(n))."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    g = gpu.reshape(gpu.shape[0], -1)
    r = ref.reshape(ref.shape[0], -1)
    n = r.shape[1]
    num = np.linalg.norm(g - r, axis=1)
    den = np.maximum(np.linalg.norm(r, axis=1), floor * np.sqrt(n))
    return float((num / den).max()) if len(num) else 0.0


def dev_act(x: dict, name: str, device="cuda"):
    """Activation tensor on the device in the workload's dtype (bf16 from the exact bits)."""
    if name + "_bits" in x:
        bits = np.ascontiguousarray(x[name + "_bits"]).view(np.int16)
        return torch.from_numpy(bits).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(x[name], np.float32)).to(device)


def dev_f32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(device)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def chain_slice(t: torch.Tensor, chains, H):
    """Rows of the given flat chain ids from a [B,H,...] device tensor, as float64 numpy."""
    flat = t.reshape(-1, *t.shape[2:])
    return to_np(flat[list(chains)])


def sample_chains(n_chains: int, k: int = 4):
    """A spread of chain ids: first, last and evenly spaced ones in between."""
    if n_chains <= k:
        return list(range(n_chains))
    return sorted(set(int(round(i)) for i in np.linspace(0, n_chains - 1, k)))
