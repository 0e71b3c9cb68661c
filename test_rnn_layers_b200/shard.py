"""Host-side multi-GPU plumbing of the scan: chain sharding and device-time reduction.

Every (batch, head) chain of the TTT scan is independent (each carries its own W, b through the
whole sequence), so the path shards across GPUs with no exchange at any mini-batch: rank r takes
a contiguous slice of the batch dimension (whole heads stay together, so each rank needs every
head's W0, ln_w, ln_b) and runs the same kernel on it.  No collective touches the forward's data
path; its only collectives are the timing barrier and the max over ranks of the device time.

The backward has one real exchange: the gradients of the parameters every chain of a head shares
(W0 and b0 when they are one per head, ln_w and ln_b) are sums over the whole batch, so each
rank's sums over its own shard are summed across ranks (`allreduce_shared_grads`, one all-reduce
over the few hundred KB of them, NCCL on GPUs).  The gradients of the activations and of lr
stay with the rank that owns those rows.
"""
from __future__ import annotations


def batch_shard(B: int, world: int, rank: int):
    """[start, stop) of the batch rows owned by `rank`: as even as possible, earlier ranks take
    the extra row.  Shards cover range(B) exactly once; a rank may own nothing when B < world."""
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError(f"bad shard request B={B} world={world} rank={rank}")
    base, extra = divmod(B, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def max_over_ranks(value: float, group=None, device=None) -> float:
    """The maximum of a per-rank scalar (a device time) over the process group."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    if device is None:
        device = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


SHARED_GRADS = ("dW0", "db0", "dln_w", "dln_b")


def allreduce_shared_grads(grads: dict, per_chain_state: bool = False, group=None) -> dict:
    """Sum, over the ranks of the process group, the shared-parameter gradients of a backward
    result (the dict ttt_linear_backward returns): dln_w and dln_b always, dW0 and db0 unless the
    initial state is per chain (then each chain's own gradient stays with its rank).  In place,
    one flat all-reduce; returns `grads`."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return grads
    names = [n for n in SHARED_GRADS if not (per_chain_state and n in ("dW0", "db0"))]
    flat = torch.cat([grads[n].reshape(-1) for n in names])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for n in names:
        k = grads[n].numel()
        grads[n].copy_(flat[off:off + k].view_as(grads[n]))
        off += k
    return grads


def aggregate_tokens_per_s(tokens_per_rank: int, world: int, ms_per_step_max: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's step time."""
    return world * tokens_per_rank / (ms_per_step_max / 1e3)
