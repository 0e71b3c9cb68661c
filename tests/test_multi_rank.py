"""The N>1 host path on CPU with the gloo backend (world size 2): sharding covers every chain
exactly once, the device-time reduction takes the slowest rank, and sharded oracle runs equal
the unsharded one (the chains are independent, so no exchange is needed)."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from test_rnn_layers_b200.shard import aggregate_tokens_per_s, batch_shard


@pytest.mark.parametrize("B,world", [(8, 1), (8, 2), (8, 3), (1, 2), (5, 4), (128, 8)])
def test_batch_shards_cover_each_row_once(B, world):
    rows = []
    for r in range(world):
        s, e = batch_shard(B, world, r)
        assert 0 <= s <= e <= B
        rows += list(range(s, e))
    assert rows == list(range(B))


def test_bad_shard_request():
    with pytest.raises(ValueError):
        batch_shard(4, 2, 2)


def test_aggregate():
    assert aggregate_tokens_per_s(1000, 4, 2.0) == 4 * 1000 / 0.002


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    import oracle
    import synth
    from test_rnn_layers_b200.shard import batch_shard, max_over_ranks
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # timing reduction: each rank reports a different "device time"
        t = max_over_ranks(1.5 + rank)
        # each rank runs the oracle on its batch shard of a small problem
        w = synth.workload(1, B=3, H=2, L=21, seed=0xD157)
        x = synth.linear_inputs(w)
        s, e = batch_shard(w.B, world, rank)
        chains = [b * w.H + h for b in range(s, e) for h in range(w.H)]
        xs = synth.linear_inputs(w, chains=chains)
        r = oracle.default().linear_forward(xs["XQ"], xs["XK"], xs["XV"], xs["lr"], x["W0"], x["b0"], x["ln_w"],
                                            x["ln_b"], w.K, w.eps, chains=chains)
        q.put((rank, t, chains, r["out"], r["W_last"]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reduce():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert all(t == 2.5 for _, t, _, _, _ in res)  # the max over ranks
    res.sort()
    chains = sum((c for _, _, c, _, _ in res), [])
    assert chains == list(range(6))
    import oracle
    import synth
    w = synth.workload(1, B=3, H=2, L=21, seed=0xD157)
    x = synth.linear_inputs(w)
    whole = oracle.default().linear_forward(x["XQ"], x["XK"], x["XV"], x["lr"], x["W0"], x["b0"], x["ln_w"],
                                            x["ln_b"], w.K, w.eps)
    assert np.array_equal(np.concatenate([o for _, _, _, o, _ in res]), whole["out"])
    assert np.array_equal(np.concatenate([W for _, _, _, _, W in res]), whole["W_last"])
