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


def _bwd_worker(rank, world, port, q):
    """One rank of data-parallel training: the backward oracle on this rank's batch shard, the
    shard's per-head sums of the shared-parameter gradients, then their all-reduce."""
    import torch
    import torch.distributed as dist

    import synth
    from oracle import ttt_backward
    from test_rnn_layers_b200.shard import allreduce_shared_grads, batch_shard
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = synth.workload(1, B=3, H=2, L=19, K=4, dtype="f32", seed=0xD158)
        s, e = batch_shard(w.B, world, rank)
        chains = [b * w.H + h for b in range(s, e) for h in range(w.H)]
        x, up = synth.linear_inputs(w, chains=chains), synth.upstream_grads(w, chains=chains)
        st = lambda a: np.stack([a[c % w.H] for c in chains])
        r = ttt_backward.linear_backward(x["XQ"], x["XK"], x["XV"], x["lr"], st(x["W0"]), st(x["b0"]), st(x["ln_w"]),
                                         st(x["ln_b"]), w.K, w.eps, up["d_out"], up["dW_last"], up["db_last"])
        grads = {}
        for n in ("dW0", "db0", "dln_w", "dln_b"):
            acc = torch.zeros((w.H,) + r[n].shape[1:], dtype=torch.float64)
            for i, c in enumerate(chains):
                acc[c % w.H] += torch.from_numpy(r[n][i])
            grads[n] = acc
        allreduce_shared_grads(grads)
        q.put((rank, chains, r["dXQ"], r["dlr"], {n: grads[n].numpy() for n in grads}))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_data_parallel_backward():
    """Sharded backward + the all-reduce of the shared-parameter gradients = the whole batch's."""
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_bwd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=180) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda t: t[0])
    import synth
    from oracle import ttt_backward
    w = synth.workload(1, B=3, H=2, L=19, K=4, dtype="f32", seed=0xD158)
    ids = list(range(w.chains))
    x, up = synth.linear_inputs(w, chains=ids), synth.upstream_grads(w, chains=ids)
    st = lambda a: np.stack([a[c % w.H] for c in ids])
    whole = ttt_backward.linear_backward(x["XQ"], x["XK"], x["XV"], x["lr"], st(x["W0"]), st(x["b0"]), st(x["ln_w"]),
                                         st(x["ln_b"]), w.K, w.eps, up["d_out"], up["dW_last"], up["db_last"])
    assert sum((c for _, c, _, _, _ in res), []) == ids
    assert np.array_equal(np.concatenate([d for _, _, d, _, _ in res]), whole["dXQ"])
    assert np.array_equal(np.concatenate([d for _, _, _, d, _ in res]), whole["dlr"])
    for n in ("dW0", "db0", "dln_w", "dln_b"):
        ref = whole[n].reshape(w.B, w.H, *whole[n].shape[1:]).sum(axis=0)
        for _, _, _, _, g in res:  # every rank holds the same, whole-batch sums
            np.testing.assert_allclose(g[n], ref, rtol=1e-12, atol=1e-12)
