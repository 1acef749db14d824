"""The token-sharded multi-process path on CPU (gloo, world size 2): shards cover every
token once, and the all-reduced shard sums give the balance statistics of the whole
batch. Each rank's per-shard sums come from the oracle (the CUDA kernel that turns
sums into f and P is checked on the GPU by test_parity_gpu)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from mixture_experts_layer_score_b200.sharded import shard_rows, reduce_balance_sums


def test_shard_rows_partition():
    for T in (0, 1, 7, 16, 4096, 8193):
        for world in (1, 2, 3, 8):
            spans = [shard_rows(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import workloads as W
        from oracle import dsmoe_oracle as O
        cfg = W.get_config("tiny").replace(T=301)
        inp = W.make_inputs(cfg, seed=5, with_weights=False)
        a, b = shard_rows(cfg.T, rank, world)
        shard = dict(inp)
        shard["x"] = inp["x"][a:b]
        r = O.route(cfg, shard)
        counts = torch.as_tensor(r["counts"], dtype=torch.int32)
        P_sum = torch.as_tensor(r["scores"].sum(axis=0), dtype=torch.float32)
        reduce_balance_sums(counts, P_sum)
        result_q.put((rank, counts.numpy(), P_sum.numpy()))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_reduce_to_whole_batch_stats():
    import workloads as W
    from oracle import dsmoe_oracle as O
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = W.get_config("tiny").replace(T=301)
    full = O.route(cfg, W.make_inputs(cfg, seed=5, with_weights=False))
    for rank, counts, P_sum in res:
        assert (counts == full["counts"]).all()
        np.testing.assert_allclose(P_sum / cfg.T, full["P"], rtol=1e-5, atol=1e-7)
        f = cfg.n_routed / (cfg.top_k * cfg.T) * counts
        np.testing.assert_allclose(f, full["f"], rtol=1e-12)
