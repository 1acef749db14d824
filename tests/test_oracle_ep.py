"""The expert-parallel oracle (oracle/dsmoe_ep.py) on gloo ranks on the CPU: with the
routed experts split across 2 or 4 ranks and the tokens split unevenly, every rank's
layer output equals the single-device oracle's rows for its tokens in both forms (the
all-to-all dispatch and the gather / all-reduce form), and the per-device loads add up to
the whole batch's slots."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _alltoall(parts):
    """Exchange a list of float64 arrays [n_j, ...] (same trailing shape) over gloo."""
    world = dist.get_world_size()
    counts = torch.tensor([p.shape[0] for p in parts], dtype=torch.int64)
    recv_counts = torch.empty_like(counts)
    dist.all_to_all_single(recv_counts, counts)
    tail = parts[0].shape[1:]
    width = int(np.prod(tail)) if tail else 1
    send = torch.from_numpy(np.concatenate([p.reshape(p.shape[0], width) for p in parts])).double()
    recv = torch.empty((int(recv_counts.sum()), width), dtype=torch.float64)
    dist.all_to_all_single(recv, send, recv_counts.tolist(), counts.tolist())
    out, o = [], 0
    for j in range(world):
        n = int(recv_counts[j])
        out.append(recv[o:o + n].numpy().reshape((n,) + tail))
        o += n
    return out


def _allgather_rows(a):
    """Every rank's float64 array [n_r, ...] (uneven n_r), in rank order, over gloo."""
    world = dist.get_world_size()
    n = torch.tensor([a.shape[0]], dtype=torch.int64)
    ns = [torch.empty_like(n) for _ in range(world)]
    dist.all_gather(ns, n)
    m = int(max(int(v) for v in ns))
    buf = torch.zeros((m,) + a.shape[1:], dtype=torch.float64)
    buf[:a.shape[0]] = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    outs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(outs, buf)
    return [o[:int(k)].numpy() for o, k in zip(outs, ns)]


def _allreduce_sum(a):
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    dist.all_reduce(t)
    return t.numpy()


def _cfg(name):
    import workloads as W
    cfg = W.get_config(name).replace(T=157)
    if cfg.d_model > 1024:  # keep the CPU test small: the same routing rules, a narrower layer
        cfg = cfg.replace(d_model=256, d_ff=128, d_ff_shared=128, n_routed=64)
    return cfg


def _worker(rank, world, port, name, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        import workloads as W
        from oracle import dsmoe_ep as EP
        cfg = _cfg(name)
        inp = W.make_inputs(cfg, seed=2)
        # uneven token shards: rank r takes a share proportional to r + 1
        w = np.arange(1, world + 1)
        bounds = np.concatenate([[0], np.cumsum(w * cfg.T // w.sum())])
        bounds[-1] = cfg.T
        a, b = int(bounds[rank]), int(bounds[rank + 1])
        local = {k: v for k, v in inp.items() if k in ("x", "W_router", "b", "token_ids")}
        local["x"] = inp["x"][a:b]
        if local.get("token_ids") is not None:
            local["token_ids"] = inp["token_ids"][a:b]
        per = cfg.n_routed // world
        mine = {e: (inp["W_gate"][e], inp["W_up"][e], inp["W_down"][e]) for e in range(rank * per, (rank + 1) * per)}
        shared = [(inp["Ws_gate"][i], inp["Ws_up"][i], inp["Ws_down"][i]) for i in range(cfg.n_shared)]
        out = EP.ep_forward_rank(cfg, local, mine, shared, world, _alltoall)
        loads = torch.as_tensor(EP.device_loads(out["counts"], cfg.n_routed, world))
        dist.all_reduce(loads)
        gath = EP.ep_gather_forward_rank(cfg, local, mine, shared, world, rank, _allgather_rows, _allreduce_sum)
        result_q.put((rank, a, b, out["h"], loads.numpy(), gath["h"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name,world", [("tiny", 2), ("tiny", 4), ("v4_hash_t16", 2)])
def test_expert_parallel_oracle_equals_single_device(name, world):
    import workloads as W
    from oracle import dsmoe_oracle as O
    cfg = _cfg(name)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, name, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    inp = W.make_inputs(cfg, seed=2)
    ref = O.forward(cfg, inp)
    for rank, a, b, h, loads, h_gather in res:
        np.testing.assert_allclose(h, ref["h"][a:b], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(h_gather, ref["h"][a:b], rtol=1e-12, atol=1e-12)
        assert loads.sum() == cfg.T * cfg.top_k


@pytest.mark.parametrize("world", [1, 2, 3])
def test_gather_partials_sum_to_the_layer(world):
    """The decode form's per-rank partial sums (uneven contiguous expert blocks, one rank
    adding the residual and the shared experts) add up to the single-device layer."""
    import workloads as W
    from oracle import dsmoe_oracle as O
    from oracle import dsmoe_ep as EP
    cfg = _cfg("tiny")
    inp = W.make_inputs(cfg, seed=2)
    ref = O.forward(cfg, inp)
    N = cfg.n_routed
    shared = [(inp["Ws_gate"][i], inp["Ws_up"][i], inp["Ws_down"][i]) for i in range(cfg.n_shared)]
    total = 0.0
    for rank in range(world):
        e0 = (N // world) * rank + min(rank, N % world)
        e1 = e0 + N // world + (1 if rank < N % world else 0)
        local = {e: (inp["W_gate"][e], inp["W_up"][e], inp["W_down"][e]) for e in range(e0, e1)}
        part = EP.gather_partial(inp["x"], ref["idx"], ref["gates"], local, range(e0, e1),
                                 shared if rank == 0 else None)
        rows = np.array([3, 0, 150])
        sub = EP.gather_partial(inp["x"], ref["idx"], ref["gates"], local, range(e0, e1),
                                shared if rank == 0 else None, rows=rows)
        np.testing.assert_allclose(sub, part[rows], rtol=1e-12, atol=1e-12)
        total = total + part
    np.testing.assert_allclose(total, ref["h"], rtol=1e-12, atol=1e-12)
