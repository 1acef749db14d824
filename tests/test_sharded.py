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


class _OracleShardLayer:
    """Stands in for binding.DSMoE on CPU ranks: forward() returns what the library's
    expert-range forward returns (fp32 partial sums of this rank's experts, plus the
    residual and shared experts on the rank that adds them), computed by the oracle."""

    def __init__(self, cfg, inp):
        from mixture_experts_layer_score_b200.binding import DSMOE_RANGE_ADD_SHARED
        self.cfg, self.inp = cfg, inp
        self.range = (0, cfg.n_routed, DSMOE_RANGE_ADD_SHARED)
        self.handle = None

    def set_expert_range(self, e_begin, e_end, partial=True, add_shared=False):
        self.range = (e_begin, e_end, bool(add_shared))

    def forward(self, x_all, token_ids=None, stream=None):
        from oracle import dsmoe_oracle as O
        from oracle import dsmoe_ep as EP
        cfg, inp = self.cfg, self.inp
        full = dict(inp, x=x_all, token_ids=token_ids)
        r = O.route(cfg, full)
        e0, e1, add_shared = self.range
        local = {e: (inp["W_gate"][e], inp["W_up"][e], inp["W_down"][e]) for e in range(e0, e1)}
        shared = [(inp["Ws_gate"][i], inp["Ws_up"][i], inp["Ws_down"][i]) for i in range(cfg.n_shared)]
        part = EP.gather_partial(x_all, r["idx"], r["gates"], local, range(e0, e1), shared if add_shared else None)
        return dict(h=torch.as_tensor(part, dtype=torch.float32), topk_idx=torch.as_tensor(r["idx"]),
                    gates=torch.as_tensor(r["gates"]), counts=torch.as_tensor(r["counts"]),
                    f=torch.as_tensor(r["f"]), P=torch.as_tensor(r["P"]))


def _decode_worker(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import workloads as W
        from mixture_experts_layer_score_b200.sharded import configure_expert_shard, expert_sharded_forward
        cfg = W.get_config("tiny").replace(T=12 * world, d_model=128, d_ff=64, d_ff_shared=64, n_routed=30)
        inp = W.make_inputs(cfg, seed=7)
        layer = _OracleShardLayer(cfg, inp)
        e0, e1 = configure_expert_shard(layer, rank, world)
        T = cfg.T // world
        x_local = inp["x"][rank * T:(rank + 1) * T]
        out = expert_sharded_forward(layer, x_local, round_bf16=lambda src, dst: dst.copy_(src.to(torch.bfloat16)))
        result_q.put((rank, e0, e1, out["h"].float().numpy(), out["topk_idx"].numpy(), out["counts"].numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_expert_sharded_decode_equals_the_layer(world):
    """The decode form's orchestration (all-gather of x, a contiguous expert block per rank,
    rank 0 adding the residual and the shared experts, reduce-scatter of the fp32
    partials, one rounding to bf16) on gloo ranks: every rank's rows equal the
    single-device layer's rows rounded once to bf16, the expert blocks tile [0, N'),
    and the routing slices and whole-batch counts agree."""
    import workloads as W
    from oracle import dsmoe_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = W.get_config("tiny").replace(T=12 * world, d_model=128, d_ff=64, d_ff_shared=64, n_routed=30)
    ref = O.forward(cfg, W.make_inputs(cfg, seed=7))
    h_ref = torch.as_tensor(ref["h"], dtype=torch.float32).to(torch.bfloat16).float().numpy()
    T = cfg.T // world
    assert res[0][1] == 0 and res[-1][2] == cfg.n_routed
    assert all(res[i][2] == res[i + 1][1] for i in range(world - 1))
    for rank, e0, e1, h, idx, counts in res:
        rows = slice(rank * T, (rank + 1) * T)
        # the fp32 sum over ranks differs from the float64 layer by rounding only; after
        # the one bf16 rounding at most one bf16 step apart
        np.testing.assert_allclose(h, h_ref[rows], rtol=2 ** -7, atol=1e-6)
        assert (idx == ref["idx"][rows]).all()
        assert (counts == ref["counts"]).all()


class _OracleEpLib:
    """Stands in for the library's three expert-parallel calls on CPU ranks, computed by the
    oracle, with the same data contract: dsmoe_ep_route leaves the token rows in expert
    order (workspace "Xp") and returns rows per destination; dsmoe_ep_experts maps the
    received rows (grouped by source, then expert) to expert outputs row for row;
    dsmoe_ep_combine adds the returned rows to the residual and the shared experts."""

    def __init__(self, cfg, inp):
        self.cfg, self.inp, self.state = cfg, inp, {}

    def dsmoe_ep_route(self, handle, T, x, ids, W_router, b, topk, gates, counts, f, P, P_sum, scores, world,
                       send_rows, stream=None):
        from oracle import dsmoe_oracle as O
        r = O.route(self.cfg, dict(self.inp, x=x, token_ids=ids))
        topk.copy_(torch.as_tensor(r["idx"]))
        gates.copy_(torch.as_tensor(r["gates"]))
        counts.copy_(torch.as_tensor(r["counts"]))
        f.copy_(torch.as_tensor(r["f"]))
        P.copy_(torch.as_tensor(r["P"]))
        K = r["idx"].shape[1]
        pairs = sorted((int(r["idx"][t, k]), t, k) for t in range(T) for k in range(K))
        slot_of = np.zeros((T, K), dtype=np.int64)
        for i, (_, t, k) in enumerate(pairs):
            slot_of[t, k] = i
        self.state = dict(Xp=x[[t for _, t, _ in pairs]].clone(), slot_of=slot_of)
        from mixture_experts_layer_score_b200.sharded import expert_block
        N = self.cfg.n_routed
        for j in range(world):
            a, b_ = expert_block(N, j, world)
            send_rows[j] = sum(1 for e, _, _ in pairs if a <= e < b_)

    def workspace_view(self, handle, name, device=0):
        return self.state[name]

    def dsmoe_ep_experts(self, handle, n_src, e0, e1, recv_counts, n_rows, rows, Wg, Wu, Wd, Y, stream=None):
        from oracle import dsmoe_oracle as O
        n_local = e1 - e0
        cnt = recv_counts.view(n_src, n_local).numpy()
        r0 = 0
        for j in range(n_src):
            for el in range(n_local):
                n = int(cnt[j, el])
                if n:
                    y = O.swiglu_ffn(rows[r0:r0 + n], Wg[el], Wu[el], Wd[el])
                    Y[r0:r0 + n] = torch.as_tensor(y, dtype=torch.float32).to(torch.bfloat16)
                r0 += n
        assert r0 == n_rows

    def dsmoe_ep_combine(self, handle, T, x, Wsg, Wsu, Wsd, gates, Y, h, stream=None):
        from oracle import dsmoe_oracle as O
        X = O._as_f64(x)
        acc = X.copy()
        for i in range(self.cfg.n_shared):
            acc += O.swiglu_ffn(X, Wsg[i], Wsu[i], Wsd[i])
        Yf = Y.float().numpy().astype(np.float64)
        g = gates.numpy().astype(np.float64)
        so = self.state["slot_of"]
        for k in range(so.shape[1]):
            acc += g[:, k:k + 1] * Yf[so[:, k]]
        h.copy_(torch.as_tensor(acc, dtype=torch.float32).to(torch.bfloat16))


class _CpuLayer:
    def __init__(self, cfg, w):
        self.cfg, self.w, self.handle, self.device, self.k_active = cfg, w, None, "cpu", cfg.top_k

    def alloc_outputs(self, T):
        c = self.cfg
        return dict(h=None, topk_idx=torch.empty((T, c.top_k), dtype=torch.int64),
                    gates=torch.empty((T, c.top_k)), counts=torch.empty((c.n_routed,), dtype=torch.int32),
                    f=torch.empty((c.n_routed,)), P=torch.empty((c.n_routed,)), P_sum=None)


def _dispatch_worker(rank, world, port, result_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import workloads as W
        from mixture_experts_layer_score_b200.sharded import expert_block, token_dispatch_forward
        cfg = W.get_config("tiny").replace(T=10 * world + 3, d_model=128, d_ff=64, d_ff_shared=64, n_routed=30)
        inp = W.make_inputs(cfg, seed=9)
        a, b = shard_rows(cfg.T, rank, world)
        e0, e1 = expert_block(cfg.n_routed, rank, world)
        w = dict(inp)
        for k in ("W_gate", "W_up", "W_down"):
            w[k] = inp[k][e0:e1]
        layer = _CpuLayer(cfg, w)
        lib = _OracleEpLib(cfg, inp)
        ids = None if inp["token_ids"] is None else inp["token_ids"][a:b]
        out = token_dispatch_forward(layer, inp["x"][a:b], ids, lib=lib)
        result_q.put((rank, a, b, out["h"].float().numpy(), out["topk_idx"].numpy(), out["counts"].numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_token_dispatch_equals_the_layer(world):
    """The token-dispatch form's orchestration on gloo ranks with uneven token shards and
    uneven expert blocks: counts to the owners, rows out and back by all-to-all with
    split sizes from the routing, owners' experts grouped by (source, expert). Every rank's
    h equals the single-device layer's rows within the layer bound (the exchanged expert
    outputs are bf16, as on the GPU), and its routing equals the oracle's for its shard."""
    import workloads as W
    from oracle import dsmoe_oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dispatch_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = W.get_config("tiny").replace(T=10 * world + 3, d_model=128, d_ff=64, d_ff_shared=64, n_routed=30)
    inp = W.make_inputs(cfg, seed=9)
    ref = O.forward(cfg, inp)
    rms = np.sqrt(np.mean(ref["h"] ** 2))
    total = np.zeros(cfg.n_routed, dtype=np.int64)
    for rank, a, b, h, idx, counts in res:
        assert np.abs(h - ref["h"][a:b]).max() / rms <= 2e-2
        assert (idx == ref["idx"][a:b]).all()
        total += counts
    assert (total == ref["counts"]).all()
