"""Reference oracle for the expert-parallel form of the DeepSeekMoE layer forward.

TEST INFRASTRUCTURE ONLY, like dsmoe_oracle.py (float64, CPU; used only by the
tests). It restates the layer for R ranks that each hold a shard of the tokens, a
replica of the router and of the shared experts, and N'/R of the routed experts
(the "DeepSeek-MoE interview card", section 4: shared experts replicated, routed
experts sharded across devices; the DeepSeekMoE summary's device-level balance
section groups experts by device the same way). Experts are assigned to ranks in
contiguous blocks: expert e lives on rank e // (N'/R).

One rank's forward, written as the steps a distributed implementation takes:
  1. route its own tokens (dsmoe_oracle.route on the local shard);
  2. order its (token, k) pairs by expert, ties by token then k: the
     expert-contiguous slot order, which is also destination-rank order;
  3. exchange the per-destination row counts, then the token rows and their
     expert ids (all-to-all);
  4. apply each received row's expert FFN (the owner holds those weights);
  5. send the outputs back along the reverse exchange;
  6. combine: h_t = u_t + sum_shared FFN(u_t) + sum_k g_{t,k} y_{t,k}.
The result equals the single-device layer on the concatenated batch, which is
what tests/test_oracle_ep.py checks on gloo ranks. ep_gather_forward_rank is the
second form (gather every token, apply the local experts, sum the partial outputs),
suited to decode batches.

`comm` supplies the exchange: alltoall(list of R numpy arrays) -> list of R arrays
(element j of the input goes to rank j; element j of the output came from rank j).
"""
from __future__ import annotations

from typing import Callable, Dict, List

import numpy as np

from oracle import dsmoe_oracle as O


def expert_owner(e, n_routed: int, world: int):
    """Rank that holds routed expert e (contiguous blocks of N'/R experts)."""
    return np.asarray(e) // (n_routed // world)


def ep_forward_rank(cfg, local_inputs: Dict, local_experts: Dict[int, tuple], shared: List[tuple],
                    world: int, alltoall: Callable[[List[np.ndarray]], List[np.ndarray]]) -> Dict:
    """The layer on this rank's tokens (local_inputs: x, W_router, b, token_ids as for
    dsmoe_oracle.route). local_experts maps each routed expert this rank owns to its
    (W_gate, W_up, W_down); shared lists the replicated shared experts.

    Returns h (float64, one row per local token) and the local routing."""
    assert cfg.n_routed % world == 0, "experts must split evenly across ranks"
    X = O._as_f64(local_inputs["x"])
    T, d = X.shape
    r = O.route(cfg, local_inputs)
    idx = np.asarray(r["idx"], dtype=np.int64)
    K = idx.shape[1]

    # 2. slot order: by expert, then token, then k
    pairs = sorted(((int(idx[t, k]), t, k) for t in range(T) for k in range(K)))
    dest = [int(expert_owner(e, cfg.n_routed, world)) for e, _, _ in pairs]

    # 3. rows and expert ids per destination, in slot order
    send_rows = [np.zeros((0, d)) for _ in range(world)]
    send_eids = [np.zeros((0,), dtype=np.int64) for _ in range(world)]
    for j in range(world):
        sel = [i for i, dj in enumerate(dest) if dj == j]
        send_rows[j] = X[[pairs[i][1] for i in sel]] if sel else np.zeros((0, d))
        send_eids[j] = np.asarray([pairs[i][0] for i in sel], dtype=np.int64)
    recv_rows = alltoall(send_rows)
    recv_eids = alltoall([e.astype(np.float64) for e in send_eids])

    # 4. the owner applies its experts, row by row grouped by expert
    outs = []
    for rows, eids in zip(recv_rows, recv_eids):
        eids = eids.astype(np.int64)
        y = np.zeros_like(rows)
        for e in np.unique(eids):
            m = eids == e
            Wg, Wu, Wd = local_experts[int(e)]
            y[m] = O.swiglu_ffn(rows[m], Wg, Wu, Wd)
        outs.append(y)

    # 5. back to the sources, in the order they were sent
    back = alltoall(outs)

    # 6. combine
    h = X.copy()
    for (Wg, Wu, Wd) in shared:
        h += O.swiglu_ffn(X, Wg, Wu, Wd)
    g = np.asarray(r["gates"], dtype=np.float64)
    cursor = [0] * world
    for (e, t, k), j in zip(pairs, dest):
        h[t] += g[t, k] * back[j][cursor[j]]
        cursor[j] += 1
    return dict(h=h, idx=idx, gates=g, counts=r["counts"], scores=r["scores"])


def device_loads(counts, n_routed: int, world: int) -> np.ndarray:
    """Rows each rank's experts receive: the per-device sums of the expert counts (the
    quantity the DeepSeekMoE summary's device-level balance loss evens out)."""
    c = np.asarray(counts, dtype=np.int64)
    return c.reshape(world, n_routed // world).sum(axis=1)


def ep_gather_forward_rank(cfg, local_inputs: Dict, local_experts: Dict[int, tuple], shared: List[tuple],
                           world: int, rank: int, allgather_rows: Callable[[np.ndarray], List[np.ndarray]],
                           allreduce_sum: Callable[[np.ndarray], np.ndarray]) -> Dict:
    """The decode-shaped expert-parallel form: every rank gathers all ranks' tokens, routes
    them (router replicated, so every rank makes the same choice), applies only the
    routed experts it owns to the rows that chose them, and the partial outputs are summed
    across ranks; each rank keeps its own tokens' rows and adds the residual and the
    (replicated) shared experts. Few tokens, many experts: each weight is read on one rank
    only, instead of once per token shard.

    allgather_rows(a) returns every rank's array (rank order); allreduce_sum(a) sums an
    array over ranks. local_inputs as for ep_forward_rank (token_ids included for hash
    routing)."""
    assert cfg.n_routed % world == 0, "experts must split evenly across ranks"
    X_local = O._as_f64(local_inputs["x"])
    parts = allgather_rows(X_local)
    X = np.concatenate(parts, axis=0)
    start = sum(p.shape[0] for p in parts[:rank])
    full = dict(local_inputs)
    full["x"] = X
    if local_inputs.get("token_ids") is not None:
        ids = allgather_rows(np.asarray(local_inputs["token_ids"], dtype=np.float64).reshape(-1, 1))
        full["token_ids"] = np.concatenate(ids, axis=0).reshape(-1).astype(np.int64)
    r = O.route(cfg, full)
    idx = np.asarray(r["idx"], dtype=np.int64)
    g = np.asarray(r["gates"], dtype=np.float64)
    owned = [e for e in range(cfg.n_routed) if int(expert_owner(e, cfg.n_routed, world)) == rank]
    partial = gather_partial(X, idx, g, local_experts, owned)
    total = allreduce_sum(partial)
    n = X_local.shape[0]
    h = X_local + total[start:start + n]
    for (Wg, Wu, Wd) in shared:
        h += O.swiglu_ffn(X_local, Wg, Wu, Wd)
    return dict(h=h, idx=idx[start:start + n], gates=g[start:start + n])


def gather_partial(X, idx, gates, local_experts: Dict[int, tuple], owned, shared: List[tuple] = None,
                   rows=None) -> np.ndarray:
    """One rank's share of the decode-shaped expert-parallel form, before the sum over
    ranks: for every gathered token t (or the given rows), sum over its picks k whose
    expert the rank owns of g_{t,k} FFN_e(u_t); with `shared` given (the one rank that
    adds them), plus u_t and the shared experts' outputs. The sum of all ranks' partials
    is the layer output (the shared-expert layer equation split by expert owner)."""
    X = O._as_f64(X)
    idx = np.asarray(idx, dtype=np.int64)
    gates = np.asarray(gates, dtype=np.float64)
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(rows, dtype=np.int64)
    Xr, ir, gr = X[rows], idx[rows], gates[rows]
    partial = np.zeros_like(Xr)
    owned = set(int(e) for e in owned)
    for e in np.unique(ir):
        if int(e) not in owned:
            continue
        rr, ks = np.nonzero(ir == e)
        Wg, Wu, Wd = local_experts[int(e)]
        partial[rr] += gr[rr, ks][:, None] * O.swiglu_ffn(Xr[rr], Wg, Wu, Wd)
    if shared is not None:
        partial += Xr
        for (Wg, Wu, Wd) in shared:
            partial += O.swiglu_ffn(Xr, Wg, Wu, Wd)
    return partial
