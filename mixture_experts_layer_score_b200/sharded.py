"""Multi-GPU forms of the layer forward, one process per GPU.

Token sharding (prefill): tokens are independent through the whole layer, so each
rank runs the forward on its own contiguous shard of the batch with a full copy of
the weights and no data-path exchange. The one step that spans ranks is the
expert-level balance statistics f_i and P_i (DeepSeekMoE summary, "Expert-level
balance loss"), which are defined over every token of the batch: each rank's token
counts and score sums are summed across ranks (one all-reduce of 2 N' words) and the
library turns the sums into f and P (dsmoe_balance_stats).

Expert sharding (decode): with few tokens and hundreds of experts, token shards would
each stream almost every expert's weights. Instead each rank holds a contiguous block
of the routed experts and all ranks replicate the router and the shared experts (the
DeepSeek-MoE interview card's deployment trade-off: shared experts on every GPU,
routed experts sharded). Every rank gathers all ranks' tokens (all-gather of x),
routes them all (the router is replicated, so every rank makes the same choice),
applies its own experts into an fp32 partial sum, one rank also adds the residual and
the shared experts, and a reduce-scatter sums the partials and hands each rank its own
tokens' rows, which the library rounds to bf16 once. Each expert's weights are then
read on one GPU only.
"""
from __future__ import annotations

from typing import Tuple

import torch
import torch.distributed as dist


def shard_rows(T_total: int, rank: int, world: int) -> Tuple[int, int]:
    """[start, stop) of rank's contiguous token shard; shard sizes differ by at most one."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    base, extra = divmod(T_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def reduce_balance_sums(counts: torch.Tensor, P_sum: torch.Tensor, group=None) -> None:
    """Sum every rank's per-expert token counts (int32) and score sums (fp32) in place."""
    dist.all_reduce(counts, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(P_sum, op=dist.ReduceOp.SUM, group=group)


def global_balance_stats(handle, T_total: int, counts: torch.Tensor, P_sum: torch.Tensor, f: torch.Tensor,
                         P: torch.Tensor, group=None, stream=None) -> None:
    """All-reduce the shard sums, then f_i and P_i over all T_total tokens (device kernel)."""
    from .binding import dsmoe_balance_stats
    reduce_balance_sums(counts, P_sum, group)
    dsmoe_balance_stats(handle, T_total, counts, P_sum, f, P, stream)


def expert_block(n_routed: int, rank: int, world: int) -> Tuple[int, int]:
    """[e_begin, e_end) of the routed experts rank holds: contiguous blocks, sizes
    differing by at most one."""
    return shard_rows(n_routed, rank, world)


def configure_expert_shard(layer, rank: int, world: int) -> Tuple[int, int]:
    """Set a layer (binding.DSMoE built with this rank's block of expert weights) to apply
    its block and write fp32 partial sums; rank 0 also adds the residual and the shared
    experts."""
    e0, e1 = expert_block(layer.cfg.n_routed, rank, world)
    layer.set_expert_range(e0, e1, partial=True, add_shared=(rank == 0))
    return e0, e1


def expert_sharded_forward(layer, x_local: torch.Tensor, token_ids_local: torch.Tensor = None, group=None,
                           stream=None, round_bf16=None):
    """The layer on this rank's tokens in the expert-sharded form. Every rank must pass the
    same number of tokens. Returns h (bf16, this rank's rows), this rank's topk_idx and
    gates, and the whole batch's counts, f and P (identical on every rank).

    round_bf16(src, dst) turns the summed fp32 rows into bf16; by default the library's
    kernel (dsmoe_round_bf16) on `stream`."""
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T, d = x_local.shape
    x_all = torch.empty((world * T, d), dtype=x_local.dtype, device=x_local.device)
    dist.all_gather_into_tensor(x_all, x_local.contiguous(), group=group)
    ids_all = None
    if token_ids_local is not None:
        ids_all = torch.empty((world * T,), dtype=token_ids_local.dtype, device=token_ids_local.device)
        dist.all_gather_into_tensor(ids_all, token_ids_local.contiguous(), group=group)
    out = layer.forward(x_all, token_ids=ids_all, stream=stream)
    mine = torch.empty((T, d), dtype=torch.float32, device=x_local.device)
    dist.reduce_scatter_tensor(mine, out["h"], op=dist.ReduceOp.SUM, group=group)
    h = torch.empty((T, d), dtype=torch.bfloat16, device=x_local.device)
    if round_bf16 is None:
        from .binding import dsmoe_round_bf16
        dsmoe_round_bf16(layer.handle, T * d, mine, h, stream)
    else:
        round_bf16(mine, h)
    rows = slice(rank * T, (rank + 1) * T)
    return dict(h=h, topk_idx=out["topk_idx"][rows], gates=out["gates"][rows], counts=out["counts"], f=out["f"],
                P=out["P"])


def token_dispatch_forward(layer, x_local: torch.Tensor, token_ids_local: torch.Tensor = None, group=None,
                           stream=None, lib=None):
    """The layer on this rank's tokens in the token-dispatch expert-parallel form (the
    "MoE: sparse activation" page's training-cost section: tokens travel by all-to-all to
    the GPUs that hold their experts; the interview card's deployment trade-off: routed
    experts sharded, shared experts replicated).

    layer: binding.DSMoE whose W_gate / W_up / W_down hold this rank's contiguous block of
    routed experts (expert_block) and whose router and shared experts are full copies;
    its handle's max_tokens must cover the rows this rank may receive (world * T at
    most). Steps: dsmoe_ep_route (route, gather the rows into expert order, which is
    destination order) -> all-to-all of the per-expert counts, then of the rows ->
    dsmoe_ep_experts (this rank's experts on what it received) -> all-to-all back ->
    dsmoe_ep_combine (shared experts, gate-weighted sum, residual). Returns h (bf16) and
    this rank's routing; counts, f and P are this rank's tokens' statistics (reduce them
    with global_balance_stats for the whole batch).

    lib: the object providing the library calls (the binding module by default)."""
    if lib is None:
        from . import binding as lib
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    cfg = layer.cfg
    T, d = x_local.shape
    N = cfg.n_routed
    dev = x_local.device
    K = layer.k_active
    out = layer.alloc_outputs(T)
    send_rows = torch.empty((world,), dtype=torch.int32, device=dev)
    w = layer.w
    lib.dsmoe_ep_route(layer.handle, T, x_local, token_ids_local, w.get("W_router"), w.get("b"), out["topk_idx"],
                       out["gates"], out["counts"], out["f"], out["P"], out["P_sum"], None, world, send_rows, stream)
    # per-expert counts to each expert's owner
    blocks = [expert_block(N, j, world) for j in range(world)]
    e0, e1 = blocks[rank]
    n_local = e1 - e0
    recv_counts = torch.empty((world * n_local,), dtype=torch.int32, device=dev)
    dist.all_to_all_single(recv_counts, out["counts"], output_split_sizes=[n_local] * world,
                           input_split_sizes=[b - a for a, b in blocks], group=group)
    # the row exchange needs its split sizes on the host
    send_splits = [int(v) for v in send_rows.cpu().tolist()]
    per_src = recv_counts.view(world, n_local).cpu().numpy().sum(axis=1)
    recv_splits = [int(v) for v in per_src]
    xp = lib.workspace_view(layer.handle, "Xp", layer.device)[:T * K]
    rows = torch.empty((sum(recv_splits), d), dtype=torch.bfloat16, device=dev)
    dist.all_to_all_single(rows, xp, output_split_sizes=recv_splits, input_split_sizes=send_splits, group=group)
    y_rows = torch.empty_like(rows)
    lib.dsmoe_ep_experts(layer.handle, world, e0, e1, recv_counts, rows.shape[0], rows, w["W_gate"], w["W_up"],
                         w["W_down"], y_rows, stream)
    y_back = torch.empty((T * K, d), dtype=torch.bfloat16, device=dev)
    dist.all_to_all_single(y_back, y_rows, output_split_sizes=send_splits, input_split_sizes=recv_splits,
                           group=group)
    h = torch.empty((T, d), dtype=torch.bfloat16, device=dev)
    lib.dsmoe_ep_combine(layer.handle, T, x_local, w.get("Ws_gate"), w.get("Ws_up"), w.get("Ws_down"), out["gates"],
                         y_back, h, stream)
    out["h"] = h
    return out
