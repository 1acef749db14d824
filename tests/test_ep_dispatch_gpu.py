"""Token-dispatch expert parallelism on one GPU: the library's three calls
(dsmoe_ep_route -> dsmoe_ep_experts -> dsmoe_ep_combine) for R "ranks", each with its own
handle, its token shard and its contiguous block of routed experts (DeepSeek-MoE interview
card, deep dive on engineering trade-offs, item 5; "MoE: sparse activation" page,
training-cost section). The ranks run one after another on the same GPU and the
all-to-all exchanges are done by the test with plain tensor copies between the ranks'
buffers, so no kernel waits on another rank.

Checked: each rank's routing against the oracle on its shard (as the parity tests do),
the rows each rank sends (its slot order gathers x exactly), the per-destination row
counts, and each rank's h against the float64 oracle layer on the same tokens within the
layer bound (max |err| / RMS <= 2e-2)."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from mixture_experts_layer_score_b200.sharded import expert_block, shard_rows
from tests import parity as PAR
from tests.gpu_cases import make_case

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)

CASES = [("tiny", 301, 2), ("gshard_c", 700, 3), ("v4_decode_t16", 16, 4), ("v4_hash_t16", 16, 2)]


@pytest.mark.parametrize("name,T,R", CASES, ids=[f"{c[0]}-R{c[2]}" for c in CASES])
def test_token_dispatch_equals_the_layer(name, T, R):
    cfg = W.get_config(name)
    gpu, cpu = make_case(cfg, T)
    N, K, d = cfg.n_routed, cfg.top_k, cfg.d_model
    shards = [shard_rows(T, r, R) for r in range(R)]
    blocks = [expert_block(N, r, R) for r in range(R)]
    layers, outs, sends = [], [], []
    try:
        for r in range(R):
            a, b = shards[r]
            e0, e1 = blocks[r]
            w = dict(gpu)
            for k in ("W_gate", "W_up", "W_down"):
                w[k] = gpu[k][e0:e1]
            layer = M.DSMoE(M.cfg_from(cfg, T), w)  # max_tokens covers every row a rank may receive
            layers.append(layer)
            o = layer.alloc_outputs(b - a, with_scores=True)
            send_rows = torch.empty((R,), dtype=torch.int32, device="cuda")
            ids = None if gpu.get("token_ids") is None else gpu["token_ids"][a:b]
            M.dsmoe_ep_route(layer.handle, b - a, gpu["x"][a:b], ids, gpu.get("W_router"), gpu.get("b"),
                             o["topk_idx"], o["gates"], o["counts"], o["f"], o["P"], o["P_sum"], o["scores"], R,
                             send_rows)
            outs.append(o)
            sends.append(send_rows)
        torch.cuda.synchronize()
        # the exchange, done by the test: rank r's rows for rank j, and the per-expert counts
        xp = [M.workspace_view(layers[r].handle, "Xp")[:(shards[r][1] - shards[r][0]) * K].clone() for r in range(R)]
        for r in range(R):
            a, b = shards[r]
            ref = PAR.reference_selection(cfg, {k: (v[a:b] if k in ("x", "token_ids") and v is not None else v)
                                                for k, v in cpu.items()}, outs[r]["topk_idx"], outs[r]["scores"])
            PAR.check_routing(cfg, ref, outs[r], b - a)
            cnt = outs[r]["counts"].cpu().numpy()
            want = [int(cnt[e0:e1].sum()) for e0, e1 in blocks]
            assert sends[r].cpu().tolist() == want
            slot = M.workspace_view(layers[r].handle, "slot_of")[:b - a, :K].long()
            assert torch.equal(xp[r][slot.reshape(-1)], gpu["x"][a:b].repeat_interleave(K, dim=0))
        starts = [[0] + list(np.cumsum(s.cpu().numpy())) for s in sends]
        y_back = [torch.empty(((b - a) * K, d), dtype=torch.bfloat16, device="cuda") for a, b in shards]
        for j in range(R):
            e0, e1 = blocks[j]
            rows = torch.cat([xp[r][starts[r][j]:starts[r][j + 1]] for r in range(R)])
            recv_counts = torch.cat([outs[r]["counts"][e0:e1] for r in range(R)]).to(torch.int32).contiguous()
            y = torch.empty_like(rows)
            M.dsmoe_ep_experts(layers[j].handle, R, e0, e1, recv_counts, rows.shape[0], rows, gpu["W_gate"][e0:e1],
                               gpu["W_up"][e0:e1], gpu["W_down"][e0:e1], y)
            torch.cuda.synchronize()
            off = 0
            for r in range(R):
                n = starts[r][j + 1] - starts[r][j]
                y_back[r][starts[r][j]:starts[r][j + 1]] = y[off:off + n]
                off += n
        for r in range(R):
            a, b = shards[r]
            h = torch.empty((b - a, d), dtype=torch.bfloat16, device="cuda")
            M.dsmoe_ep_combine(layers[r].handle, b - a, gpu["x"][a:b], gpu.get("Ws_gate"), gpu.get("Ws_up"),
                               gpu.get("Ws_down"), outs[r]["gates"], y_back[r], h)
            torch.cuda.synchronize()
            assert M.dsmoe_get_status(layers[r].handle) == M.DSMOE_OK, M.dsmoe_last_error()
            sub = {k: (v[a:b] if k in ("x", "token_ids") and v is not None else v) for k, v in cpu.items()}
            ref = PAR.reference_selection(cfg, sub, outs[r]["topk_idx"], outs[r]["scores"])
            hh = PAR.check_h(cfg, sub, ref, dict(h=h), np.arange(b - a))
            print(name, R, "rank", r, hh)
    finally:
        for layer in layers:
            layer.close()


def test_ep_argument_errors():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 8)
    layer = M.DSMoE(M.cfg_from(cfg, 8), gpu)
    try:
        cnt = torch.zeros(64, dtype=torch.int32, device="cuda")
        with pytest.raises(M.DsmoeError) as ei:  # 64 sources x 64 experts > 512 groups
            M.dsmoe_ep_experts(layer.handle, 64, 0, 64, cnt, 0, None, None, None, None, None)
        assert ei.value.status == M.DSMOE_ERR_UNSUPPORTED
        with pytest.raises(M.DsmoeError) as ei:  # more rows than the workspace holds
            M.dsmoe_ep_experts(layer.handle, 1, 0, 8, cnt, 8 * 7 + 1, None, None, None, None, None)
        assert ei.value.status == M.DSMOE_ERR_WORKSPACE
        with pytest.raises(M.DsmoeError) as ei:  # combine before any route on this handle
            M.dsmoe_ep_combine(layer.handle, 8, gpu["x"], None, None, None, None, None, None)
        assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
    finally:
        layer.close()
