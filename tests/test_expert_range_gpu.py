"""Expert-parallel pieces on one GPU: a handle restricted to a block of the routed
experts (dsmoe_set_expert_range) writes the fp32 partial sum of its experts' terms, one
rank adding the residual and the shared experts (DeepSeek-MoE interview card, deep dive
on engineering trade-offs, item 5: shared experts replicated, routed experts sharded).

The "ranks" of an R-way split run one after another on the same GPU (each is an
independent forward; none waits on another). Each partial is compared with the oracle's
partial (oracle/dsmoe_ep.py gather_partial) element-wise, max |err| <= 2e-2 RMS(h) with h
the whole layer's output that the partials add up to (a partial without the residual is
smaller than h, while its error, one bf16 rounding of each expert row it sums, is the same
as in h); the sum over ranks, rounded to bf16 by the library, must meet the layer bound
against the oracle's h; every rank's routing must equal the oracle's and each other's."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from oracle import dsmoe_ep as EP
from tests import parity as PAR
from tests.gpu_cases import make_case

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)

CASES = [("v4_decode_t16", 16, 4), ("gshard_c", 700, 3), ("tiny", 300, 2), ("v4_hash_t16", 16, 2)]
WEIGHTS = ("W_gate", "W_up", "W_down")


def _block(N, r, R):
    e0 = (N // R) * r + min(r, N % R)
    return e0, e0 + N // R + (1 if r < N % R else 0)


@pytest.mark.parametrize("name,T,R", CASES, ids=[f"{c[0]}-R{c[2]}" for c in CASES])
def test_expert_range_partials_sum_to_the_layer(name, T, R):
    cfg = W.get_config(name)
    gpu, cpu = make_case(cfg, T)
    N = cfg.n_routed
    parts, routes = [], []
    for r in range(R):
        e0, e1 = _block(N, r, R)
        w = dict(gpu)
        for k in WEIGHTS:
            w[k] = gpu[k][e0:e1]
        if r > 0:
            w["Ws_gate"] = w["Ws_up"] = w["Ws_down"] = None  # only rank 0 adds the shared experts
        layer = M.DSMoE(M.cfg_from(cfg, T), w)
        try:
            layer.set_expert_range(e0, e1, partial=True, add_shared=(r == 0))
            assert M.dsmoe_get_expert_range(layer.handle) == (e0, e1, M.DSMOE_RANGE_PARTIAL |
                                                               (M.DSMOE_RANGE_ADD_SHARED if r == 0 else 0))
            out = layer.forward(gpu["x"], token_ids=gpu.get("token_ids"), with_scores=True)
            torch.cuda.synchronize()
            assert out["h"].dtype == torch.float32
            assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK, M.dsmoe_last_error()
        finally:
            layer.close()
        parts.append((e0, e1, out["h"]))
        routes.append(out)
    for o in routes[1:]:
        for k in ("topk_idx", "gates", "counts", "f", "P"):
            assert torch.equal(o[k], routes[0][k]), k
    ref = PAR.reference_selection(cfg, cpu, routes[0]["topk_idx"], routes[0]["scores"])
    PAR.check_routing(cfg, ref, routes[0], T)
    shared = [(cpu["Ws_gate"][i], cpu["Ws_up"][i], cpu["Ws_down"][i]) for i in range(cfg.n_shared)]
    all_experts = {e: (cpu["W_gate"][e], cpu["W_up"][e], cpu["W_down"][e]) for e in np.unique(ref["idx"])}
    h_ref = EP.gather_partial(cpu["x"], ref["idx"], ref["gates"], all_experts, range(N), shared)
    rms_h = np.sqrt(np.mean(h_ref ** 2))
    worst = 0.0
    for r, (e0, e1, h32) in enumerate(parts):
        local = {e: (cpu["W_gate"][e], cpu["W_up"][e], cpu["W_down"][e]) for e in range(e0, e1)
                 if (ref["idx"] == e).any()}
        p_ref = EP.gather_partial(cpu["x"], ref["idx"], ref["gates"], local, range(e0, e1),
                                  shared if r == 0 else None)
        err = np.abs(h32.cpu().numpy().astype(np.float64) - p_ref).max() / rms_h
        worst = max(worst, float(err))
    total = parts[0][2].clone()
    for _, _, h32 in parts[1:]:
        total += h32
    h = torch.empty(total.shape, dtype=torch.bfloat16, device="cuda")
    probe = M.DSMoE(M.cfg_from(cfg, 1), gpu)
    M.dsmoe_round_bf16(probe.handle, total.numel(), total, h)
    torch.cuda.synchronize()
    probe.close()
    assert torch.equal(h, total.to(torch.bfloat16))  # round to nearest even, as torch does
    hh = PAR.check_h(cfg, cpu, ref, dict(h=h), np.arange(T))
    print(name, R, "worst partial err / RMS(h)", worst, hh)
    assert worst <= PAR.H_TOL


def test_full_range_partial_rounds_to_the_plain_forward():
    """The whole layer as an unrounded fp32 sum (full range, PARTIAL | ADD_SHARED) rounds to
    exactly the bf16 h of the default forward: same terms, same order."""
    cfg = W.get_config("gshard_c").replace(T=500)
    gpu, _ = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    try:
        a = layer.forward(gpu["x"])
        layer.set_expert_range(0, cfg.n_routed, partial=True, add_shared=True)
        b = layer.forward(gpu["x"])
        h = torch.empty_like(a["h"])
        M.dsmoe_round_bf16(layer.handle, b["h"].numel(), b["h"], h)
        torch.cuda.synchronize()
        assert torch.equal(h, a["h"])
        for k in ("topk_idx", "gates", "counts", "f", "P"):
            assert torch.equal(a[k], b[k]), k
    finally:
        layer.close()


def test_expert_range_rejects_bad_arguments():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 8)
    layer = M.DSMoE(M.cfg_from(cfg, 8), gpu)
    try:
        P, S = M.DSMOE_RANGE_PARTIAL, M.DSMOE_RANGE_ADD_SHARED
        for e0, e1, fl in ((0, 0, P), (-1, 4, P), (3, 65, P), (5, 2, P), (0, 32, S), (0, 64, 0), (0, 64, 8)):
            with pytest.raises(M.DsmoeError) as ei:
                M.dsmoe_set_expert_range(layer.handle, e0, e1, fl)
            assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
        assert M.dsmoe_get_expert_range(layer.handle) == (0, 64, S)  # unchanged default
        M.dsmoe_set_expert_range(layer.handle, 0, 32, P)
        with pytest.raises(M.DsmoeError) as ei:  # the host entry point runs the whole layer only
            M.dsmoe_forward_host(layer.handle, 0, None, None, None, None, None, None, None, None, None, None,
                                 None, None, None, torch.empty(64, dtype=torch.int32),
                                 torch.empty(64), torch.empty(64))
        assert ei.value.status == M.DSMOE_ERR_UNSUPPORTED
        with pytest.raises(M.DsmoeError):
            M.dsmoe_round_bf16(layer.handle, 7, torch.empty(8, device="cuda"),
                               torch.empty(8, dtype=torch.bfloat16, device="cuda"))
    finally:
        layer.close()
