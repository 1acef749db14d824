"""dsmoe_route_noalloc: the routing stage for callers that cannot allocate device
memory (their framework already owns the GPU's memory through its own pool, or they
must not create a handle, which allocates). It uses a fixed scratch array inside the
library instead of a workspace.

Its outputs are checked against the float64 oracle on two calls in a row (the second
call finds the scratch left over from the first), with the parity tests' tolerances:
expert indices bit-exact, in order, on every token whose oracle selection keys are
separated by more than 1e-4 at every position that decides the output; on the other
tokens the kernel's choice must be one the keys allow (every picked key within 1e-4
of the K'-th largest, listed in descending order up to that margin); gates within
1e-5 of the float64 gates at the kernel's own experts; counts equal to the histogram
of its selection; f within one fp32 ulp; P within 1e-5. The forward's own routing is
compared too (same indices wherever the oracle keys leave the margin).

This file is collected last so that a run stopping at the first failure has run every
other test first."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from oracle import dsmoe_oracle as O
from tests import parity as PAR

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)

CASES = [("v4_decode_t64", 64), ("tiny", 300), ("v3_prefill", 200), ("ds2b", 700)]


def _oracle_check(cfg, cpu, T, topk, gates, counts, f, P):
    r = O.route(cfg, cpu)
    s = r["scores"]
    b = None if cpu.get("b") is None else cpu["b"].numpy().astype(np.float64)
    key = s + (b[None, :] if cfg.bias_mode == O.BIAS_SELECT_ONLY else 0.0)
    K, N = cfg.top_k, cfg.n_routed
    srt = -np.sort(-key, axis=1)
    hi = min(K, N - 1)
    clean = ((srt[:, :hi] - srt[:, 1:hi + 1]) > PAR.GAP).all(axis=1)
    topk = topk.astype(np.int64)
    assert (topk[clean] == r["idx"][clean]).all(), "indices differ on tokens the keys separate"
    picked = np.take_along_axis(key, topk, axis=1)
    assert (np.sort(topk, axis=1)[:, 1:] != np.sort(topk, axis=1)[:, :-1]).all(), "an expert picked twice"
    assert (picked >= srt[:, K - 1:K] - PAR.GAP).all(), "a picked expert is not among the top K' keys"
    assert (picked[:, 1:] <= picked[:, :-1] + PAR.GAP).all(), "picked experts not in descending key order"
    g_ref = np.take_along_axis(s, topk, axis=1)
    if cfg.renormalize:
        g_ref = g_ref / g_ref.sum(axis=1, keepdims=True)
    gerr = np.abs(gates.astype(np.float64) - g_ref).max()
    assert gerr <= PAR.GATE_TOL, f"gate error {gerr}"
    assert (np.bincount(topk.ravel(), minlength=N) == counts).all(), "counts != histogram of the selection"
    f_ref = (N / (K * T) * counts.astype(np.float64)).astype(np.float32)
    assert (np.abs(f - f_ref) <= np.spacing(np.abs(f_ref))).all(), "f off by more than one ulp"
    perr = (np.abs(P.astype(np.float64) - r["P"]) / np.maximum(1.0, np.abs(r["P"]))).max()
    assert perr <= 1e-5, f"P error {perr}"
    return clean, int((~clean).sum()), float(gerr), float(perr)


@pytest.mark.parametrize("name,T", CASES, ids=[c[0] for c in CASES])
def test_noalloc_routing_matches_oracle(name, T):
    cfg = W.get_config(name)
    cpu = W.make_inputs(cfg, seed=0, device="cpu", T=T, with_weights=False)
    gpu = {k: (None if v is None else v.to("cuda:0")) for k, v in cpu.items()}
    c = M.cfg_from(cfg, T)
    K, N = cfg.top_k, cfg.n_routed
    for call in range(2):
        topk = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        gates = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
        counts = torch.full((N,), -1, dtype=torch.int32, device="cuda")
        f = torch.full((N,), -1.0, dtype=torch.float32, device="cuda")
        P = torch.full((N,), -1.0, dtype=torch.float32, device="cuda")
        M.dsmoe_route_noalloc(c, T, gpu["x"], gpu["W_router"], gpu.get("b"), topk, gates, counts, f, P)
        torch.cuda.synchronize()
        clean, n_near, gerr, perr = _oracle_check(cfg, cpu, T, topk.cpu().numpy(), gates.cpu().numpy(),
                                                  counts.cpu().numpy(), f.cpu().numpy(), P.cpu().numpy())
        print(name, "call", call, "near-tie tokens", n_near, "gate err", gerr, "P err", perr)
    # the forward's routing (its own workspace and kernels) picks the same experts where
    # the oracle's keys leave the margin
    fw = W.make_inputs(cfg, seed=0, device="cuda", T=T)  # expert weights (routing does not read them)
    fw.update({k: gpu[k] for k in ("x", "W_router", "b")})
    layer = M.DSMoE(M.cfg_from(cfg, T), fw)
    ref = layer.forward(fw["x"])
    torch.cuda.synchronize()
    layer.close()
    cl = torch.as_tensor(clean, device="cuda")
    assert torch.equal(topk[cl], ref["topk_idx"][cl])
    del fw


def test_noalloc_rejects_sizes_beyond_its_limits():
    cfg = W.get_config("tiny")
    cpu = W.make_inputs(cfg, seed=0, device="cpu", T=8, with_weights=False)
    gpu = {k: (None if v is None else v.to("cuda:0")) for k, v in cpu.items()}
    o = dict(topk=torch.empty((8, 7), dtype=torch.int32, device="cuda"),
             gates=torch.empty((8, 7), device="cuda"), counts=torch.empty(64, dtype=torch.int32, device="cuda"),
             f=torch.empty(64, device="cuda"), P=torch.empty(64, device="cuda"))
    small = M.cfg_from(cfg, 4)
    with pytest.raises(M.DsmoeError) as ei:  # T = 8 > max_tokens = 4
        M.dsmoe_route_noalloc(small, 8, gpu["x"], gpu["W_router"], None, o["topk"], o["gates"], o["counts"],
                              o["f"], o["P"])
    assert ei.value.status == M.DSMOE_ERR_WORKSPACE and "max_tokens" in M.dsmoe_last_error()
    hashed = M.cfg_from(W.get_config("v4_hash_t16"), 8)
    with pytest.raises(M.DsmoeError) as ei:
        M.dsmoe_route_noalloc(hashed, 8, gpu["x"], gpu["W_router"], None, o["topk"], o["gates"], o["counts"],
                              o["f"], o["P"])
    assert ei.value.status == M.DSMOE_ERR_UNSUPPORTED
