"""dsmoe_route_noalloc: the routing stage for callers that cannot allocate device
memory (their framework already owns the GPU's memory through its own pool, or they
must not create a handle, which allocates). It uses a fixed scratch array inside the
library instead of a workspace. Its outputs must equal the forward's routing outputs
within the tolerances the parity tests use, on two calls in a row (the second call
finds the scratch left over from the first).

This file is collected last so that a run stopping at the first failure has run every
other test first."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from tests import parity as PAR
from tests.gpu_cases import make_case

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)

CASES = [("v4_decode_t64", 64), ("tiny", 300), ("v3_prefill", 200), ("ds2b", 700)]


def _clear_tokens(cfg, scores, b):
    """Tokens whose selection keys (from the forward's fp32 scores) are separated by more
    than the parity tests' 1e-4 gap at every adjacent position up to K'+1."""
    key = scores.double() + (b.double()[None, :] if (b is not None and cfg.bias_mode == W.BIAS_SELECT_ONLY)
                             else 0.0)
    top = torch.sort(key, dim=1, descending=True).values[:, :cfg.top_k + 1]
    return ((top[:, :-1] - top[:, 1:]) > PAR.GAP).all(dim=1)


@pytest.mark.parametrize("name,T", CASES, ids=[c[0] for c in CASES])
def test_noalloc_routing_matches_forward(name, T):
    cfg = W.get_config(name)
    gpu, _ = make_case(cfg, T)
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    ref = layer.forward(gpu["x"], with_scores=True)
    torch.cuda.synchronize()
    layer.close()
    clear = _clear_tokens(cfg, ref["scores"], gpu.get("b"))
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
        # expert indices: identical wherever the forward's keys leave a margin of 1e-4
        assert torch.equal(topk[clear], ref["topk_idx"][clear]), f"call {call}: expert indices differ"
        same = (topk == ref["topk_idx"]).all(dim=1)
        assert (gates[same] - ref["gates"][same]).abs().max().item() <= PAR.GATE_TOL, f"call {call}: gates"
        # counts: the histogram of its own selection; equal to the forward's where selections agree
        hist = torch.bincount(topk.view(-1).long(), minlength=N).to(torch.int32)
        assert torch.equal(counts, hist), f"call {call}: counts != histogram"
        if bool(same.all()):
            assert torch.equal(counts, ref["counts"]), f"call {call}: counts"
        fr = (N / (K * T) * counts.double()).float().cpu().numpy()
        assert (np.abs(f.cpu().numpy() - fr) <= np.spacing(np.abs(fr))).all(), f"call {call}: f"
        Pr = ref["P"].cpu().numpy().astype(np.float64)
        perr = np.abs(P.cpu().numpy() - Pr) / np.maximum(1.0, np.abs(Pr))
        assert perr.max() <= 1e-5, f"call {call}: P error {perr.max()}"


def test_noalloc_rejects_sizes_beyond_its_limits():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 8)
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
