"""Parity of the selection variants (dsmoe_set_selection) with the oracle: masking each
token's top-ranked routed experts before the top-K' choice, and activating fewer routed
experts than the router was configured for (DeepSeekMoE summary, expert-specialisation
analysis). Routing, statistics and h are checked as in test_parity_gpu.py."""
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

# (workload, T, mask_top, k_active): softmax without renormalisation (DeepSeekMoE),
# sigmoid + selection-only bias + renormalisation (V3 shapes), softmax with a logit bias
CASES = [("gshard_c", 700, 1, 7), ("gshard_c", 700, 3, 4), ("gshard_c", 300, 0, 3),
         ("tiny", 257, 2, 5), ("v3_prefill", 300, 2, 8), ("v3_prefill", 300, 0, 4),
         ("ds2b", 1000, 4, 6), ("v4_decode_t16", 16, 1, 9)]


@pytest.mark.parametrize("name,T,mask_top,k_active", CASES,
                         ids=[f"{c[0]}-T{c[1]}-mask{c[2]}-k{c[3]}" for c in CASES])
def test_selection_variant_parity(name, T, mask_top, k_active):
    cfg = W.get_config(name)
    gpu, cpu = make_case(cfg, T)
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    try:
        layer.set_selection(mask_top, k_active)
        assert M.dsmoe_get_selection(layer.handle) == (mask_top, k_active)
        out = layer.forward(gpu["x"], with_scores=True)
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK, M.dsmoe_last_error()
    finally:
        layer.close()
    cfg_v = cfg.replace(top_k=k_active, mask_top=mask_top)
    assert tuple(out["topk_idx"].shape) == (T, k_active)
    ref = PAR.reference_selection(cfg_v, cpu, out["topk_idx"], out["scores"])
    rr = PAR.check_routing(cfg_v, ref, out, T)
    hh = PAR.check_h(cfg_v, cpu, ref, out, np.arange(min(T, 32)))
    print(name, T, mask_top, k_active, rr, hh)


def test_selection_defaults_reproduce_the_plain_forward():
    cfg = W.get_config("gshard_b").replace(T=500)
    gpu, _ = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    try:
        a = layer.forward(gpu["x"], with_scores=True)
        layer.set_selection(2, 5)
        b = layer.forward(gpu["x"], with_scores=True)
        layer.set_selection(0, cfg.top_k)
        c = layer.forward(gpu["x"], with_scores=True)
        torch.cuda.synchronize()
    finally:
        layer.close()
    for k in ("h", "topk_idx", "gates", "counts", "f", "scores"):
        assert torch.equal(a[k], c[k]), k
    # the masked, shortened selection is the plain order's columns 2..6
    assert torch.equal(b["topk_idx"], a["topk_idx"][:, 2:7].contiguous())
    assert torch.equal(a["P"], b["P"])  # the mean score does not depend on the variant


def test_selection_rejects_bad_arguments():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 8)
    layer = M.DSMoE(M.cfg_from(cfg, 8), gpu)
    try:
        for m, k in ((0, 0), (0, cfg.top_k + 1), (-1, 2), (cfg.n_routed - 2, 3)):
            with pytest.raises(M.DsmoeError) as ei:
                M.dsmoe_set_selection(layer.handle, m, k)
            assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
        assert M.dsmoe_get_selection(layer.handle) == (0, cfg.top_k)  # unchanged
    finally:
        layer.close()
    hcfg = W.get_config("v4_hash_t16")
    gpu, _ = make_case(hcfg, 16)
    layer = M.DSMoE(M.cfg_from(hcfg, 16), gpu)
    try:
        with pytest.raises(M.DsmoeError) as ei:
            M.dsmoe_set_selection(layer.handle, 1, hcfg.top_k)
        assert ei.value.status == M.DSMOE_ERR_UNSUPPORTED
        M.dsmoe_set_selection(layer.handle, 0, hcfg.top_k)
    finally:
        layer.close()
