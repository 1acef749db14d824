"""The parity machinery itself, on the CPU: fed the oracle's own outputs as if a kernel had
produced them, it must accept them — for the plain selection, for the selection variants
(masked top experts, fewer active experts) and for inputs where every score ties, which
exercises the near-tie re-decision path."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import dsmoe_oracle as O
from tests import parity as PAR


def _as_kernel_outputs(cfg, r, T):
    f32 = lambda a: torch.from_numpy(np.asarray(a, dtype=np.float32))
    return dict(topk_idx=torch.from_numpy(r["idx"].astype(np.int32)), gates=f32(r["gates"]),
                counts=torch.from_numpy(r["counts"].astype(np.int32)),
                f=f32(cfg.n_routed / (cfg.top_k * T) * r["counts"]), P=f32(r["P"]), scores=f32(r["scores"]))


@pytest.mark.parametrize("mask_top,k_active", [(0, 7), (2, 5), (1, 3), (0, 1)])
def test_reference_selection_accepts_the_oracle(mask_top, k_active):
    cfg = W.get_config("tiny").replace(T=96, top_k=k_active, mask_top=mask_top)
    inp = W.make_inputs(cfg, seed=4, with_weights=False)
    r = O.route(cfg, inp)
    out = _as_kernel_outputs(cfg, r, cfg.T)
    ref = PAR.reference_selection(cfg, inp, out["topk_idx"], out["scores"])
    PAR.check_routing(cfg, ref, out, cfg.T)
    np.testing.assert_array_equal(ref["idx"], r["idx"])


def test_all_tied_scores_are_redecided_not_rejected():
    cfg = W.get_config("tiny").replace(T=32, top_k=3, mask_top=2)
    inp = W.make_inputs(cfg, seed=5, with_weights=False)
    inp["W_router"] = inp["W_router"][0:1].expand_as(inp["W_router"]).contiguous()
    r = O.route(cfg, inp)
    out = _as_kernel_outputs(cfg, r, cfg.T)
    ref = PAR.reference_selection(cfg, inp, out["topk_idx"], out["scores"])
    assert ref["redecided"].all()  # every key ties: nothing is decided by a margin
    PAR.check_routing(cfg, ref, out, cfg.T)
    # ties go to the lower index: experts 0, 1 masked, 2..4 kept
    assert (ref["idx"] == np.array([2, 3, 4])).all()


def test_a_wrong_selection_is_caught():
    cfg = W.get_config("tiny").replace(T=64, top_k=4, mask_top=1)
    inp = W.make_inputs(cfg, seed=6, with_weights=False)
    r = O.route(cfg, inp)
    out = _as_kernel_outputs(cfg, r, cfg.T)
    plain = O.select_topk(r["scores"], 4, inp.get("b"), cfg.bias_mode, cfg.renormalize)[0]
    out["topk_idx"] = torch.from_numpy(plain.astype(np.int32))  # forgot the mask
    with pytest.raises(AssertionError):  # caught by the set check or the index check
        ref = PAR.reference_selection(cfg, inp, out["topk_idx"], out["scores"])
        PAR.check_routing(cfg, ref, out, cfg.T)
