"""Failure detection on the GPU without a fault: every in-kernel wait is bounded, and a
kernel role that gives up records it in the device status word instead of hanging.

A forward run with a 1 ns wait limit makes the waits run out (the epilogue's first wait
for an accumulator cannot be satisfied that soon); the kernels then wait, for at least
a second, for the copies and MMAs they already started, free their tensor memory and
return. dsmoe_get_status must report DSMOE_ERR_DEVICE_TIMEOUT, the context must stay
usable, and a forward on the same handle with the default limit must again match the
oracle."""
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


def test_wait_limit_runs_out_then_handle_recovers():
    cfg = W.get_config("tiny").replace(T=300)  # T >= 256: tensor-core router, both GEMMs
    gpu, cpu = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    try:
        with pytest.raises(M.DsmoeError) as ei:
            M.dsmoe_set_wait_limit(layer.handle, 0)
        assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK
        M.dsmoe_set_wait_limit(layer.handle, 1)
        layer.forward(gpu["x"])
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_ERR_DEVICE_TIMEOUT
        assert "status word" in M.dsmoe_last_error()
        # the status word was cleared by the read; the context is still usable
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK
        M.dsmoe_set_wait_limit(layer.handle, 2_000_000_000)
        out = layer.forward(gpu["x"], with_scores=True)
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK
    finally:
        layer.close()
    ref = PAR.reference_selection(cfg, cpu, out["topk_idx"], out["scores"])
    PAR.check_routing(cfg, ref, out, cfg.T)
    PAR.check_h(cfg, cpu, ref, out, np.arange(cfg.T))
