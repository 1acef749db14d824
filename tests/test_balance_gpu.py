"""The balance-control entry points against the oracle (float64) on statistics from real
forwards: expert- and device-level losses, sequence-wise statistics, the bias update."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from oracle import dsmoe_oracle as O
from tests.gpu_cases import make_case

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)


@pytest.mark.parametrize("name,T,seq_len,groups", [("gshard_c", 1024, 256, 7), ("v3_prefill", 512, 128, 8),
                                                   ("tiny", 300, 100, 64)])
def test_balance_control_matches_oracle(name, T, seq_len, groups):
    cfg = W.get_config(name)
    gpu, _ = make_case(cfg, T)
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    out = layer.forward(gpu["x"], with_scores=True)
    N = cfg.n_routed
    f, P = out["f"], out["P"]
    group_of = torch.arange(N, dtype=torch.int32, device="cuda") * groups // N
    f_dev = torch.empty(groups, device="cuda")
    P_dev = torch.empty(groups, device="cuda")
    losses = torch.empty(2, device="cuda")
    M.dsmoe_balance_losses(layer.handle, f, P, groups, group_of, 0.003, 0.05, f_dev, P_dev, losses)
    S = T // seq_len
    f_seq = torch.empty((S, N), device="cuda")
    p_seq = torch.empty((S, N), device="cuda")
    loss = torch.empty(1, device="cuda")
    M.dsmoe_sequence_balance(layer.handle, T, seq_len, out["topk_idx"], out["scores"], 1e-4, f_seq, p_seq, loss)
    b = (gpu["b"].clone() if gpu.get("b") is not None else torch.zeros(N, device="cuda"))
    b0 = b.clone()
    M.dsmoe_bias_update(layer.handle, T, out["counts"], 1e-3, b)
    torch.cuda.synchronize()
    layer.close()
    fn, Pn = f.cpu().double().numpy(), P.cpu().double().numpy()
    assert losses[0].item() == pytest.approx(O.expert_balance_loss(fn, Pn, 0.003), rel=1e-6)
    fd, Pd, Ld = O.device_balance(fn, Pn, group_of.cpu().numpy(), groups, 0.05)
    np.testing.assert_allclose(f_dev.cpu().numpy(), fd, rtol=1e-6)
    np.testing.assert_allclose(P_dev.cpu().numpy(), Pd, rtol=1e-6, atol=1e-9)
    assert losses[1].item() == pytest.approx(Ld, rel=1e-6)
    idx = out["topk_idx"].cpu().numpy()
    sc = out["scores"].cpu().double().numpy()
    fs, ps, L = O.sequence_balance(idx, sc, seq_len, N, 1e-4)
    np.testing.assert_allclose(f_seq.cpu().numpy(), fs, rtol=1e-6)
    np.testing.assert_allclose(p_seq.cpu().numpy(), ps, rtol=1e-6, atol=1e-9)
    assert loss.item() == pytest.approx(L, rel=1e-6)
    nb = O.bias_update(b0.cpu().double().numpy(), out["counts"].cpu().numpy(), T, cfg.top_k, 1e-3)
    np.testing.assert_allclose(b.cpu().numpy(), nb, rtol=0, atol=1e-7)
