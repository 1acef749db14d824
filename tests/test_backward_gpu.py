"""The first backward kernels against the float64 backward oracle (oracle/dsmoe_backward.py,
pinned there by finite differences, float64 autograd and closed forms): for an upstream
gradient dh, the gate gradients dg = <dh, y>, the routed experts' output gradient
g dh in slot order, and the router's backward with the expert-level balance term
(DeepSeekMoE summary, "Expert-level balance loss": P_i carries the gradient).

Bounds (max |err| / RMS(ref)):
* dg against the oracle: 2e-2 (the kernel dots dh with the forward's expert rows, which
  carry one bf16 rounding of A1 and of Y, 2^-8 relative together, the oracle with the
  exact float64 FFN outputs; the max over many tokens of a Gaussian error runs ~4x the
  RMS);
* dlogits, dx and dW_router against the oracle fed the kernel's own dg: 1e-4 (fp32
  arithmetic on fp32 scores): this is the router backward's own precision;
* dlogits against the oracle end to end: 0.1, a gross-error check only: the gate
  renormalisation (dg_k minus the gate-weighted mean of dg) and the softmax centring
  subtract nearly equal numbers, which multiplies dg's relative error;
* dY rows equal bf16(g * dh) exactly (one fp32 product, rounded to nearest even)."""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from oracle import dsmoe_backward as DB
from tests import parity as PAR
from tests.gpu_cases import make_case

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)

# (workload, T, alpha of the balance term, mask_top, k_active or None). tiny, gshard_b,
# v3_prefill and ds2b (N' a multiple of 64, T >= 256 and T >= 2 N') take the router
# backward's tensor-core path; v4_decode_t16 and gshard_c its CUDA-core path.
CASES = [("tiny", 300, 0.01, 0, None), ("gshard_b", 1000, 0.01, 0, None), ("v3_prefill", 520, 0.003, 0, None),
         ("v4_decode_t16", 16, 0.0, 0, None), ("ds2b", 700, 0.01, 0, None), ("gshard_c", 500, 0.02, 2, 5)]


def _rel(got, ref):
    return float(np.abs(np.asarray(got, dtype=np.float64) - ref).max() / max(np.sqrt(np.mean(ref ** 2)), 1e-30))


def _rel_fro_per_expert(got, ref):
    """max over the leading (expert) axis of ||got_e - ref_e||_F / ||ref_e||_F."""
    err = np.asarray(got, dtype=np.float64) - ref
    num = np.sqrt((err ** 2).reshape(err.shape[0], -1).sum(axis=1))
    den = np.sqrt((ref ** 2).reshape(ref.shape[0], -1).sum(axis=1))
    return float((num / np.maximum(den, 1e-30)).max())


@pytest.mark.parametrize("name,T,alpha,mask,k", CASES, ids=[f"{c[0]}-T{c[1]}" + (f"-m{c[3]}k{c[4]}" if c[3] else "")
                                                           for c in CASES])
def test_gate_and_router_backward(name, T, alpha, mask, k):
    cfg = W.get_config(name)
    gpu, cpu = make_case(cfg, T)
    dh = W.normal_bf16((T, cfg.d_model), 1.0, 0, "dh", 0, "cuda")
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    try:
        if mask or k:
            layer.set_selection(mask, k or cfg.top_k)
        K = layer.k_active
        out = layer.forward(gpu["x"], with_scores=True)
        dg = torch.empty((T, K), dtype=torch.float32, device="cuda")
        dY = torch.empty((T * K, cfg.d_model), dtype=torch.bfloat16, device="cuda")
        M.dsmoe_backward_gates(layer.handle, T, dh, out["gates"], dg, dY)
        slot = M.workspace_view(layer.handle, "slot_of")[:T, :K].clone()
        dl = torch.empty((T, cfg.n_routed), dtype=torch.float32, device="cuda")
        dx = torch.empty((T, cfg.d_model), dtype=torch.float32, device="cuda")
        dWr = torch.empty((cfg.n_routed, cfg.d_model), dtype=torch.float32, device="cuda")
        M.dsmoe_backward_router(layer.handle, T, gpu["x"], gpu["W_router"], out["topk_idx"], out["gates"],
                                out["scores"], dg, out["f"], alpha, dl, dx, dWr)
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK, M.dsmoe_last_error()
    finally:
        layer.close()
    cfg_v = cfg.replace(top_k=K, mask_top=mask)
    ref = PAR.reference_selection(cfg_v, cpu, out["topk_idx"], out["scores"])
    PAR.check_routing(cfg_v, ref, out, T)
    # dY: g * dh in the slot of each pick, exactly
    want = (out["gates"][:, :, None] * dh.float()[:, None, :]).to(torch.bfloat16)
    got = dY[slot.view(-1).long()].view(T, K, cfg.d_model)
    assert torch.equal(got, want)
    dh64 = dh.float().cpu().numpy().astype(np.float64)
    # dg against the oracle (exact float64 expert outputs)
    dg_ref = DB.gate_grads(cpu, ref["idx"], dh64)
    e_dg = _rel(dg.cpu().numpy(), dg_ref)
    # the router's backward fed the kernel's own dg, and end to end
    routing = dict(ref, f=out["f"].cpu().numpy().astype(np.float64))
    dl_k, dx_k, dW_k = DB.router_grads(cfg_v, routing, cpu["x"], cpu["W_router"], dg.cpu().numpy().astype(np.float64),
                                       alpha)
    e_dl = _rel(dl.cpu().numpy(), dl_k)
    dl64 = dl.cpu().numpy().astype(np.float64)
    x64 = cpu["x"].float().numpy().astype(np.float64)
    Wr64 = cpu["W_router"].float().numpy().astype(np.float64)
    e_dx = _rel(dx.cpu().numpy(), dl64 @ Wr64)
    e_dW = _rel(dWr.cpu().numpy(), dl64.T @ x64)
    dl_ref, _, _ = DB.router_grads(cfg_v, routing, cpu["x"], cpu["W_router"], dg_ref, alpha)
    e_dl_e2e = _rel(dl.cpu().numpy(), dl_ref)
    for k_ in ("W_gate", "W_up", "W_down"):
        if hasattr(cpu[k_], "cache"):
            cpu[k_].cache.clear()
    print(name, T, dict(dg=e_dg, dl=e_dl, dx=e_dx, dW=e_dW, dl_e2e=e_dl_e2e))
    assert e_dl <= 1e-4 and e_dx <= 1e-4 and e_dW <= 1e-4
    assert e_dg <= 2e-2 and e_dl_e2e <= 0.1


def test_backward_argument_errors():
    cfg = W.get_config("v4_hash_t16")
    gpu, _ = make_case(cfg, 16)
    layer = M.DSMoE(M.cfg_from(cfg, 16), gpu)
    try:
        with pytest.raises(M.DsmoeError) as ei:
            M.dsmoe_backward_router(layer.handle, 16, gpu["x"], None, None, None, None, None, None, 0.0, None, None,
                                    torch.empty(1, device="cuda"))
        assert ei.value.status == M.DSMOE_ERR_UNSUPPORTED
        with pytest.raises(M.DsmoeError) as ei:
            M.dsmoe_backward_gates(layer.handle, 17, None, None, None, None)
        assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
    finally:
        layer.close()


EXP_CASES = [("tiny", 300), ("gshard_c", 500), ("ds2b", 700), ("v3_slice", 256), ("tiny", 37)]


@pytest.mark.parametrize("name,T", EXP_CASES, ids=[f"{c[0]}-T{c[1]}" for c in EXP_CASES])
def test_expert_backward_input_gradient(name, T):
    """Weight gradients dW_gate, dW_up, dW_down of every routed and shared expert
    (dsmoe_backward_weights: ragged token reductions on the tensor cores) against the
    oracle's layer_backward, expert by expert: ||err||_F / ||ref||_F <= 1e-2 (the bf16
    operands below, each rounded once, give a few 2^-9 per rank-1 term; a token missing
    from or added to an expert's K range moves it by about 1/sqrt(rows)), and an unpicked
    expert's gradient exactly zero. (max |err| / RMS is no bound here: an expert that few
    tokens picked has a gradient of a few outer products, whose largest element is tens of
    times its RMS.) And
    dL/du through the experts (dsmoe_backward_experts: W_down^T dy -> SiLU backward with
    the saved pre-activations -> W_gate^T da + W_up^T db on the tensor cores, weights read
    MN-major) plus the router's part, against the oracle's layer_backward dx (float64):
    max |err| / RMS <= 3e-2 (bf16 operands: g dh, the saved a and b, da | db and the
    per-slot rows, each rounded once; fp32 accumulation). The shared experts' fp32 sum dXs
    is checked on its own against the oracle's SwiGLU backward within 2e-2."""
    cfg = W.get_config(name)
    gpu, cpu = make_case(cfg, T)
    dh = W.normal_bf16((T, cfg.d_model), 1.0, 0, "dh", 0, "cuda")
    alpha = 0.01
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    try:
        M.dsmoe_set_training(layer.handle, True)
        out = layer.forward(gpu["x"], with_scores=True)
        K, N, d = cfg.top_k, cfg.n_routed, cfg.d_model
        dg = torch.empty((T, K), dtype=torch.float32, device="cuda")
        dY = torch.empty((T * K, d), dtype=torch.bfloat16, device="cuda")
        M.dsmoe_backward_gates(layer.handle, T, dh, out["gates"], dg, dY)
        dl = torch.empty((T, N), dtype=torch.float32, device="cuda")
        dx_r = torch.empty((T, d), dtype=torch.float32, device="cuda")
        dWr = torch.empty((N, d), dtype=torch.float32, device="cuda")
        M.dsmoe_backward_router(layer.handle, T, gpu["x"], gpu["W_router"], out["topk_idx"], out["gates"],
                                out["scores"], dg, out["f"], alpha, dl, dx_r, dWr)
        dx = torch.empty((T, d), dtype=torch.float32, device="cuda")
        M.dsmoe_backward_experts(layer.handle, T, dh, dY, gpu["W_gate"], gpu["W_up"], gpu["W_down"],
                                 gpu.get("Ws_gate"), gpu.get("Ws_up"), gpu.get("Ws_down"), dx_r, dx)
        F, Ks, Fs = cfg.d_ff, cfg.n_shared, cfg.d_ff_shared
        dW = {k: torch.full(shp, float("nan"), device="cuda") for k, shp in (
            ("dW_gate", (N, F, d)), ("dW_up", (N, F, d)), ("dW_down", (N, d, F)))}
        dWs = {k: (torch.full(shp, float("nan"), device="cuda") if Ks else None) for k, shp in (
            ("dWs_gate", (Ks, Fs, d)), ("dWs_up", (Ks, Fs, d)), ("dWs_down", (Ks, d, Fs)))}
        M.dsmoe_backward_weights(layer.handle, T, dh, dY, gpu["x"], dW["dW_gate"], dW["dW_up"], dW["dW_down"],
                                 dWs["dWs_gate"], dWs["dWs_up"], dWs["dWs_down"])
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK, M.dsmoe_last_error()
        dxs = M.workspace_view(layer.handle, "dXs")[:T].clone() if cfg.n_shared else None
        M.dsmoe_set_training(layer.handle, False)
    finally:
        layer.close()
    ref = PAR.reference_selection(cfg, cpu, out["topk_idx"], out["scores"])
    PAR.check_routing(cfg, ref, out, T)
    dh64 = dh.float().cpu().numpy().astype(np.float64)
    bw = DB.layer_backward(cfg, cpu, dh64, routing=ref, alpha_bal=alpha)
    e_dx = _rel(dx.cpu().numpy(), bw["dx"])
    e_s = 0.0
    if cfg.n_shared:
        X = cpu["x"].float().numpy().astype(np.float64)
        ref_s = np.zeros_like(X)
        for i in range(cfg.n_shared):
            ref_s += DB.swiglu_backward(X, cpu["Ws_gate"][i], cpu["Ws_up"][i], cpu["Ws_down"][i], dh64)[0]
        e_s = _rel(dxs.cpu().numpy(), ref_s)
    # weight gradients: every expert (one no token picked is exactly zero), per matrix
    used = np.unique(ref["idx"])
    e_w = {}
    for k in ("dW_gate", "dW_up", "dW_down"):
        got = dW[k]
        unused = torch.ones(N, dtype=torch.bool)
        unused[torch.as_tensor(used)] = False
        if bool(unused.any()):
            assert bool((got[unused.cuda()] == 0).all()), f"{k}: an unused expert's gradient is not zero"
        e_w[k] = _rel_fro_per_expert(got[torch.as_tensor(used).cuda()].cpu().numpy(), bw[k][used])
    if Ks:
        for k in ("dWs_gate", "dWs_up", "dWs_down"):
            e_w[k] = _rel_fro_per_expert(dWs[k].cpu().numpy(), bw[k])
    for k_ in ("W_gate", "W_up", "W_down"):
        if hasattr(cpu[k_], "cache"):
            cpu[k_].cache.clear()
    print(name, T, "dx err/RMS", e_dx, "shared du err/RMS", e_s, "dW err/RMS", e_w)
    assert e_dx <= 3e-2 and e_s <= 2e-2
    assert all(v <= 1e-2 for v in e_w.values()), e_w


def test_expert_backward_needs_a_training_forward():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 64)
    layer = M.DSMoE(M.cfg_from(cfg, 64), gpu)
    try:
        dh = torch.zeros((64, cfg.d_model), dtype=torch.bfloat16, device="cuda")
        dY = torch.zeros((64 * cfg.top_k, cfg.d_model), dtype=torch.bfloat16, device="cuda")
        dx = torch.empty((64, cfg.d_model), dtype=torch.float32, device="cuda")
        args = (dh, dY, gpu["W_gate"], gpu["W_up"], gpu["W_down"], gpu["Ws_gate"], gpu["Ws_up"], gpu["Ws_down"], None,
                dx)
        with pytest.raises(M.DsmoeError):  # training buffers not enabled
            M.dsmoe_backward_experts(layer.handle, 64, *args)
        M.dsmoe_set_training(layer.handle, True)
        with pytest.raises(M.DsmoeError):  # no training forward yet
            M.dsmoe_backward_experts(layer.handle, 64, *args)
        layer.forward(gpu["x"])
        with pytest.raises(M.DsmoeError):  # a different T than the forward's
            M.dsmoe_backward_experts(layer.handle, 32, *args)
        M.dsmoe_backward_experts(layer.handle, 64, *args)
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK
        assert torch.equal(dx, dh.float())  # dh = 0: every part of the gradient is 0 but the residual's
    finally:
        layer.close()
