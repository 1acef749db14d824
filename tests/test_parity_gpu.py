"""Parity of the CUDA path (through the C ABI) with the float64 oracle on seeded inputs.

Small cases: every output checked, every row of h. Full-size cases (the sizes and
launch configuration the benchmark times): routing, counts, f, P over all tokens and
h on sampled rows (the layer is per-token independent, so a sampled row is exact).
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from tests import parity as PAR
from tests.gpu_cases import make_case, run_cuda, sample_rows

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)


def _check(cfg, T, rows_n=None, gen_device=None, seed=0, gemm_kernel=None):
    gpu, cpu = make_case(cfg, T, seed=seed, gen_device=gen_device)
    out = run_cuda(cfg, gpu, T, gemm_kernel=gemm_kernel)
    ref = PAR.reference_selection(cfg, cpu, out["topk_idx"], out["scores"])
    rr = PAR.check_routing(cfg, ref, out, T)
    rows = np.arange(T) if rows_n is None else sample_rows(T, rows_n)
    hh = PAR.check_h(cfg, cpu, ref, out, rows)
    print(cfg.name, T, rr, hh)
    return out, ref


SMALL = [("tiny", 512, None), ("tiny", 131, None), ("gshard_a", 1000, None), ("gshard_b", 1000, None),
         ("gshard_c", 1000, None), ("ds2b", 2000, None), ("v3_prefill", 300, 48), ("v4_decode_t16", 16, None),
         ("v4_decode_t64", 64, 32), ("v4_hash_t16", 16, None), ("v4_hash_t64", 64, None)]


@pytest.mark.parametrize("name,T,rows", SMALL, ids=[f"{n}-T{t}" for n, t, _ in SMALL])
def test_small_parity(name, T, rows):
    _check(W.get_config(name), T, rows)


PAIR = [("tiny", 131), ("gshard_c", 1000), ("v3_prefill", 300), ("v4_decode_t16", 16), ("ds2b", 2000)]


@pytest.mark.parametrize("name,T", PAIR, ids=[f"{n}-T{t}" for n, t in PAIR])
def test_small_parity_pair_gemm(name, T):
    """The CTA-pair grouped GEMM (the alternative to the default one-CTA kernel)."""
    _check(W.get_config(name), T, 48, gemm_kernel=M.DSMOE_GEMM_PAIR)


def test_gemm_kernels_agree():
    """The CTA-pair and one-CTA GEMM kernels on the same inputs: identical routing, and h
    identical too (both accumulate each output over K in the same 16-element MMA steps
    and share the epilogue arithmetic; measured bit-identical on B200)."""
    cfg = W.get_config("gshard_b").replace(T=1500)
    gpu, _ = make_case(cfg, cfg.T)
    a = run_cuda(cfg, gpu, cfg.T, gemm_kernel=M.DSMOE_GEMM_PAIR)
    b = run_cuda(cfg, gpu, cfg.T, gemm_kernel=M.DSMOE_GEMM_SINGLE)
    for k in ("topk_idx", "gates", "counts", "f", "P"):
        assert torch.equal(a[k], b[k]), k
    d = (a["h"].float() - b["h"].float()).abs()
    rms = b["h"].float().pow(2).mean().sqrt()
    print("pair vs single: bitwise equal rows", int((d.amax(1) == 0).sum()), "of", cfg.T,
          "max|diff|", float(d.max()), "rms", float(rms))
    assert float(d.max()) == 0.0


# (the V3 prefill and V4 decode T=256 layers at full size are in test_fullsize_stages_gpu.py)
FULL = [("gshard_a", 128), ("gshard_b", 128), ("gshard_c", 128), ("ds2b", 128), ("v4_hash_t256", 64)]


@pytest.mark.parametrize("name,rows", FULL, ids=[n for n, _ in FULL])
def test_full_size_parity(name, rows):
    cfg = W.get_config(name)
    _check(cfg, cfg.T, rows, gen_device="cuda")


def test_ragged_dims_and_two_shared():
    """d not a multiple of 256, F not a multiple of 128, N' not a multiple of 32, K_s=2 with F_s=64."""
    cfg = W.MoEConfig("ragged", T=333, d_model=320, n_routed=40, top_k=5, d_ff=192, n_shared=2,
                      d_ff_shared=64, score=W.SCORE_SIGMOID, renormalize=True, bias_mode=W.BIAS_SELECT_ONLY,
                      bias_kind="uniform0.1")
    _check(cfg, cfg.T)


def test_no_shared_softmax_renormalised_logit_bias():
    cfg = W.MoEConfig("nosh", T=257, d_model=128, n_routed=24, top_k=6, d_ff=64, score=W.SCORE_SOFTMAX,
                      renormalize=True, bias_mode=W.BIAS_IN_LOGITS, bias_kind="zipf")
    _check(cfg, cfg.T)


def test_all_tokens_pick_the_same_experts():
    """Identical expert centroids: every score ties, every token takes experts 0..K'-1, all
    other experts get no rows (empty groups) and a few get every token."""
    cfg = W.get_config("tiny").replace(T=300)
    gpu, cpu = make_case(cfg, cfg.T)
    gpu["W_router"][:] = gpu["W_router"][0:1]
    cpu["W_router"] = gpu["W_router"].cpu()
    out = run_cuda(cfg, gpu, cfg.T)
    assert (out["topk_idx"].cpu() == torch.arange(cfg.top_k, dtype=torch.int32)[None]).all()
    ref = PAR.reference_selection(cfg, cpu, out["topk_idx"], out["scores"])
    PAR.check_routing(cfg, ref, out, cfg.T)
    PAR.check_h(cfg, cpu, ref, out, np.arange(cfg.T))


def test_zero_tokens():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 4)
    layer = M.DSMoE(M.cfg_from(cfg, 16), gpu)
    out = layer.alloc_outputs(0)
    for k in ("counts", "f", "P", "P_sum"):
        out[k].fill_(7)
    M.dsmoe_forward(layer.handle, 0, gpu["x"], None, gpu["W_router"], None, gpu["W_gate"], gpu["W_up"],
                    gpu["W_down"], gpu["Ws_gate"], gpu["Ws_up"], gpu["Ws_down"], out["h"], out["topk_idx"],
                    out["gates"], out["counts"], out["f"], out["P"], out["P_sum"], None)
    torch.cuda.synchronize()
    for k in ("counts", "f", "P", "P_sum"):
        assert (out[k] == 0).all(), k
    layer.close()


def test_single_token_and_max_tokens():
    cfg = W.get_config("gshard_c")
    for T in (1, 128, 129):
        gpu, cpu = make_case(cfg, T, seed=T)
        out = run_cuda(cfg, gpu, T, max_tokens=T)  # T == max_tokens
        ref = PAR.reference_selection(cfg, cpu, out["topk_idx"], out["scores"])
        PAR.check_routing(cfg, ref, out, T)
        PAR.check_h(cfg, cpu, ref, out, np.arange(T))


def test_rejects_oversize_and_misaligned():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 64)
    layer = M.DSMoE(M.cfg_from(cfg, 32), gpu)
    with pytest.raises(M.DsmoeError) as ei:
        layer.forward(gpu["x"])  # T=64 > max_tokens=32
    assert ei.value.status == M.DSMOE_ERR_WORKSPACE
    x_mis = torch.empty(32 * 256 + 1, dtype=torch.bfloat16, device="cuda")[1:].view(32, 256)
    with pytest.raises(M.DsmoeError) as ei:
        layer.forward(x_mis)
    assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
    layer.close()


def test_repeatable_bitwise():
    """Two calls on one handle give bitwise-identical outputs (slot order inside an expert
    segment may differ between calls; the per-row results do not depend on it)."""
    cfg = W.get_config("gshard_c").replace(T=777)
    gpu, _ = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    a = layer.forward(gpu["x"], with_scores=True)
    b = layer.forward(gpu["x"], with_scores=True)
    torch.cuda.synchronize()
    for k in ("h", "topk_idx", "gates", "counts", "f", "P", "P_sum", "scores"):
        assert torch.equal(a[k], b[k]), k
    layer.close()


@pytest.mark.parametrize("name,T", [("ds2b", 700), ("gshard_b", 512)])
def test_forward_captured_in_a_cuda_graph(name, T):
    """The forward has no host synchronisation and no allocation, so it can be captured
    into a CUDA graph, side stream included (the shared experts' GEMMs fork from and join
    the capturing stream through events). A replay gives the eager forward's outputs bit
    for bit, and after new values are copied into the captured input buffer, a replay gives
    the eager forward of those values."""
    cfg = W.get_config(name).replace(T=T)
    gpu, _ = make_case(cfg, T)
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    x = gpu["x"].clone()
    x2 = W.normal_bf16((T, cfg.d_model), 1.0, 0, "x_graph", 1, "cuda")
    ref = {k: v.clone() for k, v in layer.forward(x).items() if v is not None}
    ref2 = {k: v.clone() for k, v in layer.forward(x2).items() if v is not None}
    out = layer.alloc_outputs(T)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm the capture stream
        layer.forward(x, out=out)
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        layer.forward(x, out=out)
    g.replay()
    torch.cuda.synchronize()
    assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK
    for k in ("h", "topk_idx", "gates", "counts", "f", "P"):
        assert torch.equal(out[k], ref[k]), k
    x.copy_(x2)
    g.replay()
    torch.cuda.synchronize()
    for k in ("h", "topk_idx", "gates", "counts", "f", "P"):
        assert torch.equal(out[k], ref2[k]), k
    del g
    layer.close()


def test_host_entry_point_matches_device_entry_point():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    d = layer.forward(gpu["x"])
    torch.cuda.synchronize()
    T, K, N = cfg.T, cfg.top_k, cfg.n_routed
    xh = gpu["x"].cpu().pin_memory()
    hh = torch.empty((T, cfg.d_model), dtype=torch.bfloat16).pin_memory()
    th = torch.empty((T, K), dtype=torch.int32).pin_memory()
    gh = torch.empty((T, K), dtype=torch.float32).pin_memory()
    ch = torch.empty((N,), dtype=torch.int32).pin_memory()
    fh = torch.empty((N,), dtype=torch.float32).pin_memory()
    ph = torch.empty((N,), dtype=torch.float32).pin_memory()
    M.dsmoe_forward_host(layer.handle, T, xh, None, gpu["W_router"], None, gpu["W_gate"], gpu["W_up"],
                         gpu["W_down"], gpu["Ws_gate"], gpu["Ws_up"], gpu["Ws_down"], hh, th, gh, ch, fh, ph)
    assert torch.equal(hh, d["h"].cpu()) and torch.equal(th, d["topk_idx"].cpu())
    assert torch.equal(gh, d["gates"].cpu()) and torch.equal(ch, d["counts"].cpu())
    assert torch.equal(fh, d["f"].cpu()) and torch.equal(ph, d["P"].cpu())
    # the pipelined entry point: three calls in flight through its two staging slots, with
    # different inputs, give each call's own results
    xs = [xh, (gpu["x"] * 0.5).cpu().pin_memory(), (gpu["x"] * 2.0).cpu().pin_memory()]
    outs = [tuple(torch.empty_like(t).pin_memory() for t in (hh, th, gh, ch, fh, ph)) for _ in xs]
    for xi, o in zip(xs, outs):
        M.dsmoe_forward_host_async(layer.handle, T, xi, None, gpu["W_router"], None, gpu["W_gate"], gpu["W_up"],
                                   gpu["W_down"], gpu["Ws_gate"], gpu["Ws_up"], gpu["Ws_down"], *o)
    M.dsmoe_host_sync(layer.handle)
    for xi, o in zip(xs, outs):
        ref = layer.forward(xi.cuda())
        torch.cuda.synchronize()
        for got, k in zip(o, ("h", "topk_idx", "gates", "counts", "f", "P")):
            assert torch.equal(got, ref[k].cpu()), k
    layer.close()


def test_balance_stats_entry_point():
    cfg = W.get_config("gshard_b").replace(T=600)
    gpu, _ = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    o = layer.forward(gpu["x"])
    f2 = torch.empty_like(o["f"])
    P2 = torch.empty_like(o["P"])
    M.dsmoe_balance_stats(layer.handle, cfg.T, o["counts"], o["P_sum"], f2, P2)
    torch.cuda.synchronize()
    assert torch.equal(f2, o["f"])
    assert torch.allclose(P2, o["P"], rtol=1e-6, atol=0)
    # shards: the statistics of two halves, reduced, equal those of the whole batch
    h1 = layer.forward(gpu["x"][:300].contiguous())
    c1, s1 = h1["counts"].clone(), h1["P_sum"].clone()
    h2 = layer.forward(gpu["x"][300:].contiguous())
    M.dsmoe_balance_stats(layer.handle, cfg.T, c1 + h2["counts"], s1 + h2["P_sum"], f2, P2)
    torch.cuda.synchronize()
    assert torch.equal(c1 + h2["counts"], o["counts"])
    assert torch.equal(f2, o["f"])
    assert torch.allclose(P2, o["P"], rtol=1e-5, atol=1e-7)
    layer.close()


def test_gemm_kernel_selector():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, 8)
    layer = M.DSMoE(M.cfg_from(cfg, 8), gpu)
    assert M.dsmoe_get_gemm_kernel(layer.handle) == M.DSMOE_GEMM_SINGLE  # the default
    M.dsmoe_set_gemm_kernel(layer.handle, M.DSMOE_GEMM_PAIR)
    assert M.dsmoe_get_gemm_kernel(layer.handle) == M.DSMOE_GEMM_PAIR
    with pytest.raises(M.DsmoeError) as ei:
        M.dsmoe_set_gemm_kernel(layer.handle, 7)
    assert ei.value.status == M.DSMOE_ERR_INVALID_ARG
    layer.close()


def test_stage_timing_and_launch_count():
    cfg = W.get_config("tiny")
    gpu, _ = make_case(cfg, cfg.T)
    layer = M.DSMoE(M.cfg_from(cfg, cfg.T), gpu)
    n0 = M.dsmoe_launch_count(layer.handle)
    M.dsmoe_set_timing(layer.handle, True)
    layer.forward(gpu["x"])
    t = M.dsmoe_stage_times(layer.handle)
    assert list(t) == M.stage_names() and all(v >= 0 for v in t.values())
    # router logits (tensor cores for T >= 256), select, scan, permute, the routed experts'
    # two GEMMs, combine; and the shared experts' two GEMMs on the side stream
    n_launch = 7 + (2 if cfg.n_shared else 0)
    assert M.dsmoe_launch_count(layer.handle) - n0 == n_launch
    M.dsmoe_set_timing(layer.handle, False)
    n1 = M.dsmoe_launch_count(layer.handle)
    layer.forward(gpu["x"][:100].contiguous())  # CUDA-core router logits below 256 tokens
    assert M.dsmoe_launch_count(layer.handle) - n1 == n_launch
    layer.close()


def test_varying_batch_sizes_on_one_handle():
    """One handle serving batches of different sizes (both routers, several split counts)
    gives the same outputs as a fresh handle per batch: no state of an earlier call leaks
    into a later one."""
    cfg = W.get_config("ds2b")
    gpu, _ = make_case(cfg, 2000)
    layer = M.DSMoE(M.cfg_from(cfg, 2000), gpu)
    for T in (2000, 100, 700, 16, 300, 2000):
        x = gpu["x"][:T].contiguous()
        a = layer.forward(x, with_scores=True)
        torch.cuda.synchronize()
        fresh = M.DSMoE(M.cfg_from(cfg, T), gpu)
        b = fresh.forward(x, with_scores=True)
        torch.cuda.synchronize()
        fresh.close()
        for k in ("h", "topk_idx", "gates", "counts", "f", "scores"):
            assert torch.equal(a[k], b[k]), (T, k)
    layer.close()
