"""Helpers for the GPU tests: build a case's inputs on the CPU or the GPU, run the CUDA
path through the C ABI, and hand the oracle CPU views of the same bytes."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W

WEIGHT_KEYS = ("W_gate", "W_up", "W_down", "Ws_gate", "Ws_up", "Ws_down")


class LazyExperts:
    """Per-expert CPU copies of a device weight tensor, fetched on first use."""

    def __init__(self, t: torch.Tensor):
        self.t = t
        self.cache = {}

    def __getitem__(self, e):
        e = int(e)
        if e not in self.cache:
            self.cache[e] = self.t[e].cpu()
        return self.cache[e]

    def __len__(self):
        return self.t.shape[0]


# Layers whose expert weights exceed this are drawn on the GPU (the oracle then copies
# only the experts it needs); drawing 20-35 GB of V3/V4-shaped weights with the CPU
# generator takes over a minute per case.
GPU_DRAW_BYTES = 1 << 30


def make_case(cfg: W.MoEConfig, T: int, seed: int = 0, gen_device: str = None):
    """Inputs drawn on gen_device (default: the GPU for layers whose weights exceed
    GPU_DRAW_BYTES, else the CPU); returns (inputs on cuda:0, CPU view for the oracle)."""
    if gen_device is None:
        big = cfg.routed_weight_bytes() + cfg.shared_weight_bytes() > GPU_DRAW_BYTES
        gen_device = "cuda" if big else "cpu"
    inp = W.make_inputs(cfg, seed=seed, device=gen_device, T=T)
    gpu, cpu = {}, {}
    for k, v in inp.items():
        if v is None:
            gpu[k] = cpu[k] = None
            continue
        gpu[k] = v.to("cuda:0").contiguous()
        if k in WEIGHT_KEYS:
            cpu[k] = v if gen_device == "cpu" else LazyExperts(gpu[k])
        else:
            cpu[k] = v.cpu()
    return gpu, cpu


def run_cuda(cfg: W.MoEConfig, gpu: dict, T: int, max_tokens: int = None, with_scores: bool = True,
             gemm_kernel: int = None):
    layer = M.DSMoE(M.cfg_from(cfg, max_tokens or max(T, 1)), gpu)
    try:
        if gemm_kernel is not None:
            M.dsmoe_set_gemm_kernel(layer.handle, gemm_kernel)
        out = layer.forward(gpu["x"], token_ids=gpu.get("token_ids"), with_scores=with_scores)
        torch.cuda.synchronize()
        st = M.dsmoe_get_status(layer.handle)
        assert st == M.DSMOE_OK, M.dsmoe_last_error()
    finally:
        layer.close()
    return out


def sample_rows(T: int, n: int, seed: int = 1):
    if T <= n:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    rows = rng.choice(T, size=n, replace=False)
    rows[0], rows[-1] = 0, T - 1  # include both ends
    return np.sort(rows)
