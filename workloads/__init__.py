"""Seeded synthetic workloads for the DeepSeekMoE layer forward.

This module only draws random numbers and names shapes. It holds none of the
layer's arithmetic, so both the CUDA path and the oracle can consume the very
same bytes without sharing any code with each other.

Shapes follow the configurations the DeepSeekMoE pages describe:

* ``tiny``: m=4 segmentation of N=16 experts (64 routed, top-7) plus one
  shared expert, softmax gates not renormalised (DeepSeekMoE expert
  specialization page, "Fine-Grained Expert Segmentation" gate equation).
* ``gshard_a/b/c``: the equal-FLOPs GShard / fine-grained / fine-grained +
  shared triple (same page, segmentation and shared-expert equations; the
  interview card's FLOPs identity k'(2 d d_ff / m) = k (2 d d_ff)).
* ``ds2b``: the 2B validation model's hidden size 1280 with 2 shared + 64
  routed experts, top-6, and a Zipf per-expert logit bias for a ~10:1 load skew.
* ``v3_prefill``: 256 routed + 1 shared, top-8, sigmoid scores with a
  selection-only bias, renormalised gates (V4 book ch. 2, section 2 and 3).
* ``v3_slice``: the V3 layer's shapes with 32 routed experts and T=1024 (the same
  256 rows per expert on average), a small case for profiler captures.
* ``v4_decode_t{16,64,256}``: 384 routed + 1 shared, top-9, sqrt(softplus)
  scores (V4 book ch. 2, section 2 equation) with a selection-only bias.
* ``v4_hash_t{16,64,256}``: hash-routed layer (V4 book ch. 2, section 5),
  expert = token_id * 2654435761 mod 384.
* ``v4_decode_slice``: the V4 decode shapes (T=16) with 48 routed experts, a small case
  for profiler captures of the weight-streaming GEMMs.

Values: x ~ N(0,1); expert weights ~ N(0, 1/fan_in); router weights
~ N(0, 1/d) unless the configuration fixes N(0, 0.02^2); bias ~ U(-0.1, 0.1).
Each tensor (and each expert's slice of an expert tensor) has its own
generator seed, derived from (seed, name, index), so any slice can be drawn on
its own. Values are drawn in fp32 by torch's generator for the requested
device and rounded to bf16 (round-to-nearest-even).
"""
from __future__ import annotations

import dataclasses
import hashlib
import math
from typing import Dict, Optional

import torch

SCORE_SOFTMAX, SCORE_SIGMOID, SCORE_SQRT_SOFTPLUS, ROUTE_HASH = 0, 1, 2, 3
BIAS_NONE, BIAS_SELECT_ONLY, BIAS_IN_LOGITS = 0, 1, 2

HASH_MULT = 2654435761
TOKEN_VOCAB = 129280

# Scale of the Zipf(1.1) logit bias of the 2B-shaped workload: c_i = -lam * 1.1 * ln(i+1).
# Chosen by oracle/calibrate_zipf.py so that the oracle's max/min expert load
# ratio at seed 0 is about 10:1.
DS2B_ZIPF_LAMBDA = 0.316162109375


@dataclasses.dataclass(frozen=True)
class MoEConfig:
    name: str
    T: int                 # tokens
    d_model: int           # d
    n_routed: int          # N'
    top_k: int             # K'
    d_ff: int              # routed expert intermediate size F
    n_shared: int = 0      # K_s
    d_ff_shared: int = 0   # F_s
    score: int = SCORE_SOFTMAX
    renormalize: bool = False
    bias_mode: int = BIAS_NONE
    bias_kind: str = "none"          # "none" | "uniform0.1" | "zipf"
    router_std: Optional[float] = None  # None -> 1/sqrt(d)
    hash_mult: int = HASH_MULT
    mask_top: int = 0      # experts masked before the top-K' choice (inference analysis variant)

    @property
    def slots(self) -> int:
        return self.T * self.top_k

    def expert_flops_per_token(self) -> int:
        """Multiply-add FLOPs of the SwiGLU experts one token activates (3 matrices)."""
        return 6 * self.d_model * (self.top_k * self.d_ff + self.n_shared * self.d_ff_shared)

    def router_flops_per_token(self) -> int:
        return 0 if self.score == ROUTE_HASH else 2 * self.d_model * self.n_routed

    def flops_per_token(self) -> int:
        return self.expert_flops_per_token() + self.router_flops_per_token()

    def routed_weight_bytes(self) -> int:
        return self.n_routed * 3 * self.d_model * self.d_ff * 2

    def shared_weight_bytes(self) -> int:
        return self.n_shared * 3 * self.d_model * self.d_ff_shared * 2

    def expert_bytes(self) -> int:
        return 3 * self.d_model * self.d_ff * 2

    def replace(self, **kw) -> "MoEConfig":
        return dataclasses.replace(self, **kw)


def _cfgs():
    c = {}
    c["tiny"] = MoEConfig("tiny", T=512, d_model=256, n_routed=64, top_k=7, d_ff=128,
                          n_shared=1, d_ff_shared=128)
    common2 = dict(T=4096, d_model=1024, router_std=0.02)
    c["gshard_a"] = MoEConfig("gshard_a", n_routed=16, top_k=2, d_ff=2816, **common2)
    c["gshard_b"] = MoEConfig("gshard_b", n_routed=64, top_k=8, d_ff=704, **common2)
    c["gshard_c"] = MoEConfig("gshard_c", n_routed=63, top_k=7, d_ff=704, n_shared=1,
                              d_ff_shared=704, **common2)
    c["ds2b"] = MoEConfig("ds2b", T=16384, d_model=1280, n_routed=64, top_k=6, d_ff=896,
                          n_shared=2, d_ff_shared=896, bias_mode=BIAS_IN_LOGITS, bias_kind="zipf")
    c["v3_prefill"] = MoEConfig("v3_prefill", T=8192, d_model=7168, n_routed=256, top_k=8,
                                d_ff=2048, n_shared=1, d_ff_shared=2048, score=SCORE_SIGMOID,
                                renormalize=True, bias_mode=BIAS_SELECT_ONLY,
                                bias_kind="uniform0.1")
    # the V3 layer's matrix shapes and rows per expert (T K' / N' = 256) with 1/8 of its
    # experts: small enough for profiler captures, weights still far above L2
    c["v3_slice"] = c["v3_prefill"].replace(name="v3_slice", T=1024, n_routed=32)
    for t in (16, 64, 256):
        c[f"v4_decode_t{t}"] = MoEConfig(f"v4_decode_t{t}", T=t, d_model=7168, n_routed=384,
                                         top_k=9, d_ff=2048, n_shared=1, d_ff_shared=2048,
                                         score=SCORE_SQRT_SOFTPLUS, renormalize=True,
                                         bias_mode=BIAS_SELECT_ONLY, bias_kind="uniform0.1")
        c[f"v4_hash_t{t}"] = MoEConfig(f"v4_hash_t{t}", T=t, d_model=7168, n_routed=384,
                                       top_k=1, d_ff=2048, n_shared=1, d_ff_shared=2048,
                                       score=ROUTE_HASH)
    # the V4 decode layer's matrix shapes with 48 of its routed experts (4.3 GB of weights):
    # a small case for profiler captures of the weight-streaming GEMMs
    c["v4_decode_slice"] = c["v4_decode_t16"].replace(name="v4_decode_slice", n_routed=48)
    return c


CONFIGS: Dict[str, MoEConfig] = _cfgs()


def get_config(name: str) -> MoEConfig:
    return CONFIGS[name]


# --------------------------------------------------------------------------------------
# seeded draws
# --------------------------------------------------------------------------------------
def derive_seed(seed: int, name: str, index: int = 0) -> int:
    h = hashlib.sha256(f"dsmoe/{seed}/{name}/{index}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _generator(device, seed: int, name: str, index: int = 0) -> torch.Generator:
    g = torch.Generator(device=torch.device(device))
    g.manual_seed(derive_seed(seed, name, index))
    return g


def normal_bf16(shape, std: float, seed: int, name: str, index: int = 0, device="cpu") -> torch.Tensor:
    g = _generator(device, seed, name, index)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        v.mul_(std)
    return v.to(torch.bfloat16)


def uniform_f32(shape, lo: float, hi: float, seed: int, name: str, device="cpu") -> torch.Tensor:
    g = _generator(device, seed, name)
    v = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    return v.mul_(hi - lo).add_(lo)


def zipf_logit_bias(n: int, lam: float = DS2B_ZIPF_LAMBDA, exponent: float = 1.1) -> torch.Tensor:
    """Per-expert Zipf(1.1) logit bias c_i = -lam * exponent * ln(i+1); expert 0 is the hottest."""
    i = torch.arange(n, dtype=torch.float64)
    return (-lam * exponent * torch.log1p(i)).to(torch.float32)


def expert_matrix(cfg: MoEConfig, which: str, e: int, seed: int = 0, device="cpu") -> torch.Tensor:
    """One expert's weight matrix, nn.Linear layout [out, in], bf16.

    which: 'W_gate' | 'W_up' | 'W_down' (routed expert e) or
           'Ws_gate' | 'Ws_up' | 'Ws_down' (shared expert e).
    """
    shared = which.startswith("Ws")
    F = cfg.d_ff_shared if shared else cfg.d_ff
    d = cfg.d_model
    if which.endswith("down"):
        shape, fan_in = (d, F), F
    else:
        shape, fan_in = (F, d), d
    return normal_bf16(shape, 1.0 / math.sqrt(fan_in), seed, which, e, device)


def make_inputs(cfg: MoEConfig, seed: int = 0, device="cpu", T: Optional[int] = None,
                with_weights: bool = True) -> Dict[str, torch.Tensor]:
    """All inputs of one layer forward, drawn on ``device``.

    Returns x [T,d] bf16, W_router [N',d] bf16 (absent for hash routing),
    b [N'] fp32 or None, token_ids [T] int32 (hash routing only), and the
    expert weights W_gate/W_up [N',F,d], W_down [N',d,F], Ws_gate/Ws_up
    [K_s,F_s,d], Ws_down [K_s,d,F_s], all bf16.
    """
    T = cfg.T if T is None else T
    d, N = cfg.d_model, cfg.n_routed
    out: Dict[str, torch.Tensor] = {}
    out["x"] = normal_bf16((T, d), 1.0, seed, "x", 0, device)
    if cfg.score == ROUTE_HASH:
        g = _generator(device, seed, "token_ids")
        out["token_ids"] = torch.randint(0, TOKEN_VOCAB, (T,), generator=g, device=device,
                                         dtype=torch.int64).to(torch.int32)
        out["W_router"] = None
        out["b"] = None
    else:
        std = cfg.router_std if cfg.router_std is not None else 1.0 / math.sqrt(d)
        out["W_router"] = normal_bf16((N, d), std, seed, "W_router", 0, device)
        out["token_ids"] = None
        if cfg.bias_kind == "uniform0.1":
            out["b"] = uniform_f32((N,), -0.1, 0.1, seed, "b", device)
        elif cfg.bias_kind == "zipf":
            out["b"] = zipf_logit_bias(N).to(device)
        else:
            out["b"] = None
    if with_weights:
        F, Ks, Fs = cfg.d_ff, cfg.n_shared, cfg.d_ff_shared
        for which, n_exp, shp in (("W_gate", N, (F, d)), ("W_up", N, (F, d)), ("W_down", N, (d, F)),
                                  ("Ws_gate", Ks, (Fs, d)), ("Ws_up", Ks, (Fs, d)),
                                  ("Ws_down", Ks, (d, Fs))):
            w = torch.empty((n_exp,) + shp, dtype=torch.bfloat16, device=device)
            for e in range(n_exp):
                w[e] = expert_matrix(cfg, which, e, seed, device)
            out[which] = w
    return out


def bf16_bits(t: torch.Tensor):
    """The raw uint16 bit patterns of a bf16 tensor, as a numpy array (CPU copy)."""
    import numpy as np
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
