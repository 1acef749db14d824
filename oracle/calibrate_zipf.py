"""Pick the scale of the 2B-shaped workload's Zipf(1.1) logit bias.

The workload asks for router logits given a Zipf(1.1) per-expert bias so that
expert loads are skewed about 10:1. The bias is c_i = -lam * 1.1 * ln(i+1);
this script bisects lam until the oracle's max/min expert count at seed 0
lies in [9.5, 10.5], and prints it. The value is stored as
workloads.DS2B_ZIPF_LAMBDA. Test infrastructure: calls only the oracle and
the seeded generators.

    python -m oracle.calibrate_zipf
"""
from __future__ import annotations

import numpy as np

import workloads as W
from oracle import dsmoe_oracle as O


def load_ratio(lam: float, seed: int = 0) -> float:
    cfg = W.get_config("ds2b")
    inp = W.make_inputs(cfg, seed=seed, with_weights=False)
    b = W.zipf_logit_bias(cfg.n_routed, lam)
    l = O.router_logits(inp["x"], inp["W_router"], b.numpy(), O.BIAS_IN_LOGITS)
    s = O.scores(l, cfg.score)
    idx, _ = O.select_topk(s, cfg.top_k)
    counts, _, _ = O.balance_stats(idx, s, cfg.n_routed, cfg.top_k)
    return counts.max() / max(counts.min(), 1)


def calibrate(lo: float = 0.0, hi: float = 2.0, target: float = 10.0, steps: int = 12) -> float:
    for _ in range(steps):
        mid = (lo + hi) / 2
        if load_ratio(mid) < target:
            lo = mid
        else:
            hi = mid
    return (lo + hi) / 2


if __name__ == "__main__":
    lam = calibrate()
    print(f"lambda={lam!r} ratio={load_ratio(lam):.3f}")
