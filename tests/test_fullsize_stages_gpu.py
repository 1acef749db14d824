"""The grouped GEMMs at full size, element by element, in the launch configuration the
benchmark times (V3-shaped prefill: T=8192, d=7168, 256 routed + 1 shared experts of
d_ff=2048, top-8; V4-shaped decode: T=256, 384 routed + 1 shared, top-9).

Routing and the balance statistics are checked over every token, h on 256 sampled rows
(the layer equation is per token, so a sampled row is exact), and the intermediate
results of the two grouped GEMMs for every slot of whole experts: A1 = SiLU(X W_gate^T)
* (X W_up^T) from the gathered rows Xp, and Y = A1 W_down^T from the kernel's own A1
(DeepSeekMoE summary, shared-expert layer equation). The experts checked are the
highest-numbered ones that received rows, whose tiles the persistent kernels reach
last (late ring phases and accumulator reuse in many CTAs), and the most loaded one;
the shared expert's A1s and the fp32 residual + shared rows Hs are checked on the
sampled token rows, the last rows included (its last tiles). Bounds are those of the
small per-stage tests: A1 and Y within 2^-8 |ref| + 1e-4 RMS(ref), Hs within 1e-4 RMS.
"""
import numpy as np
import pytest
import torch

import mixture_experts_layer_score_b200 as M
import workloads as W
from oracle import dsmoe_oracle as O
from tests import parity as PAR
from tests.gpu_cases import make_case, sample_rows

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("no GPU", allow_module_level=True)

CASES = [("v3_prefill", 8, 256), ("v4_decode_t256", 24, 256)]


def _excess(got, ref):
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.sqrt(np.mean(ref ** 2))
    return float((np.abs(got - ref) / bound).max())


@pytest.mark.parametrize("name,n_experts,n_rows", CASES, ids=[c[0] for c in CASES])
def test_full_size_stages_and_parity(name, n_experts, n_rows):
    cfg = W.get_config(name)
    T = cfg.T
    gpu, cpu = make_case(cfg, T)  # drawn on the GPU; the oracle fetches the experts it needs
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    try:
        out = layer.forward(gpu["x"], with_scores=True)
        torch.cuda.synchronize()
        assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK, M.dsmoe_last_error()
        counts = out["counts"].cpu().numpy().astype(np.int64)
        offs = M.workspace_view(layer.handle, "offsets")[0].cpu().numpy().astype(np.int64)
        assert (offs == np.concatenate([[0], np.cumsum(counts)])).all()
        used = np.nonzero(counts)[0]
        pick = list(used[-(n_experts - 1):]) + [int(np.argmax(counts))]
        pick = sorted(set(int(e) for e in pick))
        seg = {}
        xp, a1, y = (M.workspace_view(layer.handle, n) for n in ("Xp", "A1", "Y"))
        for e in pick:
            r0, r1 = int(offs[e]), int(offs[e + 1])
            seg[e] = (xp[r0:r1].cpu(), a1[r0:r1].cpu(), y[r0:r1].cpu())
        rows = sample_rows(T, n_rows)
        rows_t = torch.as_tensor(rows, device="cuda")
        a1s = M.workspace_view(layer.handle, "A1s")[:T].index_select(0, rows_t).cpu()
        hs = M.workspace_view(layer.handle, "Hs")[:T].index_select(0, rows_t).cpu()
    finally:
        layer.close()

    # routing over every token, h on the sampled rows
    ref = PAR.reference_selection(cfg, cpu, out["topk_idx"], out["scores"])
    rr = PAR.check_routing(cfg, ref, out, T)
    hh = PAR.check_h(cfg, cpu, ref, out, rows)
    print(name, rr, hh)

    # whole experts through both grouped GEMMs
    worst_a1 = worst_y = 0.0
    for e in pick:
        xp_e, a1_e, y_e = seg[e]
        A = O.swiglu_hidden(xp_e, cpu["W_gate"][e], cpu["W_up"][e])
        a1_k = O.bf16_bits_to_f64(a1_e)
        worst_a1 = max(worst_a1, _excess(a1_k, A))
        Yr = a1_k @ O.bf16_bits_to_f64(cpu["W_down"][e]).T
        worst_y = max(worst_y, _excess(O.bf16_bits_to_f64(y_e), Yr))
    # the shared expert on the sampled token rows
    x64 = O.bf16_bits_to_f64(cpu["x"])[rows]
    Fs = cfg.d_ff_shared
    a1s_k = O.bf16_bits_to_f64(a1s)
    hs_ref = x64.copy()
    worst_s = 0.0
    for s_ in range(cfg.n_shared):
        A = O.swiglu_hidden(x64, cpu["Ws_gate"][s_], cpu["Ws_up"][s_])
        blk = a1s_k[:, s_ * Fs:(s_ + 1) * Fs]
        worst_s = max(worst_s, _excess(blk, A))
        hs_ref += blk @ O.bf16_bits_to_f64(cpu["Ws_down"][s_]).T
    hs_err = float(np.abs(hs.numpy().astype(np.float64) - hs_ref).max() / np.sqrt(np.mean(hs_ref ** 2)))
    print(name, "experts", pick, "rows", [int(counts[e]) for e in pick], "A1 excess", worst_a1, "Y excess",
          worst_y, "A1s excess", worst_s, "Hs err/RMS", hs_err)
    for k in ("W_gate", "W_up", "W_down"):
        cpu[k].cache.clear()
    assert worst_a1 <= 1.0 and worst_y <= 1.0 and worst_s <= 1.0
    assert hs_err <= 1e-4
