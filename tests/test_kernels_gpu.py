"""Each stage of the CUDA path against the oracle's intermediate result, read from the
handle's workspace after a forward: router logits, segment offsets, the slot
permutation and row gather (bit-exact), the gate/up activation A1 and the expert
outputs Y per slot, and the fp32 residual + shared-expert rows Hs.

Bounds: A1 and Y are fp32 accumulations rounded once to bf16 (round to nearest
even: |err| <= 2^-9 |v|), so each element must lie within 2^-8 |ref| + 1e-4 RMS(ref)
of the float64 value; Hs is never rounded to bf16 and must lie within 1e-4 RMS."""
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

# T < 256 runs the CUDA-core router (split-K logits, then the select kernel); larger T
# the tensor-core router; both are checked through the scores they report.
# The grouped GEMMs run on the default one-CTA kernel; the "-pair" cases run the CTA-pair
# kernel.
# v3_slice at T=800 (d = 7168, 200 rows per expert on average) takes the 256-token gate/up
# tiles, with experts of one and of two (evenly split) token tiles.
CASES = [("tiny", 300, 0), ("tiny", 200, 0), ("gshard_c", 700, 0), ("ds2b", 900, 0), ("v4_decode_t64", 64, 0),
         ("v3_slice", 800, 0), ("tiny", 300, 1), ("ds2b", 900, 1)]


@pytest.mark.parametrize("name,T,pair", CASES,
                         ids=[f"{c[0]}-T{c[1]}" + ("-pair" if c[2] else "") for c in CASES])
def test_stages(name, T, pair):
    cfg = W.get_config(name)
    gpu, cpu = make_case(cfg, T)
    layer = M.DSMoE(M.cfg_from(cfg, T), gpu)
    M.dsmoe_set_gemm_kernel(layer.handle, M.DSMOE_GEMM_PAIR if pair else M.DSMOE_GEMM_SINGLE)
    out = layer.forward(gpu["x"], with_scores=True)
    torch.cuda.synchronize()
    ws = {n: M.workspace_view(layer.handle, n).clone().cpu()
          for n in ("offsets", "slot_of", "Xp", "A1", "Y") + (("A1s", "Hs") if cfg.n_shared else ())}
    assert M.dsmoe_get_status(layer.handle) == M.DSMOE_OK
    layer.close()
    K, N, S = cfg.top_k, cfg.n_routed, T * cfg.top_k
    x64 = O.bf16_bits_to_f64(cpu["x"])
    # router scores (either router) against float64
    l_ref = O.router_logits(cpu["x"], cpu["W_router"], cpu.get("b"), cfg.bias_mode)
    s_ref = O.scores(l_ref, cfg.score)
    assert np.abs(out["scores"].cpu().numpy() - s_ref).max() < 2e-5
    # offsets: exclusive scan of the counts
    counts = out["counts"].cpu().numpy()
    offs = ws["offsets"][0].numpy()
    assert (offs == np.concatenate([[0], np.cumsum(counts)])).all()
    # slots: a permutation of 0..S-1, each inside its expert's segment, rows gathered exactly
    topk = out["topk_idx"].cpu().numpy()
    slot = ws["slot_of"][:T].numpy()
    assert sorted(slot.ravel().tolist()) == list(range(S))
    assert ((slot >= offs[topk]) & (slot < offs[topk + 1])).all()
    xp = ws["Xp"][:S]
    assert torch.equal(xp[torch.as_tensor(slot.ravel(), dtype=torch.long)],
                       cpu["x"].repeat_interleave(K, dim=0))
    # A1 and Y per slot, for every expert's rows
    a1 = ws["A1"][:S].float().numpy().astype(np.float64)
    y = ws["Y"][:S].float().numpy().astype(np.float64)
    worst_a1 = worst_y = 0.0
    for e in range(N):
        rows = np.arange(offs[e], offs[e + 1])
        if rows.size == 0:
            continue
        U = O.bf16_bits_to_f64(xp[torch.as_tensor(rows)])
        A = O.swiglu_hidden(U, cpu["W_gate"][e], cpu["W_up"][e])
        worst_a1 = max(worst_a1, _excess(a1[rows], A))
        # Y is computed from the kernel's own bf16 A1
        Yr = a1[rows] @ O.bf16_bits_to_f64(cpu["W_down"][e]).T
        worst_y = max(worst_y, _excess(y[rows], Yr))
    print(name, "A1 excess", worst_a1, "Y excess", worst_y)
    assert worst_a1 <= 1.0 and worst_y <= 1.0
    if cfg.n_shared:
        Fs = cfg.d_ff_shared
        a1s = ws["A1s"][:T].float().numpy().astype(np.float64)
        hs_ref = x64.copy()
        for s_ in range(cfg.n_shared):
            A = O.swiglu_hidden(x64, cpu["Ws_gate"][s_], cpu["Ws_up"][s_])
            assert _excess(a1s[:, s_ * Fs:(s_ + 1) * Fs], A) <= 1.0
            hs_ref += a1s[:, s_ * Fs:(s_ + 1) * Fs] @ O.bf16_bits_to_f64(cpu["Ws_down"][s_]).T
        hs = ws["Hs"][:T].numpy().astype(np.float64)
        assert np.abs(hs - hs_ref).max() <= 1e-4 * np.sqrt(np.mean(hs_ref ** 2))


def _excess(got, ref):
    """max over elements of |got - ref| / (2^-8 |ref| + 1e-4 RMS(ref)); <= 1 passes."""
    bound = 2.0 ** -8 * np.abs(ref) + 1e-4 * np.sqrt(np.mean(ref ** 2))
    return float((np.abs(got - ref) / bound).max())
