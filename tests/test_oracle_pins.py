"""Pins of the oracle to things other than itself.

Each test fixes one part of the oracle against a value the pages print, a
closed form, an invariant of the definition, a library routine, or brute
force on a tiny input. A plausible slip in the oracle (a dropped term, a wrong
sign or index, a transposed operand, a wrong tie-break) fails at least one of
them; test_oracle_mutations.py plants such slips and checks that.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import workloads as W
from oracle import dsmoe_oracle as O


def _bf16(a):
    return torch.as_tensor(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)


# ------------------------------------------------------------------------------------------
# balance statistics
# ------------------------------------------------------------------------------------------
def test_balance_worked_example(golden_dir):
    """The page's worked example: N'=4, K'=2, T=3, E1 picked by every token -> f_1 = 2."""
    g = json.load(open(os.path.join(golden_dir, "balance_worked_example.json")))
    idx = np.array(g["selections_1based"]) - 1
    counts, f, P = O.balance_stats(idx, None, g["n_routed"], g["top_k"])
    assert g["top_k"] * g["T"] / g["n_routed"] == g["uniform_count_per_expert"]
    assert f[0] == pytest.approx(g["f_1"], abs=1e-15)
    assert counts.tolist() == [3, 1, 1, 1]
    # the remaining experts are each picked once: 1 / 1.5
    np.testing.assert_allclose(f[1:], 1.0 / g["uniform_count_per_expert"], rtol=1e-15)


def test_uniform_load_gives_unit_f():
    N, K, T = 8, 2, 12
    idx = np.array([[(2 * t) % N, (2 * t + 1) % N] for t in range(T)])
    counts, f, _ = O.balance_stats(idx, None, N, K)
    assert (counts == K * T // N).all()
    np.testing.assert_allclose(f, 1.0, rtol=0, atol=1e-15)


@pytest.mark.parametrize("score", [O.SCORE_SOFTMAX, O.SCORE_SIGMOID, O.SCORE_SQRT_SOFTPLUS])
def test_stats_invariants(score):
    rng = np.random.default_rng(1)
    T, N, K = 97, 24, 5
    l = rng.normal(size=(T, N))
    s = O.scores(l, score)
    idx, _ = O.select_topk(s, K)
    counts, f, P = O.balance_stats(idx, s, N, K)
    assert counts.sum() == T * K
    assert f.sum() == pytest.approx(N, rel=1e-13)  # sum_i f_i = N' by definition
    np.testing.assert_allclose(P, s.mean(axis=0), rtol=1e-13)
    if score == O.SCORE_SOFTMAX:
        assert P.sum() == pytest.approx(1.0, abs=1e-13)  # softmax over routed experts only
    # every row picks K distinct experts
    assert all(len(set(r)) == K for r in idx.tolist())


def test_identical_router_rows():
    """Identical expert centroids: every score ties, P_i = 1/N', ties go to the lowest indices."""
    T, d, N, K = 6, 16, 10, 3
    rng = np.random.default_rng(2)
    x = _bf16(rng.normal(size=(T, d)))
    row = rng.normal(size=(1, d))
    Wr = _bf16(np.repeat(row, N, axis=0))
    l = O.router_logits(x, Wr)
    s = O.scores(l, O.SCORE_SOFTMAX)
    idx, g = O.select_topk(s, K)
    assert (idx == np.arange(K)[None, :]).all()
    _, _, P = O.balance_stats(idx, s, N, K)
    np.testing.assert_allclose(P, 1.0 / N, rtol=1e-14)
    np.testing.assert_allclose(g, 1.0 / N, rtol=1e-14)


# ------------------------------------------------------------------------------------------
# score functions
# ------------------------------------------------------------------------------------------
def test_score_page_readings(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "v4_score_demo.json")))
    fns = {"sigmoid": O.sigmoid, "softplus": O.softplus, "sqrt_softplus": O.sqrt_softplus}
    for r in g["readings"]:
        v = float(fns[r["fn"]](r["logit"]))
        assert round(v, r["decimals"]) == pytest.approx(r["value"], abs=1e-12), r


def test_score_closed_forms():
    assert O.sigmoid(0.0) == 0.5
    assert O.sqrt_softplus(0.0) == pytest.approx(math.sqrt(math.log(2.0)), rel=1e-15)
    l = np.linspace(-30, 30, 121)
    # softplus(l) - softplus(-l) = l ; sigmoid(-l) = 1 - sigmoid(l)
    np.testing.assert_allclose(O.softplus(l) - O.softplus(-l), l, atol=1e-13)
    np.testing.assert_allclose(O.sigmoid(-l), 1.0 - O.sigmoid(l), atol=1e-15)
    # d/dl softplus = sigmoid (central difference)
    h = 1e-5
    np.testing.assert_allclose((O.softplus(l + h) - O.softplus(l - h)) / (2 * h), O.sigmoid(l), atol=1e-9)
    # a two-way softmax is the sigmoid of the logit difference
    a, b = np.array([1.3, -0.2, 4.0]), np.array([0.1, 2.5, -3.0])
    sm = O.softmax(np.stack([a, b], axis=1))
    np.testing.assert_allclose(sm[:, 0], O.sigmoid(a - b), rtol=1e-14)
    # softmax is invariant to a common shift and matches the textbook form
    l2 = np.array([[0.5, -1.0, 2.0, 0.0]])
    np.testing.assert_allclose(O.softmax(l2 + 100.0), O.softmax(l2), rtol=1e-13)
    e = np.exp(l2)
    np.testing.assert_allclose(O.softmax(l2), e / e.sum(), rtol=1e-14)


def test_scores_match_torch_library():
    l = torch.linspace(-12, 12, 97, dtype=torch.float64)
    np.testing.assert_allclose(O.sigmoid(l.numpy()), torch.sigmoid(l).numpy(), rtol=1e-14)
    np.testing.assert_allclose(O.sqrt_softplus(l.numpy()),
                               torch.sqrt(torch.nn.functional.softplus(l)).numpy(), rtol=1e-13)
    L = torch.randn(7, 13, dtype=torch.float64, generator=torch.Generator().manual_seed(3))
    np.testing.assert_allclose(O.softmax(L.numpy()), torch.softmax(L, dim=-1).numpy(), rtol=1e-13)


# ------------------------------------------------------------------------------------------
# top-k selection and gates
# ------------------------------------------------------------------------------------------
def _brute_topk(key, k):
    """Max-sum k-subset, ties to the lexicographically smallest index tuple; then ordered by
    (key desc, index asc)."""
    best, best_sum = None, None
    for comb in itertools.combinations(range(len(key)), k):
        sm = sum(key[i] for i in comb)
        if best_sum is None or sm > best_sum:
            best, best_sum = comb, sm
    return sorted(best, key=lambda i: (-key[i], i))


@pytest.mark.parametrize("N,K", [(4, 1), (6, 2), (9, 3), (12, 3), (7, 7)])
def test_topk_bruteforce(N, K):
    rng = np.random.default_rng(N * 31 + K)
    for trial in range(20):
        # integer-valued keys with many ties so subset sums are exact
        key = rng.integers(0, 4, size=N).astype(np.float64)
        idx, _ = O.select_topk(key[None, :], K)
        assert idx[0].tolist() == _brute_topk(key.tolist(), K)


def test_topk_bruteforce_with_selection_bias():
    rng = np.random.default_rng(5)
    N, K = 10, 3
    for trial in range(20):
        s = rng.integers(0, 5, size=N) / 4.0
        b = rng.integers(-2, 3, size=N) / 4.0
        idx, g = O.select_topk(s[None, :], K, b, O.BIAS_SELECT_ONLY)
        assert idx[0].tolist() == _brute_topk((s + b).tolist(), K)
        # the bias only decides who is selected: gates are the raw scores
        np.testing.assert_array_equal(g[0], s[idx[0]])


def _iterative_masked_pick(key, r, k):
    """The "disable the top routed experts" analysis of the DeepSeekMoE summary written as
    repeated arg-max: remove the best expert r times, then take the best k of the rest
    one at a time (ties to the lower index at every step)."""
    alive = list(range(len(key)))
    def pop_best():
        best = max(alive, key=lambda i: (key[i], -i))
        alive.remove(best)
        return best
    for _ in range(r):
        pop_best()
    return [pop_best() for _ in range(k)]


@pytest.mark.parametrize("N,K,r", [(8, 2, 1), (8, 3, 2), (12, 4, 3), (6, 1, 5), (9, 3, 0)])
def test_masked_topk_bruteforce(N, K, r):
    rng = np.random.default_rng(100 * N + 10 * K + r)
    for trial in range(20):
        s = rng.integers(0, 5, size=N) / 4.0
        b = rng.integers(-2, 3, size=N) / 8.0
        idx, g = O.select_topk(s[None, :], K, b, O.BIAS_SELECT_ONLY, mask_top=r)
        assert idx[0].tolist() == _iterative_masked_pick((s + b).tolist(), r, K)
        np.testing.assert_array_equal(g[0], s[idx[0]])  # gates stay raw scores


def test_masked_and_reduced_k_compose_with_the_plain_selection():
    """Masking the top r and keeping K' leaves exactly the plain top-(r+K') minus the plain
    top-r; a smaller K' keeps a prefix of the K' order; renormalised gates sum to one
    over the kept experts."""
    rng = np.random.default_rng(11)
    s = O.softmax(rng.normal(size=(50, 16)))
    full, _ = O.select_topk(s, 7)
    for r, k in [(1, 6), (2, 4), (3, 3), (0, 3)]:
        idx, g = O.select_topk(s, k, mask_top=r, renormalize=True)
        np.testing.assert_array_equal(idx, full[:, r:r + k])
        np.testing.assert_allclose(g.sum(axis=1), 1.0, rtol=1e-12)
    # the route of a config with mask_top equals select_topk on the same scores
    cfg = W.get_config("tiny").replace(T=40, mask_top=2, top_k=3)
    inp = W.make_inputs(cfg, seed=3, with_weights=False)
    r = O.route(cfg, inp)
    idx, _ = O.select_topk(r["scores"], 3, inp.get("b"), cfg.bias_mode, cfg.renormalize, mask_top=2)
    np.testing.assert_array_equal(r["idx"], idx)
    assert r["counts"].sum() == 40 * 3


def test_gates_raw_and_renormalised():
    rng = np.random.default_rng(6)
    s = O.sigmoid(rng.normal(size=(11, 20)))
    idx, g = O.select_topk(s, 4)
    np.testing.assert_array_equal(g, np.take_along_axis(s, idx.astype(np.int64), axis=1))
    idx2, g2 = O.select_topk(s, 4, renormalize=True)
    np.testing.assert_array_equal(idx2, idx)
    np.testing.assert_allclose(g2.sum(axis=1), 1.0, rtol=1e-14)
    np.testing.assert_allclose(g2 * g.sum(axis=1, keepdims=True), g, rtol=1e-14)
    # ordering: descending score
    assert (np.diff(g, axis=1) <= 0).all()


def test_fp32_decision_path():
    """Near-tie keys: float64 separates them, fp32 rounds them equal and the lower index wins."""
    s = np.array([[0.1, 0.1 + 1e-12, 0.0]])
    i64, _ = O.select_topk(s, 1)
    i32, _ = O.select_topk(s, 1, decision_dtype=np.float32)
    assert i64[0, 0] == 1 and i32[0, 0] == 0


def test_hash_route():
    """expert = id * 2654435761 mod 384: the multiplier is 49 mod 384 and coprime to 384,
    so ids 0..383 land on distinct experts; compare against Python's exact integers."""
    assert 2654435761 % 384 == 49 and math.gcd(49, 384) == 1
    ids = np.arange(384, dtype=np.int64)
    e, g = O.hash_route(ids, 384)
    assert sorted(e[:, 0].tolist()) == list(range(384))
    assert (g == 1).all()
    rng = np.random.default_rng(7)
    big = rng.integers(0, 129280, size=1000)
    e2, _ = O.hash_route(big, 384)
    assert e2[:, 0].tolist() == [(int(i) * 2654435761) % 384 for i in big]
    # no 32-bit wrap: the wrapped product would give other experts for large ids
    wrapped = [((int(i) * 2654435761) & 0xFFFFFFFF) % 384 for i in big]
    assert wrapped != e2[:, 0].tolist()


# ------------------------------------------------------------------------------------------
# expert FFN and the layer equation
# ------------------------------------------------------------------------------------------
def _rand_expert(rng, d, F, scale=1.0):
    return (_bf16(rng.normal(size=(F, d)) * scale / math.sqrt(d)),
            _bf16(rng.normal(size=(F, d)) * scale / math.sqrt(d)),
            _bf16(rng.normal(size=(d, F)) * scale / math.sqrt(F)))


def test_swiglu_matches_torch_library():
    rng = np.random.default_rng(8)
    d, F, m = 24, 40, 9
    Wg, Wu, Wd = _rand_expert(rng, d, F)
    U = _bf16(rng.normal(size=(m, d)))
    ref = torch.nn.functional.linear(
        torch.nn.functional.silu(torch.nn.functional.linear(U.double(), Wg.double()))
        * torch.nn.functional.linear(U.double(), Wu.double()), Wd.double())
    np.testing.assert_allclose(O.swiglu_ffn(U, Wg, Wu, Wd), ref.numpy(), rtol=1e-12, atol=1e-13)


def test_swiglu_bruteforce_tiny():
    """Pure-Python loops over the written indices, on a 3x2 case (non-square, so a transpose
    of any operand changes the answer)."""
    Wg = [[0.5, -1.0, 0.25], [1.5, 0.0, -0.5]]   # [F=2, d=3]
    Wu = [[1.0, 2.0, -1.0], [-0.5, 0.5, 1.0]]
    Wd = [[1.0, -2.0], [0.5, 0.25], [-1.0, 1.0]]  # [d=3, F=2]
    u = [0.75, -0.5, 2.0]
    z = []
    for j in range(2):
        a = sum(Wg[j][k] * u[k] for k in range(3))
        b = sum(Wu[j][k] * u[k] for k in range(3))
        z.append(a / (1.0 + math.exp(-a)) * b)
    y = [sum(Wd[i][j] * z[j] for j in range(2)) for i in range(3)]
    got = O.swiglu_ffn(_bf16([u]), _bf16(Wg), _bf16(Wu), _bf16(Wd))[0]
    np.testing.assert_allclose(got, y, rtol=1e-14)


def test_gshard_reduction_dense_gate_sum():
    """m=1, K_s=0 is the conventional top-K layer h = sum_{i=1}^{N} g_{i,t} FFN_i(u) + u with
    a dense gate vector that is zero off the top-K (DeepSeekMoE summary, GShard equation).
    Brute force: run every expert on every token and weight by the dense gates."""
    rng = np.random.default_rng(9)
    T, d, N, K, F = 13, 16, 6, 2, 24
    x = _bf16(rng.normal(size=(T, d)))
    Wr = _bf16(rng.normal(size=(N, d)) / 4)
    experts = [_rand_expert(rng, d, F) for _ in range(N)]
    s = O.scores(O.router_logits(x, Wr), O.SCORE_SOFTMAX)
    idx, g = O.select_topk(s, K)
    h = O.moe_layer(x, idx, g, lambda e: experts[e], [])
    dense_g = np.zeros((T, N))
    for t in range(T):
        for k in range(K):
            dense_g[t, idx[t, k]] = g[t, k]
    ref = O.bf16_bits_to_f64(x).copy()
    for i in range(N):
        ref += dense_g[:, i:i + 1] * O.swiglu_ffn(x, *experts[i])
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_identical_experts_reduce_to_one_dense_ffn():
    """All routed experts equal and gates renormalised: the routed sum is one dense FFN."""
    rng = np.random.default_rng(10)
    T, d, N, K, F = 11, 16, 8, 3, 32
    x = _bf16(rng.normal(size=(T, d)))
    Wr = _bf16(rng.normal(size=(N, d)) / 4)
    e0 = _rand_expert(rng, d, F)
    sh = _rand_expert(rng, d, F)
    s = O.scores(O.router_logits(x, Wr), O.SCORE_SIGMOID)
    idx, g = O.select_topk(s, K, renormalize=True)
    h = O.moe_layer(x, idx, g, lambda e: e0, [sh])
    ref = O.bf16_bits_to_f64(x) + O.swiglu_ffn(x, *sh) + O.swiglu_ffn(x, *e0)
    np.testing.assert_allclose(h, ref, rtol=1e-12, atol=1e-12)


def test_zero_weights_give_residual_exactly():
    rng = np.random.default_rng(11)
    T, d, N, K, F = 5, 8, 4, 2, 8
    x = _bf16(rng.normal(size=(T, d)))
    z = (_bf16(np.zeros((F, d))), _bf16(np.zeros((F, d))), _bf16(np.zeros((d, F))))
    idx = np.array([[0, 1]] * T)
    g = np.full((T, K), 0.5)
    h = O.moe_layer(x, idx, g, lambda e: z, [z])
    np.testing.assert_array_equal(h, O.bf16_bits_to_f64(x))


def test_layer_rows_subset_equals_full():
    """Evaluating a subset of rows gives the same rows as the full evaluation (per-token
    independence of the expert FFNs and the combine)."""
    cfg = W.get_config("tiny").replace(T=40)
    inp = W.make_inputs(cfg, seed=3)
    full = O.forward(cfg, inp)
    rows = [39, 0, 17, 5]
    sub = O.forward(cfg, inp, rows=rows, routing=full)
    np.testing.assert_allclose(sub["h"], full["h"][rows], rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------------------------------------
# configuration generator
# ------------------------------------------------------------------------------------------
def test_config_generator_combinations(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "combinations.json")))
    exact = {(r["n"], r["k"]): r["value"] for r in g["exact"]}
    a, b = W.get_config("gshard_a"), W.get_config("gshard_b")
    m = b.n_routed // a.n_routed
    assert m == 4 and b.top_k == m * a.top_k  # fine-grained segmentation N'=mN, K'=mK
    assert O.combinations(a.n_routed, a.top_k) == exact[(16, 2)] == 120
    assert O.combinations(b.n_routed, b.top_k) == exact[(64, 8)] == 4426165368
    assert O.combinations(8, 2) == exact[(8, 2)]
    for r in g["approximate"]:
        v = O.combinations(r["n"], r["k"])
        assert float(f"{v:.{r['sig'] - 1}e}") == r["value"]
    for r in g["page_errors"]:
        v = O.combinations(r["n"], r["k"])
        assert v == 455196700703112576 and abs(v - r["page_value"]) / v > 0.5


def test_config_generator_flops_identity():
    """k'(2 d d_ff / m) = k (2 d d_ff): equal expert FLOPs per token for the GShard triple."""
    fl = [W.get_config(n).expert_flops_per_token() for n in ("gshard_a", "gshard_b", "gshard_c")]
    assert fl == [34603008] * 3
    v3 = W.get_config("v3_prefill")
    assert abs(v3.routed_weight_bytes() / 1e9 - 22.5) < 0.1  # "~22.5 GB routed"
    assert v3.n_routed == 256 and v3.top_k == 8 and v3.n_shared == 1


def test_zipf_skew_is_about_ten_to_one():
    cfg = W.get_config("ds2b")
    inp = W.make_inputs(cfg, seed=0, with_weights=False)
    r = O.route(cfg, inp)
    ratio = r["counts"].max() / r["counts"].min()
    assert 9.5 <= ratio <= 10.5
    assert r["counts"].argmax() == 0
