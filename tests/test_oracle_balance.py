"""Pins of the oracle's balance-control functions (expert- and device-level losses,
the classic loss, the sequence-wise statistics and the auxiliary-loss-free bias
update) against closed forms, identities between them and the pages' worked numbers."""
import json
import os

import numpy as np
import pytest

from oracle import dsmoe_oracle as O


def _routing(T=120, N=12, K=3, seed=0):
    rng = np.random.default_rng(seed)
    s = O.softmax(rng.normal(size=(T, N)))
    idx, _ = O.select_topk(s, K)
    counts, f, P = O.balance_stats(idx, s, N, K)
    return idx, s, counts, f, P


def test_expert_loss_uniform_closed_form():
    N = 16
    f = np.ones(N)
    P = np.full(N, 1.0 / N)
    assert O.expert_balance_loss(f, P, 0.01) == pytest.approx(0.01 / N, rel=1e-15)


def test_expert_loss_doubles_with_a_concentrated_router():
    # all probability on one expert that also carries twice its share of the load
    N = 4
    f = np.array([2.0, 2 / 3, 2 / 3, 2 / 3])  # the expert-level worked example
    P = np.array([1.0, 0.0, 0.0, 0.0])
    assert O.expert_balance_loss(f, P, 1.0) == pytest.approx(2.0 / 4)


def test_device_level_reductions():
    idx, s, counts, f, P = _routing()
    N = f.shape[0]
    # one expert per device: f' = f, P' = P, L_dev = alpha2 * N' * L_exp / alpha1
    fd, Pd, L = O.device_balance(f, P, np.arange(N), N, 0.05)
    np.testing.assert_allclose(fd, f, rtol=1e-15)
    np.testing.assert_allclose(Pd, P, rtol=1e-15)
    assert L == pytest.approx(0.05 * N * O.expert_balance_loss(f, P, 1.0), rel=1e-13)
    # one device: f' = mean f = 1, P' = sum P = 1 (softmax) => L = alpha2 exactly
    fd, Pd, L = O.device_balance(f, P, np.zeros(N, int), 1, 0.05)
    assert fd[0] == pytest.approx(1.0, rel=1e-14) and Pd[0] == pytest.approx(1.0, rel=1e-14)
    assert L == pytest.approx(0.05, rel=1e-13)
    # brute force over an uneven grouping
    groups = np.array([0, 0, 0, 1, 1, 2, 2, 2, 2, 3, 3, 3])
    fd, Pd, L = O.device_balance(f, P, groups, 4, 0.05)
    for d in range(4):
        m = groups == d
        assert fd[d] == pytest.approx(f[m].mean(), rel=1e-14)
        assert Pd[d] == pytest.approx(P[m].sum(), rel=1e-14)
    assert L == pytest.approx(0.05 * sum(f[groups == d].mean() * P[groups == d].sum() for d in range(4)))


def test_classic_loss_equals_scaled_expert_loss():
    """alpha E sum (counts_i/(K'T)) P_i = alpha sum f_i P_i = alpha N' L_ExpBal / alpha_1."""
    idx, s, counts, f, P = _routing()
    N = f.shape[0]
    assert O.classic_balance_loss(counts, P, 3, 0.01) == pytest.approx(
        0.01 * N * O.expert_balance_loss(f, P, 1.0), rel=1e-13)


def test_sequence_balance_one_sequence_and_brute_force():
    idx, s, counts, f, P = _routing(T=120, N=12, K=3)
    fs, ps, L = O.sequence_balance(idx, s, 120, 12, 1e-4)
    np.testing.assert_allclose(fs[0], counts / 120, rtol=1e-15)
    np.testing.assert_allclose(ps[0], P, rtol=1e-14)
    assert L == pytest.approx(1e-4 * (3 / 12) * (f * P).sum(), rel=1e-13)
    fs, ps, L = O.sequence_balance(idx, s, 40, 12, 1e-4)
    assert fs.shape == (3, 12)
    for q in range(3):
        sub = idx[q * 40:(q + 1) * 40]
        np.testing.assert_allclose(fs[q], np.bincount(sub.ravel(), minlength=12) / 40)
        np.testing.assert_allclose(fs[q].sum(), 3.0)
    assert L == pytest.approx(np.mean([1e-4 * (fs[q] * ps[q]).sum() for q in range(3)]))


def test_sequence_expected_load_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "v4_sequence_load_example.json")))
    # uniform load: every expert takes K' T / N' assignments of the sequence
    exp = g["sequence_tokens"] * g["top_k"] / g["n_routed"]
    assert exp == g["expected_assignments_per_expert"]


def test_bias_update_rule():
    N, K, T = 8, 2, 100
    b = np.linspace(-0.1, 0.1, N)
    uniform = np.full(N, K * T // N)
    np.testing.assert_allclose(O.bias_update(b, uniform, T, K, 0.001), b, atol=1e-17)
    counts = np.array([50, 10, 25, 25, 25, 25, 20, 20])
    nb = O.bias_update(b, counts, T, K, 0.001)
    assert nb[0] < b[0] and nb[1] > b[1]          # over-loaded falls, under-loaded rises
    np.testing.assert_allclose(nb - b, 0.001 * (K / N - counts / T), rtol=1e-12)
    assert (nb - b).sum() == pytest.approx(0.001 * (K - counts.sum() / T), abs=1e-15)
