"""Pins of the backward oracle (oracle/dsmoe_backward.py) to things other than itself:
central finite differences of the forward with the selection held fixed, torch float64
autograd of the same forward, and closed forms (zero experts, the softmax's shift
invariance, renormalised gates under a uniform gate gradient)."""
import numpy as np
import pytest
import torch

import workloads as W
from oracle import dsmoe_backward as B
from oracle import dsmoe_oracle as O

WEIGHTS = ("W_router", "W_gate", "W_up", "W_down", "Ws_gate", "Ws_up", "Ws_down")


def _cfg(score, renorm, **kw):
    base = dict(name="bwd", T=12, d_model=64, n_routed=8, top_k=2, d_ff=32, n_shared=1, d_ff_shared=32,
                score=score, renormalize=renorm, bias_mode=O.BIAS_NONE)
    base.update(kw)
    return W.MoEConfig(**base)


def _inputs64(cfg, seed):
    """The workload's generators, widened to float64 numpy (so they can be perturbed)."""
    inp = W.make_inputs(cfg, seed=seed)
    out = {}
    for k, v in inp.items():
        out[k] = None if v is None else (v.double().numpy() if v.dtype != torch.int32 else v.numpy())
    if out.get("W_router") is not None:
        out["W_router"] = out["W_router"] * 4.0  # sharper scores: gate terms matter
    return out


def _forward_fixed(cfg, inp, idx, alpha):
    """L = <dh, h> + alpha * sum f P with the expert choice idx held fixed (numpy float64)."""
    X = inp["x"]
    if cfg.score == O.ROUTE_HASH:
        s, gates = None, np.ones(idx.shape)
    else:
        l = X @ inp["W_router"].T
        if cfg.bias_mode == O.BIAS_IN_LOGITS:
            l = l + inp["b"][None, :]
        s = O.scores(l, cfg.score)
        gates = np.take_along_axis(s, idx, axis=1)
        if cfg.renormalize:
            gates = gates / gates.sum(axis=1, keepdims=True)
    routed = lambda e: (inp["W_gate"][e], inp["W_up"][e], inp["W_down"][e])
    shared = [(inp["Ws_gate"][i], inp["Ws_up"][i], inp["Ws_down"][i]) for i in range(cfg.n_shared)]
    h = O.moe_layer(X, idx, gates, routed, shared)
    L = float((inp["dh"] * h).sum())
    if alpha and s is not None:
        counts = np.bincount(idx.ravel(), minlength=cfg.n_routed)
        f = cfg.n_routed / (cfg.top_k * X.shape[0]) * counts
        L += alpha * float((f * s.mean(axis=0)).sum())
    return L


def _setup(cfg, seed=0, alpha=0.0):
    inp = _inputs64(cfg, seed)
    inp["dh"] = np.random.default_rng(seed + 1).normal(size=(cfg.T, cfg.d_model))
    r = O.route(cfg, inp)
    g = B.layer_backward(cfg, inp, inp["dh"], r, alpha_bal=alpha)
    return inp, r, g


CASES = [(O.SCORE_SOFTMAX, False, {}), (O.SCORE_SIGMOID, True, {}), (O.SCORE_SQRT_SOFTPLUS, True, {}),
         (O.SCORE_SOFTMAX, True, dict(mask_top=2, top_k=3)), (O.SCORE_SIGMOID, False, dict(n_shared=2)),
         (O.SCORE_SIGMOID, True, dict(bias_mode=O.BIAS_SELECT_ONLY, bias_kind="uniform0.1")),
         (O.SCORE_SOFTMAX, False, dict(bias_mode=O.BIAS_IN_LOGITS, bias_kind="zipf"))]


@pytest.mark.parametrize("score,renorm,kw", CASES, ids=[f"score{c[0]}-renorm{int(c[1])}-{i}" for i, c in enumerate(CASES)])
def test_backward_matches_finite_differences(score, renorm, kw):
    cfg = _cfg(score, renorm, **kw)
    alpha = 0.05
    inp, r, g = _setup(cfg, seed=3, alpha=alpha)
    idx = np.asarray(r["idx"], dtype=np.int64)
    rng = np.random.default_rng(7)
    eps = 1e-5
    targets = [("x", "dx")] + [(w, "d" + w) for w in WEIGHTS]
    for name, gname in targets:
        A = inp[name]
        for _ in range(6):
            pos = tuple(rng.integers(0, n) for n in A.shape)
            old = A[pos]
            A[pos] = old + eps
            Lp = _forward_fixed(cfg, inp, idx, alpha)
            A[pos] = old - eps
            Lm = _forward_fixed(cfg, inp, idx, alpha)
            A[pos] = old
            fd = (Lp - Lm) / (2 * eps)
            an = g[gname][pos]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(fd)), (name, pos, fd, an)


def _torch_forward(cfg, P, idx, dh, alpha):
    X = P["x"]
    silu = lambda a: a * torch.sigmoid(a)
    ffn = lambda U, Wg, Wu, Wd: (silu(U @ Wg.T) * (U @ Wu.T)) @ Wd.T
    l = X @ P["W_router"].T
    if cfg.bias_mode == O.BIAS_IN_LOGITS:
        l = l + torch.from_numpy(P["_b"])[None, :]
    if cfg.score == O.SCORE_SOFTMAX:
        s = torch.softmax(l, dim=1)
    elif cfg.score == O.SCORE_SIGMOID:
        s = torch.sigmoid(l)
    else:
        s = torch.sqrt(torch.nn.functional.softplus(l))
    ti = torch.from_numpy(idx)
    gates = torch.gather(s, 1, ti)
    if cfg.renormalize:
        gates = gates / gates.sum(dim=1, keepdim=True)
    h = X.clone()
    for i in range(cfg.n_shared):
        h = h + ffn(X, P["Ws_gate"][i], P["Ws_up"][i], P["Ws_down"][i])
    for k in range(idx.shape[1]):
        for e in np.unique(idx[:, k]):
            rows = torch.from_numpy(np.nonzero(idx[:, k] == e)[0])
            y = ffn(X[rows], P["W_gate"][e], P["W_up"][e], P["W_down"][e])
            h = h.index_add(0, rows, gates[rows, k:k + 1] * y)
    counts = torch.bincount(ti.reshape(-1), minlength=cfg.n_routed).double()
    f = cfg.n_routed / (cfg.top_k * X.shape[0]) * counts
    return (torch.from_numpy(dh) * h).sum() + alpha * (f * s.mean(dim=0)).sum()


@pytest.mark.parametrize("score,renorm,kw", CASES, ids=[f"score{c[0]}-renorm{int(c[1])}-{i}" for i, c in enumerate(CASES)])
def test_backward_matches_torch_autograd(score, renorm, kw):
    cfg = _cfg(score, renorm, **kw)
    alpha = 0.1
    inp, r, g = _setup(cfg, seed=5, alpha=alpha)
    idx = np.asarray(r["idx"], dtype=np.int64)
    P = {k: torch.tensor(inp[k], dtype=torch.float64, requires_grad=True) for k in ("x",) + WEIGHTS}
    P["_b"] = None if inp.get("b") is None else np.asarray(inp["b"], dtype=np.float64)
    L = _torch_forward(cfg, P, idx, inp["dh"], alpha)
    grads = torch.autograd.grad(L, [P[k] for k in ("x",) + WEIGHTS])
    for k, gt in zip(("x",) + WEIGHTS, grads):
        np.testing.assert_allclose(g["d" + k], gt.numpy(), rtol=1e-9, atol=1e-11, err_msg=k)


def test_zero_experts_leave_only_the_residual_and_the_balance_term():
    cfg = _cfg(O.SCORE_SOFTMAX, False)
    inp = _inputs64(cfg, 9)
    for k in ("W_gate", "W_up", "W_down", "Ws_gate", "Ws_up", "Ws_down"):
        inp[k] = np.zeros_like(inp[k])
    dh = np.random.default_rng(2).normal(size=(cfg.T, cfg.d_model))
    r = O.route(cfg, inp)
    g = B.layer_backward(cfg, inp, dh, r, alpha_bal=0.0)
    np.testing.assert_array_equal(g["dx"], dh)  # h = u exactly: dx = dh
    assert not g["dW_router"].any() and not g["dW_gate"].any()
    # with the balance term only the router moves, and the softmax shift invariance makes
    # each token's logit gradient sum to zero
    g = B.layer_backward(cfg, inp, dh, r, alpha_bal=0.3)
    assert g["dW_router"].any()
    np.testing.assert_allclose(g["dlogits"].sum(axis=1), 0.0, atol=1e-15)


def test_renormalised_gates_ignore_a_uniform_gate_gradient():
    s = np.random.default_rng(4).uniform(0.1, 1.0, size=(5, 8))
    idx, gates = O.select_topk(s, 3, renormalize=True)
    ds = B.gate_backward(s, idx, gates, np.full((5, 3), 2.5), renormalize=True)
    np.testing.assert_allclose(ds, 0.0, atol=1e-14)  # sum_k g_k = 1 for every s


def test_hash_routing_has_no_router_gradient():
    cfg = W.MoEConfig("h", T=10, d_model=64, n_routed=8, top_k=1, d_ff=32, n_shared=1, d_ff_shared=32,
                      score=O.ROUTE_HASH)
    inp = W.make_inputs(cfg, seed=1)
    dh = np.random.default_rng(0).normal(size=(10, 64))
    g = B.layer_backward(cfg, inp, dh)
    assert g["dW_router"] is None
    # g = 1: the routed dW of an expert is the plain FFN backward of its rows
    r = O.route(cfg, inp)
    e = int(r["idx"][0, 0])
    rows = np.nonzero(r["idx"][:, 0] == e)[0]
    _, dWg, _, _ = B.swiglu_backward(O._as_f64(inp["x"])[rows], inp["W_gate"][e], inp["W_up"][e],
                                     inp["W_down"][e], dh[rows])
    np.testing.assert_allclose(g["dW_gate"][e], dWg, rtol=1e-12)


# plausible slips planted in the backward oracle; the finite-difference pin must catch each
def _silu_grad_without_product_term(a):
    return O.sigmoid(a)


def _score_backward_softmax_without_centering(l, s, ds, score):
    if score == O.SCORE_SOFTMAX:
        return s * ds
    return _ORIG_SCORE(l, s, ds, score)


def _gate_backward_renorm_as_raw(s, idx, gates, dg, renormalize):
    return _ORIG_GATE(s, idx, gates, dg, False)


_ORIG_SCORE, _ORIG_GATE = B.score_backward, B.gate_backward
MUTATIONS = [("silu_grad", _silu_grad_without_product_term, 0),
             ("score_backward", _score_backward_softmax_without_centering, 0),
             ("gate_backward", _gate_backward_renorm_as_raw, 1)]


@pytest.mark.parametrize("name,mut,case", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_finite_differences_catch_planted_slips(monkeypatch, name, mut, case):
    monkeypatch.setattr(B, name, mut)
    with pytest.raises(AssertionError):
        test_backward_matches_finite_differences(*CASES[case])
