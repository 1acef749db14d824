"""Plant plausible mistakes in the oracle and check that a pin catches each one.

Every mutation is applied to the oracle module on the CPU (monkeypatch) and
the named pin from test_oracle_pins.py must then fail.
"""
import numpy as np
import pytest

from oracle import dsmoe_oracle as O
import tests.test_oracle_pins as P

_orig = {n: getattr(O, n) for n in ("silu", "select_topk", "balance_stats", "sqrt_softplus",
                                     "moe_layer", "hash_route", "swiglu_ffn", "softmax")}


def _silu_without_sigmoid(a):
    return a


def _topk_ties_to_higher_index(s, top_k, b=None, bias_mode=0, renormalize=False,
                               decision_dtype=np.float64):
    s = np.asarray(s, dtype=np.float64)
    N = s.shape[1]
    rev = s[:, ::-1]
    bb = None if b is None else np.asarray(b)[::-1]
    idx, g = _orig["select_topk"](rev, top_k, bb, bias_mode, renormalize, decision_dtype)
    return (N - 1 - idx).astype(np.int32), g


def _mask_ranked_by_raw_score(s, top_k, b=None, bias_mode=0, renormalize=False,
                              decision_dtype=np.float64, mask_top=0):
    """Masks the r experts with the highest raw score instead of the highest selection key."""
    s = np.asarray(s, dtype=np.float64)
    if mask_top == 0:
        return _orig["select_topk"](s, top_k, b, bias_mode, renormalize, decision_dtype)
    masked, _ = _orig["select_topk"](s, mask_top)
    s2 = s.copy()
    np.put_along_axis(s2, masked.astype(np.int64), -np.inf, axis=1)
    idx, _ = _orig["select_topk"](s2, top_k, b, bias_mode, False, decision_dtype)
    g = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    if renormalize:
        g = g / g.sum(axis=1, keepdims=True)
    return idx, g


def _f_without_topk(idx, s, n_routed, top_k):
    c, f, p = _orig["balance_stats"](idx, s, n_routed, top_k)
    return c, f * top_k, p


def _softplus_without_sqrt(l):
    return O.softplus(l)


def _layer_drops_shared(x, idx, gates, routed_expert, shared_experts, rows=None):
    return _orig["moe_layer"](x, idx, gates, routed_expert, [], rows)


def _hash_wraps_32bit(token_ids, n_experts, mult=2654435761):
    ids = np.asarray(token_ids, dtype=np.uint64)
    e = ((ids * np.uint64(mult)) & np.uint64(0xFFFFFFFF)) % np.uint64(n_experts)
    return e.astype(np.int32).reshape(-1, 1), np.ones((ids.shape[0], 1))


def _swiglu_gate_up_swapped(U, W_gate, W_up, W_down):
    return _orig["swiglu_ffn"](U, W_up, W_gate, W_down)


def _softmax_over_wrong_axis(l):
    l = np.asarray(l, dtype=np.float64)
    e = np.exp(l - l.max(axis=0, keepdims=True))
    return e / e.sum(axis=0, keepdims=True)


MUTATIONS = [
    ("silu", _silu_without_sigmoid, P.test_swiglu_matches_torch_library, ()),
    ("select_topk", _topk_ties_to_higher_index, P.test_topk_bruteforce, (9, 3)),
    ("select_topk", _mask_ranked_by_raw_score, P.test_masked_topk_bruteforce, (8, 3, 2)),
    ("balance_stats", _f_without_topk, P.test_balance_worked_example, "golden"),
    ("sqrt_softplus", _softplus_without_sqrt, P.test_score_page_readings, "golden"),
    ("moe_layer", _layer_drops_shared, P.test_identical_experts_reduce_to_one_dense_ffn, ()),
    ("hash_route", _hash_wraps_32bit, P.test_hash_route, ()),
    ("swiglu_ffn", _swiglu_gate_up_swapped, P.test_swiglu_bruteforce_tiny, ()),
    ("softmax", _softmax_over_wrong_axis, P.test_scores_match_torch_library, ()),
]


@pytest.mark.parametrize("name,mut,pin,args", MUTATIONS, ids=[m[1].__name__.strip("_") for m in MUTATIONS])
def test_pin_catches_mutation(monkeypatch, golden_dir, name, mut, pin, args):
    monkeypatch.setattr(O, name, mut)
    call_args = (golden_dir,) if args == "golden" else args
    with pytest.raises(AssertionError):
        pin(*call_args)
