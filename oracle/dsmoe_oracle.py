"""Reference oracle for the DeepSeekMoE layer forward.

TEST INFRASTRUCTURE ONLY. This module is a plain, slow, float64 CPU
restatement of the formulas on the DeepSeekMoE pages. It exists so that the
CUDA path can be checked against it. Only the test suite, the smoke check of
the graft entry point and the CPU-baseline / reference legs of the benchmark
may import it; the library's own code path never does.

It shares no code with the CUDA path. Inputs arrive as raw bf16 bit patterns
(numpy uint16) or fp32/int arrays and are widened exactly to float64; every
step below is the written definition, with numpy matmul, exp/log and sort as
the only library primitives.

Sources (titles of the pages, with the section / equation):

* [DSMoE] "DeepSeekMoE: Towards Ultimate Expert Specialization" summary
  (heloowird.com): the GShard layer equation, the fine-grained gate equation
  g_{i,t} = s_{i,t} if s_{i,t} in Topk(...) else 0, the shared-expert layer
  equation, and the expert-level balance statistics f_i and P_i.
* [MoE-arch] "MoE architecture: how DeepSeek achieves more" (freedeepseekapi.com),
  section 2 "basic gating": G(x) = Softmax(W_g x), output = sum over Top-K of
  G_i(x) Expert_i(x).
* [V4-ch2] "DeepSeek-V4 book, ch. 2 DeepSeekMoE and MTP": section 2 (V3 sigmoid
  scores, top-k, renormalisation; V4 sqrt(softplus) equation), section 3
  (selection score s~_i = s_i + b_i), section 5 (hash routing equation).
* [MoE-learn] "MoE: sparse activation" (ai.clawlihai.cn), load-balancing
  section: the bias only affects which experts are selected.

Readings where the pages are silent or disagree are listed with each function.
"""
from __future__ import annotations

import math
from typing import Callable, Dict, Iterable, Optional, Sequence, Tuple

import numpy as np

SCORE_SOFTMAX, SCORE_SIGMOID, SCORE_SQRT_SOFTPLUS, ROUTE_HASH = 0, 1, 2, 3
BIAS_NONE, BIAS_SELECT_ONLY, BIAS_IN_LOGITS = 0, 1, 2


# ----------------------------------------------------------------------------------------
# input widening
# ----------------------------------------------------------------------------------------
def bf16_bits_to_f64(bits) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float64.

    A bf16 value is the upper half of an IEEE fp32 word, so shifting the
    pattern into the top 16 bits of a uint32 gives the fp32 value exactly.
    Torch tensors of dtype bfloat16 are accepted too (their bits are read).
    """
    if hasattr(bits, "dtype") and str(bits.dtype) == "torch.bfloat16":
        import torch  # only to read the raw bits of a torch bf16 tensor
        bits = bits.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)
    a = np.asarray(bits, dtype=np.uint16)
    return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _as_f64(a) -> np.ndarray:
    if a is None:
        return None
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        return bf16_bits_to_f64(a)
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return a.astype(np.float64)


# ----------------------------------------------------------------------------------------
# router: affinity, score, selection, gates
# ----------------------------------------------------------------------------------------
def router_logits(x, W_router, b=None, bias_mode: int = BIAS_NONE) -> np.ndarray:
    """Affinity logits l[t,i] = u_t . e_i  ([MoE-arch] section 2: W_g x).

    With bias_mode == BIAS_IN_LOGITS the per-expert bias is added to the logits
    before scoring, which is the form [MoE-arch] section 6 writes as
    Softmax(W_g x + b_i). (Reading: this form is used only for the skewed
    2B-shaped workload; the V3/V4 workloads use the selection-only form.)
    """
    X = _as_f64(x)
    W = _as_f64(W_router)
    l = X @ W.T
    if bias_mode == BIAS_IN_LOGITS:
        l = l + _as_f64(b)[None, :]
    return l


def sigmoid(l):
    """sigma(l) = 1 / (1 + e^{-l})  ([V4-ch2] section 2, V3 scores)."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-np.asarray(l, dtype=np.float64)))


def softplus(l):
    """log(1 + e^l), evaluated without overflow through the identity
    log(1+e^l) = max(l,0) + log(1 + e^{-|l|})."""
    l = np.asarray(l, dtype=np.float64)
    return np.maximum(l, 0.0) + np.log1p(np.exp(-np.abs(l)))


def sqrt_softplus(l):
    """s = sqrt(log(1 + e^l))  ([V4-ch2] section 2 equation)."""
    return np.sqrt(softplus(l))


def softmax(l):
    """Softmax over the routed experts of each token ([MoE-arch] section 2).

    Reading: the softmax runs over the routed experts only; shared experts are
    not routed ([DSMoE], expert-level balance section), so sum_i s_{i,t} = 1.
    """
    l = np.asarray(l, dtype=np.float64)
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=-1, keepdims=True)


def scores(logits, score: int) -> np.ndarray:
    if score == SCORE_SOFTMAX:
        return softmax(logits)
    if score == SCORE_SIGMOID:
        return sigmoid(logits)
    if score == SCORE_SQRT_SOFTPLUS:
        return sqrt_softplus(logits)
    raise ValueError(f"score function {score} has no router scores")


def select_topk(s, top_k: int, b=None, bias_mode: int = BIAS_NONE, renormalize: bool = False,
                decision_dtype=np.float64, mask_top: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Top-K' selection and gates ([DSMoE] gate equation; [V4-ch2] sections 2-3).

    Selection key: s~_i = s_i + b_i when the bias is selection-only
    ([V4-ch2] section 3; [MoE-learn]: the bias only decides who is selected),
    else s_i. Experts are ordered by key descending, ties to the lower index
    (reading: the pages do not say how ties break), and the first K' are kept.

    mask_top = r > 0 is the [DSMoE] expert-specialisation analysis ("disable the top
    routed experts"): per token the r experts ranked first are masked out and the top
    K' of the remaining ones are kept (reading: "ranked first" uses the same key as
    the selection). A K' below the trained one is the same analysis's "fewer
    activated routed experts". Gates are taken over the kept experts.

    Gates use the raw score: g = s_i for the selected experts ([DSMoE] gate
    equation), or g = s_i / sum_{selected} s_j when renormalize is set
    ([V4-ch2] section 2, V3: "top-k then renormalise").

    decision_dtype=np.float32 takes the selection decision in fp32 (the key
    s~ = fp32(s) + fp32(b) rounded to fp32), to re-decide near-tie tokens from
    the scores a kernel computed in fp32.
    """
    s = np.asarray(s, dtype=np.float64)
    T, N = s.shape
    if bias_mode == BIAS_SELECT_ONLY:
        bb = np.asarray(b, dtype=np.float64)[None, :]
        if decision_dtype == np.float32:
            key = (s.astype(np.float32) + bb.astype(np.float32)).astype(np.float64)
        else:
            key = s + bb
    else:
        key = s.astype(np.float32).astype(np.float64) if decision_dtype == np.float32 else s
    order = np.empty((T, N), dtype=np.int64)
    ar = np.arange(N)
    for t in range(T):
        order[t] = np.lexsort((ar, -key[t]))  # primary: key descending; secondary: index ascending
    idx = order[:, mask_top:mask_top + top_k].astype(np.int32)
    g = np.take_along_axis(s, idx.astype(np.int64), axis=1)
    if renormalize:
        g = g / g.sum(axis=1, keepdims=True)
    return idx, g


def hash_route(token_ids, n_experts: int, mult: int = 2654435761) -> Tuple[np.ndarray, np.ndarray]:
    """expert(t) = hash(token_id(t)) mod N_hash  ([V4-ch2] section 5).

    The hash is the multiplicative one the hash workload names,
    token_id * 2654435761, taken as an exact integer product (no 32-bit wrap),
    then reduced mod N. One expert per token, gate 1 (reading: a hashed token
    has no score to weight by).
    """
    ids = np.asarray(token_ids, dtype=np.uint64)
    e = (ids * np.uint64(mult)) % np.uint64(n_experts)  # ids < 2^17, product < 2^49: exact
    return e.astype(np.int32).reshape(-1, 1), np.ones((ids.shape[0], 1), dtype=np.float64)


# ----------------------------------------------------------------------------------------
# expert-level balance statistics
# ----------------------------------------------------------------------------------------
def balance_stats(idx, s, n_routed: int, top_k: int):
    """Expert-level balance statistics ([DSMoE], "Expert-level balance loss").

    counts_i = sum_t 1(token t selects expert i)
    f_i = N' / (K' T) * counts_i
    P_i = (1/T) sum_t s_{i,t}      (s = the raw router scores; zeros when the
                                    layer is hash routed and has none)
    Shared experts take no part (they are never routed).
    """
    idx = np.asarray(idx)
    T = idx.shape[0]
    counts = np.zeros(n_routed, dtype=np.int64)
    for t in range(T):
        for k in range(idx.shape[1]):
            counts[idx[t, k]] += 1
    if T == 0:
        return counts, np.zeros(n_routed), np.zeros(n_routed)
    f = (n_routed / (top_k * T)) * counts.astype(np.float64)
    if s is None:
        P = np.zeros(n_routed)
    else:
        P = np.asarray(s, dtype=np.float64).sum(axis=0) / T
    return counts, f, P


# ----------------------------------------------------------------------------------------
# expert FFN and the layer
# ----------------------------------------------------------------------------------------
def silu(a):
    """SiLU(a) = a * sigma(a) = a / (1 + e^{-a})."""
    return a * sigmoid(a)


def swiglu_ffn(U, W_gate, W_up, W_down) -> np.ndarray:
    """One expert FFN applied to rows U [m, d]: W_down (SiLU(W_gate u) * (W_up u)).

    Reading: the pages write FFN_i(u) and note that real models mostly use the
    three-matrix SwiGLU form ([MoE-learn], parameter-count snippet); no biases.
    Weights use the nn.Linear layout [out, in].
    """
    return swiglu_hidden(U, W_gate, W_up) @ _as_f64(W_down).T


def swiglu_hidden(U, W_gate, W_up) -> np.ndarray:
    """The expert's hidden activation SiLU(W_gate u) * (W_up u) for rows U [m, d]."""
    U = _as_f64(U)
    return silu(U @ _as_f64(W_gate).T) * (U @ _as_f64(W_up).T)


def moe_layer(x, idx, gates, routed_expert: Callable[[int], Tuple], shared_experts: Sequence[Tuple],
              rows: Optional[Iterable[int]] = None) -> np.ndarray:
    """h_t = u_t + sum_{i<=K_s} FFN_i(u_t) + sum_{routed i} g_{i,t} FFN_i(u_t).

    ([DSMoE] shared-expert layer equation.) routed_expert(e) returns the bf16
    (W_gate, W_up, W_down) of routed expert e; shared_experts is the list of
    shared (W_gate, W_up, W_down). rows selects which tokens to evaluate (all
    by default); the result has one row per selected token, in that order.

    Each routed expert is evaluated on the rows that selected it, which is the
    sum over the nonzero gates written expert by expert: the terms with
    g_{i,t} = 0 vanish from the layer equation.
    """
    X = _as_f64(x)
    rows = np.arange(X.shape[0]) if rows is None else np.asarray(list(rows), dtype=np.int64)
    U = X[rows]
    h = U.copy()
    for (Wg, Wu, Wd) in shared_experts:
        h += swiglu_ffn(U, Wg, Wu, Wd)
    sel = np.asarray(idx)[rows]
    g = np.asarray(gates, dtype=np.float64)[rows]
    for e in np.unique(sel):
        r, k = np.nonzero(sel == e)
        Wg, Wu, Wd = routed_expert(int(e))
        h[r] += g[r, k][:, None] * swiglu_ffn(U[r], Wg, Wu, Wd)
    return h


# ----------------------------------------------------------------------------------------
# whole forward
# ----------------------------------------------------------------------------------------
def route(cfg, inputs: Dict) -> Dict[str, np.ndarray]:
    """Router half of the forward: logits -> scores -> top-K' -> gates -> stats."""
    if cfg.score == ROUTE_HASH:
        idx, g = hash_route(inputs["token_ids"], cfg.n_routed, cfg.hash_mult)
        counts, f, P = balance_stats(idx, None, cfg.n_routed, cfg.top_k)
        return dict(idx=idx, gates=g, counts=counts, f=f, P=P, scores=None, logits=None)
    l = router_logits(inputs["x"], inputs["W_router"], inputs.get("b"), cfg.bias_mode)
    s = scores(l, cfg.score)
    idx, g = select_topk(s, cfg.top_k, inputs.get("b"), cfg.bias_mode, cfg.renormalize,
                         mask_top=getattr(cfg, "mask_top", 0))
    counts, f, P = balance_stats(idx, s, cfg.n_routed, cfg.top_k)
    return dict(idx=idx, gates=g, counts=counts, f=f, P=P, scores=s, logits=l)


def forward(cfg, inputs: Dict, rows: Optional[Iterable[int]] = None,
            routing: Optional[Dict] = None) -> Dict[str, np.ndarray]:
    """The full layer forward. Returns the routing outputs and h (float64) for ``rows``."""
    r = route(cfg, inputs) if routing is None else routing
    routed = lambda e: (inputs["W_gate"][e], inputs["W_up"][e], inputs["W_down"][e])
    shared = [(inputs["Ws_gate"][s], inputs["Ws_up"][s], inputs["Ws_down"][s])
              for s in range(cfg.n_shared)]
    h = moe_layer(inputs["x"], r["idx"], r["gates"], routed, shared, rows)
    out = dict(r)
    out["h"] = h
    return out


def combinations(n: int, k: int) -> int:
    """Number of ways a router can pick k of n experts, C(n, k) ([DSMoE] segmentation example)."""
    return math.comb(n, k)


# ----------------------------------------------------------------------------------------
# balance control on top of the statistics
# ----------------------------------------------------------------------------------------
def expert_balance_loss(f, P, alpha1: float) -> float:
    """L_ExpBal = alpha_1 * (1/N') * sum_i f_i P_i  ([DSMoE], "Expert-level balance loss").

    Reading: the page writes the 1/N' factor in front of the sum; it is kept as written.
    """
    f = np.asarray(f, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    return float(alpha1 * (f * P).sum() / f.shape[0])


def device_balance(f, P, group_of, n_groups: int, alpha2: float):
    """Device-level balance ([DSMoE], "Device-level balance loss").

    The routed experts are split into D groups E_1..E_D (group_of[i] = the group of
    expert i); f'_d = (1/|E_d|) sum_{j in E_d} f_j, P'_d = sum_{j in E_d} P_j and
    L_DevBal = alpha_2 * sum_d f'_d P'_d. Returns (f', P', L_DevBal).
    """
    f = np.asarray(f, dtype=np.float64)
    P = np.asarray(P, dtype=np.float64)
    g = np.asarray(group_of)
    f_dev = np.zeros(n_groups)
    P_dev = np.zeros(n_groups)
    size = np.zeros(n_groups)
    for i in range(f.shape[0]):
        f_dev[g[i]] += f[i]
        P_dev[g[i]] += P[i]
        size[g[i]] += 1
    f_dev = np.where(size > 0, f_dev / np.maximum(size, 1), 0.0)
    return f_dev, P_dev, float(alpha2 * (f_dev * P_dev).sum())


def classic_balance_loss(counts, P, top_k: int, alpha: float) -> float:
    """L = alpha * E * sum_i f_i P_i with f_i the fraction of routed assignments that went to
    expert i ("MoE architecture", section 6). Reading: with K' experts per token the
    fraction is counts_i / (K' T), so sum_i f_i = 1 as in the top-1 form."""
    c = np.asarray(counts, dtype=np.float64)
    E = c.shape[0]
    frac = c / c.sum()
    return float(alpha * E * (frac * np.asarray(P, dtype=np.float64)).sum())


def sequence_balance(idx, s, seq_len: int, n_routed: int, beta: float):
    """Sequence-wise balance ([V4-ch2] section 3): for each sequence (consecutive runs of
    seq_len tokens), f_i^seq = fraction of the sequence's tokens that selected expert i and
    p_i^seq = the mean router score of expert i over the sequence; the loss of a sequence is
    beta * sum_i f_i^seq p_i^seq. Reading: the batch loss is the mean over its sequences.
    Returns (f_seq [S, N'], p_seq [S, N'], loss)."""
    idx = np.asarray(idx)
    s = np.asarray(s, dtype=np.float64)
    T = idx.shape[0]
    S = T // seq_len
    f_seq = np.zeros((S, n_routed))
    p_seq = np.zeros((S, n_routed))
    for q in range(S):
        rows = range(q * seq_len, (q + 1) * seq_len)
        for t in rows:
            for e in idx[t]:
                f_seq[q, e] += 1.0
        f_seq[q] /= seq_len
        p_seq[q] = s[q * seq_len:(q + 1) * seq_len].mean(axis=0)
    loss = float(beta * (f_seq * p_seq).sum(axis=1).mean()) if S else 0.0
    return f_seq, p_seq, loss


def bias_update(b, counts, T: int, top_k: int, alpha: float) -> np.ndarray:
    """Auxiliary-loss-free bias update b_i <- b_i + alpha * (f* - f_i) ([V4-ch2] section 3),
    with f_i = counts_i / T the fraction of tokens that selected expert i and f* = K'/N'
    its uniform value. An over-loaded expert's bias falls, an under-loaded one's rises
    ("MoE architecture", section 6 sign rule)."""
    b = np.asarray(b, dtype=np.float64)
    c = np.asarray(counts, dtype=np.float64)
    return b + alpha * (top_k / c.shape[0] - c / T)
