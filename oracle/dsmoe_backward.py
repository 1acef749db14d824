"""Reference oracle for the backward pass of the DeepSeekMoE layer.

TEST INFRASTRUCTURE ONLY, like dsmoe_oracle.py (same rules: a plain, slow,
float64 CPU restatement; only the tests, the smoke check and the benchmark's
CPU legs may use it; it shares no code with the CUDA path).

The pages define the forward; the backward is its derivative, written out step
by step below, for an upstream gradient dh = dL/dh of the layer output and an
optional expert-level balance term:

    h_t = u_t + sum_{i<=K_s} FFN_i(u_t) + sum_k g_{t,k} FFN_{e(t,k)}(u_t)
          ([DSMoE] shared-expert layer equation)
    L_bal = alpha * sum_i f_i P_i, P_i = (1/T) sum_t s_{t,i}
          ([DSMoE] "Expert-level balance loss"; the page explains that f_i comes
          from the top-K' indicator, which gives no useful gradient, while P_i
          carries the gradient to the router)

Readings (where the pages say nothing about training):
* the top-K' selection (and its mask / K' variants) is held fixed, as the
  indicator has no gradient; f_i is a constant in L_bal;
* the selection-only bias b receives no gradient ([V4-ch2] section 3 updates it
  by its own rule); a bias added to the logits is a fixed input as well;
* hash-routed tokens have g = 1 and no router, so only the experts and the
  residual carry gradient;
* FFN is the bias-free SwiGLU W_down (SiLU(W_gate u) * (W_up u)) of the forward.

Derivatives used (exact, not approximated):
* SwiGLU: a = W_gate u, b = W_up u, m = SiLU(a) b, y = W_down m. With dy:
  dm = W_down^T dy, dW_down = dy m^T, da = dm b SiLU'(a), db = dm SiLU(a),
  du = W_gate^T da + W_up^T db, dW_gate = da u^T, dW_up = db u^T, where
  SiLU'(a) = sigma(a) (1 + a (1 - sigma(a))).
* gates: dg_{t,k} = <dh_t, FFN_{e(t,k)}(u_t)>. Without renormalisation g = s at
  the kept experts, so ds += dg there; with it, g_k = s_k / Z over the kept set
  and ds_{e(j)} += (dg_j - sum_k dg_k g_k) / Z.
* balance: dL_bal/ds_{t,i} = alpha f_i / T for every token and expert.
* scores: softmax over the routed experts ds -> dl = s (ds - <s, ds>); sigmoid
  dl = s (1 - s) ds; sqrt(softplus(l)) dl = sigma(l) / (2 sqrt(softplus(l))) ds.
* router: l = u W_router^T (+ b), so du += dl W_router and dW_router = dl^T u.
"""
from __future__ import annotations

from typing import Dict, Optional

import numpy as np

from oracle import dsmoe_oracle as O


def silu_grad(a):
    """d SiLU(a) / da = sigma(a) (1 + a (1 - sigma(a)))."""
    sg = O.sigmoid(a)
    return sg * (1.0 + a * (1.0 - sg))


def swiglu_backward(U, W_gate, W_up, W_down, dY):
    """Backward of one expert FFN over rows U [m, d] with output gradient dY [m, d].

    Returns (dU [m, d], dW_gate [F, d], dW_up [F, d], dW_down [d, F]) in float64.
    """
    U = O._as_f64(U)
    Wg, Wu, Wd = O._as_f64(W_gate), O._as_f64(W_up), O._as_f64(W_down)
    dY = np.asarray(dY, dtype=np.float64)
    a = U @ Wg.T
    b = U @ Wu.T
    m = O.silu(a) * b
    dm = dY @ Wd
    dW_down = dY.T @ m
    da = dm * b * silu_grad(a)
    db = dm * O.silu(a)
    dU = da @ Wg + db @ Wu
    return dU, da.T @ U, db.T @ U, dW_down


def score_backward(l, s, ds, score: int):
    """dL/dl from dL/ds for the score function of the router ([MoE-arch] section 2
    softmax; [V4-ch2] section 2 sigmoid and sqrt(softplus))."""
    l = np.asarray(l, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    ds = np.asarray(ds, dtype=np.float64)
    if score == O.SCORE_SOFTMAX:
        return s * (ds - (s * ds).sum(axis=1, keepdims=True))
    if score == O.SCORE_SIGMOID:
        return s * (1.0 - s) * ds
    if score == O.SCORE_SQRT_SOFTPLUS:
        return O.sigmoid(l) / (2.0 * np.sqrt(O.softplus(l))) * ds
    raise ValueError(f"score {score} has no gradient")


def gate_backward(s, idx, gates, dg, renormalize: bool):
    """dL/ds [T, N'] from dL/dg [T, K'] for the kept experts idx [T, K'] (the
    [DSMoE] gate equation g = s, or [V4-ch2] section 2 g = s / sum_kept s)."""
    s = np.asarray(s, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    dg = np.asarray(dg, dtype=np.float64)
    ds = np.zeros_like(s)
    if renormalize:
        g = np.asarray(gates, dtype=np.float64)
        Z = np.take_along_axis(s, idx, axis=1).sum(axis=1, keepdims=True)
        contrib = (dg - (dg * g).sum(axis=1, keepdims=True)) / Z
    else:
        contrib = dg
    for k in range(idx.shape[1]):
        np.add.at(ds, (np.arange(s.shape[0]), idx[:, k]), contrib[:, k])
    return ds


def layer_backward(cfg, inputs: Dict, dh, routing: Optional[Dict] = None, alpha_bal: float = 0.0) -> Dict:
    """Gradients of L = <dh, h> + alpha_bal * sum_i f_i P_i with respect to the layer's
    input and weights, the selection held fixed (module docstring).

    inputs: as for dsmoe_oracle.forward (bf16 bit patterns or arrays). routing: the
    forward's routing (dsmoe_oracle.route) to differentiate through; computed when None.
    Returns float64 dx [T, d], dW_router [N', d] (None for hash routing),
    dW_gate / dW_up [N', F, d], dW_down [N', d, F] and the shared experts' dWs_*.
    """
    r = O.route(cfg, inputs) if routing is None else routing
    X = O._as_f64(inputs["x"])
    dh = np.asarray(dh, dtype=np.float64)
    T, d = X.shape
    N, F = cfg.n_routed, cfg.d_ff
    idx = np.asarray(r["idx"], dtype=np.int64)
    gates = np.asarray(r["gates"], dtype=np.float64)

    dx = dh.copy()  # the residual u_t
    out = dict(dW_gate=np.zeros((N, F, d)), dW_up=np.zeros((N, F, d)), dW_down=np.zeros((N, d, F)))
    Ks, Fs = cfg.n_shared, cfg.d_ff_shared
    out.update(dWs_gate=np.zeros((Ks, Fs, d)), dWs_up=np.zeros((Ks, Fs, d)), dWs_down=np.zeros((Ks, d, Fs)))

    # shared experts: every token, unit weight
    for i in range(Ks):
        dU, dWg, dWu, dWd = swiglu_backward(X, inputs["Ws_gate"][i], inputs["Ws_up"][i], inputs["Ws_down"][i], dh)
        dx += dU
        out["dWs_gate"][i], out["dWs_up"][i], out["dWs_down"][i] = dWg, dWu, dWd

    # routed experts: the rows that kept each expert, output gradient g * dh; the gate
    # gradient dg = <dh, FFN(u)> on the same rows (gate_grads)
    dg = gate_grads(inputs, idx, dh)
    for e in np.unique(idx):
        rows, ks = np.nonzero(idx == e)
        U = X[rows]
        Wg, Wu, Wd = inputs["W_gate"][e], inputs["W_up"][e], inputs["W_down"][e]
        dU, dWg, dWu, dWd = swiglu_backward(U, Wg, Wu, Wd, gates[rows, ks][:, None] * dh[rows])
        np.add.at(dx, rows, dU)
        out["dW_gate"][e], out["dW_up"][e], out["dW_down"][e] = dWg, dWu, dWd

    if cfg.score == O.ROUTE_HASH:
        out.update(dx=dx, dW_router=None, dg=dg, dlogits=None)
        return out

    dl, dx_router, dW_router = router_grads(cfg, r, inputs["x"], inputs["W_router"], dg, alpha_bal)
    dx += dx_router
    out.update(dx=dx, dW_router=dW_router, dg=dg, dlogits=dl)
    return out


def gate_grads(inputs: Dict, idx, dh) -> np.ndarray:
    """dg_{t,k} = <dh_t, FFN_{e(t,k)}(u_t)> [T, K'] for the picks idx, each expert
    evaluated on the rows that kept it (inputs as for dsmoe_oracle.forward)."""
    X = O._as_f64(inputs["x"])
    dh = np.asarray(dh, dtype=np.float64)
    idx = np.asarray(idx, dtype=np.int64)
    dg = np.zeros(idx.shape)
    for e in np.unique(idx):
        rows, ks = np.nonzero(idx == e)
        y = O.swiglu_ffn(X[rows], inputs["W_gate"][e], inputs["W_up"][e], inputs["W_down"][e])
        dg[rows, ks] = (dh[rows] * y).sum(axis=1)
    return dg


def router_grads(cfg, routing: Dict, x, W_router, dg, alpha_bal: float = 0.0):
    """The router's backward: the gate gradients dg and the balance term reach the scores
    (gate_backward, plus alpha f_i / T), then the logits (score_backward), then
    du = dl W_router and dW_router = dl^T u. Returns (dlogits, du, dW_router)."""
    X = O._as_f64(x)
    T = X.shape[0]
    idx = np.asarray(routing["idx"], dtype=np.int64)
    s = np.asarray(routing["scores"], dtype=np.float64)
    ds = gate_backward(s, idx, routing["gates"], dg, cfg.renormalize)
    if alpha_bal:
        ds += alpha_bal * np.asarray(routing["f"], dtype=np.float64)[None, :] / T
    dl = score_backward(routing["logits"], s, ds, cfg.score)
    W_r = O._as_f64(W_router)
    return dl, dl @ W_r, dl.T @ X
