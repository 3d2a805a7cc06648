"""CPU oracle for the backward pass of one Mixture-of-Experts FFN layer.

TEST INFRASTRUCTURE ONLY, like oracle.moe_oracle (which it builds on): only the
test suite, the package's smoke entry and the benchmark's CPU-baseline leg may
import it.  Plain numpy in float64, the chain rule written out stage by stage
in the order the forward pass runs backwards.  It shares no code with the CUDA
library.

Sources (cited by page title and section):
  [EP]  "Expert-parallel MoE training" explainer: the backward pass runs the
        forward's two all-to-alls with their roles swapped (combine's gradient
        travels the dispatch path and vice versa); the aux loss is
        differentiable only through P_i, f_i coming from the non-differentiable
        top-k; the z-loss acts on the router logits directly.
  [SWITCH] "Switch Routing", 2.1: y = p_i(x) E_i(x) (the gate multiplies the
        expert output, so the router learns through the gate).

The discrete decisions of the forward pass (top-k ids, the random second
dispatch, capacity slots) are constants of the backward pass: gradients flow
through the gates, the expert outputs, P_i and the z-loss only.

Readings (also in the design notes):
  * the upstream gradients are dy [T,H] for the layer output and scalars d_aux,
    d_z for the aux loss and the z-loss (1 when both are added to the loss);
  * a choice that is dropped (capacity) or not dispatched (random second
    expert) adds nothing to y, so its gate receives no gradient from y, but it
    still enters the renormalisation of the gates it was selected with;
  * f_i counts selections before any drop and is a constant;
  * the logits are the forward's float32 values, differentiated as reals.

Pinned by tests/test_oracle_bwd_pins.py: torch autograd in float64 on the same
forward with the decisions fixed, central finite differences, closed forms.
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

from oracle import moe_oracle as O


# ---------------------------------------------------------------- activations
def gelu_grad(z: np.ndarray) -> np.ndarray:
    """d/dz of z Phi(z): Phi(z) + z phi(z)."""
    from scipy.special import erf
    z = np.asarray(z, dtype=np.float64)
    return 0.5 * (1.0 + erf(z / math.sqrt(2.0))) + z * np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)


def act_backward(act: int, a: np.ndarray, b: Optional[np.ndarray], dh: np.ndarray):
    """Gradients of the pre-activations from dh.  ReLU/GELU: h = act(a) -> da.
    SwiGLU: h = silu(a) * b -> (da, db), silu'(a) = s (1 + a (1 - s)), s = sigmoid(a)."""
    if act == O.ACT_RELU:
        return dh * (a > 0), None
    if act == O.ACT_GELU:
        return dh * gelu_grad(a), None
    if act == O.ACT_SWIGLU:
        s = 1.0 / (1.0 + np.exp(-a))
        return dh * b * s * (1.0 + a * (1.0 - s)), dh * (a * s)
    raise ValueError(f"unknown activation {act}")


def expert_backward(X: np.ndarray, w1, w2, act: int, w3, dyrow: np.ndarray, inter: Optional[dict] = None):
    """One expert on rows X [n,H] with output gradient dyrow [n,H] (already
    gate-weighted).  Returns (yrow, dX, dW1, dW2, dW3); the forward is
    yrow = act(X W1^T) W2^T, or (silu(X W1^T) * (X W3^T)) W2^T for SwiGLU.
    `inter` (optional dict) receives the intermediates a, b, h, dh, da, db."""
    X = np.asarray(X, dtype=np.float64)
    W1 = np.asarray(w1, dtype=np.float64)
    W2 = np.asarray(w2, dtype=np.float64)
    W3 = None if w3 is None else np.asarray(w3, dtype=np.float64)
    a = X @ W1.T
    b = X @ W3.T if act == O.ACT_SWIGLU else None
    if act == O.ACT_RELU:
        h = np.maximum(a, 0.0)
    elif act == O.ACT_GELU:
        h = O.gelu(a)
    else:
        h = O.silu(a) * b
    yrow = h @ W2.T
    dh = dyrow @ W2                      # yrow = h W2^T
    dW2 = dyrow.T @ h
    da, db = act_backward(act, a, b, dh)
    dW1 = da.T @ X
    dX = da @ W1
    if inter is not None:
        inter.update(a=a, b=b, h=h, dh=dh, da=da, db=db)
    dW3 = None
    if db is not None:
        dW3 = db.T @ X
        dX = dX + db @ W3
    return yrow, dX, dW1, dW2, dW3


# ---------------------------------------------------------------- router
def router_backward(layer: O.OracleLayer, logits: np.ndarray, selected: np.ndarray, dgate: np.ndarray,
                    d_aux: float = 1.0, d_z: float = 1.0) -> np.ndarray:
    """dL/dlogits [T,E] from the gate gradients dgate [T,k] (zero for choices
    that add nothing to y), the aux loss (through P_i) and the z-loss.

    Gates as functions of the logits l of one token (S the sum over the k
    selected of the quantity before renormalisation):
      SOFTMAX_TOPK  g_r = p_{e_r}, or p_{e_r} / S  with p = softmax(l)
      TOPK_SOFTMAX  g = softmax(l_{e_1..e_k})
      SIGMOID_TOPK  g_r = s_{e_r}, or s_{e_r} / S  with s = sigmoid(l)
    aux = alpha E sum_i f_i P_i, P_i = mean_t p_i(t) (softmax, or the sigmoids
    normalised over the experts), f_i = selections / (T k), a constant.
    z-loss = coef mean_t lse_t^2: dl_t = 2 coef lse_t softmax(l_t) / T."""
    l = np.asarray(logits, dtype=np.float64)
    T, E = l.shape
    k = selected.shape[1]
    dl = np.zeros((T, E))
    if T == 0:
        return dl
    t_idx = np.arange(T)[:, None]
    f = np.bincount(selected.reshape(-1), minlength=E).astype(np.float64) / (T * k)
    d_prob = np.tile(d_aux * layer.aux_alpha * E * f / T, (T, 1))   # dL/dP_i(t) from the aux loss
    if layer.score == O.SCORE_SIGMOID_TOPK:
        s = O.sigmoid(l)
        ds = np.zeros((T, E))
        g = s[t_idx, selected]
        if layer.renorm:
            S = g.sum(axis=1, keepdims=True)
            gn = g / S
            ds_sel = (dgate - (dgate * gn).sum(axis=1, keepdims=True)) / S
        else:
            ds_sel = dgate
        np.add.at(ds, (np.repeat(np.arange(T), k), selected.reshape(-1)), ds_sel.reshape(-1))
        # aux: q = s / sum(s) over all experts
        Ss = s.sum(axis=1, keepdims=True)
        q = s / Ss
        ds += (d_prob - (d_prob * q).sum(axis=1, keepdims=True)) / Ss
        dl += ds * s * (1.0 - s)
    else:
        p = O.softmax(l)
        dp = d_prob.copy()
        if layer.score == O.SCORE_SOFTMAX_TOPK:
            g = p[t_idx, selected]
            if layer.renorm:
                S = g.sum(axis=1, keepdims=True)
                gn = g / S
                dp_sel = (dgate - (dgate * gn).sum(axis=1, keepdims=True)) / S
            else:
                dp_sel = dgate
            np.add.at(dp, (np.repeat(np.arange(T), k), selected.reshape(-1)), dp_sel.reshape(-1))
        else:                                                        # TOPK_SOFTMAX
            gs = O.softmax(l[t_idx, selected])
            dl_sel = gs * (dgate - (dgate * gs).sum(axis=1, keepdims=True))
            np.add.at(dl, (np.repeat(np.arange(T), k), selected.reshape(-1)), dl_sel.reshape(-1))
        dl += p * (dp - (dp * p).sum(axis=1, keepdims=True))      # softmax backward
    if layer.z_coef:
        m = l.max(axis=1, keepdims=True)
        lse = m + np.log(np.exp(l - m).sum(axis=1, keepdims=True))
        dl += d_z * 2.0 * layer.z_coef * lse * O.softmax(l) / T
    return dl


# ---------------------------------------------------------------- layer
def layer_backward(layer: O.OracleLayer, x, wg, w1, w2, w3=None, sw1=None, sw2=None, sw3=None, dy=None,
                   logit_add=None, logits=None, uniform=None, d_aux: float = 1.0, d_z: float = 1.0,
                   fwd: Optional[dict] = None, want_rows: bool = False) -> dict:
    """Gradients of L = sum(dy * y) + d_aux * aux + d_z * zloss with respect to
    x, Wg and every expert matrix.  `fwd` (optional) is layer_forward's result
    for the same inputs; `logits` replaces the router GEMM as in layer_forward.
    Returns dx [T,H], dwg [E,H], dw1/dw3 [E,F,H], dw2 [E,H,F], dsw1/dsw3 [1,F,H],
    dsw2 [1,H,F] (None where absent), and dgate [T,k], dlogits [T,E].  With
    want_rows, "experts" maps each expert (E for the shared one) to its tokens
    and row intermediates (ts, rs, dyrow, a, b, h, dh, da, db)."""
    T, E, k, H, F = layer.T, layer.E, layer.k, layer.H, layer.F
    if fwd is None:
        fwd = O.layer_forward(layer, x, wg, w1, w2, w3, sw1, sw2, sw3, logit_add=logit_add, logits=logits,
                              uniform=uniform)
    X = np.asarray(x, dtype=np.float64)
    dY = np.asarray(dy, dtype=np.float64)
    ids, slot, gates, selected = fwd["ids"], fwd["slot"], fwd["gates"], fwd["selected"]
    dX = np.zeros((T, H))
    dgate = np.zeros((T, k))
    dW1 = np.zeros((E, F, H))
    dW2 = np.zeros((E, H, F))
    dW3 = np.zeros((E, F, H)) if layer.act == O.ACT_SWIGLU else None
    rows_out = {}
    # experts: the combine's gradient goes to each kept row (dispatch path), the
    # rows' input gradients return to their tokens (combine path)
    for e in range(E):
        tr = [(t, r) for r in range(k) for t in range(T) if slot[t, r] >= 0 and ids[t, r] == e]
        if not tr:
            continue
        ts = np.array([t for t, _ in tr])
        rs = np.array([r for _, r in tr])
        dyrow = gates[ts, rs][:, None] * dY[ts]
        inter = dict(ts=ts, rs=rs, dyrow=dyrow) if want_rows else None
        yrow, dXr, d1, d2, d3 = expert_backward(X[ts], w1[e], w2[e], layer.act,
                                                None if w3 is None else w3[e], dyrow, inter)
        if want_rows:
            rows_out[e] = inter
        dgate[ts, rs] = (dY[ts] * yrow).sum(axis=1)
        dW1[e], dW2[e] = d1, d2
        if d3 is not None:
            dW3[e] = d3
        np.add.at(dX, ts, dXr)
    out = dict(dsw1=None, dsw2=None, dsw3=None)
    if layer.n_shared:
        inter = dict(ts=np.arange(T), rs=-np.ones(T, dtype=np.int64), dyrow=dY) if want_rows else None
        _, dXs, d1, d2, d3 = expert_backward(X, sw1[0], sw2[0], layer.act, None if sw3 is None else sw3[0], dY,
                                             inter)
        if want_rows:
            rows_out[E] = inter
        dX += dXs
        out.update(dsw1=d1[None], dsw2=d2[None], dsw3=None if d3 is None else d3[None])
    dl = router_backward(layer, fwd["logits"], selected, dgate, d_aux, d_z)
    Wg = np.asarray(wg, dtype=np.float64)
    dWg = dl.T @ X
    dX += dl @ Wg
    out.update(dx=dX, dwg=dWg, dw1=dW1, dw2=dW2, dw3=dW3, dgate=dgate, dlogits=dl, fwd=fwd)
    if want_rows:
        out["experts"] = rows_out
    return out
