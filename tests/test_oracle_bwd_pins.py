"""Pins for the backward oracle: torch autograd in float64 on the same forward
with the discrete decisions held fixed, central finite differences of the
oracle's own forward, and closed forms.  CPU only."""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
import oracle.moe_oracle_bwd as OB


def _inputs(T, H, F, E, act, n_shared, seed, bias=0.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) * 0.6
    wg[0] += bias
    w1 = rng.standard_normal((E, F, H)) * 0.4
    w2 = rng.standard_normal((E, H, F)) * 0.4
    w3 = rng.standard_normal((E, F, H)) * 0.4 if act == O.ACT_SWIGLU else None
    sh = [None, None, None]
    if n_shared:
        sh = [rng.standard_normal((1, F, H)) * 0.4, rng.standard_normal((1, H, F)) * 0.4,
              rng.standard_normal((1, F, H)) * 0.4 if act == O.ACT_SWIGLU else None]
    dy = rng.standard_normal((T, H))
    u = rng.random(T)
    return x, wg, w1, w2, w3, sh, dy, u


def _torch_grads(layer, x, wg, w1, w2, w3, sh, dy, fwd, d_aux, d_z):
    """L = sum(dy * y) + d_aux aux + d_z zloss in float64 autograd, with the
    forward's ids, dispatch and slots fixed and the logits pinned to the
    forward's float32 values (value shifted, gradient unchanged)."""
    T, E, k = layer.T, layer.E, layer.k
    tt = lambda a: None if a is None else torch.tensor(a, dtype=torch.float64, requires_grad=True)
    X, Wg, W1, W2, W3 = tt(x), tt(wg), tt(w1), tt(w2), tt(w3)
    S1, S2, S3 = tt(sh[0]), tt(sh[1]), tt(sh[2])
    l64 = X @ Wg.T
    l = l64 + (torch.tensor(fwd["logits"], dtype=torch.float64) - l64).detach()
    sel = torch.tensor(fwd["selected"], dtype=torch.long)
    ti = torch.arange(T)[:, None]
    if layer.score == O.SCORE_SIGMOID_TOPK:
        s = torch.sigmoid(l)
        g = s[ti, sel]
        P = (s / s.sum(1, keepdim=True)).mean(0)
    else:
        p = torch.softmax(l, 1)
        g = p[ti, sel] if layer.score == O.SCORE_SOFTMAX_TOPK else torch.softmax(l[ti, sel], 1)
        P = p.mean(0)
    if layer.renorm and layer.score != O.SCORE_TOPK_SOFTMAX:
        g = g / g.sum(1, keepdim=True)

    def ffn(xr, a1, a2, a3):
        a = xr @ a1.T
        if layer.act == O.ACT_RELU:
            h = torch.relu(a)
        elif layer.act == O.ACT_GELU:
            h = torch.nn.functional.gelu(a)
        else:
            h = torch.nn.functional.silu(a) * (xr @ a3.T)
        return h @ a2.T

    y = torch.zeros((T, layer.H), dtype=torch.float64)
    ids, slot = fwd["ids"], fwd["slot"]
    for t in range(T):
        for r in range(k):
            if slot[t, r] >= 0:
                e = int(ids[t, r])
                y = y.index_add(0, torch.tensor([t]),
                                g[t, r] * ffn(X[t:t + 1], W1[e], W2[e], None if W3 is None else W3[e]))
    if layer.n_shared:
        y = y + ffn(X, S1[0], S2[0], None if S3 is None else S3[0])
    f = torch.tensor(np.bincount(fwd["selected"].reshape(-1), minlength=E) / (T * k), dtype=torch.float64)
    aux = layer.aux_alpha * E * (f * P).sum()
    lse = torch.logsumexp(l, 1)
    L = (torch.tensor(dy) * y).sum() + d_aux * aux + d_z * layer.z_coef * (lse ** 2).mean()
    L.backward()
    g_ = lambda a: None if a is None else a.grad.numpy()
    return dict(dx=g_(X), dwg=g_(Wg), dw1=g_(W1), dw2=g_(W2), dw3=g_(W3), dsw1=g_(S1), dsw2=g_(S2), dsw3=g_(S3))


CASES = [
    # act, score, renorm, k, n_shared, capacity(cf num, den) or None, random_second, z_coef
    (O.ACT_RELU, O.SCORE_SOFTMAX_TOPK, 0, 1, 0, (5, 4), 0, 0.0),
    (O.ACT_GELU, O.SCORE_SOFTMAX_TOPK, 1, 2, 0, (1, 1), 0, 1e-2),
    (O.ACT_GELU, O.SCORE_SOFTMAX_TOPK, 0, 3, 1, None, 0, 0.0),
    (O.ACT_SWIGLU, O.SCORE_TOPK_SOFTMAX, 0, 2, 1, None, 0, 1e-2),
    (O.ACT_RELU, O.SCORE_SIGMOID_TOPK, 1, 2, 0, (1, 1), 0, 0.0),
    (O.ACT_SWIGLU, O.SCORE_SIGMOID_TOPK, 0, 2, 0, None, 0, 5e-3),
    (O.ACT_GELU, O.SCORE_SOFTMAX_TOPK, 1, 2, 0, (1, 1), 1, 1e-2),
    (O.ACT_RELU, O.SCORE_TOPK_SOFTMAX, 0, 2, 0, (1, 2), 1, 0.0),
]


@pytest.mark.parametrize("case", CASES, ids=[f"c{i}" for i in range(len(CASES))])
def test_backward_matches_autograd(case):
    act, score, renorm, k, n_shared, cf, rnd, zc = case
    T, H, F, E = 40, 6, 10, 5
    x, wg, w1, w2, w3, sh, dy, u = _inputs(T, H, F, E, act, n_shared, seed=hash(case) % 1000, bias=0.8)
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, act=act, score=score, renorm=renorm,
                          cap_mode=O.CAP_DROPLESS if cf is None else O.CAP_CAPACITY,
                          cf_num=1 if cf is None else cf[0], cf_den=1 if cf is None else cf[1],
                          n_shared=n_shared, random_second=rnd, z_coef=zc, aux_alpha=0.05)
    got = OB.layer_backward(layer, x, wg, w1, w2, w3, *sh, dy=dy, uniform=u, d_aux=1.7, d_z=0.9)
    fwd = got["fwd"]
    want = _torch_grads(layer, x, wg, w1, w2, w3, sh, dy, fwd, 1.7, 0.9)
    for n in ("dx", "dwg", "dw1", "dw2", "dw3", "dsw1", "dsw2", "dsw3"):
        if want[n] is None:
            assert got[n] is None or n in ("dw3", "dsw1", "dsw2", "dsw3") and not np.any(got[n]), n
            continue
        np.testing.assert_allclose(got[n], want[n], rtol=1e-9, atol=1e-11, err_msg=n)


def test_some_cases_drop_and_skip():
    """The autograd cases above really exercise dropped and undispatched choices."""
    T, H, F, E = 40, 6, 10, 5
    x, wg, w1, w2, w3, sh, dy, u = _inputs(T, H, F, E, O.ACT_GELU, 0, seed=3, bias=0.8)
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=2, act=O.ACT_GELU, renorm=1, cf_num=1, cf_den=1, random_second=1)
    fwd = O.layer_forward(layer, x, wg, w1, w2, uniform=u)
    assert (fwd["ids"] == -1).any()
    assert ((fwd["ids"] >= 0) & (fwd["slot"] < 0)).any()


def _loss(layer, x, wg, w1, w2, w3, sh, dy, u, d_aux, d_z):
    f = O.layer_forward(layer, x, wg, w1, w2, w3, *sh, uniform=u)
    return float((dy * f["y"]).sum() + d_aux * f["aux"] + d_z * f["zloss"])


@pytest.mark.parametrize("act", [O.ACT_RELU, O.ACT_GELU, O.ACT_SWIGLU])
def test_expert_weight_gradients_finite_differences(act):
    """Expert weights do not move the routing, so central differences of the
    oracle's own forward check dW1, dW2, dW3 and the shared expert's."""
    T, H, F, E = 30, 5, 7, 4
    x, wg, w1, w2, w3, sh, dy, u = _inputs(T, H, F, E, act, 1, seed=7)
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=2, act=act, renorm=1, cf_num=1, cf_den=1, n_shared=1, aux_alpha=0.05)
    got = OB.layer_backward(layer, x, wg, w1, w2, w3, *sh, dy=dy)
    rng = np.random.default_rng(1)
    eps = 1e-6
    mats = {"dw1": w1, "dw2": w2, "dsw1": sh[0], "dsw2": sh[1]}
    if act == O.ACT_SWIGLU:
        mats.update(dw3=w3, dsw3=sh[2])
    for name, W in mats.items():
        for _ in range(6):
            idx = tuple(int(rng.integers(0, s)) for s in W.shape)
            old = W[idx]
            W[idx] = old + eps
            lp = _loss(layer, x, wg, w1, w2, w3, sh, dy, u, 1.0, 1.0)
            W[idx] = old - eps
            lm = _loss(layer, x, wg, w1, w2, w3, sh, dy, u, 1.0, 1.0)
            W[idx] = old
            fd = (lp - lm) / (2 * eps)
            assert abs(got[name][idx] - fd) <= 1e-6 * max(1.0, abs(fd)), (name, idx, got[name][idx], fd)


@pytest.mark.parametrize("score,renorm", [(0, 0), (0, 1), (1, 0), (2, 0), (2, 1)])
def test_router_gradient_finite_differences(score, renorm):
    """dL/dlogits against central differences of gates, aux and z-loss written
    as functions of float64 logits, with the selection held fixed."""
    T, E, k = 12, 6, 2
    rng = np.random.default_rng(10 + score)
    l = rng.standard_normal((T, E)) * 1.5
    layer = O.OracleLayer(T=T, H=1, F=1, E=E, k=k, score=score, renorm=renorm, aux_alpha=0.07, z_coef=0.03)
    sel = O.topk_ids(l.astype(np.float32), k)
    dgate = rng.standard_normal((T, k))
    dgate[3, 1] = 0.0                                    # a choice that adds nothing to y

    def L(lv):
        probs = O.router_probs(lv, score)
        g = O.gate_values(lv, probs, sel, score, renorm)
        return float((dgate * g).sum() + 1.3 * O.aux_loss(probs, sel, E, layer.aux_alpha)
                     + 0.8 * O.z_loss(lv, layer.z_coef))

    got = OB.router_backward(layer, l, sel, dgate, d_aux=1.3, d_z=0.8)
    eps = 1e-6
    for t in range(T):
        for e in range(E):
            lp, lm = l.copy(), l.copy()
            lp[t, e] += eps
            lm[t, e] -= eps
            fd = (L(lp) - L(lm)) / (2 * eps)
            assert abs(got[t, e] - fd) <= 2e-7 * max(1.0, abs(fd)), (t, e, got[t, e], fd)


def test_router_gradient_closed_forms():
    """Equal logits and uniform f: the aux loss is stationary (its gradient is
    zero); the z-loss gradient is 2 coef lse / (E T) per logit."""
    T, E, k = 8, 4, 1
    l = np.zeros((T, E))
    sel = np.array([[t % E] for t in range(T)], dtype=np.int32)
    layer = O.OracleLayer(T=T, H=1, F=1, E=E, k=k, aux_alpha=0.1, z_coef=0.0)
    np.testing.assert_allclose(OB.router_backward(layer, l, sel, np.zeros((T, k))), 0.0, atol=1e-15)
    layer.z_coef = 0.5
    want = 2 * 0.5 * np.log(E) / (E * T)
    np.testing.assert_allclose(OB.router_backward(layer, l, sel, np.zeros((T, k))), want, rtol=1e-13)
    # planted slip: ignoring the renormalisation Jacobian breaks the difference check
    layer = O.OracleLayer(T=2, H=1, F=1, E=3, k=2, renorm=1)
    lv = np.array([[0.3, -0.2, 0.9], [1.1, 0.0, -0.4]])
    s2 = O.topk_ids(lv.astype(np.float32), 2)
    dg = np.array([[1.0, 0.0], [0.5, -0.2]])
    p = O.softmax(lv)
    wrong = np.zeros_like(lv)
    np.add.at(wrong, (np.repeat(np.arange(2), 2), s2.reshape(-1)), dg.reshape(-1))
    wrong = p * (wrong - (wrong * p).sum(1, keepdims=True))
    right = OB.router_backward(layer, lv, s2, dg, d_aux=0.0)
    assert np.abs(wrong - right).max() > 1e-3


# ---------------------------------------------------------------- planted mistakes
# Each plants one plausible slip in the backward oracle (on the CPU, by
# replacing one of its functions for the duration of the test) and checks that
# the autograd pin above catches it.
_orig_router = OB.router_backward
_orig_expert = OB.expert_backward
_orig_act = OB.act_backward


def _gelu_grad_without_z_phi(z):
    from scipy.special import erf
    return 0.5 * (1.0 + erf(np.asarray(z, dtype=np.float64) / np.sqrt(2.0)))


def _swiglu_db_without_sigmoid(act, a, b, dh):
    da, db = _orig_act(act, a, b, dh)
    return (da, dh * a) if act == O.ACT_SWIGLU else (da, db)


def _router_without_aux(layer, logits, selected, dgate, d_aux=1.0, d_z=1.0):
    return _orig_router(layer, logits, selected, dgate, 0.0, d_z)


def _router_zloss_halved(layer, logits, selected, dgate, d_aux=1.0, d_z=1.0):
    return _orig_router(layer, logits, selected, dgate, d_aux, 0.5 * d_z)


def _router_ignores_renorm(layer, logits, selected, dgate, d_aux=1.0, d_z=1.0):
    import dataclasses
    return _orig_router(dataclasses.replace(layer, renorm=0), logits, selected, dgate, d_aux, d_z)


def _expert_dw2_sign(*a, **kw):
    yrow, dX, d1, d2, d3 = _orig_expert(*a, **kw)
    return yrow, dX, d1, -d2, d3


def _expert_dx_without_up(*a, **kw):
    yrow, dX, d1, d2, d3 = _orig_expert(*a, **kw)
    if d3 is None:
        return yrow, dX, d1, d2, d3
    X, w1, w2, act, w3, dyrow = a[:6]
    inter = {}
    _orig_expert(X, w1, w2, act, w3, dyrow, inter)
    return yrow, dX - inter["db"] @ np.asarray(w3, dtype=np.float64), d1, d2, d3


PLANTED = {
    "gelu_grad_without_z_phi": ("gelu_grad", _gelu_grad_without_z_phi, 1),
    "swiglu_db_without_sigmoid": ("act_backward", _swiglu_db_without_sigmoid, 3),
    "router_without_aux": ("router_backward", _router_without_aux, 0),
    "router_zloss_halved": ("router_backward", _router_zloss_halved, 1),
    "router_ignores_renorm": ("router_backward", _router_ignores_renorm, 1),
    "expert_dw2_sign": ("expert_backward", _expert_dw2_sign, 0),
    "expert_dx_without_up": ("expert_backward", _expert_dx_without_up, 3),
}


@pytest.mark.parametrize("name", list(PLANTED))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fake, ci = PLANTED[name]
    act, score, renorm, k, n_shared, cf, rnd, zc = CASES[ci]
    T, H, F, E = 40, 6, 10, 5
    x, wg, w1, w2, w3, sh, dy, u = _inputs(T, H, F, E, act, n_shared, seed=hash(CASES[ci]) % 1000, bias=0.8)
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, act=act, score=score, renorm=renorm,
                          cap_mode=O.CAP_DROPLESS if cf is None else O.CAP_CAPACITY,
                          cf_num=1 if cf is None else cf[0], cf_den=1 if cf is None else cf[1],
                          n_shared=n_shared, random_second=rnd, z_coef=zc, aux_alpha=0.05)
    monkeypatch.setattr(OB, attr, fake)
    got = OB.layer_backward(layer, x, wg, w1, w2, w3, *sh, dy=dy, uniform=u, d_aux=1.7, d_z=0.9)
    monkeypatch.undo()
    want = _torch_grads(layer, x, wg, w1, w2, w3, sh, dy, got["fwd"], 1.7, 0.9)
    caught = [n for n in ("dx", "dwg", "dw1", "dw2", "dw3", "dsw1", "dsw2", "dsw3")
              if want[n] is not None and not np.allclose(got[n], want[n], rtol=1e-9, atol=1e-11)]
    assert caught, f"planted mistake {name} not caught by the autograd pin"
