"""GPU parity of the backward pass (moe_layer_bwd) against the backward oracle.

The oracle runs the forward on the library's own float32 logits, so both sides
take the same discrete decisions, then differentiates it in float64.

Tolerances, derived from the arithmetic:
  * dx sums a token's rows dxrow = da W1 (+ db W3) (bf16, fp32 accumulation)
    and adds dlogits Wg.  Each row carries the rounded dz's noise carried
    through the contraction over F (sigma^2 = sum_f sigma_dz^2 W1_fh^2, with
    sigma_dz as for the weight gradients below) and its own bf16 rounding
    (relative sigma s_u); the token's rows add in quadrature, and dx's final
    rounding adds at most 2^-8 |dx|: 7 sigma of the rows' noise + 2^-8 |ref|.
  * weight gradients are sums over rows of products of bf16 operands.  One
    rounding to bf16 has relative sigma s_u = 2^-8 / sqrt 3 (8 significant
    bits).  dW2 = dyrow^T h carries two roundings per product.  dW1 (dW3)
    = dz^T x: dz's noise is act'(z) times dh's, plus dz's own rounding; dh sums
    the rounded dyrow against W2, so its noise is s_u sqrt(sum_h dyrow_h^2
    W2_hf^2) (not s_u |dh|: dh may cancel), plus dh's own rounding.  The sums
    over rows cancel, so the error scales with the root of the sum of the
    squared noise terms, not with the result: 7 sigma of that (a Gaussian tail
    beyond it has probability 2.6e-12 per entry), plus 1e-3 |ref| + 1e-6.
  * ReLU's derivative is ambiguous where a pre-activation lies within the fp32
    accumulation bound of zero ((H + 2) 2^-24 sum_h |x_h w_h|): either value is
    correct there, so such a (row, f) pair's whole contribution (|dh| times |x|
    or |W1|) joins the tolerance of dW1 and dx.
  * gate gradients dgate = dy . y_row read the forward's bf16 expert rows: each
    element carries its bf16 rounding (relative sigma s_u) and the forward's
    own noise (sigma = 2.25e-3 rms_row, the figure behind the forward's
    tolerance), so dgate has
        sigma_g = sqrt(sum_h dy_h^2 (s_u^2 y_h^2 + (2.25e-3 rms_row(y))^2))
    and is compared within 6 sigma_g.
  * dlogits is linear in dgate (plus the aux and z-loss terms, which are exact
    up to fp32): its error is J^T (dgate error), J the gate Jacobian.  The bound
    is sum_r |J_rj| 6 sigma_g(r) + 1e-3 |ref| + 1e-7.  When two gates of one token
    have nearly equal dgate, dlogits is their small difference and this bound is
    what keeps the comparison honest.
  * dx adds that propagated router error through |Wg|.  dWg = dlogits^T x sums
    independent per-token errors, each bounded by the dlogits bound (a 6 sigma
    figure): 7/6 of their root-sum-square against x, plus the fp32 accumulation
    bound over T terms, gamma_T sum_t |dlogits x|.
"""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
import oracle.moe_oracle_bwd as OB
from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import synth
from tests.parity_utils import LazyExperts, condition_uniform, oracle_layer, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


def run_fwd_bwd(shape, inp, dy, d_aux, d_z, packed=False, unfused=False):
    cfg = B.make_cfg(shape, flags=B.MOE_FLAG_TRAINING | (B.MOE_FLAG_PACKED_WEIGHTS if packed else 0)
                     | (B.MOE_FLAG_UNFUSED if unfused else 0))
    ws = B.alloc_workspace(cfg)
    T, H, F, E = shape.T, shape.H, shape.F, shape.E
    dev = "cuda"
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    aux = torch.full((2,), float("nan"), device=dev)
    wsrc = B.pack_weights(inp) if packed else inp       # the packed buffers must outlive both calls
    wts = B.make_weights(wsrc)
    B.moe_layer_fwd(cfg, inp["x"], inp["wg"], inp["logit_add"], inp.get("uniform"), wts, y, aux, None, ws)
    sw = shape.act == synth.ACT_SWIGLU
    g = dict(dw1=torch.full((E, F, H), float("nan"), device=dev), dw2=torch.full((E, H, F), float("nan"), device=dev),
             dw3=torch.full((E, F, H), float("nan"), device=dev) if sw else None)
    if shape.n_shared:
        g.update(dsw1=torch.full((1, F, H), float("nan"), device=dev), dsw2=torch.full((1, H, F), float("nan"), device=dev),
                 dsw3=torch.full((1, F, H), float("nan"), device=dev) if sw else None)
    dx = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device=dev)
    dwg = torch.full((E, H), float("nan"), device=dev)
    B.moe_layer_bwd(cfg, inp["x"], inp["wg"], wts, dy, d_aux, d_z, dx, dwg, B.make_weight_grads(g), ws)
    st = B.moe_sync_status(ws)
    assert st == B.MOE_OK, B.strerror(st)
    out = B.workspace_tensors(cfg, ws)
    out.update(y=y, aux=aux, dx=dx, dwg=dwg, grads=g, weights=wsrc)
    return out


# relative sigma of one rounding to bf16: 8 significant bits, so the error is
# uniform within half an ulp and at most the unit roundoff 2^-8 of the value
S_U = 2.0 ** -8 / np.sqrt(3.0)
# weight-gradient bound in sigmas: a Gaussian tail beyond 7 sigma has
# probability 2.6e-12, so the 1.5e8 entries of the largest case expect 4e-4
# false alarms; a wrong term is of the order of the value itself
K_SIG = 7.0


def _worst(got, ref, tol):
    r = np.abs(got - ref) / tol
    i = np.unravel_index(int(np.argmax(r)), r.shape)
    return f"worst at {tuple(int(v) for v in i)}: got {got[i]:.6g} ref {ref[i]:.6g} tol {tol[i]:.3g} ({r[i]:.2f}x)"


def check_backward(shape, inp, out, dy, d_aux, d_z):
    layer = oracle_layer(shape)
    lg = out["logits"].cpu().numpy()
    x64, wg64 = to64(inp["x"]), to64(inp["wg"])
    w1, w2 = LazyExperts(inp["w1"]), LazyExperts(inp["w2"])
    w3 = None if inp["w3"] is None else LazyExperts(inp["w3"])
    sw = [None if inp[n] is None else to64(inp[n]) for n in ("sw1", "sw2", "sw3")]
    uni = None if inp.get("uniform") is None else inp["uniform"].cpu().numpy()
    fwd = O.layer_forward(layer, x64, wg64, w1, w2, w3, sw[0], sw[1], sw[2], logits=lg, uniform=uni)
    np.testing.assert_array_equal(out["ids"].cpu().numpy(), fwd["ids"])
    np.testing.assert_array_equal(out["slot"].cpu().numpy(), fwd["slot"])
    ref = OB.layer_backward(layer, x64, wg64, w1, w2, w3, sw[0], sw[1], sw[2], dy=to64(dy), d_aux=d_aux, d_z=d_z,
                            fwd=fwd, want_rows=True)
    # gate gradients within their derived error (6 sigma_g)
    rows = O.layer_forward(layer, x64, wg64, w1, w2, w3, sw[0], sw[1], sw[2], logits=lg, uniform=uni,
                           want_rows=True)["rows"]
    dy64 = to64(dy)
    T, k, E, H = shape.T, shape.k, shape.E, shape.H
    sig_g = np.zeros((T, k))
    for (t, r), yr in rows.items():
        if r < 0:
            continue
        rms_y = np.sqrt(np.mean(yr ** 2))
        sig_g[t, r] = np.sqrt(np.sum(dy64[t] ** 2 * (S_U ** 2 * yr ** 2 + (2.25e-3 * rms_y) ** 2)))
    gdg = out["dgate"].double().cpu().numpy()
    err = np.abs(gdg - ref["dgate"])
    assert (err <= 6 * sig_g + 1e-6).all(), f"dgate: {int((err > 6 * sig_g + 1e-6).sum())} outside 6 sigma"
    # dlogits: J^T (dgate error) plus fp32 rounding
    sel = fwd["selected"]
    bound_dl = np.zeros((T, E))
    for r in range(k):
        onehot = np.zeros((T, k))
        onehot[:, r] = 1.0
        J = OB.router_backward(layer, lg, sel, onehot, d_aux=0.0, d_z=0.0)
        bound_dl += np.abs(J) * (6 * sig_g[:, r:r + 1])
    gdl = out["dlogits"].double().cpu().numpy()
    tol_dl = bound_dl + 1e-3 * np.abs(ref["dlogits"]) + 1e-7
    bad = np.abs(gdl - ref["dlogits"]) > tol_dl
    assert not bad.any(), f"dlogits: {int(bad.sum())} of {bad.size} outside the propagated bound"
    # Expert rows.  ReLU's derivative at a pre-activation within the fp32
    # accumulation error of zero is ambiguous: such (row, f) pairs may take
    # either value, so their whole contribution joins the tolerance.
    flip_dx = np.zeros((T, H))
    var_dx = np.zeros((T, H))          # noise variance of the sum of a token's dxrow rows
    tol_w = {}
    for e, it in ref["experts"].items():
        ts = it["ts"]
        Xr = x64[ts]
        W1 = sw[0][0] if e == E else w1[e]
        amb = np.zeros_like(it["a"], dtype=bool)
        if shape.act == synth.ACT_RELU:
            delta = (H + 2) * 2.0 ** -24 * (np.abs(Xr) @ np.abs(W1).T)
            amb = np.abs(it["a"]) <= delta
        flip = np.where(amb, np.abs(it["dh"]), 0.0)
        np.add.at(flip_dx, ts, flip @ np.abs(W1))
        # Noise of the bf16 rows (relative sigma s_u per rounding): dh sums the
        # rounded dyrow against W2, so its noise scales with the root of the sum
        # of the squared terms, not with |dh|; dh and dz are rounded once more.
        W2 = sw[1][0] if e == E else w2[e]
        a_, dh = it["a"], it["dh"]
        n_dh = S_U * np.sqrt((it["dyrow"] ** 2) @ (W2 ** 2)) + S_U * np.abs(dh)
        if shape.act == synth.ACT_RELU:
            d_act = (a_ > 0).astype(np.float64)
        elif shape.act == synth.ACT_GELU:
            d_act = OB.gelu_grad(a_)
        else:
            sg = 1.0 / (1.0 + np.exp(-a_))
            d_act = np.abs(it["b"] * sg * (1.0 + a_ * (1.0 - sg)))
        s_da = np.abs(d_act) * n_dh + S_U * np.abs(it["da"])
        t2 = K_SIG * np.sqrt(2.0) * S_U * np.sqrt((it["dyrow"] ** 2).T @ (it["h"] ** 2))
        t1 = K_SIG * np.sqrt((s_da ** 2).T @ (Xr ** 2)) + flip.T @ np.abs(Xr)
        t3 = None
        # dxrow = da W1 (+ db W3): the rounded dz's noise propagated through the
        # contraction over F, and the row's own bf16 rounding
        var_row = (s_da ** 2) @ (W1 ** 2)
        dxr = it["da"] @ W1
        if it["db"] is not None:
            s_db = np.abs(O.silu(a_)) * n_dh + S_U * np.abs(it["db"])
            t3 = K_SIG * np.sqrt((s_db ** 2).T @ (Xr ** 2))
            W3 = sw[2][0] if e == E else w3[e]
            var_row = var_row + (s_db ** 2) @ (W3 ** 2)
            dxr = dxr + it["db"] @ W3
        np.add.at(var_dx, ts, var_row + (S_U * dxr) ** 2)
        tol_w[e] = (t1, t2, t3)
    gx = out["grads"]
    for n, idx in (("dw1", 0), ("dw2", 1), ("dw3", 2), ("dsw1", 0), ("dsw2", 1), ("dsw3", 2)):
        if gx.get(n) is None:
            continue
        gw = gx[n].double().cpu().numpy()
        rw = ref[n]
        tol = np.full(rw.shape, 1e-6) + 1e-3 * np.abs(rw)
        for e, tw in tol_w.items():
            if (e == E) != n.startswith("ds"):
                continue
            tol[0 if e == E else e] += tw[idx]
        bad = np.abs(gw - rw) > tol
        assert np.isfinite(gw).all() and not bad.any(), \
            f"{n}: {int(bad.sum())} of {bad.size} outside the derived bound; {_worst(gw, rw, tol)}"
    # dx = the token's dxrow rows summed in fp32 + dlogits Wg, rounded once to bf16:
    # K_SIG sigma of the rows' noise, the final rounding (at most 2^-8 |dx|), the
    # dlogits bound carried through |Wg|, and the ambiguous ReLU terms
    gdx = out["dx"].double().cpu().numpy()
    tol_dx = K_SIG * np.sqrt(var_dx) + 2.0 ** -8 * np.abs(ref["dx"]) + tol_dl @ np.abs(wg64) + flip_dx + 1e-9
    bad = np.abs(gdx - ref["dx"]) > tol_dx
    assert np.isfinite(gdx).all() and not bad.any(), \
        f"dx: {int(bad.sum())} of {bad.size} outside tolerance in {int(bad.any(axis=1).sum())} rows; " \
        f"{_worst(gdx, ref['dx'], tol_dx)}"
    # dWg = dlogits^T x in fp32: each dlogits error is bounded by tol_dl (a 6 sigma
    # bound), so the weighted sum over tokens has K_SIG sigma <= K_SIG/6 of the
    # root-sum-square of the bounds; plus fp32 accumulation over T terms
    gwg = out["dwg"].double().cpu().numpy()
    gam_t = T * 2.0 ** -24 / (1.0 - T * 2.0 ** -24)
    tol_wg = (K_SIG / 6.0) * np.sqrt((tol_dl ** 2).T @ (x64 ** 2)) \
        + gam_t * (np.abs(ref["dlogits"]).T @ np.abs(x64)) + 1e-12
    bad = np.abs(gwg - ref["dwg"]) > tol_wg
    assert np.isfinite(gwg).all() and not bad.any(), \
        f"dWg: {int(bad.sum())} of {bad.size} outside tolerance; {_worst(gwg, ref['dwg'], tol_wg)}"
    return ref


BWD_SHAPES = {
    "switch_top1": synth.SWITCH_TOP1.replace(name="switch_top1_small", T=1000, H=200, F=392, E=16),
    "gshard_top2": synth.GSHARD_TOP2.replace(name="gshard_top2_small", T=777, H=136, F=520, E=8),
    "ds_k4": synth.DS_HIGHK.replace(name="ds_k4_small", T=1500, H=64, F=256, cf_den=2),
    "wideep": synth.WIDEEP_DROPLESS.replace(name="wideep_small", T=300, H=264, F=136, E=16, k=4),
    "relu_dropless_shared": synth.SWITCH_TOP1.replace(name="relu_dropless_shared", T=517, H=96, F=264, E=6, k=2,
                                                      cap_mode=synth.CAP_DROPLESS, n_shared=1, bias_row0=0.0),
    "sigmoid_zloss_random": synth.GSHARD_TOP2.replace(name="gshard_sigmoid", T=640, H=128, F=192, E=8,
                                                      score=synth.SCORE_SIGMOID_TOPK, renorm=1, z_coef=1e-2,
                                                      random_second=1),
    # T*k/E = 200: the weight gradients take the deep variant (four-stage ring)
    "swiglu_shared_deep": synth.WIDEEP_DROPLESS.replace(name="swiglu_shared_deep", T=800, H=128, F=136, E=8, k=2),
    "swiglu_softmax_renorm": synth.WIDEEP_DROPLESS.replace(name="swiglu_renorm", T=400, H=128, F=128, E=8, k=2,
                                                           score=synth.SCORE_SOFTMAX_TOPK, renorm=1, n_shared=0,
                                                           cap_mode=synth.CAP_CAPACITY, cf_num=1, cf_den=1,
                                                           zipf_skew=0.0, z_coef=1e-3),
}


# T*k > 256*E with H > 512: dh and dxrow run on pairs of SMs with the weights
# read along their columns.  SwiGLU + shared expert: 512-feature tiles in both
# (F = 584, H = 1032: ragged last tiles and a ragged last k block), the W1 -> W3
# switch at Fp = 640; GELU + capacity: 256-feature dh tiles (F = 392).
BWD_PAIR_SHAPES = {
    "swiglu_shared_pairs": synth.WIDEEP_DROPLESS.replace(name="swiglu_shared_pairs", T=1200, H=1032, F=584, E=4,
                                                         k=2),
    "gelu_capacity_pairs": synth.GSHARD_TOP2.replace(name="gelu_capacity_pairs", T=1500, H=520, F=392, E=4),
}


@pytest.mark.parametrize("name", list(BWD_PAIR_SHAPES))
def test_backward_pairs(name):
    shape = BWD_PAIR_SHAPES[name]
    inp = synth.make_inputs(shape, seed=5, device="cuda", scale="unit")
    condition_uniform(shape, inp)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(19)
    dy = torch.randn((shape.T, shape.H), generator=gen, device="cuda").to(torch.bfloat16)
    out = run_fwd_bwd(shape, inp, dy, 1.1, 0.9)
    check_backward(shape, inp, out, dy, 1.1, 0.9)


@pytest.mark.parametrize("name", list(BWD_PAIR_SHAPES))
def test_backward_pairs_packed_matches_unpacked(name):
    """The pair kernels read packed weights as half blocks and plain ones as
    64 x 64 boxes: the same bytes reach shared memory, so every output is
    bitwise the same."""
    shape = BWD_PAIR_SHAPES[name]
    inp = synth.make_inputs(shape, seed=8, device="cuda", scale="unit")
    condition_uniform(shape, inp)
    dy = torch.randn((shape.T, shape.H), device="cuda").to(torch.bfloat16)
    a = run_fwd_bwd(shape, inp, dy, 1.0, 1.0)
    a = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in a.items()}
    b = run_fwd_bwd(shape, inp, dy, 1.0, 1.0, packed=True)
    for n in ("y", "dx", "dwg", "dgate", "dlogits"):
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    for n, v in a["grads"].items():
        if v is not None:
            assert torch.equal(v.view(torch.uint8), b["grads"][n].view(torch.uint8)), n


@pytest.mark.parametrize("name", list(BWD_SHAPES))
def test_backward_small(name):
    shape = BWD_SHAPES[name]
    inp = synth.make_inputs(shape, seed=5, device="cuda", scale="unit")
    condition_uniform(shape, inp)
    gen = torch.Generator(device="cuda")
    gen.manual_seed(17)
    dy = torch.randn((shape.T, shape.H), generator=gen, device="cuda").to(torch.bfloat16)
    out = run_fwd_bwd(shape, inp, dy, 1.3, 0.7)
    check_backward(shape, inp, out, dy, 1.3, 0.7)


def test_backward_full_switch_top1():
    shape = synth.SWITCH_TOP1
    inp = synth.make_inputs(shape, seed=0, device="cuda", scale="unit")
    gen = torch.Generator(device="cuda")
    gen.manual_seed(3)
    dy = torch.randn((shape.T, shape.H), generator=gen, device="cuda").to(torch.bfloat16)
    out = run_fwd_bwd(shape, inp, dy, 1.0, 1.0)
    check_backward(shape, inp, out, dy, 1.0, 1.0)


@pytest.mark.parametrize("name", ["switch_top1", "wideep", "relu_dropless_shared", "swiglu_softmax_renorm"])
def test_backward_packed_matches_unpacked(name):
    """Packed weights change only where the contractions read the weights from:
    every output is bitwise the same (ragged F and the SwiGLU k switch included)."""
    shape = BWD_SHAPES[name]
    inp = synth.make_inputs(shape, seed=8, device="cuda", scale="unit")
    condition_uniform(shape, inp)
    dy = torch.randn((shape.T, shape.H), device="cuda").to(torch.bfloat16)
    a = run_fwd_bwd(shape, inp, dy, 1.0, 1.0)
    b = run_fwd_bwd(shape, inp, dy, 1.0, 1.0, packed=True)
    for n in ("y", "dx", "dwg", "dgate", "dlogits"):
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    for n, v in a["grads"].items():
        if v is not None:
            assert torch.equal(v.view(torch.uint8), b["grads"][n].view(torch.uint8)), n


@pytest.mark.parametrize("name", list(BWD_SHAPES))
def test_backward_fused_matches_unfused(name):
    """dz from the fused dh/dz kernel (dh rounded to bf16 in registers) is
    bitwise the unfused pair's (dh stored in bf16, then read); so is every
    gradient downstream.  Packed weights on the fused side.  Every shape here
    has H <= 512, where the library fuses by default."""
    shape = BWD_SHAPES[name]
    inp = synth.make_inputs(shape, seed=9, device="cuda", scale="unit")
    condition_uniform(shape, inp)
    dy = torch.randn((shape.T, shape.H), device="cuda").to(torch.bfloat16)
    a = run_fwd_bwd(shape, inp, dy, 1.0, 1.0, unfused=True)
    a = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in a.items()}
    b = run_fwd_bwd(shape, inp, dy, 1.0, 1.0, packed=True)
    R = int(a["expert_offset"][-1].item())
    assert torch.equal(a["dz"][:R].view(torch.uint8), b["dz"][:R].view(torch.uint8)), "dz"
    for n in ("dx", "dwg", "dgate", "dlogits"):
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    for n, v in a["grads"].items():
        if v is not None:
            assert torch.equal(v.view(torch.uint8), b["grads"][n].view(torch.uint8)), n


def test_backward_is_deterministic():
    shape = BWD_SHAPES["gshard_top2"]
    inp = synth.make_inputs(shape, seed=6, device="cuda", scale="unit")
    dy = torch.randn((shape.T, shape.H), device="cuda").to(torch.bfloat16)
    a = run_fwd_bwd(shape, inp, dy, 1.0, 1.0)
    b = run_fwd_bwd(shape, inp, dy, 1.0, 1.0)
    for n in ("dx", "dwg"):
        assert torch.equal(a[n].view(torch.uint8), b[n].view(torch.uint8)), n
    for n, v in a["grads"].items():
        if v is not None:
            assert torch.equal(v.view(torch.uint8), b["grads"][n].view(torch.uint8)), n


def test_backward_rejects_unsupported():
    shape = synth.SWITCH_TINY_F32
    cfg = B.make_cfg(shape, flags=B.MOE_FLAG_TRAINING)
    ws = B.alloc_workspace(cfg)
    z = torch.zeros(16, device="cuda")
    w = B.moe_weights(*([z.data_ptr()] * 6))
    g = B.moe_weight_grads(*([z.data_ptr()] * 6))
    with pytest.raises(B.MoeError) as ei:
        B.moe_layer_bwd(cfg, z, z, w, z, 1.0, 1.0, z, z, g, ws)
    assert ei.value.code == B.MOE_EUNSUPPORTED
    cfg2 = B.make_cfg(BWD_SHAPES["switch_top1"])          # forward run without MOE_FLAG_TRAINING
    ws2 = B.alloc_workspace(cfg2)
    with pytest.raises(B.MoeError) as ei:
        B.moe_layer_bwd(cfg2, z, z, w, z, 1.0, 1.0, z, z, g, ws2)
    assert ei.value.code == B.MOE_EINVAL
