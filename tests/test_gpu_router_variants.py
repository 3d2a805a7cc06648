"""GPU parity of the router variants: sigmoid scores, the router z-loss and
GShard's random second-expert dispatch, through the C ABI against the oracle."""
import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import synth
from tests.parity_utils import check_layer, condition_uniform, oracle_layer, run_layer

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


GSHARD_SMALL = synth.GSHARD_TOP2.replace(name="gshard_top2_small", T=777, H=136, F=520, E=8)
SWITCH_SMALL = synth.SWITCH_TOP1.replace(name="switch_top1_small", T=1000, H=200, F=392, E=16)
DS_SMALL = synth.DS_HIGHK.replace(name="ds_k4_small_cf05", T=1500, H=64, F=256, cf_den=2)
WIDE_SMALL = synth.WIDEEP_DROPLESS.replace(name="wideep_small", T=300, H=264, F=136, E=16, k=4)

CASES = {
    "gshard_random_second": GSHARD_SMALL.replace(random_second=1),
    "gshard_random_second_zloss": GSHARD_SMALL.replace(random_second=1, z_coef=1e-3),
    "gshard_sigmoid_renorm": GSHARD_SMALL.replace(score=synth.SCORE_SIGMOID_TOPK, renorm=1),
    "switch_sigmoid": SWITCH_SMALL.replace(score=synth.SCORE_SIGMOID_TOPK),
    "switch_zloss": SWITCH_SMALL.replace(z_coef=1e-3),
    "ds_k4_random_second_sigmoid": DS_SMALL.replace(random_second=1, score=synth.SCORE_SIGMOID_TOPK, renorm=1),
    "wideep_zloss_random_second": WIDE_SMALL.replace(z_coef=1e-2, random_second=1),
    "tiny_f32_sigmoid_zloss": synth.SWITCH_TINY_F32.replace(score=synth.SCORE_SIGMOID_TOPK, z_coef=1e-3, k=2,
                                                            random_second=1, renorm=1),
}


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("seed", [1, 2])
def test_layer_variants(name, seed):
    shape = CASES[name]
    inp = synth.make_inputs(shape, seed=seed, device="cuda")
    condition_uniform(shape, inp)
    out = run_layer(shape, inp)
    ref = check_layer(shape, inp, out)
    if shape.random_second:
        # some second choices go, some stay; the first choice always goes
        ids = out["ids"].cpu().numpy()
        assert (ids[:, 0] >= 0).all()
        n_off = int((ids[:, 1] < 0).sum())
        assert 0 < n_off < shape.T
        assert (ids[:, 2:] >= 0).all()
        # the aux loss counts selections, so it equals the no-dispatch-drop value
        assert (ref["selected"][:, 1] >= 0).all()


def test_layer_variants_full_size_switch_zloss_sigmoid():
    shape = synth.SWITCH_TOP1.replace(score=synth.SCORE_SIGMOID_TOPK, z_coef=1e-3)
    inp = synth.make_inputs(shape, seed=0, device="cuda")
    out = run_layer(shape, inp)
    rng = np.random.default_rng(1)
    tokens = np.sort(rng.choice(shape.T, 512, replace=False))
    check_layer(shape, inp, out, tokens=tokens, logit_rows=tokens)


def _route_logits(shape, lg, uni):
    cfg = B.make_cfg(shape)
    ws = B.alloc_workspace(cfg)
    T, k = shape.T, shape.k
    ids = torch.full((T, k), -9, dtype=torch.int32, device="cuda")
    gates = torch.full((T, k), float("nan"), dtype=torch.float32, device="cuda")
    B.moe_route_from_logits(cfg, lg.cuda(), None if uni is None else uni.cuda(), ids, gates, ws)
    aux = torch.full((2,), float("nan"), dtype=torch.float32, device="cuda")
    B.moe_aux_loss(cfg, ws, aux)
    assert B.moe_sync_status(ws) == B.MOE_OK
    return ids.cpu().numpy(), gates.cpu().numpy(), aux.cpu().numpy()


@pytest.mark.parametrize("score,renorm", [(0, 0), (0, 1), (1, 0), (2, 0), (2, 1)])
def test_route_from_logits_variants(score, renorm):
    rng = np.random.default_rng(10 + 3 * score + renorm)
    for E, k, T in [(8, 2, 333), (64, 2, 1000), (256, 8, 129), (1000, 4, 50)]:
        shape = synth.LayerShape("route_variants", T=T, H=64, F=64, E=E, k=k, score=score, renorm=renorm,
                                 z_coef=5e-3, random_second=1)
        lg = torch.from_numpy((rng.standard_normal((T, E)) * 2).astype(np.float32))
        layer = oracle_layer(shape)
        probs, sel, ids0, g0 = O.route_and_dispatch(layer, lg.numpy(), np.zeros(T))
        _, _, g_full = O.route(layer, lg.numpy())
        u = rng.random(T)
        two_g = 2 * g_full[:, 1]
        near = np.abs(u - two_g) < 1e-4
        u[near] = np.clip(two_g[near] + 2e-4, 0, 0.99999)
        uni = torch.from_numpy(u.astype(np.float32))
        ids, gates, aux = _route_logits(shape, lg, uni)
        _, sel, d_ids, d_g = O.route_and_dispatch(layer, lg.numpy(), uni.numpy())
        np.testing.assert_array_equal(ids, d_ids)
        np.testing.assert_allclose(gates, d_g, rtol=0, atol=1e-5)
        ref_aux = O.aux_loss(probs, sel, E, layer.aux_alpha)
        assert abs(aux[0] - ref_aux) <= 1e-5 * abs(ref_aux) + 1e-12
        ref_z = O.z_loss(lg.numpy(), layer.z_coef)
        assert abs(aux[1] - ref_z) <= 1e-5 * abs(ref_z)


def test_random_second_edge_draws():
    """u = 0 keeps every second choice with a positive gate; equal top-2 logits
    under renormalisation give 2 g = 1, so every u in [0, 1) keeps it; a second
    gate of exactly zero (its logit 200 below the first) is never kept."""
    T, E = 64, 8
    shape = synth.LayerShape("edge", T=T, H=64, F=64, E=E, k=2, score=synth.SCORE_TOPK_SOFTMAX,
                             random_second=1)
    lg = torch.full((T, E), -3.0)
    lg[:, 2] = 1.5
    lg[:, 5] = 1.5
    u = torch.linspace(0, 0.999999, T)
    ids, gates, _ = _route_logits(shape, lg, u)
    assert (ids == np.array([2, 5])).all() and (gates == 0.5).all()
    lg2 = torch.full((T, E), -100.0)
    lg2[:, 1] = 100.0
    ids, gates, _ = _route_logits(shape, lg2, torch.zeros(T))
    assert (ids[:, 0] == 1).all() and (ids[:, 1] == -1).all() and (gates[:, 1] == 0).all()
    lg3 = torch.from_numpy(np.random.default_rng(3).standard_normal((T, E)).astype(np.float32))
    ids, gates, _ = _route_logits(shape, lg3, torch.zeros(T))
    assert (ids[:, 1] >= 0).all()


def test_slots_skip_undispatched_choices():
    """An id of -1 takes no slot; the other assignments keep their order."""
    rng = np.random.default_rng(21)
    for E, k, T, mode in [(8, 2, 3000, 0), (16, 4, 777, 1), (3, 2, 4, 0)]:
        shape = synth.LayerShape("slots_minus1", T=T, H=64, F=64, E=E, k=k, cap_mode=mode, cf_num=1, cf_den=2)
        ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
        ids[rng.random(T) < 0.4, 1] = -1
        cfg = B.make_cfg(shape)
        ws = B.alloc_workspace(cfg)
        rows = B.moe_rows_max(cfg)
        d_ids = torch.from_numpy(ids).cuda()
        slot = torch.full((T, k), -9, dtype=torch.int32, device="cuda")
        ec = torch.zeros(E, dtype=torch.int32, device="cuda")
        kc = torch.zeros(E, dtype=torch.int32, device="cuda")
        off = torch.zeros(E + 2, dtype=torch.int32, device="cuda")
        rt = torch.full((rows,), -9, dtype=torch.int32, device="cuda")
        B.moe_assign_slots(cfg, d_ids, None, slot, ec, kc, off, rt, ws)
        assert B.moe_sync_status(ws) == B.MOE_OK
        C = O.layer_capacity(oracle_layer(shape))
        r_slot, r_count, r_kept = O.assign_slots(ids, E, C)
        np.testing.assert_array_equal(slot.cpu().numpy(), r_slot)
        np.testing.assert_array_equal(ec.cpu().numpy(), r_count)
        np.testing.assert_array_equal(kc.cpu().numpy(), r_kept)
        r_off = O.row_layout(r_kept, T, 0)
        np.testing.assert_array_equal(off.cpu().numpy(), r_off)
        used = int(r_off[-1])
        np.testing.assert_array_equal(rt[:used].cpu().numpy(), O.row_tokens(ids, r_slot, r_off, 0))


# ------------------------------------------------------------ "probs" drop policy
def _slots_probs_gpu(shape, ids, gates):
    cfg = B.make_cfg(shape)
    ws = B.alloc_workspace(cfg)
    T, k, E = shape.T, shape.k, shape.E
    rows = B.moe_rows_max(cfg)
    slot = torch.full((T, k), -9, dtype=torch.int32, device="cuda")
    ec = torch.zeros(E, dtype=torch.int32, device="cuda")
    kc = torch.zeros(E, dtype=torch.int32, device="cuda")
    off = torch.zeros(E + 2, dtype=torch.int32, device="cuda")
    rt = torch.full((max(rows, 1),), -9, dtype=torch.int32, device="cuda")
    B.moe_assign_slots(cfg, torch.from_numpy(ids).cuda(), torch.from_numpy(gates).cuda(), slot, ec, kc, off, rt, ws)
    assert B.moe_sync_status(ws) == B.MOE_OK
    return slot.cpu().numpy(), ec.cpu().numpy(), kc.cpu().numpy(), off.cpu().numpy(), rt.cpu().numpy()


@pytest.mark.parametrize("E,k,T,cf,quant,minus1", [
    (3, 2, 4, (1, 2), 0, False), (8, 2, 3001, (1, 2), 0, True), (12, 4, 32768, (1, 2), 64, False),
    (12, 4, 32768, (1, 4), 0, False), (64, 1, 8192, (5, 4), 16, False), (256, 8, 4099, (1, 1), 8, True),
    (5, 3, 20000, (1, 8), 1, False), (4, 2, 40000, (1, 4), 0, False)])
def test_slots_probs_policy_exact(E, k, T, cf, quant, minus1):
    """Exact parity of the per-expert top-C selection, including many equal gates
    (quantised gates; quant=1 makes every gate equal), undispatched ids, and an
    expert with more assignments than the select kernel stages on chip."""
    rng = np.random.default_rng(E * 7 + k)
    skew = np.linspace(0, 2.0, E)
    ids = np.argsort(-(rng.gumbel(size=(T, E)) + skew), axis=1)[:, :k].astype(np.int32)
    if minus1:
        ids[rng.random(T) < 0.3, 1] = -1
    g = rng.random((T, k)).astype(np.float32)
    if quant:
        g = (np.floor(g * quant) / quant).astype(np.float32)
    shape = synth.LayerShape("slots_probs", T=T, H=8, F=8, E=E, k=k, cf_num=cf[0], cf_den=cf[1],
                             drop_policy=synth.DROP_PROBS)
    slot, ec, kc, off, rt = _slots_probs_gpu(shape, ids, g)
    C = O.capacity(T, E, k, *cf)
    r_slot, r_count, r_kept = O.assign_slots_probs(ids, g.astype(np.float64), E, C)
    assert (r_count > C).any()                   # some expert overflows
    if T == 40000:
        assert r_count.max() > 24576
    np.testing.assert_array_equal(slot, r_slot)
    np.testing.assert_array_equal(ec, r_count)
    np.testing.assert_array_equal(kc, r_kept)
    r_off = O.row_layout(r_kept, T, 0)
    np.testing.assert_array_equal(off, r_off)
    used = int(r_off[-1])
    np.testing.assert_array_equal(rt[:used], O.row_tokens(ids, r_slot, r_off, 0))
    if quant == 1:                               # all gates equal: the position policy
        p_slot, _, _ = O.assign_slots(ids, E, C)
        np.testing.assert_array_equal(slot, p_slot)


PROBS_CASES = {
    "switch_probs": SWITCH_SMALL.replace(drop_policy=synth.DROP_PROBS),
    "ds_k4_probs": DS_SMALL.replace(drop_policy=synth.DROP_PROBS),
    "gshard_probs_random_second": GSHARD_SMALL.replace(drop_policy=synth.DROP_PROBS, random_second=1, cf_num=1,
                                                       cf_den=2),
}


@pytest.mark.parametrize("name", list(PROBS_CASES))
def test_layer_probs_policy(name):
    shape = PROBS_CASES[name]
    inp = synth.make_inputs(shape, seed=4, device="cuda")
    condition_uniform(shape, inp)
    out = run_layer(shape, inp)
    ref = check_layer(shape, inp, out)
    assert (ref["count"] > ref["capacity"]).any()


def test_probs_policy_static_variant_unsupported():
    shape = DS_SMALL.replace(drop_policy=synth.DROP_PROBS)
    cfg = B.make_cfg(shape)
    z = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as ei:
        B.moe_assign_slots_static(cfg, z, z, z, z, z, z)
    assert ei.value.code == B.MOE_EUNSUPPORTED
