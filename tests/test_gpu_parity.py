"""GPU parity: every stage of the library against the CPU oracle, through the
C ABI, on seeded synthetic inputs."""
import itertools

import numpy as np
import pytest
import torch

import oracle.moe_oracle as O
from expert_dispatch_router_b200 import binding as B
from expert_dispatch_router_b200 import build as build_mod
from expert_dispatch_router_b200 import synth
from tests.parity_utils import check_layer, condition_uniform, run_layer, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")
    build_mod.build()
    B.load()


# Reduced shapes: several tiles in every dimension plus ragged tails
# (H % 64 != 0 -> K tail, F % 256 != 0 -> N tail, T % 128 != 0 -> M tail).
SMALL = {
    "tiny_f32": synth.SWITCH_TINY_F32,
    "switch_top1": synth.SWITCH_TOP1.replace(name="switch_top1_small", T=1000, H=200, F=392, E=16),
    "gshard_top2": synth.GSHARD_TOP2.replace(name="gshard_top2_small", T=777, H=136, F=520, E=8),
    "ds_k4_cf1": synth.DS_HIGHK.replace(name="ds_k4_small", T=1500, H=64, F=256),
    "ds_k4_cf05": synth.DS_HIGHK.replace(name="ds_k4_small_cf05", T=1500, H=64, F=256, cf_den=2),
    "ds_k4_cf025": synth.DS_HIGHK.replace(name="ds_k4_small_cf025", T=1500, H=64, F=256, cf_den=4),
    "wideep": synth.WIDEEP_DROPLESS.replace(name="wideep_small", T=300, H=264, F=136, E=16, k=4),
    "switch_relu_dropless_shared": synth.SWITCH_TOP1.replace(name="relu_dropless_shared", T=517, H=96, F=264,
                                                             E=6, k=2, cap_mode=synth.CAP_DROPLESS, n_shared=1,
                                                             bias_row0=0.0),
    "tiny_f32_swiglu_shared": synth.SWITCH_TINY_F32.replace(name="tiny_f32_swiglu", act=synth.ACT_SWIGLU, k=2,
                                                            n_shared=1, score=synth.SCORE_TOPK_SOFTMAX),
    # more than two 128-row blocks per expert on average: the contractions run on
    # pairs of SMs (256-row tiles; odd block counts leave half a pair tile idle)
    "wideep_2sm": synth.WIDEEP_DROPLESS.replace(name="wideep_2sm", T=600, H=200, F=200, E=4, k=2),
    "gshard_2sm": synth.GSHARD_TOP2.replace(name="gshard_2sm", T=1200, H=136, F=520, E=4),
    "relu_2sm_shared": synth.SWITCH_TOP1.replace(name="relu_2sm_shared", T=900, H=96, F=264, E=3, k=2,
                                                 cap_mode=synth.CAP_DROPLESS, n_shared=1, bias_row0=0.0),
    # skewed loads over 8 experts: groups from a handful of tokens (16-token MMA
    # tiles) to several 256-token tiles, T not a multiple of 16
    "skewed_2sm": synth.WIDEEP_DROPLESS.replace(name="skewed_2sm", T=701, H=136, F=72, E=8, k=3, zipf_skew=2.5),
    # plain (ReLU) contractions of 512 output features per pair tile (two
    # accumulators share each token tile) in both GEMMs: H = 2 * 512 + 8 and
    # F = 512 + 72 leave a ragged last tile, with a shared expert
    "wide_2sm_shared": synth.SWITCH_TOP1.replace(name="wide_2sm_shared", T=1100, H=1032, F=584, E=4, k=2,
                                                 cap_mode=synth.CAP_DROPLESS, n_shared=1, bias_row0=0.0),
    # one SM per tile with 192-column tiles (about 40 row blocks: 3 x 192 columns
    # fit one wave where 128-column tiles need two); H = 568 and F = 392 leave
    # ragged last tiles.  Top-1 with the fused gather and scatter; then k = 2
    # with a shared expert (its weights in half-block boxes too)
    "tiles192_top1": synth.SWITCH_TOP1.replace(name="tiles192_top1", T=4000, H=568, F=392, E=40),
    "tiles192_shared": synth.SWITCH_TOP1.replace(name="tiles192_shared", T=1200, H=568, F=392, E=24, k=2,
                                                 cap_mode=synth.CAP_DROPLESS, n_shared=1, bias_row0=0.0),
    # 384-column tiles (two 192-column accumulators sharing each A stage) in the
    # second contraction: about 40-50 row blocks, so those tiles fit one wave
    # where 192-column ones need two; H = 760 leaves a ragged second tile
    "wide384_top1": synth.SWITCH_TOP1.replace(name="wide384_top1", T=4000, H=760, F=392, E=40),
    "wide384_shared": synth.SWITCH_TOP1.replace(name="wide384_shared", T=1800, H=760, F=392, E=36, k=2,
                                                cap_mode=synth.CAP_DROPLESS, n_shared=1, bias_row0=0.0),
}


@pytest.mark.parametrize("name", list(SMALL))
@pytest.mark.parametrize("seed", [1, 2])
@pytest.mark.parametrize("mode", ["fused", "unfused"])
def test_layer_small(name, seed, mode):
    shape = SMALL[name]
    inp = synth.make_inputs(shape, seed=seed, device="cuda")
    out = run_layer(shape, inp, unfused=mode == "unfused")
    check_layer(shape, inp, out)


@pytest.mark.parametrize("name", ["switch_top1", "gshard_top2", "wideep", "ds_k4_cf05", "wideep_2sm", "gshard_2sm",
                                  "relu_2sm_shared", "skewed_2sm", "wide_2sm_shared"])
def test_fused_matches_unfused(name):
    """Fusing dispatch into the first contraction changes nothing but where A
    comes from: routing, slots, h and the expert outputs are bitwise equal.  The
    fused top-1 combine rounds gate * accumulator once instead of twice.  Layers
    whose contractions run on SM pairs never fuse: every output is bitwise
    equal."""
    shape = SMALL[name]
    inp = synth.make_inputs(shape, seed=9, device="cuda")
    a = run_layer(shape, inp)
    snap = {n: a[n].clone() for n in ("ids", "slot", "expert_offset", "y", "hbuf", "ybuf")}
    b = run_layer(shape, inp, unfused=True)
    used = int(b["expert_offset"][-1])
    live = b["row_token"][:used] >= 0
    for n in ("ids", "slot", "expert_offset"):
        assert torch.equal(snap[n], b[n]), n
    assert torch.equal(snap["hbuf"][:used][live], b["hbuf"][:used][live])
    ya, yb = snap["y"].float(), b["y"].float()
    if a["fused_combine"]:
        assert ((ya - yb).abs() <= 2.0 ** -7 * yb.abs()).all()   # one bf16 rounding apart
    else:
        assert torch.equal(snap["ybuf"][:used][live], b["ybuf"][:used][live])
        assert torch.equal(snap["y"], b["y"])


@pytest.mark.parametrize("name", ["switch_top1", "gshard_top2", "wideep", "ds_k4_cf05", "wideep_2sm", "gshard_2sm"])
def test_layer_small_unit_scale(name):
    shape = SMALL[name]
    inp = synth.make_inputs(shape, seed=3, device="cuda", scale="unit")
    out = run_layer(shape, inp)
    check_layer(shape, inp, out, literal=False)


def test_layer_full_tiny_and_switch():
    for shape in (synth.SWITCH_TINY_F32, synth.SWITCH_TOP1):
        inp = synth.make_inputs(shape, seed=0, device="cuda")
        out = run_layer(shape, inp)
        ref = check_layer(shape, inp, out)
        if shape is synth.SWITCH_TOP1:
            # the biased expert overflows its 160 slots
            assert ref["count"][0] > 160 and ref["kept"][0] == 160


@pytest.mark.slow
@pytest.mark.parametrize("shape", [synth.GSHARD_TOP2, synth.DS_HIGHK, synth.WIDEEP_DROPLESS],
                         ids=["gshard_top2", "ds_k4", "wideep"])
def test_layer_full_size_sampled(shape):
    inp = synth.make_inputs(shape, seed=0, device="cuda")
    out = run_layer(shape, inp)
    rng = np.random.default_rng(0)
    n = 48 if shape is synth.WIDEEP_DROPLESS else 384
    tokens = np.sort(rng.choice(shape.T, n, replace=False))
    tokens[0], tokens[-1] = 0, shape.T - 1
    check_layer(shape, inp, out, tokens=tokens, logit_rows=tokens)


def _layer_ms(shape, inp, reps=7):
    """Median device time of one moe_layer_fwd call (CUDA events)."""
    cfg = B.make_cfg(shape)
    ws = B.alloc_workspace(cfg)
    y = torch.empty((shape.T, shape.H), dtype=torch.bfloat16, device="cuda")
    aux = torch.empty(2, device="cuda")
    w = B.make_weights(inp)
    call = lambda: B.moe_layer_fwd(cfg, inp["x"], inp["wg"], inp["logit_add"], None, w, y, aux, None, ws)
    for _ in range(3):
        call()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        call()
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    assert B.moe_sync_status(ws) == 0
    return float(np.median(times))


def test_ds_k4_cost_follows_kept_rows():
    """The DeepSpeed k=4 capacity sweep ([DS7508] follow-ups: with a fixed
    capacity buffer the step time grows with cf).  Here rows used follow the
    kept assignments, not E*C: at cf = 2.0, E*C is twice the assignments, yet
    the rows (and the time) stay those of cf = 1.0, and halving cf below 1
    shrinks both."""
    used, kept, ms = {}, {}, {}
    for num, den in ((2, 1), (1, 1), (1, 2), (1, 4)):
        shape = synth.DS_HIGHK.replace(cf_num=num, cf_den=den)
        inp = synth.make_inputs(shape, seed=0, device="cuda", experts=shape.E)
        out = run_layer(shape, inp, keep_logits=False)
        cf = num / den
        kept[cf] = int(out["kept_count"].sum())
        rows = int(out["expert_offset"][-1])
        assert rows - kept[cf] < 128 * shape.E
        used[cf] = rows
        ms[cf] = _layer_ms(shape, inp)
    E, A = synth.DS_HIGHK.E, synth.DS_HIGHK.T * synth.DS_HIGHK.k
    C2 = O.capacity(synth.DS_HIGHK.T, E, synth.DS_HIGHK.k, 2, 1)
    assert kept[2.0] == A and E * C2 >= 2 * A                  # nothing dropped, capacity far above the load
    assert used[2.0] < 0.6 * E * C2                            # rows follow kept, not E*C
    assert used[2.0] >= used[1.0] > used[0.5] > used[0.25]
    assert ms[2.0] < 1.25 * ms[1.0]                            # doubling C costs ~nothing
    assert ms[0.25] < ms[1.0]


def test_route_from_logits_bitexact_with_ties():
    rng = np.random.default_rng(5)
    for E, k, T in [(4, 1, 100), (12, 4, 333), (32, 2, 257), (64, 1, 300), (256, 8, 129), (1000, 16, 40)]:
        base = rng.standard_normal((T, E)).astype(np.float32)
        base[: T // 3] = np.round(base[: T // 3] * 2) / 2          # many exact ties
        base[0] = 0.0
        for score, renorm in [(0, 0), (0, 1), (1, 0)]:
            shape = synth.LayerShape("route", T=T, H=8, F=8, E=E, k=k, score=score, renorm=renorm)
            cfg = B.make_cfg(shape)
            ws = B.alloc_workspace(cfg)
            lg = torch.from_numpy(base).cuda()
            ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
            gates = torch.empty((T, k), dtype=torch.float32, device="cuda")
            B.moe_route_from_logits(cfg, lg, None, ids, gates, ws)
            aux = torch.empty(1, device="cuda")
            B.moe_aux_loss(cfg, ws, aux)
            assert B.moe_sync_status(ws) == 0
            layer = O.OracleLayer(T=T, H=8, F=8, E=E, k=k, score=score, renorm=renorm)
            probs, rids, rg = O.route(layer, base)
            np.testing.assert_array_equal(ids.cpu().numpy(), rids)
            np.testing.assert_allclose(gates.cpu().numpy(), rg, rtol=0, atol=1e-5)
            ra = O.aux_loss(probs, rids, E, shape.aux_alpha)
            assert abs(aux.item() - ra) <= 1e-5 * ra


def _slots_gpu(ids_np, E, cap_mode, cf=(1, 1), n_shared=0):
    T, k = ids_np.shape
    shape = synth.LayerShape("slots", T=T, H=8, F=8, E=E, k=k, cap_mode=cap_mode, cf_num=cf[0], cf_den=cf[1],
                             n_shared=n_shared)
    cfg = B.make_cfg(shape)
    ws = B.alloc_workspace(cfg)
    R = B.moe_rows_max(cfg)
    ids = torch.from_numpy(ids_np.astype(np.int32)).cuda()
    slot = torch.empty((T, k), dtype=torch.int32, device="cuda")
    cnt = torch.empty(E, dtype=torch.int32, device="cuda")
    kept = torch.empty(E, dtype=torch.int32, device="cuda")
    off = torch.empty(E + 2, dtype=torch.int32, device="cuda")
    rt = torch.empty(max(R, 1), dtype=torch.int32, device="cuda")
    B.moe_assign_slots(cfg, ids, None, slot, cnt, kept, off, rt, ws)
    st = B.moe_sync_status(ws)
    return st, slot.cpu().numpy(), cnt.cpu().numpy(), kept.cpu().numpy(), off.cpu().numpy(), rt.cpu().numpy()


def test_slots_every_pattern_tiny():
    E, k, T = 3, 2, 4
    pats = list(itertools.permutations(range(E), k))
    for combo in itertools.product(pats, repeat=T):
        ids = np.array(combo, np.int32)
        for cf in [(1, 3), (2, 3), (1, 1)]:      # C = 1, 2, 3
            st, slot, cnt, kept, off, rt = _slots_gpu(ids, E, synth.CAP_CAPACITY, cf)
            assert st == 0
            C = O.capacity(T, E, k, *cf)
            rs, rc, rk = O.assign_slots(ids, E, C)
            np.testing.assert_array_equal(slot, rs)
            np.testing.assert_array_equal(cnt, rc)
            np.testing.assert_array_equal(kept, rk)


@pytest.mark.parametrize("E,k,T,mode", [(64, 1, 5000, 0), (12, 4, 32768, 0), (256, 8, 16384, 1), (1024, 3, 7001, 1),
                                         (7, 7, 2049, 0), (1, 1, 3000, 0),
                                         # beyond the one-launch path: more than 148 CTAs of 1024
                                         # assignments, and E * CTAs above its limit of 32768
                                         (64, 2, 80000, 0), (1024, 2, 20000, 1)])
def test_slots_random_large(E, k, T, mode):
    rng = np.random.default_rng(E * 7 + k)
    w = rng.dirichlet(np.ones(E) * 0.5)
    ids = np.stack([rng.choice(E, k, replace=False, p=w) for _ in range(T)]).astype(np.int32)
    st, slot, cnt, kept, off, rt = _slots_gpu(ids, E, mode, (5, 4), n_shared=1)
    assert st == 0
    C = None if mode == 1 else O.capacity(T, E, k, 5, 4)
    rs, rc, rk = O.assign_slots(ids, E, C)
    np.testing.assert_array_equal(slot, rs)
    np.testing.assert_array_equal(cnt, rc)
    np.testing.assert_array_equal(kept, rk)
    roff = O.row_layout(rk, T, 1)
    np.testing.assert_array_equal(off, roff)
    np.testing.assert_array_equal(rt[:roff[-1]], O.row_tokens(ids, rs, roff, 1))


def test_bad_expert_id_sets_device_status():
    ids = np.zeros((64, 2), np.int32)
    ids[:, 1] = 1
    ids[5, 1] = 9          # E = 4: out of range
    st, slot, *_ = _slots_gpu(ids, 4, synth.CAP_CAPACITY)
    assert st == B.MOE_EDEVICE
    assert slot[5, 1] == -1
    # the status is cleared by the read
    st2, *_ = _slots_gpu(np.zeros((8, 1), np.int32), 4, synth.CAP_CAPACITY)
    assert st2 == 0


def test_empty_batch_layer():
    shape = SMALL["wideep"].replace(T=0)
    inp = synth.make_inputs(shape, seed=0, device="cuda")
    cfg = B.make_cfg(shape)
    ws = B.alloc_workspace(cfg)
    y = torch.empty((0, shape.H), dtype=torch.bfloat16, device="cuda")
    aux = torch.full((1,), float("nan"), device="cuda")
    B.moe_layer_fwd(cfg, inp["x"], inp["wg"], inp["logit_add"], None, B.make_weights(inp), y, aux, None, ws)
    assert B.moe_sync_status(ws) == 0
    assert aux.item() == 0.0


def test_single_token_and_all_to_one_expert():
    shape = SMALL["switch_top1"].replace(T=1)
    inp = synth.make_inputs(shape, seed=4, device="cuda")
    check_layer(shape, inp, run_layer(shape, inp))
    # every token to expert 0 through a large logit offset: all but C dropped, y = 0 for them
    shape = SMALL["switch_top1"]
    inp = synth.make_inputs(shape, seed=4, device="cuda")
    add = torch.zeros((shape.T, shape.E), dtype=torch.float32, device="cuda")
    add[:, 0] = 50.0
    inp["logit_add"] = add
    out = run_layer(shape, inp)
    ref = check_layer(shape, inp, out)
    C = O.capacity(shape.T, shape.E, shape.k, shape.cf_num, shape.cf_den)
    assert ref["kept"][0] == C and ref["kept"].sum() == C
    assert (out["y"][C:] == 0).all()


def test_deterministic_bitwise():
    shape = SMALL["wideep"]
    inp = synth.make_inputs(shape, seed=6, device="cuda")
    a = run_layer(shape, inp)
    snap = {n: a[n].clone() for n in ("ids", "gates", "slot", "expert_offset", "y", "aux")}
    snap["row_token"] = a["row_token"][: int(a["expert_offset"][-1])].clone()
    b = run_layer(shape, inp)
    for n, v in snap.items():
        w = b[n] if n != "row_token" else b["row_token"][: int(b["expert_offset"][-1])]
        assert torch.equal(v.contiguous().view(torch.uint8), w.contiguous().view(torch.uint8)), n   # bits, NaN too


@pytest.mark.parametrize("variant", ["plain", "zloss_random_second", "sigmoid_zloss"])
def test_stage_entry_points_match_layer(variant):
    shape = SMALL["gshard_top2"].replace(n_shared=1)
    if variant == "zloss_random_second":
        shape = shape.replace(z_coef=1e-3, random_second=1)
    elif variant == "sigmoid_zloss":
        shape = shape.replace(z_coef=1e-3, score=synth.SCORE_SIGMOID_TOPK)
    inp = synth.make_inputs(shape, seed=7, device="cuda")
    condition_uniform(shape, inp)
    full = run_layer(shape, inp)
    cfg = B.make_cfg(shape)
    ws = B.alloc_workspace(cfg)
    T, k, E, H = shape.T, shape.k, shape.E, shape.H
    R = B.moe_rows_max(cfg)
    dev = "cuda"
    ids = torch.empty((T, k), dtype=torch.int32, device=dev)
    gates = torch.empty((T, k), dtype=torch.float32, device=dev)
    logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    slot = torch.empty_like(ids)
    cnt = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    off = torch.empty(E + 2, dtype=torch.int32, device=dev)
    rt = torch.empty(R, dtype=torch.int32, device=dev)
    xbuf = torch.empty((R, H), dtype=torch.bfloat16, device=dev)
    ybuf = torch.empty((R, H), dtype=torch.bfloat16, device=dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    aux = torch.full((2,), float("nan"), device=dev)
    B.moe_route(cfg, inp["x"], inp["wg"], None, inp["uniform"], ids, gates, logits, ws)
    B.moe_assign_slots(cfg, ids, gates, slot, cnt, kept, off, rt, ws)
    B.moe_dispatch(cfg, inp["x"], ids, slot, off, xbuf)
    B.moe_expert_ffn(cfg, xbuf, inp["x"], off, B.make_weights(inp), ybuf, ws)
    B.moe_combine(cfg, ybuf, ids, slot, gates, off, y)
    B.moe_aux_loss(cfg, ws, aux)
    assert B.moe_sync_status(ws) == 0
    assert torch.equal(logits, full["logits"])
    for n, v in dict(ids=ids, gates=gates, slot=slot, expert_offset=off, y=y).items():
        assert torch.equal(v, full[n]), n
    # the standalone aux kernel and the slot-fused reduction sum in different orders
    torch.testing.assert_close(aux[0], full["aux"][0], rtol=1e-6, atol=0)
    if shape.z_coef:
        torch.testing.assert_close(aux[1], full["aux"][1], rtol=1e-6, atol=0)
    else:
        assert torch.isnan(aux[1]) and torch.isnan(full["aux"][1])
    used = int(off[-1])
    assert torch.equal(rt[:used], full["row_token"][:used])
    assert torch.equal(ybuf[:used][rt[:used] >= 0], full["ybuf"][:used][full["row_token"][:used] >= 0])


@pytest.mark.parametrize("G,N,K", [(3, 200, 136), (1, 128, 64), (2, 300, 520)])
def test_pack_weight_layout(G, N, K):
    """moe_pack_weight is pure data movement into [G][N/128][K/64][128][64]."""
    w = (torch.arange(G * N * K, device="cuda", dtype=torch.float32) % 251).to(torch.bfloat16).reshape(G, N, K)
    nb, kb = (N + 127) // 128, (K + 63) // 64
    assert B.moe_packed_weight_bytes(G, N, K) == G * nb * kb * 128 * 64 * 2
    got = torch.full((G * nb * kb * 128 * 64,), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.moe_pack_weight(w, got)
    torch.cuda.synchronize()
    pad = torch.zeros((G, nb * 128, kb * 64), dtype=torch.bfloat16, device="cuda")
    pad[:, :N, :K] = w
    want = pad.reshape(G, nb, 128, kb, 64).permute(0, 1, 3, 2, 4).reshape(-1)
    assert torch.equal(got.view(torch.int16), want.view(torch.int16))


@pytest.mark.parametrize("name", ["switch_top1", "gshard_top2", "wideep", "ds_k4_cf05", "tiles192_top1", "tiles192_shared",
                                  "wide384_top1", "wide384_shared", "switch_relu_dropless_shared",
                                  "wideep_2sm", "gshard_2sm", "relu_2sm_shared", "wide_2sm_shared"])
def test_packed_weights_bitwise(name):
    """Packed weights change only where the contractions read B from."""
    shape = SMALL[name]
    inp = synth.make_inputs(shape, seed=11, device="cuda")
    a = run_layer(shape, inp)
    snap = {n: a[n].clone() for n in ("y", "hbuf", "ybuf", "expert_offset", "row_token")}
    b = run_layer(shape, inp, packed=True)
    used = int(b["expert_offset"][-1])
    live = b["row_token"][:used] >= 0
    assert torch.equal(snap["y"], b["y"])
    assert torch.equal(snap["hbuf"][:used][live], b["hbuf"][:used][live])
    if not a["fused_combine"]:
        assert torch.equal(snap["ybuf"][:used][live], b["ybuf"][:used][live])
    check_layer(shape, inp, b)


@pytest.mark.slow
def test_wideep_full_size_repeat_bitwise():
    """Three calls of the full WideEP layer (its contractions run on SM pairs
    over many tiles per pair) give bitwise the same rows and output, packed
    weights or not: nothing in the pipeline depends on timing."""
    shape = synth.WIDEEP_DROPLESS
    inp = synth.make_inputs(shape, seed=0, device="cuda")
    first = None
    for i in range(3):
        out = run_layer(shape, inp, keep_logits=False, packed=i == 1)
        used = int(out["expert_offset"][-1])
        live = out["row_token"][:used] >= 0
        cur = (out["hbuf"][:used][live].clone(), out["ybuf"][:used][live].clone(), out["y"].clone())
        if first is None:
            first = cur
        else:
            for a, b, n in zip(first, cur, ("h", "ybuf", "y")):
                assert torch.equal(a.view(torch.int16), b.view(torch.int16)), (i, n)
        del out
