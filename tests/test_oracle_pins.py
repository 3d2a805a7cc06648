"""Pins for the CPU oracle: printed values from the pages, closed forms,
brute force on tiny inputs, special cases that reduce to library routines, and
planted mistakes that these pins must catch.  CPU only."""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

import oracle.moe_oracle as O
from expert_dispatch_router_b200 import synth


# ------------------------------------------------------------ printed values
def test_capacity_printed_values(golden):
    for c in golden["capacity"]:
        n, d = c["cf"]
        assert O.capacity(c["T"], c["E"], c["k"], n, d) == c["C"], c["source"]


def test_capacity_of_the_five_workloads():
    # capacities stated beside the workload definitions (80, 160, 2048, 10923)
    assert O.capacity(256, 4, 1, 5, 4) == 80
    assert O.capacity(8192, 64, 1, 5, 4) == 160
    assert O.capacity(16384, 32, 2, 2, 1) == 2048
    assert O.capacity(32768, 12, 4, 1, 1) == 10923
    # the DeepSpeed k>2 form ceil((T/E)*cf*k) in exact rationals equals the same C
    from fractions import Fraction
    for (T, E, k, n, d) in [(32768, 12, 4, 1, 2), (32768, 12, 4, 1, 4), (1000, 7, 3, 5, 4)]:
        ds = math.ceil(Fraction(T, E) * Fraction(n, d) * k)
        assert O.capacity(T, E, k, n, d) == ds


def test_min_capacity_clamp():
    assert O.capacity(10, 8, 1, 1, 1) == 2
    assert O.capacity(10, 8, 1, 1, 1, min_capacity=4) == 4


def test_dense_mask_sizes(golden):
    for m in golden["dense_mask_gib"]:
        n, d = m["cf"]
        C = O.capacity(m["T"], m["E"], m["k"], n, d)
        gib = O.dense_mask_bytes(m["T"], m["E"], C, m["elem_bytes"]) / 2**30
        if "gib_2dp" in m:
            assert f"{gib:.2f}" == m["gib_2dp"], m["source"]
        else:
            assert abs(gib - m["gib_approx"]) < 0.1, m["source"]
    # capacities behind those sizes
    assert O.capacity(32768, 12, 4, 1, 2) == 5462
    assert O.capacity(32768, 12, 4, 1, 4) == 2731


def _overflow_example_routing(ex):
    """Tokens 0..511 pick expert 0 first; every other choice goes round-robin
    over experts 1..63, so only expert 0 exceeds C (worked example)."""
    T, E, k = ex["T_local"], ex["E"], ex["k"]
    hot = ex["hot_assignments"]
    choices = []
    rr = 0
    for t in range(T):
        row = []
        if t < hot:
            row.append(0)
        while len(row) < k:
            e = 1 + (rr % (E - 1))
            rr += 1
            if e not in row:
                row.append(e)
        choices.append(row)
    return choices


def test_worked_overflow_example(golden):
    ex = golden["overflow_example"]
    T, E, k = ex["T_local"], ex["E"], ex["k"]
    n, d = ex["cf"]
    logits = synth.constructed_logits(_overflow_example_routing(ex), E, k).numpy()
    layer = O.OracleLayer(T=T, H=8, F=8, E=E, k=k, cf_num=n, cf_den=d)
    probs, ids, gates = O.route(layer, logits)
    C = O.layer_capacity(layer)
    assert T * k == ex["A"] and C == ex["C"]
    slot, count, kept = O.assign_slots(ids, E, C)
    assert count[0] == ex["hot_assignments"] == round(ex["hot_share"] * ex["A"])
    dropped = int((slot < 0).sum())
    assert dropped == ex["dropped"]
    assert f"{100.0 * dropped / ex['A']:.1f}" == ex["drop_pct_1dp"]
    # position policy: the first 40 of expert 0's assignments are kept
    assert (slot[:40, 0] == np.arange(40)).all() and (slot[40:512, 0] == -1).all()
    assert (kept <= C).all()
    # pad vs dropless send bytes
    pad_rows, dl_rows = E * C, T * k
    assert pad_rows == ex["pad_rows"] and dl_rows == ex["dropless_rows"]
    mib = lambda rows: rows * ex["H"] * ex["elem_bytes"] / 2**20
    assert f"{mib(pad_rows):.1f}" == ex["pad_mib_1dp"]
    assert f"{mib(dl_rows):.1f}" == ex["dropless_mib_1dp"]


def test_param_example(golden):
    ex = golden["param_example"]
    p = O.expert_param_count(ex["H"], ex["F"], ex["n_mats"])
    assert p == ex["per_expert"]
    assert f"{ex['experts_per_rank'] * p * 2 / 2**30:.3f}" == ex["rank_gib_3dp"]
    assert f"{ex['E'] * p * 2 / 2**30:.3f}" == ex["total_gib_3dp"]


# ------------------------------------------------------------ top-k / softmax
@pytest.mark.parametrize("E", [2, 3, 4, 5])
def test_topk_bruteforce_all_orderings(E):
    for perm in itertools.permutations(range(E)):
        l = np.array([perm], dtype=np.float32) * 0.5 - 1.0
        for k in range(1, E + 1):
            ids = O.topk_ids(l, k)[0]
            want = [perm.index(v) for v in range(E - 1, E - 1 - k, -1)]
            assert list(ids) == want


def test_topk_ties_go_to_lower_index():
    l = np.zeros((1, 6), dtype=np.float32)
    assert list(O.topk_ids(l, 3)[0]) == [0, 1, 2]
    l = np.array([[0.0, 2.0, 1.0, 2.0, 1.0, -0.0]], dtype=np.float32)
    assert list(O.topk_ids(l, 6)[0]) == [1, 3, 2, 4, 0, 5]


def test_softmax_against_scipy_and_uniform():
    from scipy.special import softmax as sp_softmax
    rng = np.random.default_rng(3)
    l = rng.standard_normal((50, 17)).astype(np.float32) * 3
    np.testing.assert_allclose(O.softmax(l), sp_softmax(l.astype(np.float64), axis=-1), rtol=1e-13, atol=0)
    np.testing.assert_allclose(O.softmax(np.zeros((2, 8), np.float32)), 1 / 8, rtol=0, atol=1e-15)
    # two experts: softmax reduces to the logistic function of the difference
    a, b = 0.7, -0.4
    p = O.softmax(np.array([[a, b]], np.float32))[0]
    assert abs(p[0] - 1 / (1 + math.exp(-(float(np.float32(a)) - float(np.float32(b)))))) < 1e-15


def test_gate_modes():
    rng = np.random.default_rng(4)
    l = rng.standard_normal((64, 9)).astype(np.float32)
    probs = O.softmax(l)
    ids = O.topk_ids(l, 3)
    g_plain = O.gate_values(l, probs, ids, O.SCORE_SOFTMAX_TOPK, 0)
    g_renorm = O.gate_values(l, probs, ids, O.SCORE_SOFTMAX_TOPK, 1)
    g_pre = O.gate_values(l, probs, ids, O.SCORE_TOPK_SOFTMAX, 0)
    np.testing.assert_allclose(g_renorm.sum(1), 1.0, atol=1e-14)
    # top-k-then-softmax equals softmax-then-top-k renormalised
    np.testing.assert_allclose(g_pre, g_renorm, rtol=1e-12, atol=0)
    # gate is the selected probability and is the largest first
    assert (np.diff(g_plain, axis=1) <= 0).all()
    # equal logits: gates 1/E (plain) and 1/k (renormalised)
    z = np.zeros((3, 8), np.float32)
    pz = O.softmax(z)
    idz = O.topk_ids(z, 2)
    np.testing.assert_allclose(O.gate_values(z, pz, idz, 0, 0), 1 / 8, atol=1e-15)
    np.testing.assert_allclose(O.gate_values(z, pz, idz, 0, 1), 1 / 2, atol=1e-15)


def test_router_logits_is_fp32_rounded_dot():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 33)).astype(np.float32)
    wg = rng.standard_normal((5, 33)).astype(np.float32)
    l = O.router_logits(x, wg)
    assert l.dtype == np.float32
    ref = torch.from_numpy(x).double() @ torch.from_numpy(wg).double().T
    np.testing.assert_array_equal(l, ref.float().numpy())
    add = rng.standard_normal((7, 5)).astype(np.float32)
    np.testing.assert_array_equal(O.router_logits(x, wg, add), (ref + torch.from_numpy(add).double()).float().numpy())


# ------------------------------------------------------------ slots
def _slots_by_counting(ids, E, C):
    """Independent definition: pos(t,r) = number of earlier assignments of the
    same expert in (choice rank, token) order."""
    T, k = ids.shape
    slot = np.full((T, k), -1, np.int32)
    for t in range(T):
        for r in range(k):
            e = ids[t, r]
            pos = sum(1 for t2 in range(T) for r2 in range(k)
                      if ids[t2, r2] == e and (r2 < r or (r2 == r and t2 < t)))
            if C is None or pos < C:
                slot[t, r] = pos
    return slot


def test_slots_bruteforce_all_patterns():
    E, k, T = 3, 2, 4
    pats = list(itertools.permutations(range(E), k))          # 6 ordered choices
    for combo in itertools.product(pats, repeat=T):          # 6^4 = 1296
        ids = np.array(combo, dtype=np.int32)
        for C in (1, 2, 3, None):
            slot, count, kept = O.assign_slots(ids, E, C)
            np.testing.assert_array_equal(slot, _slots_by_counting(ids, E, C))
            assert (count == np.bincount(ids.ravel(), minlength=E)).all()


def test_slots_through_routing_on_constructed_logits():
    E, k, T = 3, 2, 4
    rng = np.random.default_rng(6)
    pats = list(itertools.permutations(range(E), k))
    for _ in range(200):
        choices = [pats[i] for i in rng.integers(0, len(pats), T)]
        l = synth.constructed_logits(choices, E, k).numpy()
        ids = O.topk_ids(l, k)
        assert (ids == np.array(choices)).all()
        slot, _, _ = O.assign_slots(ids, E, 2)
        np.testing.assert_array_equal(slot, _slots_by_counting(ids, E, 2))


@pytest.mark.parametrize("E,k,T,cf", [(8, 2, 300, (1, 1)), (5, 3, 257, (1, 2)), (16, 1, 1000, (5, 4)), (6, 4, 129, None)])
def test_slot_invariants(E, k, T, cf):
    rng = np.random.default_rng(E * 100 + k)
    l = (rng.standard_normal((T, E)) + np.linspace(0, 1.5, E)).astype(np.float32)
    ids = O.topk_ids(l, k)
    C = None if cf is None else O.capacity(T, E, k, *cf)
    slot, count, kept = O.assign_slots(ids, E, C)
    assert int(kept.sum()) + int((slot < 0).sum()) == T * k
    for e in range(E):
        s = np.sort(slot[(ids == e) & (slot >= 0)])
        assert (s == np.arange(kept[e])).all()
        assert kept[e] == (count[e] if C is None else min(count[e], C))
    off = O.row_layout(kept, T, 1)
    assert (np.diff(off) >= 0).all() and (off % 128 == 0).all()
    assert all(off[e + 1] - off[e] >= kept[e] for e in range(E))
    rt = O.row_tokens(ids, slot, off, 1)
    for t in range(T):
        for r in range(k):
            if slot[t, r] >= 0:
                assert rt[off[ids[t, r]] + slot[t, r]] == t
    assert (rt[off[E]:off[E] + T] == np.arange(T)).all()
    assert int((rt >= 0).sum()) == int(kept.sum()) + T


# ------------------------------------------------------------ aux loss
def test_aux_closed_forms(golden):
    alpha = golden["aux_uniform"]["alpha"]
    E, k, T = 8, 2, 64
    rng = np.random.default_rng(7)
    # uniform P (equal logits) -> alpha, whatever f is
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    assert abs(O.aux_loss(np.full((T, E), 1 / E), ids, E, alpha) - alpha) < 1e-15
    # uniform f (round robin choices) -> alpha, whatever P is
    ids = np.array([[(t * k + r) % E for r in range(k)] for t in range(T)], np.int32)
    P = O.softmax(rng.standard_normal((T, E)).astype(np.float32))
    assert abs(O.aux_loss(P, ids, E, alpha) - alpha) < 1e-15
    # everything on one expert with one-hot probabilities -> alpha * E
    l = np.full((T, E), -1e4, np.float32)
    l[:, 3] = 0.0
    P1 = O.softmax(l)
    ids1 = np.full((T, 1), 3, np.int32)
    assert abs(O.aux_loss(P1, ids1, E, alpha) - alpha * E) < 1e-12


# ------------------------------------------------------------ expert FFN / layer
def _torch_mlp(x, w1, w2, act, w3=None):
    x = torch.from_numpy(np.asarray(x, np.float64))
    a = Fnn.linear(x, torch.from_numpy(np.asarray(w1, np.float64)))
    if act == O.ACT_RELU:
        h = Fnn.relu(a)
    elif act == O.ACT_GELU:
        h = Fnn.gelu(a, approximate="none")
    else:
        h = Fnn.silu(a) * Fnn.linear(x, torch.from_numpy(np.asarray(w3, np.float64)))
    return Fnn.linear(h, torch.from_numpy(np.asarray(w2, np.float64))).numpy()


@pytest.mark.parametrize("act", [O.ACT_RELU, O.ACT_GELU, O.ACT_SWIGLU])
def test_single_expert_is_dense_mlp(act):
    T, H, F = 40, 24, 40
    rng = np.random.default_rng(8)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((1, H)).astype(np.float32)
    w1 = rng.standard_normal((1, F, H)) / 5
    w2 = rng.standard_normal((1, H, F)) / 6
    w3 = rng.standard_normal((1, F, H)) / 5
    layer = O.OracleLayer(T=T, H=H, F=F, E=1, k=1, act=act, cf_num=1, cf_den=1)
    out = O.layer_forward(layer, x, wg, w1, w2, w3 if act == O.ACT_SWIGLU else None)
    np.testing.assert_array_equal(out["gates"], 1.0)
    ref = _torch_mlp(x, w1[0], w2[0], act, w3[0])
    np.testing.assert_allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def test_all_experts_dropless_is_probability_mixture():
    T, H, F, E = 30, 16, 24, 5
    rng = np.random.default_rng(9)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)).astype(np.float32)
    w1 = rng.standard_normal((E, F, H)) / 4
    w2 = rng.standard_normal((E, H, F)) / 5
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=E, act=O.ACT_GELU, cap_mode=O.CAP_DROPLESS)
    out = O.layer_forward(layer, x, wg, w1, w2)
    p = O.softmax(O.router_logits(x, wg))
    ref = sum(p[:, e:e + 1] * _torch_mlp(x, w1[e], w2[e], O.ACT_GELU) for e in range(E))
    np.testing.assert_allclose(out["y"], ref, rtol=1e-11, atol=1e-12)


def test_dropped_token_is_exactly_zero_and_shared_expert_alone():
    T, H, F, E, k = 12, 8, 16, 2, 1
    rng = np.random.default_rng(10)
    x = rng.standard_normal((T, H))
    choices = [[0]] * T                                    # all to expert 0
    logits = synth.constructed_logits(choices, E, k).numpy()
    w1 = rng.standard_normal((E, F, H))
    w2 = rng.standard_normal((E, H, F))
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, cf_num=1, cf_den=4)   # C = 2
    out = O.layer_forward(layer, x, None, w1, w2, logits=logits)
    assert out["capacity"] == 2
    assert (out["y"][2:] == 0.0).all() and (np.abs(out["y"][:2]).sum() > 0)
    # shared expert with zero routed weights: y = shared FFN(x)
    sw1 = rng.standard_normal((1, F, H))
    sw2 = rng.standard_normal((1, H, F))
    layer_s = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, cap_mode=O.CAP_DROPLESS, n_shared=1)
    out = O.layer_forward(layer_s, x, None, np.zeros_like(w1), np.zeros_like(w2), sw1=sw1, sw2=sw2, logits=logits)
    np.testing.assert_allclose(out["y"], _torch_mlp(x, sw1[0], sw2[0], O.ACT_RELU), rtol=1e-12, atol=1e-12)


def test_token_sample_matches_full_layer():
    T, H, F, E, k = 50, 8, 12, 6, 2
    rng = np.random.default_rng(11)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)).astype(np.float32)
    w1 = rng.standard_normal((E, F, H))
    w2 = rng.standard_normal((E, H, F))
    layer = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, renorm=1, cf_num=3, cf_den=4)
    full = O.layer_forward(layer, x, wg, w1, w2)
    tok = [3, 17, 49, 0]
    part = O.layer_forward(layer, x, wg, w1, w2, tokens=tok)
    # same rows, different matmul batch: equal up to the library's rounding order
    np.testing.assert_allclose(part["y"], full["y"][tok], rtol=1e-13, atol=1e-13)


# ------------------------------------------------------------ planted mistakes
def test_planted_mistakes_are_caught(monkeypatch, golden):
    """Each plausible slip in the oracle must make one of the pins above fail."""
    # 1. floor instead of ceil in the capacity
    bad_cap = lambda T, E, k, n, d, m=0: max((T * k * n) // (E * d), m)
    assert any(bad_cap(c["T"], c["E"], c["k"], *c["cf"]) != c["C"] for c in golden["capacity"])

    # 2. slot walk in (token, rank) order instead of (rank, token)
    def bad_walk(ids, E, C):
        T, k = ids.shape
        fill = [0] * E
        slot = np.full((T, k), -1, np.int32)
        for t in range(T):
            for r in range(k):
                e = ids[t, r]
                if C is None or fill[e] < C:
                    slot[t, r] = fill[e]
                fill[e] += 1
        return slot
    found = False
    for combo in itertools.product(list(itertools.permutations(range(3), 2)), repeat=4):
        ids = np.array(combo, np.int32)
        if not np.array_equal(bad_walk(ids, 3, 2), _slots_by_counting(ids, 3, 2)):
            found = True
            break
    assert found

    # 3. aux loss without k in the denominator of f
    T, E, k = 64, 8, 2
    ids = np.array([[(t * k + r) % E for r in range(k)] for t in range(T)], np.int32)
    f_bad = np.bincount(ids.ravel(), minlength=E) / T
    assert abs(golden["aux_uniform"]["alpha"] * E * np.sum(f_bad / E) - golden["aux_uniform"]["alpha"]) > 1e-3

    # 4. tie broken toward the higher index
    l = np.zeros((1, 6), np.float32)
    bad = np.lexsort((-np.arange(6)[None, :], -l), axis=-1)[0, :3]
    assert list(bad) != [0, 1, 2]

    # 5. weight used untransposed (x @ w1 instead of x @ w1.T) breaks the MLP pin
    T, H, F = 6, 4, 4
    rng = np.random.default_rng(12)
    x, w1, w2 = rng.standard_normal((T, H)), rng.standard_normal((F, H)), rng.standard_normal((H, F))
    bad_y = np.maximum(x @ w1, 0) @ w2
    assert not np.allclose(bad_y, _torch_mlp(x, w1, w2, O.ACT_RELU))

    # 6. renormalisation forgotten breaks sum-to-one
    lg = rng.standard_normal((5, 6)).astype(np.float32)
    pr = O.softmax(lg)
    idk = O.topk_ids(lg, 2)
    assert not np.allclose(pr[np.arange(5)[:, None], idk].sum(1), 1.0)


# ------------------------------------------------------------ router variants
def test_sigmoid_scores_against_expit():
    from scipy.special import expit
    rng = np.random.default_rng(31)
    l = (rng.standard_normal((40, 11)) * 5).astype(np.float32)
    np.testing.assert_allclose(O.sigmoid(l), expit(l.astype(np.float64)), rtol=1e-14, atol=0)
    assert O.sigmoid(np.float32(0.0)) == 0.5
    assert O.sigmoid(np.float32(-200.0)) < 1e-80 and O.sigmoid(np.float32(200.0)) == 1.0
    # P for sigmoid scores: normalised over the experts
    P = O.router_probs(l, O.SCORE_SIGMOID_TOPK)
    np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-14)
    a, b = 0.3, -1.2
    P2 = O.router_probs(np.array([[a, b]], np.float32), O.SCORE_SIGMOID_TOPK)[0]
    sa, sb = expit(float(np.float32(a))), expit(float(np.float32(b)))
    assert abs(P2[0] - sa / (sa + sb)) < 1e-15
    # equal logits: P = 1/E, so the aux loss is alpha whatever f is
    z = np.full((16, 8), 0.7, np.float32)
    Pz = O.router_probs(z, O.SCORE_SIGMOID_TOPK)
    np.testing.assert_allclose(Pz, 1 / 8, atol=1e-15)
    ids = np.array([[t % 3, 3 + t % 5] for t in range(16)], np.int32)
    assert abs(O.aux_loss(Pz, ids, 8, 1e-2) - 1e-2) < 1e-15
    # softmax scores are unchanged by the new branch
    np.testing.assert_array_equal(O.router_probs(l, O.SCORE_SOFTMAX_TOPK), O.softmax(l))


def test_sigmoid_gates():
    from scipy.special import expit
    rng = np.random.default_rng(32)
    l = rng.standard_normal((50, 9)).astype(np.float32)
    layer = O.OracleLayer(T=50, H=1, F=1, E=9, k=3, score=O.SCORE_SIGMOID_TOPK)
    probs, ids, g = O.route(layer, l)
    # selection is the same as under softmax (sigmoid is monotone)
    np.testing.assert_array_equal(ids, O.topk_ids(l, 3))
    sel = l.astype(np.float64)[np.arange(50)[:, None], ids]
    np.testing.assert_allclose(g, expit(sel), rtol=1e-14)
    assert (np.diff(g, axis=1) <= 0).all()
    g_r = O.gate_values(l, probs, ids, O.SCORE_SIGMOID_TOPK, 1)
    np.testing.assert_allclose(g_r.sum(1), 1.0, atol=1e-14)
    np.testing.assert_allclose(g_r, expit(sel) / expit(sel).sum(1, keepdims=True), rtol=1e-14)


def test_z_loss_closed_forms():
    from scipy.special import logsumexp
    rng = np.random.default_rng(33)
    l = (rng.standard_normal((70, 13)) * 4).astype(np.float32)
    want = 1e-3 * np.mean(logsumexp(l.astype(np.float64), axis=1) ** 2)
    assert abs(O.z_loss(l, 1e-3) - want) <= 1e-15 * want
    # equal logits c over E experts: lse = c + ln E
    for c, E in [(0.0, 8), (2.5, 64), (-7.0, 3)]:
        z = np.full((5, E), c, np.float32)
        assert abs(O.z_loss(z, 0.1) - 0.1 * (c + math.log(E)) ** 2) < 1e-13
    # one dominant logit: lse -> that logit, stable at large magnitudes
    big = np.full((2, 4), -1e4, np.float32)
    big[:, 1] = 1000.0
    assert abs(O.z_loss(big, 1.0) - 1e6) < 1e-6
    assert O.z_loss(np.zeros((0, 4), np.float32), 1.0) == 0.0
    assert O.z_loss(l, 0.0) == 0.0
    # planted slips: the mean of lse (not squared) and the max instead of lse
    assert abs(1e-3 * np.mean(logsumexp(l.astype(np.float64), axis=1)) - want) > 1e-6
    assert abs(1e-3 * np.mean(l.max(axis=1).astype(np.float64) ** 2) - want) > 1e-6


def test_random_second_dispatch_rule():
    T = 1000
    ids = np.tile(np.array([[3, 5]], np.int32), (T, 1))
    # second gate g: kept iff u < 2 g; on the grid u = i / T exactly ceil(2 g T) are kept
    for g1 in (0.0, 0.05, 0.25, 0.3125, 0.5):
        gates = np.tile(np.array([[1 - g1, g1]]), (T, 1))
        u = np.arange(T) / T
        d_ids, d_g = O.random_second_dispatch(ids, gates, u)
        kept = d_ids[:, 1] >= 0
        assert int(kept.sum()) == math.ceil(2 * g1 * T)
        assert (d_ids[:, 0] == 3).all() and (d_g[:, 0] == 1 - g1).all()
        assert (d_g[~kept, 1] == 0).all() and (d_g[kept, 1] == g1).all()
        assert (d_ids[kept, 1] == 5).all() and (d_ids[~kept, 1] == -1).all()
    # u = 0 keeps any positive gate; the inputs are not modified
    gates = np.tile(np.array([[0.9, 1e-30]]), (T, 1))
    d_ids, _ = O.random_second_dispatch(ids, gates, np.zeros(T))
    assert (d_ids[:, 1] == 5).all() and (ids[:, 1] == 5).all()
    # k=3: only the rank-1 choice is subject to the draw
    ids3 = np.tile(np.array([[0, 1, 2]], np.int32), (4, 1))
    g3 = np.tile(np.array([[0.5, 0.3, 0.2]]), (4, 1))
    d3, _ = O.random_second_dispatch(ids3, g3, np.array([0.1, 0.59, 0.6, 0.99]))
    np.testing.assert_array_equal(d3, [[0, 1, 2], [0, 1, 2], [0, -1, 2], [0, -1, 2]])


def test_slots_skip_minus_one_equals_extra_expert():
    """An undispatched choice (-1) takes no slot: the slots equal those of the
    same assignments with -1 sent to an extra expert E that nobody reads."""
    E, k, T = 3, 2, 4
    pats = list(itertools.permutations(range(E), k))
    rng = np.random.default_rng(34)
    for combo in itertools.product(pats, repeat=T):
        ids = np.array(combo, dtype=np.int32)
        ids[rng.random(T) < 0.5, 1] = -1
        alt = np.where(ids < 0, E, ids).astype(np.int32)
        for C in (1, 2, None):
            slot, count, kept = O.assign_slots(ids, E, C)
            s2, c2, k2 = O.assign_slots(alt, E + 1, C)
            np.testing.assert_array_equal(slot[ids >= 0], s2[ids >= 0])
            assert (slot[ids < 0] == -1).all()
            np.testing.assert_array_equal(count, c2[:E])
            np.testing.assert_array_equal(kept, k2[:E])


def test_layer_random_second_counts_selections_and_drops_rows():
    E, k, T, H, F = 4, 2, 40, 8, 16
    rng = np.random.default_rng(35)
    x = rng.standard_normal((T, H))
    wg = rng.standard_normal((E, H)) * 0.5
    w1 = rng.standard_normal((E, F, H)) * 0.3
    w2 = rng.standard_normal((E, H, F)) * 0.3
    base = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, score=O.SCORE_TOPK_SOFTMAX, cap_mode=O.CAP_DROPLESS)
    rnd = O.OracleLayer(T=T, H=H, F=F, E=E, k=k, score=O.SCORE_TOPK_SOFTMAX, cap_mode=O.CAP_DROPLESS,
                        random_second=1, z_coef=1e-2)
    keep_all = O.layer_forward(rnd, x, wg, w1, w2, uniform=np.zeros(T))
    ref = O.layer_forward(base, x, wg, w1, w2)
    np.testing.assert_allclose(keep_all["y"], ref["y"], rtol=1e-13, atol=1e-13)
    drop_all = O.layer_forward(rnd, x, wg, w1, w2, uniform=np.full(T, 0.999999))
    assert drop_all["aux"] == ref["aux"]               # f counts the selections
    assert int(drop_all["kept"].sum()) == T
    # with every second choice gone, y is the first choice's output times g_t0
    for t in range(T):
        e = int(ref["ids"][t, 0])
        h = np.maximum(w1[e] @ x[t], 0)
        np.testing.assert_allclose(drop_all["y"][t], ref["gates"][t, 0] * (w2[e] @ h), rtol=1e-12, atol=1e-13)
    assert drop_all["zloss"] == O.z_loss(drop_all["logits"], 1e-2)


# ------------------------------------------------------------ "probs" drop policy
def test_probs_policy_equal_gates_is_position_policy():
    E, k, T = 3, 2, 4
    pats = list(itertools.permutations(range(E), k))
    for combo in itertools.product(pats, repeat=T):
        ids = np.array(combo, dtype=np.int32)
        g = np.full((T, k), 0.25)
        for C in (1, 2, 3, None):
            a = O.assign_slots_probs(ids, g, E, C)
            b = O.assign_slots(ids, E, C)
            for u, v in zip(a, b):
                np.testing.assert_array_equal(u, v)


def test_probs_policy_keeps_the_best_subset_bruteforce():
    """With distinct gates the kept set of each expert is the unique size-C
    subset of largest gate sum; slots follow (rank, token) order."""
    rng = np.random.default_rng(41)
    E, k, T = 3, 2, 5
    for _ in range(300):
        ids = np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32)
        if rng.random() < 0.3:
            ids[rng.random(T) < 0.5, 1] = -1
        g = rng.permutation(T * k).reshape(T, k) / (T * k) + 0.01
        for C in (1, 2, 3):
            slot, count, kept = O.assign_slots_probs(ids, g, E, C)
            for e in range(E):
                arr = [(t, r) for r in range(k) for t in range(T) if ids[t, r] == e]
                assert count[e] == len(arr) and kept[e] == min(len(arr), C)
                best = max(itertools.combinations(range(len(arr)), min(C, len(arr))),
                           key=lambda s: sum(g[arr[i]] for i in s))
                got = [i for i, (t, r) in enumerate(arr) if slot[t, r] >= 0]
                assert sorted(got) == sorted(best)
                assert [slot[arr[i]] for i in got] == list(range(len(got)))
            assert (slot[ids < 0] == -1).all()
    # planted slip: dropping the highest gates instead fails the subset check
    ids = np.array([[0, 1], [0, 1], [0, 1]], np.int32)
    g = np.array([[0.9, 0.1], [0.5, 0.5], [0.2, 0.8]])
    slot, _, _ = O.assign_slots_probs(ids, g, 2, 1)
    assert list(slot[:, 0]) == [0, -1, -1] and list(slot[:, 1]) == [-1, -1, 0]


def test_probs_policy_ties_keep_earlier_arrivals():
    ids = np.array([[0, 1], [0, 1], [0, 1], [1, 0]], np.int32)
    g = np.array([[0.5, 0.3], [0.5, 0.3], [0.7, 0.3], [0.3, 0.5]])
    slot, count, kept = O.assign_slots_probs(ids, g, 2, 2)
    # expert 0: arrivals (t0,r0)=.5 (t1,r0)=.5 (t2,r0)=.7 (t3,r1)=.5 -> keep t2 and t0
    assert [slot[0, 0], slot[1, 0], slot[2, 0], slot[3, 1]] == [0, -1, 1, -1]
    # expert 1: arrivals (t3,r0)=.3 (t0,r1)=.3 (t1,r1)=.3 (t2,r1)=.3 -> first two arrivals
    assert [slot[3, 0], slot[0, 1], slot[1, 1], slot[2, 1]] == [0, 1, -1, -1]
    assert list(count) == [4, 4] and list(kept) == [2, 2]
