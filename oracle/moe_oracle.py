"""CPU oracle for the forward pass of one Mixture-of-Experts FFN layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the package's smoke entry and
the benchmark's CPU-baseline leg may import this module; the product path never
does.  It is deliberately plain and slow: numpy in float64, one library matmul
per contraction, Python loops where the method is a walk, and no blocking,
fusion or reordering beyond what each step's definition states.  It shares no
code with the CUDA library.

Sources (cited by page title and section):
  [EP]     "Expert-parallel MoE training" explainer (blog.vllbc.top, visual-reading
           series): router section (linear gate W_g in R^{HxE}, softmax then top-k,
           Megatron pre_softmax=False), capacity section (C = ceil((T*k/E)*cf)),
           drop/pad section ("position" policy, residual bypass), aux-loss section
           (f_i * P_i dot product times E, top-k in the denominator, = alpha under
           uniform routing), worked example "capacity overflow" and worked example
           "parameter and dispatch bytes", shared-expert paragraph.
  [DS7508] "The MoE spends too much time on the gate network" (DeepSpeed
           discussion 7508): k>2 capacity ceil((tokens/experts)*cf*k) = 10,923 at
           T=32768, E=12, k=4, cf=1.0, and the dense [T,E,C] mask sizes.
  [SWITCH] "Switch Routing - MoE Routing, Communication, and Stability"
           (AI Top Papers 7): section 2.1 "Routing math" (softmax, argmax,
           y = p_i(x) E_i(x)), "Load balance & capacity" (alpha*N*sum f_i P_i,
           alpha = 1e-2, overflow bypasses through the residual), section 2.2
           "Selective precision" (router in float32).
  [MB]     MegaBlocks as summarised in [EP] (dropless, each expert batch padded
           to a multiple of 128 rows).

Precision: every floating-point step is float64, except that the router logits
are rounded to float32 because [SWITCH] 2.2 fixes the router's precision to
float32; top-k is decided on those float32 values with an exact comparison.

Readings where the pages are silent or loose (each also listed in the design
notes):
  * capacity: the Megatron and DeepSpeed k>2 forms are the same rational number;
    it is evaluated exactly in integers with cf given as num/den.
  * slot order for k>1: (choice rank, token index), i.e. every first choice in
    token order, then every second choice ("position" drop policy).
  * top-k ties: larger logit first, equal logits go to the lower expert index.
  * gates are fixed before capacity; a dropped choice contributes zero and the
    kept gates are not renormalised again.
  * "probs" drop policy ([EP] drop/pad section names it: drop the lowest
    probability): the probability is the assignment's gate, compared in float32
    (the precision gates are stored in); equal gates keep the earlier
    assignment in (rank, token) order; kept assignments take slots in that
    order, so equal gates reduce it to the "position" policy.
  * f_i counts pre-drop selections over T*k; P_i is the mean full softmax.
  * sigmoid scores ([EP] router section names sigmoid as the alternative to
    softmax and says nothing more): top-k on the logits as for softmax (the
    sigmoid is monotone), gate = sigmoid(logit), optionally renormalised over
    the k selected; for the aux loss P_i averages the sigmoids divided by their
    sum over the E experts, so that equal logits still give aux = alpha.
  * z-loss ([EP] aux-loss section, z_loss_func): coef * mean_t lse(logits_t)^2
    on the float32 logits, reported beside the aux loss rather than added to it.
  * GShard random second expert ([EP] router section: sent at random according
    to its weight): the rank-1 choice is dispatched iff u_t < 2 g_t1, GShard's
    own rule (with top-2 renormalised gates 2 g_t1 <= 1), u_t ~ U[0, 1) an
    input.  A choice that is not dispatched keeps its place in f_i (selected),
    takes no slot and adds nothing to y; g_t0 is not changed.
  * the layer returns the MoE branch only (y = 0 for a fully dropped token); the
    caller adds the residual.
  * GELU is the exact erf form; SwiGLU is silu(x W_gate) * (x W_up) then W_down.
  * rows are laid out per expert, each expert's block padded to 128 rows, the
    shared expert's block (if any) last.

Every function here is pinned by tests/test_oracle_pins.py.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np

ACT_RELU, ACT_GELU, ACT_SWIGLU = 0, 1, 2
SCORE_SOFTMAX_TOPK, SCORE_TOPK_SOFTMAX, SCORE_SIGMOID_TOPK = 0, 1, 2
CAP_CAPACITY, CAP_DROPLESS = 0, 1
DROP_POSITION, DROP_PROBS = 0, 1
ROW_PAD = 128


@dataclass
class OracleLayer:
    """Layer options the oracle needs (kept independent of the CUDA binding)."""
    T: int
    H: int
    F: int
    E: int
    k: int
    act: int = ACT_RELU
    score: int = SCORE_SOFTMAX_TOPK
    renorm: int = 0
    cap_mode: int = CAP_CAPACITY
    cf_num: int = 1
    cf_den: int = 1
    min_capacity: int = 0
    n_shared: int = 0
    aux_alpha: float = 1e-2
    z_coef: float = 0.0          # router z-loss coefficient, 0 = off
    random_second: int = 0       # GShard: dispatch the second choice at random
    drop_policy: int = DROP_POSITION

    @classmethod
    def from_mapping(cls, m) -> "OracleLayer":
        names = cls.__dataclass_fields__.keys()
        return cls(**{n: m[n] for n in names if n in m})


# ---------------------------------------------------------------- capacity
def capacity(T: int, E: int, k: int, cf_num: int, cf_den: int, min_capacity: int = 0) -> int:
    """Expert capacity C = ceil((T*k/E) * cf)  ([EP] capacity section; Megatron
    get_capacity uses ceil).  [DS7508]'s k>2 form ceil((T/E)*cf*k) is the same
    rational number.  cf = cf_num/cf_den is exact, so the ceiling is taken on
    the exact fraction T*k*cf_num / (E*cf_den).  DeepSpeed's min_capacity
    ([EP], drop/pad section) is a lower clamp, 0 = none."""
    num = int(T) * int(k) * int(cf_num)
    den = int(E) * int(cf_den)
    c = -((-num) // den)
    return max(c, int(min_capacity))


def dense_mask_bytes(T: int, E: int, C: int, elem_bytes: int = 8) -> int:
    """Size of the dense one-hot [T, E, C] dispatch mask [DS7508] builds; the
    library never materialises it, the number is kept for comparison."""
    return int(T) * int(E) * int(C) * int(elem_bytes)


def expert_param_count(H: int, F: int, n_mats: int) -> int:
    """Parameters of one expert FFN with n_mats matrices of H x F ([EP] worked
    example "parameter and dispatch bytes", step 1)."""
    return int(n_mats) * int(H) * int(F)


# ---------------------------------------------------------------- router
def router_logits(x: np.ndarray, wg: np.ndarray, logit_add: Optional[np.ndarray] = None) -> np.ndarray:
    """logits[t, e] = sum_h x[t, h] * Wg[e, h]  ([EP] router section: a linear
    gate with E outputs; [SWITCH] 2.1 h(x) = W_r x).  Wg is held with one row
    per expert.  Computed in float64 and rounded once to float32 ([SWITCH] 2.2:
    the router runs in float32).  `logit_add` is a harness-only offset."""
    l = np.asarray(x, dtype=np.float64) @ np.asarray(wg, dtype=np.float64).T
    if logit_add is not None:
        l = l + np.asarray(logit_add, dtype=np.float64)
    return l.astype(np.float32)


def softmax(logits: np.ndarray) -> np.ndarray:
    """p = softmax over the last axis, float64 ([SWITCH] 2.1 p_i(x))."""
    l = np.asarray(logits, dtype=np.float64)
    m = l.max(axis=-1, keepdims=True)
    e = np.exp(l - m)
    return e / e.sum(axis=-1, keepdims=True)


def topk_ids(logits: np.ndarray, k: int) -> np.ndarray:
    """Top-k experts per token in rank order: larger logit first, equal logits
    broken toward the smaller expert index.  Selecting on logits picks the same
    experts as selecting on softmax probabilities (softmax is monotone)."""
    l = np.asarray(logits, dtype=np.float32)
    T, E = l.shape
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, -l), axis=-1)      # primary: -logit, secondary: index
    return order[:, :k].astype(np.int32)


def sigmoid(logits: np.ndarray) -> np.ndarray:
    """sigma(l) = 1 / (1 + exp(-l)), float64 ([EP] router section: softmax or sigmoid)."""
    return 1.0 / (1.0 + np.exp(-np.asarray(logits, dtype=np.float64)))


def router_probs(logits: np.ndarray, score: int) -> np.ndarray:
    """The per-expert probabilities P_i averages ([EP] aux-loss section).  Softmax
    for the softmax scores; for sigmoid scores the sigmoids normalised over the
    experts (so that they sum to one per token and uniform routing still gives
    aux = alpha)."""
    if score == SCORE_SIGMOID_TOPK:
        s = sigmoid(logits)
        return s / s.sum(axis=-1, keepdims=True)
    return softmax(logits)


def gate_values(logits: np.ndarray, probs: np.ndarray, ids: np.ndarray, score: int, renorm: int) -> np.ndarray:
    """Gate of each selected expert.
    SOFTMAX_TOPK: g = p[e] (Switch: y = p_i(x) E_i(x)), optionally divided by the
    sum over the k selected.  TOPK_SOFTMAX ([EP] router section, Megatron
    pre_softmax=False): softmax taken over the k selected logits only.
    SIGMOID_TOPK ([EP] router section, sigmoid scores): g = sigmoid(l[e]),
    optionally divided by the sum over the k selected."""
    t = np.arange(ids.shape[0])[:, None]
    sel = np.asarray(logits, dtype=np.float64)[t, ids]
    if score == SCORE_SOFTMAX_TOPK:
        g = probs[t, ids]
    elif score == SCORE_SIGMOID_TOPK:
        g = sigmoid(sel)
    else:
        return softmax(sel)
    if renorm:
        g = g / g.sum(axis=1, keepdims=True)
    return g


def random_second_dispatch(ids: np.ndarray, gates: np.ndarray, uniform: np.ndarray):
    """GShard top-2 ([EP] router section: the second expert receives the token at
    random, in proportion to its weight): the rank-1 choice of token t is
    dispatched iff u_t < 2 g_t1 (g renormalised over the two, so 2 g_t1 <= 1);
    otherwise its id becomes -1 (not dispatched) and its gate 0.  The uniforms
    u_t in [0,1) are an input."""
    ids = ids.copy()
    gates = gates.copy()
    u = np.asarray(uniform, dtype=np.float64)
    for t in range(ids.shape[0]):
        if not (u[t] < 2.0 * gates[t, 1]):
            ids[t, 1] = -1
            gates[t, 1] = 0.0
    return ids, gates


def z_loss(logits: np.ndarray, coef: float) -> float:
    """Router z-loss ([EP] aux-loss section, z_loss_func): coef * mean over tokens
    of logsumexp(logits_t)^2."""
    l = np.asarray(logits, dtype=np.float64)
    m = l.max(axis=-1)
    lse = m + np.log(np.exp(l - m[:, None]).sum(axis=-1))
    return float(coef * np.mean(lse ** 2)) if l.shape[0] else 0.0


# ---------------------------------------------------------------- slots
def assign_slots(ids: np.ndarray, E: int, C: Optional[int]):
    """Literal walk of the 'position' drop policy ([EP] drop/pad section):
    assignments are visited choice rank first, then token order; each takes the
    next free position of its expert and is kept iff that position < C
    (C=None: dropless, always kept).  An id of -1 is a choice that is not
    dispatched (GShard random second expert): it takes no position.  Returns
    (slot[T,k] with -1 = dropped or not dispatched, count[E] assignments per
    expert before the capacity drop, kept[E])."""
    T, k = ids.shape
    fill = [0] * E
    slot = np.full((T, k), -1, dtype=np.int32)
    for r in range(k):
        for t in range(T):
            e = int(ids[t, r])
            if e < 0:
                continue
            pos = fill[e]
            fill[e] += 1
            if C is None or pos < C:
                slot[t, r] = pos
    count = np.asarray(fill, dtype=np.int64)
    kept = count.copy() if C is None else np.minimum(count, C)
    return slot, count.astype(np.int32), kept.astype(np.int32)


def assign_slots_probs(ids: np.ndarray, gates: np.ndarray, E: int, C: Optional[int]):
    """The 'probs' drop policy ([EP] drop/pad section: Megatron-Core's
    moe_token_drop_policy="probs" drops the lowest-probability assignments).
    Each expert keeps the C of its assignments with the largest gate; among
    equal gates the one earlier in (choice rank, token) order is kept.  Kept
    assignments take slots 0.. in (choice rank, token) order.  Ids of -1 take no
    slot.  Same returns as assign_slots."""
    T, k = ids.shape
    per = [[] for _ in range(E)]               # (t, r) of each assignment, arrival order
    for r in range(k):
        for t in range(T):
            e = int(ids[t, r])
            if e >= 0:
                per[e].append((t, r))
    slot = np.full((T, k), -1, dtype=np.int32)
    g = np.asarray(gates, dtype=np.float64)
    for e in range(E):
        lst = per[e]
        if C is None or len(lst) <= C:
            keep = set(range(len(lst)))
        else:
            order = sorted(range(len(lst)), key=lambda i: (-g[lst[i]], i))
            keep = set(order[:C])
        j = 0
        for i, (t, r) in enumerate(lst):
            if i in keep:
                slot[t, r] = j
                j += 1
    count = np.array([len(p) for p in per], dtype=np.int64)
    kept = count.copy() if C is None else np.minimum(count, C)
    return slot, count.astype(np.int32), kept.astype(np.int32)


def round_up(n: int, m: int = ROW_PAD) -> int:
    return -(-int(n) // m) * m


def row_layout(kept: np.ndarray, T: int, n_shared: int):
    """Per-expert row blocks: expert e owns rows [off[e], off[e] + kept[e]) of a
    block padded to a multiple of 128 rows ([MB] via [EP]); the shared expert's
    block of T rows (padded) follows at off[E].  Returns off[E+2]."""
    E = len(kept)
    off = np.zeros(E + 2, dtype=np.int64)
    for e in range(E):
        off[e + 1] = off[e] + round_up(kept[e])
    off[E + 1] = off[E] + (round_up(T) if n_shared else 0)
    return off.astype(np.int32)


def row_tokens(ids: np.ndarray, slot: np.ndarray, off: np.ndarray, n_shared: int) -> np.ndarray:
    """Source token of every row, -1 for padding rows."""
    T, k = ids.shape
    E = len(off) - 2
    rt = np.full(int(off[E + 1]), -1, dtype=np.int32)
    for t in range(T):
        for r in range(k):
            if slot[t, r] >= 0:
                rt[off[ids[t, r]] + slot[t, r]] = t
    if n_shared:
        rt[off[E]:off[E] + T] = np.arange(T, dtype=np.int32)
    return rt


# ---------------------------------------------------------------- experts
def gelu(z: np.ndarray) -> np.ndarray:
    """Exact GELU, 0.5 z (1 + erf(z / sqrt 2))."""
    from scipy.special import erf
    return 0.5 * z * (1.0 + erf(np.asarray(z, dtype=np.float64) / math.sqrt(2.0)))


def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def expert_ffn(X: np.ndarray, w1: np.ndarray, w2: np.ndarray, act: int,
               w3: Optional[np.ndarray] = None) -> np.ndarray:
    """One expert applied to rows X [n, H], float64 throughout.
    Weights are stored like a linear layer: w1 [F, H] (W_in transposed, the
    gate projection for SwiGLU), w3 [F, H] (SwiGLU up projection), w2 [H, F].
    ReLU/GELU: act(X W_in) W_out.  SwiGLU ([EP] worked example: gate / up /
    down matrices): (silu(X W_gate) * (X W_up)) W_down."""
    X = np.asarray(X, dtype=np.float64)
    a = X @ np.asarray(w1, dtype=np.float64).T
    if act == ACT_RELU:
        h = np.maximum(a, 0.0)
    elif act == ACT_GELU:
        h = gelu(a)
    elif act == ACT_SWIGLU:
        h = silu(a) * (X @ np.asarray(w3, dtype=np.float64).T)
    else:
        raise ValueError(f"unknown activation {act}")
    return h @ np.asarray(w2, dtype=np.float64).T


# ---------------------------------------------------------------- aux loss
def aux_loss(probs: np.ndarray, ids: np.ndarray, E: int, alpha: float) -> float:
    """Switch load-balancing loss alpha * N * sum_i f_i P_i ([SWITCH] 2.1, [EP]
    aux-loss section): f_i = selections of expert i / (T*k) (top-k in the
    denominator, pre-drop), P_i = mean over tokens of the router probabilities
    p_i (softmax, or the normalised sigmoids of router_probs)."""
    T, k = ids.shape
    f = np.bincount(ids.reshape(-1), minlength=E).astype(np.float64) / (T * k)
    P = np.asarray(probs, dtype=np.float64).mean(axis=0)
    return float(alpha * E * np.sum(f * P))


# ---------------------------------------------------------------- layer
def route(layer: OracleLayer, logits: np.ndarray):
    """Router steps after the logits: scores, top-k, gates."""
    probs = router_probs(logits, layer.score)
    ids = topk_ids(logits, layer.k)
    gates = gate_values(logits, probs, ids, layer.score, layer.renorm)
    return probs, ids, gates


def route_and_dispatch(layer: OracleLayer, logits: np.ndarray, uniform=None):
    """route(), then GShard's random second-expert dispatch when enabled.
    Returns (probs, selected ids, dispatched ids, gates): the aux loss counts
    the selected ids, slots take the dispatched ones."""
    probs, ids, gates = route(layer, logits)
    disp = ids
    if layer.random_second and layer.k >= 2:
        disp, gates = random_second_dispatch(ids, gates, uniform)
    return probs, ids, disp, gates


def layer_capacity(layer: OracleLayer) -> Optional[int]:
    if layer.cap_mode == CAP_DROPLESS:
        return None
    return capacity(layer.T, layer.E, layer.k, layer.cf_num, layer.cf_den, layer.min_capacity)


def layer_forward(layer: OracleLayer, x, wg, w1, w2, w3=None, sw1=None, sw2=None, sw3=None,
                  logit_add=None, logits=None, tokens=None, want_rows=False, uniform=None) -> dict:
    """The whole forward pass, stage by stage.

    `logits` (optional) replaces the router GEMM with given float32 logits, so
    routing can be compared bit-exactly against another implementation's
    logits.  `tokens` (optional) restricts the expert FFN and combine to those
    token indices (tokens are independent once slots are fixed); routing, slots
    and the aux loss always cover every token.  Returns a dict with logits,
    probs, ids, gates, capacity, slot, count, kept, offsets, row_token, aux,
    y (for `tokens`, or all) and, with want_rows, the un-gated expert output of
    every kept (token, choice) of those tokens.  `uniform` [T] drives GShard's
    random second-expert dispatch when the layer enables it; `ids` are then the
    dispatched ids (-1 = not dispatched) and `selected` the top-k ids.
    """
    T, E, k = layer.T, layer.E, layer.k
    if logits is None:
        logits = router_logits(x, wg, logit_add)
    logits = np.asarray(logits, dtype=np.float32)
    probs, selected, ids, gates = route_and_dispatch(layer, logits, uniform)
    C = layer_capacity(layer)
    if layer.drop_policy == DROP_PROBS:
        # the decision compares gates in float32, the precision they are stored in
        slot, count, kept = assign_slots_probs(ids, gates.astype(np.float32), E, C)
    else:
        slot, count, kept = assign_slots(ids, E, C)
    off = row_layout(kept, T, layer.n_shared)
    rt = row_tokens(ids, slot, off, layer.n_shared)
    aux = aux_loss(probs, selected, E, layer.aux_alpha)
    zl = z_loss(logits, layer.z_coef)

    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    X = np.asarray(x, dtype=np.float64)
    y = np.zeros((len(tok), layer.H), dtype=np.float64)
    rows = {}
    bucket = [[] for _ in range(E)]          # kept (sample index, choice) per expert
    for i, t in enumerate(tok):
        for r in range(k):
            if slot[t, r] >= 0:
                bucket[int(ids[t, r])].append((i, r))
    for e in range(E):
        sel = bucket[e]
        if not sel:
            continue
        ii = np.array([i for i, _ in sel])
        Ye = expert_ffn(X[tok[ii]], w1[e], w2[e], layer.act, None if w3 is None else w3[e])
        for j, (i, r) in enumerate(sel):
            y[i] += gates[tok[i], r] * Ye[j]
            if want_rows:
                rows[(int(tok[i]), int(r))] = Ye[j]
    if layer.n_shared:
        Ys = expert_ffn(X[tok], sw1[0], sw2[0], layer.act, None if sw3 is None else sw3[0])
        y += Ys
        if want_rows:
            for i, t in enumerate(tok):
                rows[(int(t), -1)] = Ys[i]
    out = dict(logits=logits, probs=probs, ids=ids, selected=selected, gates=gates, capacity=C, slot=slot, zloss=zl,
               count=count, kept=kept, offsets=off, row_token=rt, aux=aux, y=y, tokens=tok)
    if want_rows:
        out["rows"] = rows
    return out
