"""Seeded synthetic inputs for the MoE FFN forward pass.

This module only draws numbers: it holds none of the layer's arithmetic.  Both
the CUDA path and the CPU oracle consume exactly the tensors it returns, so a
parity check compares the two on identical bytes.

Workload shapes follow the five layer configurations this library is built
for (tiny Switch top-1 in fp32; Switch top-1 with one overflowing expert;
GShard-style top-2; the high-k DeepSpeed stress shape from "The MoE spends too
much time on the gate network"; the DeepSeek-R1-shaped dropless layer from the
InferenceX "WideEP" note).  Value distributions follow the Switch explainer's
initialisation rule ("Switch Routing", section 2.2 "Init & regularization":
scale s = 0.1, sigma = sqrt(s / fan_in)).

Recipe (documented once here, used by tests and the benchmark):
  * x ~ N(0, 1) for the fp32 tiny layer, N(0, 1)/sqrt(H) otherwise.
  * router weight Wg [E, H] fp32 ~ N(0, 0.1/H).  The Switch top-1 workload adds
    +0.5 to every element of row 0 so that expert 0 overflows its capacity.
  * expert weights are stored like a linear layer ([out_features, in_features]):
    w1 [E, F, H] (W_in transposed; gate projection for SwiGLU), w3 [E, F, H]
    (SwiGLU up projection), w2 [E, H, F] (W_out / down projection transposed),
    all ~ N(0, 0.1/fan_in) with fan_in = H for w1/w3 and F for w2.
  * the dropless WideEP workload adds a harness-only logit offset
    logit_add[t, e] = ln p_e + G[t, e], p_e proportional to (pi(e)+1)^-1.1 over
    a seeded permutation pi and G standard Gumbel noise, so that top-8 routing
    draws experts with Zipf(1.1)-skewed loads.
  * "unit" scale variant: x ~ N(0, 1), weights ~ N(0, 1/fan_in), used where the
    configuration's tiny output scale would make an absolute tolerance vacuous.
  * layers with GShard's random second-expert dispatch get uniform [T] fp32
    draws in [0, 1), drawn after everything else (the other tensors are the
    same as without the option).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch

# Activation / scoring / capacity / dtype enumerations shared by the harness.
ACT_RELU, ACT_GELU, ACT_SWIGLU = 0, 1, 2
SCORE_SOFTMAX_TOPK, SCORE_TOPK_SOFTMAX, SCORE_SIGMOID_TOPK = 0, 1, 2
CAP_CAPACITY, CAP_DROPLESS = 0, 1
DROP_POSITION, DROP_PROBS = 0, 1
DTYPE_F32, DTYPE_BF16 = 0, 1


@dataclasses.dataclass(frozen=True)
class LayerShape:
    """Shape and routing options of one MoE FFN layer (plain data)."""
    name: str
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
    dtype: int = DTYPE_BF16
    bias_row0: float = 0.0        # added to router row 0 (overflowing expert)
    zipf_skew: float = 0.0        # >0: Gumbel/Zipf logit offset exponent
    z_coef: float = 0.0           # router z-loss coefficient (0 = off)
    random_second: int = 0        # GShard random dispatch of the second choice
    drop_policy: int = DROP_POSITION

    def replace(self, **kw) -> "LayerShape":
        return dataclasses.replace(self, **kw)

    def as_dict(self) -> dict:
        return dataclasses.asdict(self)


# The five layer workloads.
SWITCH_TINY_F32 = LayerShape("switch_top1_tiny_f32", T=256, H=64, F=128, E=4, k=1,
                             act=ACT_RELU, cf_num=5, cf_den=4, dtype=DTYPE_F32)
SWITCH_TOP1 = LayerShape("switch_top1_T8192_H768_E64", T=8192, H=768, F=3072, E=64, k=1,
                         act=ACT_RELU, cf_num=5, cf_den=4, bias_row0=0.5)
GSHARD_TOP2 = LayerShape("gshard_top2_T16384_H1024_E32", T=16384, H=1024, F=4096, E=32, k=2,
                         act=ACT_GELU, renorm=1, cf_num=2, cf_den=1)
DS_HIGHK = LayerShape("deepspeed_k4_T32768_H512_E12", T=32768, H=512, F=2048, E=12, k=4,
                      act=ACT_GELU, cf_num=1, cf_den=1)
WIDEEP_DROPLESS = LayerShape("wideep_dropless_T16384_H7168_E256_k8", T=16384, H=7168, F=2048,
                             E=256, k=8, act=ACT_SWIGLU, score=SCORE_TOPK_SOFTMAX,
                             cap_mode=CAP_DROPLESS, n_shared=1, zipf_skew=1.1)

# Profiling slice of the WideEP layer: the same H, F, SwiGLU, shared expert and
# top-8 skewed routing, with 16 experts and T chosen so that an expert gets the
# same ~512 rows on average (T*k/E = 512), in ~1.5 GB of weights.
WIDEEP_SLICE = WIDEEP_DROPLESS.replace(name="wideep_slice_T1024_H7168_E16_k8", T=1024, E=16)

WORKLOADS = {s.name: s for s in (SWITCH_TINY_F32, SWITCH_TOP1, GSHARD_TOP2, DS_HIGHK,
                                  WIDEEP_DROPLESS, WIDEEP_SLICE)}


def _normal(gen, shape, std, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * std


def make_inputs(shape: LayerShape, seed: int = 0, device: str = "cpu",
                scale: str = "config", experts: Optional[int] = None) -> dict:
    """Draw the layer inputs for `shape` with a seeded generator.

    Returns a dict of torch tensors on `device`:
      x [T,H] (bf16, or fp32 for the fp32 layer), wg [E,H] fp32,
      w1 [E,F,H], w2 [E,H,F], w3 [E,F,H] or None, and for a shared expert
      sw1 [1,F,H], sw2 [1,H,F], sw3 [1,F,H] or None; logit_add [T,E] fp32 or None;
      uniform [T] fp32 in [0,1) or None (random second-expert dispatch).
    `experts` (optional) draws only that many routed experts' weights, for
    host-side tests that never route to the others.
    """
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    T, H, F, E = shape.T, shape.H, shape.F, shape.E
    wdt = torch.float32 if shape.dtype == DTYPE_F32 else torch.bfloat16
    unit = scale == "unit"
    if unit:
        x = _normal(gen, (T, H), 1.0, device)
    else:
        x = _normal(gen, (T, H), 1.0 if shape.dtype == DTYPE_F32 else 1.0 / math.sqrt(H), device)
    wg_std = math.sqrt((1.0 if unit else 0.1) / H)
    wg = _normal(gen, (E, H), wg_std, device)
    if shape.bias_row0:
        wg[0] += shape.bias_row0
    s = 1.0 if unit else 0.1
    nE = E if experts is None else experts
    w1 = _normal(gen, (nE, F, H), math.sqrt(s / H), device).to(wdt)
    w3 = _normal(gen, (nE, F, H), math.sqrt(s / H), device).to(wdt) if shape.act == ACT_SWIGLU else None
    w2 = _normal(gen, (nE, H, F), math.sqrt(s / F), device).to(wdt)
    out = dict(x=x.to(wdt), wg=wg.contiguous(), w1=w1, w2=w2, w3=w3,
               sw1=None, sw2=None, sw3=None, logit_add=None, uniform=None)
    if shape.n_shared:
        out["sw1"] = _normal(gen, (1, F, H), math.sqrt(s / H), device).to(wdt)
        out["sw3"] = (_normal(gen, (1, F, H), math.sqrt(s / H), device).to(wdt)
                      if shape.act == ACT_SWIGLU else None)
        out["sw2"] = _normal(gen, (1, H, F), math.sqrt(s / F), device).to(wdt)
    if shape.zipf_skew:
        perm = torch.randperm(E, generator=gen, device=device)
        rank = torch.empty(E, dtype=torch.float64, device=device)
        rank[perm] = torch.arange(E, dtype=torch.float64, device=device)
        logp = -shape.zipf_skew * torch.log(rank + 1.0)
        logp = logp - torch.logsumexp(logp, 0)
        u = torch.rand((T, E), generator=gen, device=device, dtype=torch.float64)
        u = u.clamp_(min=1e-300)
        gumbel = -torch.log(-torch.log(u))
        out["logit_add"] = (logp[None, :] + gumbel).to(torch.float32).contiguous()
    if shape.random_second:
        out["uniform"] = torch.rand((T,), generator=gen, device=device, dtype=torch.float32)
    return out


def constructed_logits(choices, E: int, k: int, base: float = 4.0, step: float = 1.0):
    """fp32 router logits [T,E] whose top-k (descending, ties to lower index)
    is exactly `choices` [T,k] in rank order; every other expert gets -base.
    Used to realise a prescribed routing pattern through the routing epilogue."""
    T = len(choices)
    l = torch.full((T, E), -base, dtype=torch.float32)
    for t, row in enumerate(choices):
        for r, e in enumerate(row):
            l[t, int(e)] = base + (k - r) * step
    return l
