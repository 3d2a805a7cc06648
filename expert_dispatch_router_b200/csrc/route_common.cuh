// Per-token routing on a warp: scores, top-k, gates, and the per-lane sums the
// aux loss and the z-loss reduce.  Shared by the SIMT router (router.cu) and
// the tensor-core router's epilogue (grouped_gemm.cu).
//
// Method: "Expert-parallel MoE training" explainer, router section (a linear
// gate with E outputs, softmax then top-k, Megatron pre_softmax=False; sigmoid
// scores) and aux-loss section; "Switch Routing", 2.1 (p_i(x) softmax, gate =
// p_i(x)).  Top-k order: larger logit first, equal logits -> smaller expert.
#pragma once
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// Expert held by (lane, j): EJ==1 -> lane; EJ==2 -> 2*lane+j; EJ>=4 -> groups of
// four consecutive experts per lane, 128 experts per group row.
template <int EJ>
__device__ __forceinline__ int lane_expert(int lane, int j) {
  if constexpr (EJ == 1) return lane;
  else if constexpr (EJ == 2) return 2 * lane + j;
  else return 4 * lane + 128 * (j >> 2) + (j & 3);
}

// Top-k order: larger logit first (order-preserving keys, to_ordered), equal
// logits -> smaller expert index.  Each round finds the warp's best remaining
// (logit, lower index) key with two 32-bit max reductions: first the
// order-preserving logit bits, then, among lanes holding that logit, the
// complemented expert index.  Lane r < k receives the rank-r choice (its logit
// and expert); the return value marks, per lane, which of its EJ experts were
// chosen.
template <int EJ>
__device__ __forceinline__ unsigned select_topk(const float (&l)[EJ], int lane, int E, int k, float& my_l,
                                                int& my_e) {
  unsigned selected = 0u;
  my_l = -INFINITY;
  my_e = -1;
  uint32_t bh = 0u, bl = 0u;      // this lane's best unselected candidate
  int bj = -1;
  auto lane_best = [&]() {
    bh = 0u; bl = 0u; bj = -1;
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      const int e = lane_expert<EJ>(lane, j);
      if (e < E && !((selected >> j) & 1u)) {
        const uint32_t h = to_ordered(l[j]), lo = 0xffffffffu - (uint32_t)e;
        if (h > bh || (h == bh && lo > bl)) { bh = h; bl = lo; bj = j; }
      }
    }
  };
  lane_best();
#pragma unroll 1
  for (int r = 0; r < k; ++r) {
    const uint32_t wh = __reduce_max_sync(0xffffffffu, bh);
    const uint32_t wl = __reduce_max_sync(0xffffffffu, bh == wh ? bl : 0u);
    if (lane == r) { my_l = from_ordered(wh); my_e = (int)(0xffffffffu - wl); }
    if (bj >= 0 && bh == wh && bl == wl) {      // this lane owned the winner
      selected |= 1u << bj;
      lane_best();
    }
  }
  return selected;
}


// Scores, top-k and gates of token t from its E values spread over the warp's
// lanes (val[j] belongs to expert lane_expert(lane, j)), adding the logit offset
// and storing the logits if asked.  Accumulates this lane's sums of the
// probabilities the aux loss averages (softmax, or sigmoids normalised over the
// experts), its selection counts, and (zacc, same value in every lane) the
// squared log-sum-exp of the z-loss.
template <int EJ>
__device__ __forceinline__ void route_token(const RouterParams& p, int64_t t, int lane, const float (&val)[EJ],
                                            float (&psum)[EJ], int (&cnt)[EJ], float& zacc) {
  const int E = p.E;
  float l[EJ];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    const int e = lane_expert<EJ>(lane, j);
    float v = val[j];
    if (e < E) {
      if (p.logit_add != nullptr) v += p.logit_add[t * E + e];
      if (p.logits_out != nullptr) p.logits_out[t * E + e] = v;
      l[j] = v;
      m = fmaxf(m, v);
    } else {
      l[j] = -INFINITY;
    }
  }
  m = from_ordered(__reduce_max_sync(0xffffffffu, to_ordered(m)));
  float s = 0.0f, ex[EJ];
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    ex[j] = lane_expert<EJ>(lane, j) < E ? expf(l[j] - m) : 0.0f;
    s += ex[j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const bool sigmoid = p.score == MOE_SCORE_SIGMOID_TOPK;
  if (sigmoid) {
    float ss = 0.0f, sg[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      sg[j] = lane_expert<EJ>(lane, j) < E ? 1.0f / (1.0f + expf(-l[j])) : 0.0f;
      ss += sg[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    const float inv_ss = 1.0f / ss;
#pragma unroll
    for (int j = 0; j < EJ; ++j) psum[j] += sg[j] * inv_ss;
  } else {
    const float inv_s = 1.0f / s;
#pragma unroll
    for (int j = 0; j < EJ; ++j) psum[j] += ex[j] * inv_s;
  }
  if (p.zsum_part != nullptr) {
    const float lse = m + logf(s);
    zacc += lse * lse;
  }

  float my_l;
  int my_e;
  const unsigned selected = select_topk<EJ>(l, lane, E, p.k, my_l, my_e);
#pragma unroll
  for (int j = 0; j < EJ; ++j) cnt[j] += (selected >> j) & 1u;
  // gates: lane r holds the rank-r selection
  float g = 0.0f;
  if (lane < p.k) g = sigmoid ? 1.0f / (1.0f + expf(-my_l)) : expf(my_l - m);   // top-1 logit equals m
  if (p.score == MOE_SCORE_TOPK_SOFTMAX || p.renorm) {
    float gs = g;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) gs += __shfl_xor_sync(0xffffffffu, gs, o);
    g = g / gs;
  } else if (p.score == MOE_SCORE_SOFTMAX_TOPK) {
    g = g / s;
  }
  // GShard top-2: the second choice is dispatched iff u_t < 2 g_t1
  if (p.uniform != nullptr && lane == 1 && !(p.uniform[t] < 2.0f * g)) {
    my_e = -1;
    g = 0.0f;
  }
  if (lane < p.k) {
    p.ids[t * p.k + lane] = my_e;
    p.gates[t * p.k + lane] = g;
  }
}

}  // namespace moe
