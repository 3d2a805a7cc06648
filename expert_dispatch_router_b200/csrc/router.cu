// Router (fp32 logits GEMM + fused softmax / top-k / gates) and the Switch
// load-balancing loss reduction.
//
// Method: "Expert-parallel MoE training" explainer, router section (a linear
// gate with E outputs, softmax then top-k, Megatron pre_softmax=False) and
// aux-loss section (alpha * E * sum f_i P_i with top-k in f's denominator);
// "Switch Routing", 2.1 (p_i(x) softmax, gate = p_i(x)) and 2.2 (the router
// runs in float32).
//
// Design: one CTA of four warps owns BT tokens and all E experts.  The H
// reduction walks 16-wide chunks: x (bf16 or fp32) is widened to fp32 into
// shared memory, the Wg chunk is stored transposed so that a lane reads its
// experts with one conflict-free vector load, and every lane accumulates a
// TW x EJ register tile with FFMA.  The epilogue keeps each token's E logits
// spread over the 32 lanes of a warp and does max, sum-of-exp and k rounds of
// arg-max with warp shuffles, so no logit row ever goes back to memory.  Per-CTA
// sums of p and selection counts are reduced over the warps in a fixed order
// (deterministic) and left in the workspace for the aux-loss kernel.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "route_common.cuh"

namespace moe {

constexpr int kRouterWarps = 4;
constexpr int kRouterThreads = kRouterWarps * 32;
constexpr int kKC = 16;   // H chunk

// lane_expert, select_topk and route_token: route_common.cuh.

// Sums the warps' per-expert partials (and z-loss sums) in a fixed order and
// stores this CTA's row of psum_part / cnt_part (and zsum_part).  `smem` must
// hold 2 * WARPS * 32 * EJ + WARPS words.
template <int EJ, int WARPS>
__device__ __forceinline__ void write_partials(const RouterParams& p, float* smem, const float (&psum)[EJ],
                                               const int (&cnt)[EJ], float zacc) {
  constexpr int EP = 32 * EJ;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  float* rp = smem;                                     // [WARPS][EP]
  int* rc = reinterpret_cast<int*>(smem + WARPS * EP);
  float* rz = smem + 2 * WARPS * EP;                    // [WARPS]
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    const int e = lane_expert<EJ>(lane, j);
    rp[warp * EP + e] = psum[j];
    rc[warp * EP + e] = cnt[j];
  }
  if (lane == 0) rz[warp] = zacc;
  __syncthreads();
  for (int e = tid; e < p.E; e += WARPS * 32) {
    float ps = 0.0f;
    int cs = 0;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) { ps += rp[w * EP + e]; cs += rc[w * EP + e]; }
    p.psum_part[(int64_t)blockIdx.x * p.E + e] = ps;
    p.cnt_part[(int64_t)blockIdx.x * p.E + e] = cs;
  }
  if (tid == 0 && p.zsum_part != nullptr) {
    float z = 0.0f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) z += rz[w];
    p.zsum_part[blockIdx.x] = z;
  }
}

template <int EJ, int TW>
constexpr int router_smem_floats() {
  constexpr int EP = 32 * EJ;
  constexpr int main_ = kRouterWarps * TW * kKC + kKC * (EP + 4);
  constexpr int red = 2 * kRouterWarps * EP + kRouterWarps;
  return main_ > red ? main_ : red;
}

template <int EJ, int TW, typename XT>
__global__ void __launch_bounds__(kRouterThreads) router_kernel(RouterParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int EP = 32 * EJ;
  constexpr int BT = kRouterWarps * TW;
  constexpr int WS = EP + 4;
  extern __shared__ __align__(16) float smem[];
  float* xs = smem;                       // [BT][kKC]
  float* wgs = smem + BT * kKC;           // [kKC][WS]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * BT;
  const int E = p.E, H = p.H;
  if (blockIdx.x == 0 && tid == 0 && p.aux_counter != nullptr) *p.aux_counter = 0u;

  float acc[TW][EJ];
#pragma unroll
  for (int i = 0; i < TW; ++i)
#pragma unroll
    for (int j = 0; j < EJ; ++j) acc[i][j] = 0.0f;

  {
    constexpr int XV = 16 / sizeof(XT);              // elements per 16-byte vector
    constexpr int XVEC = BT * kKC / XV;              // x vectors per chunk
    constexpr int XM = (XVEC + kRouterThreads - 1) / kRouterThreads;
    int4 xraw[XM];
    float4 wr[EJ];
    // global -> registers for the chunk at k0 (issued one chunk ahead of its use)
    auto fetch = [&](int k0) {
#pragma unroll
      for (int m = 0; m < XM; ++m) {
        const int q = tid + m * kRouterThreads;
        const int tok = q / (kKC / XV), kv = q % (kKC / XV);
        const int64_t t = t0 + tok;
        const int kk = k0 + kv * XV;
        xraw[m] = make_int4(0, 0, 0, 0);
        if (q < XVEC && t < p.T && kk < H) xraw[m] = ld_nc_v4(static_cast<const XT*>(p.x) + t * H + kk);
      }
#pragma unroll
      for (int m = 0; m < EJ; ++m) {
        const int q = tid + m * kRouterThreads;      // float4 index in [0, EP*4)
        const int e = q >> 2, kq = q & 3;
        wr[m] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (e < E && k0 + 4 * kq < H)
          wr[m] = __ldg(reinterpret_cast<const float4*>(p.wg + (int64_t)e * H + k0 + 4 * kq));
      }
    };
    fetch(0);
    for (int k0 = 0; k0 < H; k0 += kKC) {
      float xr[XM][XV];
#pragma unroll
      for (int m = 0; m < XM; ++m) {
        const XT* e = reinterpret_cast<const XT*>(&xraw[m]);
#pragma unroll
        for (int c = 0; c < XV; ++c) xr[m][c] = Elem<XT>::to_f(e[c]);
      }
      __syncthreads();  // previous chunk consumed
#pragma unroll
      for (int m = 0; m < XM; ++m) {
        const int q = tid + m * kRouterThreads;
        if (q < XVEC) {
          const int tok = q / (kKC / XV), kv = q % (kKC / XV);
#pragma unroll
          for (int c = 0; c < XV; ++c) xs[tok * kKC + kv * XV + c] = xr[m][c];
        }
      }
#pragma unroll
      for (int m = 0; m < EJ; ++m) {
        const int q = tid + m * kRouterThreads;
        const int e = q >> 2, kq = q & 3;
        wgs[(4 * kq + 0) * WS + e] = wr[m].x;
        wgs[(4 * kq + 1) * WS + e] = wr[m].y;
        wgs[(4 * kq + 2) * WS + e] = wr[m].z;
        wgs[(4 * kq + 3) * WS + e] = wr[m].w;
      }
      __syncthreads();
      if (k0 + kKC < H) fetch(k0 + kKC);             // next chunk's loads overlap this chunk's FFMAs
#pragma unroll
      for (int kk = 0; kk < kKC; kk += 4) {
        float4 xv[TW];
#pragma unroll
        for (int i = 0; i < TW; ++i)
          xv[i] = *reinterpret_cast<const float4*>(&xs[(warp * TW + i) * kKC + kk]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float* wrow = wgs + (kk + c) * WS;
          float wv[EJ];
          if constexpr (EJ == 1) {
            wv[0] = wrow[lane];
          } else if constexpr (EJ == 2) {
            float2 v = *reinterpret_cast<const float2*>(wrow + 2 * lane);
            wv[0] = v.x; wv[1] = v.y;
          } else {
#pragma unroll
            for (int g = 0; g < EJ / 4; ++g) {
              float4 v = *reinterpret_cast<const float4*>(wrow + 4 * lane + 128 * g);
              wv[4 * g + 0] = v.x; wv[4 * g + 1] = v.y; wv[4 * g + 2] = v.z; wv[4 * g + 3] = v.w;
            }
          }
#pragma unroll
          for (int i = 0; i < TW; ++i) {
            const float xc = c == 0 ? xv[i].x : c == 1 ? xv[i].y : c == 2 ? xv[i].z : xv[i].w;
#pragma unroll
            for (int j = 0; j < EJ; ++j) acc[i][j] = fmaf(xc, wv[j], acc[i][j]);
          }
        }
      }
    }
  }

  // ---------------- epilogue: softmax, top-k, gates, partial sums
  float psum[EJ], zacc = 0.0f;
  int cnt[EJ];
#pragma unroll
  for (int j = 0; j < EJ; ++j) { psum[j] = 0.0f; cnt[j] = 0; }
#pragma unroll
  for (int i = 0; i < TW; ++i) {
    const int64_t t = t0 + warp * TW + i;
    if (t < p.T) route_token<EJ>(p, t, lane, acc[i], psum, cnt, zacc);
  }

  // ---------------- fixed-order reduction of the per-warp partials
  __syncthreads();
  write_partials<EJ, kRouterWarps>(p, smem, psum, cnt, zacc);
}

// Routing from given fp32 logits (the tensor-core router's output, or the
// caller's for moe_route_from_logits): the same BT tokens per CTA as the FFMA
// router so the partial-sum rows line up; a warp routes one token at a time with
// nothing but that token's logits in registers.  Warps per CTA: 32 (one token
// each) for E <= 64, 16 for E <= 128 (the register budget of 1024 threads is
// too small there), 8 for wider E, whose partial sums need more shared memory.
template <int EJ>
constexpr int logit_warps() { return EJ <= 2 ? 32 : EJ == 4 ? 16 : 8; }

template <int EJ>
__global__ void __launch_bounds__(logit_warps<EJ>() * 32, 1) route_logits_kernel(RouterParams p, int bt) {
  constexpr int kLogitWarps = logit_warps<EJ>();
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) float smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * bt;
  if (blockIdx.x == 0 && tid == 0 && p.aux_counter != nullptr) *p.aux_counter = 0u;
  float psum[EJ], zacc = 0.0f;
  int cnt[EJ];
#pragma unroll
  for (int j = 0; j < EJ; ++j) { psum[j] = 0.0f; cnt[j] = 0; }
  for (int i = warp; i < bt; i += kLogitWarps) {
    const int64_t t = t0 + i;
    if (t >= p.T) break;
    float val[EJ];
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      const int e = lane_expert<EJ>(lane, j);
      float v = 0.0f;
      if (e < p.E) {
        v = p.logits_in[t * p.E + e];
        for (int q = 1; q < p.logits_parts; ++q) v += p.logits_in[(int64_t)q * p.T * p.E + t * p.E + e];
      }
      val[j] = v;
    }
    route_token<EJ>(p, t, lane, val, psum, cnt, zacc);
  }
  __syncthreads();
  write_partials<EJ, kLogitWarps>(p, smem, psum, cnt, zacc);
}

// Tokens per CTA of the router for E experts (the host needs it to size the
// partial-sum arrays).
int router_tile_tokens(int E) {
  const int ej = E <= 32 ? 1 : E <= 64 ? 2 : E <= 128 ? 4 : E <= 256 ? 8 : E <= 512 ? 16 : 32;
  const int tw = ej <= 8 ? 8 : ej == 16 ? 4 : 2;
  return kRouterWarps * tw;
}

template <int EJ, int TW>
static cudaError_t launch_router_ej(const RouterParams& p, bool bf16, cudaStream_t stream) {
  constexpr int BT = kRouterWarps * TW;
  const size_t smem = sizeof(float) * router_smem_floats<EJ, TW>();
  const unsigned grid = (unsigned)((p.T + BT - 1) / BT);
  if (bf16) {
    auto k = router_kernel<EJ, TW, __nv_bfloat16>;
    cudaError_t e = ensure_smem(k, smem);
    if (e != cudaSuccess) return e;
    launch_pdl(k, grid, kRouterThreads, smem, stream, p);
  } else {
    auto k = router_kernel<EJ, TW, float>;
    cudaError_t e = ensure_smem(k, smem);
    if (e != cudaSuccess) return e;
    launch_pdl(k, grid, kRouterThreads, smem, stream, p);
  }
  return cudaGetLastError();
}

template <int EJ>
static cudaError_t launch_route_logits_ej(const RouterParams& p, cudaStream_t stream) {
  const int bt = router_tile_tokens(p.E);
  constexpr int kLogitWarps = logit_warps<EJ>();
  const size_t smem = sizeof(float) * (2 * kLogitWarps * 32 * EJ + kLogitWarps);
  const unsigned grid = (unsigned)((p.T + bt - 1) / bt);
  auto k = route_logits_kernel<EJ>;
  cudaError_t e = ensure_smem(k, smem);
  if (e != cudaSuccess) return e;
  launch_pdl(k, grid, kLogitWarps * 32, smem, stream, p, bt);
  return cudaGetLastError();
}

cudaError_t launch_router(const RouterParams& p, bool bf16, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  const int E = p.E;
  if (p.logits_in != nullptr) {
    if (E <= 32) return launch_route_logits_ej<1>(p, stream);
    if (E <= 64) return launch_route_logits_ej<2>(p, stream);
    if (E <= 128) return launch_route_logits_ej<4>(p, stream);
    if (E <= 256) return launch_route_logits_ej<8>(p, stream);
    if (E <= 512) return launch_route_logits_ej<16>(p, stream);
    return launch_route_logits_ej<32>(p, stream);
  }
  if (E <= 32) return launch_router_ej<1, 8>(p, bf16, stream);
  if (E <= 64) return launch_router_ej<2, 8>(p, bf16, stream);
  if (E <= 128) return launch_router_ej<4, 8>(p, bf16, stream);
  if (E <= 256) return launch_router_ej<8, 8>(p, bf16, stream);
  if (E <= 512) return launch_router_ej<16, 4>(p, bf16, stream);
  return launch_router_ej<32, 2>(p, bf16, stream);
}

// ---------------------------------------------------------------- backward
// dL/dlogits of one token ("Expert-parallel MoE training" explainer, aux-loss
// section: the aux loss reaches the router only through P_i, f_i being a
// constant; the z-loss acts on the logits; "Switch Routing" 2.1: the gate is the
// router's probability).  The selection is recomputed from the forward's logits
// with the forward's own top-k; dgate is zero for choices that add nothing to y.
template <int EJ>
__device__ __forceinline__ void route_token_bwd(const RouterBwdParams& p, int64_t t, int lane) {
  const int E = p.E;
  float l[EJ];
  float m = -INFINITY;
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    const int e = lane_expert<EJ>(lane, j);
    l[j] = e < E ? p.logits[t * E + e] : -INFINITY;
    m = fmaxf(m, l[j]);
  }
  m = from_ordered(__reduce_max_sync(0xffffffffu, to_ordered(m)));
  float pr[EJ], s = 0.0f;
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    pr[j] = lane_expert<EJ>(lane, j) < E ? expf(l[j] - m) : 0.0f;
    s += pr[j];
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float inv_s = 1.0f / s;
#pragma unroll
  for (int j = 0; j < EJ; ++j) pr[j] *= inv_s;                 // softmax
  float my_l;
  int my_e;
  select_topk<EJ>(l, lane, E, p.k, my_l, my_e);
  const int e_top = __shfl_sync(0xffffffffu, my_e, 0);         // argmax of the logits, p, the sigmoids
  const bool sigmoid = p.score == MOE_SCORE_SIGMOID_TOPK;
  const bool tks = p.score == MOE_SCORE_TOPK_SOFTMAX;
  const bool norm = tks || p.renorm;
  // Renormalised softmax gates are the softmax of the selected logits, the
  // same function as TOPK_SOFTMAX: their gradient goes straight to the
  // selected logits (through the full softmax it would cancel exactly for every
  // other expert, in exact arithmetic only).
  const bool direct = tks || (p.score == MOE_SCORE_SOFTMAX_TOPK && p.renorm);
  // Every "v_j - sum_i w_i v_i" below (weights summing to one, the largest one
  // w_m) is evaluated as (v_j - v_m) + sum_{i != m} w_i (v_m - v_i): equal in
  // exact arithmetic, and free of the cancellation that the direct form suffers
  // in fp32 when w_m is within rounding of 1 (a confidently routed token).
  // gate of rank r (lane r) before renormalisation, and the normaliser S
  float graw = 0.0f, dg = 0.0f;
  if (lane < p.k) {
    graw = sigmoid ? 1.0f / (1.0f + expf(-my_l)) : tks ? expf(my_l - m) : expf(my_l - m) * inv_s;
    dg = p.dgate[t * p.k + lane];
  }
  float S = graw;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) S += __shfl_xor_sync(0xffffffffu, S, o);
  const float g = norm ? graw / S : graw;
  const float dg0 = __shfl_sync(0xffffffffu, dg, 0);
  float rg = lane > 0 && lane < p.k ? g * (dg0 - dg) : 0.0f;     // sum_{r != 0} g_r (dg_0 - dg_r)
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) rg += __shfl_xor_sync(0xffffffffu, rg, o);
  const float centred = (dg - dg0) + rg;                          // dg_r - sum_q g_q dg_q
  // gradient with respect to the rank-r quantity before normalisation: the
  // logit (TOPK_SOFTMAX, renormalised SOFTMAX_TOPK), p (SOFTMAX_TOPK) or the
  // sigmoid (SIGMOID_TOPK)
  const float val = direct ? g * centred : norm ? centred / S : dg;
  float dpre[EJ], dl[EJ];
#pragma unroll
  for (int j = 0; j < EJ; ++j) { dpre[j] = 0.0f; dl[j] = 0.0f; }
#pragma unroll 1
  for (int r = 0; r < p.k; ++r) {
    const int er = __shfl_sync(0xffffffffu, my_e, r);
    const float vr = __shfl_sync(0xffffffffu, val, r);
#pragma unroll
    for (int j = 0; j < EJ; ++j)
      if (lane_expert<EJ>(lane, j) == er) {
        if (direct) dl[j] += vr;
        else dpre[j] += vr;
      }
  }
  // value v at the top expert, broadcast from the lane that holds it
  auto at_top = [&](const float (&v)[EJ]) -> float {
    float x = 0.0f;
#pragma unroll
    for (int j = 0; j < EJ; ++j)
      if (lane_expert<EJ>(lane, j) == e_top) x = v[j];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);   // one lane holds it
    return x;
  };
  if (sigmoid) {
    // aux: P uses q = sigmoid / sum(sigmoid), dL/dq_i = fcoef_i;
    // ds_j = dpre_j + (fcoef_j - sum_i q_i fcoef_i) / sum(sigmoid)
    float sg[EJ], sgc[EJ], fc[EJ], Ss = 0.0f;
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      const int e = lane_expert<EJ>(lane, j);
      sg[j] = e < E ? 1.0f / (1.0f + expf(-l[j])) : 0.0f;
      sgc[j] = e < E ? 1.0f / (1.0f + expf(l[j])) : 0.0f;        // 1 - sigmoid, without cancellation
      fc[j] = e < E ? p.fcoef[e] : 0.0f;
      Ss += sg[j];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) Ss += __shfl_xor_sync(0xffffffffu, Ss, o);
    const float f_top = at_top(fc);
    float rq = 0.0f;
#pragma unroll
    for (int j = 0; j < EJ; ++j)
      if (lane_expert<EJ>(lane, j) < E && lane_expert<EJ>(lane, j) != e_top) rq += sg[j] * (f_top - fc[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rq += __shfl_xor_sync(0xffffffffu, rq, o);
    rq /= Ss;
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      const int e = lane_expert<EJ>(lane, j);
      if (e < E) {
        const float ds = dpre[j] + ((fc[j] - f_top) + rq) / Ss;
        dl[j] += ds * sg[j] * sgc[j];
      }
    }
  } else {
    // softmax backward of dp = (gate part) + aux part
#pragma unroll
    for (int j = 0; j < EJ; ++j) {
      const int e = lane_expert<EJ>(lane, j);
      if (e < E) dpre[j] += p.fcoef[e];
    }
    const float d_top = at_top(dpre);
    float rp = 0.0f;                                              // sum_{i != top} p_i (dp_top - dp_i)
#pragma unroll
    for (int j = 0; j < EJ; ++j)
      if (lane_expert<EJ>(lane, j) < E && lane_expert<EJ>(lane, j) != e_top) rp += pr[j] * (d_top - dpre[j]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rp += __shfl_xor_sync(0xffffffffu, rp, o);
#pragma unroll
    for (int j = 0; j < EJ; ++j) dl[j] += pr[j] * ((dpre[j] - d_top) + rp);
  }
  if (p.zc != 0.0f) {
    const float c = 2.0f * p.zc * (m + logf(s)) / (float)p.T;
#pragma unroll
    for (int j = 0; j < EJ; ++j) dl[j] += c * pr[j];
  }
#pragma unroll
  for (int j = 0; j < EJ; ++j) {
    const int e = lane_expert<EJ>(lane, j);
    if (e < E) p.dlogits[t * E + e] = dl[j];
  }
}

constexpr int kBwdRouterWarps = 8;

template <int EJ>
__global__ void __launch_bounds__(kBwdRouterWarps * 32) router_bwd_kernel(RouterBwdParams p) {
  pdl_wait();
  pdl_trigger();
  const int64_t t = (int64_t)blockIdx.x * kBwdRouterWarps + (threadIdx.x >> 5);
  if (t < p.T) route_token_bwd<EJ>(p, t, threadIdx.x & 31);
}

// fcoef[e] = d_aux * alpha * E * f_e / T, f_e = selections of e / (T k) from the
// router's per-CTA counts: one warp per expert, lanes striding over the CTAs
// (integer sums, exact in any order).
constexpr int kPrepWarps = 8;

__global__ void __launch_bounds__(kPrepWarps * 32) aux_grad_prep_kernel(const int32_t* cnt_part, int nblk, int E,
                                                                         int64_t T, int k, float scale, float* fcoef) {
  pdl_wait();
  pdl_trigger();
  const int e = blockIdx.x * kPrepWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (e >= E) return;
  long long c = 0;
  for (int b = lane; b < nblk; b += 32) c += cnt_part[(int64_t)b * E + e];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
  if (lane == 0)
    fcoef[e] = T > 0 ? (float)((double)scale * (double)E * ((double)c / ((double)T * k)) / (double)T) : 0.0f;
}

template <int EJ>
static void launch_router_bwd_ej(const RouterBwdParams& p, cudaStream_t stream) {
  launch_pdl(router_bwd_kernel<EJ>, (unsigned)((p.T + kBwdRouterWarps - 1) / kBwdRouterWarps), kBwdRouterWarps * 32,
             0, stream, p);
}

cudaError_t launch_router_bwd(const RouterBwdParams& p, const int32_t* cnt_part, int nblk, float d_aux_alpha,
                              float* fcoef, cudaStream_t stream) {
  launch_pdl(aux_grad_prep_kernel, (unsigned)((p.E + kPrepWarps - 1) / kPrepWarps), kPrepWarps * 32, 0, stream,
             cnt_part, nblk, p.E, p.T, p.k, d_aux_alpha, fcoef);
  if (p.T > 0) {
    const int E = p.E;
    if (E <= 32) launch_router_bwd_ej<1>(p, stream);
    else if (E <= 64) launch_router_bwd_ej<2>(p, stream);
    else if (E <= 128) launch_router_bwd_ej<4>(p, stream);
    else if (E <= 256) launch_router_bwd_ej<8>(p, stream);
    else if (E <= 512) launch_router_bwd_ej<16>(p, stream);
    else launch_router_bwd_ej<32>(p, stream);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------- aux loss
// Warp per expert: its lanes stride over the router blocks' partials in fp64
// and reduce with a fixed butterfly into term[e] = f_e * P_e.  The last CTA to
// finish (a ticket counter) sums the terms in a fixed order, so the result is
// deterministic, and re-arms the counter.  The router also re-arms it.
constexpr int kAuxWarps = 8;

__global__ void __launch_bounds__(kAuxWarps * 32) aux_kernel(const float* psum_part, const int32_t* cnt_part,
                                                             const float* zsum_part, int nblk, int E, int64_t T,
                                                             int k, float alpha, float z_coef, double* term,
                                                             unsigned* counter, float* aux) {
  pdl_wait();
  pdl_trigger();
  __shared__ double sh[kAuxWarps * 32];
  __shared__ bool last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, tid = threadIdx.x;
  if (T == 0) {
    if (tid == 0) {
      aux[0] = 0.0f;
      if (zsum_part != nullptr) aux[1] = 0.0f;
    }
    return;
  }
  const int e = blockIdx.x * kAuxWarps + warp;
  if (e < E) {
    double ps = 0.0;
    long long cs = 0;
    for (int b = lane; b < nblk; b += 32) {
      ps += (double)psum_part[(int64_t)b * E + e];
      cs += cnt_part[(int64_t)b * E + e];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ps += __shfl_xor_sync(0xffffffffu, ps, o);
      cs += __shfl_xor_sync(0xffffffffu, cs, o);
    }
    if (lane == 0) term[e] = ((double)cs / ((double)T * k)) * (ps / (double)T);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) last = atomicAdd(counter, 1u) == gridDim.x - 1;
  __syncthreads();
  if (!last) return;
  __threadfence();
  double v = 0.0;
  for (int i = tid; i < E; i += kAuxWarps * 32) v += __ldcg(term + i);
  sh[tid] = v;
  __syncthreads();
  for (int s2 = kAuxWarps * 16; s2 > 0; s2 >>= 1) {
    if (tid < s2) sh[tid] += sh[tid + s2];
    __syncthreads();
  }
  if (tid == 0) aux[0] = (float)((double)alpha * (double)E * sh[0]);
  if (zsum_part != nullptr) {
    // z-loss = coef * mean_t lse_t^2 over the router CTAs' sums, fixed tree
    __syncthreads();
    double z = 0.0;
    for (int b = tid; b < nblk; b += kAuxWarps * 32) z += (double)zsum_part[b];
    sh[tid] = z;
    __syncthreads();
    for (int s2 = kAuxWarps * 16; s2 > 0; s2 >>= 1) {
      if (tid < s2) sh[tid] += sh[tid + s2];
      __syncthreads();
    }
    if (tid == 0) aux[1] = (float)((double)z_coef * sh[0] / (double)T);
  }
  if (tid == 0) *counter = 0u;
}

cudaError_t launch_aux(const float* psum_part, const int32_t* cnt_part, const float* zsum_part, int nblk, int E,
                       int64_t T, int k, float alpha, float z_coef, double* term, float* aux, cudaStream_t stream) {
  unsigned* counter = reinterpret_cast<unsigned*>(term + E);
  const int grid = T == 0 ? 1 : (E + kAuxWarps - 1) / kAuxWarps;
  launch_pdl(aux_kernel, grid, kAuxWarps * 32, 0, stream, psum_part, cnt_part, zsum_part, nblk, E, T, k, alpha, z_coef,
                                                  term, counter, aux);
  return cudaGetLastError();
}

}  // namespace moe
