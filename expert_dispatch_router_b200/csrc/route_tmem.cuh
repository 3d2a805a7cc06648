// Routing of a router tile's 128 tokens from its fp32 accumulator in tensor
// memory, shared by the one-SM router (grouped_gemm.cu) and the SM-pair router
// (router_pair.cu).  Method: "Expert-parallel MoE training" explainer, router
// section (softmax then top-k, Megatron pre_softmax=False; sigmoid scores) and
// aux-loss section; "Switch Routing", 2.1 (gate = p_i(x)); ST-MoE's router
// z-loss; GShard's random dispatch of the second choice.
//
// The kernel calling it has 16 epilogue warps (512 threads, named barrier 1
// among them), four per TMEM sub-partition, and at least 22 KB of shared
// staging for the exchange below; named barriers 2-5 belong to it.
#pragma once
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace moe {

constexpr int kRouteTokens = 128;               // tokens of one router tile (TMEM lanes)
constexpr int kRouteThreads = 512;              // the 16 epilogue warps
constexpr int kRouteStagingBytes = 512 * 4 * 3 + 1024 * 8 + 1024 * 4 + 256 * 4 + 16;

// 8 columns of this warp's 32 lanes from / to tensor memory (one load shape:
// the routing's code runs once per tile and is fetched cold).
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const float (&v)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};"
               :: "r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                  "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                  "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
               : "memory");
}

// The routing's top-k bound for k choices: one instantiation each for k = 1,
// 2, <= 4, <= 8 and <= 16 (the sorted key lists live in registers).
inline int route_km_of(int k) { return k <= 1 ? 1 : k <= 2 ? 2 : k <= 4 ? 4 : k <= 8 ? 8 : 16; }

__device__ __forceinline__ void route_bar() {
  asm volatile("bar.sync 1, %0;" :: "r"(kRouteThreads) : "memory");
}

// Routing of one router tile's 128 tokens straight from its accumulator
// (lane = token, columns = experts), a token per thread.  The four warps of a
// TMEM sub-partition (the same 32 tokens) take four ranges of W columns each
// and meet at their own named barrier (2 + sub) to combine, in a fixed order:
// the maximum, the sums of exp(l - m) (and of the sigmoids), and the top-k,
// chosen one rank at a time from the four ranges' sorted lists (keys: larger
// logit first, equal logits -> smaller expert; the order the oracle uses).
// Selection counts add up in shared memory (integers: any order gives the same
// total); each expert's probability sum over the tile's tokens is a fixed
// reduce-scatter butterfly over the lanes, then the four sub-partitions in order.  The tile's
// sums go to row 4 * mt of the 32-token partial arrays and rows 4 mt + 1 ..
// 4 mt + 3 are zeroed.  The logit offset, where there is one, is added once
// and the sums written back to TMEM for the later passes.
__device__ __forceinline__ void sub_bar(int sub) {
  asm volatile("bar.sync %0, 128;" :: "r"(2 + sub) : "memory");
}
__device__ __forceinline__ unsigned long long route_key(float l, int e) {
  return ((unsigned long long)to_ordered(l) << 32) | (unsigned long long)(0xffffffffu - (uint32_t)e);
}
template <int KM>
__device__ __forceinline__ void route_tile_tmem(const RouterParams& rp, int64_t nblk, int64_t mt, int sub, int quarter,
                                                int lane, uint8_t* staging, uint32_t tacc, int ncols) {
  using namespace tcx;
  const int E = rp.E, k = rp.k;
  const int tid = (sub * 4 + quarter) * 32 + lane;                 // 0 .. 511, unique per thread
  const int64_t t = mt * kRouteTokens + sub * 32 + lane;
  const bool tv = t < rp.T;
  // columns per quarter: 8, 16, 32 or 64 (a multiple of the columns of one
  // TMEM access, so that no access reaches into the next quarter's range);
  // columns at or past E are masked
  const int q4 = (ncols + 3) / 4;
  const int W = q4 <= 8 ? 8 : q4 <= 16 ? 16 : q4 <= 32 ? 32 : 64;
  const int c0 = quarter * W;
  const bool sigmoid = rp.score == MOE_SCORE_SIGMOID_TOPK;
  float* xmax = reinterpret_cast<float*>(staging);                 // [4 sub][4 quarter][32]
  float* xsum = xmax + 512;
  float* xss = xsum + 512;
  unsigned long long* xhead = reinterpret_cast<unsigned long long*>(xss + 512);   // [2][4][4][32]
  float* xps = reinterpret_cast<float*>(xhead + 1024);            // [4 sub][256]
  int* xcnt = reinterpret_cast<int*>(xps + 1024);                 // [256]
  float* xz = reinterpret_cast<float*>(xcnt + 256);               // [4]
  
  if (tid < 256) xcnt[tid] = 0;
  route_bar();                                                  // the staging area is free; counts zeroed

  // 1. logits (+ offset) -> this range's maximum and sorted top-k keys
  unsigned long long key[KM];
#pragma unroll
  for (int i = 0; i < KM; ++i) key[i] = 0ull;
  float m = -INFINITY;
#pragma unroll 1
  for (int cc = 0; cc < W; cc += 8) {
    float v[8];
    tmem_ld8(tacc + (uint32_t)(c0 + cc), v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = c0 + cc + j;
      if (tv && e < E) {
        if (rp.logit_add != nullptr) v[j] += rp.logit_add[t * E + e];
        if (rp.logits_out != nullptr) rp.logits_out[t * E + e] = v[j];
        m = fmaxf(m, v[j]);
        unsigned long long x = route_key(v[j], e);
#pragma unroll
        for (int i = 0; i < KM; ++i)
          if (i < k) {
            const unsigned long long hi = key[i] > x ? key[i] : x;
            x = key[i] > x ? x : key[i];
            key[i] = hi;
          }
      }
    }
    if (rp.logit_add != nullptr) tmem_st8(tacc + (uint32_t)(c0 + cc), v);
  }
  if (rp.logit_add != nullptr) tmem_wait_st();
  xmax[tid] = m;
  sub_bar(sub);
  {
    const float* q = xmax + sub * 128 + lane;
    m = fmaxf(fmaxf(q[0], q[32]), fmaxf(q[64], q[96]));
  }

  // 2. sums of exp(l - m) (and of sigmoid(l)) over the whole token
  float s = 0.0f, ss = 0.0f;
#pragma unroll 1
  for (int cc = 0; cc < W; cc += 8) {
    float v[8];
    tmem_ld8(tacc + (uint32_t)(c0 + cc), v);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (tv && c0 + cc + j < E) {
        s += expf(v[j] - m);
        if (sigmoid) ss += 1.0f / (1.0f + expf(-v[j]));
      }
    }
  }
  xsum[tid] = s;
  xss[tid] = ss;
  sub_bar(sub);
  {
    const float* q = xsum + sub * 128 + lane;
    s = ((q[0] + q[32]) + q[64]) + q[96];
    const float* r = xss + sub * 128 + lane;
    ss = ((r[0] + r[32]) + r[64]) + r[96];
  }

  // 3. the top-k, one rank at a time: the best of the four ranges' heads
  unsigned long long sel[KM];
  int pos = 0;
#pragma unroll
  for (int r = 0; r < KM; ++r) {
    sel[r] = 0ull;
    if (r < k) {
      unsigned long long h = 0ull;
#pragma unroll
      for (int i = 0; i < KM; ++i)
        if (i == pos) h = key[i];
      unsigned long long* buf = xhead + (r & 1) * 512 + sub * 128 + lane;
      buf[quarter * 32] = h;
      sub_bar(sub);
      unsigned long long w = 0ull;
      int wq = 0;
#pragma unroll
      for (int q2 = 0; q2 < 4; ++q2) {
        const unsigned long long hq = buf[q2 * 32];
        if (hq > w) { w = hq; wq = q2; }
      }
      sel[r] = w;
      if (wq == quarter && w != 0ull) {
        ++pos;
        if (tv) atomicAdd(xcnt + (int)(0xffffffffu - (uint32_t)(w & 0xffffffffull)), 1);
      }
    }
  }

  // 4. gates and ids (the first quarter's warp writes its tokens' rows)
  if (quarter == 0 && tv) {
    float g[KM];
    float gs = 0.0f;
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      g[r] = 0.0f;
      if (r < k) {
        const float l = from_ordered((uint32_t)(sel[r] >> 32));
        g[r] = sigmoid ? 1.0f / (1.0f + expf(-l)) : expf(l - m);
        gs += g[r];
      }
    }
    const bool renorm = rp.score == MOE_SCORE_TOPK_SOFTMAX || rp.renorm;
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      if (r >= k) break;
      if (renorm) g[r] = g[r] / gs;
      else if (rp.score == MOE_SCORE_SOFTMAX_TOPK) g[r] = g[r] / s;
    }
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      if (r >= k) break;
      int e = sel[r] != 0ull ? (int)(0xffffffffu - (uint32_t)(sel[r] & 0xffffffffull)) : -1;
      float gr = g[r];
      // GShard top-2: the second choice is dispatched iff u_t < 2 g_t1
      if (r == 1 && rp.uniform != nullptr && !(rp.uniform[t] < 2.0f * gr)) { e = -1; gr = 0.0f; }
      rp.ids[t * k + r] = e;
      rp.gates[t * k + r] = gr;
    }
  }

  // 5. z-loss: lse^2 summed over the tile's tokens
  if (rp.zsum_part != nullptr && quarter == 0) {
    float z = 0.0f;
    if (tv) {
      const float lse = m + logf(s);
      z = lse * lse;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
    if (lane == 0) xz[sub] = z;
  }

  // 6. each expert's probability sum over the tile's tokens: per 8 columns a
  // reduce-scatter butterfly over the lanes (lane bits 4, 3, 2 halve the
  // columns each lane carries; bits 1, 0 finish the sum), after which lanes
  // 4c .. 4c + 3 hold column c's sum
  if (rp.psum_part != nullptr) {
    const float inv = 1.0f / (sigmoid ? ss : s);
    const bool b16 = (lane & 16) != 0, b8 = (lane & 8) != 0, b4 = (lane & 4) != 0;
#pragma unroll 1
    for (int cc = 0; cc < W; cc += 8) {
      float v[8];
      tmem_ld8(tacc + (uint32_t)(c0 + cc), v);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int e = c0 + cc + j;
        v[j] = (tv && e < E) ? (sigmoid ? 1.0f / (1.0f + expf(-v[j])) : expf(v[j] - m)) * inv : 0.0f;
      }
      float q4[4], q2[2];
#pragma unroll
      for (int i = 0; i < 4; ++i)      // bit 4 clear keeps columns 0-3, set keeps 4-7
        q4[i] = (b16 ? v[i + 4] : v[i]) + __shfl_xor_sync(0xffffffffu, b16 ? v[i] : v[i + 4], 16);
#pragma unroll
      for (int i = 0; i < 2; ++i)
        q2[i] = (b8 ? q4[i + 2] : q4[i]) + __shfl_xor_sync(0xffffffffu, b8 ? q4[i] : q4[i + 2], 8);
      float q1 = (b4 ? q2[1] : q2[0]) + __shfl_xor_sync(0xffffffffu, b4 ? q2[0] : q2[1], 4);
      q1 += __shfl_xor_sync(0xffffffffu, q1, 2);
      q1 += __shfl_xor_sync(0xffffffffu, q1, 1);
      const int e = c0 + cc + ((lane >> 2) & 7);
      if ((lane & 3) == 0 && e < E) xps[sub * 256 + e] = q1;
    }
  }
  route_bar();
  const int64_t row0 = 4 * mt;
  for (int idx = tid; idx < 4 * E; idx += kRouteThreads) {
    const int q = idx / E, e = idx - q * E;
    const int64_t row = row0 + q;
    if (row >= nblk) continue;
    float ps = 0.0f;
    int cs = 0;
    if (q == 0) {
      ps = ((xps[e] + xps[256 + e]) + xps[512 + e]) + xps[768 + e];
      cs = xcnt[e];
    }
    if (rp.psum_part != nullptr) rp.psum_part[row * E + e] = ps;
    if (rp.cnt_part != nullptr) rp.cnt_part[row * E + e] = cs;
  }
  if (tid == 0) {
    if (rp.zsum_part != nullptr) {
      const float z = ((xz[0] + xz[1]) + xz[2]) + xz[3];
      for (int q = 0; q < 4; ++q)
        if (row0 + q < nblk) rp.zsum_part[row0 + q] = q == 0 ? z : 0.0f;
    }
    if (mt == 0 && rp.aux_counter != nullptr) *rp.aux_counter = 0u;   // re-armed for moe_aux_loss
  }
  route_bar();                                                  // the staging area is free again
}

}  // namespace moe
