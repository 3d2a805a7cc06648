// Dispatch permutation and gate-weighted combine: the single-GPU replacements of
// the dispatch and combine all-to-alls ("Expert-parallel MoE training"
// explainer: token dispatch to experts and the unpermute / multiply-by-gate /
// sum step; "Switch Routing" 2.1: y = p_i(x) E_i(x); dropped tokens contribute
// nothing and reach the output through the caller's residual).
//
// Both kernels are token-centric and HBM-bound: one warp per token, 16-byte
// vectors, every source row read exactly once.  Dispatch writes the token's
// row to each of its kept destination rows; combine reads the token's kept
// expert rows (plus its shared-expert row), accumulates in fp32 in choice-rank
// order and rounds once.  KM (a power of two >= k) bounds the per-token row
// arrays at compile time; U vector positions are in flight per lane, so every
// lane keeps U*KM 16-byte loads outstanding instead of one round trip at a time.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kPermWarps = 8;

// Source / destination row of each choice of token t (-1 when dropped) and its gate.
template <int KM>
__device__ __forceinline__ void token_rows(const PermuteParams& p, int64_t t, int (&row)[KM], float (&g)[KM]) {
#pragma unroll
  for (int r = 0; r < KM; ++r) {
    row[r] = -1;
    g[r] = 0.0f;
    if (r < p.k) {
      const int s = p.slot[t * p.k + r];
      const int e = p.ids[t * p.k + r];
      if (s >= 0 && e >= 0 && e < p.E && (int64_t)p.expert_offset[e] + s < p.rows_max) {
        row[r] = p.expert_offset[e] + s;
        if (p.gates != nullptr) g[r] = p.gates[t * p.k + r];
      }
    }
  }
}

template <int KM, int U>
__global__ void __launch_bounds__(kPermWarps * 32) dispatch_kernel(PermuteParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kPermWarps + (threadIdx.x >> 5);
  if (t >= p.T) return;
  int row[KM];
  float g[KM];
  token_rows<KM>(p, t, row, g);
  const int64_t rowbytes = (int64_t)p.H * p.elem_bytes;
  const int nvec = (int)(rowbytes / 16);
  const char* src = static_cast<const char*>(p.src) + t * rowbytes;
  char* dst = static_cast<char*>(p.dst);
  for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
    int4 val[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * 32;
      if (v < nvec) val[u] = ld_nc_v4(src + (int64_t)v * 16);
    }
#pragma unroll
    for (int r = 0; r < KM; ++r) {
      if (row[r] >= 0) {
        char* d = dst + (int64_t)row[r] * rowbytes;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int v = v0 + u * 32;
          if (v < nvec) st_v4(d + (int64_t)v * 16, val[u]);
        }
      }
    }
  }
}

template <typename ET, int KM, int U>
__global__ void __launch_bounds__(kPermWarps * 32) combine_kernel(PermuteParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int NE = 16 / sizeof(ET);
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kPermWarps + (threadIdx.x >> 5);
  if (t >= p.T) return;
  int row[KM];
  float g[KM];
  token_rows<KM>(p, t, row, g);
  const int64_t shared_row = p.n_shared ? (int64_t)p.expert_offset[p.E] + t : -1;
  const int64_t rowbytes = (int64_t)p.H * sizeof(ET);
  const int nvec = (int)(rowbytes / 16);
  const char* ybuf = static_cast<const char*>(p.src);
  char* y = static_cast<char*>(p.dst) + t * rowbytes;
  for (int v0 = lane; v0 < nvec; v0 += 32 * U) {
    int4 val[U][KM];
    int4 sv[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * 32;
      if (v < nvec) {
#pragma unroll
        for (int r = 0; r < KM; ++r)
          if (row[r] >= 0) val[u][r] = ld_nc_v4(ybuf + (int64_t)row[r] * rowbytes + (int64_t)v * 16);
        if (shared_row >= 0) sv[u] = ld_nc_v4(ybuf + shared_row * rowbytes + (int64_t)v * 16);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * 32;
      if (v >= nvec) continue;
      float acc[NE];
#pragma unroll
      for (int c = 0; c < NE; ++c) acc[c] = 0.0f;
#pragma unroll
      for (int r = 0; r < KM; ++r) {
        if (row[r] >= 0) {
          const ET* e = reinterpret_cast<const ET*>(&val[u][r]);
#pragma unroll
          for (int c = 0; c < NE; ++c) acc[c] = fmaf(g[r], Elem<ET>::to_f(e[c]), acc[c]);
        }
      }
      if (shared_row >= 0) {
        const ET* e = reinterpret_cast<const ET*>(&sv[u]);
#pragma unroll
        for (int c = 0; c < NE; ++c) acc[c] += Elem<ET>::to_f(e[c]);
      }
      int4 out;
      ET* o = reinterpret_cast<ET*>(&out);
#pragma unroll
      for (int c = 0; c < NE; ++c) o[c] = Elem<ET>::from_f(acc[c]);
      st_v4(y + (int64_t)v * 16, out);
    }
  }
}

// Instantiation for k <= KM, with U*KM loads in flight per lane.
template <int KM>
static void launch_dispatch_km(const PermuteParams& p, unsigned grid, cudaStream_t s) {
  constexpr int U = KM >= 8 ? 2 : 4;
  launch_pdl(dispatch_kernel<KM, U>, grid, kPermWarps * 32, 0, s, p);
}

// U: vector positions per lane in flight, at most what one row needs (a
// lane's U * KM loads are held in registers, which bound the warps per SM).
template <typename ET, int KM>
static void launch_combine_km(const PermuteParams& p, unsigned grid, cudaStream_t s) {
  constexpr int UMAX = KM >= 16 ? 1 : KM >= 8 ? 2 : 4;
  const int64_t nvec = (int64_t)p.H * (int64_t)sizeof(ET) / 16;
  if (UMAX >= 2 && nvec <= 32) launch_pdl(combine_kernel<ET, KM, 1>, grid, kPermWarps * 32, 0, s, p);
  else if (UMAX >= 4 && nvec <= 64) launch_pdl(combine_kernel<ET, KM, 2>, grid, kPermWarps * 32, 0, s, p);
  else launch_pdl(combine_kernel<ET, KM, UMAX>, grid, kPermWarps * 32, 0, s, p);
}

cudaError_t launch_dispatch(const PermuteParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((p.T + kPermWarps - 1) / kPermWarps);
  if (p.k <= 1) launch_dispatch_km<1>(p, grid, stream);
  else if (p.k <= 2) launch_dispatch_km<2>(p, grid, stream);
  else if (p.k <= 4) launch_dispatch_km<4>(p, grid, stream);
  else if (p.k <= 8) launch_dispatch_km<8>(p, grid, stream);
  else launch_dispatch_km<16>(p, grid, stream);
  return cudaGetLastError();
}

template <typename ET>
static void launch_combine_t(const PermuteParams& p, unsigned grid, cudaStream_t stream) {
  if (p.k <= 1) launch_combine_km<ET, 1>(p, grid, stream);
  else if (p.k <= 2) launch_combine_km<ET, 2>(p, grid, stream);
  else if (p.k <= 4) launch_combine_km<ET, 4>(p, grid, stream);
  else if (p.k <= 8) launch_combine_km<ET, 8>(p, grid, stream);
  else launch_combine_km<ET, 16>(p, grid, stream);
}

cudaError_t launch_combine(const PermuteParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((p.T + kPermWarps - 1) / kPermWarps);
  if (p.elem_bytes == 2) launch_combine_t<__nv_bfloat16>(p, grid, stream);
  else launch_combine_t<float>(p, grid, stream);
  return cudaGetLastError();
}

}  // namespace moe
