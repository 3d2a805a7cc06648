// Grouped GEMM on pairs of SMs (tcgen05.mma.cta_group::2), for the expert
// contractions when they are compute-bound.
//
// Method: the per-expert FFN of an MoE layer ("Expert-parallel MoE training"
// explainer: experts as grouped MLPs, SwiGLU experts with gate / up / down
// matrices in worked example 2; MegaBlocks' dropless layout with every expert
// batch padded to a multiple of 128 rows).  Same contraction as the 1-SM
// grouped GEMM (grouped_gemm.cu): for every group g and its rows,
//     D[rows, n-tile] = epi( A[rows, :] * B_g[n-tile, :]^T ),
// bf16 operands, fp32 accumulation in tensor memory, bf16 output.
//
// Why a pair: a 128 x 256 tile on one SM needs 48 KB of operands per 64-k step
// for 2*128*256*64 flops, ~96 bytes per clock per SM at the MMA rate, more than
// L2 feeds.  Two SMs of a cluster multiply a 256 x 256 tile together: each loads
// its own 128 rows of A and one half of the 256 B rows (32 KB per step), and one
// MMA instruction issued by the even CTA reads both CTAs' shared memory and
// writes each CTA's 128 accumulator rows into that CTA's tensor memory.
//
// A pair tile covers two consecutive 128-row blocks of one group, so both
// halves use the group's weights.  A group with an odd number of blocks ends
// with a pair tile whose second half lies past the group: that half's rows are
// not loaded and not stored.  The pair tiles of each group are numbered by a
// prefix over the groups (pair_prefix_kernel), and the tiles are walked
// pair-block-major, n fastest, one cluster per two SMs, persistent.
//
// Roles, per CTA of the pair (576 threads):
//   warp 0      TMA producer (both CTAs): A rows and this CTA's half of B into
//               a 6-stage ring of 32 KB.  Every copy completes on the EVEN CTA's
//               full barrier (.cta_group::2 form), which the even CTA's producer
//               arms with the bytes of both CTAs.
//   warp 1      even CTA: issues tcgen05.mma.cta_group::2 (M = 256, N = 256,
//               K = 16) from one lane and commits with a multicast to both CTAs'
//               empty / accumulator-full barriers.  Both CTAs: allocate and free
//               512 TMEM columns together (two 256-column accumulators).
//   warps 2-17  epilogue (both CTAs): tcgen05.ld of this CTA's 128 rows, the
//               activation, bf16 staging in shared memory and TMA stores; then
//               one arrival per warp on the even CTA's accumulator-empty barrier.
// No load in this file uses cluster multicast.  Every mbarrier wait is bounded:
// on expiry the CTA records MOE_ETIMEOUT, raises both CTAs' abort flags, stops
// issuing, waits (bounded) for what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace moe {
namespace g2 {

using namespace tcx;

constexpr int BM = 128;                         // rows per CTA (256 per pair)
constexpr int BH = 128;                         // B rows per CTA (MMA N = 256)
constexpr int BK = 64;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BH * BK * 2;            // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
constexpr int STAGES = 6;
constexpr int RING_BYTES = STAGES * STAGE_BYTES;
constexpr int EPI_WARPS = 16;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int ACC_COLS = 256;
constexpr int TMEM_COLS = 2 * ACC_COLS;
constexpr int STAGE_OUT_BYTES = 32 * 32 * 2;
constexpr int STAGING_BYTES = EPI_WARPS * STAGE_OUT_BYTES;
constexpr int SMEM_BYTES = RING_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct KParams {
  CUtensorMap tmA, tmAs, tmB0, tmB1, tmSB0, tmSB1;
  CUtensorMap tmD;       // bf16 output [rows, N_out], box 32 x 32, 64-byte swizzle
  const int32_t* off;    // [ngroups + 1] row offsets (multiples of 128)
  const int32_t* pp;     // [ngroups + 1] exclusive prefix of the groups' pair tiles
  DevStatus* status;
  int64_t rows_max;
  int K, N_out, E, n_shared, epi;
  int as_sep;            // 1: the shared block's A rows come from tmAs (row - off[E])
  int b_packed;          // 1: B maps are 5-D over packed weights
};

// ---------------------------------------------------------------- cluster helpers
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_count() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
  return r;
}
// Shared::cluster address of `local` (a shared::cta address) in CTA `rank`.
__device__ __forceinline__ uint32_t map_to(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" :: "r"(cluster_addr), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}
// Acquire at cluster scope: the barrier may complete through the peer CTA's
// copies or arrivals.
__device__ __forceinline__ bool mbar_try_wait_cl(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_cl(uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  if (mbar_try_wait_cl(bar, parity)) return true;
  const long long t0 = clock64();
  while (true) {
    if (mbar_try_wait_cl(bar, parity)) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitCycles) return false;
  }
}
// Drain wait (no abort check): bounded by kWaitCycles.
__device__ __forceinline__ void mbar_drain_cl(uint32_t bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait_cl(bar, parity) && clock64() - t0 < kWaitCycles) {}
}

// TMA loads whose completion goes to a barrier that may sit in the peer CTA.
__device__ __forceinline__ void tma2_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile("cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3}], [%4];"
               :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void tma2_load_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z,
                                             uint32_t bar) {
  asm volatile("cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %3, %4}], [%5];"
               :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar) : "memory");
}
// Packed weights: coordinates (0, 0, k block, n block, group).
__device__ __forceinline__ void tma2_load_5d(uint32_t dst, const CUtensorMap* map, int c2, int c3, int c4,
                                             uint32_t bar) {
  asm volatile("cp.async.bulk.tensor.5d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
               " [%0], [%1, {%2, %2, %3, %4, %5}], [%6];"
               :: "r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(c2), "r"(c3), "r"(c4), "r"(bar)
               : "memory");
}

__device__ __forceinline__ void umma2(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                      uint32_t accum) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
               :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accum) : "memory");
}
// Arrive once on the barrier at this offset in both CTAs of the pair when the
// MMAs issued so far have completed.
__device__ __forceinline__ void umma2_commit_both(uint32_t bar) {
  const uint16_t mask = 3;
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               :: "r"(bar), "h"(mask) : "memory");
}

// Pair tile -> (group, rows).  pp is nondecreasing with pp[0] = 0.
__device__ __forceinline__ int find_pair_group(const int32_t* pp, int ngroups, int64_t pm) {
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(pp + mid) <= pm) lo = mid; else hi = mid - 1;
  }
  return lo;
}

struct Tile {
  int g;           // group
  int64_t row0;    // first row of the pair tile
  int64_t end;     // end of the group's rows
  int nt;          // n tile
};
__device__ __forceinline__ Tile decode(const KParams& p, int ngroups, int n_tiles_n, int64_t tile) {
  Tile t;
  const int64_t pm = tile / n_tiles_n;
  t.nt = (int)(tile - pm * n_tiles_n);
  t.g = find_pair_group(p.pp, ngroups, pm);
  const int64_t beg = min((int64_t)__ldg(p.off + t.g), p.rows_max);
  t.end = min((int64_t)__ldg(p.off + t.g + 1), p.rows_max);
  t.row0 = beg + (pm - __ldg(p.pp + t.g)) * (2 * BM);
  return t;
}

__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_2sm_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* staging = smem + RING_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES + STAGING_BYTES);
  // bars: full[STAGES], empty[STAGES], tfull[2], tempty[2], drain
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * STAGES), tempty0 = smem_u32(bars + 2 * STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const bool swiglu = p.epi == MOE_ACT_SWIGLU;
  const int ngroups = p.E + (p.n_shared ? 1 : 0);
  // raise the abort flag of both CTAs of the pair
  auto abort_pair = [&](int info) {
    *abort_flag = 1;
    st_cluster_u32(map_to(smem_u32((const void*)abort_flag), rank ^ 1u), 1u);
    set_status(p.status, MOE_ETIMEOUT, info);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull0 + 8 * b, 1); mbar_init(tempty0 + 8 * b, 2 * EPI_WARPS); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_map(&p.tmA); prefetch_map(&p.tmB0); prefetch_map(&p.tmD);
    if (p.n_shared) { prefetch_map(&p.tmAs); prefetch_map(&p.tmSB0); }
    if (swiglu) { prefetch_map(&p.tmB1); if (p.n_shared) prefetch_map(&p.tmSB1); }
  }
  if (warp == 1) {
    // both CTAs allocate together: the same columns in each CTA's TMEM
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();               // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The MMA writes both CTAs' accumulators at the even CTA's column address:
  // the joint allocation must have given both CTAs the same columns (checked
  // symmetrically, so both CTAs skip the work together if not).
  const bool tmem_same = ld_cluster_u32(map_to(smem_u32(tmem_slot), rank ^ 1u)) == tmem_base;
  pdl_wait();
  if (!tmem_same && threadIdx.x == 0) set_status(p.status, MOE_EDEVICE, 30);

  const int64_t n_pairs = tmem_same ? __ldg(p.pp + ngroups) : 0;
  const int n_step = swiglu ? BH : 2 * BH;                 // output columns per tile
  const int n_tiles_n = (p.N_out + n_step - 1) / n_step;
  const int64_t n_tiles = n_pairs * n_tiles_n;
  const int nk = (p.K + BK - 1) / BK;
  const int64_t cid = cluster_id(), ncl = cluster_count();

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to(full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[STAGES] = {0, 0, 0, 0, 0, 0};
      bool ok = true;
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        const Tile t = decode(p, ngroups, n_tiles_n, tile);
        const bool sh = t.g == p.E;
        const bool sep = sh && p.as_sep;
        const int64_t my_row = t.row0 + rank * BM;
        const bool a_live = my_row < t.end;
        const bool peer_live = t.row0 + BM < t.end;
        const CUtensorMap* ma = sep ? &p.tmAs : &p.tmA;
        const int arow = (int)(sep ? my_row - __ldg(p.off + p.E) : my_row);
        const int z = sh ? 0 : t.g;
        // B half: rows [n0 + 128 rank, +128) of W, or SwiGLU: gate rows (even
        // CTA) / up rows (odd CTA) [n0, n0 + 128)
        const CUtensorMap* mb = (swiglu && rank == 1) ? (sh ? &p.tmSB1 : &p.tmB1) : (sh ? &p.tmSB0 : &p.tmB0);
        const int nrow = swiglu ? t.nt * BH : t.nt * 2 * BH + (int)rank * BH;
        const uint32_t tx = 2 * B_BYTES + A_BYTES * (peer_live ? 2 : 1);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_cl(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = full_leader0 + 8 * stage;
          if (leader) mbar_expect_tx(full0 + 8 * stage, tx);
          if (a_live) tma2_load_2d(sa, ma, kb * BK, arow, fb);
          if (p.b_packed) tma2_load_5d(sb, mb, kb, nrow / 128, z, fb);
          else tma2_load_3d(sb, mb, kb * BK, nrow, z, fb);
          fills[stage]++;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) abort_pair(20);
      // never leave with a copy still writing shared memory: the even CTA's full
      // barrier completes only when both CTAs' copies of a stage have landed;
      // the odd CTA's copies of a stage have landed once the MMAs consumed it
      for (int s = 0; s < STAGES; ++s)
        if (fills[s]) {
          if (leader) mbar_drain_cl(full0 + 8 * s, (fills[s] - 1) & 1u);
          else mbar_drain_cl(empty0 + 8 * s, (fills[s] - 1) & 1u);
        }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA)
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc(2 * BH, 2 * BM);
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        if (!mbar_wait_cl(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * ACC_COLS);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_cl(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * STAGE_BYTES);
          const uint64_t ad = sw128_desc(sa), bd = sw128_desc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)         // 16 elements = 32 bytes along K
            umma2(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma2_commit_both(empty0 + 8 * stage);      // both CTAs' stage is free once these finish
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(tfull0 + 8 * acc);          // both CTAs' accumulators are ready
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) abort_pair(21);
      umma2_commit_both(drain);                       // every MMA issued, in both CTAs' view
    }
    if (lane == 0) mbar_drain_cl(drain, 0);           // both CTAs: no MMA still reads or writes
  } else {
    // ---------------- epilogue (both CTAs): this CTA's 128 rows of the pair tile
    const int ew = warp - 2;
    const int sub = warp & 3;                   // TMEM sub-partition this warp may access
    const int quarter = ew >> 2;
    const uint32_t stage_out = smem_u32(staging + ew * STAGE_OUT_BYTES);
    const uint32_t tempty_leader0 = map_to(tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = cid; tile < n_tiles; tile += ncl) {
      const Tile t = decode(p, ngroups, n_tiles_n, tile);   // before the wait: off its critical path
      if (!mbar_wait_cl(tfull0 + 8 * acc, acc_phase, abort_flag)) {
        if (lane == 0) abort_pair(22);
        break;
      }
      tc_fence_after();
      const int64_t my_row = t.row0 + rank * BM;
      if (my_row < t.end) {
        const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * ACC_COLS);
        const int ncol0 = t.nt * n_step;
        for (int c = quarter * 32; c < n_step; c += 4 * 32) {
          __syncwarp();
          float v[32];
          tmem_ld(tbase + (uint32_t)c, v, 32);
          if (swiglu) {
            float u[32];
            tmem_ld(tbase + (uint32_t)(BH + c), u, 32);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = act_silu(v[i]) * u[i];
          } else {
            tmem_wait_ld();
            if (p.epi == MOE_ACT_RELU) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = act_relu(v[i]);
            } else if (p.epi == MOE_ACT_GELU) {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = act_gelu(v[i]);
            }
          }
          // 32 rows x 32 columns through the warp's staging buffer (16-byte chunk
          // j of row r at j ^ ((r >> 1) & 3): the TMA 64-byte swizzle) and out
          // with one TMA store
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q)
            st_shared_v4(stage_out + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                         pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                         pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&p.tmD, stage_out, ncol0 + c, (int)(my_row + sub * 32));
            bulk_commit();
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();               // the peer's MMAs and epilogue are done with both CTAs' memory
  tc_fence_after();
  pdl_trigger();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// One warp: pp[g] = sum over g' < g of ceil(blocks(g') / 2), blocks(g') the
// 128-row blocks of group g' clipped to rows_max; pp[ngroups] = the total.
__global__ void pair_prefix_kernel(const int32_t* off, int ngroups, int64_t rows_max, int32_t* pp) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x;
  const int seg = (ngroups + 31) / 32;
  const int g0 = min(ngroups, lane * seg), g1 = min(ngroups, g0 + seg);
  auto pairs = [&](int g) {
    const int64_t b = min((int64_t)off[g], rows_max), e = min((int64_t)off[g + 1], rows_max);
    const int64_t blocks = e > b ? (e - b + BM - 1) / BM : 0;
    return (int)((blocks + 1) / 2);
  };
  int s = 0;
  for (int g = g0; g < g1; ++g) s += pairs(g);
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - s;
  for (int g = g0; g < g1; ++g) {
    pp[g] = run;
    run += pairs(g);
  }
  if (lane == 31) pp[ngroups] = incl;
}

// 2-D map over a row-major bf16 matrix [rows, K], box 64 x 128.
static bool map_rows(CUtensorMap* m, const void* base, int64_t rows, int K) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 2;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)K;
  key.dims[1] = (cuuint64_t)rows;
  key.strides[0] = (cuuint64_t)K * 2;
  key.box[0] = BK;
  key.box[1] = BM;
  return encode_cached(m, key);
}

// 3-D map over stacked weights [G, N, K], box 64 x 128 x 1 (rows past N read as zero).
static bool map_weights(CUtensorMap* m, const void* base, int G, int N, int K) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 3;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)K;
  key.dims[1] = (cuuint64_t)N;
  key.dims[2] = (cuuint64_t)G;
  key.strides[0] = (cuuint64_t)K * 2;
  key.strides[1] = (cuuint64_t)N * K * 2;
  key.box[0] = BK;
  key.box[1] = BH;
  key.box[2] = 1;
  return encode_cached(m, key);
}

// 5-D map over packed weights [G][N/128][K/64][128][64]: one box = one 16 KB block.
static bool map_packed(CUtensorMap* m, const void* base, int G, int N, int K) {
  const cuuint64_t kb = (cuuint64_t)((K + BK - 1) / BK), nb = (cuuint64_t)((N + 127) / 128);
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 5;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = BK;
  key.dims[1] = 128;
  key.dims[2] = kb;
  key.dims[3] = nb;
  key.dims[4] = (cuuint64_t)G;
  key.strides[0] = BK * 2;
  key.strides[1] = (cuuint64_t)BK * 128 * 2;
  key.strides[2] = key.strides[1] * kb;
  key.strides[3] = key.strides[2] * nb;
  key.box[0] = BK;
  key.box[1] = 128;
  key.box[2] = key.box[3] = key.box[4] = 1;
  return encode_cached(m, key);
}

// 2-D map over the bf16 output [rows, N], box 32 x 32, 64-byte swizzle (TMA store).
static bool map_out(CUtensorMap* m, const void* base, int64_t rows, int N) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 2;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_64B;
  key.dims[0] = (cuuint64_t)N;
  key.dims[1] = (cuuint64_t)rows;
  key.strides[0] = (cuuint64_t)N * 2;
  key.box[0] = 32;
  key.box[1] = 32;
  return encode_cached(m, key);
}

// Clusters of two CTAs (one per SM) that can be resident at once (cached per device).
static int resident_pairs() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& c = cache[dev & 63];
  if (c == 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * sm_count());
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_2sm_kernel, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = sm_count() / 2;
    }
    c = n;
  }
  return c;
}

}  // namespace g2

bool grouped_gemm_2sm_supported(const GemmParams& p) {
  return p.gather_src == nullptr && p.scatter_dst == nullptr && p.pair_prefix != nullptr;
}

cudaError_t launch_grouped_gemm_2sm(const GemmParams& p, cudaStream_t stream) {
  using namespace g2;
  if (p.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  KParams k{};
  bool ok = map_rows(&k.tmA, p.a_routed, p.rows_max, p.K);
  ok = ok && map_rows(&k.tmAs, p.a_shared ? p.a_shared : p.a_routed, p.a_shared ? p.T : p.rows_max, p.K);
  const void* b1 = p.b1 ? p.b1 : p.b0;
  const void* s0 = p.sb0 ? p.sb0 : p.b0;
  const void* s1 = p.sb1 ? p.sb1 : s0;
  if (p.b_packed) {
    ok = ok && map_packed(&k.tmB0, p.b0, p.E, p.Nw, p.K);
    ok = ok && map_packed(&k.tmB1, b1, p.E, p.Nw, p.K);
    ok = ok && map_packed(&k.tmSB0, s0, 1, p.Nw, p.K);
    ok = ok && map_packed(&k.tmSB1, s1, 1, p.Nw, p.K);
  } else {
    ok = ok && map_weights(&k.tmB0, p.b0, p.E, p.Nw, p.K);
    ok = ok && map_weights(&k.tmB1, b1, p.E, p.Nw, p.K);
    ok = ok && map_weights(&k.tmSB0, s0, 1, p.Nw, p.K);
    ok = ok && map_weights(&k.tmSB1, s1, 1, p.Nw, p.K);
  }
  ok = ok && map_out(&k.tmD, p.d, p.rows_max, p.Nw);
  if (!ok) return cudaErrorInvalidValue;
  const int ngroups = p.E + (p.n_shared ? 1 : 0);
  if (p.pair_prefix_ready == 0)
    launch_pdl(pair_prefix_kernel, 1, 32, 0, stream, p.expert_offset, ngroups, p.rows_max, p.pair_prefix);
  k.off = p.expert_offset;
  k.pp = p.pair_prefix;
  k.status = p.status;
  k.rows_max = p.rows_max;
  k.K = p.K;
  k.N_out = p.Nw;
  k.E = p.E;
  k.n_shared = p.n_shared;
  k.epi = p.epi;
  k.as_sep = p.a_shared != nullptr;
  k.b_packed = p.b_packed;
  cudaError_t e = ensure_smem(grouped_gemm_2sm_kernel, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2 * resident_pairs());
  cfg.blockDim = dim3(THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, grouped_gemm_2sm_kernel, k);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
