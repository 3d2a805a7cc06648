// Grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Method: the per-expert FFN of an MoE layer ("Expert-parallel MoE training"
// explainer: experts as grouped MLPs, SwiGLU experts with gate / up / down
// matrices in worked example 2; MegaBlocks' dropless layout with every expert
// batch padded to a multiple of 128 rows).  The expert FFN is the only dense
// contraction of the layer; "The MoE spends too much time on the gate network"
// measures it at 87-99% of the layer once dispatch is fixed.  The same kernel
// also computes the router logits (one group, fp32 store; see
// launch_router_gemm).
//
// One launch computes, for every 128-row block of every group g,
//     D[rows, n-tile] = epi( A[rows, :] * B_g[n-tile, :]^T )
// with bf16 operands and fp32 accumulation in tensor memory.
//   GEMM1: A = dispatched rows (the shared expert's block reads x directly),
//          B = W_in^T (or W_gate^T | W_up^T stacked for SwiGLU), epi = act, bf16 out.
//   GEMM2: A = activations h, B = W_out^T, epi = none, bf16 out.
//   router: A = x (its k coordinate wraps every H' columns), B = the three bf16
//          planes of Wg laid side by side along K, fp32 out.
//
// Kernel structure (one persistent CTA per SM, 576 threads):
//   warp 0      TMA producer: A box 64x128 and B boxes 64 x (<=128) per stage,
//               128-byte swizzle, a 4-8 stage ring guarded by full/empty mbarriers.
//   warp 1      allocates 512 TMEM columns and issues tcgen05.mma
//               (M=128, N<=256, K=16, kind::f16) from one lane; commits free the
//               smem stage and, per tile, signal the accumulator as full.
//   warps 2-17  epilogue: tcgen05.ld of the fp32 accumulator (four warps per
//               32-lane TMEM sub-partition, interleaving column chunks), the
//               activation, packing and 16-byte global stores.
// Two accumulators of 256 columns let the epilogue of one tile overlap the
// main loop of the next.  Tiles are walked m-block-major, n fastest, so CTAs
// running at the same time share the A block and the group's weights in L2.
// The group of an m-block comes from a binary search over the device-side
// offsets, so no host synchronisation is needed between routing and the GEMM.
// Every mbarrier wait is bounded; on expiry the CTA records MOE_ETIMEOUT, stops
// issuing work, drains what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"
#include "route_tmem.cuh"
#include "tc_common.cuh"

namespace moe {
namespace gg {

using namespace tcx;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB
constexpr int RING_BYTES = 4 * (A_BYTES + BN * BK * 2);   // 192 KB: 4 stages at N=256, more when narrower
constexpr int MAX_STAGES = 8;
constexpr int EPI_WARPS = 16;                      // 4 per TMEM sub-partition
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int GATHER_WARPS = 2;                    // fused dispatch: cp.async row gathers, 64 rows each
constexpr int THREADS_GATHER = THREADS + GATHER_WARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int STAGE_OUT_BYTES = 32 * 32 * 2;       // one warp's 32 x 32 bf16 output sub-tile
constexpr int STAGING_BYTES = EPI_WARPS * STAGE_OUT_BYTES;   // 32 KB
constexpr int SMEM_BYTES = RING_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct KParams {
  CUtensorMap tmA, tmAs, tmB0, tmB1, tmSB0, tmSB1;
  CUtensorMap tmB0h, tmSB0h;   // 192-column tiles: the same weights in 64-row boxes (half a packed block)
  CUtensorMap tmD;       // bf16 output [rows, N_out], box 32 x 32, 64-byte swizzle (TMA store)
  void* d;
  const int32_t* off;
  DevStatus* status;
  int64_t ld_d, rows_max;
  int64_t rows_static;   // >= 0: one group of this many rows (off unused)
  int64_t rows_store;    // rows >= rows_store are not stored
  int K, N_out, E, n_shared, epi;
  int as_sep;            // 1: the shared block's A rows come from tmAs (row - off[E]); 0: from tmA in place
  int bn_fixed;          // 0: N tile chosen on the device (256, 192 or 128); else this MMA N (multiple of 16)
  int allow192;          // 1: 192-column tiles may be chosen (tmB0h / tmSB0h are set)
  int bbox;              // rows of one B TMA box (128, or bn_fixed when smaller)
  int b_planes;          // router: 3 weight planes laid side by side along B's K; one stage holds the A
                         // chunk and the matching chunk of every plane, multiplied into one accumulator
  int plane_k;           // elements between planes along B's K
  int k_split;           // fp32 output only: each tile's k blocks split over this many tiles, each
                         // storing its partial sums to d + part * rows_store * ld_d
  int out_f32;           // 1: store the raw fp32 accumulator
  int b_packed;          // 1: B maps are 5-D over packed weights (16 KB blocks of 128 rows x 64 k)
  // fused dispatch: routed A rows gathered from gsrc [rows of K elements] by gidx
  // (warp 0 issues cp.async with the 128-byte swizzle applied by hand)
  const __nv_bfloat16* gsrc;
  const int32_t* gidx;
  // fused top-1 combine: routed rows stored to sdst[gidx[row]] * sgate[gidx[row]];
  // warp 0's idle lanes also zero sdst[t] for every token t with sslot[t] < 0
  __nv_bfloat16* sdst;
  const float* sgate;
  const int32_t* sslot;
  int64_t sT;
  // router: planes_per_stage 3 = a stage holds the A chunk and the matching
  // chunk of all three planes; 1 = one plane per stage (the k loop visits
  // (k block, plane) in the same order), for wide N where three planes would
  // leave too few stages.
  int planes_per_stage;
  // router with routing fused (ROUTE_KM > 0): the epilogue routes the tile's
  // 128 tokens from the accumulator (route_tile_tmem) and stores the tile's
  // partial sums in row 4 * m-block of the 32-token partial arrays (the other
  // three rows of the tile are zero).
  RouterParams rp;
  int64_t nblk;          // rows of the partial arrays (32 tokens each)
};

__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, %0;" :: "r"(EPI_WARPS * 32) : "memory");
}
// True iff `v` holds in every epilogue thread (a barrier: every epilogue warp
// takes the same branch after it, so none is left waiting at a later barrier).
__device__ __forceinline__ bool epilogue_all(bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred pi, po;\n\t"
               "setp.ne.u32 pi, %1, 0;\n\t"
               "bar.red.and.pred po, 1, %2, pi;\n\t"
               "selp.u32 %0, 1, 0, po;\n\t}"
               : "=r"(r) : "r"((uint32_t)v), "r"(EPI_WARPS * 32) : "memory");
  return r != 0;
}

// GATHER: routed A rows are gathered from p.gsrc by warps 18-19 (fused
// dispatch).  SCATTER: routed output rows go to p.sdst[token] * gate (fused
// top-1 combine).  Both false: every operand moves by TMA.  ROUTE_KM > 0:
// router logits with routing fused into the epilogue (E <= 256, k <= ROUTE_KM).
template <bool GATHER, bool SCATTER, int ROUTE_KM = 0>
__global__ void __launch_bounds__(GATHER ? THREADS_GATHER : THREADS, 1)
    grouped_gemm_kernel(const __grid_constant__ KParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* staging = smem + RING_BYTES;                 // per epilogue warp: 32 x 32 bf16, swizzled
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES + STAGING_BYTES);
  // bars: full[MAX_STAGES], empty[MAX_STAGES], tfull[2], tempty[2], drain
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + MAX_STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * MAX_STAGES), tempty0 = smem_u32(bars + 2 * MAX_STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * MAX_STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * MAX_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool swiglu = p.epi == MOE_ACT_SWIGLU;
  const bool grouped = p.rows_static < 0;
  const int ngroups = p.E + (p.n_shared ? 1 : 0);
  // full barrier arrivals per stage: the TMA lane's arrive.expect_tx, plus one
  // per gather lane
  const uint32_t full_count = GATHER ? 1u + GATHER_WARPS * 32u : 1u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) { mbar_init(full0 + 8 * s, full_count); mbar_init(empty0 + 8 * s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull0 + 8 * b, 1); mbar_init(tempty0 + 8 * b, EPI_WARPS * 32); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_map(&p.tmA); prefetch_map(&p.tmB0);
    if (p.n_shared) { prefetch_map(&p.tmAs); prefetch_map(&p.tmSB0); }
    if (swiglu) { prefetch_map(&p.tmB1); if (p.n_shared) prefetch_map(&p.tmSB1); }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  pdl_wait();                                    // inputs of earlier launches are complete from here on

  const int64_t rows_used = grouped ? min((int64_t)p.off[ngroups], p.rows_max) : p.rows_static;
  const int64_t n_mtiles = (rows_used + BM - 1) / BM;
  const int nk = (p.K + BK - 1) / BK;
  // Tile width: SwiGLU tiles hold 128 gate + 128 up columns (128 outputs),
  // the router a fixed N.  Otherwise 256, 192 or 128 columns, whichever keeps
  // the busiest SM's operand bytes lowest: a tile loads BM + bn rows of K per
  // k step through an SM whose intake rate is fixed, and the SM with the most
  // tiles (ceil(tiles / grid)) finishes last.  Ties go to the wider tile.
  // A 384-column tile (two 192-column accumulators, both TMEM buffers, sharing
  // each A stage: the A rows load half as often) when such tiles fit one wave,
  // so that no tile waits for the previous one's epilogue (not with the fused
  // gather, whose instance keeps its registers for the gather warps).
  int bn_auto = 256;
  bool wide = false;
  if (!swiglu && p.bn_fixed == 0) {
    auto cost = [&](int b) {
      const int64_t t = n_mtiles * ((p.N_out + b - 1) / b);
      return ((t + gridDim.x - 1) / gridDim.x) * (int64_t)(BM + b);
    };
    int64_t best = cost(256);
    if (p.allow192 && cost(192) < best) { best = cost(192); bn_auto = 192; }
    if (cost(128) < best) { best = cost(128); bn_auto = 128; }
    if (!GATHER && p.allow192 && n_mtiles * ((p.N_out + 383) / 384) <= (int64_t)gridDim.x &&
        (int64_t)(BM + 384) < best) {
      wide = true;
      bn_auto = 192;
    }
  }
  const int bn = p.bn_fixed ? p.bn_fixed : bn_auto;                 // MMA N
  const int n_step = swiglu ? BN / 2 : (wide ? 2 * bn : bn);        // output columns per tile
  const int n_tiles_n = (p.N_out + n_step - 1) / n_step;
  // tile = (m-block, n-tile, k part), k part fastest; part q owns k blocks
  // [q * nk_part, min(nk, (q + 1) * nk_part))
  const int n_parts = p.k_split;
  const int nk_part = (nk + n_parts - 1) / n_parts;
  const int64_t n_tiles = n_mtiles * n_tiles_n * n_parts;
  const int box_bytes = p.bbox * BK * 2;
  const int brows = wide ? 2 * bn : bn;                 // B rows of a tile
  const int n_boxes = swiglu ? 2 : brows / p.bbox;      // (192: a 128-row and a 64-row box)
  const int plane_bytes = swiglu ? 2 * box_bytes : brows * BK * 2;   // one plane's B chunk
  const int pps = p.b_planes == 1 ? 1 : p.planes_per_stage;   // planes per stage
  const int pass = p.b_planes / pps;                    // stages per k block
  const int stage_bytes = A_BYTES + pps * plane_bytes;
  const int n_stages = min(MAX_STAGES, RING_BYTES / stage_bytes);

  if (warp == 0) {
    if (SCATTER && lane > 0) {
      // fused top-1 combine: rows of fully dropped tokens are zero
      const int64_t nthr = (int64_t)gridDim.x * 31;
      const int nvec = p.N_out / 8;
      for (int64_t t = (int64_t)blockIdx.x * 31 + (lane - 1); t < p.sT; t += nthr)
        if (__ldg(p.sslot + t) < 0)
          for (int v = 0; v < nvec; ++v) st_v4(p.sdst + t * p.N_out + 8 * v, make_int4(0, 0, 0, 0));
    }
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[MAX_STAGES] = {0, 0, 0, 0, 0, 0, 0, 0};
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const int part = (int)(tile % n_parts);
        const int64_t mt = tile / n_parts / n_tiles_n;
        const int nt = (int)(tile / n_parts % n_tiles_n);
        const int kb0 = part * nk_part, kb1 = min(nk, kb0 + nk_part);
        const int64_t row0 = mt * BM;
        const int g = grouped ? find_group(p.off, ngroups, row0) : 0;
        const bool sh = grouped && g == p.E;
        const bool sep = sh && p.as_sep;
        const bool gat = GATHER && !sh;          // the gather warps fill this tile's A
        const CUtensorMap* ma = sep ? &p.tmAs : &p.tmA;
        const CUtensorMap* mb0 = sh ? &p.tmSB0 : &p.tmB0;
        const CUtensorMap* mb1 = sh ? &p.tmSB1 : &p.tmB1;
        const int arow = (int)(sep ? row0 - p.off[p.E] : row0);
        const int z = sh ? 0 : g;
        const int n0 = nt * n_step;
        for (int ks = kb0 * pass; ks < kb1 * pass; ++ks) {
          const int kb = ks / pass, j1 = ks - kb * pass;   // k block; its plane when pps == 1
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = full0 + 8 * stage;
          const int ka = kb * BK, kbb = kb * BK;
          mbar_expect_tx(fb, gat ? stage_bytes - A_BYTES : stage_bytes);
          if (!gat) tma_load_2d(sa, ma, ka, arow, fb);
          if (bn == 192 && !wide) {
            // a 128-row box and a 64-row half box in row order (n0 is a multiple of 64)
            const CUtensorMap* mh = sh ? &p.tmSB0h : &p.tmB0h;
            const bool lead_half = (n0 & 127) != 0;
            if (p.b_packed) {
              if (lead_half) {
                tma_load_5d_at(sb, mh, 64, kbb / BK, n0 / 128, z, fb);
                tma_load_5d(sb + 8192, mb0, kbb / BK, n0 / 128 + 1, z, fb);
              } else {
                tma_load_5d(sb, mb0, kbb / BK, n0 / 128, z, fb);
                tma_load_5d_at(sb + 16384, mh, 0, kbb / BK, n0 / 128 + 1, z, fb);
              }
            } else if (lead_half) {
              tma_load_3d(sb, mh, kbb, n0, z, fb);
              tma_load_3d(sb + 8192, mb0, kbb, n0 + 64, z, fb);
            } else {
              tma_load_3d(sb, mb0, kbb, n0, z, fb);
              tma_load_3d(sb + 16384, mh, kbb, n0 + 128, z, fb);
            }
          } else if (p.b_packed) {
            // packed weights: every box is one contiguous 16 KB block
            if (swiglu) {
              tma_load_5d(sb, mb0, kbb / BK, n0 / 128, z, fb);
              tma_load_5d(sb + box_bytes, mb1, kbb / BK, n0 / 128, z, fb);
            } else {
              for (int b = 0; b < n_boxes; ++b) tma_load_5d(sb + b * box_bytes, mb0, kbb / BK, n0 / 128 + b, z, fb);
            }
          } else if (swiglu) {
            tma_load_3d(sb, mb0, kbb, n0, z, fb);                 // gate rows
            tma_load_3d(sb + box_bytes, mb1, kbb, n0, z, fb);     // up rows
          } else {
            for (int j = 0; j < pps; ++j)
              for (int b = 0; b < n_boxes; ++b)
                tma_load_3d(sb + j * plane_bytes + b * box_bytes, mb0, (j + j1) * p.plane_k + kbb,
                            n0 + b * p.bbox, z, fb);
          }
          fills[stage]++;
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ETIMEOUT, 10);
      }
      // never leave with a bulk copy still writing this CTA's shared memory
      for (int s = 0; s < n_stages; ++s)
        if (fills[s]) {
          const long long t0 = clock64();
          while (!mbar_try_wait(full0 + 8 * s, (fills[s] - 1) & 1u) && clock64() - t0 < kWaitCycles) {}
        }
    }
  } else if (GATHER && warp >= 2 + EPI_WARPS) {
    // ---------------- gather producers (fused dispatch): warp gw fills A rows
    // [64 gw, 64 gw + 64) of every routed tile with 16-byte cp.async copies of x
    // rows, applying the 128-byte swizzle (chunk c of row r at c ^ (r & 7)).
    // Lane l copies chunk (l & 7) of rows 64 gw + 4 i + (l >> 3), i < 16.
    const int gw = warp - 2 - EPI_WARPS;
    const int c = lane & 7, lr = lane >> 3;
    const uint32_t sw_even = (uint32_t)((c ^ (lr & 7)) << 4), sw_odd = (uint32_t)((c ^ ((4 + lr) & 7)) << 4);
    const uint32_t row_off = (uint32_t)((64 * gw + lr) * 128);
    const int64_t rowbytes = (int64_t)p.K * 2;
    const char* xsrc = reinterpret_cast<const char*>(p.gsrc);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
      const int64_t mt = tile / n_parts / n_tiles_n;
      const int kb0 = (int)(tile % n_parts) * nk_part, kb1 = min(nk, kb0 + nk_part);
      const int64_t row0 = mt * BM;
      const int g = find_group(p.off, ngroups, row0);
      const bool gat = g != p.E;
      int tok[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) tok[i] = gat ? __ldg(p.gidx + row0 + 64 * gw + 4 * i + lr) : -1;
      for (int kb = kb0; kb < kb1; ++kb) {
        int good = 1;
        if (lane == 0) good = mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag);
        good = __shfl_sync(0xffffffffu, good, 0);
        if (!good) { ok = false; break; }
        const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
        const uint32_t fb = full0 + 8 * stage;
        if (gat) {
          const int kk = kb * BK + c * 8;
          const bool kin = kk < p.K;
          const char* kbase = xsrc + (int64_t)kk * 2;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t dst = sa + row_off + (uint32_t)(i * 512) + ((i & 1) ? sw_odd : sw_even);
            const bool live = kin && tok[i] >= 0;
            cp_async16(dst, live ? kbase + (int64_t)tok[i] * rowbytes : xsrc, live ? 16u : 0u);
          }
          cp_async_arrive(fb);
        } else {
          mbar_arrive(fb);                       // this tile's A comes by TMA
        }
        if (++stage == n_stages) { stage = 0; phase ^= 1u; }
      }
    }
    cp_async_wait_all();                         // no copy still writing shared memory
    if (!ok && lane == 0) {
      *abort_flag = 1;
      set_status(p.status, MOE_ETIMEOUT, 13);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc(bn);
      // wide: both accumulator buffers per tile, one 192-column MMA into each per
      // 16-k step, the B rows of the second starting 192 rows into the stage
      for (int64_t tile = blockIdx.x; tile < n_tiles && ok && wide; tile += gridDim.x) {
        const int kb0 = (int)(tile % n_parts) * nk_part, kb1 = min(nk, kb0 + nk_part);
        if (!mbar_wait(tempty0, acc_phase ^ 1u, abort_flag) || !mbar_wait(tempty0 + 8, acc_phase ^ 1u, abort_flag)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int ks = kb0; ks < kb1; ++ks) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          if (GATHER) fence_async_smem();
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          const uint64_t ad = sw128_desc(sa), bd0 = sw128_desc(sb), bd1 = sw128_desc(sb + (uint32_t)(bn * 128));
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint32_t acc_in = ((ks - kb0) | kk) != 0 ? 1u : 0u;
            umma(tmem_base, ad + (uint64_t)(kk * 2), bd0 + (uint64_t)(kk * 2), idesc, acc_in);
            umma(tmem_base + (uint32_t)BN, ad + (uint64_t)(kk * 2), bd1 + (uint64_t)(kk * 2), idesc, acc_in);
          }
          umma_commit(empty0 + 8 * stage);
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tfull0);
        acc_phase ^= 1u;
      }
      for (int64_t tile = blockIdx.x; tile < n_tiles && ok && !wide; tile += gridDim.x) {
        const int kb0 = (int)(tile % n_parts) * nk_part, kb1 = min(nk, kb0 + nk_part);
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int ks = kb0 * pass; ks < kb1 * pass; ++ks) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          if (GATHER) fence_async_smem();       // cp.async data (generic proxy) -> tensor-core reads
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          const uint64_t ad = sw128_desc(sa);
          for (int j = 0; j < pps; ++j) {
            const uint64_t bd = sw128_desc(sb + j * plane_bytes);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)   // advance 16 elements = 32 bytes along K
              umma(d_tmem, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc,
                   ((ks - kb0 * pass) | kk | j) != 0 ? 1u : 0u);
          }
          umma_commit(empty0 + 8 * stage);      // stage free once these MMAs finish
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * acc);          // accumulator ready for the epilogue
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ETIMEOUT, 11);
      }
      // wait for every MMA issued by this CTA before TMEM is released
      umma_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {}
    }
  } else if (warp < 2 + EPI_WARPS) {
    // ---------------- epilogue
    const int ew = warp - 2;
    const int sub = warp & 3;                  // TMEM sub-partition this warp may access
    const int quarter = ew >> 2;               // the four warps of a sub-partition split the chunks
    const int row_in_tile = sub * 32 + lane;
    const int chunk = n_step >= 128 ? 32 : n_step >= 64 ? 16 : 8;   // columns per tcgen05.ld
    const uint32_t stage_out = smem_u32(staging + ew * STAGE_OUT_BYTES);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      bool got = mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag);
      if constexpr (ROUTE_KM > 0) got = epilogue_all(got);   // the routing below has barriers
      if (!got) {
        *abort_flag = 1;
        set_status(p.status, MOE_ETIMEOUT, 12);
        break;
      }
      tc_fence_after();
      const int part = (int)(tile % n_parts);
      const int64_t mt = tile / n_parts / n_tiles_n;
      const int nt = (int)(tile / n_parts % n_tiles_n);
      const int64_t grow = mt * BM + row_in_tile;
      const bool row_ok = grow < p.rows_store;
      // fused top-1 combine: this lane's row is token st of the batch, weighted by sg
      int st = -1;
      float sg = 0.0f;
      if (SCATTER && row_ok) {
        st = __ldg(p.gidx + grow);
        if (st >= 0) sg = __ldg(p.sgate + st);
      }
      const int ncol0 = nt * n_step;                           // first output column of the tile
      const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BN);
      if constexpr (ROUTE_KM > 0) {
        // the router: route the tile's tokens from the accumulator itself
        route_tile_tmem<ROUTE_KM>(p.rp, p.nblk, mt, sub, quarter, lane, staging, tbase, bn);
      } else {
        for (int c = quarter * chunk; c < n_step; c += 4 * chunk) {
          __syncwarp();                                // converged for the warp-wide tcgen05.ld
          float v[32];
          const int acol = (wide && c >= bn) ? BN + (c - bn) : c;   // accumulator column (wide: second buffer)
          tmem_ld(tbase + (uint32_t)acol, v, chunk);
          if (swiglu) {
            float u[32];
            tmem_ld(tbase + (uint32_t)(BN / 2 + acol), u, chunk);
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
          const int col = ncol0 + c;
          if (p.out_f32) {
            if (!row_ok) continue;
            float* drow = static_cast<float*>(p.d) + (int64_t)part * p.rows_store * p.ld_d + grow * p.ld_d;
            const bool vec = (p.ld_d & 3) == 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              if (4 * q >= chunk) continue;
              const int cc = col + 4 * q;
              if (vec && cc + 4 <= p.N_out) {
                *reinterpret_cast<float4*>(drow + cc) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
              } else {
#pragma unroll
                for (int i = 0; i < 4; ++i)
                  if (cc + i < p.N_out) drow[cc + i] = v[4 * q + i];
              }
            }
          } else if (SCATTER) {
            // the warp's 32 rows x 32 columns go through its staging buffer (same
            // swizzle as below), then out row by row: lanes 4j..4j+3 write the 64
            // bytes of one row, eight rows per store instruction
            __syncwarp();                              // the previous chunk's reads are done
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_shared_v4(stage_out + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                           pack_bf16(sg * v[8 * q + 0], sg * v[8 * q + 1]), pack_bf16(sg * v[8 * q + 2], sg * v[8 * q + 3]),
                           pack_bf16(sg * v[8 * q + 4], sg * v[8 * q + 5]), pack_bf16(sg * v[8 * q + 6], sg * v[8 * q + 7]));
            __syncwarp();
            const int j = lane & 3;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int r = 8 * q + (lane >> 2);
              const int tr = __shfl_sync(0xffffffffu, st, r);
              if (tr >= 0 && 8 * j < chunk && col + 8 * j < p.N_out) {
                int4 val;
                asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                             : "=r"(val.x), "=r"(val.y), "=r"(val.z), "=r"(val.w)
                             : "r"(stage_out + r * 64 + ((j ^ ((r >> 1) & 3)) << 4)));
                st_v4(p.sdst + (int64_t)tr * p.N_out + col + 8 * j, val);
              }
            }
          } else {
            // bf16: this warp's 32 rows x 32 columns go through its staging buffer
            // (16-byte chunk j of row r at chunk j ^ ((r >> 1) & 3): the TMA 64-byte
            // swizzle, bank-conflict free) and out with one TMA store of full lines.
            if (lane == 0) bulk_wait_read0();          // the previous store has read the buffer
            __syncwarp();
#pragma unroll
            for (int q = 0; q < 4; ++q)
              st_shared_v4(stage_out + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                           pack_bf16(v[8 * q + 0], v[8 * q + 1]), pack_bf16(v[8 * q + 2], v[8 * q + 3]),
                           pack_bf16(v[8 * q + 4], v[8 * q + 5]), pack_bf16(v[8 * q + 6], v[8 * q + 7]));
            fence_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_store_2d(&p.tmD, stage_out, col, (int)(mt * BM + sub * 32));
              bulk_commit();
            }
          }
        }
      }
      tc_fence_before();
      if (wide) {
        mbar_arrive(tempty0);
        mbar_arrive(tempty0 + 8);
        acc_phase ^= 1u;
      } else {
        mbar_arrive(tempty0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
    }
    if (lane == 0) bulk_wait0();                 // this warp's output stores are complete
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // The next launch may start only now: its CTAs could otherwise sit on this
  // SM beside the GEMM while they wait for it.
  pdl_trigger();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// 2-D map over a row-major bf16 matrix [rows, K], box 64 x 128.
static bool make_map_a(CUtensorMap* m, const void* base, int64_t rows, int K) {
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

// 3-D map over stacked weights [G, N, K], box 64 x box_n x 1 (rows past N read as zero).
static bool make_map_b(CUtensorMap* m, const void* base, int G, int N, int K, int box_n) {
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
  key.box[1] = (cuuint32_t)box_n;
  key.box[2] = 1;
  return encode_cached(m, key);
}

// 5-D map over packed weights [G][N/128][K/64][128][64] (see launch_pack_weight):
// dims (64, 128, K/64, N/128, G), box 64 x 128 x 1 x 1 x 1 = one 16 KB block.
static bool make_map_b_packed(CUtensorMap* m, const void* base, int G, int N, int K, int box_rows = 128) {
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
  key.box[1] = (cuuint32_t)box_rows;
  key.box[2] = key.box[3] = key.box[4] = 1;
  return encode_cached(m, key);
}

// 2-D map over the bf16 output [rows, N], box 32 x 32, 64-byte swizzle (TMA store).
static bool make_map_d(CUtensorMap* m, const void* base, int64_t rows, int N) {
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

template <bool GATHER, bool SCATTER, int ROUTE_KM = 0>
static cudaError_t launch_variant(KParams& k, int grid, cudaStream_t stream) {
  auto kern = grouped_gemm_kernel<GATHER, SCATTER, ROUTE_KM>;
  cudaError_t e = ensure_smem(kern, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  launch_pdl(kern, grid, GATHER ? THREADS_GATHER : THREADS, SMEM_BYTES, stream, k);
  return cudaGetLastError();
}

static cudaError_t launch_kernel(KParams& k, int64_t max_tiles, cudaStream_t stream, int route_km = 0) {
  const int sms = sm_count();
  // grid: one CTA per SM, never more than the largest possible tile count
  const int grid = (int)(max_tiles < sms ? (max_tiles > 0 ? max_tiles : 1) : sms);
  if (route_km == 1) return launch_variant<false, false, 1>(k, grid, stream);
  if (route_km == 2) return launch_variant<false, false, 2>(k, grid, stream);
  if (route_km == 4) return launch_variant<false, false, 4>(k, grid, stream);
  if (route_km == 8) return launch_variant<false, false, 8>(k, grid, stream);
  if (route_km == 16) return launch_variant<false, false, 16>(k, grid, stream);
  const bool gather = k.gsrc != nullptr, scatter = k.sdst != nullptr;
  if (gather) return scatter ? launch_variant<true, true>(k, grid, stream) : launch_variant<true, false>(k, grid, stream);
  return scatter ? launch_variant<false, true>(k, grid, stream) : launch_variant<false, false>(k, grid, stream);
}

}  // namespace gg

cudaError_t launch_grouped_gemm(const GemmParams& p, cudaStream_t stream) {
  using namespace gg;
  if (p.rows_max == 0) return cudaSuccess;
  if (p.two_sm && p.gather_src == nullptr && p.scatter_dst == nullptr && p.pair_prefix != nullptr)
    return launch_grouped_gemm_tn(p, stream);
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  const int box_n = 128;
  KParams k{};
  bool ok = make_map_a(&k.tmA, p.a_routed ? p.a_routed : p.gather_src, p.a_routed ? p.rows_max : p.T, p.K);
  ok = ok && make_map_a(&k.tmAs, p.a_shared ? p.a_shared : p.a_routed, p.a_shared ? p.T : p.rows_max, p.K);
  if (p.b_packed) {
    ok = ok && make_map_b_packed(&k.tmB0, p.b0, p.E, p.Nw, p.K);
    ok = ok && make_map_b_packed(&k.tmB1, p.b1 ? p.b1 : p.b0, p.E, p.Nw, p.K);
    ok = ok && make_map_b_packed(&k.tmSB0, p.sb0 ? p.sb0 : p.b0, 1, p.Nw, p.K);
    ok = ok && make_map_b_packed(&k.tmSB1, p.sb1 ? p.sb1 : (p.sb0 ? p.sb0 : p.b0), 1, p.Nw, p.K);
  } else {
    ok = ok && make_map_b(&k.tmB0, p.b0, p.E, p.Nw, p.K, box_n);
    ok = ok && make_map_b(&k.tmB1, p.b1 ? p.b1 : p.b0, p.E, p.Nw, p.K, box_n);
    ok = ok && make_map_b(&k.tmSB0, p.sb0 ? p.sb0 : p.b0, 1, p.Nw, p.K, box_n);
    ok = ok && make_map_b(&k.tmSB1, p.sb1 ? p.sb1 : (p.sb0 ? p.sb0 : p.b0), 1, p.Nw, p.K, box_n);
  }
  // 192-column tiles (no SwiGLU): the same weights in 64-row boxes
  const bool allow192 = p.epi != MOE_ACT_SWIGLU && p.Nw > 128;
  if (allow192) {
    if (p.b_packed) {
      ok = ok && make_map_b_packed(&k.tmB0h, p.b0, p.E, p.Nw, p.K, 64);
      ok = ok && make_map_b_packed(&k.tmSB0h, p.sb0 ? p.sb0 : p.b0, 1, p.Nw, p.K, 64);
    } else {
      ok = ok && make_map_b(&k.tmB0h, p.b0, p.E, p.Nw, p.K, 64);
      ok = ok && make_map_b(&k.tmSB0h, p.sb0 ? p.sb0 : p.b0, 1, p.Nw, p.K, 64);
    }
  }
  ok = ok && make_map_d(&k.tmD, p.d, p.rows_max, p.Nw);
  if (!ok) return cudaErrorInvalidValue;
  k.allow192 = allow192 ? 1 : 0;
  k.d = p.d;
  k.off = p.expert_offset;
  k.status = p.status;
  k.ld_d = p.Nw;
  k.rows_max = p.rows_max;
  k.rows_static = -1;
  k.rows_store = p.rows_max;
  k.as_sep = p.a_shared != nullptr;
  k.K = p.K;
  k.N_out = p.Nw;
  k.E = p.E;
  k.n_shared = p.n_shared;
  k.epi = p.epi;
  k.bn_fixed = 0;
  k.bbox = box_n;
  k.b_planes = 1;
  k.plane_k = 0;
  k.k_split = 1;
  k.out_f32 = 0;
  k.b_packed = p.b_packed;
  k.planes_per_stage = 1;
  k.gsrc = static_cast<const __nv_bfloat16*>(p.gather_src);
  k.gidx = p.gather_idx;
  k.sdst = static_cast<__nv_bfloat16*>(p.scatter_dst);
  k.sgate = p.scatter_gate;
  k.sslot = p.scatter_slot;
  k.sT = p.T;
  return launch_kernel(k, (p.rows_max / BM) * ((p.Nw + box_n - 1) / box_n), stream);
}

// ---------------------------------------------------------------- router logits on tensor cores
// Wg (fp32) is split into three bf16 planes hi + mid + lo (each the bf16
// rounding of what the previous planes leave), laid side by side along K with
// each plane padded to Hp = H rounded up to 64.  x is bf16, so every product
// x_h * plane_j(w) is exact in fp32 and the tensor core's fp32 accumulation
// gives fp32 logits of the same quality as an fp32 dot product.
__global__ void split_router_weight_kernel(const float* wg, __nv_bfloat16* planes, int E, int H, int Hp) {
  pdl_wait();
  pdl_trigger();
  const int64_t n = (int64_t)E * Hp;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const int e = (int)(i / Hp), h = (int)(i % Hp);
    const float w = h < H ? wg[(int64_t)e * H + h] : 0.0f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(w);
    const float r1 = w - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(mid);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r2);
    __nv_bfloat16* row = planes + (int64_t)e * 3 * Hp;
    row[h] = hi;
    row[Hp + h] = mid;
    row[2 * Hp + h] = lo;
  }
}

int router_plane_width(int H) { return (H + gg::BK - 1) / gg::BK * gg::BK; }

cudaError_t launch_split_router_weight(const float* wg, void* planes, int E, int H, cudaStream_t stream) {
  const int Hp = router_plane_width(H);
  const int64_t n = (int64_t)E * Hp;
  const int64_t blocks = (n + 255) / 256;
  launch_pdl(split_router_weight_kernel, (unsigned)(blocks < 2048 ? blocks : 2048), 256, 0, stream, wg,
             static_cast<__nv_bfloat16*>(planes), E, H, Hp);
  return cudaGetLastError();
}

cudaError_t launch_router_gemm(const void* x, const float* wg, void* planes, bool planes_ready, float* logits,
                               int64_t T, int H, int E, DevStatus* status, const RouterParams* route, int64_t nblk,
                               int* parts, bool* routed, cudaStream_t stream) {
  using namespace gg;
  *routed = false;
  if (T == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  const int Hp = router_plane_width(H);
  if (!planes_ready) {
    cudaError_t e = launch_split_router_weight(wg, planes, E, H, stream);
    if (e != cudaSuccess) return e;
  }
  // Routing fused into the epilogue needs a token's E logits in one tile
  // (N <= 256).  A stage holds the A chunk and the matching chunk of all three
  // planes while that leaves three stages (N <= 128); wider tiles take one
  // plane per stage.
  const bool fuse = route != nullptr && E <= 256;
  if (fuse && router_pair_fits(T, H, E)) {
    *routed = true;
    *parts = 1;
    return launch_router_pair(x, planes, T, H, E, status, *route, nblk, stream);
  }
  const int bn = fuse ? (E + 15) / 16 * 16 : (E >= 128 ? 128 : (E + 15) / 16 * 16);
  const int bbox = bn;
  KParams k{};
  bool ok = make_map_a(&k.tmA, x, T, H);
  ok = ok && make_map_b(&k.tmB0, planes, 1, E, 3 * Hp, bbox);
  if (!ok) return cudaErrorInvalidValue;
  k.tmAs = k.tmA;
  k.tmB1 = k.tmSB0 = k.tmSB1 = k.tmB0;
  k.tmD = k.tmA;                                   // unused: fp32 output is stored directly
  k.d = logits;
  k.off = nullptr;
  k.status = status;
  k.ld_d = E;
  k.rows_max = T;
  k.rows_static = T;
  k.rows_store = T;
  k.K = Hp;
  k.N_out = E;
  k.E = 1;
  k.n_shared = 0;
  k.epi = -1;
  k.as_sep = 0;
  k.bn_fixed = bn;
  k.bbox = bbox;
  k.b_planes = 3;
  k.plane_k = Hp;
  k.planes_per_stage = 3 * (A_BYTES + 3 * bn * BK * 2) <= RING_BYTES ? 3 : 1;
  k.out_f32 = 1;
  // One tile per (m-block, n-tile); each k step multiplies the A chunk by the
  // hi, mid and lo planes in that order, into one fp32 accumulator.  Unfused,
  // when the tiles cannot fill half the SMs, each tile's k blocks are split in
  // two and the partial logits are added by the routing kernel.
  const int64_t tiles = ((T + BM - 1) / BM) * ((E + bn - 1) / bn);
  const int nk = Hp / BK;
  k.k_split = (!fuse && tiles * 2 <= sm_count() && nk >= 4) ? 2 : 1;
  *parts = k.k_split;
  int km = 0;
  if (fuse) {
    k.rp = *route;
    k.nblk = nblk;
    km = route_km_of(route->k);
    *routed = true;
  }
  return launch_kernel(k, tiles * k.k_split, stream, km);
}

}  // namespace moe
