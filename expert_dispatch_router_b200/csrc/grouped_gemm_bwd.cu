// Grouped GEMMs of the expert FFN's backward pass on the sm_100a tensor cores.
//
// Method: the backward of "Expert-parallel MoE training"'s grouped expert MLPs
// (the two permutations swap roles; every expert's rows are a 128-padded block
// of the row layout).  For one expert with rows X, pre-activations z = X W1^T,
// h = act(z), Y = h W2^T and output gradient dY (already gate-weighted):
//   DGRAD  dh = dY W2,  dX = dz W1 (+ dz_up W3)   A = rows (K-major), B = weights
//                                                  read along N (MN-major)
//   DACT   dz = dh * act'(z) with z recomputed     A = X, B = W1 (| W3), like the
//          on the tensor cores (SwiGLU: da, db)    forward's first contraction
//   WGRAD  dW2 = dY^T h,  dW1 = dz^T X            A and B both rows read along
//          (one output matrix per expert, K =      their feature dimension
//          that expert's rows)                     (MN-major)
//   DHZ    DGRAD dh and DACT fused per tile: the   k runs twice over H: dY W2
//          tile's dh and z accumulate side by      (MN-major B), then X W1^T
//          side in TMEM, dz = bf16(dh) * act'(z)   (K-major B); dh never
//                                                  reaches HBM
// All three use the forward kernel's structure: one persistent CTA per SM, warp
// 0 issues TMA loads into a ring of stages, warp 1 issues tcgen05.mma
// (M=128, K=16, kind::f16, fp32 accumulators in TMEM, two 256-column buffers),
// warps 2-17 drain the accumulators.  MN-major operands are loaded as boxes of
// 64 features x 64 k (128-byte swizzle; 64-feature chunks 8 KB apart, 8-row k
// groups 1 KB apart) and described to the MMA with the MN-major bit.
// Every mbarrier wait is bounded.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace moe {
namespace gb {

using namespace tcx;

constexpr int BM = 128, BK = 64, BNMAX = 256;
constexpr int A_BYTES = BM * BK * 2;                        // 16 KB
constexpr int RING_BYTES = 4 * (A_BYTES + BNMAX * BK * 2);  // 192 KB
constexpr int MAX_STAGES = 8;
constexpr int EPI_WARPS = 16;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int STAGE_OUT_BYTES = 32 * 32 * 2;
constexpr int STAGING_BYTES = EPI_WARPS * STAGE_OUT_BYTES;
constexpr int SMEM_BYTES = RING_BYTES + STAGING_BYTES + 1024 + 256;
// WGRAD: the k loop of a tile is one expert's rows (a few blocks), and the fp32
// output dominates, so the ring shrinks to two stages and each epilogue warp
// gets two 4 KB buffers (32 rows x 32 fp32, 128-byte swizzle) for TMA stores.
constexpr int WG_OUT_BYTES = 32 * 32 * 4;
constexpr int WG_STAGING_BYTES = EPI_WARPS * 2 * WG_OUT_BYTES;   // 128 KB
constexpr int WG_RING_BYTES = RING_BYTES + STAGING_BYTES - WG_STAGING_BYTES;
static_assert(WG_RING_BYTES >= 2 * (A_BYTES + BNMAX * BK * 2), "WGRAD ring holds two stages");
constexpr int MN_CHUNK_BYTES = 64 * BK * 2;                 // one 64-feature x 64-k box: 8 KB

enum Mode { DGRAD = 0, DACT = 1, WGRAD = 2, DHZ = 3 };

struct BParams {
  CUtensorMap tmA, tmAs;          // A (and the shared block's A when as_sep)
  CUtensorMap tmB0, tmB1;         // routed B (DGRAD: map 1 after k_switch k blocks; DACT: SwiGLU up)
  CUtensorMap tmSB0, tmSB1;       // shared expert's B (or, WGRAD with b_sep: the shared rows' B)
  CUtensorMap tmD;                // bf16 output, box 32 x 32, 64-byte swizzle
  const int32_t* off;             // [E+2]
  DevStatus* status;
  int mode, E, n_shared, act;
  int64_t rows_max;
  int K, N;                       // contraction length (DGRAD, DACT), output columns
  int M;                          // WGRAD: output rows per expert
  int k_switch;                   // DGRAD: k blocks read from tmB0 before tmB1 (0: never)
  int as_sep, b_sep;              // shared block's A (DACT) / B (WGRAD) from a separate map, rows - off[E]
  const __nv_bfloat16* dh;        // DACT: [rows_max, N] upstream gradient of h
  int dz_ld;                      // DACT: row length of dz (N, or 2N for SwiGLU: da | db)
  CUtensorMap tmW, tmW2;          // WGRAD: fp32 outputs [E, m_valid, N] (rows >= m_split: tmW2), box 32 x 32 x 1
  CUtensorMap tmWs, tmWs2;        // WGRAD: the shared expert's, [1, m_valid, N]
  int m_split;                    // WGRAD: output rows >= m_split go to tmW2 / tmWs2 (a multiple of 64)
  int m_valid;                    // WGRAD: rows of each output part (rows beyond are padding, not stored)
  int b_packed;                   // DGRAD / DACT / DHZ: weight maps are 5-D over packed 128 x 64 blocks
  int wg_deep;                    // WGRAD: the deep variant (maps' box 16 x 32 x 1, 64-byte swizzle)
  CUtensorMap tmA2;               // DHZ: dyrow rows (K-major A of the dh pass)
  CUtensorMap tmV, tmSV;          // DHZ: W2 (routed, shared) read along F (MN-major B of the dh pass)
};

// MN-major operand descriptor (128-byte swizzle): 64-feature chunks `lbo`
// bytes apart, 8-row k groups 1 KB apart.
__device__ __forceinline__ uint64_t mn_desc(uint32_t saddr, uint32_t lbo) { return sw128_mn_desc(saddr, lbo); }


// MODE and V are template parameters so that each variant's epilogue gets its
// own register allocation.  V: SwiGLU for DACT and DHZ; for WGRAD the deep
// variant (the four-stage ring of the other modes, fp32 stored through one
// 2 KB buffer per warp as 32 x 16 blocks), for layers whose experts have
// many rows, where the k loop is long and the output a small part of the work.
template <int MODE, bool V>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_bwd_kernel(const __grid_constant__ BParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  constexpr bool wgrad = MODE == WGRAD;
  constexpr bool wdeep = wgrad && V;
  constexpr bool wshallow = wgrad && !V;
  uint8_t* stage_base = smem;
  uint8_t* staging = smem + (wshallow ? WG_RING_BYTES : RING_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES + STAGING_BYTES);
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + MAX_STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * MAX_STAGES), tempty0 = smem_u32(bars + 2 * MAX_STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * MAX_STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * MAX_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr bool dhz = MODE == DHZ;
  constexpr bool swiglu = (MODE == DACT || dhz) && V;
  constexpr int a_mn = wgrad ? 1 : 0, b_mn = MODE == DACT ? 0 : 1;
  const int ngroups = p.E + (p.n_shared ? 1 : 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull0 + 8 * b, 1); mbar_init(tempty0 + 8 * b, EPI_WARPS * 32); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
  pdl_wait();

  // Tiles.  DGRAD / DACT: (128-row block of the row layout, N tile), the block's
  // group by binary search.  WGRAD: (group, 128-row tile of M, N tile), the k
  // blocks being the group's rows.
  // output columns per tile; DHZ holds dh (n_step columns) and z (n_step, or
  // gate | up for SwiGLU) in one 256-column accumulator buffer
  constexpr int n_step = dhz ? (swiglu ? 64 : 128) : (swiglu ? BNMAX / 2 : BNMAX);
  const int bn = BNMAX;                                    // MMA N
  const int n_tiles_n = (p.N + n_step - 1) / n_step;
  const int64_t rows_used = min((int64_t)p.off[ngroups], p.rows_max);
  const int m_tiles = wgrad ? (p.M + BM - 1) / BM : 0;
  const int64_t n_tiles = wgrad ? (int64_t)ngroups * m_tiles * n_tiles_n : ((rows_used + BM - 1) / BM) * n_tiles_n;
  const int nk = (p.K + BK - 1) / BK;
  struct Tile {
    int g, nt, kb0, kb1;
    int64_t row0;                                          // DGRAD / DACT: first row; WGRAD: first output row m0
  };
  auto decode = [&](int64_t tile) -> Tile {
    Tile d;
    if (wgrad) {
      d.nt = (int)(tile % n_tiles_n);
      const int64_t rest = tile / n_tiles_n;
      d.row0 = (rest % m_tiles) * BM;
      d.g = (int)(rest / m_tiles);
      d.kb0 = p.off[d.g] / BK;
      d.kb1 = p.off[d.g + 1] / BK;
    } else {
      d.nt = (int)(tile % n_tiles_n);
      d.row0 = (tile / n_tiles_n) * BM;
      d.g = find_group(p.off, ngroups, d.row0);
      d.kb0 = 0;
      d.kb1 = dhz ? 2 * nk : nk;                           // DHZ: the dh pass, then the z pass
    }
    return d;
  };
  const int b_bytes = dhz ? 128 * BK * 2 : bn * BK * 2;    // 16 KB (DHZ) or 32 KB
  const int stage_bytes = A_BYTES + b_bytes;
  const int n_stages = min(MAX_STAGES, (wshallow ? WG_RING_BYTES : RING_BYTES) / stage_bytes);

  if (warp == 0) {
    // ---------------- TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[MAX_STAGES] = {0, 0, 0, 0, 0, 0, 0, 0};
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const Tile d = decode(tile);
        const bool sh = d.g == p.E;
        const int n0 = d.nt * n_step;
        for (int kb = d.kb0; kb < d.kb1; ++kb) {
          if (!mbar_wait(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = full0 + 8 * stage;
          if constexpr (!dhz) mbar_expect_tx(fb, stage_bytes);
          if constexpr (dhz) {
            const bool zp = kb >= nk;                      // z pass
            const int kk = (zp ? kb - nk : kb) * BK;
            const int z = sh ? 0 : d.g;
            if (!zp) {
              mbar_expect_tx(fb, A_BYTES + n_step * BK * 2);
              tma_load_2d(sa, &p.tmA2, kk, (int)d.row0, fb);
              const CUtensorMap* mv = sh ? &p.tmSV : &p.tmV;
              for (int j = 0; j < n_step / 64; ++j) {
                if (p.b_packed)
                  tma_load_5d_at(sb + j * MN_CHUNK_BYTES, mv, kk & 127, (n0 >> 6) + j, kk >> 7, z, fb);
                else
                  tma_load_3d(sb + j * MN_CHUNK_BYTES, mv, n0 + 64 * j, kk, z, fb);
              }
            } else {
              const bool sep = sh && p.as_sep;
              mbar_expect_tx(fb, A_BYTES + (swiglu ? 2 : 1) * n_step * BK * 2);
              tma_load_2d(sa, sep ? &p.tmAs : &p.tmA, kk, (int)(sep ? d.row0 - p.off[p.E] : d.row0), fb);
              const CUtensorMap* m0 = sh ? &p.tmSB0 : &p.tmB0;
              const CUtensorMap* m1 = sh ? &p.tmSB1 : &p.tmB1;
              // W1 rows n0..n0+n_step (then W3's): one box each, n_step x 64 k
              if (p.b_packed) {
                tma_load_5d_at(sb, m0, n0 & 127, kb - nk, n0 >> 7, z, fb);
                if (swiglu) tma_load_5d_at(sb + n_step * BK * 2, m1, n0 & 127, kb - nk, n0 >> 7, z, fb);
              } else {
                tma_load_3d(sb, m0, kk, n0, z, fb);
                if (swiglu) tma_load_3d(sb + n_step * BK * 2, m1, kk, n0, z, fb);
              }
            }
          } else if constexpr (MODE == WGRAD) {
            // A: rows kb*64.. of the M-wide source, two 64-feature chunks
            for (int i = 0; i < 2; ++i) tma_load_2d(sa + i * MN_CHUNK_BYTES, &p.tmA, (int)d.row0 + 64 * i, kb * BK, fb);
            const bool bs = sh && p.b_sep;
            const int krow = bs ? kb * BK - p.off[p.E] : kb * BK;
            for (int j = 0; j < bn / 64; ++j)
              tma_load_2d(sb + j * MN_CHUNK_BYTES, bs ? &p.tmSB0 : &p.tmB0, n0 + 64 * j, krow, fb);
          } else {
            const bool sep = sh && p.as_sep;
            const int arow = (int)(sep ? d.row0 - p.off[p.E] : d.row0);
            tma_load_2d(sa, sep ? &p.tmAs : &p.tmA, kb * BK, arow, fb);
            const int z = sh ? 0 : d.g;
            if constexpr (MODE == DGRAD) {
              const bool second = p.k_switch > 0 && kb >= p.k_switch;
              const CUtensorMap* mb = sh ? (second ? &p.tmSB1 : &p.tmSB0) : (second ? &p.tmB1 : &p.tmB0);
              const int kk = (second ? kb - p.k_switch : kb) * BK;
              // packed: the weight's rows are this contraction's k, its columns
              // the output features; a 64 x 64 box is 8 KB of one block
              for (int j = 0; j < bn / 64; ++j) {
                if (p.b_packed)
                  tma_load_5d_at(sb + j * MN_CHUNK_BYTES, mb, kk & 127, (n0 >> 6) + j, kk >> 7, z, fb);
                else
                  tma_load_3d(sb + j * MN_CHUNK_BYTES, mb, n0 + 64 * j, kk, z, fb);
              }
            } else if (p.b_packed) {
              const CUtensorMap* m0 = sh ? &p.tmSB0 : &p.tmB0;
              if (swiglu) {
                tma_load_5d(sb, m0, kb, n0 >> 7, z, fb);                                         // gate rows
                tma_load_5d(sb + b_bytes / 2, sh ? &p.tmSB1 : &p.tmB1, kb, n0 >> 7, z, fb);     // up rows
              } else {
                for (int b = 0; b < 2; ++b) tma_load_5d(sb + b * (b_bytes / 2), m0, kb, (n0 >> 7) + b, z, fb);
              }
            } else if (swiglu) {
              tma_load_3d(sb, sh ? &p.tmSB0 : &p.tmB0, kb * BK, n0, z, fb);                // gate rows
              tma_load_3d(sb + b_bytes / 2, sh ? &p.tmSB1 : &p.tmB1, kb * BK, n0, z, fb);  // up rows
            } else {
              for (int b = 0; b < 2; ++b) tma_load_3d(sb + b * (b_bytes / 2), sh ? &p.tmSB0 : &p.tmB0, kb * BK, n0 + 128 * b, z, fb);
            }
          }
          fills[stage]++;
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ETIMEOUT, 20);
      }
      for (int s = 0; s < n_stages; ++s)
        if (fills[s]) {
          const long long t0 = clock64();
          while (!mbar_try_wait(full0 + 8 * s, (fills[s] - 1) & 1u) && clock64() - t0 < kWaitCycles) {}
        }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc(bn, BM, a_mn, b_mn);
      // DHZ: the dh pass (N = n_step, MN-major B) into columns [0, n_step), the
      // z pass (N = n_step, or gate | up = 2 n_step, K-major B) after them
      const uint32_t idesc_dh = make_idesc(n_step, BM, 0, 1);
      const uint32_t idesc_z = make_idesc(swiglu ? 2 * n_step : n_step, BM, 0, 0);
      for (int64_t tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x) {
        const Tile d = decode(tile);
        if (!mbar_wait(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BNMAX);
        for (int kb = d.kb0; kb < d.kb1; ++kb) {
          if (!mbar_wait(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          if constexpr (dhz) {
            const bool zp = kb >= nk;
            const uint64_t ad = sw128_desc(sa);
            const uint64_t bd = zp ? sw128_desc(sb) : mn_desc(sb, MN_CHUNK_BYTES);
            const uint64_t bstep = zp ? 2 : 128;
            const uint32_t dt = d_tmem + (zp ? (uint32_t)n_step : 0u);
            const uint32_t id = zp ? idesc_z : idesc_dh;
            const int kfirst = zp ? nk : 0;
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma(dt, ad + 2 * kk, bd + bstep * kk, id, ((kb - kfirst) | kk) != 0 ? 1u : 0u);
          } else {
            const uint64_t ad = a_mn ? mn_desc(sa, MN_CHUNK_BYTES) : sw128_desc(sa);
            const uint64_t bd = b_mn ? mn_desc(sb, MN_CHUNK_BYTES) : sw128_desc(sb);
            const uint64_t astep = a_mn ? 128 : 2, bstep = b_mn ? 128 : 2;   // 16 k: 2 KB (MN-major) or 32 B
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma(d_tmem, ad + astep * kk, bd + bstep * kk, idesc, ((kb - d.kb0) | kk) != 0 ? 1u : 0u);
          }
          umma_commit(empty0 + 8 * stage);
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(tfull0 + 8 * acc);         // also when the group had no rows: nothing to wait for
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) {
        *abort_flag = 1;
        set_status(p.status, MOE_ETIMEOUT, 21);
      }
      umma_commit(drain);
      const long long t0 = clock64();
      while (!mbar_try_wait(drain, 0) && clock64() - t0 < kWaitCycles) {}
    }
  } else {
    // ---------------- epilogue
    const int ew = warp - 2;
    const int sub = warp & 3;
    const int quarter = ew >> 2;
    const int row_in_tile = sub * 32 + lane;
    const uint32_t stage_out = smem_u32(staging + ew * (wshallow ? 2 * WG_OUT_BYTES : STAGE_OUT_BYTES));
    int wbuf = 0;                                    // WGRAD: staging buffer of the next store
    int acc = 0;
    uint32_t acc_phase = 0;
    // bf16 store of this warp's 32 x 32 sub-tile through its staging buffer
    auto store_bf16 = [&](const float (&v)[32], int col, int64_t row_base) {
      if (lane == 0) bulk_wait_read0();
      __syncwarp();
#pragma unroll
      for (int q = 0; q < 4; ++q)
        st_shared_v4(stage_out + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4), pack_bf16(v[8 * q], v[8 * q + 1]),
                     pack_bf16(v[8 * q + 2], v[8 * q + 3]), pack_bf16(v[8 * q + 4], v[8 * q + 5]),
                     pack_bf16(v[8 * q + 6], v[8 * q + 7]));
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&p.tmD, stage_out, col, (int)row_base);
        bulk_commit();
      }
    };
    for (int64_t tile = blockIdx.x; tile < n_tiles; tile += gridDim.x) {
      const Tile d = decode(tile);
      const int ncol0 = d.nt * n_step;
      // DACT: this thread's dh (its row, 32 columns of each of its chunks) is
      // loaded before the accumulator is ready, so the loads overlap the MMA
      int4 dhv[2][4];
      if constexpr (MODE == DACT) {
        const int64_t grow = d.row0 + row_in_tile;
#pragma unroll
        for (int ci = 0; ci < 2; ++ci) {
          const int col = ncol0 + quarter * 32 + ci * 128;
          const __nv_bfloat16* src = p.dh + grow * (int64_t)p.N + col;
#pragma unroll
          for (int q = 0; q < 4; ++q)     // columns past N read as zero, so dz is zero there
            dhv[ci][q] = quarter * 32 + ci * 128 < n_step && grow < p.rows_max && col + 8 * q < p.N
                             ? ld_nc_v4(src + 8 * q) : make_int4(0, 0, 0, 0);
        }
      }
      if (!mbar_wait(tfull0 + 8 * acc, acc_phase, abort_flag)) {
        *abort_flag = 1;
        set_status(p.status, MOE_ETIMEOUT, 22);
        break;
      }
      tc_fence_after();
      const bool empty = d.kb1 <= d.kb0;
      const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * BNMAX);
      for (int c = quarter * 32; c < n_step; c += 4 * 32) {
        const int col = ncol0 + c;
        if (col >= p.N) break;
        __syncwarp();                                // converged for the warp-wide tcgen05.ld
        float v[32];
        if (empty) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.0f;
        } else {
          tmem_ld(tbase + (uint32_t)c, v, 32);
        }
        if constexpr (MODE == WGRAD) {
          tmem_wait_ld();
          // this warp's 32 output rows lie on one side of m_split (a multiple
          // of 64); rows past m_valid and columns past N are clipped by the map
          const int m0 = (int)d.row0 + sub * 32;
          if (m0 >= p.M) continue;
          const bool hi = m0 >= p.m_split;
          const bool sh = d.g == p.E;
          const CUtensorMap* mw = sh ? (hi ? &p.tmWs2 : &p.tmWs) : (hi ? &p.tmW2 : &p.tmW);
          if constexpr (wdeep) {
            // two 32 x 16 fp32 blocks (64-byte rows, 64-byte swizzle) through the
            // warp's one 2 KB buffer
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (lane == 0) bulk_wait_read0();
              __syncwarp();
#pragma unroll
              for (int q = 0; q < 4; ++q)
                st_shared_v4(stage_out + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4),
                             __float_as_uint(v[16 * h + 4 * q]), __float_as_uint(v[16 * h + 4 * q + 1]),
                             __float_as_uint(v[16 * h + 4 * q + 2]), __float_as_uint(v[16 * h + 4 * q + 3]));
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(mw, stage_out, col + 16 * h, hi ? m0 - p.m_split : m0, sh ? 0 : d.g);
                bulk_commit();
              }
            }
            continue;
          }
          const uint32_t buf = stage_out + wbuf * WG_OUT_BYTES;
          if (lane == 0) bulk_wait_read1();          // the store that last read `buf` is done with it
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 8; ++q)
            st_shared_v4(buf + lane * 128 + ((q ^ (lane & 7)) << 4), __float_as_uint(v[4 * q]),
                         __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(mw, buf, col, hi ? m0 - p.m_split : m0, sh ? 0 : d.g);
            bulk_commit();
          }
          wbuf ^= 1;
          continue;
        }
        const int64_t row_base = d.row0 + sub * 32;
        if constexpr (MODE == DGRAD) {
          tmem_wait_ld();
          store_bf16(v, col, row_base);
          continue;
        }
        if constexpr (dhz) {
          // v = dh; zv = z (SwiGLU: the gate pre-activation); u = the up projection.
          // dh is rounded to bf16 first, as the unfused path stores it.
          float zv[32];
          tmem_ld(tbase + (uint32_t)(n_step + c), zv, 32);
          float u[32];
          if constexpr (swiglu) tmem_ld(tbase + (uint32_t)(2 * n_step + c), u, 32);
          tmem_wait_ld();
          if constexpr (!swiglu) {
            if (p.act == MOE_ACT_GELU) {                        // GELU' two values at a time
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                float g0 = zv[i], g1 = zv[i + 1];
                gelu_grad_x2(g0, g1);
                v[i] = __bfloat162float(__float2bfloat16_rn(v[i])) * g0;
                v[i + 1] = __bfloat162float(__float2bfloat16_rn(v[i + 1])) * g1;
              }
              store_bf16(v, col, row_base);
              continue;
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float gi = __bfloat162float(__float2bfloat16_rn(v[i]));
            const float z = zv[i];
            if constexpr (swiglu) {
              const float s = rcp_approx(1.0f + __expf(-z));
              v[i] = gi * u[i] * s * (1.0f + z * (1.0f - s));    // da
              zv[i] = gi * z * s;                                 // db = dh * silu(a)
            } else {
              v[i] = p.act == MOE_ACT_RELU ? (z > 0.0f ? gi : 0.0f) : gi * gelu_grad(z);
            }
          }
          store_bf16(v, col, row_base);
          if constexpr (swiglu) store_bf16(zv, p.dz_ld / 2 + col, row_base);
          continue;
        }
        // DACT: z (and the SwiGLU up projection) recomputed; dz = dh * act'(z)
        float u[32];
        if constexpr (swiglu) tmem_ld(tbase + (uint32_t)(BNMAX / 2 + c), u, 32);
        tmem_wait_ld();
        const int ci = c >= 128 ? 1 : 0;
        if constexpr (!swiglu) {
          if (p.act == MOE_ACT_GELU) {                          // GELU' two values at a time
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int4 w = ci ? dhv[1][q] : dhv[0][q];
              const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                float g0 = v[8 * q + i], g1 = v[8 * q + i + 1];
                gelu_grad_x2(g0, g1);
                v[8 * q + i] = __bfloat162float(e[i]) * g0;
                v[8 * q + i + 1] = __bfloat162float(e[i + 1]) * g1;
              }
            }
            store_bf16(v, col, row_base);
            continue;
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int4 w = ci ? dhv[1][q] : dhv[0][q];
          const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&w);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float gi = __bfloat162float(e[i]);
            const float z = v[8 * q + i];
            if constexpr (swiglu) {
              const float s = rcp_approx(1.0f + __expf(-z));
              v[8 * q + i] = gi * u[8 * q + i] * s * (1.0f + z * (1.0f - s));   // da
              u[8 * q + i] = gi * z * s;                                        // db = dh * silu(a)
            } else {
              v[8 * q + i] = p.act == MOE_ACT_RELU ? (z > 0.0f ? gi : 0.0f) : gi * gelu_grad(z);
            }
          }
        }
        store_bf16(v, col, row_base);
        if constexpr (swiglu) store_bf16(u, p.dz_ld / 2 + col, row_base);             // db at column Fp + col
      }
      tc_fence_before();
      mbar_arrive(tempty0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_trigger();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// ---------------------------------------------------------------- host side
// [rows, W] bf16 read along W: box 64 x 64 (MN-major operand)
static bool make_map_mn_rows(CUtensorMap* m, const void* base, int64_t rows, int W) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 2;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)W;
  key.dims[1] = (cuuint64_t)rows;
  key.strides[0] = (cuuint64_t)W * 2;
  key.box[0] = 64;
  key.box[1] = 64;
  return encode_cached(m, key);
}
// weights [G, K, N] bf16 read along N: box 64 x 64 x 1 (MN-major operand)
static bool make_map_mn_weights(CUtensorMap* m, const void* base, int G, int K, int N) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 3;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)N;
  key.dims[1] = (cuuint64_t)K;
  key.dims[2] = (cuuint64_t)G;
  key.strides[0] = (cuuint64_t)N * 2;
  key.strides[1] = (cuuint64_t)K * N * 2;
  key.box[0] = 64;
  key.box[1] = 64;
  key.box[2] = 1;
  return encode_cached(m, key);
}
// packed weights (the layout of moe_pack_weight: [G][N/128][K/64][128][64] for a
// [G, N, K] matrix) as 5-D (64 k, 128 n, K/64, N/128, G).  Box 64 x 128 (one
// block) or, with `half`, 64 x 64 (half a block: an MN-major box, whose block k
// are the output features, or a 64-row K-major box).
static bool make_map_packed(CUtensorMap* m, const void* base, int G, int N, int K, bool half) {
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
  key.box[1] = half ? 64 : 128;
  key.box[2] = key.box[3] = key.box[4] = 1;
  return encode_cached(m, key);
}
// [rows, K] bf16 read along K: box 64 x 128 (K-major A)
static bool make_map_k_rows(CUtensorMap* m, const void* base, int64_t rows, int K) {
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
// weights [G, N, K] bf16 read along K: box 64 x box_n x 1 (K-major B)
static bool make_map_k_weights(CUtensorMap* m, const void* base, int G, int N, int K, int box_n = 128) {
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
  key.box[1] = box_n;
  key.box[2] = 1;
  return encode_cached(m, key);
}
// fp32 weight gradients [G, rows, W], box 32 x 32 x 1 with 128-byte swizzle, or
// (deep) 16 x 32 x 1 with 64-byte swizzle (TMA store)
static bool make_map_wout(CUtensorMap* m, const float* base, int G, int rows, int W, bool deep) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 3;
  key.f32 = 1;
  key.swizzle = deep ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)W;
  key.dims[1] = (cuuint64_t)rows;
  key.dims[2] = (cuuint64_t)G;
  key.strides[0] = (cuuint64_t)W * 4;
  key.strides[1] = (cuuint64_t)rows * W * 4;
  key.box[0] = deep ? 16 : 32;
  key.box[1] = 32;
  key.box[2] = 1;
  return encode_cached(m, key);
}
// bf16 output [rows, W], box 32 x 32, 64-byte swizzle (TMA store)
static bool make_map_out(CUtensorMap* m, const void* base, int64_t rows, int W) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 2;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_64B;
  key.dims[0] = (cuuint64_t)W;
  key.dims[1] = (cuuint64_t)rows;
  key.strides[0] = (cuuint64_t)W * 2;
  key.box[0] = 32;
  key.box[1] = 32;
  return encode_cached(m, key);
}

template <int MODE, bool SWI>
static cudaError_t launch_variant(BParams& k, int grid, cudaStream_t stream) {
  cudaError_t e = ensure_smem(grouped_gemm_bwd_kernel<MODE, SWI>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  launch_pdl(grouped_gemm_bwd_kernel<MODE, SWI>, grid, THREADS, SMEM_BYTES, stream, k);
  return cudaGetLastError();
}

static cudaError_t launch(BParams& k, int64_t max_tiles, cudaStream_t stream) {
  const int sms = sm_count();
  const int grid = (int)(max_tiles < sms ? (max_tiles > 0 ? max_tiles : 1) : sms);
  if (k.mode == DGRAD) return launch_variant<DGRAD, false>(k, grid, stream);
  if (k.mode == WGRAD)
    return k.wg_deep ? launch_variant<WGRAD, true>(k, grid, stream) : launch_variant<WGRAD, false>(k, grid, stream);
  if (k.mode == DHZ)
    return k.act == MOE_ACT_SWIGLU ? launch_variant<DHZ, true>(k, grid, stream)
                                   : launch_variant<DHZ, false>(k, grid, stream);
  return k.act == MOE_ACT_SWIGLU ? launch_variant<DACT, true>(k, grid, stream)
                                 : launch_variant<DACT, false>(k, grid, stream);
}

}  // namespace gb

cudaError_t launch_bwd_dgrad(const BwdGemm& q, cudaStream_t stream) {
  using namespace gb;
  if (q.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  BParams k{};
  const int G = q.E;
  bool ok = make_map_k_rows(&k.tmA, q.a, q.rows_max, q.K);
  k.tmAs = k.tmA;
  // map 0 covers the first q.K0 k of B (rows beyond read as zero); with
  // k_switch, A's k blocks from k_switch on use map 1 (also q.K0 deep)
  const void* b1 = q.b1 ? q.b1 : q.b0;
  const void* s0 = q.sb0 ? q.sb0 : q.b0;
  const void* s1 = q.sb1 ? q.sb1 : s0;
  if (q.b_packed) {                                 // packed [G, K0, N]: rows K0, columns N
    ok = ok && make_map_packed(&k.tmB0, q.b0, G, q.K0, q.N, true);
    ok = ok && make_map_packed(&k.tmB1, b1, G, q.K0, q.N, true);
    ok = ok && make_map_packed(&k.tmSB0, s0, 1, q.K0, q.N, true);
    ok = ok && make_map_packed(&k.tmSB1, s1, 1, q.K0, q.N, true);
  } else {
    ok = ok && make_map_mn_weights(&k.tmB0, q.b0, G, q.K0, q.N);
    ok = ok && make_map_mn_weights(&k.tmB1, b1, G, q.K0, q.N);
    ok = ok && make_map_mn_weights(&k.tmSB0, s0, 1, q.K0, q.N);
    ok = ok && make_map_mn_weights(&k.tmSB1, s1, 1, q.K0, q.N);
  }
  k.b_packed = q.b_packed;
  ok = ok && make_map_out(&k.tmD, q.out, q.rows_max, q.N);
  if (!ok) return cudaErrorInvalidValue;
  k.off = q.off;
  k.status = q.status;
  k.mode = DGRAD;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.rows_max = q.rows_max;
  k.K = q.K;
  k.N = q.N;
  k.k_switch = q.k_switch;
  return launch(k, (q.rows_max / BM) * ((q.N + BNMAX - 1) / BNMAX), stream);
}

cudaError_t launch_bwd_dact(const BwdGemm& q, cudaStream_t stream) {
  using namespace gb;
  if (q.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  BParams k{};
  bool ok = make_map_k_rows(&k.tmA, q.a, q.rows_max, q.K);
  ok = ok && make_map_k_rows(&k.tmAs, q.a_shared ? q.a_shared : q.a, q.a_shared ? q.T : q.rows_max, q.K);
  const void* b1 = q.b1 ? q.b1 : q.b0;
  const void* s0 = q.sb0 ? q.sb0 : q.b0;
  const void* s1 = q.sb1 ? q.sb1 : s0;
  if (q.b_packed) {
    ok = ok && make_map_packed(&k.tmB0, q.b0, q.E, q.N, q.K, false);
    ok = ok && make_map_packed(&k.tmB1, b1, q.E, q.N, q.K, false);
    ok = ok && make_map_packed(&k.tmSB0, s0, 1, q.N, q.K, false);
    ok = ok && make_map_packed(&k.tmSB1, s1, 1, q.N, q.K, false);
  } else {
    ok = ok && make_map_k_weights(&k.tmB0, q.b0, q.E, q.N, q.K);
    ok = ok && make_map_k_weights(&k.tmB1, b1, q.E, q.N, q.K);
    ok = ok && make_map_k_weights(&k.tmSB0, s0, 1, q.N, q.K);
    ok = ok && make_map_k_weights(&k.tmSB1, s1, 1, q.N, q.K);
  }
  k.b_packed = q.b_packed;
  const int ld = q.act == MOE_ACT_SWIGLU ? 2 * ((q.N + BK - 1) / BK * BK) : q.N;   // da | db, db at column Fp
  ok = ok && make_map_out(&k.tmD, q.out, q.rows_max, ld);
  if (!ok) return cudaErrorInvalidValue;
  k.off = q.off;
  k.status = q.status;
  k.mode = DACT;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.act = q.act;
  k.rows_max = q.rows_max;
  k.K = q.K;
  k.N = q.N;
  k.as_sep = q.a_shared != nullptr;
  k.dh = static_cast<const __nv_bfloat16*>(q.dh);
  k.dz_ld = ld;
  const int n_step = q.act == MOE_ACT_SWIGLU ? BNMAX / 2 : BNMAX;
  return launch(k, (q.rows_max / BM) * ((q.N + n_step - 1) / n_step), stream);
}

cudaError_t launch_bwd_dhz(const BwdGemm& q, cudaStream_t stream) {
  using namespace gb;
  if (q.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  BParams k{};
  const bool sw = q.act == MOE_ACT_SWIGLU;
  const int n_step = sw ? 64 : 128;
  const int G = q.E;
  // z pass: A = dispatched rows (shared block: x), B = W1 (| W3) rows, n_step x 64 k boxes
  bool ok = make_map_k_rows(&k.tmA, q.a, q.rows_max, q.K);
  ok = ok && make_map_k_rows(&k.tmAs, q.a_shared ? q.a_shared : q.a, q.a_shared ? q.T : q.rows_max, q.K);
  const void* b1 = q.b1 ? q.b1 : q.b0;
  const void* s0 = q.sb0 ? q.sb0 : q.b0;
  const void* s1 = q.sb1 ? q.sb1 : s0;
  // dh pass: A = dyrow, B = W2 [G, K, N] read along N
  ok = ok && make_map_k_rows(&k.tmA2, q.a2, q.rows_max, q.K);
  const void* v0 = q.v;
  const void* sv = q.sv ? q.sv : q.v;
  if (q.b_packed) {
    ok = ok && make_map_packed(&k.tmB0, q.b0, G, q.N, q.K, sw);
    ok = ok && make_map_packed(&k.tmB1, b1, G, q.N, q.K, sw);
    ok = ok && make_map_packed(&k.tmSB0, s0, 1, q.N, q.K, sw);
    ok = ok && make_map_packed(&k.tmSB1, s1, 1, q.N, q.K, sw);
    ok = ok && make_map_packed(&k.tmV, v0, G, q.K, q.N, true);
    ok = ok && make_map_packed(&k.tmSV, sv, 1, q.K, q.N, true);
  } else {
    ok = ok && make_map_k_weights(&k.tmB0, q.b0, G, q.N, q.K, n_step);
    ok = ok && make_map_k_weights(&k.tmB1, b1, G, q.N, q.K, n_step);
    ok = ok && make_map_k_weights(&k.tmSB0, s0, 1, q.N, q.K, n_step);
    ok = ok && make_map_k_weights(&k.tmSB1, s1, 1, q.N, q.K, n_step);
    ok = ok && make_map_mn_weights(&k.tmV, v0, G, q.K, q.N);
    ok = ok && make_map_mn_weights(&k.tmSV, sv, 1, q.K, q.N);
  }
  const int ld = sw ? 2 * ((q.N + BK - 1) / BK * BK) : q.N;   // da | db, db at column Fp
  ok = ok && make_map_out(&k.tmD, q.out, q.rows_max, ld);
  if (!ok) return cudaErrorInvalidValue;
  k.b_packed = q.b_packed;
  k.off = q.off;
  k.status = q.status;
  k.mode = DHZ;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.act = q.act;
  k.rows_max = q.rows_max;
  k.K = q.K;
  k.N = q.N;
  k.as_sep = q.a_shared != nullptr;
  k.dz_ld = ld;
  return launch(k, (q.rows_max / BM) * ((q.N + n_step - 1) / n_step), stream);
}

cudaError_t launch_bwd_wgrad(const BwdGemm& q, cudaStream_t stream) {
  using namespace gb;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  BParams k{};
  bool ok = make_map_mn_rows(&k.tmA, q.a, q.rows_max > 0 ? q.rows_max : 1, q.M);
  ok = ok && make_map_mn_rows(&k.tmB0, q.b0, q.rows_max > 0 ? q.rows_max : 1, q.N);
  ok = ok && make_map_mn_rows(&k.tmSB0, q.b_shared ? q.b_shared : q.b0, q.b_shared ? q.T : (q.rows_max > 0 ? q.rows_max : 1),
                              q.N);
  k.tmAs = k.tmA;
  k.tmB1 = k.tmB0;
  k.tmSB1 = k.tmSB0;
  k.tmD = k.tmA;                                    // unused: fp32 stores
  if (!ok) return cudaErrorInvalidValue;
  k.off = q.off;
  k.status = q.status;
  k.mode = WGRAD;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.rows_max = q.rows_max;
  k.K = 0;
  k.N = q.N;
  k.M = q.M;
  k.b_sep = q.b_shared != nullptr;
  k.m_split = q.m_split > 0 ? q.m_split : q.M;
  k.m_valid = q.m_valid > 0 ? q.m_valid : q.M;
  if (k.m_split < q.M && k.m_split % 64 != 0) return cudaErrorInvalidValue;
  const bool deep = q.wg_deep != 0;
  ok = make_map_wout(&k.tmW, q.w_out, q.E, k.m_valid, q.N, deep);
  ok = ok && make_map_wout(&k.tmW2, q.w_out2 ? q.w_out2 : q.w_out, q.E, k.m_valid, q.N, deep);
  ok = ok && make_map_wout(&k.tmWs, q.w_sh ? q.w_sh : q.w_out, 1, k.m_valid, q.N, deep);
  ok = ok && make_map_wout(&k.tmWs2, q.w_sh2 ? q.w_sh2 : (q.w_sh ? q.w_sh : q.w_out), 1, k.m_valid, q.N, deep);
  k.wg_deep = deep ? 1 : 0;
  if (!ok) return cudaErrorInvalidValue;
  const int64_t tiles = (int64_t)(q.E + (q.n_shared ? 1 : 0)) * ((q.M + BM - 1) / BM) * ((q.N + BNMAX - 1) / BNMAX);
  return launch(k, tiles, stream);
}

}  // namespace moe
