// Grouped GEMM with the tokens on the MMA's N side, on pairs of SMs
// (tcgen05.mma.cta_group::2), for the expert contractions of compute-bound
// layers.
//
// Method: the per-expert FFN of an MoE layer ("Expert-parallel MoE training"
// explainer: experts as grouped MLPs, SwiGLU experts with gate / up / down
// matrices in worked example 2; MegaBlocks' dropless layout with every expert
// batch padded to a multiple of 128 rows).  For every group g and its rows,
//     D[rows, features] = epi( X_g[rows, :] * W_g[features, :]^T ),
// bf16 operands, fp32 accumulation in tensor memory, bf16 output.
//
// Why tokens on N: with the rows of a group on the MMA's M side, every group
// is computed in whole 128-row blocks (256 on a pair of SMs), and a group's
// padding rows cost as much as its tokens: 23% extra work on the WideEP layer
// (skewed loads over 256 experts).  Here the MMA computes D^T = W_g * X_g^T:
// M = 256 output features (128 per SM of the pair), N = the group's next
// tokens, at most 256 and rounded up to 16, so a group costs its token count
// rounded up to 16.  The buffers keep the 128-row-padded layout; only the
// computation skips the padding.
//
// Per pair tile (group g, token tile j, feature tile f):
//   tokens r0 = off[g] + 256 j .. r0 + N, N = round_up(min(256, valid_g - 256 j), 16);
//   the even CTA computes features 256 f .. +128, the odd CTA the next 128.
// Each CTA loads its 128 weight rows (A, 16 KB per 64-k step) and half of the
// token rows (B: rows r0 + rank * N/2, a 128-row box of which the MMA reads
// N/2); one MMA instruction issued by the even CTA reads both CTAs' shared
// memory.  SwiGLU: two MMAs per k step, gate and up rows of the same features
// (A 32 KB per step), into two accumulators, so a thread holds gate and up of
// its feature; plain: double-buffered accumulators.
//
// Roles per CTA (576 threads): warp 0 issues the TMA loads (both CTAs; each
// copy completes on the even CTA's full barrier, armed by the even CTA with
// both CTAs' bytes); warp 1 of the even CTA issues the MMAs and commits with a
// multicast to both CTAs' barriers; warps 2-17 read the accumulator (lane =
// feature, columns = tokens), apply the activation, transpose 32 x 32 tiles
// through shared memory and store them by TMA.
//
// No load in this file uses cluster multicast.  Every wait is bounded: on
// expiry the CTA records MOE_ETIMEOUT, raises both CTAs' abort flags, and the
// pair drains what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "pair_common.cuh"
#include "tc_common.cuh"

namespace moe {
namespace gtn {

using namespace tcx;
using namespace pairx;

constexpr int BK = 64;
constexpr int FT = 256;                         // output features per pair tile
constexpr int TT = 256;                         // tokens per pair tile at most
constexpr int HALF = 128;                       // rows of one CTA's A (and of its B box)
constexpr int A_BYTES = HALF * BK * 2;          // 16 KB
constexpr int B_BYTES = HALF * BK * 2;          // 16 KB
constexpr int RING_BYTES = 192 * 1024;
constexpr int MAX_STAGES = 6;
constexpr int EPI_WARPS = 16;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int STAGE_OUT_BYTES = 32 * 32 * 2;
constexpr int STAGING_BYTES = EPI_WARPS * STAGE_OUT_BYTES;
constexpr int SMEM_BYTES = RING_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;

struct KParams {
  CUtensorMap tmA, tmA1, tmSA, tmSA1;   // weights [G, N_out, K] (SwiGLU: gate, up); the shared expert's
  CUtensorMap tmB, tmBs;                // token rows [rows_max, K]; the shared block's rows from x [T, K]
  CUtensorMap tmD;                      // bf16 output [rows_max, N_out], box 32 x 32, 64-byte swizzle
  const int32_t* off;                   // [ngroups + 1] row offsets (multiples of 128)
  const int32_t* tp;                    // [ngroups + 1] exclusive prefix of the groups' token tiles
  const int32_t* valid;                 // [E] rows of each routed group (kept counts), or null: whole blocks
  DevStatus* status;
  int64_t rows_max, T;
  int K, N_out, E, n_shared, epi;
  int as_sep;                           // 1: the shared block's token rows come from tmBs (row - off[E])
  int b_packed;                         // 1: weight maps are 5-D over packed blocks
  int wide;                             // 1 (no SwiGLU): 512 features per pair tile, two MMAs share each B tile
  // 1: the weights are read along their columns (MN-major A; the backward's
  // dh = dY W2 and dX = dz [W1; W3]): stored [G, K, N_out], so this CTA's 128
  // output features are two 64-column boxes of 64 k rows; k blocks >= k_switch
  // (when > 0) come from tmA1 / tmSA1 at k - 64 k_switch
  int a_mn;
  int k_switch;
  // 1: the backward's dz = dh * act'(z) from the recomputed z (the epilogue
  // reads dh [rows_max, N_out]; SwiGLU writes da at column f and db at
  // dz_half + f of the output)
  int dact;
  int dz_half;
  const __nv_bfloat16* dh;
  // weight gradients (the WGRAD instance): per expert g, out[g] = A_g^T B_g
  // (fp32 [m_valid, N_out]) with A rows [rows_max, M_out] (tmA) and B rows
  // [rows_max, N_out] (tmB; the shared block's from tmBs at row - off[E] when
  // b_sep), both read along their columns; output rows >= m_split go to
  // w_out2 / w_sh2 at m - m_split
  int M_out, m_split, m_valid, b_sep;
  float *w_out, *w_out2, *w_sh, *w_sh2;
  CUtensorMap tmW, tmW2, tmWs, tmWs2;   // those outputs [G, m_valid, N_out] fp32, box 16 x 32 x 1, 64-byte swizzle
};

// Rows of group g that carry tokens: the routed groups' kept counts, the
// shared block's T, clipped to the group's rows (<= rows_max).
__device__ __forceinline__ int64_t group_rows(const int32_t* off, const int32_t* valid, int g, int E, int64_t T,
                                              int64_t rows_max) {
  const int64_t b = min((int64_t)off[g], rows_max), e = min((int64_t)off[g + 1], rows_max);
  const int64_t pad = e > b ? e - b : 0;
  const int64_t v = g == E ? T : (valid != nullptr ? (int64_t)valid[g] : pad);
  return v < pad ? (v > 0 ? v : 0) : pad;
}

struct Tile {
  int g;           // group
  int ft;          // feature tile
  int n;           // MMA N: tokens of the tile rounded up to 16
  int64_t r0;      // first row of the tile
};
__device__ __forceinline__ Tile decode(const KParams& p, int ngroups, int nf, int64_t tile) {
  Tile t;
  const int64_t tt = tile / nf;
  t.ft = (int)(tile - tt * nf);
  int lo = 0, hi = ngroups - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (__ldg(p.tp + mid) <= tt) lo = mid; else hi = mid - 1;
  }
  t.g = lo;
  const int64_t j = tt - __ldg(p.tp + lo);
  t.r0 = min((int64_t)__ldg(p.off + lo), p.rows_max) + j * TT;
  const int64_t v = group_rows(p.off, p.valid, lo, p.E, p.T, p.rows_max) - j * TT;
  const int64_t nv = v < TT ? v : TT;
  t.n = (int)((nv + 15) / 16 * 16);
  return t;
}

// MODE 0: the forward's contractions and the backward's dh / dX (a_mn);
// MODE 1: the backward's dz epilogue (KParams::dact); MODE 2: the weight
// gradients.  Separate instances keep the forward's register allocation.
template <int MODE>
__global__ void __launch_bounds__(THREADS, 1) grouped_gemm_tn_kernel(const __grid_constant__ KParams p) {
  constexpr bool DACT = MODE == 1, WG = MODE == 2;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stage_base = smem;
  uint8_t* staging = smem + RING_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + RING_BYTES + STAGING_BYTES);
  // bars: full[MAX_STAGES], empty[MAX_STAGES], tfull[2], tempty[2], drain
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + MAX_STAGES);
  const uint32_t tfull0 = smem_u32(bars + 2 * MAX_STAGES), tempty0 = smem_u32(bars + 2 * MAX_STAGES + 2);
  const uint32_t drain = smem_u32(bars + 2 * MAX_STAGES + 4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * MAX_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const bool swiglu = p.epi == MOE_ACT_SWIGLU;
  // two accumulators per tile, fed by one B tile: gate | up (SwiGLU), or two
  // 256-feature halves of a 512-feature tile (wide); they fill all 512 columns
  const bool two = swiglu || p.wide;
  const int span = p.wide ? 2 * FT : FT;        // output features per pair tile
  const int ngroups = p.E + (p.n_shared ? 1 : 0);
  const int stage_bytes = (two ? 2 : 1) * A_BYTES + B_BYTES;
  const int n_stages = min(MAX_STAGES, RING_BYTES / stage_bytes);
  const int n_acc = two ? 1 : 2;
  auto abort_pair = [&](int info) {
    *abort_flag = 1;
    st_cluster_u32(map_to(smem_u32((const void*)abort_flag), rank ^ 1u), 1u);
    set_status(p.status, MOE_ETIMEOUT, info);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < MAX_STAGES; ++s) { mbar_init(full0 + 8 * s, 1); mbar_init(empty0 + 8 * s, 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(tfull0 + 8 * b, 1); mbar_init(tempty0 + 8 * b, 2 * EPI_WARPS); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefetch_map(&p.tmA); prefetch_map(&p.tmB); prefetch_map(&p.tmD);
    if (swiglu) prefetch_map(&p.tmA1);
    if (p.n_shared) { prefetch_map(&p.tmSA); prefetch_map(&p.tmBs); if (swiglu) prefetch_map(&p.tmSA1); }
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the pair's MMA writes both CTAs' accumulators at the even CTA's columns
  const bool tmem_same = ld_cluster_u32(map_to(smem_u32(tmem_slot), rank ^ 1u)) == tmem_base;
  pdl_wait();
  if (!tmem_same && threadIdx.x == 0) set_status(p.status, MOE_EDEVICE, 31);

  const int nf = (p.N_out + span - 1) / span;                  // feature tiles
  // WG: tiles (group, 256 output rows, 256 output columns), columns fastest
  const int wg_nm = WG ? (p.M_out + 2 * HALF - 1) / (2 * HALF) : 0, wg_nn = WG ? (p.N_out + 2 * HALF - 1) / (2 * HALF) : 0;
  const int64_t n_tok_tiles = tmem_same && !WG ? __ldg(p.tp + ngroups) : 0;
  const int64_t n_tiles = WG ? (tmem_same ? (int64_t)ngroups * wg_nm * wg_nn : 0) : n_tok_tiles * nf;
  // WG: a tile's group, output row and column blocks, and 64-row k blocks
  auto wg_tile = [&](int64_t tile, int& g, int& mt, int& nt, int& nkb, int64_t& r0) {
    const int64_t per = (int64_t)wg_nm * wg_nn;
    g = (int)(tile / per);
    const int rest = (int)(tile - (int64_t)g * per);
    mt = rest / wg_nn;
    nt = rest - mt * wg_nn;
    r0 = min((int64_t)__ldg(p.off + g), p.rows_max);
    nkb = (int)((group_rows(p.off, p.valid, g, p.E, p.T, p.rows_max) + BK - 1) / BK);
  };
  const int nk = (p.K + BK - 1) / BK;
  const int64_t cid = cluster_id(), ncl = cluster_count();

  if (WG && warp == 0) {
    // ---------------- TMA producer, weight gradients (both CTAs): per 64-row
    // k block, this CTA's 128 A columns and 128 B columns as 64 x 64 boxes
    if (lane == 0) {
      const uint32_t full_leader0 = map_to(full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[MAX_STAGES] = {0, 0, 0, 0, 0, 0};
      bool ok = true;
      const uint32_t tx = 2u * (uint32_t)stage_bytes;
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        int g, mt, nt, nkb;
        int64_t r0;
        wg_tile(tile, g, mt, nt, nkb, r0);
        const bool bsep = g == p.E && p.b_sep;
        const CUtensorMap* mb = bsep ? &p.tmBs : &p.tmB;
        const int64_t rb0 = bsep ? r0 - __ldg(p.off + p.E) : r0;
        const int m0 = mt * 2 * HALF + (int)rank * HALF, n0 = nt * 2 * HALF + (int)rank * HALF;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_cl(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = full_leader0 + 8 * stage;
          if (leader) mbar_expect_tx(full0 + 8 * stage, tx);
          const int ra = (int)(r0 + kb * BK), rb = (int)(rb0 + kb * BK);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            tma2_load_2d(sa + (uint32_t)(j * 8192), &p.tmA, m0 + 64 * j, ra, fb);
            tma2_load_2d(sb + (uint32_t)(j * 8192), mb, n0 + 64 * j, rb, fb);
          }
          fills[stage]++;
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) abort_pair(43);
      for (int s = 0; s < n_stages; ++s)
        if (fills[s]) {
          if (leader) mbar_drain_cl(full0 + 8 * s, (fills[s] - 1) & 1u);
          else mbar_drain_cl(empty0 + 8 * s, (fills[s] - 1) & 1u);
        }
    }
  } else if (WG && warp == 1) {
    // ---------------- MMA issuer, weight gradients (even CTA): both operands
    // MN-major; a group with no rows commits an untouched accumulator, which
    // the epilogue replaces by zeros
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      const uint32_t idesc = make_idesc(2 * HALF, 2 * HALF, 1, 1);
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        int g, mt, nt, nkb;
        int64_t r0;
        wg_tile(tile, g, mt, nt, nkb, r0);
        if (!mbar_wait_cl(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_cl(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint64_t ad = sw128_mn_desc(sa, 8192), bd = sw128_mn_desc(sa + A_BYTES, 8192);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)                // 16 rows = 2 KB in both operands
            umma2(d0, ad + (uint64_t)(128 * kk), bd + (uint64_t)(128 * kk), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma2_commit_both(empty0 + 8 * stage);
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) abort_pair(44);
      umma2_commit_both(drain);
    }
    if (lane == 0) mbar_drain_cl(drain, 0);
  } else if (WG) {
    // ---------------- epilogue, weight gradients (both CTAs): lane = output
    // row m; each 32-column TMEM load leaves as two 32-row x 16-column fp32
    // blocks through this warp's staging buffer (rows of 64 bytes, 16-byte
    // chunk q of row j at q ^ ((j >> 1) & 3): the TMA 64-byte swizzle)
    const int ew = warp - 2;
    const int sub = warp & 3;
    const int quarter = ew >> 2;
    const uint32_t stage_out = smem_u32(staging + ew * STAGE_OUT_BYTES);
    const uint32_t tempty_leader0 = map_to(tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = cid; tile < n_tiles; tile += ncl) {
      int g, mt, nt, nkb;
      int64_t r0;
      wg_tile(tile, g, mt, nt, nkb, r0);
      if (!mbar_wait_cl(tfull0 + 8 * acc, acc_phase, abort_flag)) {
        if (lane == 0) abort_pair(45);
        break;
      }
      tc_fence_after();
      const bool sh = g == p.E;
      // this warp's 32 rows: m0w .. m0w + 31, all in one output part (m_split
      // is a multiple of 64)
      const int m0w = mt * 2 * HALF + (int)rank * HALF + sub * 32;
      const bool second = m0w >= p.m_split;
      const int mr0 = second ? m0w - p.m_split : m0w;
      const CUtensorMap* mw = second ? (sh ? &p.tmWs2 : &p.tmW2) : (sh ? &p.tmWs : &p.tmW);
      const bool part_ok = (second ? (sh ? p.w_sh2 : p.w_out2) : (sh ? p.w_sh : p.w_out)) != nullptr &&
                           mr0 < p.m_valid && (second || m0w < p.m_split);
      const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * 256);
      for (int c = quarter * 32; c < 2 * HALF; c += 4 * 32) {
        const int n = nt * 2 * HALF + c;
        if (n >= p.N_out) break;                                 // warp-uniform
        __syncwarp();
        float v[32];
        tmem_ld(tbase + (uint32_t)c, v, 32);
        tmem_wait_ld();
        if (!part_ok) continue;                                  // warp-uniform
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (n + 16 * h >= p.N_out) break;
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t addr = stage_out + (uint32_t)(lane * 64) + (((uint32_t)q ^ (((uint32_t)lane >> 1) & 3u)) << 4);
            const float* x4 = v + 16 * h + 4 * q;
            const uint32_t z = nkb > 0 ? 0xffffffffu : 0u;       // a group with no rows stores zeros
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                         :: "r"(addr), "r"(__float_as_uint(x4[0]) & z), "r"(__float_as_uint(x4[1]) & z),
                            "r"(__float_as_uint(x4[2]) & z), "r"(__float_as_uint(x4[3]) & z) : "memory");
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(mw, stage_out, n + 16 * h, mr0, sh ? 0 : g);
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
  } else if (warp == 0) {
    // ---------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to(full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[MAX_STAGES] = {0, 0, 0, 0, 0, 0};
      bool ok = true;
      const uint32_t tx = 2u * (uint32_t)stage_bytes;          // both CTAs load whole boxes
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        const Tile t = decode(p, ngroups, nf, tile);
        const bool sh = t.g == p.E;
        const bool sep = sh && p.as_sep;
        const CUtensorMap* ma = sh ? &p.tmSA : &p.tmA;
        const CUtensorMap* ma1 = sh ? &p.tmSA1 : &p.tmA1;
        const CUtensorMap* mb = sep ? &p.tmBs : &p.tmB;
        const int z = sh ? 0 : t.g;
        const int wrow = t.ft * span + (int)rank * HALF;        // this CTA's weight rows
        const CUtensorMap* ma2 = swiglu ? ma1 : ma;             // the second accumulator's rows
        const int wrow2 = swiglu ? wrow : wrow + FT;
        const int64_t brow64 = (sep ? t.r0 - __ldg(p.off + p.E) : t.r0) + (int64_t)rank * (t.n / 2);
        const int brow = (int)brow64;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_cl(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + (two ? 2 : 1) * A_BYTES;
          const uint32_t fb = full_leader0 + 8 * stage;
          if (leader) mbar_expect_tx(full0 + 8 * stage, tx);
          if (p.a_mn) {
            const bool up = p.k_switch > 0 && kb >= p.k_switch;
            const CUtensorMap* mk = up ? ma1 : ma;
            const int kr = (up ? kb - p.k_switch : kb) * BK;    // k row of the stored weights
#pragma unroll
            for (int acc2 = 0; acc2 < 2; ++acc2) {
              if (acc2 == 1 && !two) break;
              const int col0 = acc2 == 0 ? wrow : wrow2;
              const uint32_t dst = sa + (uint32_t)(acc2 * A_BYTES);
#pragma unroll
              for (int j = 0; j < 2; ++j) {                     // 64-feature chunks, 8 KB apart
                const int col = col0 + 64 * j;
                if (p.b_packed) tma2_load_5d_half(dst + (uint32_t)(j * 8192), mk, kr % 128, col / 64, kr / 128, z, fb);
                else tma2_load_3d(dst + (uint32_t)(j * 8192), mk, col, kr, z, fb);
              }
            }
          } else if (p.b_packed) {
            tma2_load_5d(sa, ma, kb, wrow / 128, z, fb);
            if (two) tma2_load_5d(sa + A_BYTES, ma2, kb, wrow2 / 128, z, fb);
          } else {
            tma2_load_3d(sa, ma, kb * BK, wrow, z, fb);
            if (two) tma2_load_3d(sa + A_BYTES, ma2, kb * BK, wrow2, z, fb);
          }
          tma2_load_2d(sb, mb, kb * BK, brow, fb);
          fills[stage]++;
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) abort_pair(40);
      for (int s = 0; s < n_stages; ++s)
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
      // A descriptors: K-major, or MN-major (64-feature chunks 8 KB apart); a
      // 16-k step moves 32 bytes (K-major) or 2 KB (MN-major), in 16-byte units
      auto a_desc = [&](uint32_t a) { return p.a_mn ? sw128_mn_desc(a, 8192) : sw128_desc(a); };
      const uint64_t astep = p.a_mn ? 128 : 2;
      for (int64_t tile = cid; tile < n_tiles && ok && p.wide; tile += ncl) {
        // wide: the epilogue frees accumulator 0 (columns 0-255) before
        // accumulator 1, so this tile's MMAs into accumulator 0 start as soon
        // as it is free; a stage whose accumulator-1 MMAs cannot go yet is held
        // (at most n_stages - 1 of them) until accumulator 1 is free too
        const Tile t = decode(p, ngroups, nf, tile);
        const uint32_t idesc = make_idesc(t.n, 2 * HALF, p.a_mn);
        if (!mbar_wait_cl(tempty0, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        bool have1 = false;
        int held = 0, held_stage = 0;
        // k step nk only flushes what is still held (K shorter than the ring)
        for (int kb = 0; kb <= nk; ++kb) {
          const bool past = kb == nk;
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint64_t bd = sw128_desc(sa + 2 * A_BYTES);
          if (!past) {
            if (!mbar_wait_cl(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
            tc_fence_after();
            const uint64_t ad = a_desc(sa);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma2(tmem_base, ad + astep * kk, bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          if (!have1) {
            if (!past && held + 1 < n_stages && !mbar_test_cl(tempty0 + 8, acc_phase ^ 1u)) {
              if (held++ == 0) held_stage = stage;
              if (++stage == n_stages) { stage = 0; phase ^= 1u; }
              continue;
            }
            // accumulator 1 is free: the held stages' accumulator-1 MMAs, in
            // k order (the last held stage is k step kb - 1), then their release
            if (!mbar_wait_cl(tempty0 + 8, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
            tc_fence_after();
            have1 = true;
            for (int h = 0, hs = held_stage; h < held; ++h) {
              const uint32_t ha = smem_u32(stage_base + hs * stage_bytes);
              const uint64_t hb = sw128_desc(ha + 2 * A_BYTES), hu = a_desc(ha + A_BYTES);
              const int hk = kb - held + h;
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                umma2(tmem_base + 256, hu + astep * kk, hb + (uint64_t)(kk * 2), idesc,
                      (hk | kk) != 0 ? 1u : 0u);
              umma2_commit_both(empty0 + 8 * hs);
              if (++hs == n_stages) hs = 0;
            }
            held = 0;
          }
          if (past) break;
          const uint64_t ud = a_desc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma2(tmem_base + 256, ud + astep * kk, bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma2_commit_both(empty0 + 8 * stage);
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(tfull0);
        acc_phase ^= 1u;
      }
      for (int64_t tile = cid; tile < n_tiles && ok && !p.wide; tile += ncl) {
        const Tile t = decode(p, ngroups, nf, tile);
        const uint32_t idesc = make_idesc(t.n, 2 * HALF, p.a_mn);
        if (!mbar_wait_cl(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_cl(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint64_t bd = sw128_desc(sa + (two ? 2 : 1) * A_BYTES);
          const uint64_t ad = a_desc(sa);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)               // 16 elements along K
            umma2(d0, ad + astep * kk, bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          if (two) {
            const uint64_t ud = a_desc(sa + A_BYTES);
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma2(d0 + 256, ud + astep * kk, bd + (uint64_t)(kk * 2), idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma2_commit_both(empty0 + 8 * stage);
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(tfull0 + 8 * acc);
        if (++acc == n_acc) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) abort_pair(41);
      umma2_commit_both(drain);
    }
    if (lane == 0) mbar_drain_cl(drain, 0);
  } else {
    // ---------------- epilogue (both CTAs)
    const int ew = warp - 2;
    const int sub = warp & 3;                   // TMEM sub-partition: features 32 sub .. +32 of this CTA
    const int quarter = ew >> 2;                // token columns quarter * 32, + 128
    const uint32_t stage_out = smem_u32(staging + ew * STAGE_OUT_BYTES);
    const uint32_t tempty_leader0 = map_to(tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = cid; tile < n_tiles; tile += ncl) {
      // lane = feature f0 + lane, columns = the tile's tokens
      const Tile t = decode(p, ngroups, nf, tile);           // before the wait: off its critical path
      if (!mbar_wait_cl(tfull0 + 8 * acc, acc_phase, abort_flag)) {
        if (lane == 0) abort_pair(42);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * 256);
      // wide: accumulator a (columns 256 a ..) holds features 256 a .. of the tile
      for (int a = 0; a < (p.wide ? 2 : 1); ++a) {
        const int f0 = t.ft * span + a * FT + (int)rank * HALF + sub * 32;
        const uint32_t tb = tbase + (uint32_t)(a * 256);
        for (int c = quarter * 32; c < t.n && f0 < p.N_out; c += 4 * 32) {
          __syncwarp();
          if constexpr (DACT) {
            // dz = dh * act'(z): the chunk's 32 x 32 dh block comes in by
            // 16-byte loads into the staging buffer (its layout below), then
            // each lane takes its feature's column (features past N_out read
            // as zero); da (or dz) and SwiGLU's db go out as two stores
            // the chunk in the forward's 16-lane fragment layout (below): the dh
            // block comes in by 16-byte loads into the staging buffer (features
            // past N_out read as zero) and back by transposing matrix loads, so
            // gk[4 tg + fg] holds dh of features 8 fg + lane / 4 at tokens
            // 8 tg + 2 (lane % 4) and + 1, the elements v[4 tg + 2 h + e] of load
            // L = fg / 2, h = fg % 2 multiply; da (or dz) and SwiGLU's db go out as
            // two stores
            if (lane == 0) bulk_wait_read0();
            __syncwarp();
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int q = lane + 32 * i, j = q >> 2, ch = q & 3;
              const int64_t row = t.r0 + c + j;
              const int fc = f0 + 8 * ch;
              int4 w = make_int4(0, 0, 0, 0);
              if (fc < p.N_out && row < p.rows_max) w = ld_nc_v4(p.dh + row * p.N_out + fc);
              const uint32_t addr = stage_out + (uint32_t)(j * 64) + (((uint32_t)ch ^ (((uint32_t)j >> 1) & 3u)) << 4);
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                           :: "r"(addr), "r"(w.x), "r"(w.y), "r"(w.z), "r"(w.w) : "memory");
            }
            __syncwarp();
            uint32_t gk[16];
#pragma unroll
            for (int tg = 0; tg < 4; ++tg) {
              const uint32_t jr = (uint32_t)(8 * tg + (lane & 7));
              const uint32_t addr = stage_out + jr * 64u + ((((uint32_t)lane >> 3) ^ ((jr >> 1) & 3u)) << 4);
              asm volatile("ldmatrix.sync.aligned.x4.trans.m8n8.shared.b16 {%0, %1, %2, %3}, [%4];"
                           : "=r"(gk[4 * tg]), "=r"(gk[4 * tg + 1]), "=r"(gk[4 * tg + 2]), "=r"(gk[4 * tg + 3])
                           : "r"(addr) : "memory");
            }
            uint32_t pa[16], pb[16];
#pragma unroll
            for (int L = 0; L < 2; ++L) {
              const uint32_t lo = ((uint32_t)(16 * L) << 16) + (uint32_t)c;
              float z[16], u[16];
              tmem_ld_16x256b(tb + lo, z);
              if (swiglu) tmem_ld_16x256b(tbase + 256u + lo, u);
              tmem_wait_ld();
#pragma unroll
              for (int tg = 0; tg < 4; ++tg)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                  const int k = 4 * tg + 2 * L + h;
                  const __nv_bfloat162 g2 = *reinterpret_cast<const __nv_bfloat162*>(&gk[k]);
                  float da[2], db[2];
#pragma unroll
                  for (int e = 0; e < 2; ++e) {
                    const float gi = __bfloat162float(e == 0 ? g2.x : g2.y);
                    const float zz = z[4 * tg + 2 * h + e];
                    if (swiglu) {
                      const float sg = rcp_approx(1.0f + __expf(-zz));
                      da[e] = gi * u[4 * tg + 2 * h + e] * sg * (1.0f + zz * (1.0f - sg));
                      db[e] = gi * zz * sg;                         // dh * silu(a)
                    } else {
                      da[e] = p.epi == MOE_ACT_RELU ? (zz > 0.0f ? gi : 0.0f) : gi * gelu_grad(zz);
                      db[e] = 0.0f;
                    }
                  }
                  const __nv_bfloat162 a2 = __floats2bfloat162_rn(da[0], da[1]);
                  const __nv_bfloat162 b2 = __floats2bfloat162_rn(db[0], db[1]);
                  pa[k] = *reinterpret_cast<const uint32_t*>(&a2);
                  pb[k] = *reinterpret_cast<const uint32_t*>(&b2);
                }
            }
            for (int o = 0; o < (swiglu ? 2 : 1); ++o) {
              if (lane == 0) bulk_wait_read0();
              __syncwarp();
#pragma unroll
              for (int tg = 0; tg < 4; ++tg) {
                const uint32_t jr = (uint32_t)(8 * tg + (lane & 7));
                const uint32_t addr = stage_out + jr * 64u + ((((uint32_t)lane >> 3) ^ ((jr >> 1) & 3u)) << 4);
                const uint32_t* pk = o == 0 ? pa : pb;
                asm volatile("stmatrix.sync.aligned.x4.trans.m8n8.shared.b16 [%0], {%1, %2, %3, %4};"
                             :: "r"(addr), "r"(pk[4 * tg]), "r"(pk[4 * tg + 1]), "r"(pk[4 * tg + 2]),
                                "r"(pk[4 * tg + 3]) : "memory");
              }
              fence_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_2d(&p.tmD, stage_out, (o == 0 ? 0 : p.dz_half) + f0, (int)(t.r0 + c));
                bulk_commit();
              }
            }
            continue;
          }
          // the chunk in the 16-lane shape: load L holds features 16 L + lane / 4
          // (v[4 i], v[4 i + 1]) and 16 L + 8 + lane / 4 (v[4 i + 2], v[4 i + 3])
          // at tokens 8 i + 2 (lane % 4) and + 1, the fragment layout of an 8 x 8
          // matrix; pk[4 tg + fg] is the bf16 fragment of features 8 fg .. + 8 by
          // tokens 8 tg .. + 8
          uint32_t pk[16];
#pragma unroll
          for (int L = 0; L < 2; ++L) {
            const uint32_t ta = tb + ((uint32_t)(16 * L) << 16) + (uint32_t)c;
            float v[16];
            tmem_ld_16x256b(ta, v);
            if (swiglu) {
              float u[16];
              tmem_ld_16x256b(ta + 256u, u);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) v[i] = act_silu(v[i]) * u[i];
            } else {
              tmem_wait_ld();
              if (p.epi == MOE_ACT_RELU) {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = act_relu(v[i]);
              } else if (p.epi == MOE_ACT_GELU) {
#pragma unroll
                for (int i = 0; i < 16; i += 2) act_gelu_x2(v[i], v[i + 1]);
              }
            }
#pragma unroll
            for (int tg = 0; tg < 4; ++tg)
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                const __nv_bfloat162 b2 = __floats2bfloat162_rn(v[4 * tg + 2 * h], v[4 * tg + 2 * h + 1]);
                pk[4 * tg + 2 * L + h] = *reinterpret_cast<const uint32_t*>(&b2);
              }
          }
          // transpose into the staging buffer: token j's 32 features form a
          // 64-byte row (16-byte chunk q of row j at q ^ ((j >> 1) & 3): the TMA
          // 64-byte swizzle); one transposing matrix store per token group, this
          // lane giving the address of token 8 tg + lane % 8 in feature group lane / 8
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int tg = 0; tg < 4; ++tg) {
            const uint32_t jr = (uint32_t)(8 * tg + (lane & 7));
            const uint32_t addr = stage_out + jr * 64u + ((((uint32_t)lane >> 3) ^ ((jr >> 1) & 3u)) << 4);
            asm volatile("stmatrix.sync.aligned.x4.trans.m8n8.shared.b16 [%0], {%1, %2, %3, %4};"
                         :: "r"(addr), "r"(pk[4 * tg]), "r"(pk[4 * tg + 1]), "r"(pk[4 * tg + 2]), "r"(pk[4 * tg + 3])
                         : "memory");
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            // rows past the tile's tokens lie in the group's padding: harmless
            tma_store_2d(&p.tmD, stage_out, f0, (int)(t.r0 + c));
            bulk_commit();
          }
        }
        if (p.wide) {
          // accumulator a is read: the next tile's MMAs may write it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * a);
        }
      }
      if (!p.wide) {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
      }
      if (++acc == n_acc) { acc = 0; acc_phase ^= 1u; }
    }
    if (lane == 0) bulk_wait0();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();
  pdl_trigger();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
}

// One warp: tp[g] = sum over g' < g of ceil(rows(g') / 256) token tiles, rows
// as in group_rows; tp[ngroups] = the total.
__global__ void token_tile_prefix_kernel(const int32_t* off, const int32_t* valid, int ngroups, int E, int64_t T,
                                         int64_t rows_max, int32_t* tp) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x;
  const int seg = (ngroups + 31) / 32;
  const int g0 = min(ngroups, lane * seg), g1 = min(ngroups, g0 + seg);
  auto tiles = [&](int g) { return (int)((group_rows(off, valid, g, E, T, rows_max) + TT - 1) / TT); };
  int s = 0;
  for (int g = g0; g < g1; ++g) s += tiles(g);
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - s;
  for (int g = g0; g < g1; ++g) {
    tp[g] = run;
    run += tiles(g);
  }
  if (lane == 31) tp[ngroups] = incl;
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
  key.box[1] = HALF;
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
  key.box[1] = HALF;
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

// 5-D map over packed weights [G][N/128][K/64][128][64] (a stored [G, N, K]
// matrix) read along K, the columns: box 64 x 64, half a block.
static bool map_packed_half(CUtensorMap* m, const void* base, int G, int N, int K) {
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
  key.box[1] = 64;
  key.box[2] = key.box[3] = key.box[4] = 1;
  return encode_cached(m, key);
}

// 3-D map over stacked weights [G, N, K] read along K: box 64 x 64 x 1.
static bool map_weights_half(CUtensorMap* m, const void* base, int G, int N, int K) {
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
  key.box[1] = 64;
  key.box[2] = 1;
  return encode_cached(m, key);
}

// 2-D map over a row-major bf16 matrix [rows, W] read along W: box 64 x 64.
static bool map_rows_half(CUtensorMap* m, const void* base, int64_t rows, int W) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 2;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)W;
  key.dims[1] = (cuuint64_t)rows;
  key.strides[0] = (cuuint64_t)W * 2;
  key.box[0] = BK;
  key.box[1] = 64;
  return encode_cached(m, key);
}

// 3-D map over an fp32 output [G, rows, N], box 16 x 32 x 1, 64-byte swizzle (TMA store).
static bool map_out_f32(CUtensorMap* m, const void* base, int G, int rows, int N) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 3;
  key.f32 = 1;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_64B;
  key.dims[0] = (cuuint64_t)N;
  key.dims[1] = (cuuint64_t)rows;
  key.dims[2] = (cuuint64_t)G;
  key.strides[0] = (cuuint64_t)N * 4;
  key.strides[1] = (cuuint64_t)rows * N * 4;
  key.box[0] = 16;
  key.box[1] = 32;
  key.box[2] = 1;
  return encode_cached(m, key);
}

// 2-D map over a bf16 output [rows, N], box 32 x 32, 64-byte swizzle (TMA store).
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
    if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_tn_kernel<0>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = sm_count() / 2;
    }
    c = n;
  }
  return c;
}

static cudaError_t launch_pairs(const KParams& k, cudaStream_t stream);

}  // namespace gtn

cudaError_t launch_grouped_gemm_tn(const GemmParams& p, cudaStream_t stream) {
  using namespace gtn;
  if (p.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  KParams k{};
  const void* b1 = p.b1 ? p.b1 : p.b0;
  const void* s0 = p.sb0 ? p.sb0 : p.b0;
  const void* s1 = p.sb1 ? p.sb1 : s0;
  bool ok = true;
  if (p.b_packed) {
    ok = ok && map_packed(&k.tmA, p.b0, p.E, p.Nw, p.K);
    ok = ok && map_packed(&k.tmA1, b1, p.E, p.Nw, p.K);
    ok = ok && map_packed(&k.tmSA, s0, 1, p.Nw, p.K);
    ok = ok && map_packed(&k.tmSA1, s1, 1, p.Nw, p.K);
  } else {
    ok = ok && map_weights(&k.tmA, p.b0, p.E, p.Nw, p.K);
    ok = ok && map_weights(&k.tmA1, b1, p.E, p.Nw, p.K);
    ok = ok && map_weights(&k.tmSA, s0, 1, p.Nw, p.K);
    ok = ok && map_weights(&k.tmSA1, s1, 1, p.Nw, p.K);
  }
  ok = ok && map_rows(&k.tmB, p.a_routed, p.rows_max, p.K);
  ok = ok && map_rows(&k.tmBs, p.a_shared ? p.a_shared : p.a_routed, p.a_shared ? p.T : p.rows_max, p.K);
  ok = ok && map_out(&k.tmD, p.d, p.rows_max, p.Nw);
  if (!ok) return cudaErrorInvalidValue;
  const int ngroups = p.E + (p.n_shared ? 1 : 0);
  if (p.pair_prefix_ready == 0)
    launch_pdl(token_tile_prefix_kernel, 1, 32, 0, stream, p.expert_offset, p.valid_rows, ngroups, p.E, p.T,
               p.rows_max, p.pair_prefix);
  k.off = p.expert_offset;
  k.tp = p.pair_prefix;
  k.valid = p.valid_rows;
  k.status = p.status;
  k.rows_max = p.rows_max;
  k.T = p.T;
  k.K = p.K;
  k.N_out = p.Nw;
  k.E = p.E;
  k.n_shared = p.n_shared;
  k.epi = p.epi;
  k.as_sep = p.a_shared != nullptr;
  k.b_packed = p.b_packed;
  // 512-feature tiles where the epilogue is cheap (no activation, or ReLU): two
  // accumulators share every B tile, so a pair moves 48 KB per 64-k step for
  // twice the MMA work of a 32 KB step.  They are single-buffered, so an
  // expensive epilogue (GELU) would stall the MMAs: those keep 256-feature,
  // double-buffered tiles.
  k.wide = ((p.epi < 0 || p.epi == MOE_ACT_RELU) && p.Nw >= 2 * FT) ? 1 : 0;
  return launch_pairs(k, stream);
}

// The backward's weight-side contractions on pairs of SMs (see KParams::a_mn):
// out[rows, N] = a[rows, K] * W, W stored [G, K0, N] and read along N, k blocks
// >= k_switch from b1; the same token tiles as the forward (kept rows rounded up
// to 16 per group, the shared block's T rows in place).
cudaError_t launch_bwd_dgrad_pair(const BwdGemm& q, int32_t* pair_prefix, const int32_t* valid,
                                  cudaStream_t stream) {
  using namespace gtn;
  if (q.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  KParams k{};
  const void* b1 = q.b1 ? q.b1 : q.b0;
  const void* s0 = q.sb0 ? q.sb0 : q.b0;
  const void* s1 = q.sb1 ? q.sb1 : s0;
  bool ok = true;
  if (q.b_packed) {
    ok = ok && map_packed_half(&k.tmA, q.b0, q.E, q.K0, q.N);
    ok = ok && map_packed_half(&k.tmA1, b1, q.E, q.K0, q.N);
    ok = ok && map_packed_half(&k.tmSA, s0, 1, q.K0, q.N);
    ok = ok && map_packed_half(&k.tmSA1, s1, 1, q.K0, q.N);
  } else {
    ok = ok && map_weights_half(&k.tmA, q.b0, q.E, q.K0, q.N);
    ok = ok && map_weights_half(&k.tmA1, b1, q.E, q.K0, q.N);
    ok = ok && map_weights_half(&k.tmSA, s0, 1, q.K0, q.N);
    ok = ok && map_weights_half(&k.tmSA1, s1, 1, q.K0, q.N);
  }
  ok = ok && map_rows(&k.tmB, q.a, q.rows_max, q.K);
  ok = ok && map_rows(&k.tmBs, q.a, q.rows_max, q.K);
  ok = ok && map_out(&k.tmD, q.out, q.rows_max, q.N);
  if (!ok) return cudaErrorInvalidValue;
  const int ngroups = q.E + (q.n_shared ? 1 : 0);
  launch_pdl(token_tile_prefix_kernel, 1, 32, 0, stream, q.off, valid, ngroups, q.E, q.T, q.rows_max, pair_prefix);
  k.off = q.off;
  k.tp = pair_prefix;
  k.valid = valid;
  k.status = q.status;
  k.rows_max = q.rows_max;
  k.T = q.T;
  k.K = q.K;
  k.N_out = q.N;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.epi = -1;
  k.as_sep = 0;
  k.b_packed = q.b_packed;
  k.wide = q.N >= 2 * FT ? 1 : 0;
  k.a_mn = 1;
  k.k_switch = q.k_switch;
  return launch_pairs(k, stream);
}

// The backward's dz = dh * act'(z) on pairs of SMs: z (and SwiGLU's up
// projection) recomputed from the dispatched rows as the forward's first
// contraction does, dh read in the epilogue, dz [rows_max, dz_ld] written with
// SwiGLU's db at column dz_ld / 2.
cudaError_t launch_bwd_dact_pair(const BwdGemm& q, int dz_ld, int32_t* pair_prefix, const int32_t* valid,
                                 cudaStream_t stream) {
  using namespace gtn;
  if (q.rows_max == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  KParams k{};
  const bool swiglu = q.act == MOE_ACT_SWIGLU;
  const void* b1 = q.b1 ? q.b1 : q.b0;
  const void* s0 = q.sb0 ? q.sb0 : q.b0;
  const void* s1 = q.sb1 ? q.sb1 : s0;
  bool ok = true;
  if (q.b_packed) {
    ok = ok && map_packed(&k.tmA, q.b0, q.E, q.N, q.K);
    ok = ok && map_packed(&k.tmA1, b1, q.E, q.N, q.K);
    ok = ok && map_packed(&k.tmSA, s0, 1, q.N, q.K);
    ok = ok && map_packed(&k.tmSA1, s1, 1, q.N, q.K);
  } else {
    ok = ok && map_weights(&k.tmA, q.b0, q.E, q.N, q.K);
    ok = ok && map_weights(&k.tmA1, b1, q.E, q.N, q.K);
    ok = ok && map_weights(&k.tmSA, s0, 1, q.N, q.K);
    ok = ok && map_weights(&k.tmSA1, s1, 1, q.N, q.K);
  }
  ok = ok && map_rows(&k.tmB, q.a, q.rows_max, q.K);
  ok = ok && map_rows(&k.tmBs, q.a_shared ? q.a_shared : q.a, q.a_shared ? q.T : q.rows_max, q.K);
  ok = ok && map_out(&k.tmD, q.out, q.rows_max, dz_ld);
  if (!ok) return cudaErrorInvalidValue;
  const int ngroups = q.E + (q.n_shared ? 1 : 0);
  launch_pdl(token_tile_prefix_kernel, 1, 32, 0, stream, q.off, valid, ngroups, q.E, q.T, q.rows_max, pair_prefix);
  k.off = q.off;
  k.tp = pair_prefix;
  k.valid = valid;
  k.status = q.status;
  k.rows_max = q.rows_max;
  k.T = q.T;
  k.K = q.K;
  k.N_out = q.N;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.epi = q.act;
  k.as_sep = q.a_shared != nullptr;
  k.b_packed = q.b_packed;
  k.wide = (q.act == MOE_ACT_RELU && q.N >= 2 * FT) ? 1 : 0;
  k.dact = 1;
  k.dz_half = swiglu ? dz_ld / 2 : 0;
  k.dh = static_cast<const __nv_bfloat16*>(q.dh);
  return launch_pairs(k, stream);
}

// The weight gradients on pairs of SMs: per expert g, w_out[g] = a_g^T b_g in
// fp32, over the group's kept rows in 64-row blocks (the padding rows past them
// in a block are zero in b for dW1 and in a for dW2); tiles of 256 output rows
// x 256 columns; output rows >= m_split go to w_out2 (m_valid rows each); the
// shared expert's to w_sh / w_sh2, its b rows from b_shared (row - off[E]).
cudaError_t launch_bwd_wgrad_pair(const BwdGemm& q, const int32_t* valid, cudaStream_t stream) {
  using namespace gtn;
  if (q.rows_max == 0 && q.E == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  KParams k{};
  bool ok = true;
  const int64_t rows = q.rows_max > 0 ? q.rows_max : 1;
  ok = ok && map_rows_half(&k.tmA, q.a, rows, q.M);
  ok = ok && map_rows_half(&k.tmB, q.b0, rows, q.N);
  ok = ok && map_rows_half(&k.tmBs, q.b_shared ? q.b_shared : q.b0, q.b_shared ? (q.T > 0 ? q.T : 1) : rows, q.N);
  // absent outputs map the first one: the kernel never stores through them
  ok = ok && map_out_f32(&k.tmW, q.w_out, q.E > 0 ? q.E : 1, q.m_valid, q.N);
  ok = ok && map_out_f32(&k.tmW2, q.w_out2 ? q.w_out2 : q.w_out, q.E > 0 ? q.E : 1, q.m_valid, q.N);
  ok = ok && map_out_f32(&k.tmWs, q.w_sh ? q.w_sh : q.w_out, 1, q.m_valid, q.N);
  ok = ok && map_out_f32(&k.tmWs2, q.w_sh2 ? q.w_sh2 : (q.w_sh ? q.w_sh : q.w_out), 1, q.m_valid, q.N);
  if (!ok) return cudaErrorInvalidValue;
  k.off = q.off;
  k.valid = valid;
  k.status = q.status;
  k.rows_max = q.rows_max;
  k.T = q.T;
  k.N_out = q.N;
  k.M_out = q.M;
  k.E = q.E;
  k.n_shared = q.n_shared;
  k.epi = -1;
  k.m_split = q.m_split;
  k.m_valid = q.m_valid;
  k.b_sep = q.b_shared != nullptr;
  k.w_out = q.w_out;
  k.w_out2 = q.w_out2;
  k.w_sh = q.w_sh;
  k.w_sh2 = q.w_sh2;
  return launch_pairs(k, stream);
}

namespace gtn {
static cudaError_t launch_pairs(const KParams& k, cudaStream_t stream) {
  auto kern = k.M_out > 0 ? grouped_gemm_tn_kernel<2> : k.dact ? grouped_gemm_tn_kernel<1> : grouped_gemm_tn_kernel<0>;
  cudaError_t e = ensure_smem(kern, SMEM_BYTES);
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
  e = cudaLaunchKernelEx(&cfg, kern, k);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}
}  // namespace gtn

}  // namespace moe
