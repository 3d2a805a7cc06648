// Router logits and routing on pairs of SMs (tcgen05.mma.cta_group::2), for
// every router with E <= 256 and at least 256 tokens: 256 tokens per pair tile,
// each CTA holding 128 tokens (A) and half of the experts of every weight plane (B).
//
// Method: the router of an MoE layer ("Expert-parallel MoE training"
// explainer, router section: a linear gate with E outputs in fp32; "Switch
// Routing", 2.1 and 2.2, selective precision: the router in fp32).  The fp32
// router weight is split into three bf16 planes, hi + mid + lo = Wg exactly
// (moe_pack_router_weight), so x (bf16) times each plane is exact in fp32 and
// one fp32 accumulator gives fp32 logits.  The k loop multiplies, per 64-k
// step, the A chunk by the hi, mid and lo planes in that order: the order of
// the one-SM router (grouped_gemm.cu), so the logits are bitwise the same.
//
// Why a pair: an SM takes in its operands at a fixed rate (about 45 GB/s on
// a B200 SM, from L2 or HBM alike), so the router's k loop costs what its CTA
// loads.  On one SM a 128-token tile loads its A chunk and all E rows of every
// plane per k step (16 + 3 * 32 KB at E = 256; 16 + 3 * 8 KB at E = 64).  A
// pair shares the plane rows: each CTA loads its own 128 tokens and E/2 rows
// of each plane, and one MMA instruction from the even CTA writes every CTA's
// 128 rows x E columns into that CTA's tensor memory, so each CTA still holds
// its tokens' complete logits and routes them as the one-SM router does
// (route_tmem.cuh).  The CTA count is the one-SM router's (two CTAs per
// 256 tokens), each loading less.
//
// Roles per CTA (576 threads): warp 0 issues the TMA loads (both CTAs; every
// copy completes on the even CTA's full barrier, armed with both CTAs'
// bytes); warp 1 of the even CTA issues the MMAs and commits with a multicast
// to both CTAs; warps 2-17 route the tile's tokens from the accumulator and
// arrive on the even CTA's accumulator-empty barrier.  Two 256-column
// accumulators overlap one tile's routing with the next tile's k loop.
// No load in this file uses cluster multicast.  Every wait is bounded: on
// expiry the CTA records MOE_ETIMEOUT, raises both CTAs' abort flags, and the
// pair drains what it issued and frees TMEM.
#include <cuda.h>
#include <cuda_runtime.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"
#include "pair_common.cuh"
#include "route_tmem.cuh"
#include "tc_common.cuh"

namespace moe {
namespace rpair {

using namespace tcx;
using namespace pairx;

constexpr int BK = 64;
constexpr int HALF = 128;                        // tokens of one CTA
constexpr int A_BYTES = HALF * BK * 2;           // 16 KB
constexpr int RING_BYTES = 192 * 1024;
constexpr int MAX_STAGES = 6;
constexpr int EPI_WARPS = 16;
constexpr int THREADS = 64 + EPI_WARPS * 32;
constexpr int TMEM_COLS = 512;
constexpr int STAGING_BYTES = 32 * 1024;         // the routing's exchange area
constexpr int SMEM_BYTES = RING_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;
static_assert(kRouteStagingBytes <= STAGING_BYTES, "routing exchange area");
static_assert(EPI_WARPS * 32 == kRouteThreads, "routing threads");

struct RParams {
  CUtensorMap tmA;          // x [T, H] bf16, box 64 x 128
  CUtensorMap tmB;          // planes [E, 3 Hp] bf16 as [1, E, 3 Hp], box 64 x N/2 x 1
  RouterParams rp;
  DevStatus* status;
  int64_t nblk, T;
  int Hp, N;                // plane width (k); MMA N = E rounded up to 16 (<= 256)
};

// True iff `v` holds in every epilogue thread (named barrier 1 with a reduction:
// the warps leave together or not at all, before the routing's barriers).
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred pi, po;\n\t"
               "setp.ne.u32 pi, %1, 0;\n\t"
               "bar.red.and.pred po, 1, %2, pi;\n\t"
               "selp.u32 %0, 1, 0, po;\n\t}"
               : "=r"(r) : "r"((uint32_t)v), "r"(EPI_WARPS * 32) : "memory");
  return r != 0;
}

template <int KM>
__global__ void __launch_bounds__(THREADS, 1) router_pair_kernel(const __grid_constant__ RParams p) {
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
  const int half_n = p.N / 2;
  const int plane_bytes = half_n * BK * 2;
  const int stage_bytes = A_BYTES + 3 * plane_bytes;
  const int n_stages = min(MAX_STAGES, RING_BYTES / stage_bytes);
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
    prefetch_map(&p.tmA);
    prefetch_map(&p.tmB);
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
  if (!tmem_same && threadIdx.x == 0) set_status(p.status, MOE_EDEVICE, 32);

  const int64_t n_tiles = tmem_same ? (p.T + 2 * HALF - 1) / (2 * HALF) : 0;
  const int nk = p.Hp / BK;
  const int64_t cid = cluster_id(), ncl = cluster_count();

  if (warp == 0) {
    // ---------------- TMA producer (both CTAs)
    if (lane == 0) {
      const uint32_t full_leader0 = map_to(full0, 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t fills[MAX_STAGES] = {0, 0, 0, 0, 0, 0};
      bool ok = true;
      const uint32_t tx = 2u * (uint32_t)stage_bytes;           // both CTAs' boxes
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        const int arow = (int)(tile * 2 * HALF + (int64_t)rank * HALF);
        const int brow = (int)rank * half_n;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_cl(empty0 + 8 * stage, phase ^ 1u, abort_flag)) { ok = false; break; }
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = full_leader0 + 8 * stage;
          if (leader) mbar_expect_tx(full0 + 8 * stage, tx);
          tma2_load_2d(sa, &p.tmA, kb * BK, arow, fb);
#pragma unroll
          for (int pl = 0; pl < 3; ++pl)
            tma2_load_3d(sb + (uint32_t)(pl * plane_bytes), &p.tmB, pl * p.Hp + kb * BK, brow, 0, fb);
          fills[stage]++;
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) abort_pair(50);
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
      const uint32_t idesc = make_idesc(p.N, 2 * HALF);
      for (int64_t tile = cid; tile < n_tiles && ok; tile += ncl) {
        if (!mbar_wait_cl(tempty0 + 8 * acc, acc_phase ^ 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * 256);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_cl(full0 + 8 * stage, phase, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(stage_base + stage * stage_bytes);
          const uint64_t ad = sw128_desc(sa);
#pragma unroll
          for (int pl = 0; pl < 3; ++pl) {                      // hi, mid, lo
            const uint64_t bd = sw128_desc(sa + A_BYTES + (uint32_t)(pl * plane_bytes));
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              umma2(d, ad + (uint64_t)(kk * 2), bd + (uint64_t)(kk * 2), idesc, (kb | pl | kk) != 0 ? 1u : 0u);
          }
          umma2_commit_both(empty0 + 8 * stage);
          if (++stage == n_stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma2_commit_both(tfull0 + 8 * acc);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok) abort_pair(51);
      umma2_commit_both(drain);
    }
    if (lane == 0) mbar_drain_cl(drain, 0);
  } else {
    // ---------------- routing (both CTAs): this CTA's 128 tokens of the tile
    const int ew = warp - 2;
    const int sub = warp & 3;                    // TMEM sub-partition: tokens 32 sub .. +32
    const int quarter = ew >> 2;                 // expert column range of the routing
    const uint32_t tempty_leader0 = map_to(tempty0, 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int64_t tile = cid; tile < n_tiles; tile += ncl) {
      const bool got = epi_all(mbar_wait_cl(tfull0 + 8 * acc, acc_phase, abort_flag));
      if (!got) {
        if (lane == 0) abort_pair(52);
        break;
      }
      tc_fence_after();
      const uint32_t tbase = tmem_base + ((uint32_t)(sub * 32) << 16) + (uint32_t)(acc * 256);
      route_tile_tmem<KM>(p.rp, p.nblk, 2 * tile + rank, sub, quarter, lane, staging, tbase, p.N);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader0 + 8 * acc);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
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

// 2-D map over x [T, H] (bf16), box 64 x 128, 128-byte swizzle.
static bool map_x(CUtensorMap* m, const void* base, int64_t T, int H) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 2;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)H;
  key.dims[1] = (cuuint64_t)T;
  key.strides[0] = (cuuint64_t)H * 2;
  key.box[0] = BK;
  key.box[1] = HALF;
  return encode_cached(m, key);
}

// 3-D map over the planes [1, E, 3 Hp] (bf16), box 64 x rows x 1 (rows past E read as zero).
static bool map_planes(CUtensorMap* m, const void* base, int E, int Hp3, int rows) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.base = base;
  key.rank = 3;
  key.swizzle = CU_TENSOR_MAP_SWIZZLE_128B;
  key.dims[0] = (cuuint64_t)Hp3;
  key.dims[1] = (cuuint64_t)E;
  key.dims[2] = 1;
  key.strides[0] = (cuuint64_t)Hp3 * 2;
  key.strides[1] = (cuuint64_t)E * Hp3 * 2;
  key.box[0] = BK;
  key.box[1] = (cuuint32_t)rows;
  key.box[2] = 1;
  return encode_cached(m, key);
}

template <int KM>
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
    if (cudaOccupancyMaxActiveClusters(&n, router_pair_kernel<KM>, &cfg) != cudaSuccess || n < 1) {
      cudaGetLastError();
      n = sm_count() / 2;
    }
    c = n;
  }
  return c;
}

template <int KM>
static cudaError_t launch_km(const RParams& k, int64_t n_tiles, cudaStream_t stream) {
  cudaError_t e = ensure_smem(router_pair_kernel<KM>, SMEM_BYTES);
  if (e != cudaSuccess) return e;
  const int64_t pairs = min((int64_t)resident_pairs<KM>(), n_tiles);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)(2 * (pairs > 0 ? pairs : 1)));
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
  e = cudaLaunchKernelEx(&cfg, router_pair_kernel<KM>, k);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace rpair

bool router_pair_fits(int64_t T, int H, int E) {
  return E <= 256 && T >= 256 && router_plane_width(H) >= rpair::BK;
}

cudaError_t launch_router_pair(const void* x, const void* planes, int64_t T, int H, int E, DevStatus* status,
                               const RouterParams& route, int64_t nblk, cudaStream_t stream) {
  using namespace rpair;
  if (T == 0) return cudaSuccess;
  if (encode_fn() == nullptr) return cudaErrorNotSupported;
  const int Hp = router_plane_width(H);
  RParams k{};
  k.N = (E + 15) / 16 * 16;
  bool ok = map_x(&k.tmA, x, T, H);
  ok = ok && map_planes(&k.tmB, planes, E, 3 * Hp, k.N / 2);
  if (!ok) return cudaErrorInvalidValue;
  k.rp = route;
  k.status = status;
  k.nblk = nblk;
  k.T = T;
  k.Hp = Hp;
  const int64_t n_tiles = (T + 2 * HALF - 1) / (2 * HALF);
  switch (route_km_of(route.k)) {
    case 1: return launch_km<1>(k, n_tiles, stream);
    case 2: return launch_km<2>(k, n_tiles, stream);
    case 4: return launch_km<4>(k, n_tiles, stream);
    case 8: return launch_km<8>(k, n_tiles, stream);
    default: return launch_km<16>(k, n_tiles, stream);
  }
}

}  // namespace moe
