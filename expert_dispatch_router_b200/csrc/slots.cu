// Capacity-slot assignment without a dense [T,E,C] mask.
//
// Method: "Expert-parallel MoE training" explainer, drop/pad section ("position"
// policy: overflow beyond the expert's capacity is dropped in arrival order) and
// capacity section; "The MoE spends too much time on the gate network"
// (DeepSpeed discussion 7508) for why the one-hot [T,E,C] mask must not exist.
//
// The assignment sequence is a = r*T + t (every first choice in token order,
// then every second choice, ...).  slot(a) = number of earlier assignments of
// the same expert.  Three small kernels, all deterministic:
//   1. count   : CTA c counts its 256-assignment chunk (kSlotChunk) per expert
//                (shared-memory histogram) -> chunk_cnt[e][c].
//   2. scan    : CTA e scans chunk_cnt[e][*] -> chunk base offsets, the expert's
//                pre-drop count and kept count, and its aux-loss term.  The CTA
//                that finishes last (an atomic ticket; no CTA waits for another)
//                scans the 128-padded kept counts into the per-expert row
//                blocks, sums the aux loss (and z-loss) and writes row_token's
//                padding and shared rows, then resets the ticket.
//   3. rank    : CTA c re-reads its chunk; warps rank equal experts inside each
//                32-assignment step with match_any, carry per-warp running counts,
//                prefix them over the warps in order, and add the chunk base.
// Total metadata traffic is O(T*k + E*chunks); nothing scales with C.
// Layers whose assignments fit one resident CTA per SM (1024 assignments each)
// and that use the "position" policy or none run the same steps in one launch
// with two grid barriers (slot_fused_kernel below).
//
// "probs" policy (same section: drop the lowest-probability assignments): the
// rank kernel lists every assignment of an over-full expert, in arrival order,
// as (order-preserving gate key, assignment index); one CTA per such expert
// then finds the C-th largest key with a 4 x 8-bit radix select and makes one
// ordered pass that keeps the keys above it plus the earliest arrivals equal to
// it, numbering the kept ones in arrival order.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kSlotThreads = 256;
constexpr int kSlotWarps = kSlotThreads / 32;
constexpr int kStepsPerWarp = kSlotChunk / (kSlotWarps * 32);   // 32-assignment steps per warp

__device__ __forceinline__ int load_assignment(const SlotParams& p, int64_t a, int64_t A) {
  if (a >= A) return -1;
  const int64_t r = a / p.T, t = a - r * p.T;
  return p.ids[t * p.k + r];
}

__global__ void __launch_bounds__(kSlotThreads) slot_count_kernel(SlotParams p, int nchunk) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int hist[];
  const int64_t A = p.T * p.k;
  for (int e = threadIdx.x; e < p.E; e += kSlotThreads) hist[e] = 0;
  __syncthreads();
  const int64_t a0 = (int64_t)blockIdx.x * kSlotChunk;
  for (int i = threadIdx.x; i < kSlotChunk; i += kSlotThreads) {
    const int e = load_assignment(p, a0 + i, A);
    if (a0 + i >= A) break;
    if (e == -1) continue;                      // a choice that is not dispatched
    if (e < 0 || e >= p.E) { set_status(p.status, MOE_EDEVICE, 1); continue; }
    atomicAdd(&hist[e], 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < p.E; e += kSlotThreads)
    p.chunk_cnt[(int64_t)e * nchunk + blockIdx.x] = hist[e];
}

// Exclusive scan of one int per thread over a block of NW warps: returns the
// thread's exclusive prefix and sets `total`.  `sh` holds NW ints; the trailing
// barrier lets the caller reuse it at once.
template <int NW>
__device__ __forceinline__ int block_scan_excl(int v, int* sh, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sh[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < NW ? sh[lane] : 0;
#pragma unroll
    for (int o = 1; o < NW; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) sh[lane] = w;             // inclusive warp totals
  }
  __syncthreads();
  const int excl = (warp == 0 ? 0 : sh[warp - 1]) + x - v;
  total = sh[NW - 1];
  __syncthreads();
  return excl;
}

// Row blocks (exclusive scan of the 128-padded kept counts; the shared block
// last), the "probs" lists' starts, the aux-loss and z-loss totals, and
// row_token's padding and shared rows.  Run by one CTA of kSlotThreads threads.
__device__ __forceinline__ void slot_offsets(const SlotParams& p) {
  __shared__ int sh[kSlotWarps];
  __shared__ int sh_off[kMaxE + 2];
  __shared__ int sh_kept[kMaxE];
  __shared__ double red[kSlotThreads];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  constexpr int kPer = (kMaxE + kSlotThreads - 1) / kSlotThreads;   // experts per thread, contiguous
  const int e0 = tid * kPer;
  int loc = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (e0 + i < p.E) {
      const int kept = __ldcg(p.kept_count + e0 + i);
      sh_kept[e0 + i] = kept;
      loc += (int)round_up(kept, kRowPad);
    }
  int routed;
  int run = block_scan_excl<kSlotWarps>(loc, sh, routed);
#pragma unroll
  for (int i = 0; i < kPer; ++i)
    if (e0 + i < p.E) {
      sh_off[e0 + i] = run;
      run += (int)round_up(sh_kept[e0 + i], kRowPad);
    }
  if (p.gates != nullptr) {
    // "probs" policy: where each expert's arrival-ordered list starts
    int loc_c = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (e0 + i < p.E) loc_c += __ldcg(p.expert_count + e0 + i);
    int total;
    int c = block_scan_excl<kSlotWarps>(loc_c, sh, total);
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (e0 + i < p.E) {
        p.cum[e0 + i] = c;
        c += __ldcg(p.expert_count + e0 + i);
      }
  }
  if (tid == 0) {
    sh_off[p.E] = routed;
    const int64_t end = routed + (p.n_shared ? round_up(p.T, kRowPad) : 0);
    sh_off[p.E + 1] = (int)end;
    if (end > p.rows_max) set_status(p.status, MOE_EDEVICE, 2);
  }
  __syncthreads();
  for (int i = tid; i < p.E + 2; i += kSlotThreads) p.expert_offset[i] = sh_off[i];
  if (p.aux != nullptr) {
    // aux loss = alpha * E * sum_e term[e]: per-thread sums in expert order, then a fixed tree
    double t = 0.0;
    for (int e = tid; e < p.E; e += kSlotThreads) t += p.T > 0 ? __ldcg(p.aux_term + e) : 0.0;
    red[tid] = t;
    __syncthreads();
    for (int s = kSlotThreads / 2; s > 0; s >>= 1) {
      if (tid < s) red[tid] += red[tid + s];
      __syncthreads();
    }
    if (tid == 0) *p.aux = (float)((double)p.aux_alpha * (double)p.E * red[0]);
    __syncthreads();
    if (p.zsum_part != nullptr) {
      // z-loss = coef * mean_t lse_t^2 from the router's per-block sums, fixed order
      double z = 0.0;
      for (int b = tid; b < p.nblk_router; b += kSlotThreads) z += (double)p.zsum_part[b];
      red[tid] = z;
      __syncthreads();
      for (int s = kSlotThreads / 2; s > 0; s >>= 1) {
        if (tid < s) red[tid] += red[tid + s];
        __syncthreads();
      }
      if (tid == 0) p.aux[1] = p.T > 0 ? (float)((double)p.z_coef * red[0] / (double)p.T) : 0.0f;
    }
  }
  // padding rows of each routed block -> -1; the shared block's rows -> their tokens
  for (int e = warp; e < p.E; e += kSlotWarps) {
    const int start = sh_off[e] + sh_kept[e], stop = sh_off[e + 1];
    for (int r = start + lane; r < stop; r += 32) p.row_token[r] = -1;
  }
  if (p.n_shared) {
    const int64_t s0 = sh_off[p.E], n = round_up(p.T, kRowPad);
    for (int64_t i = tid; i < n; i += kSlotThreads)
      if (s0 + i < p.rows_max) p.row_token[s0 + i] = i < p.T ? (int)i : -1;
  }
}

__global__ void __launch_bounds__(kSlotThreads) slot_scan_kernel(SlotParams p, int nchunk) {
  pdl_wait();
  pdl_trigger();
  __shared__ int sh[kSlotWarps];
  const int e = blockIdx.x;
  int* row = p.chunk_cnt + (int64_t)e * nchunk;
  int running = 0;
  for (int base = 0; base < nchunk; base += kSlotThreads) {
    const int c = base + threadIdx.x;
    const int v = c < nchunk ? row[c] : 0;
    int tot;
    const int excl = block_scan_excl<kSlotWarps>(v, sh, tot);
    if (c < nchunk) row[c] = running + excl;        // chunk base, in place
    running += tot;
  }
  if (threadIdx.x == 0) {
    p.expert_count[e] = running;
    const int kept = p.capacity < 0 ? running : (int)min((int64_t)running, p.capacity);
    p.kept_count[e] = kept;
  }
  if (p.psum_part != nullptr) {
    // this expert's aux-loss term f_e * P_e: f from the pre-drop count (or, when
    // some choices were not dispatched, from the router's selection counts), P
    // from the router's per-CTA sums of p (fp64, fixed block-then-tree order)
    __shared__ double red[kSlotThreads];
    __shared__ long long redc[kSlotThreads];
    double ps = 0.0;
    long long cs = 0;
    for (int b = threadIdx.x; b < p.nblk_router; b += kSlotThreads) {
      ps += (double)p.psum_part[(int64_t)b * p.E + e];
      if (p.cnt_part != nullptr) cs += p.cnt_part[(int64_t)b * p.E + e];
    }
    red[threadIdx.x] = ps;
    redc[threadIdx.x] = cs;
    __syncthreads();
    for (int s = kSlotThreads / 2; s > 0; s >>= 1) {
      if ((int)threadIdx.x < s) {
        red[threadIdx.x] += red[threadIdx.x + s];
        redc[threadIdx.x] += redc[threadIdx.x + s];
      }
      __syncthreads();
    }
    if (threadIdx.x == 0) {
      const double f = (double)(p.cnt_part != nullptr ? redc[0] : running) / ((double)p.T * p.k);
      p.aux_term[e] = f * (red[0] / (double)p.T);
    }
  }
  // The last expert CTA to finish (fence + ticket; no CTA waits for another)
  // lays out the row blocks from every expert's kept count.
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(p.ticket, 1u) == (unsigned)(p.E - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  slot_offsets(p);
  if (threadIdx.x == 0) *p.ticket = 0u;       // ready for the next call
}

__global__ void __launch_bounds__(kSlotThreads) slot_rank_kernel(SlotParams p, int nchunk) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int wcnt[];                 // [warps][E]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t A = p.T * p.k;
  for (int i = tid; i < kSlotWarps * p.E; i += kSlotThreads) wcnt[i] = 0;
  __syncthreads();
  const int64_t a_warp = (int64_t)blockIdx.x * kSlotChunk + (int64_t)warp * (kStepsPerWarp * 32);
  const unsigned lt_mask = (1u << lane) - 1u;
  int local[kStepsPerWarp];
  int expert[kStepsPerWarp];
#pragma unroll
  for (int s = 0; s < kStepsPerWarp; ++s) {
    const int64_t a = a_warp + s * 32 + lane;
    int e = load_assignment(p, a, A);          // -1 past the end
    if (a < A && (e < 0 || e >= p.E)) e = -2;  // bad id: reported by the count kernel
    expert[s] = e;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int prior = 0;
    if (e >= 0) prior = wcnt[warp * p.E + e];
    local[s] = prior + __popc(peers & lt_mask);
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) wcnt[warp * p.E + e] = prior + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < p.E; e += kSlotThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kSlotWarps; ++w) {
      const int v = wcnt[w * p.E + e];
      wcnt[w * p.E + e] = run;
      run += v;
    }
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < kStepsPerWarp; ++s) {
    const int e = expert[s];
    if (e == -1) continue;
    const int64_t a = a_warp + s * 32 + lane;
    const int64_t r = a / p.T, t = a - r * p.T;
    if (e < 0) { p.slot[t * p.k + r] = -1; continue; }
    const int pos = p.chunk_cnt[(int64_t)e * nchunk + blockIdx.x] + wcnt[warp * p.E + e] + local[s];
    if (p.gates != nullptr && p.expert_count[e] > p.capacity) {
      // over-full expert under the "probs" policy: list it for the select kernel
      const int64_t li = (int64_t)p.cum[e] + pos;
      p.list_key[li] = to_ordered(p.gates[t * p.k + r]);
      p.list_idx[li] = (uint32_t)(t * p.k + r);
      continue;
    }
    const bool kept = p.capacity < 0 || pos < p.capacity;
    p.slot[t * p.k + r] = kept ? pos : -1;
    const int64_t row = (int64_t)p.expert_offset[e] + pos;
    if (kept && row < p.rows_max) p.row_token[row] = (int)t;
  }
}

// One CTA per expert; only experts with more than C assignments do work.  An
// expert's list (keys and slot indices) is staged in shared memory when it fits
// (kSelSmemElems); otherwise it is read from global memory.
constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelSmemElems = 24576;         // 192 KB of (key, index) pairs

__global__ void __launch_bounds__(kSelThreads) slot_select_kernel(SlotParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint32_t sbuf[];           // [kSelSmemElems] keys, then [kSelSmemElems] indices
  __shared__ int hist[256];
  __shared__ int sh[kSelWarps];
  __shared__ uint32_t s_prefix;
  __shared__ int s_need;
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n = p.expert_count[e];
  if ((int64_t)n <= p.capacity) return;
  const int64_t base = p.cum[e];
  const bool staged = n <= kSelSmemElems;
  if (staged) {
    for (int i = tid; i < n; i += kSelThreads) {
      sbuf[i] = p.list_key[base + i];
      sbuf[kSelSmemElems + i] = p.list_idx[base + i];
    }
    __syncthreads();
  }
  const uint32_t* key = staged ? sbuf : p.list_key + base;
  const uint32_t* idx = staged ? sbuf + kSelSmemElems : p.list_idx + base;

  // radix select: after the four 8-bit passes, `prefix` is the C-th largest key
  // and `need` is how many of the keys equal to it are kept (the earliest ones)
  uint32_t prefix = 0u, mask = 0u;
  int need = (int)p.capacity;
  if (need <= 0) prefix = 0xffffffffu;         // nothing is kept (C = 0 cannot arise with T*k > 0)
  for (int shift = 24; shift >= 0 && need > 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = 0; i0 < n; i0 += kSelThreads) {   // warp-uniform trip count for match_any
      const int i = i0 + tid;
      const uint32_t kv = i < n ? key[i] : 0u;
      const int bin = (i < n && (kv & mask) == prefix) ? (int)((kv >> shift) & 255u) : -1;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (bin >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (warp == 0) {
      // lane l holds bins 255-8l .. 248-8l (descending); find where the count from
      // the top reaches `need`
      int loc[8], s = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { loc[j] = hist[255 - (8 * lane + j)]; s += loc[j]; }
      int incl = s;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const int excl = incl - s;
      if (excl < need && need <= incl) {
        int run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run < need && need <= run + loc[j]) {
            s_prefix = prefix | ((uint32_t)(255 - (8 * lane + j)) << shift);
            s_need = need - run;
          }
          run += loc[j];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    mask |= 255u << shift;
    __syncthreads();
  }

  // ordered pass.  Kept = every key above the threshold and the first `need`
  // keys equal to it, so the kept elements before position i number
  // gt_before(i) + min(eq_before(i), need).  Warp w owns a contiguous segment of
  // the arrival order: one block scan of the warps' (eq, gt) totals, then each
  // warp walks its segment with ballots, free of block barriers.
  const int seg = ((n + kSelWarps - 1) / kSelWarps + 31) & ~31;
  const int s0 = min(n, warp * seg), s1 = min(n, s0 + seg);
  int my_eq = 0, my_gt = 0;
  for (int i = s0 + lane; i < s1; i += 32) {
    const uint32_t kv = key[i];
    my_eq += kv == prefix;
    my_gt += kv > prefix;
  }
  my_eq = __reduce_add_sync(0xffffffffu, my_eq);
  my_gt = __reduce_add_sync(0xffffffffu, my_gt);
  int tot;
  // only lane 0 carries its warp's totals, so the exclusive prefix at lane 0 is
  // the warp's base
  int eq_before = __shfl_sync(0xffffffffu, block_scan_excl<kSelWarps>(lane == 0 ? my_eq : 0, sh, tot), 0);
  int gt_before = __shfl_sync(0xffffffffu, block_scan_excl<kSelWarps>(lane == 0 ? my_gt : 0, sh, tot), 0);
  const int64_t off = p.expert_offset[e];
  const unsigned lt = (1u << lane) - 1u;
  for (int i0 = s0; i0 < s1; i0 += 32) {
    const int i = i0 + lane;
    const bool valid = i < s1;
    const uint32_t kv = valid ? key[i] : 0u;
    const unsigned beq = __ballot_sync(0xffffffffu, valid && kv == prefix);
    const unsigned bgt = __ballot_sync(0xffffffffu, valid && kv > prefix);
    if (valid) {
      const int eqb = eq_before + __popc(beq & lt), gtb = gt_before + __popc(bgt & lt);
      const bool keep = kv > prefix || (kv == prefix && eqb < need);
      const int rank = gtb + min(eqb, need);
      const uint32_t flat = idx[i];                // t * k + r
      p.slot[flat] = keep ? rank : -1;
      if (keep && off + rank < p.rows_max) p.row_token[off + rank] = (int)(flat / (uint32_t)p.k);
    }
    eq_before += __popc(beq);
    gt_before += __popc(bgt);
  }
}

// ---------------------------------------------------------------- one launch
// The same assignment in one launch, for the "position" policy and dropless
// layers whose assignments fit one resident CTA per SM at kFuseSpan each.
//   phase 1: CTA c ranks its span warp by warp (match_any, as the rank kernel
//            does) and publishes its per-expert totals at chunk_cnt[e][c]; its
//            warps also sum the router's partials of the experts it owns
//            (e = c, c + G, ...: a warp each);
//   grid barrier;
//   phase 2: the owner warp of expert e scans chunk_cnt[e][*] in place into the
//            spans' bases and writes the expert's count, kept count and aux term;
//   grid barrier;
//   (with E * G <= kFuseSmallTotals every CTA instead reads all span totals
//   after the first barrier and adds up those before its span and all of
//   them, and the second barrier goes);
//   phase 3: every CTA reads its base and the kept count of every expert, lays
//            out the 128-padded row blocks (the same scan in every CTA) and
//            writes its slots and row_token entries; the owner CTAs write the
//            padding rows, every CTA a share of the shared block, and CTA 0 the
//            offsets and the aux loss.
// The grid barriers are one counter with bounded waits.  Every CTA is resident
// at once: the grid is at most one CTA per SM and no CTA waits on a later
// kernel.  Slots, counts, offsets and row_token equal the three-kernel path's
// bit for bit (integers); the aux loss is summed in this path's own fixed order.
constexpr int kFuseSteps = 4;                                  // 32-assignment steps per warp
constexpr int kFuseSpan = kSlotWarps * 32 * kFuseSteps;        // assignments per CTA
constexpr int kFuseMaxPer = 5;                                 // chunk counts per lane in the scan (G <= 160)
constexpr int kFuseSmallTotals = 4096;                         // E * G read by every CTA on the one-barrier path

// Thread 0 of each CTA: arrive at grid barrier number `n` (1, 2, ...) and wait
// until all G CTAs have arrived (bounded; false and MOE_ETIMEOUT in the status
// word if the wait runs out).
__device__ __forceinline__ bool slot_grid_barrier(unsigned* ctr, unsigned G, unsigned n, DevStatus* st) {
  __threadfence();
  atomicAdd(ctr, 1u);
  const long long t0 = clock64();
  unsigned v = 0;
  while (true) {
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
    if (v >= n * G) return true;
    if (clock64() - t0 > kWaitCycles) {
      set_status(st, MOE_ETIMEOUT, 3);
      return false;
    }
    __nanosleep(64);
  }
}

__global__ void __launch_bounds__(kSlotThreads) slot_fused_kernel(SlotParams p, int G) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int fsm[];
  const int E = p.E;
  int* wcnt = fsm;                          // [warps][E]: counts, then exclusive prefixes over the warps
  int* s_base = wcnt + kSlotWarps * E;      // [E] this span's base per expert
  int* s_kept = s_base + E;                 // [E]
  int* s_tot = s_kept + E;                  // [E] (one-barrier path)
  int* s_off = s_tot + E;                   // [E + 2]
  __shared__ int sh[kSlotWarps];
  __shared__ double red[kSlotWarps];
  __shared__ int s_ok;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, c = blockIdx.x;
  const int64_t A = p.T * p.k;
  const bool aux = p.aux != nullptr;
  for (int i = tid; i < kSlotWarps * E; i += kSlotThreads) wcnt[i] = 0;
  for (int i = tid; i < E; i += kSlotThreads) {
    s_base[i] = 0;
    s_tot[i] = 0;
  }
  __syncthreads();

  // phase 1: ranks inside each warp's 128 assignments (in sequence order)
  const int64_t a_warp = (int64_t)c * kFuseSpan + (int64_t)warp * (kFuseSteps * 32);
  const unsigned lt_mask = (1u << lane) - 1u;
  int local[kFuseSteps], expert[kFuseSteps];
#pragma unroll
  for (int s = 0; s < kFuseSteps; ++s) {
    const int64_t a = a_warp + s * 32 + lane;
    int e = load_assignment(p, a, A);          // -1 past the end
    if (a < A && (e < 0 || e >= E)) {
      if (e != -1) set_status(p.status, MOE_EDEVICE, 1);   // -1: a choice that is not dispatched
      e = -2;
    }
    expert[s] = e;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    int prior = 0;
    if (e >= 0) prior = wcnt[warp * E + e];
    local[s] = prior + __popc(peers & lt_mask);
    __syncwarp();
    if (e >= 0 && lane == __ffs(peers) - 1) wcnt[warp * E + e] = prior + __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int e = tid; e < E; e += kSlotThreads) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < kSlotWarps; ++w) {
      const int v = wcnt[w * E + e];
      wcnt[w * E + e] = run;
      run += v;
    }
    __stcg(p.chunk_cnt + (int64_t)e * G + c, run);
  }
  if (aux) {
    // P_e / T of the experts this CTA owns (and, with selection counts, the
    // whole term f_e * P_e): lanes stride the router's partial rows in fp64
    // (rows between the strided ones hold zeros), then a fixed butterfly
    const int rs = p.part_stride > 1 ? p.part_stride : 1;
    for (int e = c + G * warp; e < E; e += G * kSlotWarps) {
      double ps = 0.0;
      long long cs = 0;
#pragma unroll 4
      for (int b = lane * rs; b < p.nblk_router; b += 32 * rs) {
        ps += (double)__ldcg(p.psum_part + (int64_t)b * E + e);
        if (p.cnt_part != nullptr) cs += __ldcg(p.cnt_part + (int64_t)b * E + e);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        ps += __shfl_xor_sync(0xffffffffu, ps, o);
        cs += __shfl_xor_sync(0xffffffffu, cs, o);
      }
      const double pt = ps / (double)p.T;
      if (lane == 0) __stcg(p.aux_term + e, p.cnt_part != nullptr ? ((double)cs / ((double)p.T * p.k)) * pt : pt);
    }
    if (c == 0 && warp == kSlotWarps - 1 && p.zsum_part != nullptr) {
      // z-loss = coef * mean_t lse_t^2 from the router's per-block sums
      double z = 0.0;
      for (int b = lane * rs; b < p.nblk_router; b += 32 * rs) z += (double)__ldcg(p.zsum_part + b);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
      if (lane == 0) p.aux[1] = (float)((double)p.z_coef * z / (double)p.T);
    }
  }
  // with few span totals (E * G <= kFuseSmallTotals) every CTA reads them all
  // after the first barrier, and the second barrier is not needed
  const bool one = (int64_t)E * G <= kFuseSmallTotals;
  __syncthreads();
  if (tid == 0) {
    s_ok = slot_grid_barrier(p.ticket, (unsigned)G, 1u, p.status) ? 1 : 0;
    // the last CTA to leave re-arms the counter for the next call
    if (one && s_ok && atomicAdd(p.ticket, 1u) == 2u * G - 1u) atomicExch(p.ticket, 0u);
  }
  __syncthreads();
  if (!s_ok) return;

  if (one) {
    // all E * G span totals at once (coalesced, one round trip), added into this
    // span's bases (spans before it) and the experts' totals with integer
    // shared-memory atomics (zeroed in phase 1; any order gives the same sums)
    constexpr int kPerThread = kFuseSmallTotals / kSlotThreads;
    const int n = E * G;
    int v[kPerThread];
#pragma unroll
    for (int m = 0; m < kPerThread; ++m) {
      const int idx = m * kSlotThreads + tid;
      v[m] = idx < n ? __ldcg(p.chunk_cnt + idx) : 0;
    }
#pragma unroll
    for (int m = 0; m < kPerThread; ++m) {
      const int idx = m * kSlotThreads + tid;
      if (idx < n && v[m] != 0) {
        const int e = idx / G, j = idx - e * G;
        atomicAdd(s_tot + e, v[m]);
        if (j < c) atomicAdd(s_base + e, v[m]);
      }
    }
    __syncthreads();
    for (int e = tid; e < E; e += kSlotThreads) {
      const int all = s_tot[e];
      const int kept = p.capacity < 0 ? all : (int)min((int64_t)all, p.capacity);
      s_kept[e] = kept;
      if (c == 0) {
        p.expert_count[e] = all;
        p.kept_count[e] = kept;
      }
    }
  } else {
  // phase 2: the owner warp scans expert e's span totals into bases, in place;
  // lane l holds the contiguous entries [l * per, (l + 1) * per)
  {
    const int per = (G + 31) / 32;
    for (int e = c + G * warp; e < E; e += G * kSlotWarps) {
      int* row = p.chunk_cnt + (int64_t)e * G;
      int v[kFuseMaxPer];
      int mine = 0;
#pragma unroll
      for (int i = 0; i < kFuseMaxPer; ++i) {
        const int j = lane * per + i;
        v[i] = (i < per && j < G) ? __ldcg(row + j) : 0;
        mine += v[i];
      }
      int incl = mine;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      int run = incl - mine;
#pragma unroll
      for (int i = 0; i < kFuseMaxPer; ++i) {
        const int j = lane * per + i;
        if (i < per && j < G) __stcg(row + j, run);
        run += v[i];
      }
      const int tot = __shfl_sync(0xffffffffu, incl, 31);
      if (lane == 0) {
        const int kept = p.capacity < 0 ? tot : (int)min((int64_t)tot, p.capacity);
        p.expert_count[e] = tot;
        __stcg(p.kept_count + e, kept);
        if (aux && p.T > 0 && p.cnt_part == nullptr)
          __stcg(p.aux_term + e, ((double)tot / ((double)p.T * p.k)) * __ldcg(p.aux_term + e));
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    s_ok = slot_grid_barrier(p.ticket, (unsigned)G, 2u, p.status) ? 1 : 0;
    // the last CTA to leave re-arms the counter for the next call
    if (s_ok && atomicAdd(p.ticket, 1u) == 3u * G - 1u) atomicExch(p.ticket, 0u);
  }
  __syncthreads();
  if (!s_ok) return;

  // phase 3: this span's bases, every expert's kept count, the row blocks
  for (int e = tid; e < E; e += kSlotThreads) {
    s_base[e] = __ldcg(p.chunk_cnt + (int64_t)e * G + c);
    s_kept[e] = __ldcg(p.kept_count + e);
  }
  }
  __syncthreads();
  {
    constexpr int kPer = (kMaxE + kSlotThreads - 1) / kSlotThreads;   // experts per thread, contiguous
    const int e0 = tid * kPer;
    int loc = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (e0 + i < E) loc += (int)round_up(s_kept[e0 + i], kRowPad);
    int routed;
    int run = block_scan_excl<kSlotWarps>(loc, sh, routed);
#pragma unroll
    for (int i = 0; i < kPer; ++i)
      if (e0 + i < E) {
        s_off[e0 + i] = run;
        run += (int)round_up(s_kept[e0 + i], kRowPad);
      }
    if (tid == 0) {
      s_off[E] = routed;
      const int64_t end = routed + (p.n_shared ? round_up(p.T, kRowPad) : 0);
      s_off[E + 1] = (int)end;
      if (c == 0 && end > p.rows_max) set_status(p.status, MOE_EDEVICE, 2);
    }
  }
  __syncthreads();
#pragma unroll
  for (int s = 0; s < kFuseSteps; ++s) {
    const int e = expert[s];
    if (e == -1) continue;
    const int64_t a = a_warp + s * 32 + lane;
    const int64_t r = a / p.T, t = a - r * p.T;
    if (e < 0) { p.slot[t * p.k + r] = -1; continue; }
    const int pos = s_base[e] + wcnt[warp * E + e] + local[s];
    const bool kept = p.capacity < 0 || pos < p.capacity;
    p.slot[t * p.k + r] = kept ? pos : -1;
    const int64_t row = (int64_t)s_off[e] + pos;
    if (kept && row < p.rows_max) p.row_token[row] = (int)t;
  }
  // padding rows of the experts this CTA owns -> -1; a share of the shared block
  for (int e = c + G * warp; e < E; e += G * kSlotWarps) {
    const int start = s_off[e] + s_kept[e], stop = s_off[e + 1];
    for (int r = start + lane; r < stop; r += 32) p.row_token[r] = -1;
  }
  if (p.n_shared) {
    const int64_t s0 = s_off[E], n = round_up(p.T, kRowPad);
    for (int64_t i = (int64_t)c * kSlotThreads + tid; i < n; i += (int64_t)G * kSlotThreads)
      if (s0 + i < p.rows_max) p.row_token[s0 + i] = i < p.T ? (int)i : -1;
  }
  if (c != 0) return;
  for (int i = tid; i < E + 2; i += kSlotThreads) p.expert_offset[i] = s_off[i];
  if (aux) {
    // aux loss = alpha * E * sum_e f_e * P_e: thread-strided sums in expert
    // order, a fixed butterfly per warp, then the warps in order
    double v = 0.0;
    if (p.T > 0)
      for (int e = tid; e < E; e += kSlotThreads) {
        // the whole term, or P_e / T still to be scaled by f_e (one-barrier path)
        const double pt = __ldcg(p.aux_term + e);
        v += (one && p.cnt_part == nullptr) ? ((double)s_tot[e] / ((double)p.T * p.k)) * pt : pt;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (tid == 0) {
      double s = 0.0;
#pragma unroll
      for (int w = 0; w < kSlotWarps; ++w) s += red[w];
      p.aux[0] = (float)((double)p.aux_alpha * (double)E * s);
    }
  }
}

// The one-launch path applies when every CTA can be resident at once (one per
// SM at most) and no "probs" lists are needed.
static int fused_slot_grid(const SlotParams& p) {
  const int64_t A = p.T * p.k;
  if (A <= 0 || p.gates != nullptr) return 0;
  const int64_t G = (A + kFuseSpan - 1) / kFuseSpan;
  if (G > sm_count() || G > 32 * kFuseMaxPer) return 0;
  return (int)G;
}

cudaError_t launch_slots(const SlotParams& p, cudaStream_t stream) {
  const int64_t A = p.T * p.k;
  if (const int G = fused_slot_grid(p)) {
    const size_t sm = ((size_t)(kSlotWarps + 4) * p.E + 2) * sizeof(int);   // wcnt, base, kept, tot, off
    cudaError_t e = ensure_smem(slot_fused_kernel, sm);
    if (e != cudaSuccess) return e;
    launch_pdl(slot_fused_kernel, G, kSlotThreads, sm, stream, p, G);
    return cudaGetLastError();
  }
  const int nchunk = (int)((A + kSlotChunk - 1) / kSlotChunk);
  if (A > 0) launch_pdl(slot_count_kernel, nchunk, kSlotThreads, p.E * sizeof(int), stream, p, nchunk);
  // one CTA per expert; the last one to finish lays out the row blocks
  launch_pdl(slot_scan_kernel, p.E, kSlotThreads, 0, stream, p, nchunk);
  if (A > 0) {
    const size_t sm = (size_t)kSlotWarps * p.E * sizeof(int);
    cudaError_t e = ensure_smem(slot_rank_kernel, sm);
    if (e != cudaSuccess) return e;
    launch_pdl(slot_rank_kernel, nchunk, kSlotThreads, sm, stream, p, nchunk);
    if (p.gates != nullptr) {
      const size_t ssm = 2 * sizeof(uint32_t) * kSelSmemElems;
      e = ensure_smem(slot_select_kernel, ssm);
      if (e != cudaSuccess) return e;
      launch_pdl(slot_select_kernel, p.E, kSelThreads, ssm, stream, p);
    }
  }
  return cudaGetLastError();
}

}  // namespace moe
