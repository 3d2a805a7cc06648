// Internal launch interface between the C ABI (moe_abi.cu) and the kernels.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {

struct RouterParams {
  const void* x;            // [T,H] bf16 or fp32 (unused when logits_in is set)
  const float* wg;          // [E,H]
  const float* logit_add;   // [T,E] or null
  const float* logits_in;   // [T,E] or null: skip the GEMM, route these logits
  int logits_parts;         // logits_in holds this many [T,E] partials to add in order (1 or 3)
  int32_t* ids;             // [T,k]
  float* gates;             // [T,k]
  float* logits_out;        // [T,E] or null
  float* psum_part;         // [nblk,E]
  int32_t* cnt_part;        // [nblk,E]
  unsigned* aux_counter;    // ticket counter of the aux-loss kernel (re-armed here)
  float* zsum_part;         // [nblk] per-CTA sums of lse^2 (z-loss), or null
  const float* uniform;     // [T] GShard random second dispatch, or null
  int64_t T;
  int H, E, k, score, renorm;
};
int router_tile_tokens(int E);
// bf16 x: fp32 router logits [T,E] on the tensor cores from three bf16 planes
// of Wg (hi + mid + lo = Wg exactly), laid out [E][3][router_plane_width(H)].
int router_plane_width(int H);
cudaError_t launch_split_router_weight(const float* wg, void* planes, int E, int H, cudaStream_t stream);
// `planes` holds the planes already (planes_ready) or receives them from wg.
// `logits` holds 3*T*E floats; *parts (1 or 2) is how many fp32 partial [T,E]
// arrays were written (their sum, in order, is the logits).  With `route`
// (E <= 256) the same launch also routes every token (ids, gates, partial sums
// in rows of 32 tokens, nblk rows) and *routed is set: no launch_router needed.
cudaError_t launch_router_gemm(const void* x, const float* wg, void* planes, bool planes_ready, float* logits,
                               int64_t T, int H, int E, DevStatus* status, const RouterParams* route, int64_t nblk,
                               int* parts, bool* routed, cudaStream_t stream);
cudaError_t launch_router(const RouterParams& p, bool bf16, cudaStream_t stream);
// Routers with E <= 256 and T >= 256: logits and routing on pairs of SMs from
// precomputed planes (router_pair.cu).
bool router_pair_fits(int64_t T, int H, int E);
cudaError_t launch_router_pair(const void* x, const void* planes, int64_t T, int H, int E, DevStatus* status,
                               const RouterParams& route, int64_t nblk, cudaStream_t stream);
// term: E doubles of scratch followed by one unsigned ticket counter.
// zsum_part (or null): per-CTA sums of lse^2; aux[1] = z_coef * their mean.
cudaError_t launch_aux(const float* psum_part, const int32_t* cnt_part, const float* zsum_part, int nblk, int E,
                       int64_t T, int k, float alpha, float z_coef, double* term, float* aux, cudaStream_t stream);
// Router backward: dlogits [T,E] from dgate [T,k], the aux loss (through P_i,
// fcoef[e] = d_aux * alpha * E * f_e / T, computed here from cnt_part) and the
// z-loss (zc = d_z * z_coef).
struct RouterBwdParams {
  const float* logits;      // [T,E] the forward's
  const float* dgate;       // [T,k]
  const float* fcoef;       // [E]
  float* dlogits;           // [T,E]
  int64_t T;
  int E, k, score, renorm;
  float zc;
};
cudaError_t launch_router_bwd(const RouterBwdParams& p, const int32_t* cnt_part, int nblk, float d_aux_alpha,
                              float* fcoef, cudaStream_t stream);

// Backward permutations (backward.cu).
struct CombineBwdParams {
  const __nv_bfloat16* dy;  // [T,H]
  const __nv_bfloat16* ybuf;// [rows,H] the forward's un-gated expert rows
  const int32_t* ids;
  const int32_t* slot;
  const float* gates;
  const int32_t* off;
  __nv_bfloat16* dyrow;     // [rows,H]
  float* dgate;             // [T,k]
  int64_t T, rows_max;
  int H, E, k, n_shared;
};
cudaError_t launch_combine_bwd(const CombineBwdParams& p, cudaStream_t stream);
struct DispatchBwdParams {
  const __nv_bfloat16* dxrow;   // [rows,H]
  const float* dlogits;         // [T,E]
  const float* wg;              // [E,H]
  const int32_t* ids;
  const int32_t* slot;
  const int32_t* off;
  __nv_bfloat16* dx;            // [T,H]
  int64_t T, rows_max;
  int H, E, k, n_shared;
};
cudaError_t launch_dispatch_bwd(const DispatchBwdParams& p, cudaStream_t stream);
cudaError_t launch_zero_pad_rows(void* buf, int width, const int32_t* row_token, const int32_t* off, int ngroups,
                                 int64_t rows_max, cudaStream_t stream);
int dwg_chunks(int64_t T, int E, int H);
// dwg [E,H] = dlogits^T x (part: dwg_chunks(T, E, H) * E * H floats of scratch)
cudaError_t launch_router_wgrad(const float* dlogits, const void* x, int64_t T, int E, int H, float* part,
                                float* dwg, cudaStream_t stream);

// Evaluates the GEMM epilogue's activation: out = act(z) (ReLU, GELU) or silu(z) * u (SwiGLU).
cudaError_t launch_activation_eval(int act, const float* z, const float* u, float* out, int64_t n,
                                   cudaStream_t stream);

struct SlotParams {
  const int32_t* ids;       // [T,k]
  int32_t* slot;            // [T,k]
  int32_t* expert_count;    // [E]
  int32_t* kept_count;      // [E]
  int32_t* expert_offset;   // [E+2]
  int32_t* row_token;       // [rows_max]
  int32_t* chunk_cnt;       // [E, nchunk] scratch
  int64_t T;
  int E, k, n_shared;
  int64_t capacity;         // < 0: dropless
  int64_t rows_max;
  DevStatus* status;
  // optional aux loss (fused layer path): router partial sums of p, one fp64 term
  // per expert, and the output scalar
  const float* psum_part;   // [nblk_router, E] or null
  const int32_t* cnt_part;  // [nblk_router, E] selection counts, or null: count the dispatched ids
  int nblk_router;
  int part_stride;          // only every part_stride-th partial row is non-zero (0 or 1: all)
  double* aux_term;         // [E]
  float* aux;               // [1], or [2] with the z-loss in aux[1]
  float aux_alpha;
  const float* zsum_part;   // [nblk_router] router sums of lse^2, or null: no z-loss
  float z_coef;
  // "probs" drop policy (capacity mode only): experts with more assignments than
  // C keep the C largest gates.  Their assignments are listed in arrival order at
  // list_*[cum[e] .. cum[e] + count[e]) and resolved by a per-expert select.
  const float* gates;       // [T,k] or null: "position" policy
  int32_t* cum;             // [E] exclusive prefix of expert_count
  uint32_t* list_key;       // [T*k] order-preserving gate keys
  uint32_t* list_idx;       // [T*k] the assignment's flat index t*k + r
  unsigned* ticket;         // zero between calls: counts the count kernel's finished CTAs
};
constexpr int kSlotChunk = 256;    // assignments per CTA of the slot kernels (one per thread)
cudaError_t launch_slots(const SlotParams& p, cudaStream_t stream);

struct PermuteParams {
  const void* src;          // dispatch: x [T,H]; combine: ybuf [rows,H]
  void* dst;                // dispatch: xbuf [rows,H]; combine: y [T,H]
  const int32_t* ids;
  const int32_t* slot;
  const float* gates;
  const int32_t* expert_offset;
  int64_t T, rows_max;
  int H, E, k, n_shared;
  int elem_bytes;           // 2 (bf16) or 4 (fp32)
};
cudaError_t launch_dispatch(const PermuteParams& p, cudaStream_t stream);
cudaError_t launch_combine(const PermuteParams& p, cudaStream_t stream);

// fp32 SIMT grouped FFN (one GEMM per call).
struct FfnF32Params {
  const float* a_routed;    // [rows_max, K]
  const float* a_shared;    // [T, K], or null: the shared block's rows sit in a_routed in place
  const float* b0;          // routed [E, N, K]
  const float* b1;          // SwiGLU up [E, N, K] or null
  const float* sb0;         // shared [1, N, K] or null
  const float* sb1;
  float* d;                 // [rows_max, N]
  const int32_t* expert_offset;
  int64_t T, rows_max;
  int K, N, E, n_shared, epi;  // epi: -1 none, else MOE_ACT_*
};
cudaError_t launch_ffn_f32(const FfnF32Params& p, cudaStream_t stream);

// tcgen05 grouped GEMM (bf16 in, fp32 accumulate in TMEM, bf16 out).
struct GemmParams {
  const void* a_routed;     // [rows_max, K] bf16
  const void* a_shared;     // [T, K] bf16, or null: the shared block's rows sit in a_routed in place
  const void* b0;           // routed [E, Nw, K] (W_in^T, W_gate^T or W_out^T)
  const void* b1;           // routed SwiGLU up [E, Nw, K] or null
  const void* sb0;          // shared [1, Nw, K] or null
  const void* sb1;
  void* d;                  // [rows_max, N_out] bf16
  const int32_t* expert_offset;   // [E+2]
  int64_t T, rows_max;
  int K, Nw, E, n_shared, epi;    // epi: -1 none, else MOE_ACT_*
  DevStatus* status;
  // Fused dispatch: routed A rows are gathered from gather_src [T, K] by
  // gather_idx (row_token; -1 = padding row, read as zeros); a_routed unused.
  const void* gather_src;
  const int32_t* gather_idx;
  // Fused top-1 combine: routed output rows go to scatter_dst[token] scaled by
  // scatter_gate[token] instead of d (no shared expert, k = 1); rows of tokens
  // with scatter_slot[token] < 0 (dropped) are zeroed by the same launch.
  void* scatter_dst;
  const float* scatter_gate;
  const int32_t* scatter_slot;
  int b_packed;             // 1: b0/b1/sb0/sb1 are packed (launch_pack_weight)
  // Pairs of SMs (tcgen05 cta_group::2, 256 output features x up to 256
  // tokens, tokens on the MMA's N) instead of one SM per 128 x 256 tile: for
  // compute-bound layers, without gather or scatter.  pair_prefix: ngroups + 1
  // ints of scratch for the groups' token-tile prefix, computed by this launch
  // unless pair_prefix_ready (same offsets and valid_rows as the launch that
  // computed it).  valid_rows: rows of each routed group that carry tokens
  // (kept counts, [E]), or null: whole 128-row blocks; the shared block has T.
  int two_sm;
  int32_t* pair_prefix;
  int pair_prefix_ready;
  const int32_t* valid_rows;
};
cudaError_t launch_grouped_gemm(const GemmParams& p, cudaStream_t stream);
cudaError_t launch_grouped_gemm_tn(const GemmParams& p, cudaStream_t stream);

// Grouped GEMMs of the backward pass (grouped_gemm_bwd.cu).
//   dgrad: out[rows, N] = a[rows, K] * B, B the weights [G, K0, N] read along N
//          (k blocks >= k_switch from b1: SwiGLU's [W1; W3]); shared rows use sb0/sb1.
//   dact:  out = dz[rows, ld] from z = a[rows, K] * b0^T (and the up projection
//          b1 for SwiGLU, ld = 2 round_up(N, 64), db at column ld / 2) and dh[rows, N].
//   wgrad: per expert g, w_out[g] = a[rows_g, M]^T * b0[rows_g, N] (fp32); output rows
//          >= m_split go to w_out2 (m_valid rows each); the shared block to w_sh / w_sh2,
//          its b rows from b_shared (row - off[E]) when given.
struct BwdGemm {
  const void* a;
  const void* a_shared;     // dact: the shared block's A rows (x), or null
  const void* b0;
  const void* b1;
  const void* sb0;
  const void* sb1;
  const void* b_shared;     // wgrad: the shared block's B rows (x), or null
  void* out;                // dgrad / dact: bf16 output
  const void* dh;           // dact
  float *w_out, *w_out2, *w_sh, *w_sh2;
  const int32_t* off;
  DevStatus* status;
  int64_t T, rows_max;
  int K, K0, N, M, E, n_shared, act, k_switch, m_split, m_valid;
  int b_packed;             // dgrad / dact / dhz: weights in the packed block layout
  const void* a2;           // dhz: dyrow (A of the dh pass)
  const void* v;            // dhz: W2 [E, K, N] (B of the dh pass, read along N)
  const void* sv;           // dhz: the shared expert's W2, or null
  int wg_deep;              // wgrad: four-stage ring, fp32 stored as 32 x 16 blocks (experts with many rows)
};
cudaError_t launch_bwd_dgrad(const BwdGemm& q, cudaStream_t stream);
cudaError_t launch_bwd_dact(const BwdGemm& q, cudaStream_t stream);
cudaError_t launch_bwd_wgrad(const BwdGemm& q, cudaStream_t stream);
// dz = bf16(dyrow W2) * act'(x_rows W1^T) in one kernel (dh is not stored)
cudaError_t launch_bwd_dhz(const BwdGemm& q, cudaStream_t stream);
// dgrad on pairs of SMs (grouped_gemm_tn.cu), for layers with T*k > 256*E:
// the same product as launch_bwd_dgrad, computed for each group's kept rows
// rounded up to 16 (valid: the routed groups' kept counts; pair_prefix:
// ngroups + 1 ints of scratch).  Rows past them in each 128-row block are not
// written.
cudaError_t launch_bwd_dgrad_pair(const BwdGemm& q, int32_t* pair_prefix, const int32_t* valid,
                                  cudaStream_t stream);
// dact on pairs of SMs (grouped_gemm_tn.cu), same rows as launch_bwd_dgrad_pair;
// dz [rows_max, dz_ld], SwiGLU's db at column dz_ld / 2.
cudaError_t launch_bwd_dact_pair(const BwdGemm& q, int dz_ld, int32_t* pair_prefix, const int32_t* valid,
                                 cudaStream_t stream);
// wgrad on pairs of SMs (grouped_gemm_tn.cu): the same outputs as
// launch_bwd_wgrad, over each group's kept rows (valid) in 64-row blocks.
cudaError_t launch_bwd_wgrad_pair(const BwdGemm& q, const int32_t* valid, cudaStream_t stream);

// Packed weight layout for the grouped GEMM: w [G, N, K] bf16 (K contiguous) ->
// [G][ceil(N/128)][ceil(K/64)][128][64], zero-padded, so every TMA box of 128
// rows x 64 k is one contiguous 16 KB block.
size_t packed_weight_bytes(int G, int N, int K);
cudaError_t launch_pack_weight(const void* w, int G, int N, int K, void* packed, cudaStream_t stream);

}  // namespace moe
