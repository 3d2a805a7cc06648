/*
 * moe_b200.h — C ABI of the B200 (sm_100a) forward pass of one
 * Mixture-of-Experts FFN layer on a single GPU.
 *
 * The pass: router (fp32 logits, softmax, top-k, optional renormalisation),
 * capacity-slot assignment ("position" policy, or dropless with each expert's
 * rows padded to a multiple of 128), dispatch permutation into per-expert row
 * blocks, grouped expert FFN, gate-weighted combine, and the Switch
 * load-balancing loss.  The two all-to-alls of the multi-device method are
 * replaced by a local permutation; the dense one-hot [T,E,C] dispatch mask is
 * never built.
 *
 * Sources, cited by page title and section:
 *   [EP]     "Expert-parallel MoE training" explainer (blog.vllbc.top):
 *            router, capacity, drop/pad, aux-loss and shared-expert sections,
 *            worked examples "capacity overflow" and "parameter and dispatch bytes".
 *   [DS7508] "The MoE spends too much time on the gate network" (DeepSpeed
 *            discussion 7508): k>2 capacity, dense [T,E,C] mask, cost that must
 *            follow real tokens rather than capacity.
 *   [SWITCH] "Switch Routing — MoE Routing, Communication, and Stability":
 *            2.1 routing math, load balance & capacity; 2.2 selective precision.
 *   [WIDEEP] InferenceX v2 "WideEP" note: 256 routed + 1 shared expert, top-8.
 *
 * Conventions for every entry point below:
 *   - Pointers named x, wg, ids, ... are DEVICE pointers owned by the caller;
 *     `cfg` and `w` point to HOST structs read during the call only.
 *   - The library never allocates device memory.  Scratch lives in a caller
 *     workspace of moe_workspace_size() bytes, 256-byte aligned, zero-filled
 *     before its first use (the calls leave the parts that must start at zero,
 *     the status word and the kernels' tickets, at zero).
 *   - Every compute call is asynchronous on `stream` and never synchronises.
 *     The return value reports host-side validation and launch errors only;
 *     errors found on the device (a bad expert id, an exhausted wait) are
 *     written to a status word in the workspace and read by moe_sync_status().
 *   - Inputs are read-only; no output may alias an input.
 *   - Row-major layouts throughout.  Matrices of expert weights are stored the
 *     way a linear layer stores them, [out_features, in_features].
 *   - ids, slot, expert_count, kept_count, expert_offset and row_token are
 *     deterministic: identical inputs give bitwise identical outputs.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* moe_stream_t;   /* a cudaStream_t; NULL = legacy default stream */
typedef struct CUevent_st* moe_event_t;     /* a cudaEvent_t */

/* Status codes. */
enum {
  MOE_OK = 0,
  MOE_EINVAL = 1,        /* null pointer or inconsistent configuration (before any launch) */
  MOE_EUNSUPPORTED = 2,  /* valid but outside this build's limits (see moe_cfg) */
  MOE_ECUDA = 3,         /* a CUDA launch or runtime call failed */
  MOE_ETIMEOUT = 4,      /* device: a bounded wait inside a kernel ran out */
  MOE_EDEVICE = 5,       /* device: an index check failed (e.g. expert id outside [0,E)) */
  MOE_EWORKSPACE = 6     /* workspace smaller than moe_workspace_size() */
};

enum { MOE_ACT_RELU = 0, MOE_ACT_GELU = 1, MOE_ACT_SWIGLU = 2 };
/* SOFTMAX_TOPK: gates are full-softmax probabilities of the selected experts
 * ([SWITCH] 2.1), optionally renormalised over the k selected.
 * TOPK_SOFTMAX: softmax over the k selected logits only ([EP] router section,
 * Megatron pre_softmax=False).
 * SIGMOID_TOPK: gates are sigmoid(logit) of the selected experts ([EP] router
 * section: sigmoid instead of softmax), optionally renormalised over the k
 * selected; the aux loss's P_i then averages the sigmoids divided by their sum
 * over the E experts.  Every score selects the k largest logits. */
enum { MOE_SCORE_SOFTMAX_TOPK = 0, MOE_SCORE_TOPK_SOFTMAX = 1, MOE_SCORE_SIGMOID_TOPK = 2 };
/* CAPACITY: C = ceil(T*k*cf/E) slots per expert, overflow dropped ([EP]
 * capacity and drop/pad sections; [DS7508]).  DROPLESS: every assignment kept
 * (MegaBlocks as summarised in [EP]). */
enum { MOE_CAP_CAPACITY = 0, MOE_CAP_DROPLESS = 1 };
/* Which assignments an over-full expert drops in MOE_CAP_CAPACITY mode ([EP]
 * drop/pad section, Megatron-Core moe_token_drop_policy).  POSITION: the
 * latest in (choice rank, token) order.  PROBS: the lowest gates; each expert
 * keeps its C largest gates (fp32 comparison), equal gates keep the earlier
 * assignment, and kept assignments take slots in (choice rank, token) order. */
enum { MOE_DROP_POSITION = 0, MOE_DROP_PROBS = 1 };
/* Element type of x, expert weights, dispatch buffers and y.  The router
 * weight, logits, gates and the aux loss are always fp32 ([SWITCH] 2.2). */
enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 };
/* moe_cfg.flags
 * KEEP_LOGITS: moe_layer_fwd also stores fp32 logits in the workspace.
 * TRAINING (bf16): moe_layer_fwd keeps everything
 *   moe_layer_bwd needs in the workspace (logits, dispatched rows with zeroed
 *   padding rows, activations, un-gated expert rows; it runs unfused), and
 *   moe_workspace_size includes the backward pass's buffers.
 * PACKED_WEIGHTS (bf16 only): every pointer of moe_weights is a packed buffer
 *   written by moe_pack_weight (see there); results are bitwise the same.
 * PACKED_ROUTER (bf16 only): the `wg` argument of moe_route and moe_layer_fwd
 *   points to the router planes written by moe_pack_router_weight instead of
 *   the fp32 [E,H] weight (which those calls otherwise split into the same
 *   planes on every call); results are bitwise the same.  moe_layer_bwd still
 *   takes the fp32 weight.
 * UNFUSED: moe_layer_fwd runs dispatch and combine as separate kernels (the
 *   pages' literal sequence, filling xbuf and ybuf).  Without it, a bf16 layer
 *   with T*k <= 256*E (at most two 128-row blocks per expert on average, where
 *   the expert contractions stream weights from HBM) runs fused: the first
 *   expert contraction gathers its rows straight from x (xbuf is not written)
 *   and, for k == 1 without a shared expert, the second contraction writes
 *   gate * row to y[token] and zeroes the rows of fully dropped tokens (ybuf's
 *   routed rows are not written).  Larger layers run the separate kernels.
 *   moe_layer_bwd with UNFUSED computes and stores dh, then dz, in two kernels
 *   (default for T*k <= 256*E or H <= 512: one kernel, dh kept on chip); results are
 *   bitwise the same.
 * RANDOM_SECOND: GShard top-2 ([EP] router section: the second expert receives
 *   the token at random, according to its weight).  For k >= 2 the rank-1
 *   choice of token t is dispatched iff uniform[t] < 2 * gate[t,1], with
 *   uniform [T] fp32 in [0,1) supplied by the caller; otherwise its id becomes
 *   -1 and its gate 0 (it takes no slot and adds nothing to y).  The aux loss
 *   still counts it as selected.  No effect when k == 1. */
enum {
  MOE_FLAG_KEEP_LOGITS = 1,
  MOE_FLAG_RANDOM_SECOND = 2,
  MOE_FLAG_UNFUSED = 4,
  MOE_FLAG_PACKED_WEIGHTS = 8,
  MOE_FLAG_TRAINING = 16,
  MOE_FLAG_PACKED_ROUTER = 32
};

/* Layer configuration.  Limits of this build: 1 <= E <= 1024, 1 <= k <= min(E,16),
 * H and F multiples of 8, n_shared in {0,1}, T >= 0 with T*k < 2^31 and every
 * row count below 2^31.  bf16 uses the tcgen05 tensor-core expert FFN; fp32 uses
 * an fp32 SIMT expert FFN. */
typedef struct moe_cfg {
  int64_t T;             /* tokens */
  int32_t H;             /* hidden size */
  int32_t F;             /* expert FFN inner size */
  int32_t E;             /* routed experts */
  int32_t k;             /* experts per token */
  int32_t n_shared;      /* 0 or 1 always-on shared expert ([EP] shared-expert paragraph; [WIDEEP]) */
  int32_t act;           /* MOE_ACT_* */
  int32_t score;         /* MOE_SCORE_* */
  int32_t renorm;        /* 1: divide SOFTMAX_TOPK gates by their sum over the k selected */
  int32_t cap_mode;      /* MOE_CAP_* */
  int32_t dtype;         /* MOE_DTYPE_* */
  int64_t cf_num;        /* capacity factor cf = cf_num / cf_den (exact) */
  int64_t cf_den;
  int64_t min_capacity;  /* lower clamp of C (DeepSpeed min_capacity), 0 = none */
  float aux_alpha;       /* alpha of the load-balancing loss ([SWITCH] 2.1: 1e-2) */
  int32_t flags;         /* MOE_FLAG_* */
  float z_coef;          /* router z-loss coefficient ([EP] aux-loss section), >= 0; 0 = no z-loss */
  int32_t drop_policy;   /* MOE_DROP_* (ignored when dropless) */
} moe_cfg;

/* Expert weights (device pointers, element type cfg->dtype).
 *   w1  [E, F, H]  W_in transposed (ReLU/GELU) or W_gate transposed (SwiGLU)
 *   w3  [E, F, H]  W_up transposed (SwiGLU only, else NULL)
 *   w2  [E, H, F]  W_out / W_down transposed
 *   sw1, sw3, sw2  the shared expert's matrices with the same shapes and E=1
 *                  (NULL when n_shared == 0). */
typedef struct moe_weights {
  const void* w1;
  const void* w3;
  const void* w2;
  const void* sw1;
  const void* sw3;
  const void* sw2;
} moe_weights;

/* Device pointers into a workspace after moe_layer_fwd (see moe_workspace_views). */
typedef struct moe_ws_views {
  int32_t* ids;            /* [T,k] selected experts, rank order (largest logit first) */
  float* gates;            /* [T,k] gate of each selection */
  int32_t* slot;           /* [T,k] position in the expert's slots, -1 = dropped */
  int32_t* expert_count;   /* [E] dispatched choices per expert before the capacity drop */
  int32_t* kept_count;     /* [E] kept assignments per expert */
  int32_t* expert_offset;  /* [E+2] first row of each expert's block; [E] shared block; [E+1] end */
  int32_t* row_token;      /* [rows_max] source token of each row, -1 for padding rows */
  float* logits;           /* [T,E] fp32 logits (written only with MOE_FLAG_KEEP_LOGITS) */
  void* xbuf;              /* [rows_max, H] dispatched rows (moe_layer_fwd: MOE_FLAG_UNFUSED or fp32 only) */
  void* hbuf;              /* [rows_max, F] expert activations (bf16; fp32 for MOE_DTYPE_F32) */
  void* ybuf;              /* [rows_max, H] un-gated expert outputs (routed rows not written by a fused top-1 combine) */
  int64_t rows_max;
  /* MOE_FLAG_TRAINING only (else NULL), after moe_layer_bwd: */
  float* dgate;            /* [T,k] gradient of each gate (0 for choices that add nothing to y) */
  float* dlogits;          /* [T,E] gradient of the router logits */
  void* dyrow;             /* [rows_max, H] gate-weighted output gradient of every row (bf16) */
  void* dh;                /* [rows_max, F] gradient of the activations (written with MOE_FLAG_UNFUSED only) */
  void* dz;                /* [rows_max, F] gradient of the pre-activations ([rows_max, 2*round_up(F,64)] for SwiGLU) */
  void* dxrow;             /* [rows_max, H] input gradient of every row */
} moe_ws_views;

/* ---- sizing (host only, no CUDA calls) ------------------------------------ */

/* Capacity C of cfg ([EP] capacity section: ceil((T*k/E)*cf), evaluated exactly
 * in integers; [DS7508]'s ceil((T/E)*cf*k) is the same number), clamped below by
 * min_capacity.  Writes -1 for MOE_CAP_DROPLESS.  Returns MOE_EINVAL on a bad cfg. */
MOE_API int moe_capacity(const moe_cfg* cfg, int64_t* capacity);

/* Upper bound on the number of rows of the per-expert buffers (xbuf, hbuf, ybuf):
 * every expert block padded to 128 rows plus the shared block.  */
MOE_API int moe_rows_max(const moe_cfg* cfg, int64_t* rows_max);

/* Bytes of workspace needed by moe_layer_fwd; the same workspace serves every
 * per-stage entry point.  O(T*k + rows_max*(2H+F) + E*blocks) bytes: never the
 * T*E*C of a dense dispatch mask. */
MOE_API int moe_workspace_size(const moe_cfg* cfg, size_t* bytes);

/* Device pointers of the workspace regions (host arithmetic on `ws` only). */
MOE_API int moe_workspace_views(const moe_cfg* cfg, void* ws, moe_ws_views* views);

/* ---- stages ---------------------------------------------------------------- */

/* Router ([EP] router section; [SWITCH] 2.1, 2.2).
 *   x [T,H] (cfg->dtype), wg [E,H] fp32 (one row per expert), logit_add [T,E] fp32
 *   or NULL (an additive offset on the logits, e.g. for synthetic load skew),
 *   uniform [T] fp32 in [0,1): the random draws of MOE_FLAG_RANDOM_SECOND
 *   (required with that flag and k >= 2, else ignored and may be NULL).
 *   logits[t,e] = sum_h x[t,h]*wg[e,h] (+ logit_add) accumulated in fp32;
 *   p = softmax(logits[t,:]) (normalised sigmoids for SIGMOID_TOPK); top-k on
 *   the logits (ties to the lower index); gates per cfg->score / cfg->renorm.
 * Writes ids [T,k] int32 (-1: a second choice not dispatched), gates [T,k]
 * fp32, logits_out [T,E] fp32 if non-NULL, and per-block sums of p, selection
 * counts and, when cfg->z_coef != 0, squared log-sum-exps into `ws` for
 * moe_aux_loss.
 * bf16 x: the logits come from the tensor cores, with wg split into three bf16
 * planes whose sum is wg exactly (so every product is exact and the sum is
 * accumulated in fp32); for E <= 256 the same launch also routes the tokens.
 * With MOE_FLAG_PACKED_ROUTER, wg points to planes from moe_pack_router_weight. */
MOE_API int moe_route(const moe_cfg* cfg, const void* x, const float* wg, const float* logit_add,
                      const float* uniform, int32_t* ids, float* gates, float* logits_out, void* ws,
                      moe_stream_t stream);

/* Same as moe_route after the logits: takes fp32 logits [T,E] (so routing can be
 * reproduced bit-exactly from given logits). */
MOE_API int moe_route_from_logits(const moe_cfg* cfg, const float* logits, const float* uniform, int32_t* ids,
                                  float* gates, void* ws, moe_stream_t stream);

/* Slot assignment ([EP] drop/pad section; [DS7508] without the [T,E,C] mask).
 * Assignments are ordered by (choice rank, token).  "position" policy: an
 * assignment's slot is the number of earlier assignments of its expert and it
 * is kept iff slot < C (always, when dropless).  "probs" policy
 * (cfg->drop_policy, capacity mode): gates [T,k] fp32 decide which C
 * assignments an over-full expert keeps (see MOE_DROP_PROBS); gates may be NULL
 * otherwise.  Outputs: slot [T,k] (-1 dropped),
 * expert_count [E] (pre-drop), kept_count [E], expert_offset [E+2] (expert e owns
 * rows [off[e], off[e]+kept[e]) of a 128-row-padded block; the shared block
 * [off[E], off[E]+T) follows; off[E+1] = rows used), row_token [rows_max]
 * (-1 on padding rows).  An id of -1 is a choice that is not dispatched: it
 * takes no slot and gets slot -1.  Other ids outside [0,E) set MOE_EDEVICE. */
MOE_API int moe_assign_slots(const moe_cfg* cfg, const int32_t* ids, const float* gates, int32_t* slot,
                             int32_t* expert_count, int32_t* kept_count, int32_t* expert_offset, int32_t* row_token,
                             void* ws, moe_stream_t stream);

/* moe_assign_slots ("position" policy only: MOE_DROP_PROBS in capacity mode
 * returns MOE_EUNSUPPORTED) for callers that cannot allocate device memory.  No source
 * page has a counterpart: this is a deployment variant.  Some callers get
 * only their input and output buffers and may not allocate anything else, for
 * example a plugin inside a framework whose memory pool owns the whole device,
 * or a latency-critical path where an allocation (and the synchronisation it
 * can imply) is not allowed.  This entry point takes no workspace and calls no
 * allocator; it computes exactly what moe_assign_slots computes (same
 * arguments, same outputs, same kernels).
 * Scratch: a fixed 1 MiB device array inside the library, held by every GPU that
 * loads the library until the process exits.  It fits E * ceil(T*k/256) <=
 * 262080 (e.g. E=256 with T*k up to 262,080 assignments); larger configurations
 * return MOE_EUNSUPPORTED before any launch.
 * All calls on a device share that array and it keeps the last call's contents;
 * the call clears the part that must start at zero.  Calls whose work
 * overlaps on the GPU (concurrent streams) race on the array: order them.
 * The first call on each device looks up the array's device address (with that
 * device current), and so does the first call in each later context of the
 * device (after cudaDeviceReset the module, and the array, are loaded again);
 * make that first call before any stream capture.  An expert
 * id outside [0,E) gives slot -1 for that assignment; this variant has no
 * status word for the caller to read. */
MOE_API int moe_assign_slots_static(const moe_cfg* cfg, const int32_t* ids, int32_t* slot, int32_t* expert_count,
                                    int32_t* kept_count, int32_t* expert_offset, int32_t* row_token,
                                    moe_stream_t stream);

/* Dispatch permutation (the local replacement of the dispatch all-to-all, [EP]):
 * xbuf[off[e]+slot[t,r], :] = x[t, :] for every kept (t,r).  Padding rows are not
 * written.  xbuf has rows_max rows. */
MOE_API int moe_dispatch(const moe_cfg* cfg, const void* x, const int32_t* ids, const int32_t* slot,
                 const int32_t* expert_offset, void* xbuf, moe_stream_t stream);

/* Grouped expert FFN over the variable per-expert row blocks ([EP] experts and
 * worked example 2; SwiGLU = silu(x W_gate) * (x W_up) then W_down).  For every
 * 128-row block of every expert: ybuf = act(xbuf W_in) W_out with fp32
 * accumulation and the activation rounded once to cfg->dtype.  The shared
 * expert's block reads its rows straight from x (NULL when n_shared == 0).
 * Padding rows of ybuf hold unspecified values. */
MOE_API int moe_expert_ffn(const moe_cfg* cfg, const void* xbuf, const void* x, const int32_t* expert_offset,
                   const moe_weights* w, void* ybuf, void* ws, moe_stream_t stream);

/* Gate-weighted combine (the local replacement of the combine all-to-all, [EP];
 * [SWITCH] 2.1 y = p_i(x) E_i(x)): y[t] = sum_{r kept} gates[t,r]*ybuf[row(t,r)]
 * (+ ybuf[off[E]+t] with weight 1 for the shared expert), fp32 accumulation,
 * one rounding.  A fully dropped token gets y[t] = 0: the residual is the
 * caller's ([EP] drop/pad section; [SWITCH] overflow bypass). */
MOE_API int moe_combine(const moe_cfg* cfg, const void* ybuf, const int32_t* ids, const int32_t* slot,
                const float* gates, const int32_t* expert_offset, void* y, moe_stream_t stream);

/* Switch load-balancing loss ([SWITCH] 2.1; [EP] aux-loss section):
 * aux = alpha * E * sum_i f_i * P_i, f_i = pre-drop selections of i / (T*k),
 * P_i = mean_t p_i(t).  With cfg->z_coef != 0 also the router z-loss ([EP]
 * aux-loss section): aux[1] = z_coef * mean_t logsumexp(logits[t,:])^2.
 * Reads the partials left in `ws` by the last moe_route / moe_route_from_logits
 * with the same cfg; writes aux[0] (and aux[1]) fp32 on the device. */
MOE_API int moe_aux_loss(const moe_cfg* cfg, const void* ws, float* aux, moe_stream_t stream);

/* The whole layer: route -> assign slots -> dispatch -> expert FFN -> combine,
 * plus the aux loss, on `stream` (dispatch and the top-1 combine fused into the
 * expert contractions unless MOE_FLAG_UNFUSED; see the flags).  y [T,H] (cfg->dtype) and aux (one fp32, two
 * with the z-loss: see moe_aux_loss) are device outputs; uniform is moe_route's;
 * expert_count [E] (optional, NULL to skip) counts dispatched choices.  The
 * intermediates stay in `ws` (see moe_workspace_views).  `stage_events`, if
 * non-NULL, is an array of MOE_N_STAGE_EVENTS events recorded on `stream` before
 * the router and after each of: router, slots (which here also reduce the aux
 * loss), dispatch (an empty interval when fused), expert FFN first contraction
 * (with the activation), expert FFN second contraction, combine (an empty
 * interval when fused), and the end of the call (the copy of expert_count, if
 * requested). */
enum { MOE_N_STAGE_EVENTS = 8 };
MOE_API int moe_layer_fwd(const moe_cfg* cfg, const void* x, const float* wg, const float* logit_add,
                          const float* uniform, const moe_weights* w, void* y, float* aux, int32_t* expert_count,
                          void* ws, size_t ws_bytes, const moe_event_t* stage_events, moe_stream_t stream);

/* The activation exactly as the expert-FFN epilogues evaluate it, on n fp32
 * values (device pointers): out = relu(z) or gelu(z) = 0.5 z (1 + erf(z/sqrt 2))
 * with erf from Abramowitz & Stegun formula 7.1.26 (|error| <= 1.5e-7), or for
 * MOE_ACT_SWIGLU out = silu(z) * u.  Exposed so the approximation can be
 * checked against its error bound. */
MOE_API int moe_activation_eval(int act, const float* z, const float* u, float* out, int64_t n, moe_stream_t stream);

/* Expert weights in the grouped GEMM's block layout.  No source page has a
 * counterpart: this is weight preprocessing, done once per weight.  The
 * contractions read weights in boxes of 128 rows x 64 k; in the linear-layer
 * layout a box is 128 pieces of 128 bytes K*2 bytes apart, which HBM serves at
 * a fraction of its streaming rate.  Packed, each box is one contiguous 16 KB
 * block: P[g][n/128][k/64][n%128][k%64], zero-padded to whole blocks.
 *   moe_packed_weight_bytes: bytes of the packed form of a [G, N, K] bf16 matrix.
 *   moe_pack_weight: w [G, N, K] bf16 (device, K % 8 == 0) -> packed (device,
 *   moe_packed_weight_bytes bytes, 16-byte aligned), asynchronous on `stream`.
 * Pack w1 and w3 as [E, F, H], w2 as [E, H, F], the shared matrices with G = 1,
 * then set MOE_FLAG_PACKED_WEIGHTS. */
MOE_API int moe_packed_weight_bytes(int32_t G, int32_t N, int32_t K, size_t* bytes);
MOE_API int moe_pack_weight(const void* w, int32_t G, int32_t N, int32_t K, void* packed, moe_stream_t stream);

/* One-time split of the fp32 router weight for the tensor-core router ([SWITCH]
 * 2.2: the router computes in fp32).  Each element w of wg [E,H] (device, fp32)
 * becomes three bf16 values hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi -
 * mid) with hi + mid + lo = w exactly, stored in `planes` (device, 16-byte
 * aligned, moe_router_planes_bytes bytes) as [E][3][Hp], Hp = H rounded up to
 * 64, zero-padded.  Pass `planes` as wg with MOE_FLAG_PACKED_ROUTER.
 * Asynchronous on `stream`.  Errors: MOE_EINVAL (NULL, misaligned, E or H < 1),
 * MOE_EUNSUPPORTED (E > 1024 or H % 8 != 0), MOE_ECUDA. */
MOE_API int moe_router_planes_bytes(int32_t E, int32_t H, size_t* bytes);
MOE_API int moe_pack_router_weight(const float* wg, int32_t E, int32_t H, void* planes, moe_stream_t stream);

/* Gradients of the expert weights (device pointers, fp32, the shapes of
 * moe_weights: dw1/dw3 [E,F,H], dw2 [E,H,F], shared [1,...]; NULL where absent). */
typedef struct moe_weight_grads {
  float* dw1;
  float* dw3;
  float* dw2;
  float* dsw1;
  float* dsw3;
  float* dsw2;
} moe_weight_grads;

/* Backward pass of the layer ([EP]: the backward runs the forward's
 * permutations with their roles swapped; the aux loss is differentiable only
 * through P_i; the z-loss acts on the logits; [SWITCH] 2.1 y = p_i E_i).
 * Requires the workspace of a moe_layer_fwd call with MOE_FLAG_TRAINING on the
 * same cfg, x, wg and w, untouched since.  Discrete decisions (top-k, random
 * second dispatch, capacity) are constants.  Upstream gradients: dy [T,H]
 * (bf16) of y, and scalars d_aux, d_z of the aux loss and the z-loss (1 when
 * both are added to the loss).  Outputs (device, overwritten): dx [T,H] bf16,
 * dwg [E,H] fp32, and the expert weight gradients in `dw` (fp32).
 * Kernels: combine backward (gate-weighted rows of dy, gate gradients), the
 * second contraction's data and weight gradients, the first contraction
 * recomputed with the activation's derivative applied (no pre-activations are
 * stored), its data and weight gradients, the router backward, the dispatch
 * backward (tokens sum their rows, plus dlogits Wg), and dWg = dlogits^T x.
 * When T*k <= 256*E (the weight-streaming regime, as for the forward's fusion)
 * or H <= 512, dh and dz come from one kernel (dz = bf16(dh) * act'(z), dh
 * not stored: ws views' dh is left unwritten); otherwise, or with
 * MOE_FLAG_UNFUSED, two kernels compute and store dh, then dz.  Results are
 * bitwise the same.
 * `stage_events`, if non-NULL, is an array of MOE_N_BWD_STAGE_EVENTS events
 * recorded on `stream` before the first kernel and after each of: combine
 * backward (with the zeroing of padding rows), dh (fused: dh and dz), dW2, dz
 * (fused: an empty interval), dW1/dW3, router backward, the rows' input
 * gradients, dispatch backward, dWg.
 * With MOE_FLAG_PACKED_WEIGHTS the data-gradient contractions read the packed
 * blocks (the weight gradients are always written in the linear-layer layout);
 * results are bitwise the same.
 * Ownership: every buffer is the caller's; nothing is allocated.  Gradients are
 * written, not accumulated (add them into a master copy to accumulate).
 * Asynchronous on `stream`; deterministic (fixed reduction orders).
 * Errors: MOE_EUNSUPPORTED for fp32 layers; MOE_EINVAL for a bad cfg, a cfg
 * without MOE_FLAG_TRAINING, a NULL input/output or a missing weight gradient
 * (dw3 for SwiGLU, the shared ones with n_shared); MOE_EWORKSPACE when ws_bytes
 * is below moe_workspace_size of the training cfg; MOE_ECUDA for a launch
 * failure.  Bounded in-kernel waits that run out report MOE_ETIMEOUT through
 * moe_sync_status. */
enum { MOE_N_BWD_STAGE_EVENTS = 10 };
MOE_API int moe_layer_bwd(const moe_cfg* cfg, const void* x, const float* wg, const moe_weights* w, const void* dy,
                          float d_aux, float d_z, void* dx, float* dwg, const moe_weight_grads* dw, void* ws,
                          size_t ws_bytes, const moe_event_t* stage_events, moe_stream_t stream);

/* ---- status ---------------------------------------------------------------- */

/* Synchronises `stream`, returns the device status word of `ws` (MOE_OK,
 * MOE_ETIMEOUT or MOE_EDEVICE) and clears it.  MOE_ECUDA if the sync fails. */
MOE_API int moe_sync_status(void* ws, moe_stream_t stream);

/* Clears the device status word of `ws` (asynchronously on `stream`). */
MOE_API int moe_clear_status(void* ws, moe_stream_t stream);

/* Self-check of the device-side failure detection (no page counterpart: it
 * exercises this library's bounded waits).  Launches one tiny kernel on
 * `stream` whose warp waits on an mbarrier that nothing arrives at, with the
 * same bounded-wait routine every tensor-core kernel here uses, limited to
 * `limit_cycles` SM clock cycles (0 .. about 1 s worth, the kernels' own limit).
 * With abort_after_cycles >= 0 a second warp raises the CTA's abort flag after
 * that many cycles and the wait must end through the flag instead.  Either way
 * the kernel records MOE_ETIMEOUT in the status word at the start of `ws` (any
 * workspace of at least 256 bytes) and returns: read it with moe_sync_status.
 * *waited_cycles (DEVICE pointer to one int64) receives the cycles the wait
 * lasted.  No copy or MMA is in flight when the wait gives up, so the context
 * stays usable.  Errors: MOE_EINVAL for NULL pointers or limits above the
 * kernels' own; MOE_ECUDA for a launch failure. */
MOE_API int moe_selftest_bounded_wait(int64_t limit_cycles, int64_t abort_after_cycles, int64_t* waited_cycles,
                                      void* ws, moe_stream_t stream);

/* Static description of a status code. */
MOE_API const char* moe_strerror(int status);

/* Version string of the library build. */
MOE_API const char* moe_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H */
