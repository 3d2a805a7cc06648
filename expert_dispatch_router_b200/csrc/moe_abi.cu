// Host side of the C ABI declared in include/moe_b200.h: validation, the exact
// capacity, the row bound, the workspace layout, and the stage launches.
// Nothing here allocates device memory or synchronises (moe_sync_status
// excepted, which exists to do exactly that).
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

constexpr int64_t kMaxCf = int64_t(1) << 20;

struct Layout {
  size_t status, psum, cnt, zsum, term, chunk, cum, lkey, lidx, ids, gates, slot, ecount, kept, off, pairs, rowtok,
      logits, lparts, planes, xbuf,
      hbuf, ybuf, dyrow, dh, dz, dxrow, dgate, dlog, fcoef, dwgp;
  size_t total;
  int nblk_router, nchunk;
  int64_t rows_max;
};

bool valid_cfg(const moe_cfg* c) {
  if (c == nullptr) return false;
  if (c->T < 0 || c->E < 1 || c->k < 1 || c->H < 1 || c->F < 1) return false;
  if (c->k > c->E) return false;
  if (c->n_shared != 0 && c->n_shared != 1) return false;
  if (c->act < MOE_ACT_RELU || c->act > MOE_ACT_SWIGLU) return false;
  if (c->score < MOE_SCORE_SOFTMAX_TOPK || c->score > MOE_SCORE_SIGMOID_TOPK) return false;
  if (c->renorm != 0 && c->renorm != 1) return false;
  if (c->cap_mode != MOE_CAP_CAPACITY && c->cap_mode != MOE_CAP_DROPLESS) return false;
  if (c->dtype != MOE_DTYPE_F32 && c->dtype != MOE_DTYPE_BF16) return false;
  if (c->cap_mode == MOE_CAP_CAPACITY && (c->cf_num <= 0 || c->cf_den <= 0)) return false;
  if (c->min_capacity < 0) return false;
  if (!(c->z_coef >= 0.0f) || isinf(c->z_coef)) return false;
  if (c->flags & ~(MOE_FLAG_KEEP_LOGITS | MOE_FLAG_RANDOM_SECOND | MOE_FLAG_UNFUSED | MOE_FLAG_PACKED_WEIGHTS |
                   MOE_FLAG_TRAINING | MOE_FLAG_PACKED_ROUTER))
    return false;
  if ((c->flags & (MOE_FLAG_PACKED_WEIGHTS | MOE_FLAG_PACKED_ROUTER)) && c->dtype != MOE_DTYPE_BF16) return false;
  if (c->drop_policy != MOE_DROP_POSITION && c->drop_policy != MOE_DROP_PROBS) return false;
  return true;
}

// MOE_OK, MOE_EINVAL or MOE_EUNSUPPORTED.
int check_cfg(const moe_cfg* c) {
  if (!valid_cfg(c)) return MOE_EINVAL;
  if (c->E > kMaxE || c->k > kMaxK) return MOE_EUNSUPPORTED;
  if (c->H % 8 != 0 || c->F % 8 != 0) return MOE_EUNSUPPORTED;
  if (c->cap_mode == MOE_CAP_CAPACITY && (c->cf_num > kMaxCf || c->cf_den > kMaxCf)) return MOE_EUNSUPPORTED;
  if (c->T * (int64_t)c->k >= (int64_t(1) << 31)) return MOE_EUNSUPPORTED;
  return MOE_OK;
}

bool training(const moe_cfg* c) { return (c->flags & MOE_FLAG_TRAINING) != 0; }
int dz_width(const moe_cfg* c) {                 // dz row length: F, or da | db with db at round_up(F, 64)
  return c->act == MOE_ACT_SWIGLU ? 2 * ((c->F + 63) / 64 * 64) : c->F;
}

int64_t capacity_of(const moe_cfg* c) {
  if (c->cap_mode == MOE_CAP_DROPLESS) return -1;
  const int64_t num = c->T * c->k * c->cf_num;
  const int64_t den = (int64_t)c->E * c->cf_den;
  int64_t cap = (num + den - 1) / den;              // exact ceiling of the rational T*k*cf/E
  return cap > c->min_capacity ? cap : c->min_capacity;
}

int64_t rows_max_of(const moe_cfg* c) {
  const int64_t A = c->T * c->k;
  const int64_t nonempty = A < c->E ? A : c->E;     // experts that can own a block
  int64_t routed = A + (kRowPad - 1) * nonempty;
  if (c->cap_mode == MOE_CAP_CAPACITY) {
    const int64_t C = capacity_of(c);
    const int64_t kept = A < (int64_t)c->E * C ? A : (int64_t)c->E * C;
    const int64_t b1 = kept + (kRowPad - 1) * nonempty;
    const int64_t b2 = (int64_t)c->E * round_up(C, kRowPad);
    routed = b1 < b2 ? b1 : b2;
  }
  routed = round_up(routed, kRowPad);
  return routed + (c->n_shared ? round_up(c->T, kRowPad) : 0);
}

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

bool drop_probs(const moe_cfg* c) { return c->cap_mode == MOE_CAP_CAPACITY && c->drop_policy == MOE_DROP_PROBS; }

Layout layout_of(const moe_cfg* c) {
  Layout L{};
  const size_t T = (size_t)c->T, E = (size_t)c->E, k = (size_t)c->k;
  const size_t esz = c->dtype == MOE_DTYPE_BF16 ? 2 : 4;
  L.rows_max = rows_max_of(c);
  const int bt = router_tile_tokens(c->E);
  L.nblk_router = (int)((c->T + bt - 1) / bt);
  L.nchunk = (int)((c->T * c->k + kSlotChunk - 1) / kSlotChunk);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + (bytes ? bytes : 1)); return at; };
  L.status = take(sizeof(DevStatus));
  L.psum = take(sizeof(float) * L.nblk_router * E);
  L.cnt = take(sizeof(int32_t) * L.nblk_router * E);
  L.zsum = take(sizeof(float) * L.nblk_router);
  L.term = take(sizeof(double) * (E + 2));      // E terms, the aux ticket counter, the slot ticket
  L.chunk = take(sizeof(int32_t) * E * (size_t)L.nchunk);
  const bool probs = drop_probs(c);
  L.cum = take(probs ? sizeof(int32_t) * E : 0);
  L.lkey = take(probs ? sizeof(uint32_t) * T * k : 0);
  L.lidx = take(probs ? sizeof(uint32_t) * T * k : 0);
  L.ids = take(sizeof(int32_t) * T * k);
  L.gates = take(sizeof(float) * T * k);
  L.slot = take(sizeof(int32_t) * T * k);
  L.ecount = take(sizeof(int32_t) * E);
  L.kept = take(sizeof(int32_t) * E);
  L.off = take(sizeof(int32_t) * (E + 2));
  L.pairs = take(sizeof(int32_t) * (E + 2));
  L.rowtok = take(sizeof(int32_t) * (size_t)L.rows_max);
  const bool tc_router = c->dtype == MOE_DTYPE_BF16;   // bf16 x: router logits on the tensor cores
  L.logits = take(((c->flags & (MOE_FLAG_KEEP_LOGITS | MOE_FLAG_TRAINING)) || tc_router) ? sizeof(float) * T * E : 0);
  L.lparts = take(tc_router ? sizeof(float) * 3 * T * E : 0);   // router GEMM partials
  L.planes = take(tc_router ? sizeof(uint16_t) * E * 3 * (size_t)router_plane_width(c->H) : 0);
  L.xbuf = take(esz * (size_t)L.rows_max * c->H);
  L.hbuf = take(esz * (size_t)L.rows_max * c->F);
  L.ybuf = take(esz * (size_t)L.rows_max * c->H);
  const bool tr = training(c);
  L.dyrow = take(tr ? esz * (size_t)L.rows_max * c->H : 0);
  L.dh = take(tr ? esz * (size_t)L.rows_max * c->F : 0);
  L.dz = take(tr ? esz * (size_t)L.rows_max * dz_width(c) : 0);
  L.dxrow = take(tr ? esz * (size_t)L.rows_max * c->H : 0);
  L.dgate = take(tr ? sizeof(float) * T * k : 0);
  L.dlog = take(tr ? sizeof(float) * T * E : 0);
  L.fcoef = take(tr ? sizeof(float) * E : 0);
  L.dwgp = take(tr ? sizeof(float) * (size_t)dwg_chunks(c->T, E, c->H) * E * c->H : 0);
  L.total = o;
  return L;
}

template <typename P>
P* at(void* ws, size_t off) { return reinterpret_cast<P*>(static_cast<char*>(ws) + off); }

cudaStream_t S(moe_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ECUDA; }

bool random_second(const moe_cfg* c) { return (c->flags & MOE_FLAG_RANDOM_SECOND) && c->k >= 2; }
bool has_zloss(const moe_cfg* c) { return c->z_coef != 0.0f; }

RouterParams router_params(const moe_cfg* c, const Layout& L, void* ws) {
  RouterParams p{};
  p.psum_part = at<float>(ws, L.psum);
  p.cnt_part = at<int32_t>(ws, L.cnt);
  p.aux_counter = reinterpret_cast<unsigned*>(at<double>(ws, L.term) + c->E);
  p.zsum_part = has_zloss(c) ? at<float>(ws, L.zsum) : nullptr;
  p.T = c->T;
  p.H = c->H;
  p.E = c->E;
  p.k = c->k;
  p.score = c->score;
  p.renorm = c->renorm;
  return p;
}

int run_route(const moe_cfg* c, const Layout& L, const void* x, const float* wg, const float* logit_add,
              const float* logits_in, const float* uniform, int32_t* ids, float* gates, float* logits_out, void* ws,
              cudaStream_t s) {
  if (random_second(c) && c->T > 0 && uniform == nullptr) return MOE_EINVAL;
  RouterParams p = router_params(c, L, ws);
  p.uniform = random_second(c) ? uniform : nullptr;
  p.logits_parts = 1;
  p.x = x;
  p.wg = wg;
  p.logit_add = logit_add;
  p.ids = ids;
  p.gates = gates;
  p.logits_out = logits_out;
  if (logits_in == nullptr && c->dtype == MOE_DTYPE_BF16 && c->T > 0) {
    // logits on the tensor cores; for E <= 256 the same launch routes the
    // tokens, otherwise the softmax / top-k / gate kernel runs on the logits.
    // With MOE_FLAG_PACKED_ROUTER, wg already holds the three bf16 planes.
    float* buf = at<float>(ws, L.lparts);
    int parts = 1;
    bool routed = false;
    const bool ready = (c->flags & MOE_FLAG_PACKED_ROUTER) != 0;
    void* planes = ready ? const_cast<float*>(wg) : at<void>(ws, L.planes);
    if (launch_router_gemm(x, wg, planes, ready, buf, c->T, c->H, c->E, at<DevStatus>(ws, L.status), &p,
                           L.nblk_router, &parts, &routed, s) != cudaSuccess)
      return MOE_ECUDA;
    if (routed) return MOE_OK;
    logits_in = buf;
    p.logits_parts = parts;
  }
  p.logits_in = logits_in;
  return cuda_status(launch_router(p, c->dtype == MOE_DTYPE_BF16, s));
}

int run_slots(const moe_cfg* c, const Layout& L, const int32_t* ids, const float* gates, int32_t* slot,
              int32_t* ecount, int32_t* kept, int32_t* off, int32_t* rowtok, void* ws, cudaStream_t s,
              float* aux = nullptr) {
  SlotParams p{};
  if (drop_probs(c)) {
    if (c->T > 0 && gates == nullptr) return MOE_EINVAL;
    p.gates = gates;
    p.cum = at<int32_t>(ws, L.cum);
    p.list_key = at<uint32_t>(ws, L.lkey);
    p.list_idx = at<uint32_t>(ws, L.lidx);
  }
  p.ids = ids;
  p.slot = slot;
  p.expert_count = ecount;
  p.kept_count = kept;
  p.expert_offset = off;
  p.row_token = rowtok;
  p.chunk_cnt = at<int32_t>(ws, L.chunk);
  p.ticket = reinterpret_cast<unsigned*>(at<double>(ws, L.term) + c->E + 1);
  p.T = c->T;
  p.E = c->E;
  p.k = c->k;
  p.n_shared = c->n_shared;
  p.capacity = capacity_of(c);
  p.rows_max = L.rows_max;
  p.status = at<DevStatus>(ws, L.status);
  if (aux != nullptr) {            // fuse the aux loss into the slot kernels
    p.psum_part = at<float>(ws, L.psum);
    p.nblk_router = L.nblk_router;
    // bf16 layers with E <= 256 are routed from the router GEMM's accumulator,
    // 128 tokens a tile: one partial row in every 128 / router_tile_tokens
    // holds the tile's sums and the rows between hold zeros
    p.part_stride = (c->dtype == MOE_DTYPE_BF16 && c->E <= 256) ? 128 / router_tile_tokens(c->E) : 1;
    p.aux_term = at<double>(ws, L.term);
    p.aux = aux;
    p.aux_alpha = c->aux_alpha;
    p.cnt_part = random_second(c) ? at<int32_t>(ws, L.cnt) : nullptr;   // f counts selections, not dispatches
    p.zsum_part = has_zloss(c) ? at<float>(ws, L.zsum) : nullptr;
    p.z_coef = c->z_coef;
  }
  return cuda_status(launch_slots(p, s));
}

PermuteParams permute_params(const moe_cfg* c, const Layout& L) {
  PermuteParams p{};
  p.T = c->T;
  p.rows_max = L.rows_max;
  p.H = c->H;
  p.E = c->E;
  p.k = c->k;
  p.n_shared = c->n_shared;
  p.elem_bytes = c->dtype == MOE_DTYPE_BF16 ? 2 : 4;
  return p;
}

int record(const moe_event_t* ev, int i, cudaStream_t s) {
  if (ev == nullptr) return MOE_OK;
  return cuda_status(cudaEventRecord(reinterpret_cast<cudaEvent_t>(ev[i]), s));
}

// Compute-bound expert contractions (more than two 128-row blocks per expert
// on average) run on pairs of SMs; the others stream their weights and run one
// SM per tile (where dispatch and the top-1 combine can be fused in).
bool two_sm_ffn(const moe_cfg* c) {
  return c->dtype == MOE_DTYPE_BF16 && c->T * c->k > 2 * kRowPad * (int64_t)c->E;
}

// Both contractions of the expert FFN; `ev_mid`, if non-NULL, is recorded between them.
// bf16 only: with `rowtok`, GEMM1 gathers its routed A rows from x (fused
// dispatch; xbuf unused); with `y_top1` as well, GEMM2 writes gate * row to
// y[token] (fused top-1 combine; ybuf's routed rows are not written).  `kept`
// (optional): the routed groups' kept counts, so the SM-pair contractions skip
// the padding rows.
int run_ffn(const moe_cfg* c, const Layout& L, const void* xbuf, const void* x, const int32_t* off,
            const moe_weights* w, void* ybuf, void* ws, cudaStream_t s, const moe_event_t* ev_mid = nullptr,
            const int32_t* rowtok = nullptr, void* y_top1 = nullptr, const float* gates_top1 = nullptr,
            const int32_t* slot_top1 = nullptr, const int32_t* kept = nullptr) {
  void* hbuf = at<void>(ws, L.hbuf);
  const bool sh = c->n_shared != 0;
  if (c->dtype == MOE_DTYPE_BF16) {
    GemmParams g1{};
    g1.a_routed = xbuf;
    g1.a_shared = sh ? x : nullptr;
    g1.b0 = w->w1;
    g1.b1 = c->act == MOE_ACT_SWIGLU ? w->w3 : nullptr;
    g1.sb0 = sh ? w->sw1 : nullptr;
    g1.sb1 = sh && c->act == MOE_ACT_SWIGLU ? w->sw3 : nullptr;
    g1.d = hbuf;
    g1.expert_offset = off;
    g1.T = c->T;
    g1.rows_max = L.rows_max;
    g1.K = c->H;
    g1.Nw = c->F;
    g1.E = c->E;
    g1.n_shared = c->n_shared;
    g1.epi = c->act;
    g1.status = at<DevStatus>(ws, L.status);
    g1.b_packed = (c->flags & MOE_FLAG_PACKED_WEIGHTS) ? 1 : 0;
    g1.two_sm = two_sm_ffn(c) ? 1 : 0;
    g1.pair_prefix = at<int32_t>(ws, L.pairs);
    g1.pair_prefix_ready = 0;
    g1.valid_rows = kept;
    if (rowtok != nullptr) {
      g1.a_routed = nullptr;
      g1.gather_src = x;
      g1.gather_idx = rowtok;
    }
    cudaError_t e = launch_grouped_gemm(g1, s);
    if (e != cudaSuccess) return MOE_ECUDA;
    if (record(ev_mid, 0, s) != MOE_OK) return MOE_ECUDA;
    GemmParams g2 = g1;
    g2.a_routed = hbuf;
    g2.a_shared = nullptr;
    g2.b0 = w->w2;
    g2.b1 = nullptr;
    g2.sb0 = sh ? w->sw2 : nullptr;
    g2.sb1 = nullptr;
    g2.d = ybuf;
    g2.K = c->F;
    g2.Nw = c->H;
    g2.epi = -1;
    g2.gather_src = nullptr;
    g2.gather_idx = nullptr;
    g2.pair_prefix_ready = 1;                   // same offsets as GEMM1
    if (y_top1 != nullptr) {
      g2.gather_idx = rowtok;
      g2.scatter_dst = y_top1;
      g2.scatter_gate = gates_top1;
      g2.scatter_slot = slot_top1;
    }
    return cuda_status(launch_grouped_gemm(g2, s));
  }
  FfnF32Params f1{};
  f1.a_routed = static_cast<const float*>(xbuf);
  f1.a_shared = sh ? static_cast<const float*>(x) : nullptr;
  f1.b0 = static_cast<const float*>(w->w1);
  f1.b1 = c->act == MOE_ACT_SWIGLU ? static_cast<const float*>(w->w3) : nullptr;
  f1.sb0 = sh ? static_cast<const float*>(w->sw1) : nullptr;
  f1.sb1 = sh && c->act == MOE_ACT_SWIGLU ? static_cast<const float*>(w->sw3) : nullptr;
  f1.d = static_cast<float*>(hbuf);
  f1.expert_offset = off;
  f1.T = c->T;
  f1.rows_max = L.rows_max;
  f1.K = c->H;
  f1.N = c->F;
  f1.E = c->E;
  f1.n_shared = c->n_shared;
  f1.epi = c->act;
  cudaError_t e = launch_ffn_f32(f1, s);
  if (e != cudaSuccess) return MOE_ECUDA;
  if (record(ev_mid, 0, s) != MOE_OK) return MOE_ECUDA;
  FfnF32Params f2 = f1;
  f2.a_routed = static_cast<const float*>(hbuf);
  f2.a_shared = nullptr;
  f2.b0 = static_cast<const float*>(w->w2);
  f2.b1 = nullptr;
  f2.sb0 = sh ? static_cast<const float*>(w->sw2) : nullptr;
  f2.sb1 = nullptr;
  f2.d = static_cast<float*>(ybuf);
  f2.K = c->F;
  f2.N = c->H;
  f2.epi = -1;
  return cuda_status(launch_ffn_f32(f2, s));
}

int check_weights(const moe_cfg* c, const moe_weights* w) {
  if (w == nullptr || w->w1 == nullptr || w->w2 == nullptr) return MOE_EINVAL;
  if (c->act == MOE_ACT_SWIGLU && w->w3 == nullptr) return MOE_EINVAL;
  if (c->n_shared) {
    if (w->sw1 == nullptr || w->sw2 == nullptr) return MOE_EINVAL;
    if (c->act == MOE_ACT_SWIGLU && w->sw3 == nullptr) return MOE_EINVAL;
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

int moe_capacity(const moe_cfg* cfg, int64_t* capacity) {
  if (capacity == nullptr) return MOE_EINVAL;
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  *capacity = capacity_of(cfg);
  return MOE_OK;
}

int moe_rows_max(const moe_cfg* cfg, int64_t* rows_max) {
  if (rows_max == nullptr) return MOE_EINVAL;
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  const int64_t r = rows_max_of(cfg);
  if (r >= (int64_t(1) << 31)) return MOE_EUNSUPPORTED;
  *rows_max = r;
  return MOE_OK;
}

int moe_workspace_size(const moe_cfg* cfg, size_t* bytes) {
  if (bytes == nullptr) return MOE_EINVAL;
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (rows_max_of(cfg) >= (int64_t(1) << 31)) return MOE_EUNSUPPORTED;
  *bytes = layout_of(cfg).total;
  return MOE_OK;
}

int moe_workspace_views(const moe_cfg* cfg, void* ws, moe_ws_views* v) {
  if (ws == nullptr || v == nullptr) return MOE_EINVAL;
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  const Layout L = layout_of(cfg);
  v->ids = at<int32_t>(ws, L.ids);
  v->gates = at<float>(ws, L.gates);
  v->slot = at<int32_t>(ws, L.slot);
  v->expert_count = at<int32_t>(ws, L.ecount);
  v->kept_count = at<int32_t>(ws, L.kept);
  v->expert_offset = at<int32_t>(ws, L.off);
  v->row_token = at<int32_t>(ws, L.rowtok);
  v->logits = (cfg->flags & (MOE_FLAG_KEEP_LOGITS | MOE_FLAG_TRAINING)) ? at<float>(ws, L.logits) : nullptr;
  v->xbuf = at<void>(ws, L.xbuf);
  v->hbuf = at<void>(ws, L.hbuf);
  v->ybuf = at<void>(ws, L.ybuf);
  v->rows_max = L.rows_max;
  const bool tr = training(cfg);
  v->dgate = tr ? at<float>(ws, L.dgate) : nullptr;
  v->dlogits = tr ? at<float>(ws, L.dlog) : nullptr;
  v->dyrow = tr ? at<void>(ws, L.dyrow) : nullptr;
  v->dh = tr ? at<void>(ws, L.dh) : nullptr;
  v->dz = tr ? at<void>(ws, L.dz) : nullptr;
  v->dxrow = tr ? at<void>(ws, L.dxrow) : nullptr;
  return MOE_OK;
}

int moe_route(const moe_cfg* cfg, const void* x, const float* wg, const float* logit_add, const float* uniform,
              int32_t* ids, float* gates, float* logits_out, void* ws, moe_stream_t stream) {
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (x == nullptr || wg == nullptr || ids == nullptr || gates == nullptr)) return MOE_EINVAL;
  if (ws == nullptr) return MOE_EINVAL;
  return run_route(cfg, layout_of(cfg), x, wg, logit_add, nullptr, uniform, ids, gates, logits_out, ws, S(stream));
}

int moe_route_from_logits(const moe_cfg* cfg, const float* logits, const float* uniform, int32_t* ids, float* gates,
                          void* ws, moe_stream_t stream) {
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (logits == nullptr || ids == nullptr || gates == nullptr)) return MOE_EINVAL;
  if (ws == nullptr) return MOE_EINVAL;
  return run_route(cfg, layout_of(cfg), nullptr, nullptr, nullptr, logits, uniform, ids, gates, nullptr, ws,
                   S(stream));
}

int moe_assign_slots(const moe_cfg* cfg, const int32_t* ids, const float* gates, int32_t* slot,
                     int32_t* expert_count, int32_t* kept_count, int32_t* expert_offset, int32_t* row_token, void* ws,
                     moe_stream_t stream) {
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (ws == nullptr || expert_count == nullptr || kept_count == nullptr || expert_offset == nullptr) return MOE_EINVAL;
  if (cfg->T > 0 && (ids == nullptr || slot == nullptr || row_token == nullptr)) return MOE_EINVAL;
  return run_slots(cfg, layout_of(cfg), ids, gates, slot, expert_count, kept_count, expert_offset, row_token, ws,
                   S(stream));
}

int moe_dispatch(const moe_cfg* cfg, const void* x, const int32_t* ids, const int32_t* slot,
                 const int32_t* expert_offset, void* xbuf, moe_stream_t stream) {
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (x == nullptr || ids == nullptr || slot == nullptr || expert_offset == nullptr || xbuf == nullptr))
    return MOE_EINVAL;
  PermuteParams p = permute_params(cfg, layout_of(cfg));
  p.src = x;
  p.dst = xbuf;
  p.ids = ids;
  p.slot = slot;
  p.expert_offset = expert_offset;
  return cuda_status(launch_dispatch(p, S(stream)));
}

int moe_expert_ffn(const moe_cfg* cfg, const void* xbuf, const void* x, const int32_t* expert_offset,
                   const moe_weights* w, void* ybuf, void* ws, moe_stream_t stream) {
  int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  st = check_weights(cfg, w);
  if (st != MOE_OK) return st;
  if (xbuf == nullptr || expert_offset == nullptr || ybuf == nullptr || ws == nullptr) return MOE_EINVAL;
  if (cfg->n_shared && x == nullptr) return MOE_EINVAL;
  return run_ffn(cfg, layout_of(cfg), xbuf, x, expert_offset, w, ybuf, ws, S(stream));
}

int moe_combine(const moe_cfg* cfg, const void* ybuf, const int32_t* ids, const int32_t* slot, const float* gates,
                const int32_t* expert_offset, void* y, moe_stream_t stream) {
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (cfg->T > 0 && (ybuf == nullptr || ids == nullptr || slot == nullptr || gates == nullptr ||
                     expert_offset == nullptr || y == nullptr))
    return MOE_EINVAL;
  PermuteParams p = permute_params(cfg, layout_of(cfg));
  p.src = ybuf;
  p.dst = y;
  p.ids = ids;
  p.slot = slot;
  p.gates = gates;
  p.expert_offset = expert_offset;
  return cuda_status(launch_combine(p, S(stream)));
}

int moe_aux_loss(const moe_cfg* cfg, const void* ws, float* aux, moe_stream_t stream) {
  const int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  if (ws == nullptr || aux == nullptr) return MOE_EINVAL;
  const Layout L = layout_of(cfg);
  void* w = const_cast<void*>(ws);
  return cuda_status(launch_aux(at<float>(w, L.psum), at<int32_t>(w, L.cnt),
                                has_zloss(cfg) ? at<float>(w, L.zsum) : nullptr, L.nblk_router, cfg->E, cfg->T,
                                cfg->k, cfg->aux_alpha, cfg->z_coef, at<double>(w, L.term), aux, S(stream)));
}

int moe_layer_fwd(const moe_cfg* cfg, const void* x, const float* wg, const float* logit_add, const float* uniform,
                  const moe_weights* w, void* y, float* aux, int32_t* expert_count, void* ws, size_t ws_bytes,
                  const moe_event_t* stage_events, moe_stream_t stream) {
  int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  st = check_weights(cfg, w);
  if (st != MOE_OK) return st;
  if (ws == nullptr || aux == nullptr) return MOE_EINVAL;
  if (cfg->T > 0 && (x == nullptr || wg == nullptr || y == nullptr)) return MOE_EINVAL;
  if (rows_max_of(cfg) >= (int64_t(1) << 31)) return MOE_EUNSUPPORTED;
  const Layout L = layout_of(cfg);
  if (ws_bytes < L.total) return MOE_EWORKSPACE;
  cudaStream_t s = S(stream);
  int32_t* ids = at<int32_t>(ws, L.ids);
  float* gates = at<float>(ws, L.gates);
  int32_t* slot = at<int32_t>(ws, L.slot);
  int32_t* off = at<int32_t>(ws, L.off);
  void* xbuf = at<void>(ws, L.xbuf);
  void* ybuf = at<void>(ws, L.ybuf);
  float* logits = (cfg->flags & (MOE_FLAG_KEEP_LOGITS | MOE_FLAG_TRAINING)) ? at<float>(ws, L.logits) : nullptr;

  if ((st = record(stage_events, 0, s)) != MOE_OK) return st;
  if ((st = run_route(cfg, L, x, wg, logit_add, nullptr, uniform, ids, gates, logits, ws, s)) != MOE_OK) return st;
  if ((st = record(stage_events, 1, s)) != MOE_OK) return st;
  if ((st = run_slots(cfg, L, ids, gates, slot, at<int32_t>(ws, L.ecount), at<int32_t>(ws, L.kept), off,
                      at<int32_t>(ws, L.rowtok), ws, s, aux)) != MOE_OK)
    return st;
  if ((st = record(stage_events, 2, s)) != MOE_OK) return st;
  // bf16 with at most two 128-row blocks per expert on average: the expert
  // contractions stream weights from HBM, so dispatch is fused into the first
  // one's A loads and, for top-1 without a shared expert, the combine into the
  // second one's epilogue.  With more rows per expert the contractions are fed
  // from L2, where the TMA loads of a dispatched buffer feed faster than
  // per-row cp.async gathers.
  const bool fuse = cfg->dtype == MOE_DTYPE_BF16 && !(cfg->flags & (MOE_FLAG_UNFUSED | MOE_FLAG_TRAINING)) &&
                    cfg->T * cfg->k <= 2 * kRowPad * (int64_t)cfg->E;
  const bool fuse_combine = fuse && cfg->k == 1 && cfg->n_shared == 0;
  int32_t* rowtok = at<int32_t>(ws, L.rowtok);
  PermuteParams pp = permute_params(cfg, L);
  pp.ids = ids;
  pp.slot = slot;
  pp.gates = gates;
  pp.expert_offset = off;
  pp.src = x;
  pp.dst = xbuf;
  if (!fuse && launch_dispatch(pp, s) != cudaSuccess) return MOE_ECUDA;
  // training: padding rows of xbuf are zero (the weight gradients read them)
  if (training(cfg) && launch_zero_pad_rows(xbuf, cfg->H, rowtok, off, cfg->E + (cfg->n_shared ? 1 : 0), L.rows_max,
                                            s) != cudaSuccess)
    return MOE_ECUDA;
  if ((st = record(stage_events, 3, s)) != MOE_OK) return st;
  if ((st = run_ffn(cfg, L, xbuf, x, off, w, ybuf, ws, s, stage_events ? stage_events + 4 : nullptr,
                    fuse ? rowtok : nullptr, fuse_combine ? y : nullptr, fuse_combine ? gates : nullptr,
                    fuse_combine ? slot : nullptr, at<int32_t>(ws, L.kept))) != MOE_OK)
    return st;
  if ((st = record(stage_events, 5, s)) != MOE_OK) return st;
  pp.src = ybuf;
  pp.dst = y;
  if (!fuse_combine && launch_combine(pp, s) != cudaSuccess) return MOE_ECUDA;
  if ((st = record(stage_events, 6, s)) != MOE_OK) return st;
  if (expert_count != nullptr && cfg->E > 0)
    if (cudaMemcpyAsync(expert_count, at<int32_t>(ws, L.ecount), sizeof(int32_t) * cfg->E, cudaMemcpyDeviceToDevice,
                        s) != cudaSuccess)
      return MOE_ECUDA;
  return record(stage_events, 7, s);
}

int moe_layer_bwd(const moe_cfg* cfg, const void* x, const float* wg, const moe_weights* w, const void* dy,
                  float d_aux, float d_z, void* dx, float* dwg, const moe_weight_grads* dw, void* ws, size_t ws_bytes,
                  const moe_event_t* stage_events, moe_stream_t stream) {
  int st = check_cfg(cfg);
  if (st != MOE_OK) return st;
  st = check_weights(cfg, w);
  if (st != MOE_OK) return st;
  if (!training(cfg)) return MOE_EINVAL;
  if (cfg->dtype != MOE_DTYPE_BF16) return MOE_EUNSUPPORTED;
  if (ws == nullptr || dw == nullptr || dwg == nullptr || dw->dw1 == nullptr || dw->dw2 == nullptr) return MOE_EINVAL;
  if (cfg->act == MOE_ACT_SWIGLU && dw->dw3 == nullptr) return MOE_EINVAL;
  if (cfg->n_shared && (dw->dsw1 == nullptr || dw->dsw2 == nullptr ||
                        (cfg->act == MOE_ACT_SWIGLU && dw->dsw3 == nullptr)))
    return MOE_EINVAL;
  if (cfg->T > 0 && (x == nullptr || wg == nullptr || dy == nullptr || dx == nullptr)) return MOE_EINVAL;
  const Layout L = layout_of(cfg);
  if (ws_bytes < L.total) return MOE_EWORKSPACE;
  cudaStream_t s = S(stream);
  const bool sw = cfg->act == MOE_ACT_SWIGLU, sh = cfg->n_shared != 0;
  const int H = cfg->H, F = cfg->F, E = cfg->E;
  const int ngroups = E + (sh ? 1 : 0);
  const int Fp = (F + 63) / 64 * 64;
  const int dzw = dz_width(cfg);
  int32_t* ids = at<int32_t>(ws, L.ids);
  int32_t* slot = at<int32_t>(ws, L.slot);
  int32_t* off = at<int32_t>(ws, L.off);
  int32_t* rowtok = at<int32_t>(ws, L.rowtok);
  DevStatus* status = at<DevStatus>(ws, L.status);
  auto bf = [&](size_t o) { return at<__nv_bfloat16>(ws, o); };

  if ((st = record(stage_events, 0, s)) != MOE_OK) return st;
  // 1. combine backward: gate-weighted rows of dy, gate gradients
  CombineBwdParams cb{};
  cb.dy = static_cast<const __nv_bfloat16*>(dy);
  cb.ybuf = bf(L.ybuf);
  cb.ids = ids;
  cb.slot = slot;
  cb.gates = at<float>(ws, L.gates);
  cb.off = off;
  cb.dyrow = bf(L.dyrow);
  cb.dgate = at<float>(ws, L.dgate);
  cb.T = cfg->T;
  cb.rows_max = L.rows_max;
  cb.H = H;
  cb.E = E;
  cb.k = cfg->k;
  cb.n_shared = cfg->n_shared;
  if (launch_combine_bwd(cb, s) != cudaSuccess) return MOE_ECUDA;
  if (launch_zero_pad_rows(bf(L.dyrow), H, rowtok, off, ngroups, L.rows_max, s) != cudaSuccess) return MOE_ECUDA;
  if ((st = record(stage_events, 1, s)) != MOE_OK) return st;

  BwdGemm q{};
  q.off = off;
  q.status = status;
  q.T = cfg->T;
  q.rows_max = L.rows_max;
  q.E = E;
  q.n_shared = cfg->n_shared;
  q.act = cfg->act;
  const int packed = (cfg->flags & MOE_FLAG_PACKED_WEIGHTS) ? 1 : 0;
  // 2. dh = dyrow W2 (W2 read along F); fused: dz = bf16(dh) * act'(z) straight
  //    away, with z recomputed from the dispatched rows, and dh never stored.
  //    The fused kernel's tiles are narrower (128 or 64 output columns), so it
  //    pays where the contractions stream their weights from HBM (the
  //    forward's rule, T*k <= 256*E: at most two 128-row blocks per expert on
  //    average) or where the contraction over H is short (H <= 512), which
  //    leaves the unfused dz kernel bound by its epilogue.  Otherwise the two
  //    N = 256 kernels run.
  const bool fused = !(cfg->flags & MOE_FLAG_UNFUSED) &&
                     (cfg->T * cfg->k <= 2 * kRowPad * (int64_t)E || H <= 512);
  BwdGemm g = q;
  if (fused) {
    g.a = bf(L.xbuf);
    g.a_shared = sh ? x : nullptr;
    g.b0 = w->w1;
    g.b1 = sw ? w->w3 : nullptr;
    g.sb0 = sh ? w->sw1 : nullptr;
    g.sb1 = sh && sw ? w->sw3 : nullptr;
    g.a2 = bf(L.dyrow);
    g.v = w->w2;
    g.sv = sh ? w->sw2 : nullptr;
    g.out = bf(L.dz);
    g.K = H;
    g.N = F;
    g.b_packed = packed;
    if (launch_bwd_dhz(g, s) != cudaSuccess) return MOE_ECUDA;
  } else {
    g.a = bf(L.dyrow);
    g.b0 = w->w2;
    g.sb0 = sh ? w->sw2 : nullptr;
    g.out = bf(L.dh);
    g.K = H;
    g.K0 = H;
    g.N = F;
    g.b_packed = packed;
    // compute-bound layers (the forward's rule): pairs of SMs, W2 read along F
    const cudaError_t e = two_sm_ffn(cfg) ? launch_bwd_dgrad_pair(g, at<int32_t>(ws, L.pairs), at<int32_t>(ws, L.kept), s)
                                          : launch_bwd_dgrad(g, s);
    if (e != cudaSuccess) return MOE_ECUDA;
  }
  if ((st = record(stage_events, 2, s)) != MOE_OK) return st;
  // 3. dW2 = dyrow^T h per expert.  With at least 192 rows per expert on
  //    average the k loops are long and the fp32 output a small part of the
  //    work: the deep variant (four-stage ring) runs.  With fewer, the output
  //    dominates and the two-stage ring with double-buffered stores runs.
  const int wg_deep = cfg->T * cfg->k >= 192 * (int64_t)E ? 1 : 0;
  g = q;
  g.wg_deep = wg_deep;
  g.a = bf(L.dyrow);
  g.b0 = bf(L.hbuf);
  g.M = H;
  g.N = F;
  g.m_split = H;
  g.m_valid = H;
  g.w_out = dw->dw2;
  g.w_sh = sh ? dw->dsw2 : nullptr;
  // compute-bound layers: pairs of SMs
  if ((two_sm_ffn(cfg) ? launch_bwd_wgrad_pair(g, at<int32_t>(ws, L.kept), s) : launch_bwd_wgrad(g, s)) !=
      cudaSuccess)
    return MOE_ECUDA;
  if ((st = record(stage_events, 3, s)) != MOE_OK) return st;
  // 4. dz = dh * act'(z), z recomputed from the dispatched rows
  g = q;
  g.a = bf(L.xbuf);
  g.a_shared = sh ? x : nullptr;
  g.b0 = w->w1;
  g.b1 = sw ? w->w3 : nullptr;
  g.sb0 = sh ? w->sw1 : nullptr;
  g.sb1 = sh && sw ? w->sw3 : nullptr;
  g.dh = bf(L.dh);
  g.out = bf(L.dz);
  g.K = H;
  g.N = F;
  g.b_packed = packed;
  if (!fused) {
    // compute-bound SwiGLU layers: pairs of SMs, as the forward's first
    // contraction (GShard's GELU layer measured 0.67 ms there against 0.42 ms on
    // one SM per tile: the epilogue's GELU' outweighs the feed)
    const cudaError_t e = two_sm_ffn(cfg) && sw
                              ? launch_bwd_dact_pair(g, dzw, at<int32_t>(ws, L.pairs), at<int32_t>(ws, L.kept), s)
                              : launch_bwd_dact(g, s);
    if (e != cudaSuccess) return MOE_ECUDA;
  }
  if ((st = record(stage_events, 4, s)) != MOE_OK) return st;
  // 5. dW1 (and dW3) = dz^T x_rows per expert; the shared block's rows are x
  g = q;
  g.wg_deep = wg_deep;
  g.a = bf(L.dz);
  g.b0 = bf(L.xbuf);
  g.b_shared = sh ? x : nullptr;
  g.M = dzw;
  g.N = H;
  g.m_split = sw ? Fp : dzw;
  g.m_valid = F;
  g.w_out = dw->dw1;
  g.w_out2 = sw ? dw->dw3 : nullptr;
  g.w_sh = sh ? dw->dsw1 : nullptr;
  g.w_sh2 = sh && sw ? dw->dsw3 : nullptr;
  if ((two_sm_ffn(cfg) ? launch_bwd_wgrad_pair(g, at<int32_t>(ws, L.kept), s) : launch_bwd_wgrad(g, s)) !=
      cudaSuccess)
    return MOE_ECUDA;
  if ((st = record(stage_events, 5, s)) != MOE_OK) return st;
  // 6. router backward
  RouterBwdParams rb{};
  rb.logits = at<float>(ws, L.logits);
  rb.dgate = at<float>(ws, L.dgate);
  rb.fcoef = at<float>(ws, L.fcoef);
  rb.dlogits = at<float>(ws, L.dlog);
  rb.T = cfg->T;
  rb.E = E;
  rb.k = cfg->k;
  rb.score = cfg->score;
  rb.renorm = cfg->renorm;
  rb.zc = d_z * cfg->z_coef;
  if (launch_router_bwd(rb, at<int32_t>(ws, L.cnt), L.nblk_router, d_aux * cfg->aux_alpha, at<float>(ws, L.fcoef),
                        s) != cudaSuccess)
    return MOE_ECUDA;
  if ((st = record(stage_events, 6, s)) != MOE_OK) return st;
  // 7. dxrow = dz [W1; W3] (weights read along H)
  g = q;
  g.a = bf(L.dz);
  g.b0 = w->w1;
  g.b1 = sw ? w->w3 : nullptr;
  g.sb0 = sh ? w->sw1 : nullptr;
  g.sb1 = sh && sw ? w->sw3 : nullptr;
  g.out = bf(L.dxrow);
  g.K = dzw;
  g.K0 = F;
  g.k_switch = sw ? Fp / 64 : 0;
  g.N = H;
  g.b_packed = packed;
  {
    const cudaError_t e = two_sm_ffn(cfg)
                              ? launch_bwd_dgrad_pair(g, at<int32_t>(ws, L.pairs), at<int32_t>(ws, L.kept), s)
                              : launch_bwd_dgrad(g, s);
    if (e != cudaSuccess) return MOE_ECUDA;
  }
  if ((st = record(stage_events, 7, s)) != MOE_OK) return st;
  // 8. dx: tokens sum their rows' gradients, plus the router's dlogits Wg
  DispatchBwdParams db{};
  db.dxrow = bf(L.dxrow);
  db.dlogits = at<float>(ws, L.dlog);
  db.wg = wg;
  db.ids = ids;
  db.slot = slot;
  db.off = off;
  db.dx = static_cast<__nv_bfloat16*>(dx);
  db.T = cfg->T;
  db.rows_max = L.rows_max;
  db.H = H;
  db.E = E;
  db.k = cfg->k;
  db.n_shared = cfg->n_shared;
  if (launch_dispatch_bwd(db, s) != cudaSuccess) return MOE_ECUDA;
  if ((st = record(stage_events, 8, s)) != MOE_OK) return st;
  // 9. dWg = dlogits^T x
  if (launch_router_wgrad(at<float>(ws, L.dlog), x, cfg->T, E, H, at<float>(ws, L.dwgp), dwg, s) != cudaSuccess)
    return MOE_ECUDA;
  return record(stage_events, 9, s);
}

int moe_sync_status(void* ws, moe_stream_t stream) {
  if (ws == nullptr) return MOE_EINVAL;
  cudaStream_t s = S(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ECUDA;
  DevStatus h{0, 0};
  if (cudaMemcpy(&h, ws, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ECUDA;
  if (cudaMemset(ws, 0, sizeof(DevStatus)) != cudaSuccess) return MOE_ECUDA;
  return h.code;
}

int moe_clear_status(void* ws, moe_stream_t stream) {
  if (ws == nullptr) return MOE_EINVAL;
  return cuda_status(cudaMemsetAsync(ws, 0, sizeof(DevStatus), S(stream)));
}

const char* moe_strerror(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_EINVAL: return "invalid argument or configuration";
    case MOE_EUNSUPPORTED: return "configuration outside the supported limits";
    case MOE_ECUDA: return "CUDA launch or runtime error";
    case MOE_ETIMEOUT: return "a bounded wait inside a kernel ran out";
    case MOE_EDEVICE: return "device-side index check failed";
    case MOE_EWORKSPACE: return "workspace smaller than moe_workspace_size()";
    default: return "unknown status";
  }
}

int moe_activation_eval(int act, const float* z, const float* u, float* out, int64_t n, moe_stream_t stream) {
  if (act < MOE_ACT_RELU || act > MOE_ACT_SWIGLU || n < 0) return MOE_EINVAL;
  if (n > 0 && (z == nullptr || out == nullptr || (act == MOE_ACT_SWIGLU && u == nullptr))) return MOE_EINVAL;
  return cuda_status(launch_activation_eval(act, z, u, out, n, S(stream)));
}

int moe_packed_weight_bytes(int32_t G, int32_t N, int32_t K, size_t* bytes) {
  if (bytes == nullptr || G < 1 || N < 1 || K < 1) return MOE_EINVAL;
  if (K % 8 != 0) return MOE_EUNSUPPORTED;
  *bytes = packed_weight_bytes(G, N, K);
  return MOE_OK;
}

int moe_pack_weight(const void* w, int32_t G, int32_t N, int32_t K, void* packed, moe_stream_t stream) {
  size_t bytes = 0;
  const int st = moe_packed_weight_bytes(G, N, K, &bytes);
  if (st != MOE_OK) return st;
  if (w == nullptr || packed == nullptr) return MOE_EINVAL;
  if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(packed)) & 15) return MOE_EINVAL;
  return cuda_status(launch_pack_weight(w, G, N, K, packed, S(stream)));
}

int moe_router_planes_bytes(int32_t E, int32_t H, size_t* bytes) {
  if (bytes == nullptr || E < 1 || H < 1) return MOE_EINVAL;
  if (E > kMaxE || H % 8 != 0) return MOE_EUNSUPPORTED;
  *bytes = sizeof(uint16_t) * (size_t)E * 3 * (size_t)router_plane_width(H);
  return MOE_OK;
}

int moe_pack_router_weight(const float* wg, int32_t E, int32_t H, void* planes, moe_stream_t stream) {
  size_t bytes = 0;
  const int st = moe_router_planes_bytes(E, H, &bytes);
  if (st != MOE_OK) return st;
  if (wg == nullptr || planes == nullptr) return MOE_EINVAL;
  if (reinterpret_cast<uintptr_t>(planes) & 15) return MOE_EINVAL;
  return cuda_status(launch_split_router_weight(wg, planes, E, H, S(stream)));
}

const char* moe_version(void) { return "moe_b200 0.2 sm_100a"; }

}  // extern "C"
