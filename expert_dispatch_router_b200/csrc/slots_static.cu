// Slot assignment that needs no caller workspace: moe_assign_slots_static.
//
// Some callers cannot allocate device memory at all. Examples: a plugin that
// runs inside a host framework which owns every byte of device memory through
// its own pool and gives the plugin only its input and output tensors, or code
// on a latency path where any allocation (and the device-wide synchronisation
// cudaMalloc can imply) is not allowed.  Such callers can still assign slots:
// this variant keeps its scratch (per-chunk expert counts and a status word)
// in one file-scope device array of fixed size instead of the workspace.
//
// The array is loaded with the library, so every GPU that loads the library
// holds it until the process exits.  The kernels are the same ones
// moe_assign_slots launches.
#include <cuda.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

using namespace moe;

namespace {

constexpr size_t kStaticScratchBytes = size_t(1) << 20;          // 1 MiB
constexpr size_t kStatusBytes = 256;                             // DevStatus and the ticket, padded
constexpr size_t kTicketOffset = 128;
constexpr int64_t kStaticChunkInts = (int64_t)((kStaticScratchBytes - kStatusBytes) / sizeof(int32_t));

// Shared by every call on a device; holds the last call's contents.
static __device__ __align__(256) unsigned char g_slot_scratch[kStaticScratchBytes];

// Unique id of the calling thread's current CUDA context (0 if unknown).  A
// context re-created after cudaDeviceReset gets a new id, and the module (with
// g_slot_scratch) is loaded again at a possibly different address.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext*);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long*);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

// Device address of g_slot_scratch, looked up with the device current the first
// time a device (and each later context of it) calls.  (In host code the array's
// name is only a host-side stand-in.)
void* scratch_address(int& err) {
  static void* addr[64] = {nullptr};
  static unsigned long long ctx_of[64] = {0};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    err = MOE_ECUDA;
    return nullptr;
  }
  // 0 while no context is current on this thread: then look the address up (the
  // lookup makes the device's primary context current) and note the context
  const unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_slot_scratch) != cudaSuccess || p == nullptr) {
      err = MOE_ECUDA;
      return nullptr;
    }
    addr[dev] = p;
    ctx_of[dev] = current_context_id();
  }
  err = MOE_OK;
  return addr[dev];
}

}  // namespace

extern "C" int moe_assign_slots_static(const moe_cfg* cfg, const int32_t* ids, int32_t* slot, int32_t* expert_count,
                                       int32_t* kept_count, int32_t* expert_offset, int32_t* row_token,
                                       moe_stream_t stream) {
  int64_t cap = 0, rows_max = 0;
  int st = moe_capacity(cfg, &cap);
  if (st != MOE_OK) return st;
  st = moe_rows_max(cfg, &rows_max);
  if (st != MOE_OK) return st;
  if (expert_count == nullptr || kept_count == nullptr || expert_offset == nullptr) return MOE_EINVAL;
  if (cfg->T > 0 && (ids == nullptr || slot == nullptr || row_token == nullptr)) return MOE_EINVAL;
  if (cfg->cap_mode == MOE_CAP_CAPACITY && cfg->drop_policy == MOE_DROP_PROBS) return MOE_EUNSUPPORTED;
  const int64_t nchunk = (cfg->T * cfg->k + kSlotChunk - 1) / kSlotChunk;
  if ((int64_t)cfg->E * nchunk > kStaticChunkInts) return MOE_EUNSUPPORTED;   // beyond the fixed scratch
  int err = MOE_OK;
  unsigned char* base = static_cast<unsigned char*>(scratch_address(err));
  if (base == nullptr) return err;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the status word and the ticket must start at zero; the chunk counts are
  // fully rewritten
  if (cudaMemsetAsync(base, 0, kStatusBytes, s) != cudaSuccess) return MOE_ECUDA;
  SlotParams p{};
  p.ids = ids;
  p.slot = slot;
  p.expert_count = expert_count;
  p.kept_count = kept_count;
  p.expert_offset = expert_offset;
  p.row_token = row_token;
  p.chunk_cnt = reinterpret_cast<int32_t*>(base + kStatusBytes);
  p.status = reinterpret_cast<DevStatus*>(base);
  p.ticket = reinterpret_cast<unsigned*>(base + kTicketOffset);
  p.T = cfg->T;
  p.E = cfg->E;
  p.k = cfg->k;
  p.n_shared = cfg->n_shared;
  p.capacity = cap;
  p.rows_max = rows_max;
  return launch_slots(p, s) == cudaSuccess ? MOE_OK : MOE_ECUDA;
}
