// Shared device helpers of the MoE forward library (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kRowPad = 128;          // expert row blocks are padded to this many rows
constexpr int kMaxK = 16;
constexpr int kMaxE = 1024;

// Device status word (first bytes of the workspace).  Kernels record the
// first error they see; the host reads it through moe_sync_status.
struct DevStatus {
  int code;
  int info;
};

__device__ __forceinline__ void set_status(DevStatus* st, int code, int info) {
  if (st != nullptr && atomicCAS(&st->code, 0, code) == 0) st->info = info;
}

__host__ __device__ __forceinline__ int64_t round_up(int64_t n, int64_t m) { return (n + m - 1) / m * m; }

// Element type helpers (bf16 and fp32 activations).
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// 16-byte vector helpers.
__device__ __forceinline__ int4 ld_nc_v4(const void* p) {
  int4 v;
  asm volatile("ld.global.nc.v4.s32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}
__device__ __forceinline__ void st_v4(void* p, int4 v) {
  asm volatile("st.global.v4.s32 [%0], {%1,%2,%3,%4};" :: "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w) : "memory");
}

// Activation functions on fp32 values.
__device__ __forceinline__ float act_relu(float z) { return fmaxf(z, 0.0f); }
__device__ __forceinline__ float act_gelu(float z) { return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f)); }
__device__ __forceinline__ float act_silu(float z) { return z / (1.0f + expf(-z)); }

// Upper bound on the cycles any bounded wait spins before it gives up (~1 s
// at the B200's boost clock).  Normal waits in these kernels last microseconds.
constexpr long long kWaitCycles = 2000000000LL;

}  // namespace moe

#define MOE_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t _e = (expr);                                 \
    if (_e != cudaSuccess) return MOE_ECUDA;                 \
  } while (0)
