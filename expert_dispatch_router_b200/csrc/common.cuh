// Shared device helpers of the MoE forward library (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

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

// Order-preserving map from fp32 to uint32 (a > b as floats <=> key(a) > key(b)
// as integers); -0 is mapped like +0 so equal values get equal keys.
__device__ __forceinline__ uint32_t to_ordered(float v) {
  const uint32_t b = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float from_ordered(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

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

// Activation functions on fp32 values, written for the GEMM epilogue's
// instruction budget.
__device__ __forceinline__ float act_relu(float z) { return fmaxf(z, 0.0f); }

// Reciprocal on the special-function unit (PTX rcp.approx: about 1 ulp;
// rcp(+inf) = 0).
__device__ __forceinline__ float rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}
// 2^x on the special-function unit (PTX ex2.approx, about 2 ulp).
__device__ __forceinline__ float exp2f_approx(float x) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// erf from Abramowitz & Stegun, Handbook of Mathematical Functions (1964),
// formula 7.1.26: erf(x) = 1 - (a1 t + ... + a5 t^5) exp(-x^2), t = 1/(1 + p x),
// x >= 0, absolute error <= 1.5e-7; odd symmetry for x < 0.  The exponential
// and the reciprocal use the special-function unit.
__device__ __forceinline__ float erf_as7126(float x) {
  const float ax = fabsf(x);
  const float t = rcp_approx(fmaf(0.3275911f, ax, 1.0f));
  float poly = fmaf(1.061405429f, t, -1.453152027f);
  poly = fmaf(poly, t, 1.421413741f);
  poly = fmaf(poly, t, -0.284496736f);
  poly = fmaf(poly, t, 0.254829592f);
  poly *= t;
  const float r = 1.0f - poly * __expf(-ax * ax);
  return copysignf(r, x);
}
// Exact-form GELU, 0.5 z (1 + erf(z / sqrt 2)), evaluated through erfc: formula
// 7.1.26 is erfc(x) = P(t) exp(-x^2) for x >= 0, so with x = |z| / sqrt 2,
//   z <  0:  0.5 z (1 + erf(z/sqrt 2)) = 0.5 z erfc(x)
//   z >= 0:  0.5 z (1 + erf(z/sqrt 2)) = z - 0.5 z erfc(x).
// Constants are pre-scaled: p/sqrt 2 in t, 0.5 a_i in the polynomial, and
// exp(-z^2/2) = 2^(-z^2 log2(e) / 2).  Same error bound as erf_as7126.
__device__ __forceinline__ float act_gelu(float z) {
  const float t = rcp_approx(fmaf(0.23164189f, fabsf(z), 1.0f));           // 0.3275911 / sqrt 2
  float q = fmaf(0.5307027145f, t, -0.7265760135f);                        // 0.5 * a5, 0.5 * a4
  q = fmaf(q, t, 0.7107068705f);                                            // 0.5 * a3
  q = fmaf(q, t, -0.142248368f);                                            // 0.5 * a2
  q = fmaf(q, t, 0.127414796f);                                             // 0.5 * a1
  const float e = exp2f_approx(z * z * -0.72134752044448170f);             // exp(-z^2 / 2)
  const float h = z * (q * t) * e;                                          // 0.5 z erfc(|z| / sqrt 2)
  return z >= 0.0f ? z - h : h;
}
// Two fp32 values in one 64-bit register for the packed fp32 pipes of sm_100
// (add / sub / mul / fma .f32x2: each half the same IEEE operation as the
// scalar instruction, two values per issue).
__device__ __forceinline__ unsigned long long f32x2_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f32x2_unpack(unsigned long long r, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(r));
}
__device__ __forceinline__ unsigned long long f32x2_fma(unsigned long long a, unsigned long long b,
                                                        unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f32x2_mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f32x2_sub(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// act_gelu of two values: the same steps and constants, the FMA-pipe work on
// packed pairs, the reciprocal and the exponential per value.
__device__ __forceinline__ void act_gelu_x2(float& z0, float& z1) {
  const unsigned long long z = f32x2_pack(z0, z1);
  const unsigned long long a =
      f32x2_fma(f32x2_pack(0.23164189f, 0.23164189f), f32x2_pack(fabsf(z0), fabsf(z1)), f32x2_pack(1.0f, 1.0f));
  float a0, a1;
  f32x2_unpack(a, a0, a1);
  const unsigned long long t = f32x2_pack(rcp_approx(a0), rcp_approx(a1));
  unsigned long long q = f32x2_fma(f32x2_pack(0.5307027145f, 0.5307027145f), t, f32x2_pack(-0.7265760135f, -0.7265760135f));
  q = f32x2_fma(q, t, f32x2_pack(0.7107068705f, 0.7107068705f));
  q = f32x2_fma(q, t, f32x2_pack(-0.142248368f, -0.142248368f));
  q = f32x2_fma(q, t, f32x2_pack(0.127414796f, 0.127414796f));
  const unsigned long long sq = f32x2_mul(f32x2_mul(z, z), f32x2_pack(-0.72134752044448170f, -0.72134752044448170f));
  float s0, s1;
  f32x2_unpack(sq, s0, s1);
  const unsigned long long e = f32x2_pack(exp2f_approx(s0), exp2f_approx(s1));
  const unsigned long long h = f32x2_mul(f32x2_mul(z, f32x2_mul(q, t)), e);   // 0.5 z erfc(|z| / sqrt 2)
  const unsigned long long r = f32x2_sub(z, h);
  float h0, h1, r0, r1;
  f32x2_unpack(h, h0, h1);
  f32x2_unpack(r, r0, r1);
  z0 = z0 >= 0.0f ? r0 : h0;
  z1 = z1 >= 0.0f ? r1 : h1;
}
// GELU'(z) = d/dz [z Phi(z)] = Phi(z) + z phi(z); Phi from erf (Abramowitz & Stegun 7.1.26).
__device__ __forceinline__ float gelu_grad(float z) {
  const float phi = 0.3989422804014327f * __expf(-0.5f * z * z);
  return 0.5f * (1.0f + erf_as7126(z * 0.70710678118654752f)) + z * phi;
}
// gelu_grad of two values: Phi(z) = 0.5 (1 + erf(z / sqrt 2)) from the same
// erf formula (Abramowitz & Stegun 7.1.26) and phi(z) = exp(-z^2 / 2) / sqrt(2 pi),
// the FMA-pipe work on packed pairs, exp(a) as 2^(a log2 e) and the reciprocal
// per value.
__device__ __forceinline__ void gelu_grad_x2(float& z0, float& z1) {
  const unsigned long long z = f32x2_pack(z0, z1);
  const unsigned long long a = f32x2_mul(f32x2_mul(z, z), f32x2_pack(-0.72134752044448170f, -0.72134752044448170f));
  float a0, a1;
  f32x2_unpack(a, a0, a1);
  const unsigned long long phi =
      f32x2_mul(f32x2_pack(0.3989422804014327f, 0.3989422804014327f), f32x2_pack(exp2f_approx(a0), exp2f_approx(a1)));
  const unsigned long long x = f32x2_mul(z, f32x2_pack(0.70710678118654752f, 0.70710678118654752f));
  float x0, x1;
  f32x2_unpack(x, x0, x1);
  const unsigned long long ax = f32x2_pack(fabsf(x0), fabsf(x1));
  const unsigned long long d = f32x2_fma(f32x2_pack(0.3275911f, 0.3275911f), ax, f32x2_pack(1.0f, 1.0f));
  float d0, d1;
  f32x2_unpack(d, d0, d1);
  const unsigned long long t = f32x2_pack(rcp_approx(d0), rcp_approx(d1));
  unsigned long long poly = f32x2_fma(f32x2_pack(1.061405429f, 1.061405429f), t, f32x2_pack(-1.453152027f, -1.453152027f));
  poly = f32x2_fma(poly, t, f32x2_pack(1.421413741f, 1.421413741f));
  poly = f32x2_fma(poly, t, f32x2_pack(-0.284496736f, -0.284496736f));
  poly = f32x2_fma(poly, t, f32x2_pack(0.254829592f, 0.254829592f));
  poly = f32x2_mul(poly, t);
  const unsigned long long b = f32x2_mul(f32x2_mul(ax, ax), f32x2_pack(-1.4426950408889634f, -1.4426950408889634f));
  float b0, b1;
  f32x2_unpack(b, b0, b1);
  const unsigned long long r =
      f32x2_sub(f32x2_pack(1.0f, 1.0f), f32x2_mul(poly, f32x2_pack(exp2f_approx(b0), exp2f_approx(b1))));
  float r0, r1;
  f32x2_unpack(r, r0, r1);
  const unsigned long long erf = f32x2_pack(copysignf(r0, x0), copysignf(r1, x1));
  const unsigned long long g = f32x2_fma(z, phi, f32x2_fma(f32x2_pack(0.5f, 0.5f), erf, f32x2_pack(0.5f, 0.5f)));
  f32x2_unpack(g, z0, z1);
}
// SiLU: z * sigmoid(z) = z / (1 + exp(-z)).
__device__ __forceinline__ float act_silu(float z) { return z * rcp_approx(1.0f + __expf(-z)); }

// Programmatic dependent launch.  The layer's kernels are launched so that the
// next kernel on the stream may be scheduled while this one drains: every such
// kernel calls pdl_wait() before it touches global memory that an earlier
// launch writes or reads (griddepcontrol.wait returns once the preceding grid
// has completed and its writes are visible), and pdl_trigger() to let the next
// grid launch early; its CTAs then block in their own pdl_wait().
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Host: launch `kern` with programmatic stream serialization allowed.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Upper bound on the cycles any bounded wait spins before it gives up (~1 s
// at the B200's boost clock).  Normal waits in these kernels last microseconds.
constexpr long long kWaitCycles = 2000000000LL;

// Host: raise a kernel's dynamic shared memory limit to at least `bytes` on the
// current device (the default limit counts the kernel's static shared memory
// too, so any non-zero request is set explicitly).  Remembers, per (kernel,
// device), the largest limit set.
inline cudaError_t ensure_smem_ptr(const void* k, size_t bytes) {
  if (bytes == 0) return cudaSuccess;
  int dev = 0;
  cudaGetDevice(&dev);
  struct Entry { const void* k; int dev; size_t bytes; };
  static std::mutex mu;
  static Entry tab[256];
  static int n = 0;
  std::lock_guard<std::mutex> lock(mu);
  int i = 0;
  while (i < n && !(tab[i].k == k && tab[i].dev == dev)) ++i;
  if (i < n && tab[i].bytes >= bytes) return cudaSuccess;
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  if (i < n) tab[i].bytes = bytes;
  else if (n < 256) tab[n++] = Entry{k, dev, bytes};
  return cudaSuccess;
}
template <typename Kernel>
inline cudaError_t ensure_smem(Kernel k, size_t bytes) {
  return ensure_smem_ptr(reinterpret_cast<const void*>(k), bytes);
}

// Host: multiprocessor count of the current device (cached per device).
inline int sm_count() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  int& c = cache[dev & 63];
  if (c == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    c = n > 0 ? n : 148;
  }
  return c;
}

}  // namespace moe

#define MOE_CUDA_TRY(expr)                                   \
  do {                                                       \
    cudaError_t _e = (expr);                                 \
    if (_e != cudaSuccess) return MOE_ECUDA;                 \
  } while (0)
