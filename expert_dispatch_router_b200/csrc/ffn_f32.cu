// fp32 grouped expert FFN on the FFMA pipes (the fp32 layer precision has no
// tensor-core operand kind).  One launch computes D = epi(A_g B_g^T) for every
// expert block g: GEMM1 with the activation (ReLU, GELU, or SwiGLU from two
// weight matrices) and GEMM2 without.  Expert blocks are multiples of 128 rows,
// so each 64-row tile lies inside one block; the block of a tile is found by a
// binary search over the expert offsets, entirely on the device.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kFBM = 64, kFBN = 64, kFBK = 16, kFThreads = 256;

__device__ __forceinline__ int find_group(const int32_t* off, int ngroups, int64_t row) {
  int lo = 0, hi = ngroups - 1;          // largest g with off[g] <= row
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= row) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__global__ void __launch_bounds__(kFThreads) ffn_f32_kernel(FfnF32Params p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[kFBK][kFBM + 4];
  __shared__ float Bs[2][kFBK][kFBN + 4];
  const int64_t row0 = (int64_t)blockIdx.x * kFBM;
  const int col0 = blockIdx.y * kFBN;
  const int ngroups = p.E + (p.n_shared ? 1 : 0);
  const int64_t end = min((int64_t)p.expert_offset[ngroups], p.rows_max);
  if (row0 >= end) return;
  const int g = find_group(p.expert_offset, ngroups, row0);
  const bool shared = g == p.E;
  const bool sep = shared && p.a_shared != nullptr;   // else the shared rows sit in a_routed in place
  const float* A = sep ? p.a_shared : p.a_routed;
  const int64_t arow0 = sep ? row0 - p.expert_offset[p.E] : row0;
  const int64_t arows = sep ? p.T : p.rows_max;
  const float* B0 = shared ? p.sb0 : p.b0 + (int64_t)g * p.N * p.K;
  const float* B1 = p.epi == MOE_ACT_SWIGLU ? (shared ? p.sb1 : p.b1 + (int64_t)g * p.N * p.K) : nullptr;

  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  float acc0[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < p.K; k0 += kFBK) {
    // A tile 64x16 and B tiles 64x16: 1024 elements each, 4 per thread
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int q = tid + i * kFThreads;
      const int rr = q / kFBK, kk = q % kFBK;
      const int64_t ar = arow0 + rr;
      As[kk][rr] = (ar < arows && k0 + kk < p.K) ? A[ar * p.K + k0 + kk] : 0.0f;
      const int n = col0 + rr;
      const bool okb = n < p.N && k0 + kk < p.K;
      Bs[0][kk][rr] = okb ? B0[(int64_t)n * p.K + k0 + kk] : 0.0f;
      if (B1) Bs[1][kk][rr] = okb ? B1[(int64_t)n * p.K + k0 + kk] : 0.0f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kFBK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b0[i] = Bs[0][kk][tx * 4 + i];
        b1[i] = B1 ? Bs[1][kk][tx * 4 + i] : 0.0f;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (B1) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = row0 + ty * 4 + i;
    if (r >= end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = col0 + tx * 4 + j;
      if (n >= p.N) continue;
      float v = acc0[i][j];
      if (p.epi == MOE_ACT_RELU) v = act_relu(v);
      else if (p.epi == MOE_ACT_GELU) v = act_gelu(v);
      else if (p.epi == MOE_ACT_SWIGLU) v = act_silu(v) * acc1[i][j];
      p.d[r * p.N + n] = v;
    }
  }
}

__global__ void activation_eval_kernel(int act, const float* z, const float* u, float* out, int64_t n) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float v = z[i];
    out[i] = act == MOE_ACT_RELU ? act_relu(v) : act == MOE_ACT_GELU ? act_gelu(v) : act_silu(v) * u[i];
  }
}

cudaError_t launch_activation_eval(int act, const float* z, const float* u, float* out, int64_t n,
                                   cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  activation_eval_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(act, z, u, out, n);
  return cudaGetLastError();
}

cudaError_t launch_ffn_f32(const FfnF32Params& p, cudaStream_t stream) {
  if (p.rows_max == 0) return cudaSuccess;
  dim3 grid((unsigned)((p.rows_max + kFBM - 1) / kFBM), (unsigned)((p.N + kFBN - 1) / kFBN));
  launch_pdl(ffn_f32_kernel, grid, kFThreads, 0, stream, p);
  return cudaGetLastError();
}

}  // namespace moe
