// Memory-bound kernels of the backward pass: the combine's and the dispatch's
// backward permutations, the zeroing of padding rows, and the router weight
// gradient.
//
// Method: "Expert-parallel MoE training" explainer: in the backward pass the
// combine's gradient travels the dispatch path (each kept row receives its
// token's output gradient times the gate) and the dispatch's gradient travels
// the combine path (each token sums the input gradients of its rows);
// "Switch Routing" 2.1: y = p_i E_i, so the gate's gradient is the dot product
// of the output gradient with the expert's (un-gated) output.
//
// Like the forward permutations these are token-centric, one warp per token,
// 16-byte vectors, fp32 accumulation in choice-rank order, deterministic.
#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kBwdWarps = 8;

// dyrow[row(t,r)] = gate[t,r] * dy[t]; dgate[t,r] = dy[t] . ybuf[row(t,r)];
// dyrow[off[E] + t] = dy[t] for the shared expert.  Choices without a row get
// dgate = 0.
__global__ void __launch_bounds__(kBwdWarps * 32) combine_bwd_kernel(CombineBwdParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (t >= p.T) return;
  const int nvec = p.H / 8;
  const __nv_bfloat16* dy = p.dy + t * p.H;
  for (int r = 0; r < p.k; ++r) {
    const int s = p.slot[t * p.k + r], e = p.ids[t * p.k + r];
    const bool kept = s >= 0 && e >= 0 && e < p.E && (int64_t)p.off[e] + s < p.rows_max;
    float dot = 0.0f;
    if (kept) {
      const int64_t row = (int64_t)p.off[e] + s;
      const float g = p.gates[t * p.k + r];
      const __nv_bfloat16* yr = p.ybuf + row * p.H;
      __nv_bfloat16* dr = p.dyrow + row * p.H;
      for (int v = lane; v < nvec; v += 32) {
        const int4 a = ld_nc_v4(dy + 8 * v), b = ld_nc_v4(yr + 8 * v);
        const __nv_bfloat16* ea = reinterpret_cast<const __nv_bfloat16*>(&a);
        const __nv_bfloat16* eb = reinterpret_cast<const __nv_bfloat16*>(&b);
        int4 o;
        __nv_bfloat16* eo = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float d = __bfloat162float(ea[i]);
          dot = fmaf(d, __bfloat162float(eb[i]), dot);
          eo[i] = __float2bfloat16_rn(g * d);
        }
        st_v4(dr + 8 * v, o);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    }
    if (lane == 0) p.dgate[t * p.k + r] = dot;
  }
  if (p.n_shared) {
    __nv_bfloat16* dr = p.dyrow + ((int64_t)p.off[p.E] + t) * p.H;
    for (int v = lane; v < nvec; v += 32) st_v4(dr + 8 * v, ld_nc_v4(dy + 8 * v));
  }
}

// Rows of buf [rows, width] (bf16) that hold no token (row_token < 0) are
// zeroed, up to the end of the used rows.
__global__ void __launch_bounds__(kBwdWarps * 32) zero_pad_rows_kernel(__nv_bfloat16* buf, int width,
                                                                        const int32_t* row_token,
                                                                        const int32_t* off, int ngroups,
                                                                        int64_t rows_max) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t used = min((int64_t)off[ngroups], rows_max);
  for (int64_t row = (int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5); row < used;
       row += (int64_t)gridDim.x * kBwdWarps) {
    if (row_token[row] >= 0) continue;
    __nv_bfloat16* r = buf + row * width;
    for (int v = lane; v < width / 8; v += 32) st_v4(r + 8 * v, make_int4(0, 0, 0, 0));
  }
}

// dx[t] = sum_r dxrow[row(t,r)] (+ dxrow[off[E] + t]) + sum_e dlogits[t,e] Wg[e,:],
// fp32 accumulation in choice-rank order, one rounding.
__global__ void __launch_bounds__(kBwdWarps * 32) dispatch_bwd_kernel(DispatchBwdParams p) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t t = (int64_t)blockIdx.x * kBwdWarps + (threadIdx.x >> 5);
  if (t >= p.T) return;
  int rows[kMaxK];
  int nr = 0;
  for (int r = 0; r < p.k; ++r) {
    const int s = p.slot[t * p.k + r], e = p.ids[t * p.k + r];
    if (s >= 0 && e >= 0 && e < p.E && (int64_t)p.off[e] + s < p.rows_max) rows[nr++] = p.off[e] + s;
  }
  const int64_t shared_row = p.n_shared ? (int64_t)p.off[p.E] + t : -1;
  const float* dl = p.dlogits + t * p.E;
  for (int v = lane; v < p.H / 8; v += 32) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int q = 0; q < nr; ++q) {
      const int4 a = ld_nc_v4(p.dxrow + (int64_t)rows[q] * p.H + 8 * v);
      const __nv_bfloat16* ea = reinterpret_cast<const __nv_bfloat16*>(&a);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __bfloat162float(ea[i]);
    }
    if (shared_row >= 0) {
      const int4 a = ld_nc_v4(p.dxrow + shared_row * p.H + 8 * v);
      const __nv_bfloat16* ea = reinterpret_cast<const __nv_bfloat16*>(&a);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += __bfloat162float(ea[i]);
    }
    // the router's part: dlogits[t,:] Wg (fp32)
    for (int e = 0; e < p.E; ++e) {
      const float d = __ldg(dl + e);
      const float4 w0 = __ldg(reinterpret_cast<const float4*>(p.wg + (int64_t)e * p.H + 8 * v));
      const float4 w1 = __ldg(reinterpret_cast<const float4*>(p.wg + (int64_t)e * p.H + 8 * v + 4));
      acc[0] = fmaf(d, w0.x, acc[0]); acc[1] = fmaf(d, w0.y, acc[1]);
      acc[2] = fmaf(d, w0.z, acc[2]); acc[3] = fmaf(d, w0.w, acc[3]);
      acc[4] = fmaf(d, w1.x, acc[4]); acc[5] = fmaf(d, w1.y, acc[5]);
      acc[6] = fmaf(d, w1.z, acc[6]); acc[7] = fmaf(d, w1.w, acc[7]);
    }
    int4 o;
    __nv_bfloat16* eo = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
    for (int i = 0; i < 8; ++i) eo[i] = __float2bfloat16_rn(acc[i]);
    st_v4(p.dx + t * p.H + 8 * v, o);
  }
}

// Router weight gradient dWg[e,h] = sum_t dlogits[t,e] x[t,h] in two
// deterministic steps: CTA (e block of 32, h block of 128, token chunk of 256)
// writes a partial sum; the partials are added in chunk order.
constexpr int kDwgE = 32, kDwgH = 128, kDwgT = 256, kDwgSub = 32;

__global__ void __launch_bounds__(256) dwg_partial_kernel(const float* dlogits, const __nv_bfloat16* x, int64_t T,
                                                          int E, int H, float* part) {
  pdl_wait();
  pdl_trigger();
  __shared__ float sd[kDwgSub][kDwgE];
  __shared__ float sx[kDwgSub][kDwgH];
  const int tid = threadIdx.x;
  const int e0 = blockIdx.x * kDwgE, h0 = blockIdx.y * kDwgH;
  const int64_t t0 = (int64_t)blockIdx.z * kDwgT;
  const int te = tid >> 5, th = tid & 31;            // thread: experts te*4.., columns th*4..
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int64_t ts = t0; ts < t0 + kDwgT && ts < T; ts += kDwgSub) {
    for (int i = tid; i < kDwgSub * kDwgE; i += 256) {
      const int r = i / kDwgE, c = i % kDwgE;
      const int64_t t = ts + r;
      sd[r][c] = (t < T && e0 + c < E) ? dlogits[t * E + e0 + c] : 0.0f;
    }
    for (int i = tid; i < kDwgSub * kDwgH; i += 256) {
      const int r = i / kDwgH, c = i % kDwgH;
      const int64_t t = ts + r;
      sx[r][c] = (t < T && h0 + c < H) ? __bfloat162float(x[t * H + h0 + c]) : 0.0f;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < kDwgSub; ++r)
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(sd[r][te * 4 + i], sx[r][th * 4 + j], acc[i][j]);
    __syncthreads();
  }
  float* out = part + (int64_t)blockIdx.z * E * H;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = e0 + te * 4 + i;
    if (e >= E) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (h0 + th * 4 + j < H) out[(int64_t)e * H + h0 + th * 4 + j] = acc[i][j];
  }
}

__global__ void dwg_reduce_kernel(const float* part, int nchunk, int64_t n, float* dwg) {
  pdl_wait();
  pdl_trigger();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    float s = 0.0f;
    for (int c = 0; c < nchunk; ++c) s += part[(int64_t)c * n + i];
    dwg[i] = s;
  }
}

int dwg_chunks(int64_t T) { return (int)((T + kDwgT - 1) / kDwgT); }

cudaError_t launch_combine_bwd(const CombineBwdParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  launch_pdl(combine_bwd_kernel, (unsigned)((p.T + kBwdWarps - 1) / kBwdWarps), kBwdWarps * 32, 0, stream, p);
  return cudaGetLastError();
}

cudaError_t launch_zero_pad_rows(void* buf, int width, const int32_t* row_token, const int32_t* off, int ngroups,
                                 int64_t rows_max, cudaStream_t stream) {
  if (rows_max == 0) return cudaSuccess;
  const int64_t blocks = (rows_max + kBwdWarps - 1) / kBwdWarps;
  launch_pdl(zero_pad_rows_kernel, (unsigned)(blocks < 4096 ? blocks : 4096), kBwdWarps * 32, 0, stream,
             static_cast<__nv_bfloat16*>(buf), width, row_token, off, ngroups, rows_max);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_bwd(const DispatchBwdParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  launch_pdl(dispatch_bwd_kernel, (unsigned)((p.T + kBwdWarps - 1) / kBwdWarps), kBwdWarps * 32, 0, stream, p);
  return cudaGetLastError();
}

cudaError_t launch_router_wgrad(const float* dlogits, const void* x, int64_t T, int E, int H, float* part,
                                float* dwg, cudaStream_t stream) {
  const int64_t n = (int64_t)E * H;
  if (T == 0) return cudaMemsetAsync(dwg, 0, sizeof(float) * n, stream);
  const dim3 grid((E + kDwgE - 1) / kDwgE, (H + kDwgH - 1) / kDwgH, dwg_chunks(T));
  launch_pdl(dwg_partial_kernel, grid, 256, 0, stream, dlogits, static_cast<const __nv_bfloat16*>(x), T, E, H, part);
  const int64_t blocks = (n + 255) / 256;
  launch_pdl(dwg_reduce_kernel, (unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream,
             static_cast<const float*>(part), dwg_chunks(T), n, dwg);
  return cudaGetLastError();
}

}  // namespace moe
