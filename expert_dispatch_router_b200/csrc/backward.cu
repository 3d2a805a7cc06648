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
// fp32, one rounding.  CTA: 64 tokens x 256 columns; the router's part is a
// small fp32 contraction over E, staged through shared memory in chunks of 32
// experts: warp w owns tokens 8w..8w+7, lane l columns 4l..4l+3 and
// 128+4l..128+4l+3, so each step reads two broadcast and two conflict-free
// 16-byte words for 64 FMAs.  The rows are added in choice-rank order after
// the contraction.
constexpr int kDxT = 64, kDxH = 256, kDxE = 32;

__global__ void __launch_bounds__(256) dispatch_bwd_kernel(DispatchBwdParams p) {
  __shared__ __align__(16) float sdl[kDxE][kDxT + 4];
  __shared__ __align__(16) float swg[kDxE][kDxH];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, ty = tid >> 5, tx = tid & 31;
  const int64_t t0 = (int64_t)blockIdx.x * kDxT;
  const int h0 = blockIdx.y * kDxH;
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0f;
  for (int e0 = 0; e0 < p.E; e0 += kDxE) {
#pragma unroll
    for (int j = 0; j < kDxE * kDxT / 256; ++j) {
      const int i = tid + 256 * j, tok = i / kDxE, e = i % kDxE;
      const int64_t t = t0 + tok;
      sdl[e][tok] = (t < p.T && e0 + e < p.E) ? __ldg(p.dlogits + t * p.E + e0 + e) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kDxE * kDxH / 4 / 256; ++j) {
      const int i = tid + 256 * j, r = i / (kDxH / 4), c = 4 * (i % (kDxH / 4));
      float4 w = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (e0 + r < p.E && h0 + c < p.H) w = __ldg(reinterpret_cast<const float4*>(p.wg + (int64_t)(e0 + r) * p.H + h0 + c));
      *reinterpret_cast<float4*>(&swg[r][c]) = w;
    }
    __syncthreads();
#pragma unroll 4
    for (int e = 0; e < kDxE; ++e) {
      const float4 d0 = *reinterpret_cast<const float4*>(&sdl[e][8 * ty]);
      const float4 d1 = *reinterpret_cast<const float4*>(&sdl[e][8 * ty + 4]);
      const float4 w0 = *reinterpret_cast<const float4*>(&swg[e][4 * tx]);
      const float4 w1 = *reinterpret_cast<const float4*>(&swg[e][128 + 4 * tx]);
      const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      const float wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(dv[i], wv[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t t = t0 + 8 * ty + i;
    if (t >= p.T) break;
    int rows[kMaxK + 1];
    int nr = 0;
    for (int r = 0; r < p.k; ++r) {
      const int s = p.slot[t * p.k + r], e = p.ids[t * p.k + r];
      if (s >= 0 && e >= 0 && e < p.E && (int64_t)p.off[e] + s < p.rows_max) rows[nr++] = p.off[e] + s;
    }
    if (p.n_shared) rows[nr++] = p.off[p.E] + (int)t;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int col = h0 + 128 * half + 4 * tx;
      if (col >= p.H) continue;
      float s4[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      for (int q = 0; q < nr; ++q) {
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(p.dxrow + (int64_t)rows[q] * p.H + col));
        const __nv_bfloat16* ea = reinterpret_cast<const __nv_bfloat16*>(&a);
#pragma unroll
        for (int c = 0; c < 4; ++c) s4[c] += __bfloat162float(ea[c]);
      }
      uint2 o;
      __nv_bfloat16* eo = reinterpret_cast<__nv_bfloat16*>(&o);
#pragma unroll
      for (int c = 0; c < 4; ++c) eo[c] = __float2bfloat16_rn(s4[c] + acc[i][4 * half + c]);
      *reinterpret_cast<uint2*>(p.dx + t * p.H + col) = o;
    }
  }
}

// Router weight gradient dWg[e,h] = sum_t dlogits[t,e] x[t,h] in two
// deterministic steps: CTA (64 experts, 128 columns, one token chunk) writes a
// partial sum; the partials are added in chunk order.  Warp w owns experts
// 8w..8w+7, lane l columns 4l..4l+3: per token, two broadcast and one
// conflict-free 16-byte shared read feed 32 FMAs.  The chunk count is a pure
// function of (T, E, H): enough CTAs for four per SM of a 148-SM part, at most
// one chunk per 128 tokens.
constexpr int kDwgE = 64, kDwgH = 128, kDwgSub = 32;

__global__ void __launch_bounds__(256) dwg_partial_kernel(const float* dlogits, const __nv_bfloat16* x, int64_t T,
                                                          int E, int H, int64_t tpc, float* part) {
  __shared__ __align__(16) float sd[kDwgSub][kDwgE];
  __shared__ __align__(16) float sx[kDwgSub][kDwgH];
  pdl_wait();
  pdl_trigger();
  const int tid = threadIdx.x, te = tid >> 5, th = tid & 31;
  const int e0 = blockIdx.x * kDwgE, h0 = blockIdx.y * kDwgH;
  const int64_t t0 = (int64_t)blockIdx.z * tpc;
  const int64_t t1 = min(t0 + tpc, T);
  float acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  for (int64_t ts = t0; ts < t1; ts += kDwgSub) {
#pragma unroll
    for (int j = 0; j < kDwgSub * kDwgE / 256; ++j) {
      const int i = tid + 256 * j, r = i / kDwgE, c = i % kDwgE;
      const int64_t t = ts + r;
      sd[r][c] = (t < t1 && e0 + c < E) ? __ldg(dlogits + t * E + e0 + c) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kDwgSub * kDwgH / 4 / 256; ++j) {
      const int i = tid + 256 * j, r = i / (kDwgH / 4), c = 4 * (i % (kDwgH / 4));
      const int64_t t = ts + r;
      float4 v = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (t < t1 && h0 + c < H) {
        const uint2 a = __ldg(reinterpret_cast<const uint2*>(x + t * H + h0 + c));
        const __nv_bfloat16* ea = reinterpret_cast<const __nv_bfloat16*>(&a);
        v = make_float4(__bfloat162float(ea[0]), __bfloat162float(ea[1]), __bfloat162float(ea[2]),
                        __bfloat162float(ea[3]));
      }
      *reinterpret_cast<float4*>(&sx[r][c]) = v;
    }
    __syncthreads();
#pragma unroll 8
    for (int r = 0; r < kDwgSub; ++r) {
      const float4 d0 = *reinterpret_cast<const float4*>(&sd[r][8 * te]);
      const float4 d1 = *reinterpret_cast<const float4*>(&sd[r][8 * te + 4]);
      const float4 xv = *reinterpret_cast<const float4*>(&sx[r][4 * th]);
      const float dv[8] = {d0.x, d0.y, d0.z, d0.w, d1.x, d1.y, d1.z, d1.w};
      const float xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(dv[i], xw[j], acc[i][j]);
    }
    __syncthreads();
  }
  float* out = part + (int64_t)blockIdx.z * E * H;
  const int col = h0 + 4 * th;
  if (col >= H) return;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = e0 + 8 * te + i;
    if (e < E) *reinterpret_cast<float4*>(out + (int64_t)e * H + col) = make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
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

int dwg_chunks(int64_t T, int E, int H) {
  const int64_t tiles = (int64_t)((E + kDwgE - 1) / kDwgE) * ((H + kDwgH - 1) / kDwgH);
  const int64_t by_tokens = (T + 127) / 128;
  const int64_t by_sms = (4 * 148 + tiles - 1) / tiles;
  const int64_t c = by_tokens < by_sms ? by_tokens : by_sms;
  return (int)(c > 1 ? c : 1);
}

// tokens per chunk: a multiple of 32
static int64_t dwg_tokens_per_chunk(int64_t T, int nchunk) { return ((T + nchunk - 1) / nchunk + 31) / 32 * 32; }

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
  if (p.k > kMaxK) return cudaErrorInvalidValue;
  const dim3 grid((unsigned)((p.T + kDxT - 1) / kDxT), (unsigned)((p.H + kDxH - 1) / kDxH));
  launch_pdl(dispatch_bwd_kernel, grid, 256, 0, stream, p);
  return cudaGetLastError();
}

cudaError_t launch_router_wgrad(const float* dlogits, const void* x, int64_t T, int E, int H, float* part,
                                float* dwg, cudaStream_t stream) {
  const int64_t n = (int64_t)E * H;
  if (T == 0) return cudaMemsetAsync(dwg, 0, sizeof(float) * n, stream);
  const int nchunk = dwg_chunks(T, E, H);
  const int64_t tpc = dwg_tokens_per_chunk(T, nchunk);
  const int used = (int)((T + tpc - 1) / tpc);      // chunks that hold tokens (<= nchunk)
  const dim3 grid((E + kDwgE - 1) / kDwgE, (H + kDwgH - 1) / kDwgH, used);
  launch_pdl(dwg_partial_kernel, grid, 256, 0, stream, dlogits, static_cast<const __nv_bfloat16*>(x), T, E, H, tpc,
             part);
  const int64_t blocks = (n + 255) / 256;
  launch_pdl(dwg_reduce_kernel, (unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, stream,
             static_cast<const float*>(part), used, n, dwg);
  return cudaGetLastError();
}

}  // namespace moe
