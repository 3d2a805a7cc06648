// Packing of expert weights into the grouped GEMM's block layout.
//
// A weight matrix [G, N, K] (bf16, the linear-layer layout with K contiguous)
// is read by the GEMM in boxes of 128 rows x 64 k.  In that layout one box is
// 128 pieces of 128 bytes, one per row, K*2 bytes apart, which HBM serves at a
// fraction of its streaming rate.  The packed layout
//     P[g][n / 128][k / 64][n % 128][k % 64]   (zero-padded to whole blocks)
// stores each box as one contiguous 16 KB block.  Packing is a one-time
// transformation of static weights, like any inference engine's weight
// preprocessing; the arithmetic of the layer is unchanged.
#include "common.cuh"
#include "kernels.h"

namespace moe {

size_t packed_weight_bytes(int G, int N, int K) {
  const size_t nb = (size_t)(N + 127) / 128, kb = (size_t)(K + 63) / 64;
  return (size_t)G * nb * kb * 128 * 64 * 2;
}

// One thread per 16-byte vector (8 elements) of the packed buffer.
__global__ void pack_weight_kernel(const __nv_bfloat16* w, int G, int N, int K, __nv_bfloat16* out) {
  pdl_wait();
  pdl_trigger();
  const int64_t nb = (N + 127) / 128, kb = (K + 63) / 64;
  const int64_t nvec = (int64_t)G * nb * kb * 128 * 8;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < nvec; v += (int64_t)gridDim.x * blockDim.x) {
    const int c8 = (int)(v & 7);                  // which 8-element piece of the 64-wide row
    const int r = (int)((v >> 3) & 127);          // row within the block
    const int64_t blk = v >> 10;                  // (g, n block, k block)
    const int64_t kbi = blk % kb, nbi = (blk / kb) % nb, g = blk / (kb * nb);
    const int64_t n = nbi * 128 + r, k = kbi * 64 + c8 * 8;
    int4 val = make_int4(0, 0, 0, 0);
    if (n < N && k < K) val = ld_nc_v4(w + (g * N + n) * (int64_t)K + k);   // K % 8 == 0: whole vectors
    st_v4(out + v * 8, val);
  }
}

cudaError_t launch_pack_weight(const void* w, int G, int N, int K, void* packed, cudaStream_t stream) {
  const int64_t nvec = (int64_t)packed_weight_bytes(G, N, K) / 16;
  if (nvec == 0) return cudaSuccess;
  const int64_t blocks = (nvec + 255) / 256;
  launch_pdl(pack_weight_kernel, (unsigned)(blocks < 65535 ? blocks : 65535), 256, 0, stream,
             static_cast<const __nv_bfloat16*>(w), G, N, K, static_cast<__nv_bfloat16*>(packed));
  return cudaGetLastError();
}

}  // namespace moe
