// Self-check of the failure-detection path shared by the tensor-core kernels:
// a bounded mbarrier wait that nothing will satisfy must give up, record
// MOE_ETIMEOUT in the caller's status word and let the kernel return, so the
// context stays usable and the host learns of it through moe_sync_status.
//
// The kernel issues no copy and no MMA, so nothing is in flight when the wait
// runs out.  Warp 0 waits on an mbarrier whose single expected arrival never
// comes; with `abort_after` >= 0, warp 1 raises the CTA's abort flag after that
// many cycles instead, and the wait must return early through the flag (the
// path a CTA takes when another role of it has already given up).
#include "common.cuh"
#include "kernels.h"
#include "tc_common.cuh"

namespace moe {

__global__ void bounded_wait_selftest_kernel(DevStatus* status, long long limit, long long abort_after,
                                             long long* waited) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t b = tcx::smem_u32(&bar);
  if (threadIdx.x == 0) {
    tcx::mbar_init(b, 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0 && lane == 0) {
    const long long t0 = clock64();
    const bool ok = tcx::mbar_wait_for(b, 0, &abort_flag, limit);
    *waited = clock64() - t0;
    if (!ok) set_status(status, MOE_ETIMEOUT, 99);
  } else if (warp == 1 && lane == 0 && abort_after >= 0) {
    const long long t0 = clock64();
    while (clock64() - t0 < abort_after) {}
    *reinterpret_cast<volatile int*>(&abort_flag) = 1;
  }
  __syncthreads();
  if (threadIdx.x == 0) tcx::mbar_arrive(b);   // leave the barrier's phase complete
}

cudaError_t launch_bounded_wait_selftest(DevStatus* status, long long limit, long long abort_after,
                                         long long* waited, cudaStream_t stream) {
  bounded_wait_selftest_kernel<<<1, 64, 0, stream>>>(status, limit, abort_after, waited);
  return cudaGetLastError();
}

}  // namespace moe

extern "C" int moe_selftest_bounded_wait(int64_t limit_cycles, int64_t abort_after_cycles, int64_t* waited_cycles,
                                         void* ws, moe_stream_t stream) {
  using namespace moe;
  if (ws == nullptr || waited_cycles == nullptr) return MOE_EINVAL;
  if (limit_cycles < 0 || limit_cycles > kWaitCycles) return MOE_EINVAL;
  if (abort_after_cycles > kWaitCycles) return MOE_EINVAL;
  const cudaError_t e = launch_bounded_wait_selftest(static_cast<DevStatus*>(ws), limit_cycles, abort_after_cycles,
                                                     reinterpret_cast<long long*>(waited_cycles),
                                                     reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? MOE_OK : MOE_ECUDA;
}
