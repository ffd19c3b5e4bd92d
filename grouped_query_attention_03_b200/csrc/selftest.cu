// selftest.cu -- a check of the kernels' bounded waits.
//
// Every wait inside the library's kernels (an mbarrier phase that a TMA
// copy, an MMA commit or other warps complete) gives up after a time limit,
// records GQA_ERR_TIMEOUT in the caller's status word and lets the kernel
// return, so that a stalled call reports an error instead of hanging the
// GPU ("Share key/value heads and make context explicit", section "Extend
// the existing full and cached attention paths": a failed operation
// reports and leaves nothing half done).  That path only runs when
// something has gone wrong, so this entry point runs the same two wait
// routines (the suspending mbar_wait and the polling mbar_wait_spin) on
// mbarriers that no thread arrives on, with a caller-chosen short limit, in
// a kernel that has no copy or MMA in flight: the waits run out, the kernel
// records the status and returns, and the context stays usable.  With
// `arrive` set, one thread completes both barriers first and the waits
// succeed (the control case).
#include <cstdint>

#include "../../include/gqa.h"
#include "common.cuh"

namespace {

// Warp 0 waits with mbar_wait, warp 1 with mbar_wait_spin, each on its own
// barrier; lane 0 of a warp whose wait gave up counts it in gave_up[warp].
__global__ void wait_selftest_kernel(uint64_t limit_ns, int arrive,
                                     int32_t *status, int32_t *gave_up) {
  __shared__ __align__(8) uint64_t bar[2];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    gqa::mbar_init(&bar[0], 1);
    gqa::mbar_init(&bar[1], 1);
    gqa::fence_mbar_init();
  }
  __syncthreads();
  if (arrive && threadIdx.x == 0) {
    gqa::mbar_arrive(&bar[0]);
    gqa::mbar_arrive(&bar[1]);
  }
  __syncthreads();
  bool failed = false;
  const bool ok = warp == 0 ? gqa::mbar_wait(&bar[0], 0, &failed, limit_ns)
                            : gqa::mbar_wait_spin(&bar[1], 0, &failed, limit_ns);
  const bool all_ok = __all_sync(0xffffffffu, ok) != 0;
  if (lane == 0 && !all_ok) {
    atomicAdd(&gave_up[warp], 1);
    gqa::record_status(status, gqa::kStatusTimeout);
  }
}

}  // namespace

extern "C" gqa_status gqa_selftest_wait_timeout(int64_t limit_us, int arrive,
                                                int32_t *dev_status,
                                                int32_t *gave_up,
                                                gqa_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000) return GQA_ERR_SHAPE;
  if (!dev_status || !gave_up) return GQA_ERR_NULL;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
          cudaSuccess) {
    cudaGetLastError();
    return GQA_ERR_CUDA;
  }
  if (major != 10) return GQA_ERR_DEVICE;
  wait_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (uint64_t)limit_us * 1000ull, arrive ? 1 : 0, dev_status, gave_up);
  return cudaGetLastError() == cudaSuccess ? GQA_OK : GQA_ERR_CUDA;
}
