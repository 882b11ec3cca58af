// selftest.cu — a diagnostic that makes one of the library's bounded waits run out, so the
// timeout path (abort flag, the other roles giving up, the status word) can be checked on a GPU
// without a fault: the wait is on an mbarrier that nothing ever arrives on.
#include "common.cuh"

namespace nvfp4 {
namespace {

// Warp 0 waits (limit_ns) on a barrier nobody arrives on and raises the CTA's abort flag when the
// wait runs out; warp 1 waits on a second such barrier with the default 2 s limit and must leave
// early because of the flag, as the roles of the grouped GEMM do.  Thread 0 then reports
// NVFP4_DEVERR_TIMEOUT into the status word.
__global__ void __launch_bounds__(64) wait_selftest_kernel(uint64_t limit_ns,
                                                          int32_t* __restrict__ dev_status,
                                                          uint64_t* __restrict__ elapsed_ns) {
  __shared__ __align__(8) uint64_t never_a, never_b;
  __shared__ volatile int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&never_a), 1);
    mbar_init(smem_u32(&never_b), 1);
    fence_mbar_init();
  }
  __syncthreads();
  const uint64_t t0 = global_timer_ns();
  bool ok = true;
  if (lane == 0) {
    if (warp == 0) ok = mbar_wait_bounded(smem_u32(&never_a), 0, &abort_flag, limit_ns);
    else ok = mbar_wait_bounded(smem_u32(&never_b), 0, &abort_flag);
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (abort_flag || !ok) report(dev_status, NVFP4_DEVERR_TIMEOUT);
    if (elapsed_ns) *elapsed_ns = global_timer_ns() - t0;
  }
}

}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status_t nvfp4_wait_selftest(int64_t limit_ns, int32_t* dev_status,
                                              uint64_t* elapsed_ns, nvfp4_stream_t stream) {
  using namespace nvfp4;
  if (limit_ns <= 0 || limit_ns > (int64_t)NVFP4_WAIT_TIMEOUT_NS || dev_status == nullptr)
    return NVFP4_ERR_INVALID_ARG;
  wait_selftest_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns), dev_status, elapsed_ns);
  return check_launch("wait_selftest_kernel");
}
