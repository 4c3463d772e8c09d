// moe_selftest_wait_timeout: runs the library's bounded mbarrier wait on a
// barrier that nothing ever arrives on, so that the expiry branch of every
// kernel's waits (record MOE_DEVERR_TIMEOUT, raise the abort flag that the
// other roles poll, return) can be exercised on a GPU without a fault or a
// hang.  The context stays usable afterwards.
#include "kernels.cuh"

namespace moe {
namespace {

// Warp 0 waits with the given limit and gives up on the time limit; warp 1
// waits on a second barrier with four times that limit and must leave early,
// on the abort flag that warp 0 raised.  elapsed[w] = nanoseconds warp w waited,
// with bit 63 set if its wait returned true (it never should).
__global__ void __launch_bounds__(64, 1) wait_selftest_kernel(uint64_t limit_ns, int* status,
                                                             unsigned long long* elapsed) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(smem_addr(&bar[0]), 1);
    mbar_init(smem_addr(&bar[1]), 1);
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();
  const uint64_t t0 = globaltimer_ns();
  const uint64_t lim = warp == 0 ? limit_ns : 4 * limit_ns;
  const bool ok = mbar_wait_all(smem_addr(&bar[warp]), 0, &s_abort, status, lim);
  const uint64_t t1 = globaltimer_ns();
  if ((threadIdx.x & 31) == 0 && elapsed != nullptr)
    elapsed[warp] = (t1 - t0) | (ok ? (1ull << 63) : 0ull);
}

}  // namespace
}  // namespace moe

extern "C" moe_status_t moe_selftest_wait_timeout(uint64_t limit_ns, int32_t* device_status,
                                                  uint64_t* elapsed_ns, void* stream) {
  using namespace moe;
  if (device_status == nullptr || limit_ns < 1000 || limit_ns > kWaitTimeoutNs) return MOE_ERR_INVALID_ARG;
  const moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(device_status, 0, sizeof(int32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  wait_selftest_kernel<<<1, 64, 0, s>>>(limit_ns, device_status,
                                        reinterpret_cast<unsigned long long*>(elapsed_ns));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
