// Expert capacity: a pair whose rank inside its expert's dispatch segment is
// at or past the capacity becomes the "no expert" sentinel M.
#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

// One thread per (token, slot) pair p; each thread reads and writes only idx[p].
__global__ void capacity_drop_kernel(int32_t* __restrict__ idx, const int32_t* __restrict__ slot_of,
                                     const int32_t* __restrict__ offsets, long long pairs, int M, int capacity) {
  for (long long p = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; p < pairs;
       p += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int e = idx[p];
    if (e < 0 || e >= M) continue;  // already the sentinel (or invalid: left for moe_permute to report)
    const int s = slot_of[p];
    if (s < 0) continue;
    if (s - offsets[e] >= capacity) idx[p] = M;
  }
}

}  // namespace

cudaError_t launch_capacity_drop(int32_t* idx, const int32_t* slot_of, const int32_t* offsets, int T, int k, int M,
                                 int capacity, cudaStream_t s) {
  const long long pairs = static_cast<long long>(T) * k;
  if (pairs <= 0) return cudaSuccess;
  const int blocks = static_cast<int>(std::min<long long>((pairs + 255) / 256, 8ll * num_sms()));
  capacity_drop_kernel<<<blocks, 256, 0, s>>>(idx, slot_of, offsets, pairs, M, capacity);
  return cudaGetLastError();
}

}  // namespace moe
