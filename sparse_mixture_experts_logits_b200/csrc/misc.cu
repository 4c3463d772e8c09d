// Row gather (dispatch of x into expert order) and the standalone combine.
#include "kernels.cuh"

namespace moe {

// x_perm[s, :] = x[row_token[s], :]; one warp per row, 16-byte vectors.
__global__ void gather_rows_vec_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ row_token,
                                       uint4* __restrict__ x_perm, int rows, int vecs_per_row) {
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps_total) {
    const uint4* src = x + static_cast<size_t>(row_token[r]) * vecs_per_row;
    uint4* dst = x_perm + static_cast<size_t>(r) * vecs_per_row;
    for (int v = lane; v < vecs_per_row; v += 32) dst[v] = src[v];
  }
}

__global__ void gather_rows_f32_kernel(const float* __restrict__ x, const int32_t* __restrict__ row_token,
                                       float* __restrict__ x_perm, int rows, int D) {
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps_total) {
    const float* src = x + static_cast<size_t>(row_token[r]) * D;
    for (int d = lane; d < D; d += 32) x_perm[static_cast<size_t>(r) * D + d] = src[d];
  }
}

cudaError_t launch_gather_rows(const void* x, const int32_t* row_token, void* x_perm, int rows,
                               int D, int elem_bytes, cudaStream_t s) {
  const int blocks = min((rows + 7) / 8, 4 * num_sms());
  if ((static_cast<size_t>(D) * elem_bytes) % 16 == 0) {
    gather_rows_vec_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(x), row_token,
                                                  static_cast<uint4*>(x_perm), rows,
                                                  static_cast<int>(static_cast<size_t>(D) * elem_bytes / 16));
  } else {
    gather_rows_f32_kernel<<<blocks, 256, 0, s>>>(static_cast<const float*>(x), row_token,
                                                  static_cast<float*>(x_perm), rows, D);
  }
  return cudaGetLastError();
}

// y[t, :] = sum_j out_perm[slot_of[t, j], :] (+ shared[t, :]) in fp32, in
// slot order, rounded once.  out_perm is fp32; shared and y have the layer's
// type.  One block per token.
template <typename T>
__global__ void combine_kernel(const float* __restrict__ out_perm, const int32_t* __restrict__ slot_of,
                               const T* __restrict__ shared, T* __restrict__ y, int D, int k) {
  const int t = blockIdx.x;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int slot = slot_of[static_cast<size_t>(t) * k + j];
      acc += out_perm[static_cast<size_t>(slot) * D + d];
    }
    if (shared != nullptr) acc += to_f32(shared[static_cast<size_t>(t) * D + d]);
    y[static_cast<size_t>(t) * D + d] = from_f32<T>(acc);
  }
}

// bf16 output, 8 columns per thread.
__global__ void combine_bf16x8_kernel(const float4* __restrict__ out_perm,
                                      const int32_t* __restrict__ slot_of,
                                      const uint4* __restrict__ shared, uint4* __restrict__ y,
                                      int vecs, int k) {
  const int t = blockIdx.x;
  for (int v = threadIdx.x; v < vecs; v += blockDim.x) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < k; ++j) {
      const int slot = slot_of[static_cast<size_t>(t) * k + j];
      const float4 a = out_perm[(static_cast<size_t>(slot) * vecs + v) * 2];
      const float4 b = out_perm[(static_cast<size_t>(slot) * vecs + v) * 2 + 1];
      acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
      acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
    }
    if (shared != nullptr) {
      float f[8];
      bf16x8_to_f32(shared[static_cast<size_t>(t) * vecs + v], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += f[i];
    }
    y[static_cast<size_t>(t) * vecs + v] = f32_to_bf16x8(acc);
  }
}

cudaError_t launch_combine(int dtype, const void* out_perm, const int32_t* slot_of,
                           const void* shared_out, void* y, int T, int D, int k, cudaStream_t s) {
  const float* op = static_cast<const float*>(out_perm);
  if (dtype == MOE_DTYPE_BF16 && D % 8 == 0) {
    const int vecs = D / 8;
    combine_bf16x8_kernel<<<T, min(256, ((vecs + 31) / 32) * 32), 0, s>>>(
        reinterpret_cast<const float4*>(op), slot_of, static_cast<const uint4*>(shared_out),
        static_cast<uint4*>(y), vecs, k);
  } else if (dtype == MOE_DTYPE_BF16) {
    combine_kernel<__nv_bfloat16><<<T, 256, 0, s>>>(op, slot_of,
                                                    static_cast<const __nv_bfloat16*>(shared_out),
                                                    static_cast<__nv_bfloat16*>(y), D, k);
  } else {
    combine_kernel<float><<<T, 256, 0, s>>>(op, slot_of, static_cast<const float*>(shared_out),
                                            static_cast<float*>(y), D, k);
  }
  return cudaGetLastError();
}

}  // namespace moe
