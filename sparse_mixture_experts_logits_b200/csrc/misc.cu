// Row gather (dispatch of x into expert order) and the standalone combine.
#include <algorithm>

#include "kernels.cuh"

namespace moe {

// x_perm[s, :] = x[row_token[s], :]; one warp per row, 16-byte vectors.
// Rows r < min(rows, *n_rows) are gathered (n_rows = offsets[M] of the
// dispatch, which is below T*k when pairs were dropped through the sentinel
// index); a token index outside [0, T) is reported and its row zero-filled.
__device__ __forceinline__ int gather_limit(const int32_t* n_rows, int rows) {
  return n_rows ? max(0, min(rows, *n_rows)) : rows;
}

__global__ void gather_rows_vec_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ row_token,
                                       const int32_t* __restrict__ n_rows, uint4* __restrict__ x_perm,
                                       int rows, int T, int vecs_per_row, int* status) {
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int n = gather_limit(n_rows, rows);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps_total) {
    const int tok = row_token[r];
    uint4* dst = x_perm + static_cast<size_t>(r) * vecs_per_row;
    if (tok < 0 || tok >= T) {
      if (lane == 0) set_status(status, MOE_DEVERR_BAD_ROW_TOKEN);
      for (int v = lane; v < vecs_per_row; v += 32) dst[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4* src = x + static_cast<size_t>(tok) * vecs_per_row;
    for (int v = lane; v < vecs_per_row; v += 32) dst[v] = src[v];
  }
}

__global__ void gather_rows_f32_kernel(const float* __restrict__ x, const int32_t* __restrict__ row_token,
                                       const int32_t* __restrict__ n_rows, float* __restrict__ x_perm,
                                       int rows, int T, int D, int* status) {
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  const int n = gather_limit(n_rows, rows);
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n; r += warps_total) {
    const int tok = row_token[r];
    const bool ok = tok >= 0 && tok < T;
    if (!ok && lane == 0) set_status(status, MOE_DEVERR_BAD_ROW_TOKEN);
    const float* src = x + static_cast<size_t>(ok ? tok : 0) * D;
    for (int d = lane; d < D; d += 32) x_perm[static_cast<size_t>(r) * D + d] = ok ? src[d] : 0.f;
  }
}

// The same rows written the other way round: token t's row is read once and
// stored at its k dispatch positions slot_of[t, j] (sentinel pairs, slot < 0,
// are skipped; a slot >= rows is reported and skipped).  Each x row is read
// from memory once instead of k times.
__global__ void scatter_rows_vec_kernel(const uint4* __restrict__ x, const int32_t* __restrict__ slot_of,
                                        uint4* __restrict__ x_perm, int T, int k, int rows,
                                        int vecs_per_row, int* status) {
  const int warps_total = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T; t += warps_total) {
    int my_slot = -1;
    if (lane < k) {
      my_slot = slot_of[static_cast<size_t>(t) * k + lane];
      if (my_slot >= rows) {
        set_status(status, MOE_DEVERR_BAD_ROW_TOKEN);
        my_slot = -1;
      }
    }
    const uint4* src = x + static_cast<size_t>(t) * vecs_per_row;
    for (int v = lane; v < vecs_per_row; v += 32) {
      const uint4 val = src[v];
      for (int j = 0; j < k; ++j) {
        const int slot = __shfl_sync(0xffffffffu, my_slot, j);
        if (slot >= 0) x_perm[static_cast<size_t>(slot) * vecs_per_row + v] = val;
      }
    }
  }
}

cudaError_t launch_scatter_rows(const void* x, const int32_t* slot_of, void* x_perm, int T, int k, int D,
                                int* status, cudaStream_t s) {
  const int blocks = std::max(1, std::min((T + 7) / 8, 4 * num_sms()));
  scatter_rows_vec_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(x), slot_of,
                                                 static_cast<uint4*>(x_perm), T, k, T * k, D / 8, status);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* x, const int32_t* row_token, const int32_t* n_rows, void* x_perm,
                               int rows, int T, int D, int elem_bytes, int* status, cudaStream_t s) {
  const int blocks = max(1, min((rows + 7) / 8, 4 * num_sms()));
  if ((static_cast<size_t>(D) * elem_bytes) % 16 == 0) {
    gather_rows_vec_kernel<<<blocks, 256, 0, s>>>(static_cast<const uint4*>(x), row_token, n_rows,
                                                  static_cast<uint4*>(x_perm), rows, T,
                                                  static_cast<int>(static_cast<size_t>(D) * elem_bytes / 16),
                                                  status);
  } else {
    gather_rows_f32_kernel<<<blocks, 256, 0, s>>>(static_cast<const float*>(x), row_token, n_rows,
                                                  static_cast<float*>(x_perm), rows, T, D, status);
  }
  return cudaGetLastError();
}

// y[t, :] = sum_j out_perm[slot_of[t, j], :] (+ shared[t, :]) (+ addend[t, :]) in fp32, in
// slot order (slots < 0, sentinel pairs, add nothing), rounded once.  out_perm is fp32; shared is fp32 or the layer's
// type; y has the layer's type.  Block (token, 128 four-column groups); every
// row read is contiguous, and the k rows of a token are loaded together.
template <typename TY, typename TS>
__global__ void __launch_bounds__(128) combine_vec4_kernel(const float4* __restrict__ out_perm,
                                                           const int32_t* __restrict__ slot_of,
                                                           const TS* __restrict__ shared,
                                                           const TY* __restrict__ addend, TY* __restrict__ y,
                                                           int D4, int k) {
  __shared__ int s_slot[kMaxTopK];
  const int t = blockIdx.x;
  if (threadIdx.x < k) s_slot[threadIdx.x] = slot_of[static_cast<size_t>(t) * k + threadIdx.x];
  __syncthreads();
  for (int v = blockIdx.y * blockDim.x + threadIdx.x; v < D4; v += blockDim.x * gridDim.y) {
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
    for (int j = 0; j < k; ++j) {
      if (s_slot[j] < 0) continue;  // sentinel pair
      const float4 a = out_perm[static_cast<size_t>(s_slot[j]) * D4 + v];
      acc.x += a.x; acc.y += a.y; acc.z += a.z; acc.w += a.w;
    }
    if (shared != nullptr) {
      const size_t e = (static_cast<size_t>(t) * D4 + v) * 4;
      acc.x += to_f32(shared[e]); acc.y += to_f32(shared[e + 1]);
      acc.z += to_f32(shared[e + 2]); acc.w += to_f32(shared[e + 3]);
    }
    if (addend != nullptr) {
      const size_t e = (static_cast<size_t>(t) * D4 + v) * 4;
      acc.x += to_f32(addend[e]); acc.y += to_f32(addend[e + 1]);
      acc.z += to_f32(addend[e + 2]); acc.w += to_f32(addend[e + 3]);
    }
    const size_t o = (static_cast<size_t>(t) * D4 + v) * 4;
    if constexpr (sizeof(TY) == 2) {
      __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
      uint2 u;
      u.x = *reinterpret_cast<uint32_t*>(&lo);
      u.y = *reinterpret_cast<uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(y + o) = u;
    } else {
      *reinterpret_cast<float4*>(y + o) = acc;
    }
  }
}

// Any D: one element per thread step.
template <typename TY, typename TS>
__global__ void combine_kernel(const float* __restrict__ out_perm, const int32_t* __restrict__ slot_of,
                               const TS* __restrict__ shared, const TY* __restrict__ addend,
                               TY* __restrict__ y, int D, int k) {
  const int t = blockIdx.x;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    for (int j = 0; j < k; ++j) {
      const int slot = slot_of[static_cast<size_t>(t) * k + j];
      if (slot >= 0) acc += out_perm[static_cast<size_t>(slot) * D + d];
    }
    if (shared != nullptr) acc += to_f32(shared[static_cast<size_t>(t) * D + d]);
    if (addend != nullptr) acc += to_f32(addend[static_cast<size_t>(t) * D + d]);
    y[static_cast<size_t>(t) * D + d] = from_f32<TY>(acc);
  }
}

template <typename TY, typename TS>
static cudaError_t combine_typed(const float* op, const int32_t* slot_of, const void* shared,
                                 const void* addend, void* y, int T, int D, int k, cudaStream_t s) {
  if (D % 4 == 0) {
    // few tokens: spread a row's columns over blocks too
    dim3 grid(T, T >= 1024 ? 1 : (D / 4 + 127) / 128);
    combine_vec4_kernel<TY, TS><<<grid, 128, 0, s>>>(reinterpret_cast<const float4*>(op), slot_of,
                                                  static_cast<const TS*>(shared), static_cast<const TY*>(addend),
                                                  static_cast<TY*>(y), D / 4, k);
  } else {
    combine_kernel<TY, TS><<<T, 128, 0, s>>>(op, slot_of, static_cast<const TS*>(shared),
                                             static_cast<const TY*>(addend), static_cast<TY*>(y), D, k);
  }
  return cudaGetLastError();
}

cudaError_t launch_combine(int dtype, const void* out_perm, const int32_t* slot_of,
                           const void* shared_out, bool shared_f32, const void* addend, void* y, int T,
                           int D, int k, cudaStream_t s) {
  const float* op = static_cast<const float*>(out_perm);
  if (dtype == MOE_DTYPE_BF16) {
    return shared_f32
               ? combine_typed<__nv_bfloat16, float>(op, slot_of, shared_out, addend, y, T, D, k, s)
               : combine_typed<__nv_bfloat16, __nv_bfloat16>(op, slot_of, shared_out, addend, y, T, D, k, s);
  }
  return combine_typed<float, float>(op, slot_of, shared_out, addend, y, T, D, k, s);
}

}  // namespace moe
