// Fixed-split expert-parallel exchange: the sender packs its dispatch order
// into M blocks of `cap` rows (one per expert, so the E blocks of each owner
// rank are one contiguous piece of E * cap rows), and the receiver turns the
// [world][E][cap] blocks it gets back into an expert-major dispatch order.
// Every split is E * cap rows whatever the routing, so the all-to-alls need
// no row counts on the host and the step runs without a device-to-host read.
//
// The pages name the cost this exchange carries (the GLaM industry article,
// first route: cross-node communication between expert "buildings"; second
// route: fine-grained expert parallelism).  They give no capacity rule: the
// one used is moe_capacity_drop's, an expert keeping the first `cap` of its
// pairs in dispatch order.
#include <algorithm>

#include "kernels.cuh"

namespace {

using moe::set_status;

// One warp per packed row r = e * cap + i: the i-th row of expert e's
// segment of the dispatch order if it has one, else a zero row.  Also the
// row's gate weight (0 on padding) and, from each expert's row 0, kept[e].
template <typename V>
__global__ void ep_pack_rows_kernel(const V* __restrict__ x, const int32_t* __restrict__ offsets,
                                    const int32_t* __restrict__ row_token, const float* __restrict__ row_w,
                                    int T, int M, int cap, int vecs_per_row, V* __restrict__ x_pad,
                                    float* __restrict__ w_pad, int32_t* __restrict__ kept, int* status) {
  const long long rows = static_cast<long long>(M) * cap;
  const long long warps_total = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (long long r = static_cast<long long>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += warps_total) {
    const int e = static_cast<int>(r / cap);
    const int i = static_cast<int>(r - static_cast<long long>(e) * cap);
    const int o0 = offsets[e];
    const int n = max(0, offsets[e + 1] - o0);
    V* dst = x_pad + r * vecs_per_row;
    int tok = -1;
    float w = 0.f;
    if (i < n) {
      tok = row_token[o0 + i];
      w = row_w[o0 + i];
      if (tok < 0 || tok >= T) {
        if (lane == 0) set_status(status, MOE_DEVERR_BAD_ROW_TOKEN);
        tok = -1;
        w = 0.f;
      }
    }
    if (tok >= 0) {
      const V* src = x + static_cast<long long>(tok) * vecs_per_row;
      for (int v = lane; v < vecs_per_row; v += 32) dst[v] = src[v];
    } else {
      for (int v = lane; v < vecs_per_row; v += 32) dst[v] = V{};
    }
    if (lane == 0) {
      w_pad[r] = w;
      if (i == 0) kept[e] = min(n, cap);
    }
  }
}

// Packed position of every pair: slot s of expert e (offsets[e] <= s <
// offsets[e + 1]) goes to e * cap + (s - offsets[e]) when that is below the
// capacity, else the pair is dropped (-1); sentinel pairs (s < 0) stay -1.
__global__ void ep_pack_slots_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ slot_of,
                                     long long pairs, int M, int cap, int32_t* __restrict__ slot_pad,
                                     int* status) {
  const int n_rows = offsets[M];
  for (long long p = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; p < pairs;
       p += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int s = slot_of[p];
    int out = -1;
    if (s >= n_rows) {
      set_status(status, MOE_DEVERR_BAD_ROW_TOKEN);
    } else if (s >= 0) {
      int lo = 0, hi = M - 1;  // the last expert whose segment starts at or before s
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (offsets[mid] <= s) lo = mid; else hi = mid - 1;
      }
      const int i = s - offsets[lo];
      if (i < cap) out = lo * cap + i;
    }
    slot_pad[p] = out;
  }
}

// Block b = e * world + q handles the rows that source rank q sent for local
// expert e, i.e. arrival block (q, e) = rows (q * E + e) * cap + [0, cap).
// Its place in the expert-major dispatch order starts after every block of
// the experts before e and the blocks of e from ranks before q.
__global__ void __launch_bounds__(256) ep_unpack_kernel(const int32_t* __restrict__ recv_kept,
                                                        const float* __restrict__ w_recv, int world, int E,
                                                        int cap, int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ row_token,
                                                        float* __restrict__ row_w, int32_t* __restrict__ slot_of,
                                                        int* status) {
  __shared__ int s_part[8];
  const int e = static_cast<int>(blockIdx.x) / world;
  const int q = static_cast<int>(blockIdx.x) - e * world;
  // base = sum of the kept rows of the blocks ordered before (q, e)
  int part = 0;
  for (int j = threadIdx.x; j < world * E; j += blockDim.x) {
    const int qq = j / E, ee = j - qq * E;
    if (ee < e || (ee == e && qq < q)) part += max(0, min(recv_kept[j], cap));
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = part;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) base += s_part[w];
  const int raw = recv_kept[q * E + e];
  const int n = max(0, min(raw, cap));
  if (threadIdx.x == 0) {
    if (raw != n) set_status(status, MOE_DEVERR_BAD_COUNT);
    if (q == 0) offsets[e] = base;
    if (q == world - 1 && e == E - 1) offsets[E] = base + n;
  }
  const long long r0 = (static_cast<long long>(q) * E + e) * cap;
  for (int i = threadIdx.x; i < cap; i += blockDim.x) {
    const long long r = r0 + i;
    if (i < n) {
      row_token[base + i] = static_cast<int32_t>(r);
      row_w[base + i] = w_recv[r];
      slot_of[r] = base + i;
    } else {
      slot_of[r] = -1;
    }
  }
}

}  // namespace

extern "C" moe_status_t moe_ep_pack(const void* x, const int32_t* offsets, const int32_t* row_token,
                                    const float* row_w, const int32_t* slot_of, int T, int k, int M, int D,
                                    int dtype, int cap, void* x_pad, float* w_pad, int32_t* slot_pad,
                                    int32_t* kept, int32_t* device_status, void* stream) {
  using namespace moe;
  if (T < 0 || k < 1 || M < 1 || D < 1 || cap < 0) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_F32 && dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (M > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(M) * cap;
  const long long pairs = static_cast<long long>(T) * k;
  if (rows >= (1ll << 31) || pairs >= (1ll << 31) || rows * D >= (1ll << 40)) return MOE_ERR_UNSUPPORTED;
  if (!offsets || !kept) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && (!x_pad || !w_pad)) return MOE_ERR_INVALID_ARG;
  if (pairs > 0 && (!x || !row_token || !row_w || !slot_of || !slot_pad)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (device_status != nullptr && cudaMemsetAsync(device_status, 0, sizeof(int32_t), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  const size_t esize = dtype == MOE_DTYPE_BF16 ? 2 : 4;
  const size_t row_bytes = static_cast<size_t>(D) * esize;
  if (cap == 0) {
    if (cudaMemsetAsync(kept, 0, static_cast<size_t>(M) * 4, s) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    const int blocks = static_cast<int>(std::min<long long>((rows + 7) / 8, 148ll * 16));
    const bool vec = row_bytes % 16 == 0 && reinterpret_cast<uintptr_t>(x) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(x_pad) % 16 == 0;
    if (vec) {
      ep_pack_rows_kernel<uint4><<<blocks, 256, 0, s>>>(
          static_cast<const uint4*>(x), offsets, row_token, row_w, T, M, cap, static_cast<int>(row_bytes / 16),
          static_cast<uint4*>(x_pad), w_pad, kept, device_status);
    } else if (esize == 2) {
      ep_pack_rows_kernel<uint16_t><<<blocks, 256, 0, s>>>(
          static_cast<const uint16_t*>(x), offsets, row_token, row_w, T, M, cap, D,
          static_cast<uint16_t*>(x_pad), w_pad, kept, device_status);
    } else {
      ep_pack_rows_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(x), offsets, row_token, row_w,
                                                        T, M, cap, D, static_cast<float*>(x_pad), w_pad, kept,
                                                        device_status);
    }
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  if (pairs > 0) {
    const int blocks = static_cast<int>(std::min<long long>((pairs + 255) / 256, 148ll * 8));
    ep_pack_slots_kernel<<<blocks, 256, 0, s>>>(offsets, slot_of, pairs, M, cap, slot_pad, device_status);
    if (cudaGetLastError() != cudaSuccess) return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

extern "C" moe_status_t moe_ep_unpack(const int32_t* recv_kept, const float* w_recv, int world, int E, int cap,
                                      int32_t* offsets, int32_t* row_token, float* row_w, int32_t* slot_of,
                                      int32_t* device_status, void* stream) {
  using namespace moe;
  if (world < 1 || E < 1 || cap < 0) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(world) * E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  const long long rows = static_cast<long long>(world) * E * cap;
  if (rows >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (!recv_kept || !offsets) return MOE_ERR_INVALID_ARG;
  if (rows > 0 && (!w_recv || !row_token || !row_w || !slot_of)) return MOE_ERR_INVALID_ARG;
  moe_status_t st = check_device();
  if (st != MOE_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (device_status != nullptr && cudaMemsetAsync(device_status, 0, sizeof(int32_t), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  ep_unpack_kernel<<<world * E, 256, 0, s>>>(recv_kept, w_recv, world, E, cap, offsets, row_token, row_w, slot_of,
                                             device_status);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
