// Helpers of the tensor-core backward of bf16 layers.
//
// The weight-gradient GEMMs contract over each expert's rows in 64-row
// k-blocks, so the backward keeps its per-row tensors in a padded dispatch
// order: expert e's rows start at offsets_pad[e] = sum over e' < e of
// ceil64(counts[e']), in the same (slot j, token t) order as the forward's
// dispatch, and the padding rows are zero in every tensor a weight-gradient
// GEMM reads.  These kernels build that order, gather rows into it, zero the
// padding, finish the gate-weight gradients from the GEMM's partial dot
// products, take per-expert column sums, and zero the weight gradients of
// experts that received no rows.
#include <algorithm>

#include "kernels.cuh"

namespace moe {
namespace {

inline int grid_for(long long n, int threads) {
  const long long b = (n + threads - 1) / threads;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(b, 8ll * num_sms())));
}

// offsets_pad[0] = 0, offsets_pad[e + 1] = sum_{e' <= e} ceil64(counts[e']); one block of 1024.
__global__ void __launch_bounds__(1024) pad_offsets_kernel(const int32_t* __restrict__ counts, int M,
                                                           int32_t* __restrict__ offsets_pad) {
  __shared__ int s[1024];
  const int i = threadIdx.x;
  s[i] = i < M ? ((max(counts[i], 0) + 63) & ~63) : 0;
  __syncthreads();
  for (int d = 1; d < 1024; d <<= 1) {
    const int t = i >= d ? s[i - d] : 0;
    __syncthreads();
    s[i] += t;
    __syncthreads();
  }
  if (i < M) offsets_pad[i + 1] = s[i];
  if (i == 0) offsets_pad[0] = 0;
}

// Pair (t, j) at dispatch position p = slot_of[t, j] (expert e = idx[t, j])
// moves to q = p - offsets[e] + offsets_pad[e]; sentinel pairs get -1.
__global__ void pad_pairs_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ slot_of,
                                 const float* __restrict__ topk_w, const int32_t* __restrict__ offsets,
                                 const int32_t* __restrict__ offsets_pad, long long pairs, int k, int M,
                                 long long rows_cap, int32_t* __restrict__ slot_pad,
                                 int32_t* __restrict__ row_token_pad, float* __restrict__ row_w_pad) {
  for (long long pr = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; pr < pairs;
       pr += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int p = slot_of[pr];
    const int e = idx[pr];
    if (p < 0 || e < 0 || e >= M) {
      slot_pad[pr] = -1;
      continue;
    }
    const long long q = static_cast<long long>(p) - offsets[e] + offsets_pad[e];
    if (q < 0 || q >= rows_cap) {
      slot_pad[pr] = -1;
      continue;
    }
    slot_pad[pr] = static_cast<int32_t>(q);
    row_token_pad[q] = static_cast<int32_t>(pr / k);
    row_w_pad[q] = topk_w[pr];
  }
}

// dst[r] = src[row_token_pad[r]] for r < offsets_pad[M]; a padding row (token
// -1) is written as zeros.  Warp per row, 16-byte vectors.
__global__ void gather_pad_kernel(const uint4* __restrict__ src, const int32_t* __restrict__ row_token_pad,
                                  const int32_t* __restrict__ n_rows, uint4* __restrict__ dst, long long rows_cap,
                                  int T, int vecs) {
  const int lane = threadIdx.x & 31;
  const long long n = min(rows_cap, static_cast<long long>(max(*n_rows, 0)));
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long r = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < n; r += warps) {
    const int tok = row_token_pad[r];
    uint4* d = dst + r * vecs;
    if (tok < 0 || tok >= T) {
      for (int v = lane; v < vecs; v += 32) d[v] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    }
    const uint4* s = src + static_cast<long long>(tok) * vecs;
    for (int v = lane; v < vecs; v += 32) d[v] = s[v];
  }
}

// Zero the padding rows [offsets_pad[e] + counts[e], offsets_pad[e + 1]) of a
// [rows, vecs x 16 B] buffer; blockIdx.x is the expert, blockIdx.y a share of its rows.
__global__ void zero_pad_rows_kernel(const int32_t* __restrict__ counts, const int32_t* __restrict__ offsets_pad,
                                     uint4* __restrict__ buf, long long rows_cap, int vecs) {
  const int e = blockIdx.x;
  const long long r0 = min(rows_cap, static_cast<long long>(offsets_pad[e]) + max(counts[e], 0));
  const long long r1 = min(rows_cap, static_cast<long long>(offsets_pad[e + 1]));
  const long long n = (r1 - r0) * vecs;
  for (long long i = static_cast<long long>(blockIdx.y) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.y) * blockDim.x)
    buf[r0 * vecs + i] = make_uint4(0u, 0u, 0u, 0u);
}

// dw[t, j] = sum_p parts[q, p] (+ <dy_t, b2_e>) with q = slot_pad[t, j], in a
// fixed order; 0 for a sentinel pair.  Warp per pair.
__global__ void dw_finish_kernel(const float* __restrict__ parts, int nparts, const int32_t* __restrict__ slot_pad,
                                 const int32_t* __restrict__ idx, const __nv_bfloat16* __restrict__ dy,
                                 const __nv_bfloat16* __restrict__ b2, int D, int M, long long pairs, int k,
                                 float* __restrict__ dw) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long pr = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; pr < pairs;
       pr += warps) {
    const int q = slot_pad[pr];
    if (q < 0) {
      if (lane == 0) dw[pr] = 0.f;
      continue;
    }
    float s = 0.f;
    for (int p = lane; p < nparts; p += 32) s += parts[static_cast<long long>(q) * nparts + p];
    const int e = idx[pr];
    if (b2 != nullptr && e >= 0 && e < M) {
      const __nv_bfloat16* dyt = dy + (pr / k) * D;
      const __nv_bfloat16* be = b2 + static_cast<long long>(e) * D;
      for (int d = lane; d < D; d += 32) s = fmaf(__bfloat162float(dyt[d]), __bfloat162float(be[d]), s);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) dw[pr] = s;
  }
}

// out[g, n] = sum over rows [offsets[g], offsets[g+1]) of scale[r] Y[r, n]
// (scale = 1 when null), bf16 Y, fp32 sums in row order.
__global__ void colsum_bf16_kernel(const __nv_bfloat16* __restrict__ Y, long long ldy,
                                   const float* __restrict__ scale, const int32_t* __restrict__ offsets,
                                   long long rows_cap, int N, float* __restrict__ out) {
  const int g = blockIdx.y;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const long long b = min(rows_cap, static_cast<long long>(max(offsets[g], 0)));
  const long long e = min(rows_cap, static_cast<long long>(max(offsets[g + 1], 0)));
  float s = 0.f;
  for (long long r = b; r < e; ++r) {
    const float v = __bfloat162float(Y[r * ldy + n]);
    s = scale != nullptr ? fmaf(scale[r], v, s) : s + v;
  }
  out[static_cast<long long>(g) * N + n] = s;
}

// The same sums, two columns per thread (N and ldy even, Y 4-byte aligned):
// each warp reads 128 contiguous bytes of a row, and the loads of 16 rows are
// issued before any of them is added, so that a thread keeps 16 requests in
// flight instead of one.  Each column still adds its rows one by one in row
// order, so the sums are the scalar kernel's bit for bit.
__global__ void colsum_bf16x2_kernel(const __nv_bfloat162* __restrict__ Y, long long ldy2,
                                     const float* __restrict__ scale, const int32_t* __restrict__ offsets,
                                     long long rows_cap, int N2, float2* __restrict__ out) {
  constexpr int kRows = 16;
  const int g = blockIdx.y;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N2) return;
  const long long b = min(rows_cap, static_cast<long long>(max(offsets[g], 0)));
  const long long e = min(rows_cap, static_cast<long long>(max(offsets[g + 1], 0)));
  float s0 = 0.f, s1 = 0.f;
  long long r = b;
  for (; r + kRows <= e; r += kRows) {
    __nv_bfloat162 v[kRows];
#pragma unroll
    for (int i = 0; i < kRows; ++i) v[i] = Y[(r + i) * ldy2 + n];
#pragma unroll
    for (int i = 0; i < kRows; ++i) {
      const float2 f = __bfloat1622float2(v[i]);
      if (scale != nullptr) {
        const float c = scale[r + i];
        s0 = fmaf(c, f.x, s0);
        s1 = fmaf(c, f.y, s1);
      } else {
        s0 += f.x;
        s1 += f.y;
      }
    }
  }
  for (; r < e; ++r) {
    const float2 f = __bfloat1622float2(Y[r * ldy2 + n]);
    if (scale != nullptr) {
      const float c = scale[r];
      s0 = fmaf(c, f.x, s0);
      s1 = fmaf(c, f.y, s1);
    } else {
      s0 += f.x;
      s1 += f.y;
    }
  }
  out[static_cast<long long>(g) * N2 + n] = make_float2(s0, s1);
}

// out[g, :] = 0 (per_group floats) for every g with counts[g] == 0.
__global__ void zero_empty_groups_kernel(const int32_t* __restrict__ counts, long long per_group,
                                         float* __restrict__ out) {
  const int g = blockIdx.y;
  if (counts[g] != 0) return;
  float* o = out + static_cast<long long>(g) * per_group;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < per_group;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    o[i] = 0.f;
}

}  // namespace

cudaError_t launch_pad_dispatch(const int32_t* idx, const int32_t* slot_of, const float* topk_w,
                                const int32_t* counts, const int32_t* offsets, int T, int k, int M,
                                long long rows_cap, int32_t* offsets_pad, int32_t* slot_pad,
                                int32_t* row_token_pad, float* row_w_pad, cudaStream_t s) {
  if (M < 1 || M > 1024) return cudaErrorInvalidValue;
  if (cudaMemsetAsync(row_token_pad, 0xFF, static_cast<size_t>(rows_cap) * 4, s) != cudaSuccess ||
      cudaMemsetAsync(row_w_pad, 0, static_cast<size_t>(rows_cap) * 4, s) != cudaSuccess)
    return cudaErrorUnknown;
  pad_offsets_kernel<<<1, 1024, 0, s>>>(counts, M, offsets_pad);
  const long long pairs = static_cast<long long>(T) * k;
  if (pairs > 0)
    pad_pairs_kernel<<<grid_for(pairs, 256), 256, 0, s>>>(idx, slot_of, topk_w, offsets, offsets_pad, pairs, k, M,
                                                           rows_cap, slot_pad, row_token_pad, row_w_pad);
  return cudaGetLastError();
}

cudaError_t launch_gather_pad(const void* src, const int32_t* row_token_pad, const int32_t* n_rows, void* dst,
                              long long rows_cap, int T, int D, cudaStream_t s) {
  if (rows_cap <= 0) return cudaSuccess;
  if (D % 8 != 0) return cudaErrorInvalidValue;
  gather_pad_kernel<<<grid_for(rows_cap * 32, 256), 256, 0, s>>>(static_cast<const uint4*>(src), row_token_pad,
                                                                 n_rows, static_cast<uint4*>(dst), rows_cap, T,
                                                                 D / 8);
  return cudaGetLastError();
}

cudaError_t launch_zero_pad_rows(const int32_t* counts, const int32_t* offsets_pad, int M, void* buf,
                                 long long rows_cap, int cols_bf16, cudaStream_t s) {
  if (M <= 0) return cudaSuccess;
  if (cols_bf16 % 8 != 0) return cudaErrorInvalidValue;
  // A group pads at most 63 rows: 16 blocks per group cover them in a few
  // rounds of 16-byte stores (one block per group left the stores waiting
  // one after another).
  zero_pad_rows_kernel<<<dim3(M, 16), 256, 0, s>>>(counts, offsets_pad, static_cast<uint4*>(buf), rows_cap,
                                                   cols_bf16 / 8);
  return cudaGetLastError();
}

cudaError_t launch_dw_finish(const float* parts, int nparts, const int32_t* slot_pad, const int32_t* idx,
                             const void* dy, const void* b2, int D, int M, int T, int k, float* dw, cudaStream_t s) {
  const long long pairs = static_cast<long long>(T) * k;
  if (pairs <= 0) return cudaSuccess;
  dw_finish_kernel<<<grid_for(pairs * 32, 256), 256, 0, s>>>(parts, nparts, slot_pad, idx,
                                                            static_cast<const __nv_bfloat16*>(dy),
                                                            static_cast<const __nv_bfloat16*>(b2), D, M, pairs, k, dw);
  return cudaGetLastError();
}

cudaError_t launch_colsum_bf16(const void* Y, long long ldy, const float* scale, const int32_t* offsets, int G,
                               long long rows_cap, int N, float* out, cudaStream_t s) {
  if (G <= 0 || N <= 0) return cudaSuccess;
  if (G > 65535) return cudaErrorInvalidValue;
  if (N % 2 == 0 && ldy % 2 == 0 && reinterpret_cast<uintptr_t>(Y) % 4 == 0 &&
      reinterpret_cast<uintptr_t>(out) % 8 == 0) {
    dim3 grid((N / 2 + 255) / 256, G);
    colsum_bf16x2_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat162*>(Y), ldy / 2, scale, offsets,
                                              rows_cap, N / 2, reinterpret_cast<float2*>(out));
    return cudaGetLastError();
  }
  dim3 grid((N + 255) / 256, G);
  colsum_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(Y), ldy, scale, offsets, rows_cap, N,
                                          out);
  return cudaGetLastError();
}

cudaError_t launch_zero_empty_groups(const int32_t* counts, int G, long long per_group, float* out, cudaStream_t s) {
  if (G <= 0 || per_group <= 0) return cudaSuccess;
  if (G > 65535) return cudaErrorInvalidValue;
  dim3 grid(static_cast<unsigned>(std::min<long long>(64, (per_group + 255) / 256)), G);
  zero_empty_groups_kernel<<<grid, 256, 0, s>>>(counts, per_group, out);
  return cudaGetLastError();
}

}  // namespace moe
