// Dispatch: a deterministic counting sort of the T*k (token, slot) pairs by
// expert.
//
// The GLM-5 page's GlmMoeDsaExperts.forward builds the expert mask
// one_hot(top_k_index, M + 1).permute(2, 1, 0) of shape [M + 1, k, T], lists
// expert e's pairs with torch.where, i.e. in (slot j, token t) order, and
// skips class M, the "no expert" sentinel.  Here too a pair whose index is M
// is dispatched nowhere (slot_of = -1); an index outside [0, M] is reported
// through the status flag and skipped the same way.  Placing the
// experts' lists end to end is a stable sort by expert of the pairs taken in
// j-major order p = j*T + t.  The three kernels below compute it without
// any atomic operation deciding an order:
//   1. per chunk of kPermChunk consecutive p: a histogram of experts
//      (shared-memory counters; a count does not depend on order);
//   2. per expert: exclusive scan of its chunk counts -> chunk_base, total;
//   3. per chunk: offsets = scan of the totals; inside the chunk each pair's
//      rank among equal experts comes from warp match/ballot masks plus the
//      counts of the earlier warps, so slot = offsets[e] + chunk_base + rank.
#include "kernels.cuh"

namespace moe {

constexpr int kPermThreads = kPermChunk;  // one pair per thread
constexpr int kPermWarps = kPermThreads / 32;

// Exclusive scan of in[0..n) into out[0..n) by the whole block (blockDim.x a
// multiple of 32); returns the total to every thread.  `in` and `out` may
// be global or shared memory; s_tmp holds 33 ints of shared memory.
__device__ int block_exclusive_scan(const int* in, int* out, int n, int* s_tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nwarps = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int beg = min(n, tid * per), end = min(n, beg + per);
  int local = 0;
  for (int i = beg; i < end; ++i) local += in[i];
  int incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += t;
  }
  if (lane == 31) s_tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < nwarps ? s_tmp[lane] : 0;
    int wi = v;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, wi, d);
      if (lane >= d) wi += t;
    }
    if (lane < nwarps) s_tmp[lane] = wi - v;
    if (lane == 31) s_tmp[32] = wi;
  }
  __syncthreads();
  int run = s_tmp[warp] + incl - local;
  for (int i = beg; i < end; ++i) {
    const int v = in[i];
    out[i] = run;
    run += v;
  }
  const int total = s_tmp[32];
  __syncthreads();
  return total;
}

__device__ __forceinline__ int pair_expert(const int32_t* topk_idx, long long p, int T, int k) {
  const long long t = p % T, j = p / T;
  return topk_idx[t * k + j];
}

__global__ void __launch_bounds__(kPermThreads)
    perm_hist_kernel(const int32_t* __restrict__ topk_idx, int T, int k, int M, int nchunks,
                     int32_t* __restrict__ chunk_counts, int* status) {
  extern __shared__ int hist[];
  for (int e = threadIdx.x; e < M; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  const long long pairs = static_cast<long long>(T) * k;
  const long long p = static_cast<long long>(blockIdx.x) * kPermChunk + threadIdx.x;
  if (p < pairs) {
    const int e = pair_expert(topk_idx, p, T, k);
    if (e >= 0 && e < M) atomicAdd(&hist[e], 1);
    else if (e != M) set_status(status, MOE_DEVERR_BAD_EXPERT_INDEX);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < M; e += blockDim.x)
    chunk_counts[static_cast<size_t>(e) * nchunks + blockIdx.x] = hist[e];
}

__global__ void __launch_bounds__(256)
    perm_scan_kernel(const int32_t* __restrict__ chunk_counts, int nchunks,
                     int32_t* __restrict__ chunk_base, int32_t* __restrict__ counts) {
  __shared__ int s_tmp[33];
  const int e = blockIdx.x;
  const int total = block_exclusive_scan(chunk_counts + static_cast<size_t>(e) * nchunks,
                                         chunk_base + static_cast<size_t>(e) * nchunks, nchunks, s_tmp);
  if (threadIdx.x == 0) counts[e] = total;
}

__global__ void __launch_bounds__(kPermThreads)
    perm_scatter_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
                        int T, int k, int M, int nchunks, const int32_t* __restrict__ counts,
                        const int32_t* __restrict__ chunk_base, int32_t* __restrict__ offsets,
                        int32_t* __restrict__ slot_of, int32_t* __restrict__ row_token,
                        float* __restrict__ row_w) {
  extern __shared__ int smem[];
  int* offs = smem;                 // [M]
  int* wcnt = smem + M;             // [kPermWarps][M]
  __shared__ int s_tmp[33];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int total = block_exclusive_scan(counts, offs, M, s_tmp);
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e < M; e += blockDim.x) offsets[e] = offs[e];
    if (threadIdx.x == 0) offsets[M] = total;
  }
  for (int i = threadIdx.x; i < kPermWarps * M; i += blockDim.x) wcnt[i] = 0;
  __syncthreads();

  const long long pairs = static_cast<long long>(T) * k;
  const long long p = static_cast<long long>(blockIdx.x) * kPermChunk + threadIdx.x;
  int e = -1;
  if (p < pairs) {
    e = pair_expert(topk_idx, p, T, k);
    if (e < 0 || e >= M) e = -1;
  }
  const unsigned peers = __match_any_sync(0xffffffffu, e);
  const unsigned lt = (1u << lane) - 1u;
  const int rank = __popc(peers & lt);
  if (e >= 0 && (peers & lt) == 0) wcnt[warp * M + e] = __popc(peers);
  __syncthreads();
  if (e >= 0) {
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wcnt[w * M + e];
    const int slot = offs[e] + chunk_base[static_cast<size_t>(e) * nchunks + blockIdx.x] + before + rank;
    const long long t = p % T, j = p / T;
    slot_of[t * k + j] = slot;
    row_token[slot] = static_cast<int32_t>(t);
    row_w[slot] = topk_w[t * k + j];
  } else if (p < pairs) {
    const long long t = p % T, j = p / T;
    slot_of[t * k + j] = -1;  // sentinel (or invalid) pair: dispatched nowhere
  }
}

// Small problems (T*k <= kSmallPairs): the whole counting sort in one block.
// Pairs are staged in shared memory in j-major order; a pair's rank among
// the pairs of its expert is the number of earlier pairs with that expert.
constexpr int kSmallPairs = 2048;

__global__ void __launch_bounds__(1024)
    perm_small_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w, int T, int k,
                      int M, int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ slot_of, int32_t* __restrict__ row_token,
                      float* __restrict__ row_w, int* status) {
  extern __shared__ int sm_small[];
  int* hist = sm_small;             // [M]
  int* offs = sm_small + M;         // [M]
  int* ex = sm_small + 2 * M;       // [pairs] expert of pair p (-1 if invalid)
  __shared__ int s_tmp[33];
  const int pairs = T * k;
  for (int e = threadIdx.x; e < M; e += blockDim.x) hist[e] = 0;
  __syncthreads();
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    int e = pair_expert(topk_idx, p, T, k);
    if (e < 0 || e >= M) {
      if (e != M) set_status(status, MOE_DEVERR_BAD_EXPERT_INDEX);
      e = -1;
    } else {
      atomicAdd(&hist[e], 1);
    }
    ex[p] = e;
  }
  __syncthreads();
  const int total = block_exclusive_scan(hist, offs, M, s_tmp);
  for (int e = threadIdx.x; e < M; e += blockDim.x) {
    counts[e] = hist[e];
    offsets[e] = offs[e];
  }
  if (threadIdx.x == 0) offsets[M] = total;
  for (int p = threadIdx.x; p < pairs; p += blockDim.x) {
    const int e = ex[p];
    if (e < 0) {
      slot_of[(p % T) * k + p / T] = -1;  // sentinel (or invalid) pair: dispatched nowhere
      continue;
    }
    int rank = 0;
    for (int q = 0; q < p; ++q) rank += (ex[q] == e);
    const int slot = offs[e] + rank;
    const int t = p % T, j = p / T;
    slot_of[t * k + j] = slot;
    row_token[slot] = t;
    row_w[slot] = topk_w[t * k + j];
  }
}

cudaError_t launch_permute(const int32_t* topk_idx, const float* topk_w, int T, int k, int M,
                           int32_t* counts, int32_t* offsets, int32_t* slot_of, int32_t* row_token,
                           float* row_w, int32_t* chunk_counts, int32_t* chunk_base, int* status,
                           cudaStream_t s) {
  const long long pairs = static_cast<long long>(T) * k;
  if (pairs <= kSmallPairs) {
    const size_t smem = (2 * static_cast<size_t>(M) + pairs) * sizeof(int);
    if (smem > 48 * 1024) {
      cudaError_t e = cudaFuncSetAttribute(perm_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
      if (e != cudaSuccess) return e;
    }
    perm_small_kernel<<<1, 1024, smem, s>>>(topk_idx, topk_w, T, k, M, counts, offsets, slot_of, row_token,
                                            row_w, status);
    return cudaGetLastError();
  }
  const int nchunks = perm_num_chunks(pairs);
  perm_hist_kernel<<<nchunks, kPermThreads, M * sizeof(int), s>>>(topk_idx, T, k, M, nchunks,
                                                                  chunk_counts, status);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  perm_scan_kernel<<<M, 256, 0, s>>>(chunk_counts, nchunks, chunk_base, counts);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  const size_t smem = static_cast<size_t>(M) * (1 + kPermWarps) * sizeof(int);
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(perm_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
    if (err != cudaSuccess) return err;
  }
  perm_scatter_kernel<<<nchunks, kPermThreads, smem, s>>>(topk_idx, topk_w, T, k, M, nchunks, counts,
                                                          chunk_base, offsets, slot_of, row_token,
                                                          row_w);
  return cudaGetLastError();
}

}  // namespace moe
