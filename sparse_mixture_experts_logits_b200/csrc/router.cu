// Router: scores, top-k selection and gate weights.
//
// "GLaM" note, section "Sparse MoE Layer": r_t = softmax(W_r x_t),
// S_t = TopK(r_t, 2), MoE(x_t) = sum_{i in S_t} alpha_{t,i} E_i(x_t) with
// normalised gate weights.  GLM-4.5 "Shared Expert" note, "How it works":
// sigmoid scores plus the loss-free correction bias choose the top-k; the k
// sigmoid scores g_i are renormalised by their sum + eps and scaled by
// routed_scaling_factor.
//
// The logits s = x W_r come from the tcgen05 GEMM (bf16) or from the fp32
// SIMT kernel below; this file holds the selection kernel and the W_r
// transpose that gives the GEMM a K-major [M, D] operand.
#include "kernels.cuh"

namespace moe {

// W_r [D, M] -> W_r^T [M, D] through a 32 x 32 shared-memory tile.
__global__ void transpose_bf16_kernel(const __nv_bfloat16* __restrict__ src,
                                      __nv_bfloat16* __restrict__ dst, int rows, int cols) {
  __shared__ __nv_bfloat16 tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int r = r0 + i, c = c0 + threadIdx.x;
    if (r < rows && c < cols) tile[i][threadIdx.x] = src[static_cast<size_t>(r) * cols + c];
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int c = c0 + i, r = r0 + threadIdx.x;
    if (c < cols && r < rows) dst[static_cast<size_t>(c) * rows + r] = tile[threadIdx.x][i];
  }
}

// fp32 logits, s[t, e] = sum_d x[t, d] W_r[d, e], summed in d order.
// 32 x 32 output tile per block, 32 x 8 threads, 4 outputs per thread.
__global__ void logits_f32_kernel(const float* __restrict__ x, const float* __restrict__ w_r,
                                  float* __restrict__ logits, int T, int D, int M) {
  __shared__ float xs[32][33];
  __shared__ float ws[32][33];
  const int e = blockIdx.x * 32 + threadIdx.x;
  const int t0 = blockIdx.y * 32;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int d0 = 0; d0 < D; d0 += 32) {
    for (int i = threadIdx.y; i < 32; i += 8) {
      const int t = t0 + i, d = d0 + threadIdx.x;
      xs[i][threadIdx.x] = (t < T && d < D) ? x[static_cast<size_t>(t) * D + d] : 0.f;
      const int dd = d0 + i;
      ws[i][threadIdx.x] = (dd < D && e < M) ? w_r[static_cast<size_t>(dd) * M + e] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int d = 0; d < 32; ++d) {
      const float w = ws[d][threadIdx.x];
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[q] = fmaf(xs[threadIdx.y + 8 * q][d], w, acc[q]);
    }
    __syncthreads();
  }
  for (int q = 0; q < 4; ++q) {
    const int t = t0 + threadIdx.y + 8 * q;
    if (t < T && e < M) logits[static_cast<size_t>(t) * M + e] = acc[q];
  }
}

// Small-T bf16 logits, split over D: block (expert tile of 64, k-split ks)
// computes partial[ks][t][e] = sum over its D range of x[t, d] W_r[d, e] for
// every token t < T (T <= kSmallRouteT), each thread one expert and 16
// tokens, summing in d order.  reduce_splits_kernel then adds the partials
// in ks order, so the logits are deterministic.
constexpr int kSmallRouteT = 64;
constexpr int kSplitD = 128;

__global__ void __launch_bounds__(256)
    logits_splitk_bf16_kernel(const __nv_bfloat16* __restrict__ x, const __nv_bfloat16* __restrict__ w_r,
                              float* __restrict__ partial, int T, int D, int M) {
  __shared__ __nv_bfloat16 xs[kSmallRouteT][kSplitD + 2];
  __shared__ __nv_bfloat16 ws[kSplitD][64];
  const int el = threadIdx.x & 63;
  const int e = blockIdx.x * 64 + el;
  const int tg = threadIdx.x >> 6;  // tokens tg*16 .. tg*16+15
  const int d0 = blockIdx.y * kSplitD;
  const int dn = min(kSplitD, D - d0);
  const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
  for (int i = threadIdx.x; i < kSmallRouteT * kSplitD; i += blockDim.x) {
    const int t = i / kSplitD, d = i % kSplitD;
    xs[t][d] = (t < T && d < dn) ? x[static_cast<size_t>(t) * D + d0 + d] : zero;
  }
  for (int i = threadIdx.x; i < kSplitD * 64; i += blockDim.x) {
    const int d = i / 64, ee = blockIdx.x * 64 + (i % 64);
    ws[d][i % 64] = (d < dn && ee < M) ? w_r[static_cast<size_t>(d0 + d) * M + ee] : zero;
  }
  __syncthreads();
  float acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = 0.f;
#pragma unroll 4
  for (int d = 0; d < kSplitD; ++d) {
    const float wv = __bfloat162float(ws[d][el]);
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = fmaf(__bfloat162float(xs[tg * 16 + i][d]), wv, acc[i]);
  }
  if (e < M) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int t = tg * 16 + i;
      if (t < T) partial[(static_cast<size_t>(blockIdx.y) * T + t) * M + e] = acc[i];
    }
  }
}

// logits[i] = sum_{ks} partial[ks][i], added in ks order.
__global__ void reduce_splits_kernel(const float* __restrict__ partial, float* __restrict__ logits, int n,
                                     int nsplit) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  float acc = 0.f;
#pragma unroll 8
  for (int ks = 0; ks < nsplit; ++ks) acc += partial[static_cast<size_t>(ks) * n + i];
  logits[i] = acc;
}

int route_splits(int T, int D, int dtype) {
  return (dtype == MOE_DTYPE_BF16 && T <= kSmallRouteT) ? (D + kSplitD - 1) / kSplitD : 1;
}

cudaError_t launch_logits_splitk_bf16(const void* x, const void* w_r, float* partial, float* logits, int T,
                                      int D, int M, cudaStream_t s) {
  const int nsplit = (D + kSplitD - 1) / kSplitD;
  dim3 grid((M + 63) / 64, nsplit);
  logits_splitk_bf16_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(x),
                                                 static_cast<const __nv_bfloat16*>(w_r), partial, T, D, M);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n = T * M;
  reduce_splits_kernel<<<(n + 255) / 256, 256, 0, s>>>(partial, logits, n, nsplit);
  return cudaGetLastError();
}

// One warp per token.  Selection score: the logit (softmax) or
// sigmoid(logit) + e_bias (sigmoid router).  k rounds of a warp arg-max
// with the lower expert index winning exact ties; slot j is the j-th round.
constexpr int kTopkWarps = 8;

__global__ void __launch_bounds__(kTopkWarps * 32)
    topk_kernel(const float* __restrict__ logits, const float* __restrict__ e_bias, int T,
                int M, int k, int gate, int norm_topk_prob, float alpha, float eps, int n_group,
                int topk_group, int32_t* __restrict__ topk_idx, float* __restrict__ topk_w) {
  extern __shared__ float topk_smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* sel = topk_smem + static_cast<size_t>(warp) * 2 * M;  // selection score
  float* gv = sel + M;                                          // gate value (logit or g)
  const int t = blockIdx.x * kTopkWarps + warp;
  if (t >= T) return;
  const float* lrow = logits + static_cast<size_t>(t) * M;
  float lmax = -INFINITY;
  for (int e = lane; e < M; e += 32) {
    const float l = lrow[e];
    if (gate == MOE_GATE_SIGMOID_BIAS) {
      const float g = sigmoid_f(l);
      gv[e] = g;
      sel[e] = g + (e_bias != nullptr ? e_bias[e] : 0.0f);
    } else {
      gv[e] = l;
      sel[e] = l;
    }
    lmax = fmaxf(lmax, l);
  }
  __syncwarp();
  if (n_group > 1) {
    // Group-limited selection (the GLM-4.5 note's optional mask by expert
    // group): lane g scores group g (experts g*gsz .. g*gsz+gsz-1) by the sum
    // of its two largest selection scores; the topk_group best groups (lower
    // index on ties) stay eligible, every other expert's score becomes -inf.
    const int gsz = M / n_group;
    float gscore = -INFINITY;
    if (lane < n_group) {
      float b1 = -INFINITY, b2 = -INFINITY;
      for (int i = 0; i < gsz; ++i) {
        const float v = sel[lane * gsz + i];
        if (v > b1) { b2 = b1; b1 = v; } else if (v > b2) { b2 = v; }
      }
      gscore = gsz > 1 ? b1 + b2 : b1;
    }
    unsigned keep = 0u;
    for (int r = 0; r < topk_group; ++r) {
      const bool cand = lane < n_group && ((keep >> lane) & 1u) == 0u;
      float bv = cand ? gscore : -INFINITY;
      int bi = cand ? lane : 32;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (oi < 32 && (bi >= 32 || ov > bv || (ov == bv && oi < bi))) { bv = ov; bi = oi; }
      }
      if (bi < 32) keep |= 1u << bi;
    }
    for (int e = lane; e < M; e += 32)
      if (((keep >> (e / gsz)) & 1u) == 0u) sel[e] = -INFINITY;
    __syncwarp();
  }
  // A chosen entry's selection score is replaced by NaN, which never wins a
  // comparison.  If only NaN scores remain (NaN inputs), the lowest index
  // not yet chosen is taken so that the k indices stay distinct.
  int chosen_idx = 0;     // lane j < k keeps the j-th choice
  float chosen_val = 0.f; // and its gate value
  for (int j = 0; j < k; ++j) {
    float best = -INFINITY;
    int bi = M;
    for (int e = lane; e < M; e += 32) {
      const float s = sel[e];
      if (s > best || (s == best && e < bi)) { best = s; bi = e; }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, off);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
      if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (bi >= M) {
      int cand = M;
      for (int e = lane; e < M; e += 32) {
        bool used = false;
        for (int jj = 0; jj < j; ++jj) used |= (__shfl_sync(0xffffffffu, chosen_idx, jj) == e);
        if (!used && e < cand) cand = e;
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) cand = min(cand, __shfl_xor_sync(0xffffffffu, cand, off));
      bi = cand;
    }
    const float gsel = gv[bi];
    if (lane == j) { chosen_idx = bi; chosen_val = gsel; }
    __syncwarp();
    if (lane == 0) sel[bi] = __int_as_float(0x7fc00000);
    __syncwarp();
  }
  // weights
  float w = 0.f;
  if (gate == MOE_GATE_SIGMOID_BIAS) {
    float s = lane < k ? chosen_val : 0.f;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    w = norm_topk_prob ? alpha * chosen_val / (s + eps) : alpha * chosen_val;
  } else {
    if (norm_topk_prob) {
      const float top = __shfl_sync(0xffffffffu, chosen_val, 0);
      const float ex = lane < k ? expf(chosen_val - top) : 0.f;
      float s = ex;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      w = alpha * ex / s;
    } else {
      float m = lmax;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
      float s = 0.f;
      for (int e = lane; e < M; e += 32) s += expf(gv[e] - m);  // gv holds the logits (softmax gate)
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      w = alpha * expf(chosen_val - m) / s;
    }
  }
  if (lane < k) {
    topk_idx[static_cast<size_t>(t) * k + lane] = chosen_idx;
    topk_w[static_cast<size_t>(t) * k + lane] = w;
  }
}

size_t topk_smem_bytes(int M) { return static_cast<size_t>(kTopkWarps) * 2 * M * sizeof(float); }

cudaError_t launch_topk(const float* logits, const float* e_bias, int T, int M, int k, int gate,
                        int norm, float alpha, float eps, int n_group, int topk_group, int32_t* idx,
                        float* w, cudaStream_t s) {
  const size_t smem = topk_smem_bytes(M);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const int blocks = (T + kTopkWarps - 1) / kTopkWarps;
  topk_kernel<<<blocks, kTopkWarps * 32, smem, s>>>(logits, e_bias, T, M, k, gate, norm, alpha, eps,
                                                     n_group, topk_group, idx, w);
  return cudaGetLastError();
}

cudaError_t launch_transpose_bf16(const void* src, void* dst, int rows, int cols, cudaStream_t s) {
  dim3 grid((cols + 31) / 32, (rows + 31) / 32), block(32, 8);
  transpose_bf16_kernel<<<grid, block, 0, s>>>(static_cast<const __nv_bfloat16*>(src),
                                                static_cast<__nv_bfloat16*>(dst), rows, cols);
  return cudaGetLastError();
}

cudaError_t launch_logits_f32(const float* x, const float* w_r, float* logits, int T, int D, int M,
                              cudaStream_t s) {
  dim3 grid((M + 31) / 32, (T + 31) / 32), block(32, 8);
  logits_f32_kernel<<<grid, block, 0, s>>>(x, w_r, logits, T, D, M);
  return cudaGetLastError();
}

}  // namespace moe
