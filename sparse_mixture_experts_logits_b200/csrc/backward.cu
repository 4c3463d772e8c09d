// Kernels of the layer backward (moe_backward): a grouped GEMM with strided
// operands on the CUDA cores, and the elementwise, per-pair and per-token
// steps between the GEMMs.  Every sum runs in a fixed order, so a backward is
// bitwise repeatable.
#include <algorithm>

#include "kernels.cuh"

namespace moe {

namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kBThreads = 256;

struct BwdArgs {
  const void* A; long long a_sm, a_sk;
  const void* B; long long b_sn, b_sk, b_gstride;
  const void* bias; long long bias_gstride;
  float* C; long long ldc, c_gstride;
  int mode;
  const int32_t* offsets;
  int G;
  long long rows, K;
  int N;
  int accumulate;
  long long m_tiles;  // tiles along the output rows (mode 0: upper bound)
  int ksplit;         // mode 1 without groups: contraction split into ksplit chunks of kchunk,
  long long kchunk;   // chunk z written to C + z * c_gstride (partial sums)
};

__device__ __forceinline__ long long lmin(long long a, long long b) { return a < b ? a : b; }
__device__ __forceinline__ float ld(const float* p, long long i) { return p[i]; }
__device__ __forceinline__ float ld(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }

// One 64 x 64 output tile per block and loop step; 16-deep slices of A and B
// go through shared memory, each thread keeps a 4 x 4 block of sums.  An
// operand whose contraction index is contiguous is loaded along it, any other
// along its row index, so that neighbouring threads read neighbouring words.
template <typename TA, typename TB>
__global__ void __launch_bounds__(kBThreads) bwd_gemm_kernel(const BwdArgs p) {
  __shared__ float As[kBK][kBM + 1];
  __shared__ float Bs[kBK][kBN + 1];
  __shared__ long long s_row0, s_kb, s_ke;
  __shared__ int s_nrows, s_g;
  const TA* A = static_cast<const TA*>(p.A);
  const TB* B = static_cast<const TB*>(p.B);
  const TB* bias = static_cast<const TB*>(p.bias);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int n0 = blockIdx.x * kBN;
  for (long long mt = blockIdx.y; mt < p.m_tiles; mt += gridDim.y) {
    __syncthreads();  // the previous step's readers of s_* are done
    if (threadIdx.x == 0) {
      int g = -1;
      long long row0 = 0, kb = 0, ke = p.K;
      int nrows = 0;
      if (p.mode == 0) {
        if (p.offsets == nullptr) {
          row0 = mt * kBM;
          if (row0 < p.rows) { g = 0; nrows = static_cast<int>(lmin(kBM, p.rows - row0)); }
        } else {
          long long t = mt;
          for (int gg = 0; gg < p.G; ++gg) {
            const long long b = lmin(max(p.offsets[gg], 0), p.rows);
            const long long e = lmin(max(p.offsets[gg + 1], 0), p.rows);
            const long long tiles = e > b ? (e - b + kBM - 1) / kBM : 0;
            if (t < tiles) {
              g = gg;
              row0 = b + t * kBM;
              nrows = static_cast<int>(lmin(kBM, e - row0));
              break;
            }
            t -= tiles;
          }
        }
      } else if (p.ksplit > 1) {
        g = blockIdx.z;  // the chunk: its partial sums go to C + g * c_gstride
        row0 = mt * kBM;
        nrows = static_cast<int>(lmin(kBM, p.rows - row0));
        kb = lmin(static_cast<long long>(g) * p.kchunk, p.K);
        ke = lmin(kb + p.kchunk, p.K);
      } else {
        g = blockIdx.z;
        row0 = mt * kBM;
        nrows = static_cast<int>(lmin(kBM, p.rows - row0));
        if (p.offsets != nullptr) {
          kb = lmin(max(p.offsets[g], 0), p.K);
          ke = lmin(max(p.offsets[g + 1], 0), p.K);
          if (ke < kb) ke = kb;
        }
      }
      s_g = g; s_row0 = row0; s_nrows = nrows; s_kb = kb; s_ke = ke;
    }
    __syncthreads();
    const int g = s_g;
    if (g < 0) continue;  // uniform across the block
    const long long row0 = s_row0, kb = s_kb, ke = s_ke;
    const int nrows = s_nrows;
    const long long b_base = p.ksplit > 1 ? 0 : static_cast<long long>(g) * p.b_gstride;
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (long long k0 = kb; k0 < ke; k0 += kBK) {
      for (int i = threadIdx.x; i < kBM * kBK; i += kBThreads) {
        int r, kk;
        if (p.a_sk == 1) { kk = i & (kBK - 1); r = i / kBK; } else { r = i & (kBM - 1); kk = i / kBM; }
        const long long k = k0 + kk;
        As[kk][r] = (r < nrows && k < ke) ? ld(A, (row0 + r) * p.a_sm + k * p.a_sk) : 0.f;
        int c, kc;
        if (p.b_sk == 1) { kc = i & (kBK - 1); c = i / kBK; } else { c = i & (kBN - 1); kc = i / kBN; }
        const long long kq = k0 + kc;
        const int n = n0 + c;
        Bs[kc][c] = (n < p.N && kq < ke) ? ld(B, b_base + n * p.b_sn + kq * p.b_sk) : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kBK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
    const long long c_base = p.mode == 1 ? static_cast<long long>(g) * p.c_gstride : 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = ty + 16 * i;
      if (r >= nrows) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = n0 + tx + 16 * j;
        if (n >= p.N) continue;
        float v = acc[i][j];
        if (bias != nullptr) v += ld(bias, static_cast<long long>(g) * p.bias_gstride + n);
        float* dst = p.C + c_base + (row0 + r) * p.ldc + n;
        *dst = (p.accumulate && p.ksplit <= 1) ? *dst + v : v;
      }
    }
  }
}

// C[i] (+)= sum over z of partial[z * n + i], z in order (split-K reduction).
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int splits, long long n, float* C,
                                     int accumulate) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float v = accumulate ? C[i] : 0.f;
    for (int z = 0; z < splits; ++z) v += partial[z * n + i];
    C[i] = v;
  }
}

// Rows this launch covers: *n_rows when given (the dispatched pairs), else rows.
__device__ __forceinline__ long long live_rows(const int32_t* n_rows, long long rows) {
  return n_rows ? lmin(max(*n_rows, 0), rows) : rows;
}

// a = sigma(h) (GELU) or SiLU(gate) * up (SwiGLU, h = [gate | up]).
__global__ void bwd_act_kernel(const float* __restrict__ h, float* __restrict__ a, const int32_t* n_rows,
                               long long rows, int Ha, int swiglu) {
  const long long nr = live_rows(n_rows, rows);
  const long long n = nr * Ha;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long r = q / Ha;
    const int i = static_cast<int>(q - r * Ha);
    if (swiglu) {
      const float* hr = h + r * 2 * Ha;
      a[q] = silu_f(hr[i]) * hr[Ha + i];
    } else {
      a[q] = gelu_tanh(h[q]);
    }
  }
}

__device__ __forceinline__ float gelu_tanh_grad(float v) {
  // d/dv of 0.5 v (1 + tanh u), u = c (v + 0.044715 v^3)
  const float c = 0.7978845608028654f;
  const float th = tanhf(c * (v + 0.044715f * v * v * v));
  return 0.5f * (1.0f + th) + 0.5f * v * (1.0f - th * th) * c * (1.0f + 3.0f * 0.044715f * v * v);
}

// In place: h (pre-activations) becomes dL/dh, from da = dL/da.  The thread of
// (row, i) reads and writes only column i (and I + i for SwiGLU) of that row.
__global__ void bwd_act_grad_kernel(const float* __restrict__ da, float* h, const int32_t* n_rows, long long rows,
                                    int Ha, int swiglu) {
  const long long nr = live_rows(n_rows, rows);
  const long long n = nr * Ha;
  for (long long q = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; q < n;
       q += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float g = da[q];
    if (swiglu) {
      const long long r = q / Ha;
      const int i = static_cast<int>(q - r * Ha);
      float* hr = h + r * 2 * Ha;
      const float gate = hr[i], up = hr[Ha + i];
      const float s = sigmoid_f(gate);
      hr[i] = g * up * s * (1.0f + gate * (1.0f - s));
      hr[Ha + i] = g * gate * s;
    } else {
      h[q] = g * gelu_tanh_grad(h[q]);
    }
  }
}

// One warp per (token, slot) pair p = t k + j at dispatch row r = slot_of[p]:
// dw[p] = <dy_t, o_r> and dO_r = w_p dy_t (rows r < 0 or >= rows_cap: dw = 0).
template <typename TY>
__global__ void bwd_pair_kernel(const TY* __restrict__ dy, const float* __restrict__ o,
                                const int32_t* __restrict__ slot_of, const float* __restrict__ topk_w,
                                float* __restrict__ dw, float* __restrict__ dO, long long pairs, int k, int D,
                                long long rows_cap) {
  const int lane = threadIdx.x & 31;
  const long long warps = static_cast<long long>(gridDim.x) * (blockDim.x >> 5);
  for (long long pr = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; pr < pairs;
       pr += warps) {
    const long long r = slot_of[pr];
    if (r < 0 || r >= rows_cap) {
      if (lane == 0) dw[pr] = 0.f;
      continue;
    }
    const long long t = pr / k;
    const float wt = topk_w[pr];
    const TY* dyt = dy + t * D;
    const float* orow = o + r * D;
    float* drow = dO + r * D;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float g = to_f32(dyt[d]);
      s = fmaf(g, orow[d], s);
      drow[d] = wt * g;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) dw[pr] = s;
  }
}

// out[g, n] = sum over rows [offsets[g], offsets[g+1]) of Y[row, n], in row order.
__global__ void bwd_colsum_kernel(const float* __restrict__ Y, long long ldy, const int32_t* __restrict__ offsets,
                                  long long rows_cap, int N, float* __restrict__ out) {
  const int g = blockIdx.y;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= N) return;
  const long long b = lmin(max(offsets[g], 0), rows_cap);
  const long long e = lmin(max(offsets[g + 1], 0), rows_cap);
  float s = 0.f;
  for (long long r = b; r < e; ++r) s += Y[r * ldy + n];
  out[static_cast<long long>(g) * N + n] = s;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

// One warp per token: dL/dlogits [M] from dL/dw of its k chosen experts, through
// the weight formula of the router (lane j < k holds chosen slot j).
__global__ void bwd_router_kernel(const float* __restrict__ logits, const int32_t* __restrict__ idx,
                                  const float* __restrict__ dw, int T, int M, int k, int gate, int norm,
                                  float alpha, float eps, float* __restrict__ dl,
                                  __nv_bfloat16* __restrict__ dl_bf) {
  const int lane = threadIdx.x & 31;
  const int warps = gridDim.x * (blockDim.x >> 5);
  for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; t < T; t += warps) {
    const float* lt = logits + static_cast<long long>(t) * M;
    float* dlt = dl + static_cast<long long>(t) * M;
    int e = -1;
    float l = -INFINITY, g = 0.f;
    if (lane < k) {
      e = idx[static_cast<long long>(t) * k + lane];
      if (e >= 0 && e < M) {
        l = lt[e];
        g = dw[static_cast<long long>(t) * k + lane];
      } else {
        e = -1;
      }
    }
    const bool full_softmax = gate == MOE_GATE_SOFTMAX && !norm;
    if (full_softmax) {
      // p = softmax over all M; dl_i = alpha p_i ([i chosen] dw_i - sum_j p_j dw_j)
      float mx = -INFINITY;
      for (int i = lane; i < M; i += 32) mx = fmaxf(mx, lt[i]);
      mx = warp_max(mx);
      float z = 0.f;
      for (int i = lane; i < M; i += 32) z += expf(lt[i] - mx);
      z = warp_sum(z);
      const float pj = e >= 0 ? expf(l - mx) / z : 0.f;
      const float s = warp_sum(pj * g);
      for (int i = lane; i < M; i += 32) dlt[i] = -alpha * (expf(lt[i] - mx) / z) * s;
      __syncwarp();
      if (e >= 0) dlt[e] += alpha * pj * g;
      __syncwarp();
      if (dl_bf != nullptr)
        for (int i = lane; i < M; i += 32) dl_bf[static_cast<long long>(t) * M + i] = __float2bfloat16_rn(dlt[i]);
      continue;
    }
    for (int i = lane; i < M; i += 32) dlt[i] = 0.f;
    __syncwarp();
    if (gate == MOE_GATE_SOFTMAX) {
      // q = softmax over the chosen; dl_j = alpha q_j (dw_j - sum_i q_i dw_i)
      const float mx = warp_max(l);
      const float ex = e >= 0 ? expf(l - mx) : 0.f;
      const float z = warp_sum(ex);
      const float q = ex / z;
      const float s = warp_sum(q * g);
      if (e >= 0) dlt[e] = alpha * q * (g - s);
    } else {
      // g_j = sigmoid(l_j); w_j = alpha g_j / (sum g + eps) or alpha g_j.  Normalised:
      // dg_j = alpha / den (dw_j - sum_i gbar_i dw_i), gbar = g / den (one chosen expert:
      // gbar = 1 exactly and dg = 0, the eps-small true value)
      const float gj = e >= 0 ? sigmoid_f(l) : 0.f;
      float dg;
      if (norm) {
        const float den = warp_sum(gj) + eps;
        const float gbar = gj / den;
        const float s = warp_sum(gbar * g);
        dg = alpha / den * (g - s);
      } else {
        dg = alpha * g;
      }
      if (e >= 0) dlt[e] = dg * gj * (1.0f - gj);
    }
    __syncwarp();
    if (dl_bf != nullptr)
      for (int i = lane; i < M; i += 32) dl_bf[static_cast<long long>(t) * M + i] = __float2bfloat16_rn(dlt[i]);
  }
}

inline int grid_1d(long long n, int threads) {
  const long long b = (n + threads - 1) / threads;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(b, 8ll * num_sms())));
}

}  // namespace

cudaError_t launch_bwd_gemm(const BwdGemmLaunch& L, cudaStream_t s) {
  BwdArgs a;
  a.A = L.A; a.a_sm = L.a_sm; a.a_sk = L.a_sk;
  a.B = L.B; a.b_sn = L.b_sn; a.b_sk = L.b_sk; a.b_gstride = L.b_gstride;
  a.bias = L.bias; a.bias_gstride = L.bias_gstride;
  a.C = L.C; a.ldc = L.ldc; a.c_gstride = L.c_gstride;
  a.mode = L.mode; a.offsets = L.offsets; a.G = L.offsets ? L.G : 1;
  a.rows = L.rows; a.K = L.K; a.N = L.N; a.accumulate = L.accumulate;
  a.ksplit = 1; a.kchunk = L.K;
  if (a.rows <= 0 || a.N <= 0) return cudaSuccess;
  if (L.mode == 1 && L.offsets == nullptr && L.ksplit > 1 && L.partial != nullptr && L.ldc == L.N) {
    // one contraction cut into chunks whose partial sums are added in order
    a.ksplit = L.ksplit;
    a.kchunk = (L.K + L.ksplit - 1) / L.ksplit;
    a.kchunk = (a.kchunk + kBK - 1) / kBK * kBK;
    a.C = L.partial;
    a.c_gstride = a.rows * L.ldc;
    a.G = L.ksplit;
    a.accumulate = 0;
    a.m_tiles = (a.rows + kBM - 1) / kBM;
    dim3 grid((a.N + kBN - 1) / kBN, static_cast<unsigned>(std::min<long long>(a.m_tiles, 65535)), a.ksplit);
    if (L.a_bf16 && !L.b_bf16)
      bwd_gemm_kernel<__nv_bfloat16, float><<<grid, kBThreads, 0, s>>>(a);
    else if (L.a_bf16)
      bwd_gemm_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kBThreads, 0, s>>>(a);
    else if (L.b_bf16)
      bwd_gemm_kernel<float, __nv_bfloat16><<<grid, kBThreads, 0, s>>>(a);
    else
      bwd_gemm_kernel<float, float><<<grid, kBThreads, 0, s>>>(a);
    const long long n = a.rows * L.N;
    splitk_reduce_kernel<<<grid_1d(n, 256), 256, 0, s>>>(L.partial, L.ksplit, n, L.C, L.accumulate);
    return cudaGetLastError();
  }
  if (L.mode == 0 && L.offsets != nullptr)
    a.m_tiles = a.rows / kBM + std::min<long long>(a.G, a.rows) + 1;
  else
    a.m_tiles = (a.rows + kBM - 1) / kBM;
  if (L.mode == 1 && a.G > 65535) return cudaErrorInvalidValue;
  dim3 grid((a.N + kBN - 1) / kBN, static_cast<unsigned>(std::min<long long>(a.m_tiles, 65535)),
            L.mode == 1 ? a.G : 1);
  if (L.a_bf16 && L.b_bf16)
    bwd_gemm_kernel<__nv_bfloat16, __nv_bfloat16><<<grid, kBThreads, 0, s>>>(a);
  else if (L.a_bf16)
    bwd_gemm_kernel<__nv_bfloat16, float><<<grid, kBThreads, 0, s>>>(a);
  else if (L.b_bf16)
    bwd_gemm_kernel<float, __nv_bfloat16><<<grid, kBThreads, 0, s>>>(a);
  else
    bwd_gemm_kernel<float, float><<<grid, kBThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_bwd_act(const float* h, float* a, const int32_t* n_rows, long long rows, int Ha, bool swiglu,
                           cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  bwd_act_kernel<<<grid_1d(rows * Ha, 256), 256, 0, s>>>(h, a, n_rows, rows, Ha, swiglu ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_bwd_act_grad(const float* da, float* h, const int32_t* n_rows, long long rows, int Ha,
                                bool swiglu, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  bwd_act_grad_kernel<<<grid_1d(rows * Ha, 256), 256, 0, s>>>(da, h, n_rows, rows, Ha, swiglu ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_bwd_pairs(int dtype, const void* dy, const float* o, const int32_t* slot_of,
                             const float* topk_w, float* dw, float* dO, int T, int k, int D, long long rows_cap,
                             cudaStream_t s) {
  const long long pairs = static_cast<long long>(T) * k;
  if (pairs <= 0) return cudaSuccess;
  const int blocks = grid_1d(pairs * 32, 256);
  if (dtype == MOE_DTYPE_BF16)
    bwd_pair_kernel<__nv_bfloat16><<<blocks, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(dy), o, slot_of,
                                                          topk_w, dw, dO, pairs, k, D, rows_cap);
  else
    bwd_pair_kernel<float><<<blocks, 256, 0, s>>>(static_cast<const float*>(dy), o, slot_of, topk_w, dw, dO,
                                                  pairs, k, D, rows_cap);
  return cudaGetLastError();
}

cudaError_t launch_bwd_colsum(const float* Y, long long ldy, const int32_t* offsets, int G, long long rows_cap,
                              int N, float* out, cudaStream_t s) {
  if (G <= 0 || N <= 0) return cudaSuccess;
  if (G > 65535) return cudaErrorInvalidValue;
  dim3 grid((N + 255) / 256, G);
  bwd_colsum_kernel<<<grid, 256, 0, s>>>(Y, ldy, offsets, rows_cap, N, out);
  return cudaGetLastError();
}

cudaError_t launch_bwd_router(const float* logits, const int32_t* idx, const float* dw, int T, int M, int k,
                              int gate, int norm, float alpha, float eps, float* dl, void* dl_bf,
                              cudaStream_t s) {
  if (T <= 0) return cudaSuccess;
  bwd_router_kernel<<<grid_1d(static_cast<long long>(T) * 32, 256), 256, 0, s>>>(
      logits, idx, dw, T, M, k, gate, norm, alpha, eps, dl, static_cast<__nv_bfloat16*>(dl_bf));
  return cudaGetLastError();
}

}  // namespace moe
