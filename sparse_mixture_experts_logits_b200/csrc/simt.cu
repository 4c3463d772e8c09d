// fp32 grouped GEMM on the CUDA cores, with the same segment layout and
// epilogues as the tcgen05 kernel.  This is the path of the fp32 data type
// (the tensor cores have no full-fp32 multiply); it reads A through an
// optional row index, so the fp32 path needs no gathered copy of x.
#include <algorithm>

#include "gemm_sm100.cuh"
#include "kernels.cuh"

namespace moe {

constexpr int kSBM = 64, kSBN = 64, kSBK = 16;

struct SimtArgs {
  SimtLaunch L;
  int n_tiles;
};

template <int EPI>
__global__ void __launch_bounds__(256) simt_gemm_kernel(const SimtArgs args) {
  const SimtLaunch& L = args.L;
  __shared__ float As[kSBK][kSBM + 1];
  __shared__ float Bs[kSBK][kSBN + 1];
  __shared__ float Bu[kSBK][kSBN + 1];
  __shared__ int s_g, s_row0, s_rows;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  if (threadIdx.x == 0) {
    // locate this block's (group, m-tile) from the segment sizes
    int mt = blockIdx.y, g = -1, row0 = 0, rows = 0;
    const int G = L.num_groups;
    for (int gg = 0; gg < G; ++gg) {
      const int nr = static_cast<int>(L.rows);
      const int b = L.offsets ? min(max(L.offsets[gg], 0), nr) : 0;
      const int e = L.offsets ? min(max(L.offsets[gg + 1], 0), nr) : nr;
      const int tiles = e > b ? (e - b + kSBM - 1) / kSBM : 0;
      if (mt < tiles) { g = gg; row0 = b + mt * kSBM; rows = min(kSBM, e - row0); break; }
      mt -= tiles;
    }
    s_g = g; s_row0 = row0; s_rows = rows;
  }
  __syncthreads();
  const int g = s_g;
  if (g < 0) return;
  const int row0 = s_row0, nrows = s_rows;
  const int n0 = blockIdx.x * kSBN;
  const bool swiglu = (EPI == EPI_SWIGLU);
  float acc[4][4], accu[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) { acc[i][j] = 0.f; accu[i][j] = 0.f; }

  const size_t b_base = static_cast<size_t>(g) * L.b_rows_per_group;
  for (int k0 = 0; k0 < L.K; k0 += kSBK) {
    for (int i = threadIdx.x; i < kSBM * kSBK; i += 256) {
      const int r = i / kSBK, kk = i % kSBK;
      float v = 0.f;
      if (r < nrows && k0 + kk < L.K) {
        const int out_row = row0 + r;
        const int a_row = L.a_row_index ? L.a_row_index[out_row] : out_row;
        v = L.A[static_cast<size_t>(a_row) * L.K + k0 + kk];
      }
      As[kk][r] = v;
      const int n = n0 + r;
      float b = 0.f, bu = 0.f;
      if (n < L.out_cols && k0 + kk < L.K) {
        b = L.B[(b_base + n) * L.K + k0 + kk];
        if (swiglu) bu = L.B[(b_base + L.swiglu_hi + n) * L.K + k0 + kk];
      }
      Bs[kk][r] = b;
      Bu[kk][r] = bu;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSBK; ++kk) {
      float a[4], b[4], bu[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) { b[j] = Bs[kk][tx + 16 * j]; bu[j] = Bu[kk][tx + 16 * j]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
          if (swiglu) accu[i][j] = fmaf(a[i], bu[j], accu[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = ty + 16 * i;
    if (r >= nrows) continue;
    const int row = row0 + r;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= L.out_cols) continue;
      float v = acc[i][j];
      if constexpr (EPI == EPI_GELU_BIAS) {
        if (L.bias) v += L.bias[static_cast<size_t>(g) * L.out_cols + n];
        v = gelu_tanh(v);
      } else if constexpr (EPI == EPI_SWIGLU) {
        v = silu_f(v) * accu[i][j];
      } else if constexpr (EPI == EPI_SCALE_BIAS) {
        if (L.bias) v += L.bias[static_cast<size_t>(g) * L.out_cols + n];
        v *= L.row_scale[row];
      } else if constexpr (EPI == EPI_BIAS_ADD) {
        if (L.bias) v += L.bias[static_cast<size_t>(g) * L.out_cols + n];
        if (L.addend) v += L.addend[static_cast<size_t>(row) * L.ldo + n];
      }
      L.out[static_cast<size_t>(row) * L.ldo + n] = v;
    }
  }
}

cudaError_t launch_simt_gemm(const SimtLaunch& L, cudaStream_t s) {
  SimtArgs a;
  a.L = L;
  a.n_tiles = (L.out_cols + kSBN - 1) / kSBN;
  const long long mt_ub = L.offsets ? (L.rows / kSBM + std::min<long long>(L.num_groups, L.rows) + 1)
                                    : (L.rows + kSBM - 1) / kSBM;
  if (mt_ub <= 0) return cudaSuccess;
  dim3 grid(a.n_tiles, static_cast<unsigned>(mt_ub));
  switch (L.epi) {
    case EPI_GELU_BIAS: simt_gemm_kernel<EPI_GELU_BIAS><<<grid, 256, 0, s>>>(a); break;
    case EPI_SWIGLU: simt_gemm_kernel<EPI_SWIGLU><<<grid, 256, 0, s>>>(a); break;
    case EPI_SCALE_BIAS: simt_gemm_kernel<EPI_SCALE_BIAS><<<grid, 256, 0, s>>>(a); break;
    case EPI_BIAS_ADD: simt_gemm_kernel<EPI_BIAS_ADD><<<grid, 256, 0, s>>>(a); break;
    default: simt_gemm_kernel<EPI_STORE_F32><<<grid, 256, 0, s>>>(a); break;
  }
  return cudaGetLastError();
}

}  // namespace moe
