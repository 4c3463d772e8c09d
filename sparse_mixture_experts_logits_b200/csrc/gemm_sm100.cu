// Host side of the tcgen05 grouped GEMM: tensor maps, grid size, launch.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "gemm_sm100.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D bf16 [rows, K] row-major, box = box_rows x 64, 128-byte swizzle.
// Rows or columns outside the matrix read as zero.
bool make_tmap(CUtensorMap* map, const void* base, long long rows, int K, int box_rows) {
  auto fn = get_encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int EPI>
cudaError_t launch_epi(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args, int grid,
                       cudaStream_t s) {
  static int configured_mask = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(configured_mask & (1 << (dev & 31)))) {
    cudaError_t e = cudaFuncSetAttribute(moe_gemm_sm100_kernel<EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmDynSmem);
    if (e != cudaSuccess) return e;
    configured_mask |= 1 << (dev & 31);
  }
  moe_gemm_sm100_kernel<EPI><<<grid, kGemmThreads, kGemmDynSmem, s>>>(ta, tb, args);
  return cudaGetLastError();
}

}  // namespace

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return 148;
  if (cache[dev] == 0) {
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    cache[dev] = n > 0 ? n : 148;
  }
  return cache[dev];
}

cudaError_t launch_gemm_sm100(const GemmLaunch& L, cudaStream_t s) {
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, L.A, L.a_rows, L.K, kBM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, L.B, L.b_rows, L.K, L.bn / 2)) return cudaErrorInvalidValue;
  GemmArgs a;
  a.num_groups = L.num_groups;
  a.offsets = L.offsets;
  a.rows = static_cast<int>(L.a_rows);
  a.K = L.K;
  a.n_tiles = L.n_tiles;
  a.bn = L.bn;
  a.b_rows_per_group = L.b_rows_per_group;
  a.b_row_step = L.b_row_step;
  a.b_hi_offset = L.b_hi_offset;
  a.out_cols = L.out_cols;
  a.out_col_step = L.out_col_step;
  a.ldo = L.ldo;
  a.out = L.out;
  a.row_scale = L.row_scale;
  a.bias = static_cast<const __nv_bfloat16*>(L.bias);
  a.comb_src = static_cast<const float*>(L.comb_src);
  a.slot_of = L.slot_of;
  a.k = L.k;
  a.idesc = umma_idesc_bf16(kBM, L.bn);
  a.status = L.status;
  // upper bound of the tile count: sum_g ceil(rows_g / 128) <= rows/128 + (#non-empty groups)
  long long mt_ub = L.offsets ? L.rows_upper / kBM + std::min<long long>(L.num_groups, L.rows_upper)
                              : (L.a_rows + kBM - 1) / kBM;
  long long tiles_ub = mt_ub * L.n_tiles;
  int grid = static_cast<int>(std::min<long long>(num_sms(), std::max<long long>(1, tiles_ub)));
  switch (L.epi) {
    case EPI_STORE_F32: return launch_epi<EPI_STORE_F32>(ta, tb, a, grid, s);
    case EPI_GELU_BIAS: return launch_epi<EPI_GELU_BIAS>(ta, tb, a, grid, s);
    case EPI_SWIGLU: return launch_epi<EPI_SWIGLU>(ta, tb, a, grid, s);
    case EPI_SCALE_BIAS: return launch_epi<EPI_SCALE_BIAS>(ta, tb, a, grid, s);
    case EPI_COMBINE: return launch_epi<EPI_COMBINE>(ta, tb, a, grid, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace moe
