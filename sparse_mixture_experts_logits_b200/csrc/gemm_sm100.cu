// Host side of the tcgen05 grouped GEMM: tensor maps, grid size, launch.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
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

template <int EPI, int NCTA>
cudaError_t launch_epi(const CUtensorMap& ta, const CUtensorMap& tb, const GemmArgs& args,
                       long long tiles_ub, cudaStream_t s) {
  static std::atomic<unsigned> configured{0};  // one bit per device
  static std::atomic<int> max_units[32];       // CTAs (NCTA = 1) or clusters (NCTA = 2) per device
  int dev = 0;
  cudaGetDevice(&dev);
  auto kernel = moe_gemm_sm100_kernel<EPI, NCTA>;
  constexpr int smem = gemm_dyn_smem<NCTA>();
  const unsigned bit = 1u << (dev & 31);
  if (!(configured.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int units = num_sms();
    if (NCTA == 2) {
      e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 0);
      (void)e;
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(2 * (units / 2), 1, 1);
      q.blockDim = dim3(kGemmThreads, 1, 1);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 2;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      q.attrs = at;
      q.numAttrs = 1;
      int clusters = 0;
      if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &q) != cudaSuccess || clusters <= 0)
        clusters = units / 2;
      units = clusters;
    }
    max_units[dev & 31].store(units);
    configured.fetch_or(bit);
  }
  const long long units = std::min<long long>(max_units[dev & 31].load(), std::max<long long>(1, tiles_ub));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(units * NCTA), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = NCTA;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, ta, tb, args);
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
  const int ncta = L.ncta == 1 ? 1 : 2;
  const int tile_rows = 128 * ncta;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, L.A, L.a_rows, L.K, 128)) return cudaErrorInvalidValue;
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
  a.idesc = umma_idesc_bf16(tile_rows, L.bn);
  a.status = L.status;
  // upper bound of the tile count: sum_g ceil(rows_g / tile_rows) <= rows/tile_rows + (#non-empty groups)
  const long long mt_ub = L.offsets ? L.rows_upper / tile_rows + std::min<long long>(L.num_groups, L.rows_upper)
                                    : (L.a_rows + tile_rows - 1) / tile_rows;
  const long long tiles_ub = mt_ub * L.n_tiles;
#define MOE_GEMM_CASE(E)                                                              \
  case E:                                                                             \
    return ncta == 2 ? launch_epi<E, 2>(ta, tb, a, tiles_ub, s) : launch_epi<E, 1>(ta, tb, a, tiles_ub, s);
  switch (L.epi) {
    MOE_GEMM_CASE(EPI_STORE_F32)
    MOE_GEMM_CASE(EPI_GELU_BIAS)
    MOE_GEMM_CASE(EPI_SWIGLU)
    MOE_GEMM_CASE(EPI_SCALE_BIAS)
  }
#undef MOE_GEMM_CASE
  return cudaErrorInvalidValue;
}

}  // namespace moe
