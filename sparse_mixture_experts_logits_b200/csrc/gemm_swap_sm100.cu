// Host side of the token-on-N grouped GEMM: tensor maps, grid, cluster launch.
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <mutex>

#include "gemm_swap_sm100.cuh"
#include "kernels.cuh"

namespace moe {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// bf16 [rows, cols] row-major, box = box_rows x 64 columns, 128-byte swizzle;
// rows and columns past the end read as zero.
bool tmap_bf16(CUtensorMap* map, const void* base, long long rows, int cols, int box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(box_rows)};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 [groups][rows][cols] with row pitch `ld` and group pitch `gstride`
// elements, 32 x 32 x 1 boxes, no swizzle: the weight-gradient output.
bool tmap_f32_out(CUtensorMap* map, void* base, int cols, long long rows, int groups, long long ld,
                  long long gstride) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                        static_cast<cuuint64_t>(groups)};
  cuuint64_t strides[2] = {static_cast<cuuint64_t>(ld) * 4, static_cast<cuuint64_t>(gstride) * 4};
  cuuint32_t box[3] = {32, 32, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int EPI, int LAYOUT = kSwFwd>
cudaError_t launch_swap_epi(const SwapMaps& maps, const SwapArgs& args, long long tiles_ub, cudaStream_t s) {
  static std::atomic<unsigned> configured{0};
  static std::atomic<int> max_clusters[32];
  int dev = 0;
  cudaGetDevice(&dev);
  auto kernel = moe_gemm_swap_kernel<EPI, LAYOUT>;
  const unsigned bit = 1u << (dev & 31);
  if (!(configured.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSwDynSmem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    q.blockDim = dim3(swap_threads<EPI>(), 1, 1);
    q.dynamicSmemBytes = kSwDynSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = 2;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    q.attrs = at;
    q.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, kernel, &q) != cudaSuccess || clusters <= 0)
      clusters = num_sms() / 2;
    max_clusters[dev & 31].store(clusters);
    configured.fetch_or(bit);
  }
  const long long units = std::min<long long>(max_clusters[dev & 31].load(), std::max<long long>(1, tiles_ub));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(2 * units), 1, 1);
  cfg.blockDim = dim3(swap_threads<EPI>(), 1, 1);
  cfg.dynamicSmemBytes = kSwDynSmem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, maps, args);
}

// Row-grouped layouts: the forward and the input gradients.
cudaError_t launch_swap_rows(int layout, int epi, const SwapMaps& m, const SwapArgs& a, long long tiles_ub,
                             cudaStream_t s) {
  if (layout == kSwDgrad) {
    switch (epi) {
      case EPI_STORE_F32: return launch_swap_epi<EPI_STORE_F32, kSwDgrad>(m, a, tiles_ub, s);
      case EPI_BWD_GELU_DACT: return launch_swap_epi<EPI_BWD_GELU_DACT, kSwDgrad>(m, a, tiles_ub, s);
      case EPI_BWD_SWIGLU_DACT: return launch_swap_epi<EPI_BWD_SWIGLU_DACT, kSwDgrad>(m, a, tiles_ub, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (epi) {
    case EPI_BWD_GELU_SAVE: return launch_swap_epi<EPI_BWD_GELU_SAVE>(m, a, tiles_ub, s);
    case EPI_BWD_SWIGLU_SAVE: return launch_swap_epi<EPI_BWD_SWIGLU_SAVE>(m, a, tiles_ub, s);
    case EPI_GELU_BIAS: return launch_swap_epi<EPI_GELU_BIAS>(m, a, tiles_ub, s);
    case EPI_SWIGLU: return launch_swap_epi<EPI_SWIGLU>(m, a, tiles_ub, s);
    case EPI_SCALE_BIAS: return launch_swap_epi<EPI_SCALE_BIAS>(m, a, tiles_ub, s);
    case EPI_STORE_F32: return launch_swap_epi<EPI_STORE_F32>(m, a, tiles_ub, s);
    case EPI_STORE_BF16: return launch_swap_epi<EPI_STORE_BF16>(m, a, tiles_ub, s);
    case EPI_BIAS_ADD: return launch_swap_epi<EPI_BIAS_ADD>(m, a, tiles_ub, s);
    case EPI_ACCUM_F32: return launch_swap_epi<EPI_ACCUM_F32>(m, a, tiles_ub, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_gemm_swap(const SwapLaunch& L, cudaStream_t s) {
  SwapMaps m = {};
  // A: K-major weight rows, or (backward) an MN-major [rows, a_cols] matrix;
  // B: K-major token rows (128-row boxes), or (weight gradients) MN-major.
  const int a_inner = L.layout == kSwFwd ? L.K : L.a_cols;
  if (!tmap_bf16(&m.w, L.W, L.w_rows, a_inner, 64)) return cudaErrorInvalidValue;
  if (L.layout == kSwWgrad) {
    if (!tmap_bf16(&m.x, L.X, L.x_rows, L.b_cols, 64)) return cudaErrorInvalidValue;
    if (L.num_groups > 1 && L.out_gstride < static_cast<long long>(L.b_cols) * L.ldo) return cudaErrorInvalidValue;
    if (!tmap_f32_out(&m.out, L.out, L.out_cols, L.b_cols, L.num_groups, L.ldo,
                      L.num_groups > 1 ? L.out_gstride : static_cast<long long>(L.b_cols) * L.ldo))
      return cudaErrorInvalidValue;
  } else if (!tmap_bf16(&m.x, L.X, L.x_rows, L.K, 128)) {
    return cudaErrorInvalidValue;
  }
  SwapArgs a = {};
  a.num_groups = L.num_groups;
  a.offsets = L.offsets;
  a.rows = static_cast<int>(L.rows);
  a.K = L.K;
  a.w_rows_per_group = L.w_rows_per_group;
  a.w_tiles = L.w_tiles;
  a.w_tile_step = L.w_tile_step;
  a.w_hi_offset = L.w_hi_offset;
  a.w_cta_step = L.w_cta_step;
  a.cols_per_tile = L.cols_per_tile;
  a.out_cols = L.out_cols;
  a.ldo = L.ldo;
  a.out = L.out;
  a.row_scale = L.row_scale;
  a.bias = static_cast<const __nv_bfloat16*>(L.bias);
  a.addend = static_cast<const __nv_bfloat16*>(L.addend);
  a.status = L.status;
  a.k_rows_per_group = L.k_rows_per_group;
  a.b_tiles = L.b_tiles;
  a.b_cols = L.b_cols;
  a.out_gstride = L.out_gstride;
  a.out2 = static_cast<__nv_bfloat16*>(L.out2);
  a.out3 = static_cast<__nv_bfloat16*>(L.out3);
  a.ldo2 = L.ldo2;
  a.aux = static_cast<const float*>(L.aux);
  a.ld_aux = L.ld_aux;
  a.parts = L.parts;
  a.ld_parts = L.ld_parts;
  a.half_cols = L.half_cols;
  a.counts = L.counts;
  a.tile_ctr = L.tile_ctr;
  if (L.layout == kSwWgrad) {
    const long long tiles_ub = static_cast<long long>(L.num_groups) * L.w_tiles * L.b_tiles;
    if (L.epi != EPI_STORE_F32) return cudaErrorInvalidValue;
    return launch_swap_epi<EPI_STORE_F32, kSwWgrad>(m, a, tiles_ub, s);
  }
  // token tiles of a segment: ceil(rows_g / 256) at most, so the total is at most rows/256 + #groups
  const long long tt_ub = L.offsets ? L.rows / kSwMaxTile + std::min<long long>(L.num_groups, L.rows)
                                    : (L.rows + kSwMaxTile - 1) / kSwMaxTile;
  const long long tiles_ub = tt_ub * L.w_tiles;
  return launch_swap_rows(L.layout, L.epi, m, a, tiles_ub, s);
}

}  // namespace moe
