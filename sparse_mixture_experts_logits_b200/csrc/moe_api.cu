// C ABI of the MoE layer forward: argument checks, workspace layouts and
// the sequence of kernel launches of every entry point (see moe_b200.h).
#include <algorithm>
#include <cmath>
#include <atomic>
#include <cstring>
#include <mutex>

#include "gemm_sm100.cuh"
#include <nvtx3/nvToolsExt.h>

#include "kernels.cuh"

using namespace moe;

namespace moe {

// Every entry point runs only on compute capability 10.0 (sm_100a code).
moe_status_t check_device() {
  static std::atomic<int> arch_ok[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  int v = arch_ok[dev].load();
  if (v == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return MOE_ERR_CUDA;
    v = (major == 10 && minor == 0) ? 1 : 2;
    arch_ok[dev].store(v);
  }
  return v == 1 ? MOE_OK : MOE_ERR_UNSUPPORTED;
}

}  // namespace moe

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }
inline int round_up(int v, int m) { return (v + m - 1) / m * m; }

struct Carve {
  size_t off = 0;
  size_t take(size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  }
};

inline size_t esize(int dtype) { return dtype == MOE_DTYPE_BF16 ? 2 : 4; }

// A handful of rows per expert (decode): the routed GEMMs take the
// tokens-on-M path of run_experts.
inline bool few_rows(const moe_layer_desc_t* d) {
  return static_cast<long long>(d->T) * d->k < 4ll * d->M;
}

inline moe_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }
#define MOE_TRY(expr)                          \
  do {                                         \
    moe_status_t st_ = (expr);                 \
    if (st_ != MOE_OK) return st_;             \
  } while (0)
#define MOE_CUDA(expr) MOE_TRY(cuda_status(expr))

bool aligned_ws(const void* ws) { return (reinterpret_cast<uintptr_t>(ws) % kAlign) == 0; }
// bf16 tensors that the tensor-core kernels move with TMA, and the fp32
// weight gradients they store with it, start on a 16-byte boundary.
bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

moe_status_t check_router_args(int T, int D, int M, int k, int dtype, int gate) {
  if (T < 0 || D < 1 || M < 1 || k < 1) return MOE_ERR_INVALID_ARG;
  if (k > M) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_F32 && dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (gate != MOE_GATE_SOFTMAX && gate != MOE_GATE_SIGMOID_BIAS) return MOE_ERR_INVALID_ARG;
  if (k > kMaxTopK || M > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  if (dtype == MOE_DTYPE_BF16 && D % 16 != 0) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * std::max(D, M) >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Group-limited selection: n_group <= 1 is off; otherwise M splits into
// n_group equal groups (at most 32), 1 <= topk_group <= n_group, and the
// eligible groups hold at least k experts.
moe_status_t check_groups(int M, int k, int n_group, int topk_group) {
  if (n_group <= 1) return MOE_OK;
  if (n_group > 32) return MOE_ERR_UNSUPPORTED;
  if (M % n_group != 0 || topk_group < 1 || topk_group > n_group) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(topk_group) * (M / n_group) < k) return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

moe_status_t check_desc(const moe_layer_desc_t* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_router_args(d->T, d->D, d->M, d->k, d->dtype, d->gate));
  MOE_TRY(check_groups(d->M, d->k, d->n_group, d->topk_group));
  if (d->act != MOE_ACT_GELU_TANH && d->act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (d->I < 1 || d->I_sh < 0 || !(d->eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16 && (d->I % 16 != 0 || d->I_sh % 16 != 0)) return MOE_ERR_UNSUPPORTED;
  const long long pairs = static_cast<long long>(d->T) * d->k;
  const long long wide = std::max<long long>({d->D, 2ll * d->I, 2ll * d->I_sh});
  if (pairs * wide >= (1ll << 40) || pairs >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(d->M) * 2 * d->I * std::max(d->D, d->I) >= (1ll << 40))
    return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status_t check_weights(const moe_layer_desc_t* d, const moe_weights_t* w, bool routed, bool shared) {
  if (w == nullptr) return MOE_ERR_INVALID_ARG;
  if (routed) {
    if (w->w1 == nullptr || w->w2 == nullptr) return MOE_ERR_INVALID_ARG;
    if (d->act == MOE_ACT_GELU_TANH && d->has_bias && (w->b1 == nullptr || w->b2 == nullptr))
      return MOE_ERR_INVALID_ARG;
  }
  if (shared && d->I_sh > 0 && (w->sh_w1 == nullptr || w->sh_w2 == nullptr)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16) {
    if (routed && (!al16(w->w1) || !al16(w->w2))) return MOE_ERR_INVALID_ARG;
    if (shared && d->I_sh > 0 && (!al16(w->sh_w1) || !al16(w->sh_w2))) return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

// ---------------------------------------------------------------- layouts
// fp32 [T, M] logits, followed on the small-T path by the split partials.
inline int route_layout_splits(int T, int D, int dtype) {
  const int n = route_splits(T, D, dtype);
  return n > 1 ? n + 1 : 1;
}

struct RouteWs { size_t status, logits, wrT, total; };
RouteWs route_layout(int T, int D, int M, int dtype) {
  Carve c;
  RouteWs L;
  L.status = c.take(4);
  L.logits = c.take(static_cast<size_t>(route_layout_splits(T, D, dtype)) * T * M * 4);
  L.wrT = c.take(dtype == MOE_DTYPE_BF16 ? static_cast<size_t>(M) * D * 2 : 0);
  L.total = c.off;
  return L;
}

struct PermWs { size_t status, chunk_counts, chunk_base, total; };
PermWs perm_layout(int T, int k, int M) {
  Carve c;
  PermWs L;
  const size_t n = static_cast<size_t>(M) * perm_num_chunks(static_cast<long long>(T) * k);
  L.status = c.take(4);
  L.chunk_counts = c.take(n * 4);
  L.chunk_base = c.take(n * 4);
  L.total = c.off;
  return L;
}

struct FfnWs { size_t status, x_perm, h, total; };
FfnWs ffn_layout(const moe_layer_desc_t* d) {
  Carve c;
  FfnWs L;
  const size_t pairs = static_cast<size_t>(d->T) * d->k;
  L.status = c.take(4);
  L.x_perm = c.take(d->dtype == MOE_DTYPE_BF16 ? pairs * d->D * 2 : 0);
  L.h = c.take(pairs * d->I * esize(d->dtype));
  L.total = c.off;
  return L;
}

struct SharedWs { size_t status, h_sh, total; };
SharedWs shared_layout(const moe_layer_desc_t* d) {
  Carve c;
  SharedWs L;
  L.status = c.take(4);
  L.h_sh = c.take(static_cast<size_t>(d->T) * d->I_sh * esize(d->dtype));
  L.total = c.off;
  return L;
}

struct FwdWs {
  moe_ws_layout_t pub;
  size_t logits, wrT, chunk_counts, chunk_base, x_perm, h, h_sh, y_sh;
};
FwdWs forward_layout(const moe_layer_desc_t* d) {
  Carve c;
  FwdWs L;
  const size_t pairs = static_cast<size_t>(d->T) * d->k;
  const size_t es = esize(d->dtype);
  L.pub.status = c.take(4);
  L.pub.topk_idx = c.take(pairs * 4);
  L.pub.topk_w = c.take(pairs * 4);
  L.pub.counts = c.take(static_cast<size_t>(d->M) * 4);
  L.pub.offsets = c.take(static_cast<size_t>(d->M + 1) * 4);
  L.pub.slot_of = c.take(pairs * 4);
  L.pub.row_token = c.take(pairs * 4);
  L.pub.row_w = c.take(pairs * 4);
  L.pub.out_perm = c.take(pairs * d->D * 4);
  L.logits = c.take(static_cast<size_t>(route_layout_splits(d->T, d->D, d->dtype)) * d->T * d->M * 4);
  L.wrT = c.take(d->dtype == MOE_DTYPE_BF16 ? static_cast<size_t>(d->M) * d->D * 2 : 0);
  const size_t nch = static_cast<size_t>(d->M) * perm_num_chunks(static_cast<long long>(pairs));
  L.chunk_counts = c.take(nch * 4);
  L.chunk_base = c.take(nch * 4);
  L.x_perm = c.take(d->dtype == MOE_DTYPE_BF16 ? pairs * d->D * 2 : 0);
  L.h = c.take(pairs * d->I * es);
  L.h_sh = c.take(static_cast<size_t>(d->T) * d->I_sh * es);
  L.y_sh = c.take(d->I_sh > 0 ? static_cast<size_t>(d->T) * d->D * 4 : 0);
  L.pub.total = c.off;
  return L;
}

template <typename P> inline P at(void* ws, size_t off) {
  return reinterpret_cast<P>(static_cast<char*>(ws) + off);
}

// ------------------------------------------------------------ the stages
// Records caller-provided CUDA events at stage boundaries (profiled forward).
// NVTX range around a host-side stage (shows the stages on a profiler's
// timeline; a no-op unless a tool is attached).
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range&) = delete;
  Range& operator=(const Range&) = delete;
};

struct Marks {
  void* const* ev = nullptr;
  cudaStream_t s = nullptr;
  moe_status_t at(int i) const {
    if (ev == nullptr) return MOE_OK;
    return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s));
  }
};

moe_status_t run_route(const void* x, const void* w_r, const float* e_bias, int T, int D, int M, int k,
                       int dtype, int gate, int norm, float alpha, float eps, int n_group, int topk_group,
                       int32_t* idx, float* w, float* logits, void* wrT, int* status, cudaStream_t s) {
  const int nsplit = route_splits(T, D, dtype);
  if (dtype == MOE_DTYPE_BF16 && nsplit > 1) {
    // few tokens: split-K SIMT logits (no transpose, no tensor-core launch)
    float* partial = logits + static_cast<size_t>(T) * M;
    MOE_CUDA(launch_logits_splitk_bf16(x, w_r, partial, logits, T, D, M, s));
  } else if (dtype == MOE_DTYPE_BF16) {
    MOE_CUDA(launch_transpose_bf16(w_r, wrT, D, M, s));
    GemmLaunch L{};
    L.epi = EPI_STORE_F32;
    L.A = x; L.a_rows = T;
    L.B = wrT; L.b_rows = M;
    L.K = D;
    L.num_groups = 1; L.offsets = nullptr; L.rows_upper = T;
    L.bn = std::min(256, round_up(M, 16));
    L.n_tiles = (M + L.bn - 1) / L.bn;
    L.b_rows_per_group = M; L.b_row_step = L.bn; L.b_hi_offset = L.bn / 2;
    L.out_cols = M; L.out_col_step = L.bn; L.ldo = M;
    L.out = logits;
    L.status = status;
    MOE_CUDA(launch_gemm_sm100(L, s));
  } else {
    MOE_CUDA(launch_logits_f32(static_cast<const float*>(x), static_cast<const float*>(w_r), logits, T,
                               D, M, s));
  }
  MOE_CUDA(launch_topk(logits, gate == MOE_GATE_SIGMOID_BIAS ? e_bias : nullptr, T, M, k, gate,
                       norm, alpha, eps, n_group > 1 ? n_group : 1, topk_group, idx, w, s));
  return MOE_OK;
}

// slot_of (may be null): when given, x is copied into dispatch order by token
// (each row read once) instead of by dispatch row.
moe_status_t run_experts(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                         const int32_t* offsets, const int32_t* row_token, const float* row_w,
                         void* out_perm, void* x_perm, void* h, int* status, cudaStream_t s,
                         const Marks& mk = Marks(), const int32_t* slot_of = nullptr,
                         int* tile_ctrs = nullptr) {
  const int pairs = d->T * d->k;
  const bool swiglu = d->act == MOE_ACT_SWIGLU;
  const int n1 = swiglu ? 2 * d->I : d->I;
  const void* b1 = (!swiglu && d->has_bias) ? w->b1 : nullptr;
  const void* b2 = (!swiglu && d->has_bias) ? w->b2 : nullptr;
  // A handful of rows per expert (decode): tokens on M with single-CTA MMAs. The 128-row token
  // tile is mostly padding, but each CTA streams its own slice of the touched experts'
  // weights once (measured: GLM-4.5 decode expert GEMMs 0.837 -> 0.810 ms).
  if (d->dtype == MOE_DTYPE_BF16 && few_rows(d)) {
    MOE_CUDA(launch_gather_rows(x, row_token, offsets + d->M, x_perm, pairs, d->T, d->D, 2, status, s));
    MOE_TRY(mk.at(3));
    GemmLaunch g1{};
    g1.ncta = 1;
    g1.A = x_perm; g1.a_rows = pairs;
    g1.B = w->w1; g1.b_rows = static_cast<long long>(d->M) * n1;
    g1.K = d->D;
    g1.num_groups = d->M; g1.offsets = offsets; g1.rows_upper = pairs;
    if (swiglu) {
      const int half = std::min(128, round_up(d->I, 16));
      g1.epi = EPI_SWIGLU;
      g1.bn = 2 * half;
      g1.n_tiles = (d->I + half - 1) / half;
      g1.b_rows_per_group = n1; g1.b_row_step = half; g1.b_hi_offset = d->I;
      g1.out_col_step = half;
    } else {
      g1.epi = EPI_GELU_BIAS;
      g1.bn = std::min(256, round_up(d->I, 16));
      g1.n_tiles = (d->I + g1.bn - 1) / g1.bn;
      g1.b_rows_per_group = n1; g1.b_row_step = g1.bn; g1.b_hi_offset = g1.bn / 2;
      g1.out_col_step = g1.bn;
      g1.bias = b1;
    }
    g1.out_cols = d->I; g1.ldo = d->I; g1.out = h;
    g1.status = status;
    MOE_CUDA(launch_gemm_sm100(g1, s));
    MOE_TRY(mk.at(4));
    GemmLaunch g2{};
    g2.ncta = 1;
    g2.epi = EPI_SCALE_BIAS;
    g2.A = h; g2.a_rows = pairs;
    g2.B = w->w2; g2.b_rows = static_cast<long long>(d->M) * d->D;
    g2.K = d->I;
    g2.num_groups = d->M; g2.offsets = offsets; g2.rows_upper = pairs;
    g2.bn = std::min(256, round_up(d->D, 16));
    g2.n_tiles = (d->D + g2.bn - 1) / g2.bn;
    g2.b_rows_per_group = d->D; g2.b_row_step = g2.bn; g2.b_hi_offset = g2.bn / 2;
    g2.out_cols = d->D; g2.out_col_step = g2.bn; g2.ldo = d->D;
    g2.out = out_perm; g2.row_scale = row_w; g2.bias = b2;
    g2.status = status;
    MOE_CUDA(launch_gemm_sm100(g2, s));
    MOE_TRY(mk.at(5));
  } else if (d->dtype == MOE_DTYPE_BF16) {
    if (slot_of != nullptr)
      MOE_CUDA(launch_scatter_rows(x, slot_of, x_perm, d->T, d->k, d->D, status, s));
    else
      MOE_CUDA(launch_gather_rows(x, row_token, offsets + d->M, x_perm, pairs, d->T, d->D, 2, status, s));
    MOE_TRY(mk.at(3));
    SwapLaunch g1{};
    g1.W = w->w1; g1.w_rows = static_cast<long long>(d->M) * n1;
    g1.X = x_perm; g1.x_rows = pairs;
    g1.K = d->D;
    g1.num_groups = d->M; g1.offsets = offsets; g1.rows = pairs;
    if (swiglu) {
      g1.epi = EPI_SWIGLU;
      g1.w_rows_per_group = n1; g1.w_tile_step = 128; g1.w_hi_offset = d->I; g1.w_cta_step = 64;
      g1.cols_per_tile = 128;
    } else {
      g1.epi = EPI_GELU_BIAS;
      g1.w_rows_per_group = n1; g1.w_tile_step = 256; g1.w_hi_offset = 64; g1.w_cta_step = 128;
      g1.cols_per_tile = 256;
      g1.bias = b1;
    }
    g1.w_tiles = (d->I + g1.cols_per_tile - 1) / g1.cols_per_tile;
    g1.out_cols = d->I; g1.ldo = d->I; g1.out = h;
    g1.status = status;
    g1.tile_ctr = tile_ctrs;
    MOE_CUDA(launch_gemm_swap(g1, s));
    MOE_TRY(mk.at(4));

    SwapLaunch g2{};
    g2.epi = EPI_SCALE_BIAS;
    g2.W = w->w2; g2.w_rows = static_cast<long long>(d->M) * d->D;
    g2.X = h; g2.x_rows = pairs;
    g2.K = d->I;
    g2.num_groups = d->M; g2.offsets = offsets; g2.rows = pairs;
    g2.w_rows_per_group = d->D; g2.w_tile_step = 256; g2.w_hi_offset = 64; g2.w_cta_step = 128;
    g2.cols_per_tile = 256; g2.w_tiles = (d->D + 255) / 256;
    g2.out_cols = d->D; g2.ldo = d->D; g2.out = out_perm;
    g2.row_scale = row_w; g2.bias = b2;
    g2.status = status;
    g2.tile_ctr = tile_ctrs != nullptr ? tile_ctrs + 1 : nullptr;
    MOE_CUDA(launch_gemm_swap(g2, s));
    MOE_TRY(mk.at(5));
  } else {
    MOE_TRY(mk.at(3));
    SimtLaunch g1{};
    g1.epi = swiglu ? EPI_SWIGLU : EPI_GELU_BIAS;
    g1.A = static_cast<const float*>(x); g1.a_row_index = row_token; g1.K = d->D;
    g1.B = static_cast<const float*>(w->w1);
    g1.num_groups = d->M; g1.offsets = offsets; g1.rows = pairs;
    g1.b_rows_per_group = n1; g1.swiglu_hi = swiglu ? d->I : 0;
    g1.out_cols = d->I; g1.ldo = d->I; g1.out = static_cast<float*>(h);
    g1.bias = static_cast<const float*>(b1);
    MOE_CUDA(launch_simt_gemm(g1, s));
    MOE_TRY(mk.at(4));
    SimtLaunch g2{};
    g2.epi = EPI_SCALE_BIAS;
    g2.A = static_cast<const float*>(h); g2.a_row_index = nullptr; g2.K = d->I;
    g2.B = static_cast<const float*>(w->w2);
    g2.num_groups = d->M; g2.offsets = offsets; g2.rows = pairs;
    g2.b_rows_per_group = d->D;
    g2.out_cols = d->D; g2.ldo = d->D; g2.out = static_cast<float*>(out_perm);
    g2.row_scale = row_w; g2.bias = static_cast<const float*>(b2);
    MOE_CUDA(launch_simt_gemm(g2, s));
    MOE_TRY(mk.at(5));
  }
  return MOE_OK;
}

// Shared SwiGLU on all T tokens ([GLM45-SE] E_sh).  The down projection
// writes `out` in fp32 when out_f32 (the forward pass adds it in the
// combine), else in the layer's dtype.
moe_status_t run_shared(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x, void* out,
                        void* h_sh, bool out_f32, int* status, cudaStream_t s,
                        const Marks& mk = Marks()) {
  if (d->dtype == MOE_DTYPE_BF16) {
    SwapLaunch g1{};
    g1.epi = EPI_SWIGLU;
    g1.W = w->sh_w1; g1.w_rows = 2ll * d->I_sh;
    g1.X = x; g1.x_rows = d->T;
    g1.K = d->D;
    g1.num_groups = 1; g1.offsets = nullptr; g1.rows = d->T;
    g1.w_rows_per_group = 2 * d->I_sh; g1.w_tile_step = 128; g1.w_hi_offset = d->I_sh; g1.w_cta_step = 64;
    g1.cols_per_tile = 128; g1.w_tiles = (d->I_sh + 127) / 128;
    g1.out_cols = d->I_sh; g1.ldo = d->I_sh; g1.out = h_sh;
    g1.status = status;
    MOE_CUDA(launch_gemm_swap(g1, s));
    MOE_TRY(mk.at(6));
    SwapLaunch g2{};
    g2.epi = out_f32 ? EPI_STORE_F32 : EPI_STORE_BF16;
    g2.W = w->sh_w2; g2.w_rows = d->D;
    g2.X = h_sh; g2.x_rows = d->T;
    g2.K = d->I_sh;
    g2.num_groups = 1; g2.offsets = nullptr; g2.rows = d->T;
    g2.w_rows_per_group = d->D; g2.w_tile_step = 256; g2.w_hi_offset = 64; g2.w_cta_step = 128;
    g2.cols_per_tile = 256; g2.w_tiles = (d->D + 255) / 256;
    g2.out_cols = d->D; g2.ldo = d->D; g2.out = out;
    g2.status = status;
    MOE_CUDA(launch_gemm_swap(g2, s));
  } else {
    SimtLaunch g1{};
    g1.epi = EPI_SWIGLU;
    g1.A = static_cast<const float*>(x); g1.K = d->D;
    g1.B = static_cast<const float*>(w->sh_w1);
    g1.num_groups = 1; g1.offsets = nullptr; g1.rows = d->T;
    g1.b_rows_per_group = 2 * d->I_sh; g1.swiglu_hi = d->I_sh;
    g1.out_cols = d->I_sh; g1.ldo = d->I_sh; g1.out = static_cast<float*>(h_sh);
    MOE_CUDA(launch_simt_gemm(g1, s));
    MOE_TRY(mk.at(6));
    SimtLaunch g2{};
    g2.epi = EPI_STORE_F32;
    g2.A = static_cast<const float*>(h_sh); g2.K = d->I_sh;
    g2.B = static_cast<const float*>(w->sh_w2);
    g2.num_groups = 1; g2.offsets = nullptr; g2.rows = d->T;
    g2.b_rows_per_group = d->D;
    g2.out_cols = d->D; g2.ldo = d->D; g2.out = static_cast<float*>(out);
    MOE_CUDA(launch_simt_gemm(g2, s));
  }
  MOE_TRY(mk.at(7));
  return MOE_OK;
}

// One internal stream and two events per device and CUDA context, made on
// the first call that is not inside a stream capture.  At decode sizes the
// forward runs the shared expert there, beside the routing stage, and joins
// it back before the combine.  Lookups are serialised by `mu`, and a caller
// holds `mu` from the fork to the join, so that concurrent callers never
// interleave their records of the two events.
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr;
  cudaEvent_t join = nullptr;
  CUcontext ctx = nullptr;
  std::mutex mu;
};

CUcontext current_ctx() {
  using Fn = CUresult (*)(CUcontext*);
  static std::once_flag once;
  static Fn fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<Fn>(p);
  });
  CUcontext c = nullptr;
  if (fn == nullptr || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// The device's side stream, or nullptr (the caller then runs everything on
// its own stream): an unknown context, a capture in progress when the
// stream does not exist yet, or a failed creation.
SideStream* side_stream(cudaStream_t s) {
  constexpr int kDevices = 64;
  static SideStream sides[kDevices];
  static std::mutex make_mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return nullptr;
  const CUcontext ctx = current_ctx();
  if (ctx == nullptr) return nullptr;
  SideStream& x = sides[dev];
  std::lock_guard<std::mutex> lock(make_mu);
  if (x.st != nullptr && x.ctx == ctx) return &x;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone) return nullptr;
  // a context made anew invalidated the old handles: they are dropped, not destroyed
  x.st = nullptr;
  x.fork = x.join = nullptr;
  cudaStream_t st = nullptr;
  cudaEvent_t f = nullptr, j = nullptr;
  if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
  if (cudaEventCreateWithFlags(&f, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&j, cudaEventDisableTiming) != cudaSuccess) {
    if (f != nullptr) cudaEventDestroy(f);
    cudaStreamDestroy(st);
    return nullptr;
  }
  x.fork = f;
  x.join = j;
  x.ctx = ctx;
  x.st = st;
  return &x;
}

// Holds a side stream from the fork to the join.  The destructor joins it
// back if the caller returns early, so that no work the caller launched on
// the side stream can outlive the call's view of its workspace.
class SideFork {
 public:
  SideFork() = default;
  SideFork(const SideFork&) = delete;
  SideFork& operator=(const SideFork&) = delete;
  ~SideFork() { (void)join(); }
  // Makes the side stream wait for everything enqueued on s so far.
  moe_status_t fork(SideStream* side, cudaStream_t s) {
    lock_ = std::unique_lock<std::mutex>(side->mu);
    side_ = side;
    s_ = s;
    forked_ = true;
    if (cudaEventRecord(side->fork, s) != cudaSuccess) return MOE_ERR_CUDA;
    return cudaStreamWaitEvent(side->st, side->fork, 0) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  // Makes s wait for everything enqueued on the side stream so far.
  moe_status_t join() {
    if (!forked_) return MOE_OK;
    forked_ = false;
    moe_status_t st = MOE_OK;
    if (cudaEventRecord(side_->join, side_->st) != cudaSuccess ||
        cudaStreamWaitEvent(s_, side_->join, 0) != cudaSuccess)
      st = MOE_ERR_CUDA;
    lock_.unlock();
    return st;
  }

 private:
  std::unique_lock<std::mutex> lock_;
  SideStream* side_ = nullptr;
  cudaStream_t s_ = nullptr;
  bool forked_ = false;
};

}  // namespace

// =========================================================== public ABI
extern "C" {

const char* moe_status_string(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA";
    case MOE_ERR_DEVICE: return "MOE_ERR_DEVICE";
  }
  return "MOE_ERR_UNKNOWN";
}

const char* moe_version(void) { return "moe_b200 0.1 (sm_100a)"; }

moe_status_t moe_device_status(void* ws, void* stream, int* out) {
  if (ws == nullptr || out == nullptr) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int v = 0;
  MOE_CUDA(cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, s));
  MOE_CUDA(cudaStreamSynchronize(s));
  MOE_CUDA(cudaMemsetAsync(ws, 0, sizeof(int), s));
  *out = v;
  return MOE_OK;
}

size_t moe_route_workspace_size(int T, int D, int M, int dtype) {
  return route_layout(std::max(T, 0), std::max(D, 0), std::max(M, 0), dtype).total;
}

moe_status_t moe_route_topk(const void* x, const void* w_r, const float* e_bias, int T, int D, int M,
                            int k, int dtype, int gate, int norm_topk_prob,
                            float routed_scaling_factor, float eps, int n_group, int topk_group,
                            int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                            void* stream) {
  MOE_TRY(check_router_args(T, D, M, k, dtype, gate));
  MOE_TRY(check_groups(M, k, n_group, topk_group));
  if (!(eps >= 0.0f)) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  if (!x || !w_r || !topk_idx || !topk_w || !ws || !aligned_ws(ws)) return MOE_ERR_INVALID_ARG;
  if (dtype == MOE_DTYPE_BF16 && (!al16(x) || !al16(w_r))) return MOE_ERR_INVALID_ARG;
  const RouteWs L = route_layout(T, D, M, dtype);
  if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int*>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  return run_route(x, w_r, e_bias, T, D, M, k, dtype, gate, norm_topk_prob, routed_scaling_factor, eps,
                   n_group, topk_group, topk_idx, topk_w, at<float*>(ws, L.logits), at<void*>(ws, L.wrT),
                   status, s);
}

size_t moe_permute_workspace_size(int T, int k, int M) {
  return perm_layout(std::max(T, 0), std::max(k, 0), std::max(M, 0)).total;
}

moe_status_t moe_permute(const int32_t* topk_idx, const float* topk_w, int T, int k, int M,
                         int32_t* counts, int32_t* offsets, int32_t* slot_of, int32_t* row_token,
                         float* row_w, void* ws, size_t ws_bytes, void* stream) {
  if (T < 0 || k < 1 || M < 1 || k > M) return MOE_ERR_INVALID_ARG;
  if (M > kMaxExperts || k > kMaxTopK) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (!counts || !offsets || !ws || !aligned_ws(ws)) return MOE_ERR_INVALID_ARG;
  if (T > 0 && (!topk_idx || !topk_w || !slot_of || !row_token || !row_w)) return MOE_ERR_INVALID_ARG;
  const PermWs L = perm_layout(T, k, M);
  if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int*>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  if (T == 0) {
    MOE_CUDA(cudaMemsetAsync(counts, 0, static_cast<size_t>(M) * 4, s));
    MOE_CUDA(cudaMemsetAsync(offsets, 0, static_cast<size_t>(M + 1) * 4, s));
    return MOE_OK;
  }
  MOE_CUDA(launch_permute(topk_idx, topk_w, T, k, M, counts, offsets, slot_of, row_token, row_w,
                          at<int32_t*>(ws, L.chunk_counts), at<int32_t*>(ws, L.chunk_base), status, s));
  return MOE_OK;
}

moe_status_t moe_capacity_drop(int32_t* topk_idx, const int32_t* slot_of, const int32_t* offsets, int T, int k,
                               int M, int capacity, void* stream) {
  if (T < 0 || k < 1 || M < 1 || capacity < 0) return MOE_ERR_INVALID_ARG;
  if (M > kMaxExperts || static_cast<long long>(T) * k >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!topk_idx || !slot_of || !offsets) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  return cuda_status(launch_capacity_drop(topk_idx, slot_of, offsets, T, k, M, capacity,
                                          static_cast<cudaStream_t>(stream)));
}

int moe_expert_capacity(double factor, int T, int k, int M) {
  if (!(factor >= 0.0) || M < 1 || T < 0 || k < 1) return -1;
  const double c = std::ceil(factor * static_cast<double>(T) * k / M - 1e-12);
  return c > 2147483647.0 ? 2147483647 : static_cast<int>(c);
}

moe_status_t moe_gather_rows(const void* x, const int32_t* row_token, const int32_t* n_rows, void* x_perm,
                             int rows, int T, int D, int dtype, int32_t* device_status, void* stream) {
  if (rows < 0 || T < 0 || D < 1) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_F32 && dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!x || !row_token || !x_perm) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  return cuda_status(launch_gather_rows(x, row_token, n_rows, x_perm, rows, T, D, static_cast<int>(esize(dtype)),
                                        device_status, static_cast<cudaStream_t>(stream)));
}

size_t moe_expert_ffn_workspace_size(const moe_layer_desc_t* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return ffn_layout(d).total;
}

moe_status_t moe_expert_ffn(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                            const int32_t* offsets, const int32_t* row_token, const float* row_w,
                            void* out_perm, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_desc(d));
  MOE_TRY(check_weights(d, w, true, false));
  if (d->T == 0) return MOE_OK;
  if (!x || !offsets || !row_token || !row_w || !out_perm || !ws || !aligned_ws(ws))
    return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16 && !al16(x)) return MOE_ERR_INVALID_ARG;
  const FfnWs L = ffn_layout(d);
  if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int*>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  return run_experts(d, w, x, offsets, row_token, row_w, out_perm, at<void*>(ws, L.x_perm),
                     at<void*>(ws, L.h), status, s);
}

size_t moe_shared_expert_workspace_size(const moe_layer_desc_t* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return shared_layout(d).total;
}

moe_status_t moe_shared_expert(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                               void* y_sh, void* ws, size_t ws_bytes, void* stream) {
  MOE_TRY(check_desc(d));
  if (d->I_sh == 0) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_weights(d, w, false, true));
  if (d->T == 0) return MOE_OK;
  if (!x || !y_sh || !ws || !aligned_ws(ws)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16 && !al16(x)) return MOE_ERR_INVALID_ARG;
  const SharedWs L = shared_layout(d);
  if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = at<int*>(ws, L.status);
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  return run_shared(d, w, x, y_sh, at<void*>(ws, L.h_sh), false, status, s);
}

moe_status_t moe_combine(const moe_layer_desc_t* d, const void* out_perm, const int32_t* slot_of,
                         const void* shared_out, const void* addend, void* y, void* stream) {
  MOE_TRY(check_desc(d));
  if (d->T == 0) return MOE_OK;
  if (!out_perm || !slot_of || !y) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  MOE_CUDA(launch_combine(d->dtype, out_perm, slot_of, shared_out, false, addend, y, d->T, d->D, d->k,
                          static_cast<cudaStream_t>(stream)));
  return MOE_OK;
}

}  // extern "C"

// ------------------------------------------------------------ dense FFN layer

namespace {

moe_status_t check_dense(const moe_dense_desc_t* d) {
  if (d == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->T < 0 || d->D < 1 || d->I < 1) return MOE_ERR_INVALID_ARG;
  if (d->dtype != MOE_DTYPE_F32 && d->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (d->act != MOE_ACT_GELU_TANH && d->act != MOE_ACT_SWIGLU) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16 && (d->D % 16 != 0 || d->I % 16 != 0)) return MOE_ERR_UNSUPPORTED;
  const long long wide = std::max<long long>(d->D, 2ll * d->I);
  if (static_cast<long long>(d->T) * wide >= (1ll << 40) || d->T >= (1 << 30)) return MOE_ERR_UNSUPPORTED;
  if (2ll * d->I * std::max(d->D, d->I) >= (1ll << 40)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

struct DenseWs { size_t status, h, total; };
DenseWs dense_layout(const moe_dense_desc_t* d) {
  Carve c;
  DenseWs L;
  L.status = c.take(4);
  L.h = c.take(static_cast<size_t>(d->T) * d->I * esize(d->dtype));
  L.total = c.off;
  return L;
}

moe_status_t dense_impl(const moe_dense_desc_t* d, const void* w1, const void* b1, const void* w2,
                        const void* b2, const void* x, const void* addend, void* y, void* ws,
                        size_t ws_bytes, cudaStream_t s, void* const* events) {
  MOE_TRY(check_dense(d));
  if (d->T == 0) return MOE_OK;
  const bool swiglu = d->act == MOE_ACT_SWIGLU;
  const bool bias = !swiglu && d->has_bias;
  if (!w1 || !w2 || !x || !y || !ws || !aligned_ws(ws)) return MOE_ERR_INVALID_ARG;
  if (bias && (!b1 || !b2)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16 && (!al16(x) || !al16(w1) || !al16(w2))) return MOE_ERR_INVALID_ARG;
  const DenseWs L = dense_layout(d);
  if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  Marks mk;
  mk.ev = events;
  mk.s = s;
  int* status = at<int*>(ws, L.status);
  void* h = at<void*>(ws, L.h);
  Range whole("moe_dense_ffn");
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  MOE_TRY(mk.at(0));
  if (d->dtype == MOE_DTYPE_BF16) {
    SwapLaunch g1{};
    g1.W = w1; g1.w_rows = swiglu ? 2ll * d->I : d->I;
    g1.X = x; g1.x_rows = d->T;
    g1.K = d->D;
    g1.num_groups = 1; g1.offsets = nullptr; g1.rows = d->T;
    if (swiglu) {
      g1.epi = EPI_SWIGLU;
      g1.w_rows_per_group = 2 * d->I; g1.w_tile_step = 128; g1.w_hi_offset = d->I; g1.w_cta_step = 64;
      g1.cols_per_tile = 128;
    } else {
      g1.epi = EPI_GELU_BIAS;
      g1.w_rows_per_group = d->I; g1.w_tile_step = 256; g1.w_hi_offset = 64; g1.w_cta_step = 128;
      g1.cols_per_tile = 256;
      g1.bias = bias ? b1 : nullptr;
    }
    g1.w_tiles = (d->I + g1.cols_per_tile - 1) / g1.cols_per_tile;
    g1.out_cols = d->I; g1.ldo = d->I; g1.out = h;
    g1.status = status;
    MOE_CUDA(launch_gemm_swap(g1, s));
    MOE_TRY(mk.at(1));
    SwapLaunch g2{};
    g2.epi = EPI_BIAS_ADD;
    g2.W = w2; g2.w_rows = d->D;
    g2.X = h; g2.x_rows = d->T;
    g2.K = d->I;
    g2.num_groups = 1; g2.offsets = nullptr; g2.rows = d->T;
    g2.w_rows_per_group = d->D; g2.w_tile_step = 256; g2.w_hi_offset = 64; g2.w_cta_step = 128;
    g2.cols_per_tile = 256; g2.w_tiles = (d->D + 255) / 256;
    g2.out_cols = d->D; g2.ldo = d->D; g2.out = y;
    g2.bias = bias ? b2 : nullptr;
    g2.addend = addend;
    g2.status = status;
    MOE_CUDA(launch_gemm_swap(g2, s));
    MOE_TRY(mk.at(2));
  } else {
    SimtLaunch g1{};
    g1.epi = swiglu ? EPI_SWIGLU : EPI_GELU_BIAS;
    g1.A = static_cast<const float*>(x); g1.K = d->D;
    g1.B = static_cast<const float*>(w1);
    g1.num_groups = 1; g1.offsets = nullptr; g1.rows = d->T;
    g1.b_rows_per_group = swiglu ? 2 * d->I : d->I; g1.swiglu_hi = swiglu ? d->I : 0;
    g1.out_cols = d->I; g1.ldo = d->I; g1.out = static_cast<float*>(h);
    g1.bias = bias ? static_cast<const float*>(b1) : nullptr;
    MOE_CUDA(launch_simt_gemm(g1, s));
    MOE_TRY(mk.at(1));
    SimtLaunch g2{};
    g2.epi = EPI_BIAS_ADD;
    g2.A = static_cast<const float*>(h); g2.K = d->I;
    g2.B = static_cast<const float*>(w2);
    g2.num_groups = 1; g2.offsets = nullptr; g2.rows = d->T;
    g2.b_rows_per_group = d->D;
    g2.out_cols = d->D; g2.ldo = d->D; g2.out = static_cast<float*>(y);
    g2.bias = bias ? static_cast<const float*>(b2) : nullptr;
    g2.addend = static_cast<const float*>(addend);
    MOE_CUDA(launch_simt_gemm(g2, s));
    MOE_TRY(mk.at(2));
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_dense_ffn_workspace_size(const moe_dense_desc_t* d) {
  if (check_dense(d) != MOE_OK) return 0;
  return dense_layout(d).total;
}

moe_status_t moe_dense_ffn(const moe_dense_desc_t* d, const void* w1, const void* b1, const void* w2,
                           const void* b2, const void* x, const void* addend, void* y, void* ws,
                           size_t ws_bytes, void* stream) {
  return dense_impl(d, w1, b1, w2, b2, x, addend, y, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                    nullptr);
}

moe_status_t moe_dense_ffn_profiled(const moe_dense_desc_t* d, const void* w1, const void* b1,
                                    const void* w2, const void* b2, const void* x, const void* addend,
                                    void* y, void* ws, size_t ws_bytes, void* stream,
                                    void* const* events, int n_events) {
  if (events == nullptr || n_events != MOE_NUM_DENSE_EVENTS) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (events[i] == nullptr) return MOE_ERR_INVALID_ARG;
  return dense_impl(d, w1, b1, w2, b2, x, addend, y, ws, ws_bytes, static_cast<cudaStream_t>(stream),
                    events);
}

size_t moe_workspace_size(const moe_layer_desc_t* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return forward_layout(d).pub.total;
}

moe_status_t moe_workspace_layout(const moe_layer_desc_t* d, moe_ws_layout_t* out) {
  MOE_TRY(check_desc(d));
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = forward_layout(d).pub;
  return MOE_OK;
}

static moe_status_t forward_impl(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                                 const void* addend, void* y, void* ws, size_t ws_bytes, cudaStream_t s,
                                 void* const* events) {
  MOE_TRY(check_desc(d));
  MOE_TRY(check_weights(d, w, true, true));
  if (w->w_r == nullptr) return MOE_ERR_INVALID_ARG;
  if (d->T == 0) return MOE_OK;
  if (!x || !y || !ws || !aligned_ws(ws)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16 && (!al16(x) || !al16(w->w_r))) return MOE_ERR_INVALID_ARG;
  const FwdWs L = forward_layout(d);
  if (ws_bytes < L.pub.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  Marks mk;
  mk.ev = events;
  mk.s = s;
  int* status = at<int*>(ws, L.pub.status);
  int32_t* idx = at<int32_t*>(ws, L.pub.topk_idx);
  float* tw = at<float*>(ws, L.pub.topk_w);
  int32_t* counts = at<int32_t*>(ws, L.pub.counts);
  int32_t* offsets = at<int32_t*>(ws, L.pub.offsets);
  int32_t* slot_of = at<int32_t*>(ws, L.pub.slot_of);
  int32_t* row_token = at<int32_t*>(ws, L.pub.row_token);
  float* row_w = at<float*>(ws, L.pub.row_w);
  void* out_perm = at<void*>(ws, L.pub.out_perm);
  Range whole("moe_forward");
  // the status flag and, in the same 256-byte slot of the workspace, the
  // tile counters of the two routed expert GEMMs (ints 2 and 3), which
  // must be 0 when their launches start
  int* tile_ctrs = status + 2;
  MOE_CUDA(cudaMemsetAsync(status, 0, 4 * sizeof(int), s));
  // At decode sizes the shared expert's two GEMMs stream their weights
  // through a few CTA pairs, each waiting on its whole K in turn, while the
  // routing stage's small kernels leave most SMs idle.  The shared expert
  // reads only x, so it runs on the side stream under the routing stage and
  // joins before the combine.  Its outputs go to their own workspace
  // regions, which no other stage touches.
  void* y_sh = d->I_sh > 0 ? at<void*>(ws, L.y_sh) : nullptr;
  SideFork shared_fork;
  bool shared_done = false;
  if (d->I_sh > 0 && d->dtype == MOE_DTYPE_BF16 && few_rows(d)) {
    if (SideStream* side = side_stream(s)) {
      Range r("moe.shared_expert");
      MOE_TRY(shared_fork.fork(side, s));
      MOE_TRY(run_shared(d, w, x, y_sh, at<void*>(ws, L.h_sh), true, status, side->st));
      shared_done = true;
    }
  }
  MOE_TRY(mk.at(0));
  {
    Range r("moe.route");
    MOE_TRY(run_route(x, w->w_r, w->e_bias, d->T, d->D, d->M, d->k, d->dtype, d->gate, d->norm_topk_prob,
                      d->routed_scaling_factor, d->eps, d->n_group, d->topk_group, idx, tw,
                      at<float*>(ws, L.logits), at<void*>(ws, L.wrT), status, s));
  }
  MOE_TRY(mk.at(1));
  {
    Range r("moe.dispatch");
    MOE_CUDA(launch_permute(idx, tw, d->T, d->k, d->M, counts, offsets, slot_of, row_token, row_w,
                            at<int32_t*>(ws, L.chunk_counts), at<int32_t*>(ws, L.chunk_base), status, s));
  }
  MOE_TRY(mk.at(2));
  // x larger than half the L2: copy it into dispatch order by token, so that each row is read
  // from HBM once (measured: GLM-4.5 prefill 0.43 -> 0.30 ms); smaller x is read through L2
  // either way and the per-row gather has more parallelism (decode, GLaM)
  const bool by_token = static_cast<double>(d->T) * d->D * esize(d->dtype) > 64.0 * 1024 * 1024;
  {
    Range r("moe.experts");
    MOE_TRY(run_experts(d, w, x, offsets, row_token, row_w, out_perm, at<void*>(ws, L.x_perm),
                        at<void*>(ws, L.h), status, s, mk, by_token ? slot_of : nullptr, tile_ctrs));
  }
  if (shared_done) {
    MOE_TRY(shared_fork.join());
    MOE_TRY(mk.at(6));
    MOE_TRY(mk.at(7));
  } else if (d->I_sh > 0) {
    Range r("moe.shared_expert");
    MOE_TRY(run_shared(d, w, x, y_sh, at<void*>(ws, L.h_sh), true, status, s, mk));
  } else {
    MOE_TRY(mk.at(6));
    MOE_TRY(mk.at(7));
  }
  {
    Range r("moe.combine");
    MOE_CUDA(launch_combine(d->dtype, out_perm, slot_of, y_sh, true, addend, y, d->T, d->D, d->k, s));
  }
  MOE_TRY(mk.at(8));
  return MOE_OK;
}

moe_status_t moe_forward(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x, void* y,
                         void* ws, size_t ws_bytes, void* stream) {
  return forward_impl(d, w, x, nullptr, y, ws, ws_bytes, static_cast<cudaStream_t>(stream), nullptr);
}

moe_status_t moe_forward_add(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                             const void* addend, void* y, void* ws, size_t ws_bytes, void* stream) {
  if (d != nullptr && d->T > 0 && addend == nullptr) return MOE_ERR_INVALID_ARG;
  return forward_impl(d, w, x, addend, y, ws, ws_bytes, static_cast<cudaStream_t>(stream), nullptr);
}

moe_status_t moe_forward_profiled(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                                  void* y, void* ws, size_t ws_bytes, void* stream,
                                  void* const* events, int n_events) {
  if (events == nullptr || n_events != MOE_NUM_STAGE_EVENTS) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (events[i] == nullptr) return MOE_ERR_INVALID_ARG;
  return forward_impl(d, w, x, nullptr, y, ws, ws_bytes, static_cast<cudaStream_t>(stream), events);
}

int moe_forward_launch_count(const moe_layer_desc_t* d) {
  if (check_desc(d) != MOE_OK || d->T == 0) return 0;
  const bool bf16 = d->dtype == MOE_DTYPE_BF16;
  int n = bf16 ? 3 : 2;  // transpose + logits GEMM or split-K logits + reduction; top-k
  n += static_cast<long long>(d->T) * d->k <= 2048 ? 1 : 3;          // counting sort (1 or 3 kernels)
  n += bf16 ? 3 : 2;      // [gather,] first GEMM, second GEMM
  n += d->I_sh > 0 ? 3 : 1;  // [shared first GEMM, shared second GEMM,] combine
  return n;
}

void moe_algorithmic_work(const moe_layer_desc_t* d, const int32_t* counts_host, double* flops,
                          double* bytes) {
  double f = 0.0, b = 0.0;
  if (d != nullptr && check_desc(d) == MOE_OK) {
    const double es = static_cast<double>(esize(d->dtype));
    const double D = d->D, I = d->I, T = d->T, Ish = d->I_sh;
    const bool swiglu = d->act == MOE_ACT_SWIGLU;
    const double n1 = swiglu ? 2.0 * I : I;
    const double bias_params = (!swiglu && d->has_bias) ? (I + D) : 0.0;
    f += 2.0 * T * D * d->M;           // router
    b += D * d->M * es + T * D * es * 2.0;  // W_r, x in, y out
    if (d->gate == MOE_GATE_SIGMOID_BIAS) b += 4.0 * d->M;
    for (int e = 0; e < d->M; ++e) {
      const double c = counts_host ? counts_host[e] : 0.0;
      if (c <= 0) continue;
      f += c * (2.0 * D * n1 + 2.0 * I * D);
      b += (n1 * D + D * I + bias_params) * es;
    }
    if (Ish > 0) {
      f += T * (2.0 * D * 2.0 * Ish + 2.0 * Ish * D);
      b += 3.0 * D * Ish * es;
    }
  }
  if (flops) *flops = f;
  if (bytes) *bytes = b;
}

}  // extern "C"

// =========================================================== backward
namespace {

// The forward's layout first (route, dispatch order, out_perm = the experts'
// recomputed outputs), then the backward's fp32 rows.
struct BwdWs {
  FwdWs f;
  size_t xp, hpre, act, dO, da, dxp, dwp, dl, hs, as, das, dxs, total;
  // tensor-core path (bf16): the padded dispatch order and its bf16 tensors
  long long rows_pad;
  size_t offp, slotp, rtp, rwp, xpp, dypp, hpb, awb, dhb, dxpp, parts, hsb, asb, dhsb, rpart, dlb;
};

// Chunks of the token sum in the router's weight gradient dW_r = x^T dlogits
// (partial sums added in order): enough blocks to fill the GPU.
int router_ksplit(int T) { return std::max(1, std::min(16, T / 1024)); }

// A bf16 layer runs the router's two backward GEMMs (dW_r = x^T dlogits and
// dx += dlogits W_r^T) on the tensor cores, with dlogits rounded to bf16 as
// their operand, when every TMA box of them has whole rows: M a multiple of
// 8 and at least one 64-column box wide.  Otherwise (small test layers) on
// the CUDA cores in fp32.
bool router_bwd_tc(const moe_layer_desc_t* d) {
  return d->dtype == MOE_DTYPE_BF16 && d->M % 8 == 0 && d->M >= 64;
}

// Rows of the backward's padded dispatch order: every expert's segment is
// rounded up to 64 rows, so at most T k + 63 M rows.
long long padded_rows(const moe_layer_desc_t* d) {
  return (static_cast<long long>(d->T) * d->k + 63ll * d->M + 63) / 64 * 64;
}

BwdWs backward_layout_tc(const moe_layer_desc_t* d) {
  BwdWs L{};
  L.f = forward_layout(d);
  Carve c;
  c.off = L.f.pub.total;
  const size_t pairs = static_cast<size_t>(d->T) * d->k;
  const size_t n1 = d->act == MOE_ACT_SWIGLU ? 2ull * d->I : static_cast<size_t>(d->I);
  const size_t Ha = d->I, T = d->T, Is = d->I_sh, D = d->D;
  const size_t P = static_cast<size_t>(padded_rows(d));
  L.rows_pad = static_cast<long long>(P);
  L.offp = c.take((d->M + 1) * 4);
  L.slotp = c.take(pairs * 4);
  L.rtp = c.take(P * 4);
  L.rwp = c.take(P * 4);
  L.xpp = c.take(P * D * 2);
  L.dypp = c.take(P * D * 2);
  L.hpb = c.take(P * n1 * 4);  // fp32 pre-activations: they feed act' and <G, a> unrounded
  L.awb = c.take(P * Ha * 2);
  L.dhb = c.take(P * n1 * 2);
  L.dxpp = c.take(P * D * 4);
  L.parts = c.take(P * ((Ha + 31) / 32) * 4);
  L.dwp = c.take(pairs * 4);
  L.dl = c.take(T * d->M * 4);
  L.hsb = c.take(T * 2 * Is * 4);
  L.asb = c.take(T * Is * 2);
  L.dhsb = c.take(T * 2 * Is * 2);
  L.dxs = c.take(T * D * 4);
  L.rpart = router_bwd_tc(d) ? 0 : c.take(static_cast<size_t>(router_ksplit(d->T)) * D * d->M * 4);
  L.dlb = router_bwd_tc(d) ? c.take(T * d->M * 2) : 0;
  L.total = c.off;
  return L;
}

BwdWs backward_layout(const moe_layer_desc_t* d) {
  if (d->dtype == MOE_DTYPE_BF16) return backward_layout_tc(d);
  BwdWs L{};
  L.f = forward_layout(d);
  Carve c;
  c.off = L.f.pub.total;
  const size_t pairs = static_cast<size_t>(d->T) * d->k;
  const size_t n1 = d->act == MOE_ACT_SWIGLU ? 2ull * d->I : static_cast<size_t>(d->I);
  const size_t Ha = d->I, T = d->T, Is = d->I_sh;
  L.xp = c.take(pairs * d->D * esize(d->dtype));
  L.hpre = c.take(pairs * n1 * 4);  // pre-activations, then their gradient in place
  L.act = c.take(pairs * Ha * 4);
  L.dO = c.take(pairs * d->D * 4);
  L.da = c.take(pairs * Ha * 4);
  L.dxp = c.take(pairs * d->D * 4);
  L.dwp = c.take(pairs * 4);
  L.dl = c.take(T * d->M * 4);
  L.hs = c.take(T * 2 * Is * 4);
  L.as = c.take(T * Is * 4);
  L.das = c.take(T * Is * 4);
  L.dxs = c.take(T * d->D * 4);
  L.total = c.off;
  return L;
}

// C = A B^T with A(m, k) = A[m a_sm + k a_sk] and B(n, k) = B[g b_gstride + n b_sn + k b_sk].
BwdGemmLaunch bwd_gemm(const void* A, long long a_sm, long long a_sk, bool a_bf16, const void* B, long long b_sn,
                       long long b_sk, long long b_gstride, bool b_bf16, float* C, long long ldc, long long rows,
                       long long K, int N) {
  BwdGemmLaunch L{};
  L.A = A; L.a_sm = a_sm; L.a_sk = a_sk; L.a_bf16 = a_bf16;
  L.B = B; L.b_sn = b_sn; L.b_sk = b_sk; L.b_gstride = b_gstride; L.b_bf16 = b_bf16;
  L.C = C; L.ldc = ldc;
  L.rows = rows; L.K = K; L.N = N;
  return L;
}

moe_status_t zero_param_grads(const moe_layer_desc_t* d, const moe_grads_t* g, cudaStream_t s) {
  const bool swiglu = d->act == MOE_ACT_SWIGLU;
  const size_t n1 = swiglu ? 2ull * d->I : static_cast<size_t>(d->I);
  const size_t D = d->D, M = d->M, Ha = d->I, Is = d->I_sh;
  MOE_CUDA(cudaMemsetAsync(g->dw_r, 0, D * M * 4, s));
  MOE_CUDA(cudaMemsetAsync(g->dw1, 0, M * n1 * D * 4, s));
  MOE_CUDA(cudaMemsetAsync(g->dw2, 0, M * D * Ha * 4, s));
  if (!swiglu && d->has_bias) {
    MOE_CUDA(cudaMemsetAsync(g->db1, 0, M * Ha * 4, s));
    MOE_CUDA(cudaMemsetAsync(g->db2, 0, M * D * 4, s));
  }
  if (Is > 0) {
    MOE_CUDA(cudaMemsetAsync(g->dsh_w1, 0, 2 * Is * D * 4, s));
    MOE_CUDA(cudaMemsetAsync(g->dsh_w2, 0, D * Is * 4, s));
  }
  return MOE_OK;
}

// A tokens-on-N GEMM of the backward: A is the weight stack (K-major for
// the recomputed forward, MN-major for the input gradients) or an MN-major
// activation (weight gradients), B the token rows.
SwapLaunch bwd_swap(int epi, int layout, const void* A, long long a_rows, const void* B, long long b_rows, int K,
                    int G, const int32_t* offsets, const int32_t* counts, long long rows, int out_cols, void* out,
                    int ldo, int* status) {
  SwapLaunch L{};
  L.epi = epi;
  L.layout = layout;
  L.W = A;
  L.w_rows = a_rows;
  L.X = B;
  L.x_rows = b_rows;
  L.K = K;
  L.num_groups = G;
  L.offsets = offsets;
  L.counts = counts;
  L.rows = rows;
  L.w_tiles = (out_cols + 255) / 256;
  L.w_tile_step = 256;
  L.w_hi_offset = 64;
  L.w_cta_step = 128;
  L.cols_per_tile = 256;
  L.out_cols = out_cols;
  L.a_cols = out_cols;
  L.ldo = ldo;
  L.out = out;
  L.status = status;
  return L;
}

// The backward of a bf16 layer on the tensor cores.  Per expert segment
// (rows r of the padded dispatch order, token t(r), gate weight w_r):
//   recompute  h = x W1^T (+ b1) (fp32), a = act(h), aw = w a   (save epilogue)
//   dgrad      G = dy W2;  dh = w G act'(h);  parts = <G, a>   (fused epilogue)
//              dx_rows = dh W1                                  (fp32)
//   wgrad      dW2 = dy^T aw,  dW1 = dh^T x  over the segment   (grouped-K GEMMs)
//   dw[t, j]   = <G, a> + <dy_t, b2>  (the gradient reaching the gate weight)
// then the shared expert the same way with w = 1, the router's backward, and
// dx_t = sum_j dx_rows + shared dx + router dx, rounded once.
moe_status_t backward_tc_impl(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x, const void* dy,
                              const moe_grads_t* g, void* ws, cudaStream_t s) {
  const bool swiglu = d->act == MOE_ACT_SWIGLU;
  const bool biases = !swiglu && d->has_bias;
  const BwdWs L = backward_layout(d);
  const int T = d->T, D = d->D, M = d->M, k = d->k, Ha = d->I, Is = d->I_sh;
  const int n1 = swiglu ? 2 * d->I : d->I;
  const long long pairs = static_cast<long long>(T) * k;
  const long long P = L.rows_pad;
  const int nparts = (Ha + 31) / 32;
  int* status = at<int*>(ws, L.f.pub.status);
  int32_t* idx = at<int32_t*>(ws, L.f.pub.topk_idx);
  float* tw = at<float*>(ws, L.f.pub.topk_w);
  int32_t* counts = at<int32_t*>(ws, L.f.pub.counts);
  int32_t* offsets = at<int32_t*>(ws, L.f.pub.offsets);
  int32_t* slot_of = at<int32_t*>(ws, L.f.pub.slot_of);
  int32_t* row_token = at<int32_t*>(ws, L.f.pub.row_token);
  float* row_w = at<float*>(ws, L.f.pub.row_w);
  float* logits = at<float*>(ws, L.f.logits);
  int32_t* offp = at<int32_t*>(ws, L.offp);
  int32_t* slotp = at<int32_t*>(ws, L.slotp);
  int32_t* rtp = at<int32_t*>(ws, L.rtp);
  float* rwp = at<float*>(ws, L.rwp);
  void* xpp = at<void*>(ws, L.xpp);
  void* dypp = at<void*>(ws, L.dypp);
  void* hpb = at<void*>(ws, L.hpb);
  void* awb = at<void*>(ws, L.awb);
  void* dhb = at<void*>(ws, L.dhb);
  float* dxpp = at<float*>(ws, L.dxpp);
  float* parts = at<float*>(ws, L.parts);
  float* dwp = at<float*>(ws, L.dwp);
  float* dl = at<float*>(ws, L.dl);
  float* dxs = at<float*>(ws, L.dxs);
  const int32_t* n_rows_pad = offp + M;
  Range whole("moe_backward");
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  {
    Range r("moe.route");
    MOE_TRY(run_route(x, w->w_r, w->e_bias, T, D, M, k, d->dtype, d->gate, d->norm_topk_prob,
                      d->routed_scaling_factor, d->eps, d->n_group, d->topk_group, idx, tw, logits,
                      at<void*>(ws, L.f.wrT), status, s));
  }
  {
    Range r("moe.dispatch");
    MOE_CUDA(launch_permute(idx, tw, T, k, M, counts, offsets, slot_of, row_token, row_w,
                            at<int32_t*>(ws, L.f.chunk_counts), at<int32_t*>(ws, L.f.chunk_base), status, s));
    MOE_CUDA(launch_pad_dispatch(idx, slot_of, tw, counts, offsets, T, k, M, P, offp, slotp, rtp, rwp, s));
    MOE_CUDA(launch_gather_pad(x, rtp, n_rows_pad, xpp, P, T, D, s));
    MOE_CUDA(launch_gather_pad(dy, rtp, n_rows_pad, dypp, P, T, D, s));
    // padding rows of the weight-gradient operands that no GEMM tile writes
    MOE_CUDA(launch_zero_pad_rows(counts, offp, M, awb, P, Ha, s));
    MOE_CUDA(launch_zero_pad_rows(counts, offp, M, dhb, P, n1, s));
  }
  {
    Range r("moe.experts_backward");
    // recompute: h (fp32) and aw = w a (bf16, the operand of dW2).  The unscaled a is not kept:
    // the input-gradient epilogue forms <G, a> from h itself.
    SwapLaunch ga{};
    if (swiglu) {
      ga = bwd_swap(EPI_BWD_SWIGLU_SAVE, kSwFwd, w->w1, 1ll * M * n1, xpp, P, D, M, offp, counts, P, Ha, hpb, n1,
                    status);
      ga.w_rows_per_group = n1;
      ga.w_tiles = (Ha + 127) / 128;
      ga.w_tile_step = 128;
      ga.w_hi_offset = Ha;
      ga.w_cta_step = 64;
      ga.cols_per_tile = 128;
      ga.half_cols = Ha;
    } else {
      ga = bwd_swap(EPI_BWD_GELU_SAVE, kSwFwd, w->w1, 1ll * M * Ha, xpp, P, D, M, offp, counts, P, Ha, hpb, Ha,
                    status);
      ga.w_rows_per_group = Ha;
      ga.bias = biases ? w->b1 : nullptr;
    }
    ga.out2 = nullptr;
    ga.out3 = awb;
    ga.ldo2 = Ha;
    ga.row_scale = rwp;
    MOE_CUDA(launch_gemm_swap(ga, s));
    // G = dy W2 (W2 read MN-major); dh = w G act'(h); per-32-column <G, a>
    SwapLaunch gb = bwd_swap(swiglu ? EPI_BWD_SWIGLU_DACT : EPI_BWD_GELU_DACT, kSwDgrad, w->w2, 1ll * M * D, dypp,
                             P, D, M, offp, counts, P, Ha, dhb, n1, status);
    gb.k_rows_per_group = D;
    gb.aux = hpb;
    gb.ld_aux = n1;
    gb.half_cols = Ha;
    gb.row_scale = rwp;
    gb.parts = parts;
    gb.ld_parts = nparts;
    MOE_CUDA(launch_gemm_swap(gb, s));
    // dx rows = dh W1 (W1 read MN-major), fp32
    SwapLaunch gc = bwd_swap(EPI_STORE_F32, kSwDgrad, w->w1, 1ll * M * n1, dhb, P, n1, M, offp, counts, P, D, dxpp,
                             D, status);
    gc.k_rows_per_group = n1;
    MOE_CUDA(launch_gemm_swap(gc, s));
    // weight gradients over each expert's padded segment
    SwapLaunch gd = bwd_swap(EPI_STORE_F32, kSwWgrad, awb, P, dypp, P, 0, M, offp, nullptr, P, Ha, g->dw2, Ha,
                             status);
    gd.b_cols = D;
    gd.b_tiles = (D + 255) / 256;
    gd.out_gstride = 1ll * D * Ha;
    MOE_CUDA(launch_gemm_swap(gd, s));
    SwapLaunch ge = bwd_swap(EPI_STORE_F32, kSwWgrad, xpp, P, dhb, P, 0, M, offp, nullptr, P, D, g->dw1, D,
                             status);
    ge.b_cols = n1;
    ge.b_tiles = (n1 + 255) / 256;
    ge.out_gstride = 1ll * n1 * D;
    MOE_CUDA(launch_gemm_swap(ge, s));
    MOE_CUDA(launch_zero_empty_groups(counts, M, 1ll * D * Ha, g->dw2, s));
    MOE_CUDA(launch_zero_empty_groups(counts, M, 1ll * n1 * D, g->dw1, s));
    MOE_CUDA(launch_dw_finish(parts, nparts, slotp, idx, dy, biases ? w->b2 : nullptr, D, M, T, k, dwp, s));
    if (biases) {
      MOE_CUDA(launch_colsum_bf16(dypp, D, rwp, offp, M, P, D, g->db2, s));
      MOE_CUDA(launch_colsum_bf16(dhb, n1, nullptr, offp, M, P, Ha, g->db1, s));
    }
  }
  if (Is > 0) {
    Range r("moe.shared_expert_backward");
    void* hsb = at<void*>(ws, L.hsb);
    void* asb = at<void*>(ws, L.asb);
    void* dhsb = at<void*>(ws, L.dhsb);
    SwapLaunch sa = bwd_swap(EPI_BWD_SWIGLU_SAVE, kSwFwd, w->sh_w1, 2ll * Is, x, T, D, 1, nullptr, nullptr, T, Is,
                             hsb, 2 * Is, status);
    sa.w_rows_per_group = 2 * Is;
    sa.w_tiles = (Is + 127) / 128;
    sa.w_tile_step = 128;
    sa.w_hi_offset = Is;
    sa.w_cta_step = 64;
    sa.cols_per_tile = 128;
    sa.half_cols = Is;
    sa.out2 = asb;
    sa.ldo2 = Is;
    MOE_CUDA(launch_gemm_swap(sa, s));
    SwapLaunch sb = bwd_swap(EPI_BWD_SWIGLU_DACT, kSwDgrad, w->sh_w2, D, dy, T, D, 1, nullptr, nullptr, T, Is, dhsb,
                             2 * Is, status);
    sb.k_rows_per_group = D;
    sb.aux = hsb;
    sb.ld_aux = 2 * Is;
    sb.half_cols = Is;
    MOE_CUDA(launch_gemm_swap(sb, s));
    SwapLaunch sc = bwd_swap(EPI_STORE_F32, kSwDgrad, w->sh_w1, 2ll * Is, dhsb, T, 2 * Is, 1, nullptr, nullptr, T,
                             D, dxs, D, status);
    sc.k_rows_per_group = 2 * Is;
    MOE_CUDA(launch_gemm_swap(sc, s));
    SwapLaunch sd = bwd_swap(EPI_STORE_F32, kSwWgrad, asb, T, dy, T, 0, 1, nullptr, nullptr, T, Is, g->dsh_w2, Is,
                             status);
    sd.b_cols = D;
    sd.b_tiles = (D + 255) / 256;
    MOE_CUDA(launch_gemm_swap(sd, s));
    SwapLaunch se = bwd_swap(EPI_STORE_F32, kSwWgrad, x, T, dhsb, T, 0, 1, nullptr, nullptr, T, D, g->dsh_w1, D,
                             status);
    se.b_cols = 2 * Is;
    se.b_tiles = (2 * Is + 255) / 256;
    MOE_CUDA(launch_gemm_swap(se, s));
  }
  {
    Range r("moe.router_backward");
    const bool tc = router_bwd_tc(d);
    void* dlb = tc ? at<void*>(ws, L.dlb) : nullptr;
    MOE_CUDA(launch_bwd_router(logits, idx, dwp, T, M, k, d->gate, d->norm_topk_prob, d->routed_scaling_factor,
                               d->eps, dl, dlb, s));
    if (tc) {
      // dW_r [D, M] = x^T dlogits: the weight-gradient layout over one group of T rows,
      // dlogits (bf16) on the A side so that its M columns are the output's contiguous ones
      SwapLaunch gw = bwd_swap(EPI_STORE_F32, kSwWgrad, dlb, T, x, T, 0, 1, nullptr, nullptr, T, M, g->dw_r, M,
                               status);
      gw.b_cols = D;
      gw.b_tiles = (D + 255) / 256;
      gw.out_gstride = 1ll * D * M;
      MOE_CUDA(launch_gemm_swap(gw, s));
      // dx += dlogits W_r^T: the forward layout, W_r [D, M] as K-major weight rows (K = M),
      // added onto the shared expert's dx when there is one
      SwapLaunch gx = bwd_swap(Is > 0 ? EPI_ACCUM_F32 : EPI_STORE_F32, kSwFwd, w->w_r, D, dlb, T, M, 1, nullptr,
                               nullptr, T, D, dxs, D, status);
      MOE_CUDA(launch_gemm_swap(gx, s));
    } else {
      BwdGemmLaunch wr = bwd_gemm(x, 1, D, true, dl, 1, M, 0, false, g->dw_r, M, D, T, M);
      wr.mode = 1;
      wr.ksplit = router_ksplit(T);
      wr.partial = at<float*>(ws, L.rpart);
      MOE_CUDA(launch_bwd_gemm(wr, s));
      BwdGemmLaunch xr = bwd_gemm(dl, M, 1, false, w->w_r, M, 1, 0, true, dxs, D, T, M, D);
      xr.accumulate = Is > 0 ? 1 : 0;  // onto the shared expert's dx
      MOE_CUDA(launch_bwd_gemm(xr, s));
    }
  }
  {
    Range r("moe.combine_backward");
    MOE_CUDA(launch_combine(d->dtype, dxpp, slotp, dxs, true, nullptr, g->dx, T, D, k, s));
  }
  (void)row_token;
  (void)row_w;
  (void)pairs;
  return MOE_OK;
}

moe_status_t backward_impl(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x, const void* dy,
                           const moe_grads_t* g, void* ws, size_t ws_bytes, cudaStream_t s) {
  MOE_TRY(check_desc(d));
  MOE_TRY(check_weights(d, w, true, true));
  if (w->w_r == nullptr || g == nullptr) return MOE_ERR_INVALID_ARG;
  const bool swiglu = d->act == MOE_ACT_SWIGLU;
  const bool biases = !swiglu && d->has_bias;
  if (!g->dw_r || !g->dw1 || !g->dw2) return MOE_ERR_INVALID_ARG;
  if (biases && (!g->db1 || !g->db2)) return MOE_ERR_INVALID_ARG;
  if (d->I_sh > 0 && (!g->dsh_w1 || !g->dsh_w2)) return MOE_ERR_INVALID_ARG;
  if (d->T == 0) {
    MOE_TRY(check_device());
    return zero_param_grads(d, g, s);
  }
  if (!x || !dy || !g->dx || !ws || !aligned_ws(ws)) return MOE_ERR_INVALID_ARG;
  if (d->dtype == MOE_DTYPE_BF16) {
    if (!al16(x) || !al16(dy) || !al16(w->w_r) || !al16(g->dw1) || !al16(g->dw2)) return MOE_ERR_INVALID_ARG;
    if (d->I_sh > 0 && (!al16(g->dsh_w1) || !al16(g->dsh_w2))) return MOE_ERR_INVALID_ARG;
  }
  const BwdWs L = backward_layout(d);
  if (ws_bytes < L.total) return MOE_ERR_INVALID_ARG;
  MOE_TRY(check_device());
  if (d->dtype == MOE_DTYPE_BF16) return backward_tc_impl(d, w, x, dy, g, ws, s);
  const bool bf = d->dtype == MOE_DTYPE_BF16;
  const int T = d->T, D = d->D, M = d->M, k = d->k, Ha = d->I, Is = d->I_sh;
  const int n1 = swiglu ? 2 * d->I : d->I;
  const long long pairs = static_cast<long long>(T) * k;
  int* status = at<int*>(ws, L.f.pub.status);
  int32_t* idx = at<int32_t*>(ws, L.f.pub.topk_idx);
  float* tw = at<float*>(ws, L.f.pub.topk_w);
  int32_t* counts = at<int32_t*>(ws, L.f.pub.counts);
  int32_t* offsets = at<int32_t*>(ws, L.f.pub.offsets);
  int32_t* slot_of = at<int32_t*>(ws, L.f.pub.slot_of);
  int32_t* row_token = at<int32_t*>(ws, L.f.pub.row_token);
  float* row_w = at<float*>(ws, L.f.pub.row_w);
  float* logits = at<float*>(ws, L.f.logits);
  float* o = at<float*>(ws, L.f.pub.out_perm);
  void* xp = at<void*>(ws, L.xp);
  float* hpre = at<float*>(ws, L.hpre);
  float* act = at<float*>(ws, L.act);
  float* dO = at<float*>(ws, L.dO);
  float* da = at<float*>(ws, L.da);
  float* dxp = at<float*>(ws, L.dxp);
  float* dwp = at<float*>(ws, L.dwp);
  float* dl = at<float*>(ws, L.dl);
  float* dxs = at<float*>(ws, L.dxs);
  const int32_t* n_rows = offsets + M;  // pairs dispatched
  Range whole("moe_backward");
  MOE_CUDA(cudaMemsetAsync(status, 0, sizeof(int), s));
  {
    Range r("moe.route");
    MOE_TRY(run_route(x, w->w_r, w->e_bias, T, D, M, k, d->dtype, d->gate, d->norm_topk_prob,
                      d->routed_scaling_factor, d->eps, d->n_group, d->topk_group, idx, tw, logits,
                      at<void*>(ws, L.f.wrT), status, s));
  }
  {
    Range r("moe.dispatch");
    MOE_CUDA(launch_permute(idx, tw, T, k, M, counts, offsets, slot_of, row_token, row_w,
                            at<int32_t*>(ws, L.f.chunk_counts), at<int32_t*>(ws, L.f.chunk_base), status, s));
    MOE_CUDA(launch_gather_rows(x, row_token, n_rows, xp, static_cast<int>(pairs), T, D,
                                static_cast<int>(esize(d->dtype)), status, s));
  }
  {
    Range r("moe.experts_backward");
    // forward values: h = x W1^T (+ b1), a = act(h), o = a W2^T (+ b2), per expert segment
    BwdGemmLaunch g1 = bwd_gemm(xp, D, 1, bf, w->w1, D, 1, 1ll * n1 * D, bf, hpre, n1, pairs, D, n1);
    g1.offsets = offsets; g1.G = M;
    g1.bias = biases ? w->b1 : nullptr; g1.bias_gstride = Ha;
    MOE_CUDA(launch_bwd_gemm(g1, s));
    MOE_CUDA(launch_bwd_act(hpre, act, n_rows, pairs, Ha, swiglu, s));
    BwdGemmLaunch g2 = bwd_gemm(act, Ha, 1, false, w->w2, Ha, 1, 1ll * D * Ha, bf, o, D, pairs, Ha, D);
    g2.offsets = offsets; g2.G = M;
    g2.bias = biases ? w->b2 : nullptr; g2.bias_gstride = D;
    MOE_CUDA(launch_bwd_gemm(g2, s));
    // dw of every pair and dO = w dy at its row
    MOE_CUDA(launch_bwd_pairs(d->dtype, dy, o, slot_of, tw, dwp, dO, T, k, D, pairs, s));
    // da = dO W2, dh = da * act'(h) (in place over h), dx rows = dh W1
    BwdGemmLaunch g3 = bwd_gemm(dO, D, 1, false, w->w2, 1, Ha, 1ll * D * Ha, bf, da, Ha, pairs, D, Ha);
    g3.offsets = offsets; g3.G = M;
    MOE_CUDA(launch_bwd_gemm(g3, s));
    MOE_CUDA(launch_bwd_act_grad(da, hpre, n_rows, pairs, Ha, swiglu, s));
    BwdGemmLaunch g4 = bwd_gemm(hpre, n1, 1, false, w->w1, 1, D, 1ll * n1 * D, bf, dxp, D, pairs, n1, D);
    g4.offsets = offsets; g4.G = M;
    MOE_CUDA(launch_bwd_gemm(g4, s));
    // weight gradients: sums over each expert's rows (the contraction split by expert)
    BwdGemmLaunch g5 = bwd_gemm(dO, 1, D, false, act, 1, Ha, 0, false, g->dw2, Ha, D, pairs, Ha);
    g5.mode = 1; g5.offsets = offsets; g5.G = M; g5.c_gstride = 1ll * D * Ha;
    MOE_CUDA(launch_bwd_gemm(g5, s));
    BwdGemmLaunch g6 = bwd_gemm(hpre, 1, n1, false, xp, 1, D, 0, bf, g->dw1, D, n1, pairs, D);
    g6.mode = 1; g6.offsets = offsets; g6.G = M; g6.c_gstride = 1ll * n1 * D;
    MOE_CUDA(launch_bwd_gemm(g6, s));
    if (biases) {
      MOE_CUDA(launch_bwd_colsum(dO, D, offsets, M, pairs, D, g->db2, s));
      MOE_CUDA(launch_bwd_colsum(hpre, n1, offsets, M, pairs, Ha, g->db1, s));
    }
  }
  if (Is > 0) {
    Range r("moe.shared_expert_backward");
    float* hs = at<float*>(ws, L.hs);
    float* as = at<float*>(ws, L.as);
    float* das = at<float*>(ws, L.das);
    MOE_CUDA(launch_bwd_gemm(bwd_gemm(x, D, 1, bf, w->sh_w1, D, 1, 0, bf, hs, 2 * Is, T, D, 2 * Is), s));
    MOE_CUDA(launch_bwd_act(hs, as, nullptr, T, Is, true, s));
    MOE_CUDA(launch_bwd_gemm(bwd_gemm(dy, D, 1, bf, w->sh_w2, 1, Is, 0, bf, das, Is, T, D, Is), s));
    MOE_CUDA(launch_bwd_act_grad(das, hs, nullptr, T, Is, true, s));
    MOE_CUDA(launch_bwd_gemm(bwd_gemm(hs, 2 * Is, 1, false, w->sh_w1, 1, D, 0, bf, dxs, D, T, 2 * Is, D), s));
    BwdGemmLaunch w2g = bwd_gemm(dy, 1, D, bf, as, 1, Is, 0, false, g->dsh_w2, Is, D, T, Is);
    w2g.mode = 1;
    MOE_CUDA(launch_bwd_gemm(w2g, s));
    BwdGemmLaunch w1g = bwd_gemm(hs, 1, 2 * Is, false, x, 1, D, 0, bf, g->dsh_w1, D, 2 * Is, T, D);
    w1g.mode = 1;
    MOE_CUDA(launch_bwd_gemm(w1g, s));
  }
  {
    Range r("moe.router_backward");
    MOE_CUDA(launch_bwd_router(logits, idx, dwp, T, M, k, d->gate, d->norm_topk_prob, d->routed_scaling_factor,
                               d->eps, dl, nullptr, s));
    BwdGemmLaunch wr = bwd_gemm(x, 1, D, bf, dl, 1, M, 0, false, g->dw_r, M, D, T, M);
    wr.mode = 1;
    MOE_CUDA(launch_bwd_gemm(wr, s));
    BwdGemmLaunch xr = bwd_gemm(dl, M, 1, false, w->w_r, M, 1, 0, bf, dxs, D, T, M, D);
    xr.accumulate = Is > 0 ? 1 : 0;  // onto the shared expert's dx
    MOE_CUDA(launch_bwd_gemm(xr, s));
  }
  {
    Range r("moe.combine_backward");
    MOE_CUDA(launch_combine(d->dtype, dxp, slot_of, dxs, true, nullptr, g->dx, T, D, k, s));
  }
  return MOE_OK;
}

}  // namespace

extern "C" {

size_t moe_backward_workspace_size(const moe_layer_desc_t* d) {
  if (check_desc(d) != MOE_OK) return 0;
  return backward_layout(d).total;
}

moe_status_t moe_backward(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x, const void* dy,
                          const moe_grads_t* grads, void* ws, size_t ws_bytes, void* stream) {
  return backward_impl(d, w, x, dy, grads, ws, ws_bytes, static_cast<cudaStream_t>(stream));
}

int moe_backward_launch_count(const moe_layer_desc_t* d) {
  if (check_desc(d) != MOE_OK || d->T == 0) return 0;
  if (d->dtype == MOE_DTYPE_BF16) {
    int n = 3;  // transpose + logits GEMM or split-K logits + reduction; top-k
    n += static_cast<long long>(d->T) * d->k <= 2048 ? 1 : 3;                    // counting sort
    n += 2 + 2 + 2;        // padded order (offsets, pairs), two gathers, two padding zero-fills
    n += 5 + 2 + 1;        // five expert GEMMs, empty-expert zero-fills, gate-weight gradients
    if (d->act == MOE_ACT_GELU_TANH && d->has_bias) n += 2;        // bias gradients
    if (d->I_sh > 0) n += 5;                                         // shared expert GEMMs
    n += 3;                                                          // router backward, dW_r, router dx
    if (!router_bwd_tc(d) && router_ksplit(d->T) > 1) n += 1;        // dW_r chunk sums
    n += 1;                                                          // dx combine
    return n;
  }
  int n = d->dtype == MOE_DTYPE_BF16 ? 3 : 2;                        // router logits + top-k
  n += static_cast<long long>(d->T) * d->k <= 2048 ? 1 : 3;          // counting sort
  n += 1;                                                            // gather
  n += 9;                                                            // 6 expert GEMMs, act, pairs, act grad
  if (d->act == MOE_ACT_GELU_TANH && d->has_bias) n += 2;            // bias gradients
  if (d->I_sh > 0) n += 7;                                           // shared expert
  n += 3;                                                            // router backward, dW_r, router dx
  n += 1;                                                            // dx combine
  return n;
}

}  // extern "C"
