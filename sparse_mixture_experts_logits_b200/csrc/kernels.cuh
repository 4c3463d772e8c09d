// Host-side launchers of the library's kernels (internal interface between
// the C ABI in moe_api.cu and the kernel files).
#pragma once

#include "common.cuh"

namespace moe {

// router.cu
cudaError_t launch_transpose_bf16(const void* src, void* dst, int rows, int cols, cudaStream_t s);
cudaError_t launch_logits_f32(const float* x, const float* w_r, float* logits, int T, int D, int M,
                              cudaStream_t s);
// Small-T bf16 router: route_splits(T, D, dtype) partial logit sums
// [nsplit][T][M] (written to `partial`), added in order into `logits`.
int route_splits(int T, int D, int dtype);
cudaError_t launch_logits_splitk_bf16(const void* x, const void* w_r, float* partial, float* logits, int T,
                                      int D, int M, cudaStream_t s);
// n_group <= 1: no group limit (otherwise the caller checked M % n_group == 0,
// n_group <= 32, 1 <= topk_group <= n_group and k <= topk_group * M / n_group).
cudaError_t launch_topk(const float* logits, const float* e_bias, int T, int M, int k, int gate,
                        int norm, float alpha, float eps, int n_group, int topk_group, int32_t* idx,
                        float* w, cudaStream_t s);

// permute.cu
constexpr int kPermChunk = 512;  // (slot, token) pairs per chunk of the counting sort
inline int perm_num_chunks(long long pairs) {
  return static_cast<int>((pairs + kPermChunk - 1) / kPermChunk);
}
cudaError_t launch_permute(const int32_t* topk_idx, const float* topk_w, int T, int k, int M,
                           int32_t* counts, int32_t* offsets, int32_t* slot_of, int32_t* row_token,
                           float* row_w, int32_t* chunk_counts, int32_t* chunk_base, int* status,
                           cudaStream_t s);

// capacity.cu: idx[p] := M where slot_of[p] - offsets[idx[p]] >= capacity (in place).
cudaError_t launch_capacity_drop(int32_t* idx, const int32_t* slot_of, const int32_t* offsets, int T, int k, int M,
                                 int capacity, cudaStream_t s);

// misc.cu
// bf16 rows of x into dispatch order by token: x_perm[slot_of[t, j]] = x[t] (D % 8 == 0).
cudaError_t launch_scatter_rows(const void* x, const int32_t* slot_of, void* x_perm, int T, int k, int D,
                                int* status, cudaStream_t s);
// Gathers rows r < min(rows, *n_rows) (n_rows device, may be null).
cudaError_t launch_gather_rows(const void* x, const int32_t* row_token, const int32_t* n_rows, void* x_perm,
                               int rows, int T, int D, int elem_bytes, int* status, cudaStream_t s);
// y = sum of the k routed rows (+ shared_out) (+ addend, layer dtype), in fp32, rounded once.
cudaError_t launch_combine(int dtype, const void* out_perm, const int32_t* slot_of,
                           const void* shared_out, bool shared_f32, const void* addend, void* y, int T,
                           int D, int k, cudaStream_t s);

// gemm_sm100.cu: grouped bf16 GEMM on tcgen05.  `epi` is a GemmEpilogue.
struct GemmLaunch {
  int epi;
  int ncta;  // 1: one CTA per 128-row tile; 2 (default, 0): 2-SM MMA on CTA pairs, 256-row tiles
  const void* A; long long a_rows; // bf16 [a_rows, K]
  const void* B; long long b_rows; // bf16 [b_rows, K]
  int K;
  int num_groups;
  const int* offsets;  // device [G+1] or nullptr (single group of a_rows rows)
  long long rows_upper;  // host upper bound of the rows covered by the segments
  int bn, n_tiles, b_rows_per_group, b_row_step, b_hi_offset;
  int out_cols, out_col_step, ldo;
  void* out;
  const float* row_scale;
  const void* bias;
  int* status;
};
cudaError_t launch_gemm_sm100(const GemmLaunch& L, cudaStream_t s);
int num_sms();
// MOE_OK when the current device is compute capability 10.0 (the only
// target of this library's sm_100a code), MOE_ERR_UNSUPPORTED otherwise.
moe_status_t check_device();

// gemm_swap_sm100.cu: grouped bf16 GEMM with the token rows on the MMA's N
// side (see gemm_swap_sm100.cuh).  `epi` is a GemmEpilogue.
struct SwapLaunch {
  int epi;
  int layout;                       // kSwFwd (0), kSwDgrad (1) or kSwWgrad (2) of gemm_swap_sm100.cuh
  const void* W; long long w_rows;  // bf16 [w_rows, K] weight stack (kSwFwd), [w_rows, a_cols] otherwise
  const void* X; long long x_rows;  // bf16 [x_rows, K] token rows in dispatch order ([x_rows, b_cols]: kSwWgrad)
  int K;
  int num_groups;
  const int* offsets;        // device [G+1] or nullptr (single group of `rows` rows)
  long long rows;            // dispatch rows (upper bound when grouped)
  int w_rows_per_group, w_tiles, w_tile_step, w_hi_offset, w_cta_step, cols_per_tile;
  int out_cols, ldo;
  void* out;
  const float* row_scale;
  const void* bias;
  const void* addend;        // EPI_BIAS_ADD: bf16 [rows, ldo] or nullptr
  int* status;
  // backward layouts and epilogues (see SwapArgs)
  int a_cols;                // columns of the MN-major A matrix
  int k_rows_per_group;      // kSwDgrad
  int b_tiles, b_cols;       // kSwWgrad
  long long out_gstride;     // kSwWgrad
  void* out2; void* out3; int ldo2;
  const void* aux; int ld_aux;
  float* parts; int ld_parts;
  int half_cols;
  const int* counts;         // optional [G]: rows computed per group (segments start at offsets)
  int* tile_ctr;             // optional: 0 at launch; with many narrow groups, tiles are claimed
                             // from it as CTA pairs free up
};
cudaError_t launch_gemm_swap(const SwapLaunch& L, cudaStream_t s);

// simt.cu: fp32 grouped GEMM with the same epilogues (fp32 dtype path).
struct SimtLaunch {
  int epi;
  const float* A; const int32_t* a_row_index; int K; // A row of output row r: a_row_index[r] or r
  const float* B;                                     // [G * b_rows_per_group, K]
  int num_groups;
  const int* offsets;  // device [G+1] or nullptr
  long long rows;      // rows when offsets == nullptr; upper bound otherwise
  int b_rows_per_group;
  int swiglu_hi;       // SwiGLU: row offset of the up half (I); 0 otherwise
  int out_cols, ldo;
  float* out;
  const float* row_scale;
  const float* bias;
  const float* addend;  // EPI_BIAS_ADD: [rows, ldo] or nullptr
};
cudaError_t launch_simt_gemm(const SimtLaunch& L, cudaStream_t s);

// bwd_tc.cu: helpers of the tensor-core backward (bf16 layers), which keeps
// its per-row tensors in a dispatch order padded per expert to 64 rows.
cudaError_t launch_pad_dispatch(const int32_t* idx, const int32_t* slot_of, const float* topk_w,
                                const int32_t* counts, const int32_t* offsets, int T, int k, int M,
                                long long rows_cap, int32_t* offsets_pad, int32_t* slot_pad,
                                int32_t* row_token_pad, float* row_w_pad, cudaStream_t s);
cudaError_t launch_gather_pad(const void* src, const int32_t* row_token_pad, const int32_t* n_rows, void* dst,
                              long long rows_cap, int T, int D, cudaStream_t s);
cudaError_t launch_zero_pad_rows(const int32_t* counts, const int32_t* offsets_pad, int M, void* buf,
                                 long long rows_cap, int cols_bf16, cudaStream_t s);
cudaError_t launch_dw_finish(const float* parts, int nparts, const int32_t* slot_pad, const int32_t* idx,
                             const void* dy, const void* b2, int D, int M, int T, int k, float* dw, cudaStream_t s);
cudaError_t launch_colsum_bf16(const void* Y, long long ldy, const float* scale, const int32_t* offsets, int G,
                               long long rows_cap, int N, float* out, cudaStream_t s);
cudaError_t launch_zero_empty_groups(const int32_t* counts, int G, long long per_group, float* out, cudaStream_t s);

// backward.cu: C (+)= A B^T on the CUDA cores, fp32 sums, with strided
// operands: A(m, k) = A[m * a_sm + k * a_sk], B(n, k) = B[g * b_gstride +
// n * b_sn + k * b_sk], C(m, n) = C[g * c_gstride + m * ldc + n] (+ bias[g *
// bias_gstride + n], bias of B's type).  Groups g come from offsets [G+1]:
// mode 0 splits the rows m (absolute row indices, c_gstride unused), mode 1
// splits the contraction k (absolute k indices; rows = M extent); without
// offsets there is one group over [0, rows) or [0, K).  An empty group of
// mode 1 writes zeros.
struct BwdGemmLaunch {
  const void* A; long long a_sm, a_sk; bool a_bf16;
  const void* B; long long b_sn, b_sk, b_gstride; bool b_bf16;
  const void* bias; long long bias_gstride;
  float* C; long long ldc, c_gstride;
  int mode;
  const int32_t* offsets;
  int G;
  long long rows, K;
  int N;
  int accumulate;
  // mode 1 without groups: split the contraction into ksplit chunks whose
  // partial sums ([ksplit, rows, N] in `partial`) are added in order (ldc == N)
  int ksplit;
  float* partial;
};
cudaError_t launch_bwd_gemm(const BwdGemmLaunch& L, cudaStream_t s);
// a = GELU(h) or SiLU(gate) * up for rows < min(rows, *n_rows) (n_rows may be null).
cudaError_t launch_bwd_act(const float* h, float* a, const int32_t* n_rows, long long rows, int Ha, bool swiglu,
                           cudaStream_t s);
// h := dL/dh from da = dL/da, in place.
cudaError_t launch_bwd_act_grad(const float* da, float* h, const int32_t* n_rows, long long rows, int Ha,
                                bool swiglu, cudaStream_t s);
// dw[t, j] = <dy_t, o[slot]>, dO[slot] = topk_w[t, j] dy_t.
cudaError_t launch_bwd_pairs(int dtype, const void* dy, const float* o, const int32_t* slot_of,
                             const float* topk_w, float* dw, float* dO, int T, int k, int D, long long rows_cap,
                             cudaStream_t s);
// out[g, :] = column sums of Y over the rows of group g.
cudaError_t launch_bwd_colsum(const float* Y, long long ldy, const int32_t* offsets, int G, long long rows_cap,
                              int N, float* out, cudaStream_t s);
// dL/dlogits [T, M] from dL/dw [T, k] (fp32), and a bf16 copy when dl_bf is
// not null (the operand of the router's tensor-core backward GEMMs).
cudaError_t launch_bwd_router(const float* logits, const int32_t* idx, const float* dw, int T, int M, int k,
                              int gate, int norm, float alpha, float eps, float* dl, void* dl_bf,
                              cudaStream_t s);

}  // namespace moe
