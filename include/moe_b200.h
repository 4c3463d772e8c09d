/*
 * moe_b200.h - C ABI of the sparse Mixture-of-Experts FFN layer forward on
 * NVIDIA B200 (sm_100a).
 *
 * The layer (sources: the "GLaM" architecture note, section "Sparse MoE
 * Layer"; the GLM-4.5 "Shared Expert" study note, section "How it works";
 * the "GLM-5 - Shared expert" page of OpenModelAtlas, its quoted
 * GlmMoeDsaMoE / GlmMoeDsaExperts / GlmMoeDsaMLP forward excerpts):
 *
 *   route     s[t,e] = sum_d x[t,d] W_r[d,e]                     (fp32)
 *             softmax gate: S_t = TopK(s_t, k); w = renormalised softmax
 *             sigmoid gate: g = sigmoid(s); S_t = TopK(g + e_bias, k);
 *                           w = alpha * g / (sum_S g + eps)
 *   dispatch  pairs (t, j) grouped by expert, inside an expert by (j, t)
 *   experts   GELU:   E(x) = W2 GELU_tanh(W1 x + b1) + b2
 *             SwiGLU: E(x) = W_down(SiLU(W_gate x) * W_up x)
 *   combine   y_t = sum_j w[t,j] E_{idx[t,j]}(x_t)  (+ E_sh(x_t))
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - All tensors are dense row-major.  Weights use the nn.Linear [out, in]
 *    layout, except W_r, which is [D, M].
 *  - Every pointer argument is a DEVICE pointer to caller-owned memory on
 *    the current device, except the descriptor and weight structs, which are
 *    host structs (the pointers inside them are device pointers).  The
 *    library never allocates memory, frees or synchronises; every call only
 *    enqueues kernels on `stream` (a cudaStream_t; NULL = legacy default
 *    stream) and returns.  The one exception to "only on `stream`" is
 *    moe_forward's decode-size shared expert (below): it may run on an
 *    internal stream that waits for `stream` and that `stream` waits for
 *    before the combine, so the call's ordering is the same.
 *  - Scratch memory ("workspace") is caller-provided; each entry point has a
 *    *_workspace_size query.  Workspaces must be 256-byte aligned.  Calls
 *    that share a workspace must be ordered on one stream.
 *  - dtype MOE_DTYPE_BF16: x, W_r, expert/shared weights, biases, y are
 *    bf16; all accumulation is fp32.  MOE_DTYPE_F32: all of them are fp32.
 *    e_bias, topk_w and row_w are always fp32; indices are int32.
 *  - MOE_DTYPE_BF16 tensors that the tensor-core kernels move with TMA start
 *    on a 16-byte boundary: x, W_r, the routed and shared weight stacks, and
 *    in moe_backward also dy and the fp32 weight gradients dw1, dw2, dsh_w1,
 *    dsh_w2 (cudaMalloc and PyTorch allocations are).  A misaligned one is
 *    MOE_ERR_INVALID_ARG, found before anything is launched.
 *  - Errors: every call validates its arguments on the host and returns a
 *    status without launching anything when they are invalid.  Device-side
 *    faults are never raised: kernels that find an out-of-range expert index
 *    or whose bounded waits time out set a flag in the workspace, read back
 *    with moe_device_status().
 *  - T = 0 is valid and launches nothing.
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, k > M, workspace too small */
  MOE_ERR_UNSUPPORTED = 2, /* shape/dtype outside what the kernels implement */
  MOE_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
  MOE_ERR_DEVICE = 4       /* a kernel reported an error through the workspace flag */
} moe_status_t;

typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype_t;

/* Router kinds.  SOFTMAX: "GLaM" eq. r_t and S_t.  SIGMOID_BIAS: the GLM-4.5
 * note's sigmoid scores plus loss-free correction bias. */
typedef enum { MOE_GATE_SOFTMAX = 0, MOE_GATE_SIGMOID_BIAS = 1 } moe_gate_t;

/* Expert kinds.  GELU_TANH: "GLaM" eq. FFN with sigma = GELU (tanh form).
 * SWIGLU: W_down(SiLU(W_gate x) * W_up x). */
typedef enum { MOE_ACT_GELU_TANH = 0, MOE_ACT_SWIGLU = 1 } moe_act_t;

/* Device-side error codes written to the workspace flag. */
#define MOE_DEVERR_NONE 0
#define MOE_DEVERR_BAD_EXPERT_INDEX 1 /* topk_idx entry outside [0, M] (M: the sentinel) */
#define MOE_DEVERR_TIMEOUT 2          /* a bounded wait inside a kernel gave up */
#define MOE_DEVERR_BAD_ROW_TOKEN 3    /* row_token entry outside [0, T) (row zero-filled) */
#define MOE_DEVERR_BAD_COUNT 4        /* an exchanged row count outside [0, cap] (clamped) */

/* One MoE layer's shape and options (HF config names in brackets). */
typedef struct {
  int dtype;                   /* moe_dtype_t */
  int T;                       /* tokens (batch x sequence flattened) */
  int D;                       /* model width [hidden_size] */
  int M;                       /* routed experts [n_routed_experts] */
  int k;                       /* experts per token [num_experts_per_tok] */
  int gate;                    /* moe_gate_t */
  int act;                     /* moe_act_t */
  int I;                       /* expert hidden width [moe_intermediate_size] */
  int has_bias;                /* GELU experts: b1, b2 present */
  int norm_topk_prob;          /* renormalise the k selected gate values */
  float routed_scaling_factor; /* alpha, multiplies every routed weight */
  float eps;                   /* sigmoid renormalisation epsilon (1e-20) */
  int I_sh;                    /* shared expert width, 0 = no shared expert
                                  [moe_intermediate_size * n_shared_experts] */
  int n_group;                 /* expert groups of the group-limited selection
                                  (0 or 1 = no group limit) [n_group] */
  int topk_group;              /* groups kept per token [topk_group] */
} moe_layer_desc_t;

/* Device pointers to one layer's weights.  Unused fields may be NULL. */
typedef struct {
  const void* w_r;     /* [D, M] router weight */
  const float* e_bias; /* [M] correction bias (SIGMOID_BIAS; NULL = zeros) */
  const void* w1;      /* GELU: [M, I, D] W1.  SWIGLU: [M, 2I, D] fused
                          gate_up stack, rows 0..I-1 gate, I..2I-1 up */
  const void* b1;      /* GELU with bias: [M, I] */
  const void* w2;      /* [M, D, I] W2 / down projection */
  const void* b2;      /* GELU with bias: [M, D] */
  const void* sh_w1;   /* [2 I_sh, D] shared gate_up (gate rows first) */
  const void* sh_w2;   /* [D, I_sh] shared down projection */
} moe_weights_t;

/* Byte offsets, inside a moe_forward workspace, of the intermediates the
 * forward pass leaves there (valid after the stream reaches the end of a
 * moe_forward call).  Exposed so that tests can check every stage. */
typedef struct {
  size_t status;    /* int32 device status flag; the 256-byte slot it starts
                       also holds, as int32 words 2 and 3, the routed expert
                       GEMMs' tile counters (zeroed by each moe_forward) */
  size_t topk_idx;  /* int32 [T, k] */
  size_t topk_w;    /* fp32  [T, k] */
  size_t counts;    /* int32 [M] */
  size_t offsets;   /* int32 [M + 1] */
  size_t slot_of;   /* int32 [T, k] */
  size_t row_token; /* int32 [T k] */
  size_t row_w;     /* fp32  [T k] */
  size_t out_perm;  /* fp32  [T k, D] weighted expert outputs, dispatch order */
  size_t total;     /* bytes needed */
} moe_ws_layout_t;

/* ------------------------------------------------------------------------ */

/* Status string ("MOE_OK", ...); never NULL. */
const char* moe_status_string(moe_status_t s);

/* Library version string. */
const char* moe_version(void);

/* Reads the device status flag at the start of workspace `ws` (any entry
 * point's workspace) into *out (MOE_DEVERR_*) and clears it.  This call
 * synchronises `stream`.  Returns MOE_ERR_CUDA if the copy fails. */
moe_status_t moe_device_status(void* ws, void* stream, int* out);

/* ---- router: "GLaM" eq. r_t, S_t and MoE; GLM-4.5 note eq. g-bar ------- */

size_t moe_route_workspace_size(int T, int D, int M, int dtype);

/* Router scores, top-k and gate weights for T tokens.
 *   x [T, D], w_r [D, M] (dtype), e_bias [M] fp32 or NULL.
 *   Outputs topk_idx [T, k] int32 (slot j = j-th largest selection score,
 *   exact ties to the lower expert index) and topk_w [T, k] fp32.
 *   SOFTMAX: selection on the logits; w = alpha * softmax renormalised over
 *   the k selected (norm_topk_prob) or the full softmax probability.
 *   SIGMOID_BIAS: selection on sigmoid(s) + e_bias; w = alpha * g /
 *   (sum_S g + eps) (norm_topk_prob) or alpha * g; the bias never enters w.
 *   Group limit (the GLM-4.5 note: the router "optionally masks by expert
 *   group"), on when n_group > 1: experts [i M/n_group, (i+1) M/n_group)
 *   form group i, scored by the sum of its two largest selection scores; the
 *   topk_group best groups (lower index on ties) stay eligible and the top-k
 *   is taken over their experts only.  Needs M % n_group == 0,
 *   n_group <= 32, 1 <= topk_group <= n_group, k <= topk_group M / n_group.
 * Limits: 1 <= k <= min(M, 32), M <= 1024; bf16 needs D % 16 == 0. */
moe_status_t moe_route_topk(const void* x, const void* w_r, const float* e_bias,
                            int T, int D, int M, int k, int dtype, int gate,
                            int norm_topk_prob, float routed_scaling_factor, float eps,
                            int n_group, int topk_group,
                            int32_t* topk_idx, float* topk_w,
                            void* ws, size_t ws_bytes, void* stream);

/* ---- dispatch: the GLM-5 page's GlmMoeDsaExperts.forward expert mask --- */

size_t moe_permute_workspace_size(int T, int k, int M);

/* Deterministic dispatch order of the T*k (token, slot) pairs: a stable
 * counting sort by expert of the pairs taken in (slot j, token t) order.
 *   counts[M], offsets[M+1] (exclusive prefix sum, offsets[M] = T k),
 *   slot_of[T, k] (dispatch position of pair (t, j)), row_token[T k],
 *   row_w[T k] = topk_w[t, j] of the pair at each position.
 * Bit-exact and independent of scheduling (no atomics decide an order).
 * An entry equal to M is the "no expert" sentinel of the GLM-5 page's
 * GlmMoeDsaExperts.forward (one_hot over M + 1 classes, class M skipped):
 * the pair is dispatched nowhere, slot_of = -1, and it is not counted.  An
 * entry outside [0, M] is skipped the same way and sets
 * MOE_DEVERR_BAD_EXPERT_INDEX. */
moe_status_t moe_permute(const int32_t* topk_idx, const float* topk_w, int T, int k, int M,
                         int32_t* counts, int32_t* offsets, int32_t* slot_of,
                         int32_t* row_token, float* row_w,
                         void* ws, size_t ws_bytes, void* stream);

/* The same dispatch as moe_permute, for callers that cannot allocate device
 * memory where they route tokens (a process whose device memory is owned by
 * a pool, a latency-critical loop that cannot take cudaMalloc's implicit
 * synchronisation, a plug-in host without an allocator).  The source pages
 * have no counterpart for this entry point: it exists for those callers.
 *   Scratch: a 4 MiB array compiled into the library, reserved on every GPU
 *   that loads the library until the process exits.  Supported sizes:
 *   M * ceil(T*k / 512) <= 524288; larger requests return
 *   MOE_ERR_UNSUPPORTED without launching.  No cudaMalloc/cudaFree.
 *   device_status: optional int32 device word, cleared by the call, set to
 *   MOE_DEVERR_BAD_EXPERT_INDEX if topk_idx holds an index outside [0, M]
 *   (M itself is the sentinel, dispatched nowhere).
 *   All calls on a device share the scratch array; calls whose kernels
 *   overlap on the GPU (unordered streams) race and may give wrong results.
 *   The first call on each device (and again after the device's context is
 *   recreated, e.g. by cudaDeviceReset) looks up the array's address with
 *   that device current; make it before any stream capture begins.
 * Other arguments and outputs: as moe_permute (bit-identical results). */
moe_status_t moe_permute_static_scratch(const int32_t* topk_idx, const float* topk_w, int T, int k,
                                        int M, int32_t* counts, int32_t* offsets, int32_t* slot_of,
                                        int32_t* row_token, float* row_w, int32_t* device_status,
                                        void* stream);

/* Expert capacity (the pages give no capacity rule; this is the plain one):
 * an expert takes at most `capacity` pairs, the first ones in moe_permute's
 * dispatch order (slot j, then token t: every first choice before any
 * second choice), and every later pair's index becomes the sentinel M, which
 * the dispatch and the combine skip.  Gate weights are left as they are (a
 * dropped pair adds nothing).  topk_idx [T, k] is rewritten in place;
 * slot_of and offsets are what moe_permute produced for it.  Run
 * moe_permute again afterwards to get the dispatch of the kept pairs.
 * capacity >= 0; 0 < M <= 1024; T = 0 launches nothing. */
moe_status_t moe_capacity_drop(int32_t* topk_idx, const int32_t* slot_of, const int32_t* offsets,
                               int T, int k, int M, int capacity, void* stream);

/* ceil(factor * T * k / M): with factor 1 every expert may take exactly its
 * even share of the T k pairs.  -1 for factor < 0, M < 1, T < 0 or k < 1. */
int moe_expert_capacity(double factor, int T, int k, int M);

/* x_perm[s, :] = x[row_token[s], :] for s < min(rows, *n_rows) (n_rows a
 * device int32, e.g. offsets + M, or NULL for all `rows`): the tokens'
 * rows in dispatch order, contiguous, e.g. to send each expert owner its
 * rows in one piece (expert parallelism).  x and x_perm in dtype; a
 * row_token outside [0, T) gives a zero row and sets MOE_DEVERR_BAD_ROW_TOKEN
 * in *device_status (a device int32, may be NULL). */
moe_status_t moe_gather_rows(const void* x, const int32_t* row_token, const int32_t* n_rows,
                             void* x_perm, int rows, int T, int D, int dtype,
                             int32_t* device_status, void* stream);

/* ---- expert parallelism: fixed-split exchange (GLaM industry article,
 *      first route: cross-node communication between experts) ------------
 * The routed experts split over `world` ranks, rank q owning experts
 * [q E, (q + 1) E), E = M / world.  Every split of the exchange is E * cap
 * rows, whatever the routing, so the all-to-alls between these calls need
 * no row counts on the host and a step runs without a device-to-host read.
 * An expert keeps the first `cap` of its pairs in dispatch order (the rule
 * of moe_capacity_drop); later pairs are dropped (they add nothing to y). */

/* Sender: pack the dispatch order of moe_permute (offsets [M+1],
 * row_token, row_w, slot_of [T, k]) into M blocks of cap rows, block e
 * holding expert e's first min(counts[e], cap) rows and zeros after them:
 *   x_pad [M * cap, D] (dtype), w_pad [M * cap] fp32 (0 on padding rows),
 *   kept [M] int32 = min(counts[e], cap),
 *   slot_pad [T, k] int32 = e * cap + i for the pair at position i of
 *     expert e's segment when i < cap, else -1 (dropped or sentinel).
 * Owner q's rows are x_pad[q E cap, (q + 1) E cap): one piece per rank.
 * x and x_pad in dtype.  A row_token outside [0, T) gives a zero row with
 * weight 0 and sets MOE_DEVERR_BAD_ROW_TOKEN in *device_status (a device
 * int32 cleared by the call, may be NULL).  cap >= 0, M <= 1024. */
moe_status_t moe_ep_pack(const void* x, const int32_t* offsets, const int32_t* row_token,
                         const float* row_w, const int32_t* slot_of, int T, int k, int M, int D,
                         int dtype, int cap, void* x_pad, float* w_pad, int32_t* slot_pad,
                         int32_t* kept, int32_t* device_status, void* stream);

/* Receiver: the blocks arrive as [world][E][cap] (source rank q, local
 * expert e, row i) with recv_kept [world, E] = the senders' kept counts and
 * w_recv [world * E * cap] their w_pad.  Builds the expert-major dispatch
 * order over the arrival rows, for moe_expert_ffn with M = E and k = 1:
 *   offsets [E+1]: expert e's rows from rank 0, then rank 1, ...;
 *   row_token[p], row_w[p] for p < offsets[E]: the arrival row at dispatch
 *     position p and its gate weight;
 *   slot_of [world * E * cap]: the dispatch position of each arrival row,
 *     -1 for padding (moe_combine with k = 1 puts the expert outputs back
 *     into arrival order, padding rows zero).
 * A recv_kept entry outside [0, cap] is clamped and sets
 * MOE_DEVERR_BAD_COUNT.  world * E <= 1024. */
moe_status_t moe_ep_unpack(const int32_t* recv_kept, const float* w_recv, int world, int E, int cap,
                           int32_t* offsets, int32_t* row_token, float* row_w, int32_t* slot_of,
                           int32_t* device_status, void* stream);

/* ---- experts: "GLaM" eq. FFN; GLM-5 GlmMoeDsaExperts.forward ----------- */

size_t moe_expert_ffn_workspace_size(const moe_layer_desc_t* d);

/* Routed experts over the dispatch order:
 *   out_perm[s, :] = row_w[s] * E_e(x[row_token[s], :]) for every position s
 *   in expert e's segment [offsets[e], offsets[e+1]).
 * out_perm is fp32 [T k, D] (the accumulator, unrounded, so that the
 * combine rounds only once).  Only the offsets[M] <= T k dispatched rows
 * are read or written: when pairs were dropped through the sentinel index,
 * row_token and row_w past offsets[M] may hold anything.  A row_token entry
 * outside [0, T) is reported as MOE_DEVERR_BAD_ROW_TOKEN and read as zeros. */
moe_status_t moe_expert_ffn(const moe_layer_desc_t* d, const moe_weights_t* w,
                            const void* x, const int32_t* offsets,
                            const int32_t* row_token, const float* row_w,
                            void* out_perm, void* ws, size_t ws_bytes, void* stream);

/* ---- shared expert: GLM-4.5 note E_sh; GLM-5 GlmMoeDsaMLP.forward ------ */

size_t moe_shared_expert_workspace_size(const moe_layer_desc_t* d);

/* y_sh[T, D] = W_down(SiLU(W_gate x) * W_up x) over the pre-routing x. */
moe_status_t moe_shared_expert(const moe_layer_desc_t* d, const moe_weights_t* w,
                               const void* x, void* y_sh,
                               void* ws, size_t ws_bytes, void* stream);

/* ---- combine: "GLaM" eq. MoE; GLM-4.5 note eq. y ----------------------- */

/* y[t, :] = sum_{j=0}^{k-1} out_perm[slot_of[t, j], :] (+ shared_out[t, :])
 *           (+ addend[t, :]),
 * with slot_of < 0 (sentinel pairs) adding nothing,
 * out_perm fp32 [T k, D], shared_out, addend and y [T, D] in dtype,
 * summed in fp32 in slot order and rounded once.  shared_out and addend may
 * be NULL; addend is the other term of the "GLaM" block sum (see
 * moe_forward_add). */
moe_status_t moe_combine(const moe_layer_desc_t* d, const void* out_perm,
                         const int32_t* slot_of, const void* shared_out,
                         const void* addend, void* y, void* stream);

/* ---- the whole layer --------------------------------------------------- */

size_t moe_workspace_size(const moe_layer_desc_t* d);
moe_status_t moe_workspace_layout(const moe_layer_desc_t* d, moe_ws_layout_t* out);

/* y[T, D] = MoE-FFN(x): route, dispatch, routed experts, shared expert (when
 * I_sh > 0, its output kept in fp32) and the combine, which adds each
 * token's k weighted expert rows and its shared-expert row in fp32 and
 * rounds once.  All stages run back to back on `stream` with no host
 * synchronisation, with one exception: in bf16 with a shared expert and
 * T * k < 4 M (the decode sizes, where each expert gets a handful of rows)
 * the shared expert's two GEMMs read only x, so they run on an internal
 * stream beside the routing stage.  That stream (one per device and CUDA
 * context, with two events, made on the first such call that is not
 * inside a stream capture) waits for `stream` before them, and `stream`
 * waits for it before the combine; a call that returns early still joins
 * it.  Inside a capture the fork and join are captured as graph branches;
 * without the stream (not yet made, or a creation that failed) everything
 * runs on `stream`.  The result is the same either way. */
moe_status_t moe_forward(const moe_layer_desc_t* d, const moe_weights_t* w,
                         const void* x, void* y, void* ws, size_t ws_bytes, void* stream);

/* y[T, D] = addend[T, D] + MoE-FFN(x): the sparse layer of the "GLaM" note,
 * section "Interleaving Dense and Sparse Layers",
 *   h^{l+1} = Attention(h^l) + MoE-FFN(h^l),
 * with addend the other term (the attention output, or the residual
 * stream).  The addend is added in fp32 inside the combine, before the one
 * rounding of y.  addend (dtype) must not be NULL when T > 0 and must not
 * overlap y.  Otherwise as moe_forward. */
moe_status_t moe_forward_add(const moe_layer_desc_t* d, const moe_weights_t* w,
                             const void* x, const void* addend, void* y,
                             void* ws, size_t ws_bytes, void* stream);

/* Stage boundaries recorded by moe_forward_profiled (the "routing overhead"
 * breakdown of the GLaM note's reporting table: gate, dispatch, expert
 * batching, combination cost). */
#define MOE_NUM_STAGE_EVENTS 9
/* event 0: start; 1: route done (scores, top-k, weights); 2: dispatch order
 * done; 3: rows gathered into dispatch order; 4: routed experts' first GEMM
 * done; 5: routed experts' second GEMM done; 6: shared expert's first GEMM
 * done; 7: shared expert's second GEMM done; 8: combine (the k routed rows
 * of every token plus its shared-expert row) done.  Stages a
 * layer does not have record their event right after the previous one.
 * When the shared expert runs beside the routing stage (moe_forward),
 * events 6 and 7 are recorded on `stream` after it joins: stage 6 then
 * holds only the part of the shared expert that the routed stages did not
 * cover, and stage 7 is empty. */

/* moe_forward, recording `events[i]` (cudaEvent_t handles created by the
 * caller, n_events == MOE_NUM_STAGE_EVENTS) on `stream` at each boundary. */
moe_status_t moe_forward_profiled(const moe_layer_desc_t* d, const moe_weights_t* w,
                                  const void* x, void* y, void* ws, size_t ws_bytes, void* stream,
                                  void* const* events, int n_events);

/* Number of kernels one moe_forward call with this descriptor launches. */
int moe_forward_launch_count(const moe_layer_desc_t* d);

/* Algorithmic work of one moe_forward call given the routing counts
 * (host array counts[M], as produced by moe_permute): FLOPs of the router
 * and of the routed and shared experts, and bytes of the weights of the
 * experts that received at least one token plus x and y.  Padding and
 * intermediate buffers are not counted. */
void moe_algorithmic_work(const moe_layer_desc_t* d, const int32_t* counts_host,
                          double* flops, double* bytes);

/* ---- dense FFN layer: "GLaM" section "Interleaving Dense and Sparse
 * Layers" (DenseFFN); GLM-4.5 note: dense prefix layers are one wide SwiGLU -- */

typedef struct {
  int dtype;    /* moe_dtype_t */
  int T;        /* tokens */
  int D;        /* model width [hidden_size] */
  int I;        /* hidden width [intermediate_size] */
  int act;      /* moe_act_t */
  int has_bias; /* GELU: b1, b2 present (ignored for SWIGLU) */
} moe_dense_desc_t;

size_t moe_dense_ffn_workspace_size(const moe_dense_desc_t* d);

/* y[T, D] = (addend[T, D] +) FFN(x), the dense layer of the "GLaM" note,
 * h^{l+1} = Attention(h^l) + DenseFFN(h^l):
 *   GELU_TANH: FFN(x) = W2 GELU(W1 x + b1) + b2 ("GLaM" eq. FFN),
 *              w1 [I, D], b1 [I], w2 [D, I], b2 [D];
 *   SWIGLU:    FFN(x) = W_down(SiLU(W_gate x) * W_up x),
 *              w1 [2I, D] (gate rows first), w2 [D, I].
 * All tensors in dtype, nn.Linear layout; addend may be NULL and must not
 * overlap y.  The hidden
 * activations are kept in the workspace in dtype; the second GEMM adds b2 and
 * the addend in fp32 and rounds y once.  Limits: bf16 needs D % 16 == 0 and
 * I % 16 == 0.  Errors as moe_forward. */
moe_status_t moe_dense_ffn(const moe_dense_desc_t* d, const void* w1, const void* b1,
                           const void* w2, const void* b2, const void* x,
                           const void* addend, void* y, void* ws, size_t ws_bytes,
                           void* stream);

/* moe_dense_ffn recording events[0] at the start, events[1] after the first
 * GEMM and events[2] after the second (n_events == MOE_NUM_DENSE_EVENTS). */
#define MOE_NUM_DENSE_EVENTS 3
moe_status_t moe_dense_ffn_profiled(const moe_dense_desc_t* d, const void* w1, const void* b1,
                                    const void* w2, const void* b2, const void* x,
                                    const void* addend, void* y, void* ws, size_t ws_bytes,
                                    void* stream, void* const* events, int n_events);

/* ---- backward of the layer (training) ---------------------------------
 * The chain rule through each forward step above.  The pages describe
 * training only in prose (the GLaM notes: the router is trained with a
 * penalty on uneven expert load); this is the gradient of the layer output
 * itself.  The top-k choice is piecewise constant, so the gradient reaches
 * the router only through the weights w of the chosen experts, and e_bias
 * (which enters the choice only) has none. */

/* Gradients written by moe_backward (device pointers, caller-owned; every
 * one is overwritten, not accumulated). */
typedef struct {
  void* dx;      /* [T, D] dtype: dL/dx (routed experts + shared expert + router) */
  float* dw_r;   /* [D, M] fp32 */
  float* dw1;    /* [M, H or 2I, D] fp32 (layout of w1) */
  float* db1;    /* [M, H] fp32; required iff act = GELU_TANH and has_bias, else ignored */
  float* dw2;    /* [M, D, H or I] fp32 (layout of w2) */
  float* db2;    /* [M, D] fp32; as db1 */
  float* dsh_w1; /* [2 I_sh, D] fp32; required iff I_sh > 0, else ignored */
  float* dsh_w2; /* [D, I_sh] fp32; as dsh_w1 */
} moe_grads_t;

/* Workspace of moe_backward.  It begins with the forward's layout
 * (moe_workspace_layout: after the call the routing fields hold this
 * backward's routing); the rest holds fp32 intermediates of every
 * dispatched row (pre-activations, activations, expert outputs and their
 * gradients).  0 if the descriptor is invalid. */
size_t moe_backward_workspace_size(const moe_layer_desc_t* d);

/* Given x [T, D] and dy = dL/dy [T, D] (both dtype) of y = MoE-FFN(x), write
 * every gradient of L: the routing is recomputed (the same route and
 * dispatch order as moe_forward), the experts' forward values are recomputed
 * in fp32 from the dtype inputs, and every GEMM of the backward sums in fp32
 * in a fixed order (bitwise repeatable).  Per chosen pair (t, j) with expert
 * e and weight w:
 *   dw[t,j]   = <dy_t, E_e(x_t)>,     dE = w dy_t  through the expert;
 *   dlogits   from dw through the weight formula of the gate;
 *   dx_t      = sum_j dx of the pair + shared expert's dx + dlogits_t W_r^T;
 *   dW_r      = x^T dlogits.
 * The expert and shared weights get the sums over their rows of the usual
 * FFN weight gradients.  x, dy and the gradients must not overlap.  Errors
 * as moe_forward; required gradient pointers that are NULL give
 * MOE_ERR_INVALID_ARG.  T = 0 zero-fills the parameter gradients. */
moe_status_t moe_backward(const moe_layer_desc_t* d, const moe_weights_t* w, const void* x,
                          const void* dy, const moe_grads_t* grads, void* ws, size_t ws_bytes,
                          void* stream);

/* Number of kernels one moe_backward call with this descriptor launches. */
int moe_backward_launch_count(const moe_layer_desc_t* d);

/* ---- diagnostics (no counterpart on the source pages) ------------------- */

/* Self-test of the bounded waits that every pipelined kernel of this library
 * uses instead of unbounded spins.  One kernel of 64 threads waits on two
 * shared-memory barriers that nothing ever arrives on: warp 0 with a limit
 * of limit_ns, warp 1 with 4 x limit_ns.  Warp 0 gives up when its limit
 * passes, records MOE_DEVERR_TIMEOUT in *device_status and raises the
 * kernel's abort flag; warp 1 must then leave on that flag (as the other
 * roles of a GEMM do), well before its own limit.  No fault, no hang: the
 * context stays usable.
 *   device_status: device int32, cleared by the call, MOE_DEVERR_TIMEOUT
 *   afterwards.  elapsed_ns: NULL or device uint64 [2]: the nanoseconds
 *   each warp waited, bit 63 set if its wait succeeded (it never should).
 *   1000 <= limit_ns <= 2e9, else MOE_ERR_INVALID_ARG. */
moe_status_t moe_selftest_wait_timeout(uint64_t limit_ns, int32_t* device_status,
                                       uint64_t* elapsed_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_B200_H_ */
