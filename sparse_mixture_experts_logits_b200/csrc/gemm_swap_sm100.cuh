// Grouped GEMM with the tokens on the MMA's N side ("swap-AB"), on CTA pairs
// (tcgen05.mma.cta_group::2, M = 256 weight rows, N = 16..256 tokens).
//
//   out[r, n] = epilogue( sum_k W[g*w_rows + n', k] * X[r, k] )
//
// for every dispatch row r of group g's segment offsets[g] .. offsets[g+1]
// and every output column n.  W is a bf16 stack of per-group [rows, K]
// weight blocks (nn.Linear layout, K-major) and is the MMA's A operand;
// the token rows X[r] (dispatch order: x gathered per expert, or h) are the
// B operand.  Each CTA loads one 128-row TMA box of token rows per k-block
// and the MMA reads the first N/2 of them.  (Loading the rows by index with
// tile::gather4 instead, 4 rows per TMA instruction, measured 2-3x slower:
// the TMA instruction rate, not the bytes, became the limit.)
//
// Decode-shaped layers (a handful of rows per expert) do not come here: a
// single-CTA MMA issues much faster than a pair's, so those run on the
// tokens-on-M kernel of gemm_sm100.cuh with NCTA = 1.
//
// Why tokens on N: an expert's segment is cut into token tiles of at most
// 256 rows whose width N is rounded up only to a multiple of 16, so the
// padding per segment is at most 15 rows (instead of up to 255 with 256-row
// M tiles); and in the accumulator a TMEM lane is an output column, so each
// token's 32 (or 64) output columns leave a warp as one contiguous store.
//
// Per CTA pair and tile: 256 weight rows (128 staged by each CTA: two 64-row
// TMA boxes) x N tokens (N/2 staged by each CTA).  SwiGLU tiles stage 64 gate
// and the matching 64 up rows in each CTA, so gate and up of one output
// column sit in TMEM lanes m and m + 64 of the same CTA; the epilogue warps
// of the up lanes hand their values to the gate lanes through shared memory.
//
// Warp roles (320 threads per CTA): warp 0 TMA producer, warp 1 TMEM
// allocator and (first CTA) MMA issuer, warps 2..9 epilogue.  Every wait is
// bounded (kWaitTimeoutNs) and reports MOE_DEVERR_TIMEOUT through the status
// word instead of hanging.
//
// Three operand layouts (template LAYOUT), all with the same tiles, TMEM
// accumulator and epilogue geometry (a TMEM lane is an A index, a column a B
// index):
//   kSwFwd    A = weight rows, K-major ([rows, K], the forward GEMMs);
//             B = token rows, K-major; groups split the token rows.
//   kSwDgrad  A = a weight stack read MN-major: group g's K rows are
//             g * k_rows_per_group + k of a [G * K, A_cols] matrix (W2 or
//             W1 of the nn.Linear layout contracted over its out index, the
//             input gradients of the backward); B and groups as kSwFwd.
//   kSwWgrad  A and B both MN-major activations [rows, cols] and the groups
//             split the contraction (the rows): group g (segment offsets[g]
//             .. offsets[g+1], a multiple of 64 rows whose padding rows are
//             zero) gives out[g] = A_g^T B_g, the weight gradients of the
//             backward.  Every output tile covers 256 A columns x 256 B columns.
#pragma once

#include "gemm_sm100.cuh"

namespace moe {

// A pipeline stage holds kSwKB consecutive k-blocks of 64: the MMA thread
// waits once and commits once per stage.  Two k-blocks per stage (3 stages
// of 64 KB) measured faster than one (6 stages of 32 KB) and than three.
constexpr int kSwKB = 2;
constexpr int kSwStages = 3;
constexpr int kSwATileBytes = 128 * kBK * 2;  // 128 weight rows per CTA, one k-block
constexpr int kSwBTileBytes = 128 * kBK * 2;  // up to 128 token rows per CTA, one k-block
constexpr int kSwStageBytes = kSwKB * (kSwATileBytes + kSwBTileBytes);
constexpr int kSwXPitch = 33;                 // floats per row of the gate/up hand-off buffer
constexpr int kSwXBytes = 4 * 32 * kSwXPitch * 4;
constexpr int kSwDynSmem = kSwStages * kSwStageBytes + kSwXBytes + 1024;
constexpr int kSwMaxTile = 256;               // tokens per tile
static_assert(kBK == 64, "the MMA loop issues four K = 16 slices per stage");

// Tensor maps of one launch.  The token operand always moves 128 rows per
// CTA and k-block, whatever the tile's N: a copy per exact N / 2 rows
// (boxes of 64, 32, 16 and 8 rows) costs more in TMA instructions than the
// rows it saves.
struct SwapMaps {
  CUtensorMap w;    // A operand
  CUtensorMap x;    // B operand
  CUtensorMap out;  // kSwWgrad: fp32 [G][b_cols][out_cols] output, 32 x 32 boxes
};

// The weight-gradient layout contracts over an expert's rows only (a few
// k-blocks per tile), so its epilogue, not the MMA, sets the pace.  It runs
// a 2-stage pipeline and gives the third stage's 64 KB to its eight epilogue
// warps as two 4 KB store-staging buffers each: every 32 x 32 fp32 chunk
// leaves through one TMA store instead of 32 warp-wide scalar stores.
// Epilogue warps (a multiple of 4: one per TMEM lane quarter, then more
// chunk parts).  The fused SwiGLU epilogue is light next to its long
// contraction, and with 4 warps the producer and MMA warps share their
// schedulers with fewer epilogue warps: the gate/up GEMMs ran 2-6% faster
// (GLM-5, GLM-4.5).  The heavier epilogues (GELU, fp32 rows, the backward's)
// keep 8: with 4 they were 20-50% slower.
template <int EPI>
constexpr int swap_epi_warps() { return EPI == EPI_SWIGLU ? 4 : 8; }
template <int EPI>
constexpr int swap_threads() { return 64 + 32 * swap_epi_warps<EPI>(); }

constexpr int kSwWgStages = 2;
constexpr int kSwWgStageBufBytes = 32 * 32 * 4;
static_assert(kSwStages > kSwWgStages &&
                  swap_epi_warps<EPI_STORE_F32>() * 2 * kSwWgStageBufBytes <= kSwStageBytes,
              "the store staging buffers fill the weight-gradient pipeline's unused stage");

struct SwapArgs {
  int num_groups;
  const int* offsets;      // [G + 1] or nullptr: one group [0, rows)
  int rows;
  int K;
  int w_rows_per_group;    // weight rows of one group
  int w_tiles;             // weight tiles per group
  int w_tile_step;         // weight-row advance per weight tile (256; SwiGLU 128)
  int w_hi_offset;         // row offset of a CTA's second 64-row box (64; SwiGLU: I, the up block)
  int w_cta_step;          // row offset of the second CTA's boxes (128; SwiGLU 64)
  int cols_per_tile;       // output columns of one weight tile (256; SwiGLU 128)
  int out_cols;            // valid output columns
  int ldo;
  void* out;
  const float* row_scale;      // EPI_SCALE_BIAS: [rows]
  const __nv_bfloat16* bias;   // EPI_GELU_BIAS / EPI_SCALE_BIAS / EPI_BIAS_ADD: [G, out_cols] or nullptr
  const __nv_bfloat16* addend; // EPI_BIAS_ADD: [rows, ldo] or nullptr
  int* status;
  // kSwDgrad: K rows of A per group.  kSwWgrad: B tiles per group, valid B
  // columns (output rows) and output elements per group.
  int k_rows_per_group;
  int b_tiles;
  int b_cols;
  long long out_gstride;
  // backward epilogues: the saved fp32 pre-activations (out of SAVE, aux
  // [rows, ld_aux] of DACT), the second and third bf16 outputs [rows, ldo2]
  // (SAVE: a and w a), the per-32-column partial dot products parts
  // [rows, ld_parts] (DACT), and I, the offset of the up half in the SwiGLU
  // outputs.
  __nv_bfloat16* out2;
  __nv_bfloat16* out3;
  int ldo2;
  const float* aux;
  int ld_aux;
  float* parts;
  int ld_parts;
  int half_cols;
  // optional [G]: rows of group g's segment to compute (the segment starts
  // at offsets[g] and may be longer: zero padding that no tile covers)
  const int* counts;
  // optional: a counter that is 0 when the launch starts.  Given, and when
  // at least a quarter of the groups with rows have fewer than 64 rows, the
  // CTA pairs claim tiles from it in index order as they become free
  // (dynamic schedule); otherwise they take fixed rounds (swap_tile_at).
  int* tile_ctr;
};

// Token tiles of a segment of `cnt` rows: ceil(cnt / 256) tiles of equal
// width rounded up to 16, then as many as that width needs.
__device__ __forceinline__ void token_tiling(int cnt, int& width, int& ntiles) {
  if (cnt <= 0) { width = 16; ntiles = 0; return; }
  const int n0 = (cnt + kSwMaxTile - 1) / kSwMaxTile;
  width = (((cnt + n0 - 1) / n0) + 15) & ~15;
  ntiles = (cnt + width - 1) / width;
}

// Tile of round rd for CTA pair `unit`: rounds of `units` consecutive tiles,
// dealt in alternating directions, so that the pair that takes the last
// tile of one round takes the first of the next.  Tile costs vary with the
// width of each expert's token tiles; dealing every round in the same
// direction gave the low-numbered pairs the larger share (same-box A/B:
// GLaM layer 1.32 -> 1.29 ms, GLM-4.5 prefill 7.27-7.36 -> 7.19-7.25 ms).
__device__ __forceinline__ int swap_tile_at(int rd, int unit, int units) {
  return rd * units + ((rd & 1) ? units - 1 - unit : unit);
}

struct SwapTile {
  int g, wt, tok0, nrows, n;  // group, weight tile, first token, rows, MMA N
  int nkb;                    // k-blocks of this tile (kSwWgrad: the group's rows / 64)
};

// Tiles of one group: token tiles x weight tiles, or (kSwWgrad) the fixed
// 256 x 256 output tiles of a group that has rows.
template <int LAYOUT>
__device__ __forceinline__ int swap_group_tiles(int cnt, const SwapArgs& a) {
  if constexpr (LAYOUT == kSwWgrad) return cnt > 0 ? a.w_tiles * a.b_tiles : 0;
  int width, ntt;
  token_tiling(cnt, width, ntt);
  return ntt * a.w_tiles;
}

template <int LAYOUT>
__device__ __forceinline__ SwapTile swap_decode(int tile, int G, const int* s_tstart, const int* s_cnt,
                                                const SwapArgs& a, int num_kb) {
  const int w_tiles = a.w_tiles;
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  SwapTile t;
  t.g = lo;
  const int cnt = s_cnt[lo];
  if constexpr (LAYOUT == kSwWgrad) {
    const int local = tile - s_tstart[lo];
    t.wt = local % w_tiles;
    const int bt = local / w_tiles;
    t.tok0 = bt * kSwMaxTile;
    t.nrows = min(kSwMaxTile, a.b_cols - t.tok0);
    t.n = kSwMaxTile;
    t.nkb = (cnt + kBK - 1) / kBK;
    return t;
  }
  t.nkb = num_kb;
  int width, ntt;
  token_tiling(cnt, width, ntt);
  const int local = tile - s_tstart[lo];
  const int band = local / (kBandM * w_tiles);
  const int rem = local - band * kBandM * w_tiles;
  const int bt = min(kBandM, ntt - band * kBandM);
  t.wt = rem / bt;
  const int tt = band * kBandM + (rem - t.wt * bt);
  t.tok0 = tt * width;
  t.nrows = min(width, cnt - t.tok0);
  t.n = (t.nrows + 15) & ~15;
  return t;
}

// Stores of one token's value for this lane's output column: the warp's 32
// lanes cover 32 consecutive columns, i.e. one contiguous row segment.
template <int EPI>
__device__ __forceinline__ void swap_store(const SwapArgs& a, size_t row, int col, float v) {
  if constexpr (EPI == EPI_SCALE_BIAS || EPI == EPI_STORE_F32 || EPI == EPI_ACCUM_F32)
    static_cast<float*>(a.out)[row * a.ldo + col] = v;
  else
    static_cast<__nv_bfloat16*>(a.out)[row * a.ldo + col] = __float2bfloat16_rn(v);
}
// Same at an element offset `base` (a group's own output block).
template <int EPI>
__device__ __forceinline__ void swap_store(const SwapArgs& a, size_t base, int col, float v, size_t row) {
  if constexpr (EPI == EPI_SCALE_BIAS || EPI == EPI_STORE_F32 || EPI == EPI_ACCUM_F32)
    static_cast<float*>(a.out)[base + row * a.ldo + col] = v;
  else
    static_cast<__nv_bfloat16*>(a.out)[base + row * a.ldo + col] = __float2bfloat16_rn(v);
}

// GELU (tanh form) and its derivative from one tanh: with t = tanh u,
// u = c (v + 0.044715 v^3) and s = 0.5 (1 + t), GELU(v) = v s and
// GELU'(v) = s + 0.5 v (1 - t^2) c (1 + 3 * 0.044715 v^2).
__device__ __forceinline__ void gelu_tanh_and_grad_fast(float v, float& g, float& dg) {
  const float c = 0.7978845608028654f;
  const float u = c * fmaf(0.044715f * v, v * v, v);
  const float t = tanh_hw(u);
  const float s = fmaf(0.5f, t, 0.5f);  // 0.5 (1 + tanh u)
  g = v * s;
  dg = fmaf(0.5f * v * fmaf(-t, t, 1.0f) * c, fmaf(3.0f * 0.044715f, v * v, 1.0f), s);
}

// Sum over the warp's 32 lanes of v[i] for every i, in 31 shuffles: after
// the five halving rounds lane L holds the sum of v[L] over all lanes (the
// butterfly transpose-reduction).  Exact order fixed, so repeatable.
__device__ __forceinline__ float warp_transpose_sum(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
  return v[0];
}

template <int EPI, int LAYOUT>
__global__ void __launch_bounds__(swap_threads<EPI>(), 1)
    moe_gemm_swap_kernel(const __grid_constant__ SwapMaps maps, const SwapArgs args) {
  constexpr int S = LAYOUT == kSwWgrad ? kSwWgStages : kSwStages;
  constexpr bool kSwiglu = EPI == EPI_SWIGLU || EPI == EPI_BWD_SWIGLU_SAVE;
  constexpr bool kAMn = LAYOUT != kSwFwd;
  constexpr bool kBMn = LAYOUT == kSwWgrad;
  static_assert(!(kSwiglu && LAYOUT != kSwFwd), "the gate/up pairing reads K-major weight rows");
  extern __shared__ uint8_t dyn_smem[];
  __shared__ int s_off[kMaxExperts + 1];
  __shared__ int s_cnt[kMaxExperts];
  __shared__ int s_tstart[kMaxExperts + 1];
  __shared__ __align__(8) uint64_t s_full[S];
  __shared__ __align__(8) uint64_t s_empty[S];
  __shared__ __align__(8) uint64_t s_tfull[2];
  __shared__ __align__(8) uint64_t s_tempty[2];
  __shared__ __align__(8) uint64_t s_xfull[4];
  __shared__ __align__(8) uint64_t s_xempty[4];
  __shared__ __align__(8) uint64_t s_drain;
  // dynamic schedule: the leader CTA's producer publishes each claimed tile
  // into this ring in both CTAs of the pair
  constexpr int kTq = 8;
  __shared__ int s_tq[kTq];
  __shared__ __align__(8) uint64_t s_tq_full[kTq];   // one arrival: the leader's producer
  __shared__ __align__(8) uint64_t s_tq_empty[kTq];  // leader's: every reader releases the slot
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;
  __shared__ int s_total;
  __shared__ int s_dyn;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int unit = static_cast<int>(blockIdx.x >> 1);
  const int units = static_cast<int>(gridDim.x >> 1);
  const uint32_t smem_base = (smem_addr(dyn_smem) + 1023u) & ~1023u;
  float* xbuf = reinterpret_cast<float*>(dyn_smem + (smem_base - smem_addr(dyn_smem)) + kSwStages * kSwStageBytes);
  const int G = args.num_groups;

  // Segment bounds clamped to [0, rows], so that offsets that are not a
  // valid dispatch cannot send a tile outside the token buffer (a segment
  // whose end lies before its start gets no tile).
  for (int i = threadIdx.x; i <= G; i += blockDim.x) {
    const long long o = args.offsets != nullptr ? args.offsets[i] : (i == 0 ? 0 : args.rows);
    s_off[i] = static_cast<int>(o < 0 ? 0 : (o > args.rows ? args.rows : o));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G; i += blockDim.x) {
    const int seg = max(0, s_off[i + 1] - s_off[i]);
    s_cnt[i] = args.counts != nullptr ? max(0, min(args.counts[i], seg)) : seg;
  }
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    int busy = 0, narrow = 0;  // groups with rows; of those, groups of fewer than 64 rows
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      const int c = g < G ? s_cnt[g] : 0;
      busy += __popc(__ballot_sync(0xffffffffu, c > 0));
      narrow += __popc(__ballot_sync(0xffffffffu, c > 0 && c < 64));
      const int v = g < G ? swap_group_tiles<LAYOUT>(c, args) : 0;
      int incl = v;
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += t;
      }
      if (g < G) s_tstart[g] = carry + incl - v;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      s_tstart[G] = carry;
      s_total = carry;
      s_abort = 0;
      // Claim tiles dynamically when at least a quarter of the groups with
      // rows are narrow: their tiles stream a whole weight tile for a few
      // rows, at a cost that depends on what runs beside them, which fixed
      // rounds cannot balance (GLM-5 skewed prefill: 40% narrow, expert
      // GEMM1 6.28 -> 5.77 ms).  With few narrow groups the fixed rounds
      // were as fast or faster (GLaM: none, GEMM1 0.547 against 0.583 ms
      // dynamic; GLM-4.5: 19%, within noise).
      s_dyn = args.tile_ctr != nullptr && narrow > 0 && 4 * narrow >= busy;
      for (int s = 0; s < S; ++s) {
        mbar_init(smem_addr(&s_full[s]), 1);
        mbar_init(smem_addr(&s_empty[s]), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_addr(&s_tfull[b]), 1);
        mbar_init(smem_addr(&s_tempty[b]), swap_epi_warps<EPI>() * 32 * 2);
      }
      for (int x = 0; x < 4; ++x) {
        mbar_init(smem_addr(&s_xfull[x]), 32);
        mbar_init(smem_addr(&s_xempty[x]), 32);
      }
      mbar_init(smem_addr(&s_drain), 1);
      // readers of a ring slot: the leader's MMA warp and epilogue warps, the
      // peer's producer and epilogue warps (one elected lane each)
      for (int q = 0; q < kTq; ++q) {
        mbar_init(smem_addr(&s_tq_full[q]), 1);
        mbar_init(smem_addr(&s_tq_empty[q]), 2 + 2 * swap_epi_warps<EPI>());
      }
      fence_mbar_init();
      tma_prefetch_desc(&maps.w);
      tma_prefetch_desc(&maps.x);
      if constexpr (LAYOUT == kSwWgrad) tma_prefetch_desc(&maps.out);
    }
  } else if (warp == 1) {
    tmem_alloc_pair(smem_addr(&s_tmem_base), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int total = s_total;
  const int num_kb = (args.K + kBK - 1) / kBK;
  volatile int* abort_flag = &s_abort;
  const bool dyn = s_dyn != 0;

  // Dynamic schedule.  The leader's producer posts lane 0's `tile` as round
  // i's to ring slot i % kTq of both CTAs (warp-uniform; false when the
  // wait for a free slot gave up).  It claims each tile from the counter
  // one round before posting it, so the atomic's round trip overlaps a
  // whole tile of loads.
  auto tq_post = [&](int i, int tile) -> bool {
    const int r = i & (kTq - 1);
    if (!mbar_wait_all(smem_addr(&s_tq_empty[r]), ((i / kTq) & 1) ^ 1u, abort_flag, args.status)) return false;
    if (lane == 0) {
      s_tq[r] = tile;
      st_shared_cluster_u32(mapa_shared(smem_addr(&s_tq[r]), 1), tile);
      mbar_arrive(smem_addr(&s_tq_full[r]));
      mbar_arrive_remote(mapa_shared(smem_addr(&s_tq_full[r]), 1));
    }
    __syncwarp();
    return true;
  };
  // Every other role reads round i's tile from its own CTA's ring and
  // releases the slot to the leader (warp-uniform; okr = false on give-up).
  auto tq_take = [&](int i, bool& okr) -> int {
    const int r = i & (kTq - 1);
    if (!mbar_wait_all_cluster(smem_addr(&s_tq_full[r]), (i / kTq) & 1, abort_flag, args.status)) {
      okr = false;
      return 0;
    }
    const int tile = *reinterpret_cast<volatile int*>(&s_tq[r]);
    __syncwarp();
    if (lane == 0) {
      if (leader) mbar_arrive(smem_addr(&s_tq_empty[r]));
      else mbar_arrive_remote(mapa_shared(smem_addr(&s_tq_empty[r]), 0));
    }
    return tile;
  };

  // The producer and MMA loops run on whole warps with warp-uniform control
  // (stage, phase, tile); only lane 0 issues the TMA copies, MMAs and
  // commits.  Loop bookkeeping in a single divergent lane costs enough issue
  // cycles per k-block to leave the tensor pipe idle between MMAs.
  if (warp == 0) {
    // -------------------------------------------------------- TMA producer
    uint32_t s = 0, ph = 0;
    bool ok = true;
    // dynamic schedule, leader: `cur` is this round's tile (posted); lane 0's
    // `claimed` is the next round's, taken from the counter a round earlier
    int cur = 0, claimed = 0;
    if (dyn && leader) {
      int first = 0;
      if (lane == 0) {
        first = atomicAdd(args.tile_ctr, 1);
        claimed = atomicAdd(args.tile_ctr, 1);
      }
      ok = tq_post(0, first);
      cur = __shfl_sync(0xffffffffu, first, 0);
    }
    for (int rd = 0; ok; ++rd) {
      int tile;
      if (!dyn) {
        tile = swap_tile_at(rd, unit, units);
      } else if (leader) {
        tile = cur;
        if (tile < total) {
          if (!tq_post(rd + 1, claimed)) break;
          cur = __shfl_sync(0xffffffffu, claimed, 0);
          if (cur < total && lane == 0) claimed = atomicAdd(args.tile_ctr, 1);
        }
      } else {
        tile = tq_take(rd, ok);
        if (!ok) break;
      }
      if (tile >= total) break;
      const SwapTile t = swap_decode<LAYOUT>(tile, G, s_tstart, s_cnt, args, num_kb);
      // kSwFwd / kSwDgrad: B = this CTA's half of the token tile, K-major rows.
      // kSwWgrad: B = this CTA's 128 of the tile's 256 B columns, rows of the segment.
      const int x_row = s_off[t.g] + t.tok0 + static_cast<int>(rank) * (t.n >> 1);
      const int b_col = t.tok0 + static_cast<int>(rank) * (kSwMaxTile >> 1);
      // A: kSwFwd weight rows; otherwise the first of this CTA's 128 A columns
      const int w_base = (LAYOUT == kSwFwd ? t.g * args.w_rows_per_group : 0) + t.wt * args.w_tile_step +
                         static_cast<int>(rank) * args.w_cta_step;
      const int k_row0 = LAYOUT == kSwDgrad ? t.g * args.k_rows_per_group : s_off[t.g];
      // both CTAs' bytes of one k-block: 128 weight rows + 128 B rows each
      constexpr uint32_t kb_bytes = 2u * (kSwATileBytes + kSwBTileBytes);
      for (int kb0 = 0; kb0 < t.nkb; kb0 += kSwKB) {
        const int nk = min(kSwKB, t.nkb - kb0);
        if (!mbar_wait_all(smem_addr(&s_empty[s]), ph ^ 1u, abort_flag, args.status)) { ok = false; break; }
        if (lane == 0) {
          const uint32_t sa = smem_base + s * kSwStageBytes;
          const uint32_t sb = sa + kSwKB * kSwATileBytes;
          const uint32_t full_leader = mapa_shared(smem_addr(&s_full[s]), 0);
          if (leader) mbar_arrive_expect_tx(smem_addr(&s_full[s]), static_cast<uint32_t>(nk) * kb_bytes);
          for (int i = 0; i < nk; ++i) {
            const int kc = (kb0 + i) * kBK;
            const uint32_t ai = sa + i * kSwATileBytes;
            const uint32_t bi = sb + i * kSwBTileBytes;
            if constexpr (!kAMn) {
              tma_load_2d_pair(ai, &maps.w, full_leader, kc, w_base);
              tma_load_2d_pair(ai + 64 * kBK * 2, &maps.w, full_leader, kc, w_base + args.w_hi_offset);
            } else {
              // two boxes of 64 A columns x 64 K rows (8 KB each, 8 KB apart)
              tma_load_2d_pair(ai, &maps.w, full_leader, w_base, k_row0 + kc);
              tma_load_2d_pair(ai + 64 * kBK * 2, &maps.w, full_leader, w_base + args.w_hi_offset, k_row0 + kc);
            }
            if constexpr (!kBMn) {
              tma_load_2d_pair(bi, &maps.x, full_leader, kc, x_row);
            } else {
              tma_load_2d_pair(bi, &maps.x, full_leader, b_col, k_row0 + kc);
              tma_load_2d_pair(bi + 64 * kBK * 2, &maps.x, full_leader, b_col + 64, k_row0 + kc);
            }
          }
        }
        __syncwarp();
        if (++s == S) { s = 0; ph ^= 1u; }
      }
    }
  } else if (warp == 1) {
    if (leader) {
      // -------------------------------------------------------- MMA issuer
      uint32_t it = 0, s = 0, ph = 0;
      bool ok = true;
      // descriptors of stage 0; stage s and k-slice kk add s * stage/16 and
      // kk * (slice bytes)/16 to the 14-bit start-address field, which never
      // carries (smem < 256 KB).  A K = 16 slice is 32 bytes along a K-major
      // row, or 16 rows of 128 bytes (2048 bytes) of an MN-major tile.
      constexpr uint64_t kAStep = kAMn ? 128 : 2;
      constexpr uint64_t kBStep = kBMn ? 128 : 2;
      const uint64_t da0 = kAMn ? sw128_mnmajor_desc(smem_base, 64 * kBK * 2) : sw128_kmajor_desc(smem_base);
      const uint64_t db0 = kBMn ? sw128_mnmajor_desc(smem_base + kSwKB * kSwATileBytes, 64 * kBK * 2)
                                : sw128_kmajor_desc(smem_base + kSwKB * kSwATileBytes);
      for (int rd = 0; ok; ++rd, ++it) {
        int tile;
        if (dyn) {
          tile = tq_take(rd, ok);
          if (!ok) break;
        } else {
          tile = swap_tile_at(rd, unit, units);
        }
        if (tile >= total) break;
        const SwapTile t = swap_decode<LAYOUT>(tile, G, s_tstart, s_cnt, args, num_kb);
        const uint32_t idesc = umma_idesc_bf16_major(256, t.n, kAMn ? 1 : 0, kBMn ? 1 : 0);
        const uint32_t buf = it & 1u;
        const uint32_t tph = (it >> 1) & 1u;
        if (!mbar_wait_all(smem_addr(&s_tempty[buf]), tph ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * 256u;
        for (int kb0 = 0; kb0 < t.nkb; kb0 += kSwKB) {
          const int nk = min(kSwKB, t.nkb - kb0);
          if (!mbar_wait_all(smem_addr(&s_full[s]), ph, abort_flag, args.status)) { ok = false; break; }
          if (lane == 0) {
            const uint64_t off = static_cast<uint64_t>(s * (kSwStageBytes >> 4));
#pragma unroll
            for (int i = 0; i < kSwKB; ++i) {
              if (i < nk) {
                const uint64_t a = da0 + off + i * (kSwATileBytes >> 4);
                const uint64_t b = db0 + off + i * (kSwBTileBytes >> 4);
                umma_bf16_pair(d_tmem, a, b, idesc, (kb0 | i) != 0 ? 1u : 0u);
                umma_bf16_pair(d_tmem, a + kAStep, b + kBStep, idesc, 1u);
                umma_bf16_pair(d_tmem, a + 2 * kAStep, b + 2 * kBStep, idesc, 1u);
                umma_bf16_pair(d_tmem, a + 3 * kAStep, b + 3 * kBStep, idesc, 1u);
              }
            }
            umma_commit_pair(smem_addr(&s_empty[s]), 0x3);
          }
          __syncwarp();
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        if (lane == 0) umma_commit_pair(smem_addr(&s_tfull[buf]), 0x3);
        __syncwarp();
      }
      if (lane == 0) {
        umma_commit_pair(smem_addr(&s_drain), 0x1);
        mbar_wait_drain(smem_addr(&s_drain), 0, kWaitTimeoutNs);
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;           // TMEM lane quarter
    constexpr int kParts = swap_epi_warps<EPI>() / 4;  // epilogue warps per TMEM lane quarter
    const int part = (warp - 2) >> 2; // token chunks part, part + kParts, ...
    const int m = q * 32 + lane;      // accumulator lane = weight row inside this CTA
    const uint32_t tempty0 = mapa_shared(smem_addr(&s_tempty[0]), 0);
    const uint32_t tempty1 = mapa_shared(smem_addr(&s_tempty[1]), 0);
    const int xpair = part * 2 + (q & 1);         // SwiGLU hand-off pair (gate q, up q + 2)
    float* xs = xbuf + xpair * 32 * kSwXPitch;
    const bool up_warp = kSwiglu && q >= 2;
    uint32_t it = 0, xc = 0;
    uint32_t sc = 0;  // kSwWgrad: chunks this warp has stored (staging buffer sc & 1)
    const uint32_t stg = smem_base + kSwWgStages * kSwStageBytes + (warp - 2) * 2 * kSwWgStageBufBytes;
    float* stgp = reinterpret_cast<float*>(dyn_smem + (stg - smem_addr(dyn_smem)));
    bool ok = true;
    for (int rd = 0; ok; ++rd, ++it) {
      int tile;
      if (dyn) {
        tile = tq_take(rd, ok);
        if (!ok) break;
      } else {
        tile = swap_tile_at(rd, unit, units);
      }
      if (tile >= total) break;
      const SwapTile t = swap_decode<LAYOUT>(tile, G, s_tstart, s_cnt, args, num_kb);
      const uint32_t buf = it & 1u;
      const uint32_t tph = (it >> 1) & 1u;
      if (!mbar_wait(smem_addr(&s_tfull[buf]), tph, abort_flag, args.status)) break;
      tc_fence_after();
      const int col = kSwiglu ? t.wt * args.cols_per_tile + static_cast<int>(rank) * 64 + (m & 63)
                              : t.wt * args.cols_per_tile + static_cast<int>(rank) * 128 + m;
      const bool col_ok = col < args.out_cols;
      float bias = 0.f;
      if constexpr (EPI == EPI_GELU_BIAS || EPI == EPI_SCALE_BIAS || EPI == EPI_BIAS_ADD ||
                    EPI == EPI_BWD_GELU_SAVE) {
        if (args.bias != nullptr && col_ok)
          bias = __bfloat162float(args.bias[static_cast<size_t>(t.g) * args.out_cols + col]);
      }
      // output row of the tile's first token (kSwWgrad: the first B column of
      // the tile, in group g's own output block)
      const size_t row0 = LAYOUT == kSwWgrad ? static_cast<size_t>(t.tok0)
                                             : static_cast<size_t>(s_off[t.g]) + t.tok0;
      const size_t gofs = LAYOUT == kSwWgrad ? static_cast<size_t>(t.g) * args.out_gstride : 0;
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + buf * 256u;
      constexpr bool kScaled = EPI == EPI_SCALE_BIAS || EPI == EPI_BWD_GELU_SAVE ||
                               EPI == EPI_BWD_SWIGLU_SAVE || EPI == EPI_BWD_GELU_DACT ||
                               EPI == EPI_BWD_SWIGLU_DACT;
      constexpr bool kDact = EPI == EPI_BWD_GELU_DACT || EPI == EPI_BWD_SWIGLU_DACT;
      if constexpr (LAYOUT == kSwWgrad) {
        // Weight gradients: the warp's four 32 x 32 chunks (N = 256) are read
        // from TMEM two at a time, one wait per pair, written to a staging
        // buffer in the output's own row-major layout (lane = column, so each
        // row of 32 floats is one conflict-free store) and sent out by one
        // TMA store per chunk.  The tensor map's extents clip the rows past
        // b_cols and the columns past out_cols.
        (void)gofs;
        (void)row0;
        const int col0 = col - lane;  // the warp's first output column (a multiple of 32)
#pragma unroll 1
        for (int j0 = 0; j0 < 8 / kParts; j0 += 2) {
          uint32_t r2[2][32];
          MOE_TMEM_LD32(tacc + 32 * (part + kParts * j0), r2[0]);
          MOE_TMEM_LD32(tacc + 32 * (part + kParts * (j0 + 1)), r2[1]);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const int c = 32 * (part + kParts * (j0 + j));
            if (col0 < args.out_cols && c < t.nrows) {
              const uint32_t b = sc & 1u;
              if (lane == 0) bulk_wait_group_read<1>();  // the store that last used buffer b has read it
              __syncwarp();
              float* st = stgp + b * (kSwWgStageBufBytes / 4);
#pragma unroll
              for (int i = 0; i < 32; ++i) st[i * 32 + lane] = __uint_as_float(r2[j][i]);
              fence_proxy_async_smem();
              __syncwarp();
              if (lane == 0) {
                tma_store_3d(&maps.out, stg + b * kSwWgStageBufBytes, col0, t.tok0 + c, t.g);
                bulk_commit_group();
              }
              ++sc;
            }
          }
        }
      } else
      for (int c = 32 * part; c < t.n; c += 32 * kParts) {
        // Every value this chunk reads from memory (the input-gradient
        // epilogues' saved pre-activations, the addend, the fp32 sum added
        // onto) is requested first, all 32 rows together, so that the loads
        // overlap the TMEM read and each other's.  Read inside the store loop
        // they would wait one memory round trip per row: the compiler cannot
        // move a load above the store to `out` before it.
        float hv[32], uv[32];
        if constexpr (kDact || EPI == EPI_BIAS_ADD) {
          const int nvd = min(32, t.nrows - c);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const bool live = col_ok && i < nvd;
            const size_t row = row0 + c + i;
            if constexpr (kDact) {
              hv[i] = live ? args.aux[row * args.ld_aux + col] : 0.f;
              if constexpr (EPI == EPI_BWD_SWIGLU_DACT)
                uv[i] = live ? args.aux[row * args.ld_aux + args.half_cols + col] : 0.f;
            } else {
              hv[i] = live && args.addend != nullptr ? __bfloat162float(args.addend[row * args.ldo + col]) : 0.f;
            }
          }
        }
        if constexpr (EPI == EPI_ACCUM_F32) {
          // out += acc in place: the chunk's 32 rows read first, then the TMEM read
          const int nva = col_ok ? min(32, t.nrows - c) : 0;
          float* op = static_cast<float*>(args.out) + (row0 + c) * args.ldo + col;
          const size_t ld = args.ldo;
          const float* lp = op;
#pragma unroll
          for (int i = 0; i < 32; ++i, lp += ld) hv[i] = i < nva ? *lp : 0.f;
          uint32_t ra[32];
          MOE_TMEM_LD32(tacc + c, ra);
          tmem_ld_wait();
          float* sp = op;
#pragma unroll
          for (int i = 0; i < 32; ++i, sp += ld)
            if (i < nva) *sp = __uint_as_float(ra[i]) + hv[i];
          continue;
        }
        uint32_t r[32];
        MOE_TMEM_LD32(tacc + c, r);
        tmem_ld_wait();
        const int nv = min(32, t.nrows - c);  // tokens of this chunk that exist
        float rs = 1.f;                       // this lane's token's row scale (gate weight)
        if constexpr (kScaled) {
          if (lane < nv && args.row_scale != nullptr) rs = args.row_scale[row0 + c + lane];
        }
        if constexpr (kSwiglu) {
          if (up_warp) {
            if (!mbar_wait(smem_addr(&s_xempty[xpair]), (xc & 1u) ^ 1u, abort_flag, args.status)) { ok = false; break; }
#pragma unroll
            for (int i = 0; i < 32; ++i) xs[lane * kSwXPitch + i] = __uint_as_float(r[i]);
            mbar_arrive(smem_addr(&s_xfull[xpair]));
          } else {
            if (!mbar_wait(smem_addr(&s_xfull[xpair]), xc & 1u, abort_flag, args.status)) { ok = false; break; }
            if constexpr (EPI == EPI_SWIGLU) {
              float v[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = silu_fast(__uint_as_float(r[i])) * xs[lane * kSwXPitch + i];
              mbar_arrive(smem_addr(&s_xempty[xpair]));
              if (col_ok) {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                  if (i < nv) swap_store<EPI>(args, row0 + c + i, col, v[i]);
              }
            } else {  // EPI_BWD_SWIGLU_SAVE: g, u, a = SiLU(g) u, w a
              float u[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) u[i] = xs[lane * kSwXPitch + i];
              mbar_arrive(smem_addr(&s_xempty[xpair]));
              float* hp = static_cast<float*>(args.out);
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const float g = __uint_as_float(r[i]);
                const float a = silu_fast(g) * u[i];
                const float w = __shfl_sync(0xffffffffu, rs, i);
                if (col_ok && i < nv) {
                  const size_t row = row0 + c + i;
                  hp[row * args.ldo + col] = g;
                  hp[row * args.ldo + args.half_cols + col] = u[i];
                  if (args.out2 != nullptr) args.out2[row * args.ldo2 + col] = __float2bfloat16_rn(a);
                  if (args.out3 != nullptr) args.out3[row * args.ldo2 + col] = __float2bfloat16_rn(w * a);
                }
              }
            }
          }
          ++xc;
        } else if constexpr (EPI == EPI_BWD_GELU_DACT || EPI == EPI_BWD_SWIGLU_DACT) {
          // G = acc (the gradient reaching a, before the gate weight); dh out,
          // and per token the partial <G, a> over this warp's 32 columns
          float prod[32];
          __nv_bfloat16* dh = static_cast<__nv_bfloat16*>(args.out);
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float G = __uint_as_float(r[i]);
            const float w = __shfl_sync(0xffffffffu, rs, i);
            prod[i] = 0.f;
            if (col_ok && i < nv) {
              const size_t row = row0 + c + i;
              if constexpr (EPI == EPI_BWD_GELU_DACT) {
                float a, da_dh;
                gelu_tanh_and_grad_fast(hv[i], a, da_dh);
                dh[row * args.ldo + col] = __float2bfloat16_rn(w * G * da_dh);
                prod[i] = G * a;
              } else {
                const float g = hv[i], u = uv[i];
                const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
                const float si = g * sg;
                const float da = w * G;
                dh[row * args.ldo + col] = __float2bfloat16_rn(da * u * sg * fmaf(g, 1.0f - sg, 1.0f));
                dh[row * args.ldo + args.half_cols + col] = __float2bfloat16_rn(da * si);
                prod[i] = G * si * u;
              }
            }
          }
          const float tot = warp_transpose_sum(prod, lane);
          // one partial per 32-column chunk that holds any valid column
          if (args.parts != nullptr && lane < nv && col - lane < args.out_cols)
            args.parts[(row0 + c + lane) * args.ld_parts + ((col - lane) >> 5)] = tot;
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float v = __uint_as_float(r[i]) + bias;
            if constexpr (EPI == EPI_GELU_BIAS) v = gelu_tanh_fast(v);
            if constexpr (EPI == EPI_SCALE_BIAS) v *= __shfl_sync(0xffffffffu, rs, i);
            if constexpr (EPI == EPI_BIAS_ADD || EPI == EPI_ACCUM_F32) v += hv[i];
            if constexpr (EPI == EPI_BWD_GELU_SAVE) {
              const float a = gelu_tanh_fast(v);
              const float w = __shfl_sync(0xffffffffu, rs, i);
              if (col_ok && i < nv) {
                const size_t row = row0 + c + i;
                static_cast<float*>(args.out)[row * args.ldo + col] = v;
                if (args.out2 != nullptr) args.out2[row * args.ldo2 + col] = __float2bfloat16_rn(a);
                if (args.out3 != nullptr) args.out3[row * args.ldo2 + col] = __float2bfloat16_rn(w * a);
              }
            } else {
              if (col_ok && i < nv) swap_store<EPI>(args, gofs, col, v, row0 + c + i);
            }
          }
        }
      }
      if (!ok) break;
      tc_fence_before();
      mbar_arrive_remote(buf ? tempty1 : tempty0);
    }
    if constexpr (LAYOUT == kSwWgrad) {
      // the staged chunks are read and written before shared memory is released
      if (lane == 0) bulk_wait_group<0>();
      __syncwarp();
    }
  }

  __syncthreads();
  if (s_abort && warp == 0 && lane == 0) {
    // let TMA loads still in flight land before shared memory is released
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  __syncthreads();
  cluster_sync_all();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

}  // namespace moe
