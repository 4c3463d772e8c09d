// Grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM, fed by TMA).
//
//   out[r, n] = epilogue( sum_k A[r, k] * B[g*b_rows + n', k] )
//
// A is a bf16 [rows, K] matrix whose rows are split into G contiguous
// segments (one per expert: offsets[g] .. offsets[g+1]); B is a bf16 stack of
// per-group [n, K] weight blocks in the nn.Linear [out, in] layout (K-major).
// Both operands are K-major, the natural tcgen05 layout.
//
// Persistent CTAs (NCTA = 1) or CTA pairs (NCTA = 2, a 2-CTA cluster on two
// SMs) walk a device-side list of (128 * NCTA) x BN output tiles (BN <= 256):
// the list is built in shared memory from offsets[] at kernel start, so no
// host synchronisation is needed to learn the segment sizes.  Inside a group
// tiles are ordered in bands of up to 16 m-tiles, and within a band
// n-tile-major, so that the CTAs working at one time share their weight
// tiles and activation rows through L2.
//
// NCTA = 2 uses the 2-SM MMA: the pair's first CTA issues 256 x BN x 16
// MMAs whose A rows come 128 from each CTA and whose B rows come BN/2 from
// each CTA, so every CTA stages only half of the weight tile (32 KB per
// stage instead of 48 KB, hence 6 stages instead of 4).  No load is
// multicast: each CTA fetches its own halves.
//
// Warp roles (320 threads per CTA):
//   warp 0      TMA producer: A tile 128 x 64 and this CTA's B rows x 64
//   warp 1      TMEM allocator; MMA issuer (one thread of the first CTA)
//   warps 2..9  epilogue: tcgen05.ld of the fp32 accumulator, fused
//               activation / scaling, stores to global; warp w
//               reads TMEM lane quarter w % 4, column chunks (w - 2) / 4
//               (mod 2)
// Two TMEM accumulators (2 x 256 columns) let the epilogue of one tile
// overlap the main loop of the next.
#pragma once

#include "common.cuh"

namespace moe {

enum GemmEpilogue : int {
  EPI_STORE_F32 = 0,   // out fp32 = acc                         (router logits)
  EPI_GELU_BIAS = 1,   // out bf16 = GELU_tanh(acc + b1[g, n])  (GELU expert, first GEMM)
  EPI_SWIGLU = 2,      // out bf16 = SiLU(acc_gate) * acc_up     (SwiGLU, fused gate/up)
  EPI_SCALE_BIAS = 3,  // out fp32 = (acc + b2[g, n]) * row_scale[r]   (second GEMM)
  // 4: unused (kept free so that the values of the others stay stable)
  EPI_STORE_BF16 = 5,  // out bf16 = acc                         (standalone shared down projection)
  EPI_BIAS_ADD = 6,    // out (layer dtype) = acc + b[n] + addend[r, n]   (dense FFN down projection;
                       //            bias and addend optional)
  // Backward (tokens-on-N kernel only):
  EPI_BWD_GELU_SAVE = 7,    // v = acc + b1: out = v (fp32), out2 = GELU(v), out3 = row_scale[r] GELU(v) (bf16;
                            // out2, out3 optional)
  EPI_BWD_SWIGLU_SAVE = 8,  // g, u: out[., n] = g, out[., I + n] = u (fp32), out2 = SiLU(g) u, out3 = w out2
  EPI_BWD_GELU_DACT = 9,    // G = acc, h = aux[r, n]: out = w G GELU'(h); parts += G GELU(h)
  EPI_BWD_SWIGLU_DACT = 10, // G = acc, g = aux[r, n], u = aux[r, I + n], a = SiLU(g) u, da = w G:
                            //   out[., n] = da u SiLU'(g), out[., I + n] = da SiLU(g); parts += G a
  EPI_ACCUM_F32 = 11,       // out fp32 += acc   (the router's dx onto the shared expert's)
};

// Operand layouts of the tokens-on-N GEMM (gemm_swap_sm100.cuh): the forward
// (both operands K-major), the input gradients (weights MN-major) and the
// weight gradients (both MN-major, groups over the contraction).
enum SwapLayout : int { kSwFwd = 0, kSwDgrad = 1, kSwWgrad = 2 };

constexpr int kBK = 64;
constexpr int kATileBytes = 128 * kBK * 2;  // 16 KB: 128 rows of A per CTA
constexpr int kGemmThreads = 320;
constexpr int kEpiWarps = 8;
constexpr int kBandM = 16;

template <int NCTA> struct GemmCfg;
template <> struct GemmCfg<1> {
  static constexpr int kStages = 4;
  static constexpr int kBRowsMax = 256;
  static constexpr int kStageBytes = kATileBytes + kBRowsMax * kBK * 2;  // 48 KB
  static constexpr int kTileRows = 128;
};
template <> struct GemmCfg<2> {
  static constexpr int kStages = 6;
  static constexpr int kBRowsMax = 128;
  static constexpr int kStageBytes = kATileBytes + kBRowsMax * kBK * 2;  // 32 KB
  static constexpr int kTileRows = 256;
};
template <int NCTA>
constexpr int gemm_dyn_smem() { return GemmCfg<NCTA>::kStages * GemmCfg<NCTA>::kStageBytes + 1024; }

struct GemmArgs {
  int num_groups;          // G >= 1
  const int* offsets;      // [G + 1] row offsets of the segments, or nullptr: one group [0, rows)
  int rows;                // rows of A when offsets == nullptr
  int K;                   // reduction length
  int n_tiles;             // tiles along N per group
  int bn;                  // accumulator columns of one tile (MMA N), multiple of 16, <= 256
  int b_rows_per_group;    // rows of B per group
  int b_row_step;          // B row advance per n-tile
  int b_hi_offset;         // B row offset of the tile's second half (bn/2 rows each)
  int out_cols;            // valid output columns
  int out_col_step;        // output column advance per n-tile
  int ldo;                 // output row stride in elements
  void* out;
  const float* row_scale;        // EPI_SCALE_BIAS: [rows]
  const __nv_bfloat16* bias;     // EPI_GELU_BIAS / EPI_SCALE_BIAS: [G, out_cols] or nullptr
  uint32_t idesc;
  int* status;
};

__device__ __forceinline__ void decode_tile(int tile, int G, const int* s_tstart, const int* s_off,
                                            int n_tiles, int tile_rows, int& g, int& mt, int& nt) {
  // last group whose start is <= tile (groups with no tiles have equal starts)
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int local = tile - s_tstart[g];
  const int mtiles = (s_off[g + 1] - s_off[g] + tile_rows - 1) / tile_rows;
  const int band = local / (kBandM * n_tiles);
  const int rem = local - band * kBandM * n_tiles;
  const int bm = min(kBandM, mtiles - band * kBandM);
  nt = rem / bm;
  mt = band * kBandM + (rem - nt * bm);
}

// 32 consecutive values of one row; nvalid < 32 only at the right edge of
// the matrix (predicated, fully unrolled: no local-memory indexing).
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, const float* v, int nvalid) {
  if (nvalid >= 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d4[q] = f32_to_bf16x8(v + 8 * q);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nvalid) dst[i] = __float2bfloat16_rn(v[i]);
  }
}
__device__ __forceinline__ void store_row32_f32(float* dst, const float* v, int nvalid, bool vec_ok) {
  if (nvalid >= 32 && vec_ok) {
    float4* o4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 8; ++q) o4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nvalid) dst[i] = v[i];
  }
}
__device__ __forceinline__ void add_bias32(float* v, const __nv_bfloat16* b, int nvalid) {
  if (nvalid >= 32) {
    const uint4* b4 = reinterpret_cast<const uint4*>(b);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float f[8];
      bf16x8_to_f32(b4[q], f);
#pragma unroll
      for (int i = 0; i < 8; ++i) v[8 * q + i] += f[i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i)
      if (i < nvalid) v[i] += __bfloat162float(b[i]);
  }
}

// Epilogue of one tile for one warp: row `row` of the output (this thread's
// TMEM lane), column chunks of 32 starting at 32 * part, stepping by 64.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t tacc, int g, int nt,
                                              int row, bool valid, int part) {
  uint32_t r[32];
  float v[32];
  if constexpr (EPI == EPI_SWIGLU) {
    const int half = a.bn >> 1;
    const int col0 = nt * a.out_col_step;
    const int ncols = min(half, a.out_cols - col0);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(row) * a.ldo + col0;
    for (int c = 32 * part; c < ncols; c += 64) {
      uint32_t u[32];
      MOE_TMEM_LD32(tacc + c, r);
      MOE_TMEM_LD32(tacc + half + c, u);
      tmem_ld_wait();
      if (!valid) continue;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = silu_fast(__uint_as_float(r[i])) * __uint_as_float(u[i]);
      store_row32_bf16(out + c, v, ncols - c);
    }
  } else {
    const int col0 = nt * a.out_col_step;
    const int ncols = min(a.bn, a.out_cols - col0);
    for (int c = 32 * part; c < ncols; c += 64) {
      MOE_TMEM_LD32(tacc + c, r);
      tmem_ld_wait();
      if (!valid) continue;
      const int nv = min(32, ncols - c);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
      const int col = col0 + c;
      if constexpr (EPI == EPI_STORE_F32 || EPI == EPI_SCALE_BIAS) {
        if constexpr (EPI == EPI_SCALE_BIAS) {
          if (a.bias != nullptr) add_bias32(v, a.bias + static_cast<size_t>(g) * a.out_cols + col, nv);
          const float s = a.row_scale[row];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= s;
        }
        store_row32_f32(static_cast<float*>(a.out) + static_cast<size_t>(row) * a.ldo + col, v, nv,
                        (a.ldo & 3) == 0);
      } else {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(row) * a.ldo + col;
        if constexpr (EPI == EPI_GELU_BIAS) {
          if (a.bias != nullptr) add_bias32(v, a.bias + static_cast<size_t>(g) * a.out_cols + col, nv);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_tanh_fast(v[i]);
        }
        store_row32_bf16(out, v, nv);
      }
    }
  }
}

template <int EPI, int NCTA>
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_b, const GemmArgs args) {
  using C = GemmCfg<NCTA>;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t dyn_smem[];
  __shared__ int s_off[kMaxExperts + 1];
  __shared__ int s_tstart[kMaxExperts + 1];
  __shared__ __align__(8) uint64_t s_full[S];
  __shared__ __align__(8) uint64_t s_empty[S];
  __shared__ __align__(8) uint64_t s_tfull[2];
  __shared__ __align__(8) uint64_t s_tempty[2];
  __shared__ __align__(8) uint64_t s_drain;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;
  __shared__ int s_total;
  __shared__ uint32_t s_kiter_issued;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = NCTA == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit = NCTA == 2 ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = NCTA == 2 ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  const uint32_t smem_base = (smem_addr(dyn_smem) + 1023u) & ~1023u;
  const int G = args.num_groups;

  for (int i = threadIdx.x; i <= G; i += blockDim.x)
    s_off[i] = args.offsets != nullptr ? args.offsets[i] : (i == 0 ? 0 : args.rows);
  __syncthreads();
  if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < G; base += 32) {
      const int g = base + lane;
      int v = 0;
      if (g < G) v = ((s_off[g + 1] - s_off[g] + C::kTileRows - 1) / C::kTileRows) * args.n_tiles;
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
      s_kiter_issued = 0;
      for (int s = 0; s < S; ++s) {
        mbar_init(smem_addr(&s_full[s]), 1);
        mbar_init(smem_addr(&s_empty[s]), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_addr(&s_tfull[b]), 1);
        mbar_init(smem_addr(&s_tempty[b]), kEpiWarps * 32 * NCTA);
      }
      mbar_init(smem_addr(&s_drain), 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
    }
  } else if (warp == 1) {
    if constexpr (NCTA == 2) {
      tmem_alloc_pair(smem_addr(&s_tmem_base), 512);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(smem_addr(&s_tmem_base), 512);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (NCTA == 2) cluster_sync_all();  // peer barriers initialised before any remote use
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int total = s_total;
  const int num_kb = (args.K + kBK - 1) / kBK;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint32_t b_rows_cta = NCTA == 2 ? static_cast<uint32_t>(args.bn >> 1) : static_cast<uint32_t>(args.bn);
      const uint32_t tx_bytes = NCTA * (kATileBytes + b_rows_cta * kBK * 2);
      const uint32_t b_hi_smem = static_cast<uint32_t>((args.bn >> 1) * kBK * 2);
      uint32_t kiter = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += units) {
        int g, mt, nt;
        decode_tile(tile, G, s_tstart, s_off, args.n_tiles, C::kTileRows, g, mt, nt);
        const int a_row = s_off[g] + mt * C::kTileRows + static_cast<int>(rank) * 128;
        const int b_lo = g * args.b_rows_per_group + nt * args.b_row_step;
        const int b_hi = b_lo + args.b_hi_offset;
        for (int kb = 0; kb < num_kb; ++kb, ++kiter) {
          const int s = kiter % S;
          const uint32_t ph = (kiter / S) & 1u;
          if (!mbar_wait(smem_addr(&s_empty[s]), ph ^ 1u, abort_flag, args.status)) { ok = false; break; }
          const uint32_t sa = smem_base + s * C::kStageBytes;
          const uint32_t sb = sa + kATileBytes;
          if constexpr (NCTA == 2) {
            const uint32_t full_leader = mapa_shared(smem_addr(&s_full[s]), 0);
            if (leader) mbar_arrive_expect_tx(smem_addr(&s_full[s]), tx_bytes);
            tma_load_2d_pair(sa, &tmap_a, full_leader, kb * kBK, a_row);
            tma_load_2d_pair(sb, &tmap_b, full_leader, kb * kBK, leader ? b_lo : b_hi);
          } else {
            const uint32_t full = smem_addr(&s_full[s]);
            mbar_arrive_expect_tx(full, tx_bytes);
            tma_load_2d(sa, &tmap_a, full, kb * kBK, a_row);
            tma_load_2d(sb, &tmap_b, full, kb * kBK, b_lo);
            tma_load_2d(sb + b_hi_smem, &tmap_b, full, kb * kBK, b_hi);
          }
          s_kiter_issued = kiter + 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------------ MMA issuer
      uint32_t kiter = 0, it = 0;
      bool ok = true;
      for (int tile = unit; ok && tile < total; tile += units, ++it) {
        const uint32_t buf = it & 1u;
        const uint32_t tph = (it >> 1) & 1u;
        if (!mbar_wait(smem_addr(&s_tempty[buf]), tph ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * 256u;
        for (int kb = 0; kb < num_kb; ++kb, ++kiter) {
          const int s = kiter % S;
          const uint32_t ph = (kiter / S) & 1u;
          if (!mbar_wait(smem_addr(&s_full[s]), ph, abort_flag, args.status)) { ok = false; break; }
          const uint32_t sa = smem_base + s * C::kStageBytes;
          const uint32_t sb = sa + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            if constexpr (NCTA == 2)
              umma_bf16_pair(d_tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32),
                             args.idesc, (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16(d_tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32),
                        args.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          if constexpr (NCTA == 2) umma_commit_pair(smem_addr(&s_empty[s]), 0x3);
          else umma_commit(smem_addr(&s_empty[s]));
        }
        if (!ok) break;
        if constexpr (NCTA == 2) umma_commit_pair(smem_addr(&s_tfull[buf]), 0x3);
        else umma_commit(smem_addr(&s_tfull[buf]));
      }
      // every MMA issued by this thread has completed once s_drain flips
      if constexpr (NCTA == 2) umma_commit_pair(smem_addr(&s_drain), 0x1);
      else umma_commit(smem_addr(&s_drain));
      mbar_wait_drain(smem_addr(&s_drain), 0, kWaitTimeoutNs);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int wq = warp & 3;             // TMEM lane quarter this warp may access
    const int part = (warp - 2) >> 2;    // which column chunks (0 or 1)
    const uint32_t tempty_target0 = NCTA == 2 ? mapa_shared(smem_addr(&s_tempty[0]), 0) : 0u;
    const uint32_t tempty_target1 = NCTA == 2 ? mapa_shared(smem_addr(&s_tempty[1]), 0) : 0u;
    uint32_t it = 0;
    for (int tile = unit; tile < total; tile += units, ++it) {
      int g, mt, nt;
      decode_tile(tile, G, s_tstart, s_off, args.n_tiles, C::kTileRows, g, mt, nt);
      const uint32_t buf = it & 1u;
      const uint32_t tph = (it >> 1) & 1u;
      if (!mbar_wait(smem_addr(&s_tfull[buf]), tph, abort_flag, args.status)) break;
      tc_fence_after();
      const int r_in_tile = static_cast<int>(rank) * 128 + wq * 32 + lane;
      const int seg_rows = s_off[g + 1] - s_off[g];
      const bool valid = mt * C::kTileRows + r_in_tile < seg_rows;
      const int row = s_off[g] + mt * C::kTileRows + r_in_tile;
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + buf * 256u;
      epilogue_tile<EPI>(args, tacc, g, nt, row, valid, part);
      tc_fence_before();
      if constexpr (NCTA == 2) mbar_arrive_remote(buf ? tempty_target1 : tempty_target0);
      else mbar_arrive(smem_addr(&s_tempty[buf]));
    }
  }

  __syncthreads();
  if (s_abort && warp == 0 && lane == 0) {
    // let every TMA load still in flight land before shared memory is released
    if constexpr (NCTA == 2) {
      const uint64_t t0 = globaltimer_ns();
      while (globaltimer_ns() - t0 < 200000ull) {
      }
    } else {
      const uint32_t issued = s_kiter_issued;
      const uint32_t first = issued > S ? issued - S : 0;
      for (uint32_t q = first; q < issued; ++q)
        mbar_wait_drain(smem_addr(&s_full[q % S]), (q / S) & 1u, kWaitTimeoutNs);
    }
  }
  __syncthreads();
  if constexpr (NCTA == 2) cluster_sync_all();  // the peer's MMAs and arrivals are done
  if (warp == 1) {
    tc_fence_after();
    if constexpr (NCTA == 2) tmem_dealloc_pair(tmem_base, 512);
    else tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace moe
