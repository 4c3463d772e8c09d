// Grouped GEMM on the sm_100a tensor cores (tcgen05 + TMEM, fed by TMA).
//
//   out[r, n] = epilogue( sum_k A[r, k] * B[g*b_rows + n', k] )
//
// A is a bf16 [rows, K] matrix whose rows are split into G contiguous
// segments (one per expert: offsets[g] .. offsets[g+1]); B is a bf16 stack of
// per-group [n, K] weight blocks in the nn.Linear [out, in] layout (K-major).
// Both operands are K-major, the natural tcgen05 layout.
//
// One persistent CTA per SM walks a device-side list of 128 x BN output
// tiles (BN <= 256): the list is built in shared memory from offsets[] at
// kernel start, so no host synchronisation is needed to learn the segment
// sizes.  Inside a group tiles are ordered in bands of up to 16 m-tiles, and
// within a band n-tile-major, so that the CTAs working at one time share
// their weight tiles and activation rows through L2.
//
// Warp roles (192 threads):
//   warp 0      TMA producer: A tile 128 x 64 and B tile BN x 64 per stage
//   warp 1      TMEM allocator and MMA issuer (one thread), 128 x BN x 16 MMAs
//   warps 2..5  epilogue: tcgen05.ld of the fp32 accumulator, fused
//               activation / scaling / combine, stores to global
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
  EPI_COMBINE = 4,     // out bf16 = acc + sum_j src[slot_of[r, j], n] (shared down + combine,
                       //            src fp32)
};

constexpr int kBM = 128;
constexpr int kBK = 64;
constexpr int kStages = 4;
constexpr int kATileBytes = kBM * kBK * 2;        // 16 KB
constexpr int kBTileBytes = 256 * kBK * 2;        // 32 KB (BN <= 256)
constexpr int kStageBytes = kATileBytes + kBTileBytes;
constexpr int kGemmDynSmem = kStages * kStageBytes + 1024;
constexpr int kGemmThreads = 192;
constexpr int kBandM = 16;

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
  const float* comb_src;         // EPI_COMBINE: fp32 [*, ldo]
  const int* slot_of;            // EPI_COMBINE: [rows, k]
  int k;
  uint32_t idesc;
  int* status;
};

__device__ __forceinline__ void decode_tile(int tile, int G, const int* s_tstart, const int* s_off,
                                            int n_tiles, int& g, int& mt, int& nt) {
  // last group whose start is <= tile (groups with no tiles have equal starts)
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_tstart[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  g = lo;
  const int local = tile - s_tstart[g];
  const int mtiles = (s_off[g + 1] - s_off[g] + kBM - 1) / kBM;
  const int band = local / (kBandM * n_tiles);
  const int rem = local - band * kBandM * n_tiles;
  const int bm = min(kBandM, mtiles - band * kBandM);
  nt = rem / bm;
  mt = band * kBandM + (rem - nt * bm);
}

__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16* dst, const float* v, int nvalid) {
  if (nvalid >= 32) {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d4[q] = f32_to_bf16x8(v + 8 * q);
  } else {
    for (int i = 0; i < nvalid; ++i) dst[i] = __float2bfloat16_rn(v[i]);
  }
}

template <int EPI>
__device__ __forceinline__ void epilogue_tile(const GemmArgs& a, uint32_t tacc, int g, int nt,
                                              int row, bool valid) {
  uint32_t r[32];
  float v[32];
  if constexpr (EPI == EPI_SWIGLU) {
    const int half = a.bn >> 1;
    const int col0 = nt * a.out_col_step;
    const int ncols = min(half, a.out_cols - col0);
    __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(row) * a.ldo + col0;
    for (int c = 0; c < ncols; c += 32) {
      uint32_t u[32];
      MOE_TMEM_LD32(tacc + c, r);
      MOE_TMEM_LD32(tacc + half + c, u);
      tmem_ld_wait();
      if (!valid) continue;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = silu_f(__uint_as_float(r[i])) * __uint_as_float(u[i]);
      store_row32_bf16(out + c, v, ncols - c);
    }
  } else {
    const int col0 = nt * a.out_col_step;
    const int ncols = min(a.bn, a.out_cols - col0);
    for (int c = 0; c < ncols; c += 32) {
      MOE_TMEM_LD32(tacc + c, r);
      tmem_ld_wait();
      if (!valid) continue;
      const int nv = min(32, ncols - c);
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
      const int col = col0 + c;
      if constexpr (EPI == EPI_STORE_F32 || EPI == EPI_SCALE_BIAS) {
        if constexpr (EPI == EPI_SCALE_BIAS) {
          if (a.bias != nullptr) {
            const __nv_bfloat16* b = a.bias + static_cast<size_t>(g) * a.out_cols + col;
            for (int i = 0; i < nv; ++i) v[i] += __bfloat162float(b[i]);
          }
          const float s = a.row_scale[row];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= s;
        }
        float* out = static_cast<float*>(a.out) + static_cast<size_t>(row) * a.ldo + col;
        if (nv == 32 && (a.ldo & 3) == 0) {
          float4* o4 = reinterpret_cast<float4*>(out);
#pragma unroll
          for (int q = 0; q < 8; ++q) o4[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        } else {
          for (int i = 0; i < nv; ++i) out[i] = v[i];
        }
      } else {
        __nv_bfloat16* out = static_cast<__nv_bfloat16*>(a.out) + static_cast<size_t>(row) * a.ldo + col;
        if constexpr (EPI == EPI_GELU_BIAS) {
          if (a.bias != nullptr) {
            const __nv_bfloat16* b = a.bias + static_cast<size_t>(g) * a.out_cols + col;
            for (int i = 0; i < nv; ++i) v[i] += __bfloat162float(b[i]);
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_tanh(v[i]);
        }
        if constexpr (EPI == EPI_COMBINE) {
          float acc[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) acc[i] = 0.0f;
          for (int j = 0; j < a.k; ++j) {
            const int slot = a.slot_of[static_cast<size_t>(row) * a.k + j];
            const float* src = a.comb_src + static_cast<size_t>(slot) * a.ldo + col;
            if (nv == 32) {
              const float4* s4 = reinterpret_cast<const float4*>(src);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 f = s4[q];
                acc[4 * q] += f.x;
                acc[4 * q + 1] += f.y;
                acc[4 * q + 2] += f.z;
                acc[4 * q + 3] += f.w;
              }
            } else {
              for (int i = 0; i < nv; ++i) acc[i] += src[i];
            }
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = acc[i] + v[i];
        }
        store_row32_bf16(out, v, nv);
      }
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
    moe_gemm_sm100_kernel(const __grid_constant__ CUtensorMap tmap_a,
                          const __grid_constant__ CUtensorMap tmap_b, const GemmArgs args) {
  extern __shared__ uint8_t dyn_smem[];
  __shared__ int s_off[kMaxExperts + 1];
  __shared__ int s_tstart[kMaxExperts + 1];
  __shared__ __align__(8) uint64_t s_full[kStages];
  __shared__ __align__(8) uint64_t s_empty[kStages];
  __shared__ __align__(8) uint64_t s_tfull[2];
  __shared__ __align__(8) uint64_t s_tempty[2];
  __shared__ __align__(8) uint64_t s_drain;
  __shared__ uint32_t s_tmem_base;
  __shared__ int s_abort;
  __shared__ int s_total;
  __shared__ uint32_t s_kiter_issued;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
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
      if (g < G) v = ((s_off[g + 1] - s_off[g] + kBM - 1) / kBM) * args.n_tiles;
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
      for (int s = 0; s < kStages; ++s) {
        mbar_init(smem_addr(&s_full[s]), 1);
        mbar_init(smem_addr(&s_empty[s]), 1);
      }
      for (int b = 0; b < 2; ++b) {
        mbar_init(smem_addr(&s_tfull[b]), 1);
        mbar_init(smem_addr(&s_tempty[b]), 128);
      }
      mbar_init(smem_addr(&s_drain), 1);
      fence_mbar_init();
      tma_prefetch_desc(&tmap_a);
      tma_prefetch_desc(&tmap_b);
    }
  } else if (warp == 1) {
    tmem_alloc(smem_addr(&s_tmem_base), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  const uint32_t tmem_base = s_tmem_base;
  const int total = s_total;
  const int num_kb = (args.K + kBK - 1) / kBK;
  volatile int* abort_flag = &s_abort;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      const uint32_t tx_bytes = static_cast<uint32_t>((kBM + args.bn) * kBK * 2);
      const uint32_t b_hi_smem = static_cast<uint32_t>((args.bn >> 1) * kBK * 2);
      uint32_t kiter = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x) {
        int g, mt, nt;
        decode_tile(tile, G, s_tstart, s_off, args.n_tiles, g, mt, nt);
        const int a_row = s_off[g] + mt * kBM;
        const int b_lo = g * args.b_rows_per_group + nt * args.b_row_step;
        const int b_hi = b_lo + args.b_hi_offset;
        for (int kb = 0; kb < num_kb; ++kb, ++kiter) {
          const int s = kiter % kStages;
          const uint32_t ph = (kiter / kStages) & 1u;
          if (!mbar_wait(smem_addr(&s_empty[s]), ph ^ 1u, abort_flag, args.status)) { ok = false; break; }
          const uint32_t full = smem_addr(&s_full[s]);
          mbar_arrive_expect_tx(full, tx_bytes);
          const uint32_t sa = smem_base + s * kStageBytes;
          const uint32_t sb = sa + kATileBytes;
          tma_load_2d(sa, &tmap_a, full, kb * kBK, a_row);
          tma_load_2d(sb, &tmap_b, full, kb * kBK, b_lo);
          tma_load_2d(sb + b_hi_smem, &tmap_b, full, kb * kBK, b_hi);
          s_kiter_issued = kiter + 1;
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------ MMA issuer
      uint32_t kiter = 0, it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < total; tile += gridDim.x, ++it) {
        const uint32_t buf = it & 1u;
        const uint32_t tph = (it >> 1) & 1u;
        if (!mbar_wait(smem_addr(&s_tempty[buf]), tph ^ 1u, abort_flag, args.status)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + buf * 256u;
        for (int kb = 0; kb < num_kb; ++kb, ++kiter) {
          const int s = kiter % kStages;
          const uint32_t ph = (kiter / kStages) & 1u;
          if (!mbar_wait(smem_addr(&s_full[s]), ph, abort_flag, args.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_base + s * kStageBytes;
          const uint32_t sb = sa + kATileBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            umma_bf16(d_tmem, sw128_kmajor_desc(sa + kk * 32), sw128_kmajor_desc(sb + kk * 32),
                      args.idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(smem_addr(&s_empty[s]));
        }
        if (!ok) break;
        umma_commit(smem_addr(&s_tfull[buf]));
      }
      // every MMA issued by this thread has completed once s_drain flips
      umma_commit(smem_addr(&s_drain));
      mbar_wait_drain(smem_addr(&s_drain), 0, kWaitTimeoutNs);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------- epilogue
    const int wq = warp & 3;  // TMEM lane quarter this warp may access
    uint32_t it = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x, ++it) {
      int g, mt, nt;
      decode_tile(tile, G, s_tstart, s_off, args.n_tiles, g, mt, nt);
      const uint32_t buf = it & 1u;
      const uint32_t tph = (it >> 1) & 1u;
      if (!mbar_wait(smem_addr(&s_tfull[buf]), tph, abort_flag, args.status)) break;
      tc_fence_after();
      const int r_in_tile = wq * 32 + lane;
      const int seg_rows = s_off[g + 1] - s_off[g];
      const bool valid = mt * kBM + r_in_tile < seg_rows;
      const int row = s_off[g] + mt * kBM + r_in_tile;
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + buf * 256u;
      epilogue_tile<EPI>(args, tacc, g, nt, row, valid);
      tc_fence_before();
      mbar_arrive(smem_addr(&s_tempty[buf]));
    }
  }

  __syncthreads();
  if (s_abort && warp == 0 && lane == 0) {
    // let every TMA load still in flight land before shared memory is released
    const uint32_t issued = s_kiter_issued;
    const uint32_t first = issued > kStages ? issued - kStages : 0;
    for (uint32_t q = first; q < issued; ++q)
      mbar_wait_drain(smem_addr(&s_full[q % kStages]), (q / kStages) & 1u, kWaitTimeoutNs);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace moe
