// Grouped expert GEMMs on the 5th-generation tensor cores (tcgen05 + TMEM, TMA-fed).
//
// Each Beam expert is a SwiGLU MLP, y = W_down (silu(W_gate x) * (W_up x)), with BF16 weights,
// intermediate size 2560 and the activation in FP32 (Transformers model doc "Beam", Overview;
// BeamConfig moe_intermediate_size; news article "Reflection lança o Beam", "cada expert é um
// MLP SwiGLU").  Rows of Xp are grouped by expert (see dispatch.cu); an m-tile is up to 128
// rows of one expert.
//
//   GEMM1 (gate|up + SwiGLU): for each m-tile and each 128-column slice n of I,
//       D[128 x 256] = Xp[rows, :] . [W_gate,e[n-slice, :] ; W_up,e[n-slice, :]]^T
//       act[rows, n-slice] = bf16( silu(D[:, 0:128]) * D[:, 128:256] )
//   GEMM2 (down): for each m-tile and each 256-column slice n of d,
//       Y[rows, n-slice] = bf16( act[rows, :] . W_down,e[n-slice, :]^T )
//
// An m-tile of at most 64 rows issues M = 64 MMAs (accumulator rows in lanes 0..15 of each
// 32-lane quarter of TMEM), so absent rows cost no tensor-core work.
//
// Kernel structure (persistent, one CTA per SM, 192 threads):
//   warp 0     one thread issues TMA loads of the A (token rows) and B (weight) tiles into a
//              4-stage ring; the A load covers only the tile's rows (16/32/64/128-row boxes)
//   warp 1     allocates 512 TMEM columns; one thread issues tcgen05.mma (M=128, N=256,
//              K=16, BF16 -> FP32) into one of two 256-column accumulators and commits
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (each warp owns its 32-lane quarter),
//              FP32 SwiGLU / conversion to BF16, 16-byte stores; the accumulator is then
//              released so the MMA of the next tile overlaps this epilogue
// Tiles are visited band by band (each m-tile names its raster band: whole experts of up to
// 2 kBand - 1 m-tiles, see dispatch.cu), slice-major inside a band, so the CTAs running at the
// same time share A rows and weight slices through L2 and no expert's weights are streamed
// from HBM twice because its m-tiles fell into two bands.
//
// In calls where nearly every m-tile is tiny (decode sizes: a few rows per expert), a tile with
// at most swap_max_rows rows swaps the operand roles: the two 128-row halves of the weight tile become M and the
// tile's rows, padded to a multiple of 16, become N:
//       D_lo[128 x Np] = W[0:128, :] . X^T,   D_hi[128 x Np] = W[128:256, :] . X^T
// so the MMA work follows the rows that exist instead of a full 128-row tile.  The same shared
// memory stage serves both forms; the epilogue then owns one weight row per thread and writes
// one value per token row.
//
// Every wait is bounded (globaltimer); on a timeout the kernel records it in the workspace
// status word, raises a CTA-wide abort flag, waits for its own TMA loads and MMAs to finish,
// frees TMEM and returns.
#include "beam_moe_internal.cuh"

namespace beam {
namespace {

constexpr uint64_t kMinDrainNs = 1000000000ull;  // drains always get at least 1 s

__device__ __forceinline__ MTile load_tile(const GemmArgs& a, int t, int n_tiles, int& n) {
  int mt;
  band_decode_tile(a.mtiles, t, n_tiles, mt, n);
  return a.mtiles[mt];
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// SiLU with the fast reciprocal division (about two ulp): the epilogue's arithmetic is on the
// critical path when the K loop is short (E4M3 operands), and the result is rounded to BF16.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// FP8 epilogue: v0[j] *= sa * s0[j] and, when s1 is given, v1[j] *= sa * s1[j], for 32
// consecutive columns (s0, s1 16-byte aligned; the same addresses across the warp).
__device__ __forceinline__ void scale_columns(uint32_t (&v0)[32], uint32_t (&v1)[32], float sa,
                                              const float* s0, const float* s1) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 a4 = reinterpret_cast<const float4*>(s0)[q];
    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) v0[4 * q + i] = __float_as_uint(__uint_as_float(v0[4 * q + i]) * sa * av[i]);
    if (s1) {
      const float4 b4 = reinterpret_cast<const float4*>(s1)[q];
      const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) v1[4 * q + i] = __float_as_uint(__uint_as_float(v1[4 * q + i]) * sa * bv[i]);
    }
  }
}

template <bool kSwiGLU, bool kSwap, bool kFp8>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_kernel(const __grid_constant__ ATensorMaps tmA,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // 128-byte swizzle atoms need 1 KB alignment
  uint8_t* smem = smem_raw + (sbase - raw);
  // [kStages x (A 16 KB | B 32 KB)][barriers][TMEM address][abort flag]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  constexpr int kBarFull = 0, kBarEmpty = kStages, kBarTFull = 2 * kStages,
                kBarTEmpty = kBarTFull + 2, kBarDrain = kBarTEmpty + 2, kNumBars = kBarDrain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = *a.mt_count;
  const int n_tiles = a.n_tiles_n;
  const int ntiles = m_tiles * n_tiles;
  if (static_cast<int>(blockIdx.x) >= ntiles) return;  // uniform over the CTA
  const uint64_t limit = a.wait_limit_ns;
  const uint64_t drain_limit = limit > kMinDrainNs ? limit : kMinDrainNs;
  constexpr int kNSlice = kSwiGLU ? kN1Half : kN2;
  constexpr int kKElems = kFp8 ? 2 * kBK : kBK;  // K elements in one 128-byte stage row

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarTFull + i), 1);
      mbar_init(bar(kBarTEmpty + i), 4);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kNumABoxes; ++i) tma_prefetch_desc(&tmA.m[i]);
    tma_prefetch_desc(&tmB0);
    if (kSwiGLU) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, filled = 0, last_parity = 0;
      bool ok = true;
      // the next tile's descriptor is loaded one tile ahead, off the critical path
      int n = 0;
      MTile m = load_tile(a, blockIdx.x, n_tiles, n);
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int n_next = 0;
        const MTile m_next = load_tile(a, t + gridDim.x < ntiles ? t + gridDim.x : t,
                                       n_tiles, n_next);
        const int brow = m.e * a.b_rows_per_expert + n * kNSlice;
        // rows of A beyond the box are left from earlier stages: they only feed accumulator
        // rows that are never stored
        const int a_box = a_box_for_rows(m.nrows);
        const uint32_t a_bytes = static_cast<uint32_t>(a_box_rows(a_box)) * kBK * 2;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kBarEmpty + stage), phase ^ 1u, abort_flag, limit, a.status,
                                 kWhereProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint32_t sB = sA + kStageABytes;
          const uint32_t fb = bar(kBarFull + stage);
          mbar_arrive_expect_tx(fb, a_bytes + kStageBBytes);
          tma_load_2d(sA, &tmA.m[a_box], fb, kb * kKElems, m.row0);
          tma_load_2d(sB, &tmB0, fb, kb * kKElems, brow);
          if (kSwiGLU) tma_load_2d(sB + kStageBBytes / 2, &tmB1, fb, kb * kKElems, brow);
          filled |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        m = m_next;
        n = n_next;
      }
      // every load this thread issued must land before the CTA may exit
      int no_abort = 0;
      for (int s = 0; s < kStages; ++s)
        if ((filled >> s) & 1u)
          mbar_wait_bounded(bar(kBarFull + s), (last_parity >> s) & 1u, &no_abort, drain_limit,
                            a.status, kWhereDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      auto make_idesc = [](int M, int N) {
        return kFp8 ? umma_idesc_e4m3_f32(M, N) : umma_idesc_bf16_f32(M, N);
      };
      // one MMA covers 32 bytes of K: 16 BF16 or 32 E4M3 elements
      auto mma = [](uint32_t d, uint64_t ad, uint64_t bd, uint32_t id, uint32_t acc) {
        if constexpr (kFp8)
          umma_e4m3(d, ad, bd, id, acc);
        else
          umma_bf16(d, ad, bd, id, acc);
      };
      const uint32_t idesc_full = make_idesc(kBM, kUmmaN);
      // tiles of at most 64 rows use M = 64: half the datapath lanes, no work on absent rows
      const uint32_t idesc_m64 = make_idesc(64, kUmmaN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      int n_unused = 0;
      int nrows = load_tile(a, blockIdx.x, n_tiles, n_unused).nrows;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int nrows_next = load_tile(a, t + gridDim.x < ntiles ? t + gridDim.x : t,
                                         n_tiles, n_unused).nrows;
        const bool swap = kSwap && nrows <= a.swap_max_rows;
        const uint32_t idesc = swap ? make_idesc(kBM, (nrows + 15) & ~15)
                               : nrows <= 64 ? idesc_m64 : idesc_full;
        if (!mbar_wait_bounded(bar(kBarTEmpty + acc), acc_phase ^ 1u, abort_flag, limit, a.status,
                               kWhereMmaTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kUmmaN);
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kBarFull + stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint64_t adesc = smem_desc_k_sw128(sA);
          const uint64_t bdesc = smem_desc_k_sw128(sA + kStageABytes);
          if (swap) {
            const uint64_t bdesc_hi = smem_desc_k_sw128(sA + kStageABytes + kStageBBytes / 2);
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k) {
              const uint32_t accum = (kb | k) != 0 ? 1u : 0u;
              mma(d_tmem, bdesc + 2u * k, adesc + 2u * k, idesc, accum);
              mma(d_tmem + 128u, bdesc_hi + 2u * k, adesc + 2u * k, idesc, accum);
            }
          } else {
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k)  // +32 bytes along K per step: +2 in addr>>4
              mma(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(bar(kBarEmpty + stage));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(bar(kBarTFull + acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        nrows = nrows_next;
      }
      // all MMAs this thread issued must complete before TMEM is freed
      int no_abort = 0;
      umma_commit(bar(kBarDrain));
      mbar_wait_bounded(bar(kBarDrain), 0, &no_abort, drain_limit, a.status, kWhereDrain);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access (warps 2..5)
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int mt, n;
      band_decode_tile(a.mtiles, t, n_tiles, mt, n);
      const MTile m = a.mtiles[mt];
      int ok = 0;
      if (lane == 0)
        ok = mbar_wait_bounded(bar(kBarTFull + acc), acc_phase, abort_flag, limit, a.status,
                               kWhereEpiTmemFull);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      // the phase has completed: each lane observes it (returns at once)
      ok = mbar_wait_bounded(bar(kBarTFull + acc), acc_phase, abort_flag, limit, a.status,
                             kWhereEpiTmemFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();

      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * kUmmaN);
      if (kSwap && m.nrows <= a.swap_max_rows) {
        // weights-as-M tile: this thread owns weight row `row` of each 128-row half; TMEM
        // column j holds token row j of the tile
        const int npad = (m.nrows + 15) & ~15;
        __nv_bfloat16* base = a.out + static_cast<size_t>(m.row0) * a.out_ld + n * kNSlice + row;
        // FP8: this thread's weight rows (gate and up of one column, or two down columns)
        float sb_lo = 1.f, sb_hi = 1.f;
        if constexpr (kFp8) {
          const int64_t brow = static_cast<int64_t>(m.e) * a.b_rows_per_expert + n * kNSlice + row;
          sb_lo = a.b_scale0[brow];
          sb_hi = kSwiGLU ? a.b_scale1[brow] : a.b_scale0[brow + 128];
        }
#pragma unroll 1
        for (int c0 = 0; c0 < npad; c0 += 16) {
          uint32_t lo[16], hi[16];
          tmem_ld16_sync(tb + c0, lo);
          tmem_ld16_sync(tb + 128 + c0, hi);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int r = c0 + j;
            if (r < m.nrows) {
              __nv_bfloat16* o = base + static_cast<size_t>(r) * a.out_ld;
              float vlo = __uint_as_float(lo[j]), vhi = __uint_as_float(hi[j]);
              if constexpr (kFp8) {
                const float sa = a.a_scale[m.row0 + r];
                vlo = vlo * sa * sb_lo;
                vhi = vhi * sa * sb_hi;
              }
              if (kSwiGLU) {
                o[0] = __float2bfloat16_rn(silu(vlo) * vhi);
              } else {
                o[0] = __float2bfloat16_rn(vlo);
                o[128] = __float2bfloat16_rn(vhi);
              }
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(kBarTEmpty + acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
        continue;
      }
      // M = 128: accumulator row r sits in TMEM lane r.  M = 64 (tiles of at most 64 rows):
      // row r sits in lane (r % 16) + 32 * (r / 16), i.e. lanes 0..15 of each warp's quarter.
      const int trow = m.nrows <= 64 ? (lane < 16 ? q * 16 + lane : kBM) : row;
      const bool valid = trow < m.nrows;
      __nv_bfloat16* dst =
          a.out + static_cast<size_t>(m.row0 + (valid ? trow : 0)) * a.out_ld + n * kNSlice;
      // FP8: this row's scale and the first weight row of the slice
      float sa = 1.f;
      int64_t brow0 = 0;
      if constexpr (kFp8) {
        sa = valid ? a.a_scale[m.row0 + trow] : 0.f;
        brow0 = static_cast<int64_t>(m.e) * a.b_rows_per_expert + n * kNSlice;
      }
      if (kSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < kN1Half; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32_sync(tb + c, g);
          tmem_ld32_sync(tb + kN1Half + c, u);
          if constexpr (kFp8) scale_columns(g, u, sa, a.b_scale0 + brow0 + c, a.b_scale1 + brow0 + c);
          uint32_t p[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float h0 = silu(__uint_as_float(g[2 * j])) * __uint_as_float(u[2 * j]);
            const float h1 = silu(__uint_as_float(g[2 * j + 1])) * __uint_as_float(u[2 * j + 1]);
            p[j] = pack_bf16x2(h0, h1);
          }
          if (valid) {
            uint4* o = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) o[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < kN2; c += 32) {
          uint32_t y[32];
          tmem_ld32_sync(tb + c, y);
          if constexpr (kFp8) scale_columns(y, y, sa, a.b_scale0 + brow0 + c, nullptr);
          uint32_t p[16];
#pragma unroll
          for (int j = 0; j < 16; ++j)
            p[j] = pack_bf16x2(__uint_as_float(y[2 * j]), __uint_as_float(y[2 * j + 1]));
          if (valid) {
            uint4* o = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int v = 0; v < 4; ++v) o[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarTEmpty + acc));
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t prepare_gemm_kernels() {
  const void* kernels[] = {reinterpret_cast<const void*>(expert_gemm_kernel<true, false, false>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<true, true, false>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<false, false, false>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<false, true, false>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<true, false, true>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<true, true, true>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<false, false, true>),
                           reinterpret_cast<const void*>(expert_gemm_kernel<false, true, true>)};
  for (const void* k : kernels) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

namespace {
template <bool kSwiGLU, bool kFp8>
void launch_gemm(const ATensorMaps& tmA, const CUtensorMap& tmB0, const CUtensorMap& tmB1,
                 const GemmArgs& a, int grid, cudaStream_t s) {
  if (a.swap_max_rows > 0)
    expert_gemm_kernel<kSwiGLU, true, kFp8>
        <<<grid, kGemmThreads, kGemmSmemBytes, s>>>(tmA, tmB0, tmB1, a);
  else
    expert_gemm_kernel<kSwiGLU, false, kFp8>
        <<<grid, kGemmThreads, kGemmSmemBytes, s>>>(tmA, tmB0, tmB1, a);
}
}  // namespace

cudaError_t launch_gemm_gate_up(const ATensorMaps& tmA, const CUtensorMap& tmG,
                                const CUtensorMap& tmU, const GemmArgs& a, int grid,
                                cudaStream_t s, bool fp8) {
  if (fp8)
    launch_gemm<true, true>(tmA, tmG, tmU, a, grid, s);
  else
    launch_gemm<true, false>(tmA, tmG, tmU, a, grid, s);
  return cudaGetLastError();
}

cudaError_t launch_gemm_down(const ATensorMaps& tmA, const CUtensorMap& tmD, const GemmArgs& a,
                             int grid, cudaStream_t s, bool fp8) {
  if (fp8)
    launch_gemm<false, true>(tmA, tmD, tmD, a, grid, s);
  else
    launch_gemm<false, false>(tmA, tmD, tmD, a, grid, s);
  return cudaGetLastError();
}

}  // namespace beam
