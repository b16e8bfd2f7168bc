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
// Kernel structure (persistent, one CTA per SM, 192 threads):
//   warp 0     one thread issues TMA loads of the A and B tiles into a 4-stage ring
//   warp 1     allocates 512 TMEM columns; one thread issues tcgen05.mma (M=128, N=256,
//              K=16, BF16 -> FP32) into one of two 256-column accumulators and commits
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (each warp owns its 32-lane quarter),
//              FP32 SwiGLU / conversion to BF16, 16-byte stores; the accumulator is then
//              released so the MMA of the next tile overlaps this epilogue
// Tiles are visited in bands of kBand m-tiles, slice-major inside a band, so the CTAs running
// at the same time share A rows and weight slices through L2.
//
// Every wait is bounded (globaltimer); on a timeout the kernel records it in the workspace
// status word, raises a CTA-wide abort flag, waits for its own TMA loads and MMAs to finish,
// frees TMEM and returns.
#include "beam_moe_internal.cuh"

namespace beam {
namespace {

constexpr uint64_t kMinDrainNs = 1000000000ull;  // drains always get at least 1 s

__device__ __forceinline__ void decode_tile(int t, int m_tiles, int n_tiles, int& mt, int& n) {
  const int band_tiles = kBand * n_tiles;
  const int band = t / band_tiles;
  const int base = band * kBand;
  const int gm = min(kBand, m_tiles - base);
  const int r = t - band * band_tiles;
  n = r / gm;
  mt = base + (r - n * gm);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float silu(float g) { return g / (1.0f + __expf(-g)); }

template <bool kSwiGLU>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_kernel(const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB0,
                       const __grid_constant__ CUtensorMap tmB1, const GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;  // 128-byte swizzle atoms need 1 KB alignment
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + kStages + s); };
  auto tfull_bar = [&](int i) { return smem_u32(bars + 2 * kStages + i); };
  auto tempty_bar = [&](int i) { return smem_u32(bars + 2 * kStages + 2 + i); };
  const uint32_t drain_bar = smem_u32(bars + 2 * kStages + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = *a.mt_count;
  const int n_tiles = a.n_tiles_n;
  const int ntiles = m_tiles * n_tiles;
  if (static_cast<int>(blockIdx.x) >= ntiles) return;  // uniform over the CTA
  const uint64_t limit = a.wait_limit_ns;
  const uint64_t drain_limit = limit > kMinDrainNs ? limit : kMinDrainNs;
  constexpr int kNSlice = kSwiGLU ? kN1Half : kN2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(tfull_bar(i), 1);
      mbar_init(tempty_bar(i), 4);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
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
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int mt, n;
        decode_tile(t, m_tiles, n_tiles, mt, n);
        const MTile m = a.mtiles[mt];
        const int brow = m.e * a.b_rows_per_expert + n * kNSlice;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, limit, a.status,
                                 kWhereProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint32_t sB = sA + kStageABytes;
          mbar_arrive_expect_tx(full_bar(stage), kStageBytes);
          tma_load_2d(sA, &tmA, full_bar(stage), kb * kBK, m.row0);
          if (kSwiGLU) {
            tma_load_2d(sB, &tmB0, full_bar(stage), kb * kBK, brow);
            tma_load_2d(sB + kStageBBytes / 2, &tmB1, full_bar(stage), kb * kBK, brow);
          } else {
            tma_load_2d(sB, &tmB0, full_bar(stage), kb * kBK, brow);
          }
          filled |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every load this thread issued must land before the CTA may exit
      int no_abort = 0;
      for (int s = 0; s < kStages; ++s)
        if ((filled >> s) & 1u)
          mbar_wait_bounded(full_bar(s), (last_parity >> s) & 1u, &no_abort, drain_limit,
                            a.status, kWhereDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kBM, kUmmaN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(tempty_bar(acc), acc_phase ^ 1u, abort_flag, limit, a.status,
                               kWhereMmaTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kUmmaN);
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(full_bar(stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * kStageBytes;
          const uint64_t adesc = smem_desc_k_sw128(sA);
          const uint64_t bdesc = smem_desc_k_sw128(sA + kStageABytes);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)  // +32 bytes along K per step: +2 in addr>>4
            umma_bf16(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit(empty_bar(stage));
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(tfull_bar(acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // all MMAs this thread issued must complete before TMEM is freed
      int no_abort = 0;
      umma_commit(drain_bar);
      mbar_wait_bounded(drain_bar, 0, &no_abort, drain_limit, a.status, kWhereDrain);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
      int mt, n;
      decode_tile(t, m_tiles, n_tiles, mt, n);
      const MTile m = a.mtiles[mt];
      int ok = 0;
      if (lane == 0)
        ok = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort_flag, limit, a.status,
                               kWhereEpiTmemFull);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      // the phase has completed: each lane observes it (returns at once)
      ok = mbar_wait_bounded(tfull_bar(acc), acc_phase, abort_flag, limit, a.status,
                             kWhereEpiTmemFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();

      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * kUmmaN);
      const bool valid = row < m.nrows;
      __nv_bfloat16* dst =
          a.out + static_cast<size_t>(m.row0 + (valid ? row : 0)) * a.out_ld + n * kNSlice;
      if (kSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < kN1Half; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32_sync(tb + c, g);
          tmem_ld32_sync(tb + kN1Half + c, u);
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
      if (lane == 0) mbar_arrive(tempty_bar(acc));
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
  cudaError_t e = cudaFuncSetAttribute(expert_gemm_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(expert_gemm_kernel<false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes);
}

cudaError_t launch_gemm_gate_up(const CUtensorMap& tmA, const CUtensorMap& tmG,
                                const CUtensorMap& tmU, const GemmArgs& a, int grid,
                                cudaStream_t s) {
  expert_gemm_kernel<true><<<grid, kGemmThreads, kGemmSmemBytes, s>>>(tmA, tmG, tmU, a);
  return cudaGetLastError();
}

cudaError_t launch_gemm_down(const CUtensorMap& tmA, const CUtensorMap& tmD, const GemmArgs& a,
                             int grid, cudaStream_t s) {
  expert_gemm_kernel<false><<<grid, kGemmThreads, kGemmSmemBytes, s>>>(tmA, tmD, tmD, a);
  return cudaGetLastError();
}

}  // namespace beam
