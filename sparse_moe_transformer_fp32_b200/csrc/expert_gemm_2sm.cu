// Grouped expert GEMMs on SM pairs (tcgen05 cta_group::2), for calls with many rows per expert.
//
// Same computation as expert_gemm.cu (gate|up with the FP32 SwiGLU epilogue, then down), but a
// cluster of two CTAs on two SMs computes one 256 x 256 accumulator tile per K loop with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16):
//   - m-tiles are 256 rows of one expert; CTA rank r owns rows 128 r .. 128 r + 127 (its A tile,
//     and the accumulator rows in its own TMEM);
//   - the 256-row weight tile is split between the pair: rank 0 loads rows 0..127 (the gate
//     slice, or the first half of a down slice), rank 1 rows 128..255 (the up slice), and the
//     MMA reads both halves from the two SMs' shared memory;
// so each SM streams 16 KB of A and 16 KB of B per 64-deep K step for the same tensor work that
// costs a single-SM tile 48 KB, and the ring is 6 stages deep.
//
// Synchronisation (one producer thread per CTA, one MMA thread in rank 0, four epilogue warps
// per CTA):
//   full[s]   rank 0 only; rank 0's producer arms it with both CTAs' bytes, and both CTAs' TMA
//             loads (.cta_group::2) complete on it;
//   empty[s]  both CTAs; released by rank 0's MMA commit multicast to the pair;
//   tfull[a]  both CTAs; rank 0's commit multicast when accumulator a is complete;
//   tempty[a] rank 0 only, 8 arrivals: the four epilogue warps of each CTA (rank 1's remotely).
// Every wait is bounded as in the single-SM kernel.
#include "beam_moe_internal.cuh"

namespace beam {
namespace {

constexpr int k2Stages = 6;
constexpr int k2StageA = kBM * kBK * 2;          // 16 KB: this CTA's 128 rows
constexpr int k2StageB = 128 * kBK * 2;          // 16 KB: this CTA's half of the weight tile
constexpr int k2StageBytes = k2StageA + k2StageB;
constexpr int k2SmemBytes = k2Stages * k2StageBytes + 1024 + 1024;
constexpr uint64_t k2MinDrainNs = 1000000000ull;

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
// shared::cluster address of the same shared-memory offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                                 int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrives on barrier `bar` (same offset) in every CTA of `mask` when this thread's earlier
// tcgen05 operations have completed.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void decode_tile2(int t, int m_tiles, int n_tiles, int& mt, int& n) {
  const int band_tiles = kBand * n_tiles;
  const int band = t / band_tiles;
  const int base = band * kBand;
  const int gm = min(kBand, m_tiles - base);
  const int r = t - band * band_tiles;
  n = r / gm;
  mt = base + (r - n * gm);
}

__device__ __forceinline__ uint32_t pack_bf16x2_2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float silu2(float g) { return g / (1.0f + __expf(-g)); }

template <bool kSwiGLU>
__global__ void __launch_bounds__(kGemmThreads, 1)
    expert_gemm_2sm_kernel(const __grid_constant__ ATensorMaps tmA,
                           const __grid_constant__ CUtensorMap tmB0,
                           const __grid_constant__ CUtensorMap tmB1, const GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + k2Stages * k2StageBytes);
  constexpr int kFull = 0, kEmpty = k2Stages, kTFull = 2 * k2Stages, kTEmpty = kTFull + 2,
                kDrain = kTEmpty + 2, kNumBars = kDrain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // This kernel needs its cluster of two; any other launch does nothing but report.
  if (cluster_nctarank() != 2) {
    if (threadIdx.x == 0) record_status(a.status, kDevAssert, kWhereDrain);
    return;
  }
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int npairs = static_cast<int>(gridDim.x >> 1);
  const int m_tiles = *a.mt_count;
  const int n_tiles = a.n_tiles_n;
  const int ntiles = m_tiles * n_tiles;
  if (pair >= ntiles) return;  // uniform over the pair
  const uint64_t limit = a.wait_limit_ns;
  const uint64_t drain_limit = limit > k2MinDrainNs ? limit : k2MinDrainNs;
  constexpr int kNSlice = kSwiGLU ? kN1Half : kN2;  // output columns of a tile's weight rows

  if (threadIdx.x == 0) {
    for (int s = 0; s < k2Stages; ++s) {
      mbar_init(bar(kFull + s), 1);
      mbar_init(bar(kEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kTFull + i), 1);
      mbar_init(bar(kTEmpty + i), 8);
    }
    mbar_init(bar(kDrain), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kNumABoxes; ++i) tma_prefetch_desc(&tmA.m[i]);
    tma_prefetch_desc(&tmB0);
    if (kSwiGLU) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncwarp();    // the cluster barrier is warp-aligned
  cluster_sync();  // barriers of both CTAs initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, filled = 0, last_parity = 0;
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs) {
        int mt, n;
        decode_tile2(t, m_tiles, n_tiles, mt, n);
        const MTile m = a.mtiles[mt];
        const int rows0 = min(m.nrows, kBM);
        const int rows1 = m.nrows - rows0;
        const int my_rows = leader ? rows0 : rows1;
        const int my_box = a_box_for_rows(my_rows > 0 ? my_rows : 1);
        const uint32_t my_a_bytes =
            my_rows > 0 ? static_cast<uint32_t>(a_box_rows(my_box)) * kBK * 2 : 0u;
        const uint32_t peer_a_bytes =
            rows1 > 0 ? static_cast<uint32_t>(a_box_rows(a_box_for_rows(rows1))) * kBK * 2 : 0u;
        // this CTA's half of the weight tile: rank 0 the first 128 rows, rank 1 the next 128
        const CUtensorMap* bmap = kSwiGLU ? (leader ? &tmB0 : &tmB1) : &tmB0;
        const int brow = m.e * a.b_rows_per_expert + n * kNSlice + (kSwiGLU ? 0 : kBM * rank);
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kEmpty + stage), phase ^ 1u, abort_flag, limit, a.status,
                                 kWhereProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sA = sbase + stage * k2StageBytes;
          const uint32_t sB = sA + k2StageA;
          const uint32_t fb = map_to_rank(bar(kFull + stage), 0);
          if (leader) mbar_arrive_expect_tx(bar(kFull + stage), my_a_bytes + peer_a_bytes + 2 * k2StageB);
          if (my_rows > 0)
            tma_load_2d_pair(sA, &tmA.m[my_box], fb, kb * kBK, m.row0 + kBM * rank);
          tma_load_2d_pair(sB, bmap, fb, kb * kBK, brow);
          filled |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == k2Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // The leader's full barriers see both CTAs' loads land: it drains for the pair.  Rank 1
      // cannot observe its own loads; it waits for the MMA to release its last stages, which
      // happens at once on the normal path and otherwise ends after drain_limit (>= 1 s, far
      // longer than any load takes to land).
      int no_abort = 0;
      for (int s = 0; s < k2Stages; ++s)
        if ((filled >> s) & 1u) {
          if (leader)
            mbar_wait_bounded(bar(kFull + s), (last_parity >> s) & 1u, &no_abort, drain_limit,
                              a.status, kWhereDrain);
          else
            mbar_wait_bounded(bar(kEmpty + s), (last_parity >> s) & 1u, &no_abort, drain_limit,
                              nullptr, kWhereDrain);
        }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (rank 0)
    if (leader && lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(2 * kBM, kUmmaN);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = pair; t < ntiles && ok; t += npairs) {
        if (!mbar_wait_bounded(bar(kTEmpty + acc), acc_phase ^ 1u, abort_flag, limit, a.status,
                               kWhereMmaTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kUmmaN);
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kFull + stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * k2StageBytes;
          const uint64_t adesc = smem_desc_k_sw128(sA);
          const uint64_t bdesc = smem_desc_k_sw128(sA + k2StageA);
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)
            umma_bf16_pair(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc, (kb | k) != 0 ? 1u : 0u);
          umma_commit_pair(bar(kEmpty + stage), 0x3);
          if (++stage == k2Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit_pair(bar(kTFull + acc), 0x3);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      int no_abort = 0;
      umma_commit_pair(bar(kDrain), 0x1);
      mbar_wait_bounded(bar(kDrain), 0, &no_abort, drain_limit, a.status, kWhereDrain);
    }
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t tempty_leader[2] = {map_to_rank(bar(kTEmpty), 0),
                                       map_to_rank(bar(kTEmpty + 1), 0)};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int t = pair; t < ntiles; t += npairs) {
      int mt, n;
      decode_tile2(t, m_tiles, n_tiles, mt, n);
      const MTile m = a.mtiles[mt];
      const int my_rows = leader ? min(m.nrows, kBM) : max(m.nrows - kBM, 0);
      int ok = 0;
      if (lane == 0)
        ok = mbar_wait_bounded(bar(kTFull + acc), acc_phase, abort_flag, limit, a.status,
                               kWhereEpiTmemFull);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      ok = mbar_wait_bounded(bar(kTFull + acc), acc_phase, abort_flag, limit, a.status,
                             kWhereEpiTmemFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * kUmmaN);
      const bool valid = row < my_rows;
      __nv_bfloat16* dst = a.out +
                           static_cast<size_t>(m.row0 + kBM * rank + (valid ? row : 0)) * a.out_ld +
                           n * (kSwiGLU ? kN1Half : kN2);
      if (kSwiGLU) {
#pragma unroll 1
        for (int c = 0; c < kN1Half; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32_sync(tb + c, g);
          tmem_ld32_sync(tb + kN1Half + c, u);
          uint32_t p[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const float h0 = silu2(__uint_as_float(g[2 * j])) * __uint_as_float(u[2 * j]);
            const float h1 = silu2(__uint_as_float(g[2 * j + 1])) * __uint_as_float(u[2 * j + 1]);
            p[j] = pack_bf16x2_2(h0, h1);
          }
          if (valid) {
            uint4* o = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              o[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
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
            p[j] = pack_bf16x2_2(__uint_as_float(y[2 * j]), __uint_as_float(y[2 * j + 1]));
          if (valid) {
            uint4* o = reinterpret_cast<uint4*>(dst + c);
#pragma unroll
            for (int v = 0; v < 4; ++v)
              o[v] = make_uint4(p[4 * v], p[4 * v + 1], p[4 * v + 2], p[4 * v + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty_leader[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
  }

  tc_fence_before();
  __syncwarp();    // reconverge the role warps (one lane of warps 0 and 1 ran the loops)
  cluster_sync();  // no MMA, load or remote arrival of either CTA is still in flight
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc_pair(tmem_base, kTmemCols);
  }
}

}  // namespace

cudaError_t prepare_gemm_2sm_kernels() {
  cudaError_t e = cudaFuncSetAttribute(expert_gemm_2sm_kernel<true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, k2SmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(expert_gemm_2sm_kernel<false>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, k2SmemBytes);
}

template <bool kSwiGLU>
static cudaError_t launch_2sm(const ATensorMaps& tmA, const CUtensorMap& tmB0,
                              const CUtensorMap& tmB1, const GemmArgs& a, int grid,
                              cudaStream_t s) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid & ~1), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = k2SmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, expert_gemm_2sm_kernel<kSwiGLU>, tmA, tmB0, tmB1, a);
}

// Largest grid (in CTAs, even) whose clusters of two can all be resident at once.
int max_pair_grid(int sms) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = k2SmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, expert_gemm_2sm_kernel<true>, &cfg) != cudaSuccess ||
      clusters <= 0) {
    cudaGetLastError();
    return sms & ~1;
  }
  const int g = 2 * clusters;
  return g < sms ? g : (sms & ~1);
}

cudaError_t launch_gemm_gate_up_2sm(const ATensorMaps& tmA, const CUtensorMap& tmG,
                                    const CUtensorMap& tmU, const GemmArgs& a, int grid,
                                    cudaStream_t s) {
  return launch_2sm<true>(tmA, tmG, tmU, a, grid, s);
}

cudaError_t launch_gemm_down_2sm(const ATensorMaps& tmA, const CUtensorMap& tmD,
                                 const GemmArgs& a, int grid, cudaStream_t s) {
  return launch_2sm<false>(tmA, tmD, tmD, a, grid, s);
}

}  // namespace beam
