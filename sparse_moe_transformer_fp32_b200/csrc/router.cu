// Router of the Beam sparse-MoE layer: FP32 logits on the tensor cores, then sigmoid scores,
// selection-only bias, group-limited top-k and normalised, scaled weights.
//
// Transformers model doc "Beam", Overview: the router scores experts with a sigmoid, balances
// load with a learned per-expert bias, restricts each token to the best topk_group of n_group
// groups, normalises the routing weights and scales by routed_scaling_factor; routing runs in
// FP32 with FP32 router weights and bias.  archdb fact sheet "Beam-1.0-501B-A23B", expert-groups
// entry: group score = sum of the top-2 biased scores.  Groups are contiguous runs of
// E / n_group experts ("8 groups of 32", news article "Reflection lança o Beam").
#include "beam_moe_internal.cuh"

#include <math_constants.h>

namespace beam {
namespace {

// ---------------------------------------------------------------- W_r split
//
// The logits run on the tensor cores as BF16 x BF16 products with FP32 accumulation.  h is
// BF16 already; the FP32 router weight is written as the sum of three BF16 terms
//     w1 = bf16(W),  w2 = bf16(W - w1),  w3 = bf16(W - w1 - w2)
// (round to nearest even).  Each difference is exact in FP32 and each rounding leaves at most
// 2^-8 of what it rounds, so |W - (w1 + w2 + w3)| <= 2^-24 |W|: the FP32 weight itself, up to
// its own unit roundoff.  Products of BF16 values are exact in FP32, so h . W = h . w1 +
// h . w2 + h . w3 is an FP32-accumulated FP32 dot product.  Ws is [3, E, d] BF16, written
// into the workspace on every call (7.9 MB at Beam shapes).
__global__ void __launch_bounds__(256) router_split_kernel(const float4* __restrict__ W,
                                                           uint2* __restrict__ Ws, size_t n4) {
  for (size_t i = static_cast<size_t>(blockIdx.x) * 256 + threadIdx.x; i < n4;
       i += static_cast<size_t>(gridDim.x) * 256) {
    const float4 v = W[i];
    float r[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int term = 0; term < 3; ++term) {
      uint32_t p[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const __nv_bfloat16 lo = __float2bfloat16_rn(r[2 * j]);
        const __nv_bfloat16 hi = __float2bfloat16_rn(r[2 * j + 1]);
        r[2 * j] -= __bfloat162float(lo);
        r[2 * j + 1] -= __bfloat162float(hi);
        p[j] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
      }
      Ws[term * n4 + i] = make_uint2(p[0], p[1]);
    }
  }
}

// ---------------------------------------------------------------- logits: tcgen05 GEMM
//
// part[z, t, e] = sum over the K blocks of split z of h[t, :] . (w1 + w2 + w3)[e, :]
// One CTA per (128-token tile, 128-expert tile, K split), 192 threads:
//   warp 0     one thread issues TMA loads into a 3-stage ring; a stage holds the 128 x 64 BF16
//              h tile and one 3-D box with the three 128 x 64 weight-term tiles (64 KB)
//   warp 1     allocates 256 TMEM columns (two 128-column accumulators); one thread issues 12
//              tcgen05.mma (M=128, N=128, K=16) per stage, the three terms into the same
//              accumulator, and hands the accumulator over every kRouterChunk stages
//   warps 2-5  add each handed-over accumulator into FP32 registers (one token row per thread,
//              its warp's 32-lane TMEM quarter), then store the row's partial logits
// The tensor cores accumulate with less care than round-to-nearest FP32 adds: the logit error
// grows with the number of MMAs summed into one accumulator (measured ~1e-6 per 24 MMAs at
// d = 5120, ~6e-5 when all 960 of a full-K tile are chained).  Chunks of 24 MMAs summed by
// FP32 adds in a fixed order keep it at the level of a plain FP32 dot product.
// Rows past T and experts past E are zero-filled by TMA and never stored.  The selection
// kernel adds the K-split partials in a fixed order, so the result is deterministic.
// Waits are bounded as in the expert GEMMs: a timeout is recorded in the status word, the CTA
// drains its own TMA loads and MMAs, frees TMEM and returns.
constexpr uint64_t kRouterMinDrainNs = 1000000000ull;

__global__ void __launch_bounds__(kRouterThreads, 1)
    router_mma_kernel(const __grid_constant__ CUtensorMap tmH,
                      const __grid_constant__ CUtensorMap tmW, const RouterMmaArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  // [kRouterStages x (h 16 KB | w1, w2, w3 48 KB)][barriers][TMEM address][abort flag]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kRouterStages * kRouterStageBytes);
  constexpr int kBarFull = 0, kBarEmpty = kRouterStages, kBarCFull = 2 * kRouterStages,
                kBarCEmpty = kBarCFull + 2, kBarDrain = kBarCEmpty + 2, kNumBars = kBarDrain + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto bar = [&](int i) { return smem_u32(bars + i); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kRouterM, n0 = blockIdx.y * kRouterN;
  const int kb0 = blockIdx.z * a.kb_per_split;
  const int kb1 = min(a.k_blocks, kb0 + a.kb_per_split);
  const int nchunks = (kb1 - kb0 + kRouterChunk - 1) / kRouterChunk;
  const uint64_t limit = a.wait_limit_ns;
  const uint64_t drain_limit = limit > kRouterMinDrainNs ? limit : kRouterMinDrainNs;

  if (a.zero_counts && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int e = threadIdx.x; e < a.E; e += blockDim.x) a.zero_counts[e] = 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRouterStages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(kBarCFull + i), 1);
      mbar_init(bar(kBarCEmpty + i), 4);
    }
    mbar_init(bar(kBarDrain), 1);
    *abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmH);
    tma_prefetch_desc(&tmW);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 2 * kRouterN);
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
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait_bounded(bar(kBarEmpty + stage), phase ^ 1u, abort_flag, limit, a.status,
                               kWhereProducerEmpty))
          break;
        const uint32_t sA = sbase + stage * kRouterStageBytes;
        const uint32_t fb = bar(kBarFull + stage);
        mbar_arrive_expect_tx(fb, kRouterStageBytes);
        tma_load_2d(sA, &tmH, fb, kb * kBK, m0);
        tma_load_3d(sA + kRouterStageABytes, &tmW, fb, kb * kBK, n0, 0);
        filled |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == kRouterStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      // every load this thread issued must land before the CTA may exit
      int no_abort = 0;
      for (int s = 0; s < kRouterStages; ++s)
        if ((filled >> s) & 1u)
          mbar_wait_bounded(bar(kBarFull + s), (last_parity >> s) & 1u, &no_abort, drain_limit,
                            a.status, kWhereDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(kRouterM, kRouterN);
      constexpr uint32_t kTermBytes = kRouterN * kBK * 2;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int c = 0; c < nchunks && ok; ++c) {
        const int buf = c & 1;
        const uint32_t cphase = static_cast<uint32_t>(c >> 1) & 1u;
        if (!mbar_wait_bounded(bar(kBarCEmpty + buf), cphase ^ 1u, abort_flag, limit, a.status,
                               kWhereMmaTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(buf * kRouterN);
        const int c0 = kb0 + c * kRouterChunk;
        const int c1 = min(kb1, c0 + kRouterChunk);
        for (int kb = c0; kb < c1; ++kb) {
          if (!mbar_wait_bounded(bar(kBarFull + stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * kRouterStageBytes;
          const uint64_t adesc = smem_desc_k_sw128(sA);
#pragma unroll
          for (int term = 0; term < 3; ++term) {
            const uint64_t bdesc = smem_desc_k_sw128(sA + kRouterStageABytes + term * kTermBytes);
#pragma unroll
            for (int k = 0; k < kBK / kUmmaK; ++k)  // +32 bytes along K per step: +2 in addr>>4
              umma_bf16(d_tmem, adesc + 2u * k, bdesc + 2u * k, idesc,
                        (kb != c0 || term != 0 || k != 0) ? 1u : 0u);
          }
          umma_commit(bar(kBarEmpty + stage));
          if (++stage == kRouterStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (ok) umma_commit(bar(kBarCFull + buf));
      }
      // all MMAs this thread issued must complete before TMEM is freed
      int no_abort = 0;
      umma_commit(bar(kBarDrain));
      mbar_wait_bounded(bar(kBarDrain), 0, &no_abort, drain_limit, a.status, kWhereDrain);
    }
  } else {
    // ------------------------------------------------------------ chunk sums, then stores
    const int q = warp & 3;  // TMEM lane quarter this warp may access (warps 2..5)
    const uint32_t tq = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    float acc[kRouterN];
#pragma unroll
    for (int j = 0; j < kRouterN; ++j) acc[j] = 0.f;
    bool ok = true;
    for (int c = 0; c < nchunks; ++c) {
      const int buf = c & 1;
      const uint32_t cphase = static_cast<uint32_t>(c >> 1) & 1u;
      ok = mbar_wait_bounded(bar(kBarCFull + buf), cphase, abort_flag, limit, a.status,
                             kWhereEpiTmemFull);
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll
      for (int g = 0; g < kRouterN / 32; ++g) {
        uint32_t v[32];
        tmem_ld32_sync(tq + static_cast<uint32_t>(buf * kRouterN + g * 32), v);
#pragma unroll
        for (int j = 0; j < 32; ++j) acc[g * 32 + j] += __uint_as_float(v[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(kBarCEmpty + buf));
    }
    const int t = m0 + q * 32 + lane;
    if (ok && t < a.T) {
      float* prow = a.part + (static_cast<size_t>(blockIdx.z) * a.T + t) * a.E;
#pragma unroll
      for (int j = 0; j < kRouterN; j += 4) {
        const int e = n0 + j;  // E % 4 == 0: a group of four is wholly in or out
        if (e < a.E)
          *reinterpret_cast<float4*>(prow + e) =
              make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kRouterN);
  }
}

// ---------------------------------------------------------------- selection
//
// A block of 256 threads takes 8 tokens.  First the whole block forms the 8 x E logits (the
// K-split partials added in z order, loads of four splits in flight), scores s = sigmoid and
// biased scores sb = s + b into shared memory.  Then one warp per token:
//   group scores   lane g scans group g's E/G biased scores (sum of the top two); lanes start
//                  at different offsets of their groups so that the reads hit distinct banks
//   kept groups    rank of each group score among all (higher first, lower index on ties)
//   top-k          lane l holds experts l*c .. l*c+c-1 (c = ceil(E/32)); k rounds of a warp
//                  maximum of the lanes' best candidate scores (order-preserving bits, redux),
//                  then a warp minimum of the expert ids holding it (lower id wins a tie)
//   output         ascending expert id: lane order, then a prefix sum of the lanes' counts;
//                  the weights' denominator is summed in that order

__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSelTokens = 8;
constexpr int kSelLogitsPerThread = kSelTokens * kMaxE / 256;

__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a) {
  __shared__ float s_sh[kSelTokens][kMaxE];
  __shared__ float sb_sh[kSelTokens][kMaxE];
  __shared__ int sel_sh[kSelTokens][kMaxTopK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E, G = a.G, P = E / G;
  const int t0 = blockIdx.x * kSelTokens;
  const int ntok = min(kSelTokens, a.T - t0);

  // ---- logits, scores and biased scores of the block's tokens
  {
    const int n = ntok * E;
    const size_t zs = static_cast<size_t>(a.T) * E;
    const float* base = a.part + static_cast<size_t>(t0) * E;
    float l[kSelLogitsPerThread];
#pragma unroll
    for (int j = 0; j < kSelLogitsPerThread; ++j) l[j] = 0.f;
#pragma unroll 1
    for (int z0 = 0; z0 < a.S; z0 += 4) {
      float v[4][kSelLogitsPerThread];
#pragma unroll
      for (int zz = 0; zz < 4; ++zz)
#pragma unroll
        for (int j = 0; j < kSelLogitsPerThread; ++j) {
          const int i = threadIdx.x + 256 * j;
          v[zz][j] = (z0 + zz < a.S && i < n) ? base[(z0 + zz) * zs + i] : 0.f;
        }
#pragma unroll
      for (int zz = 0; zz < 4; ++zz)
#pragma unroll
        for (int j = 0; j < kSelLogitsPerThread; ++j)
          if (z0 + zz < a.S) l[j] += v[zz][j];
    }
#pragma unroll
    for (int j = 0; j < kSelLogitsPerThread; ++j) {
      const int i = threadIdx.x + 256 * j;
      if (i < n) {
        const int tl = i / E, e = i - tl * E;
        if (a.logits_out) a.logits_out[static_cast<size_t>(t0) * E + i] = l[j];
        const float s = 1.0f / (1.0f + expf(-l[j]));
        s_sh[tl][e] = s;
        sb_sh[tl][e] = s + a.bias[e];
      }
    }
  }
  __syncthreads();
  if (warp >= ntok) return;
  const int t = t0 + warp;
  const float* sw = s_sh[warp];
  const float* sbw = sb_sh[warp];

  // ---- group scores: lane g takes group g
  float gs = -CUDART_INF_F;
  if (lane < G) {
    const float* grp = sbw + lane * P;
    const int o = lane % P;
    float m1 = -CUDART_INF_F, m2 = -CUDART_INF_F;
#pragma unroll 8
    for (int j = 0; j < P; ++j) {
      int jj = j + o;
      if (jj >= P) jj -= P;
      const float v = grp[jj];
      if (v > m1) {
        m2 = m1;
        m1 = v;
      } else if (v > m2) {
        m2 = v;
      }
    }
    gs = P >= 2 ? m1 + m2 : m1;
  }
  int grank = 0;
#pragma unroll 8
  for (int g2 = 0; g2 < G; ++g2) {
    const float o = __shfl_sync(0xffffffffu, gs, g2);
    if (lane < G && (o > gs || (o == gs && g2 < lane))) ++grank;
  }
  const uint32_t kept = __ballot_sync(0xffffffffu, lane < G && grank < a.Gk);

  // ---- this lane's candidates
  const int c = (E + 31) / 32;
  const int e0 = lane * c;
  uint32_t bits[kMaxE / 32];
  uint32_t avail = 0;
  {
    int g = e0 / P, r = e0 - g * P;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      bits[i] = 0;
      if (i < c && e0 + i < E) {
        if ((kept >> g) & 1u) {
          bits[i] = ordered_bits(sbw[e0 + i]);
          avail |= 1u << i;
        }
        if (++r == P) {
          r = 0;
          ++g;
        }
      }
    }
  }
  auto local_best = [&](uint32_t& best, int& bi) {
    best = 0;
    bi = 0;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i)
      if (((avail >> i) & 1u) && bits[i] > best) {  // strict: the lower id keeps a tie
        best = bits[i];
        bi = i;
      }
  };
  uint32_t best;
  int bi;
  local_best(best, bi);
  uint32_t chosen = 0;
  bool short_of_candidates = false;
#pragma unroll 1
  for (int r = 0; r < a.k; ++r) {
    const uint32_t m = __reduce_max_sync(0xffffffffu, best);
    if (m == 0u) {  // no candidate left: cannot happen for a validated shape
      short_of_candidates = true;
      break;
    }
    const uint32_t mine = best == m ? static_cast<uint32_t>(e0 + bi) : 0xffffffffu;
    const uint32_t win = __reduce_min_sync(0xffffffffu, mine);
    if (mine == win) {
      chosen |= 1u << bi;
      avail &= ~(1u << bi);
      local_best(best, bi);
    }
  }

  // ---- ascending expert ids: lanes in order, each lane's experts in order
  const int cnt = __popc(chosen);
  int incl = cnt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  const int total = __shfl_sync(0xffffffffu, incl, 31);
  int pos = incl - cnt;
#pragma unroll
  for (int i = 0; i < kMaxE / 32; ++i)
    if ((chosen >> i) & 1u) sel_sh[warp][pos++] = e0 + i;
  __syncwarp();
  float denom = 0.f;
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r)
    if (r < total) denom += sw[sel_sh[warp][r]];
  if (lane < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + lane;
    if (lane >= total) {
      if (lane == total && short_of_candidates) record_status(a.status, kDevAssert, kWhereSelect);
      a.idx[slot] = 0;
      a.w[slot] = 0.f;
      if (a.cnt) a.rank[slot] = -1;
    } else {
      const int e = sel_sh[warp][lane];
      const float s = sw[e];
      a.idx[slot] = e;
      a.w[slot] = a.norm ? a.scale * s / denom : a.scale * s;
      if (a.cnt) a.rank[slot] = atomicAdd(a.cnt + e, 1);
    }
  }
}

}  // namespace

cudaError_t launch_router_split(const float* W, __nv_bfloat16* Ws, int E, int d, int sms,
                                cudaStream_t s) {
  const size_t n4 = static_cast<size_t>(E) * d / 4;
  const size_t want = (n4 + 255) / 256;
  const int grid = static_cast<int>(want < static_cast<size_t>(4 * sms) ? want : 4 * sms);
  router_split_kernel<<<grid, 256, 0, s>>>(reinterpret_cast<const float4*>(W),
                                           reinterpret_cast<uint2*>(Ws), n4);
  return cudaGetLastError();
}

cudaError_t prepare_router_kernels() {
  return cudaFuncSetAttribute(router_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kRouterSmemBytes);
}

cudaError_t launch_router_gemm(const CUtensorMap& tmH, const CUtensorMap& tmW,
                               const RouterMmaArgs& a, cudaStream_t s) {
  const dim3 grid((a.T + kRouterM - 1) / kRouterM, (a.E + kRouterN - 1) / kRouterN,
                  (a.k_blocks + a.kb_per_split - 1) / a.kb_per_split);
  router_mma_kernel<<<grid, kRouterThreads, kRouterSmemBytes, s>>>(tmH, tmW, a);
  return cudaGetLastError();
}

cudaError_t launch_router_select(const SelectArgs& a, cudaStream_t s) {
  router_select_kernel<<<(a.T + kSelTokens - 1) / kSelTokens, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
