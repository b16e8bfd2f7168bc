// Router of the Beam sparse-MoE layer: FP32 logits on the CUDA cores, then sigmoid scores,
// selection-only bias, group-limited top-k and normalised, scaled weights.
//
// Transformers model doc "Beam", Overview: the router scores experts with a sigmoid, balances
// load with a learned per-expert bias, restricts each token to the best topk_group of n_group
// groups, normalises the routing weights and scales by routed_scaling_factor; routing runs in
// FP32 with FP32 router weights and bias.  archdb fact sheet "Beam-1.0-501B-A23B", expert-groups
// entry: group score = sum of the top-2 biased scores.  Groups are contiguous runs of
// E / n_group experts ("8 groups of 32", news article "Reflection lança o Beam").
#include "beam_moe_internal.cuh"
#include "beam_moe_router.cuh"

#include <math_constants.h>

namespace beam {
namespace {

// ---------------------------------------------------------------- W_r transpose
//
// The logits GEMM streams the router weight along the expert index; a transposed copy
// W_rT [d, E] (5 MB at Beam shapes) is written into the workspace on every call.
__global__ void __launch_bounds__(256) router_transpose_kernel(const float* __restrict__ W,
                                                               float* __restrict__ WT, int E, int d) {
  __shared__ float tile[32][33];
  const int e0 = blockIdx.y * 32, k0 = blockIdx.x * 32;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 32 x 8
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + r;
    tile[r][tx] = e < E ? W[static_cast<size_t>(e) * d + k0 + tx] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int r = ty; r < 32; r += 8) {
    const int e = e0 + tx;
    if (e < E) WT[static_cast<size_t>(k0 + r) * E + e] = tile[tx][r];
  }
}

// ---------------------------------------------------------------- logits: FP32 FFMA GEMM
//
// part[z, t, e] = sum_{j in K-chunk z} float(h[t, j]) * W[e, j].  Block tile 128 tokens x 128
// experts x 16 K, 256 threads, each an 8 x 8 register tile (rows ty*4.., 64+ty*4..; columns
// tx*4.., 64+tx*4..).  h is staged through registers (BF16 -> FP32, transposed into As[k][t]
// with a warp covering 32 consecutive tokens, so the stores are conflict-free); W_rT streams
// into a 3-stage cp.async ring.  Split-K over gridDim.z fills the machine for small T; the
// selection kernel adds the partial sums in a fixed order.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_1() {
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__global__ void __launch_bounds__(kRThreads, 2) router_gemm_kernel(const RouterGemmArgs a) {
  extern __shared__ __align__(16) float router_smem[];
  auto& As = *reinterpret_cast<float(*)[2][kRK][kRM]>(router_smem);
  auto& Bs = *reinterpret_cast<float(*)[kRBStages][kRK][kRN]>(router_smem + 2 * kRK * kRM);

  const int tid = threadIdx.x;
  const int m0 = blockIdx.x * kRM;
  const int n0 = blockIdx.y * kRN;
  const int kbeg = blockIdx.z * a.kchunk;
  const int kend = min(a.d, kbeg + a.kchunk);
  const int nk = (kend - kbeg) / kRK;

  if (a.zero_counts && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int e = tid; e < a.E; e += blockDim.x) a.zero_counts[e] = 0;

  const int tx = tid & 15;
  const int ty = tid >> 4;
  // A staging: kAChunks 16-byte chunks (8 K values each) of one token per thread and K tile
  constexpr int kAChunks = kRK * kRM / 8 / kRThreads;
  static_assert(kAChunks >= 1 && kRThreads % kRM == 0, "A staging covers the tile");
  const int a_row = tid & (kRM - 1);
  const int a_kp = (tid / kRM) * 8 * kAChunks;
  const int a_t = m0 + a_row;
  const __nv_bfloat16* a_src = a.h + static_cast<size_t>(a_t < a.T ? a_t : 0) * a.d + a_kp;
  struct AChunks {
    uint4 v[kAChunks];
  };

  auto load_a = [&](int k0) -> AChunks {
    AChunks c;
#pragma unroll
    for (int i = 0; i < kAChunks; ++i)
      c.v[i] = a_t < a.T ? *reinterpret_cast<const uint4*>(a_src + k0 + 8 * i)
                         : make_uint4(0, 0, 0, 0);
    return c;
  };
  auto store_a = [&](int buf, const AChunks& c) {
#pragma unroll
    for (int i = 0; i < kAChunks; ++i) {
      const uint32_t w4[4] = {c.v[i].x, c.v[i].y, c.v[i].z, c.v[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        As[buf][a_kp + 8 * i + 2 * q][a_row] = __uint_as_float(w4[q] << 16);
        As[buf][a_kp + 8 * i + 2 * q + 1][a_row] = __uint_as_float(w4[q] & 0xffff0000u);
      }
    }
  };
  auto issue_b = [&](int stage, int k0) {
#pragma unroll
    for (int i = 0; i < (kRK * kRN / 4) / kRThreads; ++i) {
      const int c = tid + i * kRThreads;
      const int k = c / (kRN / 4), n4 = (c % (kRN / 4)) * 4;
      const int e = n0 + n4;
      const bool ok = e < a.E;  // E % 4 == 0: a chunk is wholly in or out
      const float* src = a.WT + static_cast<size_t>(k0 + k) * a.E + (ok ? e : 0);
      cp_async16(smem_u32(&Bs[stage][k][n4]), src, ok ? 16 : 0);
    }
  };

  // Packed FMAs (fma.rn.f32x2: two IEEE FMAs, so every logit sees the same sequence of
  // roundings as with scalar fmaf, in half the instructions).  Rows are paired (2r, 2r + 1)
  // and columns (2c, 2c + 1); a row pair times a column pair gives the diagonal products,
  // times the swapped column pair the anti-diagonal ones:
  //   dg[r][c] = (acc[2r][2c],     acc[2r + 1][2c + 1])
  //   ad[r][c] = (acc[2r][2c + 1], acc[2r + 1][2c])
  float2 dg[4][4], ad[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) dg[r][c] = ad[r][c] = make_float2(0.f, 0.f);

  if (nk > 0) {
    issue_b(0, kbeg);
    cp_async_commit();
    if (nk > 1) issue_b(1, kbeg + kRK);
    cp_async_commit();
    store_a(0, load_a(kbeg));
  }
#pragma unroll 1
  for (int kt = 0; kt < nk; ++kt) {
    cp_async_wait_1();  // this tile's B has landed (one newer group may be in flight)
    __syncthreads();    // ... for every thread, and As[kt & 1] is stored
    if (kt + 2 < nk) issue_b((kt + 2) % kRBStages, kbeg + (kt + 2) * kRK);
    cp_async_commit();
    AChunks next{};
    if (kt + 1 < nk) next = load_a(kbeg + (kt + 1) * kRK);
    const int buf = kt & 1, st = kt % kRBStages;
#pragma unroll
    for (int kk = 0; kk < kRK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[st][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[st][kk][64 + tx * 4]);
      const float2 ap[4] = {make_float2(a0.x, a0.y), make_float2(a0.z, a0.w),
                            make_float2(a1.x, a1.y), make_float2(a1.z, a1.w)};
      const float2 bp[4] = {make_float2(b0.x, b0.y), make_float2(b0.z, b0.w),
                            make_float2(b1.x, b1.y), make_float2(b1.z, b1.w)};
      const float2 bs[4] = {make_float2(b0.y, b0.x), make_float2(b0.w, b0.z),
                            make_float2(b1.y, b1.x), make_float2(b1.w, b1.z)};
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          dg[r][c] = __ffma2_rn(ap[r], bp[c], dg[r][c]);
          ad[r][c] = __ffma2_rn(ap[r], bs[c], ad[r][c]);
        }
    }
    if (kt + 1 < nk) store_a(buf ^ 1, next);
  }

  // acc[i][j] back from the pairs: rows i = 2r + s, columns j = 2c + u
  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      acc[2 * r][2 * c] = dg[r][c].x;
      acc[2 * r + 1][2 * c + 1] = dg[r][c].y;
      acc[2 * r][2 * c + 1] = ad[r][c].x;
      acc[2 * r + 1][2 * c] = ad[r][c].y;
    }
  float* part = a.part + static_cast<size_t>(blockIdx.z) * a.T * a.E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + (i - 4));
    if (t >= a.T) continue;
    float* prow = part + static_cast<size_t>(t) * a.E;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int e = n0 + half * 64 + tx * 4;
      if (e < a.E) {
        const float* v = &acc[i][half * 4];
        *reinterpret_cast<float4*>(prow + e) = make_float4(v[0], v[1], v[2], v[3]);
      }
    }
  }
}

// Small batches (T <= kRouterSmallT, decode): tiles of 32 tokens x 128 experts x 16 K, 256
// threads, each a 4 x 4 register tile (rows ty*4.., columns tx*4.., ty = tid / 32,
// tx = tid % 32), so that a batch of a few tokens does not spend most of its FMAs on empty
// rows of a 128-token tile.  W_r is read as stored ([E, d]) and transposed while it is staged
// through registers, so these batches need no transposed copy (one launch less).  Same
// split-K, partial layout, packed FMAs and per-logit order of operations within a K chunk as
// router_gemm_kernel.
constexpr int kRSM = 32;

__global__ void __launch_bounds__(kRThreads) router_gemm_small_kernel(const RouterGemmArgs a,
                                                                        const float* __restrict__ W) {
  __shared__ __align__(16) float As[2][kRK][kRSM];
  __shared__ __align__(16) float Bs[2][kRK][kRN];
  const int tid = threadIdx.x;
  const int m0 = blockIdx.x * kRSM;
  const int n0 = blockIdx.y * kRN;
  const int kbeg = blockIdx.z * a.kchunk;
  const int kend = min(a.d, kbeg + a.kchunk);
  const int nk = (kend - kbeg) / kRK;

  if (a.zero_counts && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int e = tid; e < a.E; e += blockDim.x) a.zero_counts[e] = 0;

  const int tx = tid & 31, ty = tid >> 5;
  // A staging: 32 tokens x 16 K, a BF16 pair along K per thread; a warp covers the 32 tokens
  // at one K pair, so the transposed stores are conflict-free
  const int a_row = tid & (kRSM - 1);
  const int a_k = (tid / kRSM) * 2;
  const int a_t = m0 + a_row;
  const __nv_bfloat16* a_src = a.h + static_cast<size_t>(a_t < a.T ? a_t : 0) * a.d + a_k;
  auto load_a = [&](int k0) -> uint32_t {
    return a_t < a.T ? *reinterpret_cast<const uint32_t*>(a_src + k0) : 0u;
  };
  auto store_a = [&](int buf, uint32_t w) {
    As[buf][a_k][a_row] = __uint_as_float(w << 16);
    As[buf][a_k + 1][a_row] = __uint_as_float(w & 0xffff0000u);
  };
  // B staging: expert b_n's 8 K values from b_k, read from its W_r row and stored down the
  // column (a warp covers 32 experts at one K, so the stores are conflict-free)
  const int b_n = tid & (kRN - 1);
  const int b_k = (tid / kRN) * 8;
  const bool b_ok = n0 + b_n < a.E;
  const float* b_src = W + static_cast<size_t>(b_ok ? n0 + b_n : 0) * a.d + b_k;
  struct BChunk {
    float4 lo, hi;
  };
  auto load_b = [&](int k0) -> BChunk {
    if (!b_ok) return {make_float4(0.f, 0.f, 0.f, 0.f), make_float4(0.f, 0.f, 0.f, 0.f)};
    return {*reinterpret_cast<const float4*>(b_src + k0),
            *reinterpret_cast<const float4*>(b_src + k0 + 4)};
  };
  auto store_b = [&](int buf, const BChunk& c) {
    const float v[8] = {c.lo.x, c.lo.y, c.lo.z, c.lo.w, c.hi.x, c.hi.y, c.hi.z, c.hi.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) Bs[buf][b_k + j][b_n] = v[j];
  };

  // dg[r][c] = (acc[2r][2c], acc[2r + 1][2c + 1]), ad[r][c] = (acc[2r][2c + 1], acc[2r + 1][2c])
  float2 dg[2][2], ad[2][2];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int c = 0; c < 2; ++c) dg[r][c] = ad[r][c] = make_float2(0.f, 0.f);

  // K tiles in groups of kGroup: the group's loads are all issued before its first tile is
  // used, so its global reads (W_r mostly from DRAM) overlap; tile kt lives in buffer kt & 1,
  // and the barrier after each store also orders it after every thread's use of the buffer
  // two tiles back
  constexpr int kGroup = 8;
#pragma unroll 1
  for (int g = 0; g < nk; g += kGroup) {
    uint32_t aq[kGroup];
    BChunk bq[kGroup];
#pragma unroll
    for (int i = 0; i < kGroup; ++i)
      if (g + i < nk) {
        aq[i] = load_a(kbeg + (g + i) * kRK);
        bq[i] = load_b(kbeg + (g + i) * kRK);
      }
#pragma unroll
    for (int i = 0; i < kGroup; ++i) {
      if (g + i < nk) {
        const int buf = (g + i) & 1;
        store_a(buf, aq[i]);
        store_b(buf, bq[i]);
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kRK; ++kk) {
          const float4 av = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
          const float4 bv = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
          const float2 ap[2] = {make_float2(av.x, av.y), make_float2(av.z, av.w)};
          const float2 bp[2] = {make_float2(bv.x, bv.y), make_float2(bv.z, bv.w)};
          const float2 bs[2] = {make_float2(bv.y, bv.x), make_float2(bv.w, bv.z)};
#pragma unroll
          for (int r = 0; r < 2; ++r)
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              dg[r][c] = __ffma2_rn(ap[r], bp[c], dg[r][c]);
              ad[r][c] = __ffma2_rn(ap[r], bs[c], ad[r][c]);
            }
        }
      }
    }
  }

  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      acc[2 * r][2 * c] = dg[r][c].x;
      acc[2 * r + 1][2 * c + 1] = dg[r][c].y;
      acc[2 * r][2 * c + 1] = ad[r][c].x;
      acc[2 * r + 1][2 * c] = ad[r][c].y;
    }
  float* part = a.part + static_cast<size_t>(blockIdx.z) * a.T * a.E;
  const int e = n0 + tx * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int t = m0 + ty * 4 + i;
    if (t < a.T && e < a.E)
      *reinterpret_cast<float4*>(part + static_cast<size_t>(t) * a.E + e) =
          make_float4(acc[i][0], acc[i][1], acc[i][2], acc[i][3]);
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
//   dispatch       per-expert slot counts and the token bitmap (bit t of expert e's row set
//                  when token t chose e); the scan turns them into ascending-token row ranks

__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// kSelTokens tokens per block; kSelZ splits of a logit in flight per thread.  Large batches
// take 8 tokens a block; small ones (decode) one, so that more blocks share the sum of the
// many splits the GEMM then uses, with more of them in flight.
template <int kSelTokens, int kSelZ>
__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a) {
  constexpr int kSelLogitsPerThread = kSelTokens * kMaxE / 256;
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
    for (int z0 = 0; z0 < a.S; z0 += kSelZ) {
      float v[kSelZ][kSelLogitsPerThread];
#pragma unroll
      for (int zz = 0; zz < kSelZ; ++zz)
#pragma unroll
        for (int j = 0; j < kSelLogitsPerThread; ++j) {
          const int i = threadIdx.x + 256 * j;
          v[zz][j] = (z0 + zz < a.S && i < n) ? base[(z0 + zz) * zs + i] : 0.f;
        }
#pragma unroll
      for (int zz = 0; zz < kSelZ; ++zz)
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
    } else {
      const int e = sel_sh[warp][lane];
      const float s = sw[e];
      a.idx[slot] = e;
      a.w[slot] = a.norm ? a.scale * s / denom : a.scale * s;
      if (a.cnt) {  // dispatch: count the slot and mark token t in expert e's bitmap
        atomicAdd(a.cnt + e, 1);
        atomicOr(a.bits + static_cast<size_t>(e) * a.words + (t >> 5), 1u << (t & 31));
      }
    }
  }
}

}  // namespace

cudaError_t launch_router_transpose(const float* W, float* WT, int E, int d, cudaStream_t s) {
  const dim3 grid(d / 32, (E + 31) / 32);
  router_transpose_kernel<<<grid, 256, 0, s>>>(W, WT, E, d);
  return cudaGetLastError();
}

constexpr int kRouterSmemBytes = (2 * kRK * kRM + kRBStages * kRK * kRN) * 4;

cudaError_t prepare_router_kernels() {
  return cudaFuncSetAttribute(router_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kRouterSmemBytes);
}

cudaError_t launch_router_gemm(const RouterGemmArgs& a, int S, cudaStream_t s) {
  const dim3 grid((a.T + kRM - 1) / kRM, (a.E + kRN - 1) / kRN, S);
  router_gemm_kernel<<<grid, kRThreads, kRouterSmemBytes, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router_gemm_small(const RouterGemmArgs& a, const float* W, int S,
                                     cudaStream_t s) {
  const dim3 grid((a.T + kRSM - 1) / kRSM, (a.E + kRN - 1) / kRN, S);
  router_gemm_small_kernel<<<grid, kRThreads, 0, s>>>(a, W);
  return cudaGetLastError();
}

cudaError_t launch_router_select(const SelectArgs& a, cudaStream_t s) {
  if (a.T <= kSelSmallT)
    router_select_kernel<1, 16><<<a.T, 256, 0, s>>>(a);
  else
    router_select_kernel<8, 4><<<(a.T + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
