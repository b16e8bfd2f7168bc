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
  __shared__ __align__(16) float As[2][kRK][kRM];
  __shared__ __align__(16) float Bs[kRBStages][kRK][kRN];

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
  // A staging: one 16-byte chunk (8 K values) of one token per thread and K tile
  const int a_row = tid & (kRM - 1);
  const int a_kp = (tid >> 7) * 8;
  const int a_t = m0 + a_row;
  const __nv_bfloat16* a_src = a.h + static_cast<size_t>(a_t < a.T ? a_t : 0) * a.d + a_kp;

  auto load_a = [&](int k0) -> uint4 {
    return a_t < a.T ? *reinterpret_cast<const uint4*>(a_src + k0) : make_uint4(0, 0, 0, 0);
  };
  auto store_a = [&](int buf, uint4 v) {
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      As[buf][a_kp + 2 * q][a_row] = __uint_as_float(w4[q] << 16);
      As[buf][a_kp + 2 * q + 1][a_row] = __uint_as_float(w4[q] & 0xffff0000u);
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

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

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
    uint4 next = make_uint4(0, 0, 0, 0);
    if (kt + 1 < nk) next = load_a(kbeg + (kt + 1) * kRK);
    const int buf = kt & 1, st = kt % kRBStages;
#pragma unroll
    for (int kk = 0; kk < kRK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[st][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[st][kk][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (kt + 1 < nk) store_a(buf ^ 1, next);
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

// ---------------------------------------------------------------- selection: one warp per token
//
// Each lane owns up to 8 consecutive experts (lane * per_lane ...).  The token's scores are
// also kept in shared memory so that any lane can read any expert's score.  Group scores are
// computed by lane g for group g (sequential scan of its E/G experts); the kept groups come
// from a rank count over all group scores; the top_k experts are taken in top_k rounds of a
// warp-wide maximum over 64-bit keys (order-preserving score bits, then inverted expert id, so
// that the lower id wins a tie).

__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a) {
  __shared__ float s_sh[8][kMaxE];
  __shared__ float sb_sh[8][kMaxE];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
  const int E = a.E, G = a.G, P = E / G;
  const int per_lane = (E + 31) / 32;
  float* s_w = s_sh[warp];
  float* sb_w = sb_sh[warp];

  // logits (sum of the split-K partials in z order), scores, biased scores
  float my_sb[kMaxE / 32];
#pragma unroll
  for (int i = 0; i < kMaxE / 32; ++i) {
    my_sb[i] = -CUDART_INF_F;
    const int e = lane * per_lane + i;
    if (i < per_lane && e < E) {
      const float* p = a.part + static_cast<size_t>(t) * E + e;
      const size_t zs = static_cast<size_t>(a.T) * E;
      float l = 0.f;
#pragma unroll 4
      for (int z = 0; z < a.S; ++z) l += p[z * zs];
      if (a.logits_out) a.logits_out[static_cast<size_t>(t) * E + e] = l;
      const float s = 1.0f / (1.0f + expf(-l));
      const float sb = s + a.bias[e];
      s_w[e] = s;
      sb_w[e] = sb;
      my_sb[i] = sb;
    }
  }
  __syncwarp();

  // group scores: lane g scans group g
  float gs = -CUDART_INF_F;
  if (lane < G) {
    float m1 = -CUDART_INF_F, m2 = -CUDART_INF_F;
#pragma unroll 1
    for (int e = lane * P; e < (lane + 1) * P; ++e) {
      const float v = sb_w[e];
      if (v > m1) {
        m2 = m1;
        m1 = v;
      } else if (v > m2) {
        m2 = v;
      }
    }
    gs = P >= 2 ? m1 + m2 : m1;
  }
  // rank of my group among all groups (higher score first, lower index on ties)
  int rank = 0;
#pragma unroll 1
  for (int g2 = 0; g2 < G; ++g2) {
    const float o = __shfl_sync(0xffffffffu, gs, g2);
    if (lane < G && (o > gs || (o == gs && g2 < lane))) ++rank;
  }
  const uint32_t kept = __ballot_sync(0xffffffffu, lane < G && rank < a.Gk);

  // candidate keys of my experts (0 = not a candidate)
  uint64_t key[kMaxE / 32];
#pragma unroll
  for (int i = 0; i < kMaxE / 32; ++i) {
    const int e = lane * per_lane + i;
    key[i] = 0;
    if (i < per_lane && e < E && ((kept >> (e / P)) & 1u))
      key[i] = (static_cast<uint64_t>(ordered_bits(my_sb[i])) << 32) |
               static_cast<uint64_t>(0xffffffffu - static_cast<uint32_t>(e));
  }
  int sel[kMaxTopK];
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    sel[r] = 0x7fffffff;
    if (r < a.k) {
      uint64_t best = 0;
#pragma unroll
      for (int i = 0; i < kMaxE / 32; ++i) best = key[i] > best ? key[i] : best;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const uint64_t o = __shfl_xor_sync(0xffffffffu, best, off);
        best = o > best ? o : best;
      }
      const int e = best ? static_cast<int>(0xffffffffu - static_cast<uint32_t>(best)) : -1;
      sel[r] = e < 0 ? 0x7fffffff : e;
#pragma unroll
      for (int i = 0; i < kMaxE / 32; ++i)
        if (key[i] == best) key[i] = 0;
    }
  }
  // ascending expert id (insertion sort, identical on every lane)
#pragma unroll
  for (int r = 1; r < kMaxTopK; ++r)
#pragma unroll
    for (int q = r; q > 0; --q)
      if (sel[q] < sel[q - 1]) {
        const int tmp = sel[q];
        sel[q] = sel[q - 1];
        sel[q - 1] = tmp;
      }
  float denom = 0.f;
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r)
    if (r < a.k && sel[r] < E) denom += s_w[sel[r]];

#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    if (r < a.k && lane == r) {
      const int e = sel[r];
      const size_t slot = static_cast<size_t>(t) * a.k + r;
      if (e < 0 || e >= E) {  // no candidate left: cannot happen for a validated shape
        record_status(a.status, kDevAssert, kWhereSelect);
        a.idx[slot] = 0;
        a.w[slot] = 0.f;
        if (a.cnt) a.rank[slot] = -1;
        continue;
      }
      const float s = s_w[e];
      a.idx[slot] = e;
      a.w[slot] = a.norm ? a.scale * s / denom : a.scale * s;
      if (a.cnt) a.rank[slot] = atomicAdd(a.cnt + e, 1);
    }
  }
}

}  // namespace

cudaError_t launch_router_transpose(const float* W, float* WT, int E, int d, cudaStream_t s) {
  const dim3 grid(d / 32, (E + 31) / 32);
  router_transpose_kernel<<<grid, 256, 0, s>>>(W, WT, E, d);
  return cudaGetLastError();
}

cudaError_t launch_router_gemm(const RouterGemmArgs& a, int S, cudaStream_t s) {
  const dim3 grid((a.T + kRM - 1) / kRM, (a.E + kRN - 1) / kRN, S);
  router_gemm_kernel<<<grid, kRThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_router_select(const SelectArgs& a, cudaStream_t s) {
  router_select_kernel<<<(a.T + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
