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

// ---------------------------------------------------------------- logits: FP32 FFMA GEMM
//
// part[z, t, e] = sum_{j in K-chunk z} float(h[t, j]) * W[e, j].  Block tile 64 tokens x 128
// experts x 32 K, 128 threads with an 8 x 8 register tile each, shared memory double buffered
// with register staging.  Split-K over gridDim.z keeps the grid wide for small T; the partial
// sums are added in a fixed order by the selection kernel.
__global__ void __launch_bounds__(kRThreads) router_gemm_kernel(const RouterGemmArgs a) {
  __shared__ __align__(16) float As[2][kRK][kRM];
  __shared__ __align__(16) float Bs[2][kRK][kRN];

  const int tid = threadIdx.x;
  const int m0 = blockIdx.x * kRM;
  const int n0 = blockIdx.y * kRN;
  const int kbeg = blockIdx.z * a.kchunk;
  const int kend = min(a.d, kbeg + a.kchunk);
  const int nk = (kend - kbeg) / kRK;

  if (a.zero_counts && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
    for (int e = tid; e < a.E; e += blockDim.x) a.zero_counts[e] = 0;

  const int tx = tid & 15;  // expert columns tx*4 .. +3 and 64 + tx*4 .. +3
  const int ty = tid >> 4;  // token rows ty*4 .. +3 and 32 + ty*4 .. +3

  uint4 ra[2];
  float4 rb[8];

  auto load_global = [&](int k0) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + i * kRThreads;  // 0..255
      const int row = c >> 2, kp = (c & 3) * 8;
      const int t = m0 + row;
      ra[i] = t < a.T ? *reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(t) * a.d + k0 + kp)
                      : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = tid + i * kRThreads;  // 0..1023
      const int row = c >> 3, kp = (c & 7) * 4;
      const int e = n0 + row;
      rb[i] = e < a.E ? *reinterpret_cast<const float4*>(a.W + static_cast<size_t>(e) * a.d + k0 + kp)
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  auto store_smem = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const int c = tid + i * kRThreads;
      const int row = c >> 2, kp = (c & 3) * 8;
      const uint32_t w4[4] = {ra[i].x, ra[i].y, ra[i].z, ra[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        As[buf][kp + 2 * q][row] = __uint_as_float(w4[q] << 16);
        As[buf][kp + 2 * q + 1][row] = __uint_as_float(w4[q] & 0xffff0000u);
      }
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = tid + i * kRThreads;
      const int row = c >> 3, kp = (c & 7) * 4;
      Bs[buf][kp + 0][row] = rb[i].x;
      Bs[buf][kp + 1][row] = rb[i].y;
      Bs[buf][kp + 2][row] = rb[i].z;
      Bs[buf][kp + 3][row] = rb[i].w;
    }
  };

  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;

  if (nk > 0) {
    load_global(kbeg);
    store_smem(0);
  }
  __syncthreads();
#pragma unroll 1
  for (int kt = 0; kt < nk; ++kt) {
    const int buf = kt & 1;
    if (kt + 1 < nk) load_global(kbeg + (kt + 1) * kRK);
#pragma unroll
    for (int kk = 0; kk < kRK; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][32 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    if (kt + 1 < nk) store_smem(buf ^ 1);
    __syncthreads();
  }

  float* part = a.part + static_cast<size_t>(blockIdx.z) * a.T * a.E;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int t = m0 + (i < 4 ? ty * 4 + i : 32 + ty * 4 + (i - 4));
    if (t >= a.T) continue;
    float* prow = part + static_cast<size_t>(t) * a.E;
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int e = n0 + half * 64 + tx * 4;
      const float* v = &acc[i][half * 4];
      if (e + 3 < a.E && (a.E & 3) == 0) {
        *reinterpret_cast<float4*>(prow + e) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (e + j < a.E) prow[e + j] = v[j];
      }
    }
  }
}

// ---------------------------------------------------------------- selection: one warp per token

__device__ __forceinline__ void top2_insert(float v, float& m1, float& m2) {
  if (v > m1) {
    m2 = m1;
    m1 = v;
  } else if (v > m2) {
    m2 = v;
  }
}

__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a) {
  constexpr int kPer = kMaxE / 32;  // experts per lane (lane-strided: e = lane + 32 i)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
  const int E = a.E, G = a.G, P = E / G;
  const float ninf = -CUDART_INF_F;

  float s[kPer], sb[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      float l = 0.f;
      for (int z = 0; z < a.S; ++z) l += a.part[(static_cast<size_t>(z) * a.T + t) * E + e];
      if (a.logits_out) a.logits_out[static_cast<size_t>(t) * E + e] = l;
      s[i] = 1.0f / (1.0f + expf(-l));
      sb[i] = s[i] + a.bias[e];
    } else {
      s[i] = 0.f;
      sb[i] = ninf;
    }
  }

  // group scores: sum of the two largest biased scores of each group
  float gs[kMaxGroups];
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) {
    gs[g] = ninf;
    if (g < G) {
      float m1 = ninf, m2 = ninf;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E && e / P == g) top2_insert(sb[i], m1, m2);
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float o1 = __shfl_xor_sync(0xffffffffu, m1, off);
        const float o2 = __shfl_xor_sync(0xffffffffu, m2, off);
        const float hi = fmaxf(m1, o1);
        const float lo = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
        m1 = hi;
        m2 = lo;
      }
      gs[g] = P >= 2 ? m1 + m2 : m1;
    }
  }
  // keep the topk_group best groups (lower index wins ties)
  uint32_t kept = 0;
#pragma unroll
  for (int g = 0; g < kMaxGroups; ++g) {
    if (g >= G) break;
    int rank = 0;
#pragma unroll
    for (int g2 = 0; g2 < kMaxGroups; ++g2)
      if (g2 < G && (gs[g2] > gs[g] || (gs[g2] == gs[g] && g2 < g))) ++rank;
    if (rank < a.Gk) kept |= 1u << g;
  }

  // top_k experts among the kept groups by biased score (lower id wins ties)
  bool taken[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) taken[i] = false;
  int sel_e[kMaxTopK];
  float sel_s[kMaxTopK];
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    sel_e[r] = 0x7fffffff;
    sel_s[r] = 0.f;
    if (r < a.k) {
      float bv = ninf;
      int be = 0x7fffffff;
      float bs = 0.f;
#pragma unroll
      for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        if (e < E && !taken[i] && ((kept >> (e / P)) & 1u)) {
          if (sb[i] > bv || (sb[i] == bv && e < be)) {
            bv = sb[i];
            be = e;
            bs = s[i];
          }
        }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oe = __shfl_xor_sync(0xffffffffu, be, off);
        const float os = __shfl_xor_sync(0xffffffffu, bs, off);
        if (ov > bv || (ov == bv && oe < be)) {
          bv = ov;
          be = oe;
          bs = os;
        }
      }
      sel_e[r] = be;
      sel_s[r] = bs;
#pragma unroll
      for (int i = 0; i < kPer; ++i)
        if (lane + 32 * i == be) taken[i] = true;
    }
  }
  // ascending expert id (insertion sort, identical on every lane)
#pragma unroll
  for (int r = 1; r < kMaxTopK; ++r) {
#pragma unroll
    for (int q = r; q > 0; --q) {
      if (sel_e[q] < sel_e[q - 1]) {
        const int te = sel_e[q];
        sel_e[q] = sel_e[q - 1];
        sel_e[q - 1] = te;
        const float ts = sel_s[q];
        sel_s[q] = sel_s[q - 1];
        sel_s[q - 1] = ts;
      }
    }
  }
  float denom = 0.f;
#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r)
    if (r < a.k) denom += sel_s[r];

#pragma unroll
  for (int r = 0; r < kMaxTopK; ++r) {
    if (r < a.k && lane == r) {
      const int e = sel_e[r];
      const size_t slot = static_cast<size_t>(t) * a.k + r;
      if (e < 0 || e >= E) {  // no candidate left: cannot happen for a validated shape
        record_status(a.status, kDevAssert, kWhereSelect);
        a.idx[slot] = 0;
        a.w[slot] = 0.f;
        if (a.cnt) a.rank[slot] = -1;
        continue;
      }
      a.idx[slot] = e;
      a.w[slot] = a.norm ? a.scale * sel_s[r] / denom : a.scale * sel_s[r];
      if (a.cnt) a.rank[slot] = atomicAdd(a.cnt + e, 1);
    }
  }
}

}  // namespace

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
