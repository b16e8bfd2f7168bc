// Combine of the expert outputs, and the block form's FP32 RMSNorms and depth-scaled residual.
//
// Combine (Transformers model doc "Beam", Overview, "Sparse MoE" bullet; no shared expert):
//   out[t] = sum_j w[t, j] * Y[rowmap[t, j]], j in ascending expert id, FP32 accumulation.
// Block (Overview, "Sandwich norms with depth-scaled residuals"; archdb fact sheet
// "Beam-1.0-501B-A23B", residual-design entry; rms_norm_eps from BeamConfig):
//   h  = bf16( x / sqrt(mean(x^2) + eps) * g_pre )
//   o  = out / sqrt(mean(out^2) + eps) * g_post
//   x' = x * sqrt((k-1)/k) + o / sqrt(k)
// One CTA per token; row sums of squares are reduced in a fixed order (per-thread strided
// partials, warp butterfly, then warps in index order), so results are deterministic.
#include "beam_moe_internal.cuh"

namespace beam {
namespace {

constexpr int kCThreads = 128;
constexpr int kMaxVec = kMaxD / 8 / kCThreads;  // 8-element vectors per thread at d = kMaxD

__device__ __forceinline__ void unpack_bf16x8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// Sum over the CTA in a fixed order; every thread gets the total.
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < kCThreads / 32; ++w) tot += red[w];
  __syncthreads();
  return tot;
}

// Loads the token's slot rows and weights into shared memory; invalid rows weigh nothing.
__device__ __forceinline__ void load_slots(const CombineArgs& a, int t, int* rows, float* ws) {
  if (threadIdx.x < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + threadIdx.x;
    int r = a.rowmap[slot];
    float w = a.w[slot];
    if (r < 0 || r >= a.R) {
      record_status(a.status, kDevAssert, kWhereCombine);
      r = 0;
      w = 0.f;
    }
    rows[threadIdx.x] = r;
    ws[threadIdx.x] = w;
  }
  __syncthreads();
}

// kPrefetch: all k row loads are issued before the sums that consume them (which stay in slot
// order); it helps the layer combine and costs the block form occupancy (more registers), so
// the block form loads a row at a time.
template <bool kPrefetch>
__device__ __forceinline__ void combine_vec(const CombineArgs& a, const int* rows, const float* ws,
                                            int c, float (&acc)[8]) {
#pragma unroll
  for (int q = 0; q < 8; ++q) acc[q] = 0.f;
  if constexpr (!kPrefetch) {
    for (int j = 0; j < a.k; ++j) {
      const uint4 v =
          reinterpret_cast<const uint4*>(a.y + static_cast<size_t>(rows[j]) * a.d)[c];
      float f[8];
      unpack_bf16x8(v, f);
#pragma unroll
      for (int q = 0; q < 8; ++q) acc[q] = fmaf(ws[j], f[q], acc[q]);
    }
  } else {
    uint4 v[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < a.k)
        v[j] = reinterpret_cast<const uint4*>(a.y + static_cast<size_t>(rows[j]) * a.d)[c];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k) {
        float f[8];
        unpack_bf16x8(v[j], f);
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] = fmaf(ws[j], f[q], acc[q]);
      }
    }
  }
}

// A token row in `chunks` CTAs (contiguous runs of its 16-byte pieces): few tokens, as at
// decode, still give every SM loads to keep in flight.
__global__ void __launch_bounds__(kCThreads) combine_kernel(const CombineArgs a, int chunks) {
  __shared__ int rows[kMaxTopK];
  __shared__ float ws[kMaxTopK];
  const int t = blockIdx.x / chunks;
  const int chunk = blockIdx.x - t * chunks;
  load_slots(a, t, rows, ws);
  const int nvec = a.d / 8;
  const int per = (nvec + chunks - 1) / chunks;
  const int c_end = min(nvec, (chunk + 1) * per);
  uint4* out = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.d);
  for (int c = chunk * per + threadIdx.x; c < c_end; c += kCThreads) {
    float acc[8];
    combine_vec<true>(a, rows, ws, c, acc);
    out[c] = make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                        pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
  }
}

__global__ void __launch_bounds__(kCThreads) combine_block_kernel(const CombineArgs a) {
  __shared__ int rows[kMaxTopK];
  __shared__ float ws[kMaxTopK];
  __shared__ float red[kCThreads / 32];
  const int t = blockIdx.x;
  load_slots(a, t, rows, ws);
  const int nvec = a.d / 8;
  float o[kMaxVec][8];
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < kMaxVec; ++v) {
    const int c = threadIdx.x + v * kCThreads;
    if (c < nvec) {
      combine_vec<false>(a, rows, ws, c, o[v]);
#pragma unroll
      for (int q = 0; q < 8; ++q) ss = fmaf(o[v][q], o[v][q], ss);
    }
  }
  const float inv = rsqrtf(block_sum(ss, red) / static_cast<float>(a.d) + a.eps);
  const float4* xr = reinterpret_cast<const float4*>(a.x + static_cast<size_t>(t) * a.d);
  const float4* gr = reinterpret_cast<const float4*>(a.g_post);
  float4* xo = reinterpret_cast<float4*>(a.x_out + static_cast<size_t>(t) * a.d);
#pragma unroll
  for (int v = 0; v < kMaxVec; ++v) {
    const int c = threadIdx.x + v * kCThreads;
    if (c < nvec) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float4 x = xr[2 * c + h];
        const float4 g = gr[2 * c + h];
        float4 r;
        r.x = fmaf(x.x, a.coef_x, o[v][4 * h + 0] * inv * g.x * a.coef_f);
        r.y = fmaf(x.y, a.coef_x, o[v][4 * h + 1] * inv * g.y * a.coef_f);
        r.z = fmaf(x.z, a.coef_x, o[v][4 * h + 2] * inv * g.z * a.coef_f);
        r.w = fmaf(x.w, a.coef_x, o[v][4 * h + 3] * inv * g.w * a.coef_f);
        xo[2 * c + h] = r;
      }
    }
  }
}

__global__ void __launch_bounds__(kCThreads) prenorm_kernel(const PreNormArgs a) {
  __shared__ float red[kCThreads / 32];
  const int t = blockIdx.x;
  const int nvec = a.d / 8;
  const float4* xr = reinterpret_cast<const float4*>(a.x + static_cast<size_t>(t) * a.d);
  const float4* gr = reinterpret_cast<const float4*>(a.g_pre);
  float4 xv[kMaxVec][2];
  float ss = 0.f;
#pragma unroll
  for (int v = 0; v < kMaxVec; ++v) {
    const int c = threadIdx.x + v * kCThreads;
    if (c < nvec) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        xv[v][h] = xr[2 * c + h];
        ss = fmaf(xv[v][h].x, xv[v][h].x, ss);
        ss = fmaf(xv[v][h].y, xv[v][h].y, ss);
        ss = fmaf(xv[v][h].z, xv[v][h].z, ss);
        ss = fmaf(xv[v][h].w, xv[v][h].w, ss);
      }
    }
  }
  const float inv = rsqrtf(block_sum(ss, red) / static_cast<float>(a.d) + a.eps);
  uint4* hr = reinterpret_cast<uint4*>(a.h + static_cast<size_t>(t) * a.d);
#pragma unroll
  for (int v = 0; v < kMaxVec; ++v) {
    const int c = threadIdx.x + v * kCThreads;
    if (c < nvec) {
      const float4 g0 = gr[2 * c], g1 = gr[2 * c + 1];
      const float4 x0 = xv[v][0], x1 = xv[v][1];
      hr[c] = make_uint4(pack_bf16x2(x0.x * inv * g0.x, x0.y * inv * g0.y),
                         pack_bf16x2(x0.z * inv * g0.z, x0.w * inv * g0.w),
                         pack_bf16x2(x1.x * inv * g1.x, x1.y * inv * g1.y),
                         pack_bf16x2(x1.z * inv * g1.z, x1.w * inv * g1.w));
    }
  }
}

}  // namespace

cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s) {
  // about four CTAs per SM at least, one piece per thread at most
  const int nvec = a.d / 8;
  const int max_chunks = (nvec + kCThreads - 1) / kCThreads;
  const int want = (4 * 148 + a.T - 1) / a.T;
  const int chunks = want < 1 ? 1 : (want > max_chunks ? max_chunks : want);
  combine_kernel<<<static_cast<unsigned>(a.T) * chunks, kCThreads, 0, s>>>(a, chunks);
  return cudaGetLastError();
}

cudaError_t launch_combine_block(const CombineArgs& a, cudaStream_t s) {
  combine_block_kernel<<<a.T, kCThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_prenorm(const PreNormArgs& a, cudaStream_t s) {
  prenorm_kernel<<<a.T, kCThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
