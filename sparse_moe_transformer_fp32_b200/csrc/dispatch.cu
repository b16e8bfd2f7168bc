// Dispatch of token slots to experts: per-expert offsets and the m-tile list (one CTA), then
// the gather of each token's hidden row into the expert-contiguous buffer Xp.
//
// The pages say only that tokens are sent to the experts (and, under expert parallelism, to the
// GPUs) that hold them ("Use HF Transformers", section Parallelism).  Here the (token, slot)
// pairs are laid out expert by expert: expert e owns rows off[e] .. off[e+1]-1, and within an
// expert the order is the arrival order of the selection kernel's atomic counter.  Row order
// inside an expert does not change any result: every row is computed independently and the
// combine reads rows back through rowmap in a fixed slot order.
#include "beam_moe_internal.cuh"

namespace beam {
namespace {

// Inclusive scan of one int per thread over a block of 256 threads.
__device__ __forceinline__ int block_inclusive_scan(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, off);
    if (lane >= off) v += o;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  __syncthreads();
  return v + base;
}

__global__ void __launch_bounds__(256) dispatch_scan_kernel(const DispatchArgs a) {
  __shared__ int warp_tot[8];
  const int e = threadIdx.x;
  const int c = e < a.E ? a.cnt[e] : 0;
  const int tr = a.tile_rows;
  const int m = (c + tr - 1) / tr;
  const int c_incl = block_inclusive_scan(c, warp_tot);
  const int m_incl = block_inclusive_scan(m, warp_tot);
  const int c_excl = c_incl - c, m_excl = m_incl - m;
  if (e < a.E) a.off[e] = c_excl;
  if (e == a.E - 1) {
    a.off[a.E] = c_incl;
    *a.mt_count = m_incl;
  }
  for (int i = 0; i < m; ++i) {
    MTile t;
    t.e = e;
    t.row0 = c_excl + i * tr;
    t.nrows = min(tr, c - i * tr);
    t.pad = 0;
    a.mtiles[m_excl + i] = t;
  }
}

// One warp per token: the row is read once and written to each of its top_k destinations.
__global__ void __launch_bounds__(256) permute_kernel(const PermuteArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
  int row = -1;
  if (lane < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + lane;
    const int e = a.idx[slot];
    const int r = a.rank[slot];
    if (e >= 0 && e < a.E && r >= 0) {
      row = a.off[e] + r;
      if (row >= a.off[e + 1]) row = -1;
    }
    if (row < 0) record_status(a.status, kDevAssert, kWherePermute);
    a.rowmap[slot] = row;
  }
  int rows[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, row, j);

  const uint4* src = reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(t) * a.d);
  const int nvec = a.d / 8;
  for (int c = lane; c < nvec; c += 32) {
    const uint4 v = src[c];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k && rows[j] >= 0)
        reinterpret_cast<uint4*>(a.xp + static_cast<size_t>(rows[j]) * a.d)[c] = v;
    }
  }
}

// Dense MLP: every token belongs to the single group 0; tiles of up to kBM consecutive rows.
__global__ void dense_tiles_kernel(int T, MTile* mtiles, int32_t* mt_count) {
  const int n = (T + kBM - 1) / kBM;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    MTile t;
    t.e = 0;
    t.row0 = i * kBM;
    t.nrows = min(kBM, T - i * kBM);
    t.pad = 0;
    mtiles[i] = t;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) *mt_count = n;
}

// bias[e] += gamma * sign(mean - cnt[e])
__global__ void bias_update_kernel(const int32_t* cnt, float* bias, int E, float mean,
                                   float gamma) {
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < E; e += gridDim.x * blockDim.x) {
    const float c = static_cast<float>(cnt[e]);
    const float sgn = c < mean ? 1.f : (c > mean ? -1.f : 0.f);
    bias[e] += gamma * sgn;
  }
}

}  // namespace

cudaError_t launch_dense_tiles(int T, MTile* mtiles, int32_t* mt_count, cudaStream_t s) {
  const int n = (T + kBM - 1) / kBM;
  const int blocks = (n + 255) / 256 < 1 ? 1 : (n + 255) / 256;
  dense_tiles_kernel<<<blocks, 256, 0, s>>>(T, mtiles, mt_count);
  return cudaGetLastError();
}

cudaError_t launch_bias_update(const int32_t* cnt, float* bias, int E, float mean, float gamma,
                               cudaStream_t s) {
  bias_update_kernel<<<1, 256, 0, s>>>(cnt, bias, E, mean, gamma);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const DispatchArgs& a, cudaStream_t s) {
  dispatch_scan_kernel<<<1, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
  permute_kernel<<<(a.T + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
