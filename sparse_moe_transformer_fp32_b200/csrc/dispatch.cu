// Dispatch of token slots to experts: per-expert offsets, the m-tile list and the prefix counts
// of the token bitmap (a warp per expert), then the gather of each token's hidden row into the
// expert-contiguous buffer Xp.
//
// The pages say only that tokens are sent to the experts (and, under expert parallelism, to the
// GPUs) that hold them ("Use HF Transformers", section Parallelism).  Here the (token, slot)
// pairs are laid out expert by expert: expert e owns rows off[e] .. off[e+1]-1, in ascending
// token order (the rank of token t among e's rows is the number of set bits before bit t in e's
// row of the token bitmap).  The layout is therefore a function of the routing alone; no result
// depends on it in any case, since every row is computed independently and the combine reads
// rows back through rowmap in a fixed slot order.
#include "beam_moe_internal.cuh"
#include "beam_moe_div.cuh"

#include <cuda_fp8.h>

namespace beam {
namespace {

// A warp per expert e: the rows and m-tiles of the experts before e give its offset and its
// first m-tile, and the m-tile counts of its neighbours its raster band; the exclusive prefix
// counts of its row of the token bitmap give each of its tokens a rank.
__global__ void __launch_bounds__(256) dispatch_scan_kernel(const DispatchArgs a) {
  __shared__ int first_sh[8][kMaxE + 1];  // per warp: first m-tile of every expert, [E] = total
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= a.E) return;  // uniform over the warp
  const int tr = a.tile_rows;
  int* first = first_sh[warp];
  // lane l takes experts l * per .. l * per + per - 1: their counts are read once and give both
  // the row offsets and the m-tile offsets; the first words of e's bitmap row are fetched
  // meanwhile
  const int per = (a.E + 31) / 32;
  int cnt_l[kMaxE / 32];
  int msum = 0, csum = 0;
#pragma unroll
  for (int i = 0; i < kMaxE / 32; ++i) {
    const int ee = lane * per + i;
    cnt_l[i] = i < per && ee < a.E ? a.cnt[ee] : 0;
    msum += (cnt_l[i] + tr - 1) / tr;
    csum += cnt_l[i];
  }
  const uint32_t word0 = lane < a.words ? a.bits[static_cast<size_t>(e) * a.words + lane] : 0u;
  int mincl = msum, cincl = csum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int om = __shfl_up_sync(0xffffffffu, mincl, off);
    const int oc = __shfl_up_sync(0xffffffffu, cincl, off);
    if (lane >= off) {
      mincl += om;
      cincl += oc;
    }
  }
  {
    int run = mincl - msum;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i) {
      const int ee = lane * per + i;
      if (i < per && ee < a.E) {
        first[ee] = run;
        run += (cnt_l[i] + tr - 1) / tr;
      }
    }
    if (lane == 31) first[a.E] = mincl;
  }
  // rows of the experts before e: the owning lane's exclusive prefix plus its own experts
  // before e
  int c_before = 0;
  {
    const int owner = e / per;
    int pre = cincl - csum;
#pragma unroll
    for (int i = 0; i < kMaxE / 32; ++i)
      if (i < e - owner * per) pre += cnt_l[i];
    c_before = __shfl_sync(0xffffffffu, pre, owner);
  }
  __syncwarp();
  const int c = a.cnt[e];
  const int m_before = first[e];
  const int m = first[e + 1] - m_before;
  if (lane == 0) {
    a.off[e] = c_before;
    if (e == a.E - 1) {
      a.off[a.E] = c_before + c;
      *a.mt_count = first[a.E];
    }
  }
  // raster band of a small expert (at most kBand m-tiles): the run of neighbouring small
  // experts whose first m-tile lies in the same block of kBand m-tiles
  int run_start = 0, run_end = 0;
  if (m > 0 && m <= kBand) {
    const int key = m_before / kBand;
    auto small_in_block = [&](int x) {
      const int mx = first[x + 1] - first[x];
      return mx <= kBand && first[x] / kBand == key;
    };
    int lo = e, hi = e;
    while (lo > 0 && small_in_block(lo - 1)) --lo;
    while (hi + 1 < a.E && small_in_block(hi + 1)) ++hi;
    run_start = first[lo];
    run_end = first[hi + 1];
  }
  for (int i = lane; i < m; i += 32) {
    MTile t;
    t.e = e;
    t.row0 = c_before + i * tr;
    t.nrows = min(tr, c - i * tr);
    if (m <= kBand) {
      t.band = pack_band(run_start, run_end - run_start);
    } else {  // a large expert: bands of kBand of its own m-tiles
      const int b0 = (i / kBand) * kBand;
      t.band = pack_band(m_before + b0, min(kBand, m - b0));
    }
    a.mtiles[m_before + i] = t;
  }
  const uint32_t* bits = a.bits + static_cast<size_t>(e) * a.words;
  int32_t* base = a.base + static_cast<size_t>(e) * a.words;
  int run = 0;
  for (int w0 = 0; w0 < a.words; w0 += 32) {
    const int w = w0 + lane;
    const int n = w < a.words ? __popc(w0 == 0 ? word0 : bits[w]) : 0;
    int incl = n;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    if (w < a.words) base[w] = run + incl - n;
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
}

// ---- E4M3 row quantisation helpers (FP8 expert weights; see quantize_rows_kernel)
//
// s = fl32(amax / 448) over the row, q = e4m3(fl32(x / s)) with round-to-nearest-even and
// saturation (cvt.rn.satfinite); an all-zero row has s = 0 and zero codes.

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Scale of a row of nvec 8-element chunks read by the 32 lanes of a warp (all lanes return it).
__device__ __forceinline__ float row_scale_e4m3(const uint4* src, int nvec, int lane) {
  float amax = 0.f;
  for (int c = lane; c < nvec; c += 32) {
    const uint4 v = src[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  }
  // non-negative floats order like their bit patterns
  amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
  return amax / 448.0f;
}

// The quotients x / s are correctly rounded (div_rn_by with r = RN(1 / s), or the division
// itself for a row scale outside div_rn_by's range).
__device__ __forceinline__ uint2 quantize8_e4m3(const uint4 v, float s, float r) {
  if (s == 0.f) return make_uint2(0u, 0u);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t p[4];
  if (div_rn_by_applies(s)) {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      p[i] = __nv_cvt_float2_to_fp8x2(
          make_float2(div_rn_by(bf16_lo(w[i]), s, r), div_rn_by(bf16_hi(w[i]), s, r)),
          __NV_SATFINITE, __NV_E4M3);
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i)
      p[i] = __nv_cvt_float2_to_fp8x2(make_float2(bf16_lo(w[i]) / s, bf16_hi(w[i]) / s),
                                      __NV_SATFINITE, __NV_E4M3);
  }
  return make_uint2(p[0] | (p[1] << 16), p[2] | (p[3] << 16));
}

// E4M3 permute, four warps per token and two tokens per CTA: the row is read once, quantised
// (each warp a quarter of it, after the four warps have combined their quarters' maxima into
// the row scale), and its codes written to each of its top_k destinations.  (One warp per
// token left the SMs a third occupied.)
constexpr int kPermWarpsPerToken = 4;
constexpr int kPermTokensPerCta = 8 / kPermWarpsPerToken;

__global__ void __launch_bounds__(256) permute_kernel(const PermuteArgs a) {
  __shared__ float part_max[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = warp % kPermWarpsPerToken;
  const int t = blockIdx.x * kPermTokensPerCta + warp / kPermWarpsPerToken;
  const bool live = t < a.T;
  const uint4* src = reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(live ? t : 0) * a.d);
  const int per = a.d / 8 / kPermWarpsPerToken;  // 8-element chunks per warp (d % 256 == 0)
  {
    float amax = 0.f;
    if (live)
      for (int c = part * per + lane; c < (part + 1) * per; c += 32) {
        const uint4 v = src[c];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
      }
    // non-negative floats order like their bit patterns
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (lane == 0) part_max[warp] = amax;
  }
  __syncthreads();
  if (!live) return;
  const int w0 = warp - part;
  const float s = fmaxf(fmaxf(part_max[w0], part_max[w0 + 1]),
                        fmaxf(part_max[w0 + 2], part_max[w0 + 3])) /
                  448.0f;  // the row scale, as row_scale_e4m3 forms it
  const float r = __frcp_rn(s);

  int row = -1;
  if (lane < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + lane;
    const int e = a.idx[slot];
    const int r = e >= 0 && e < a.E ? slot_rank(a.bits, a.base, a.words, e, t) : -1;
    if (r >= 0) {
      row = a.off[e] + r;
      if (row >= a.off[e + 1]) row = -1;
    }
    if (part == 0) {
      if (row < 0) record_status(a.status, kDevAssert, kWherePermute);
      a.rowmap[slot] = row;
      if (row >= 0) a.xs[row] = s;
    }
  }
  int rows[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, row, j);
  for (int c = part * per + lane; c < (part + 1) * per; c += 32) {
    const uint2 q = quantize8_e4m3(src[c], s, r);
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k && rows[j] >= 0)
        reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(rows[j]) * a.d)[c] = q;
    }
  }
}

constexpr uint64_t kPermuteWaitNs = 4000000000ull;  // bound of the row copy's wait for its load

// 1-D bulk copy global -> shared completing on mbarrier `bar` (16-byte aligned addresses, bytes
// a multiple of 16).
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void* src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// 1-D bulk copy shared -> global in the thread's current bulk group.
__device__ __forceinline__ void bulk_store_1d(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}

// Closes the thread's bulk group and waits until its shared-memory sources have been read.
__device__ __forceinline__ void bulk_commit_wait_read() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// BF16 permute by bulk copies: a CTA of one warp per token.  Lanes below top_k form their
// slots' rows; lane 0 reads the token row into shared memory with one bulk copy and writes it
// to each of its rows with bulk stores, then waits until those have read shared memory.
__global__ void __launch_bounds__(32) permute_bulk_kernel(const PermuteArgs a) {
  extern __shared__ __align__(128) uint8_t row_sh[];
  __shared__ __align__(8) uint64_t bar_sh;
  const int lane = threadIdx.x;
  const int t = blockIdx.x;
  int row = -1;
  if (lane < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + lane;
    const int e = a.idx[slot];
    const int r = e >= 0 && e < a.E ? slot_rank(a.bits, a.base, a.words, e, t) : -1;
    if (r >= 0) {
      row = a.off[e] + r;
      if (row >= a.off[e + 1]) row = -1;
    }
    if (row < 0) record_status(a.status, kDevAssert, kWherePermute);
    a.rowmap[slot] = row;
  }
  int rows[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) rows[j] = __shfl_sync(0xffffffffu, row, j);
  if (lane != 0) return;
  const uint32_t bar = smem_u32(&bar_sh);
  const uint32_t bytes = static_cast<uint32_t>(a.d) * 2u;
  mbar_init(bar, 1);
  fence_mbarrier_init();
  mbar_arrive_expect_tx(bar, bytes);
  bulk_load_1d(smem_u32(row_sh), a.h + static_cast<size_t>(t) * a.d, bytes, bar);
  int abort_flag = 0;
  if (!mbar_wait_bounded(bar, 0, &abort_flag, kPermuteWaitNs, a.status, kWherePermute)) {
    // the load must land before this CTA's shared memory is released
    int no_abort = 0;
    mbar_wait_bounded(bar, 0, &no_abort, 1000000000ull, a.status, kWherePermute);
    return;
  }
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < a.k && rows[j] >= 0)
      bulk_store_1d(a.xp + static_cast<size_t>(rows[j]) * a.d, smem_u32(row_sh), bytes);
  bulk_commit_wait_read();
}

// Row-wise E4M3 quantisation of a BF16 matrix [rows, cols]: one warp per row.
__global__ void __launch_bounds__(256) quantize_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                            int64_t rows, int cols,
                                                            uint8_t* __restrict__ q,
                                                            float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int64_t r = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + r * cols);
  const int nvec = cols / 8;
  const float s = row_scale_e4m3(src, nvec, lane);
  if (lane == 0) scale[r] = s;
  uint2* dst = reinterpret_cast<uint2*>(q + r * cols);
  const float rs = __frcp_rn(s);
  for (int c = lane; c < nvec; c += 32) dst[c] = quantize8_e4m3(src[c], s, rs);
}

// Dense MLP: every token belongs to the single group 0; tiles of up to kBM consecutive rows.
__global__ void dense_tiles_kernel(int T, MTile* mtiles, int32_t* mt_count) {
  const int n = (T + kBM - 1) / kBM;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    MTile t;
    t.e = 0;
    t.row0 = i * kBM;
    t.nrows = min(kBM, T - i * kBM);
    const int b0 = (i / kBand) * kBand;
    t.band = pack_band(b0, min(kBand, n - b0));
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

cudaError_t launch_quantize_rows(const __nv_bfloat16* x, int64_t rows, int cols, uint8_t* q,
                                 float* scale, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int64_t blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  quantize_rows_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, rows, cols, q, scale);
  return cudaGetLastError();
}

cudaError_t launch_dispatch_scan(const DispatchArgs& a, cudaStream_t s) {
  dispatch_scan_kernel<<<(a.E + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s) {
  if (!a.xq)  // BF16 rows: bulk copies
    permute_bulk_kernel<<<a.T, 32, static_cast<size_t>(a.d) * 2, s>>>(a);
  else        // E4M3 rows: quantised by the warps that read them
    permute_kernel<<<(a.T + kPermTokensPerCta - 1) / kPermTokensPerCta, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
