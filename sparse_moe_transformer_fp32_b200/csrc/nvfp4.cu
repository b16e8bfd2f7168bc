// NVFP4 expert weights: the quantisers and the block-scaled grouped expert GEMMs.
//
// The SwiGLU experts (Transformers model doc "Beam", Overview; news article "Reflection lança o
// Beam", "cada expert é um MLP SwiGLU") run with E2M1 weights and activations, an E4M3 scale
// per 16 elements along K and an FP32 scale per row (the format is stated in
// beam_moe_nvfp4.cuh).  The tensor cores apply the block scales
// (tcgen05.mma.kind::mxf4nvf4.block_scale.block16); the epilogue applies the two row scales.
//
//   GEMM1 (gate|up + SwiGLU): the gate and up weights are interleaved in 64-row chunks, so a
//       128-row weight tile n holds gate rows 64n..64n+63 and the same up rows:
//       D[128 x 128] = Xq[rows, :] . Wgu,e[128n .. 128n+127, :]^T     (block-scaled, FP32)
//       act[rows, 64n + c] = bf16( silu(D[:, c] sa sg) * D[:, 64 + c] sa su ),  c < 64
//   the activation is then quantised to NVFP4 per row (a kernel of its own);
//   GEMM2 (down): Y[rows, 128n + c] = bf16( Aq[rows, :] . Wd,e[128n + c, :]^T  sa sd ).
//
// Kernel structure as the BF16/E4M3 expert GEMM (persistent, one CTA per SM), plus a warp
// that copies the block scales into TMEM (224 threads):
//   warp 0     one thread issues, per 256-element K stage, TMA loads of the A codes (box sized
//              to the tile's rows) and the B codes, and bulk copies of their block scales (A 8 KB,
//              B 2 KB; layouts in beam_moe_nvfp4.cuh), into a 5-stage ring
//   warp 6     one thread copies each landed stage's block scales into that stage's 32 TMEM
//              columns (A: two tcgen05.cp.128x256b, two K steps each; B: one
//              tcgen05.cp.32x128b.warpx4 per K step, as the MMA reads B's scales in every lane
//              quarter) and commits them to the stage's scales-ready barrier
//   warp 1     allocates 512 TMEM columns (two 128-column accumulators at 0 and 128, the
//              stages' block scales at 256..415); one thread issues four M=128 N=128 K=64 MMAs
//              per stage once its codes and scales are in.  (Copies issued by the MMA thread
//              itself ran strictly between its MMAs: gate/up 15 % slower.)
//   warps 2-5  epilogue: tcgen05.ld of the accumulator, row scales, SwiGLU / BF16 conversion
// Rows of a tile beyond its valid rows read stale codes and unwritten scales; they only feed
// accumulator rows that are never stored.
//
// Every wait is bounded (globaltimer); on a timeout the kernel records it in the status word,
// raises a CTA-wide abort flag, waits for its own copies and MMAs, frees TMEM and returns.
#include "beam_moe_nvfp4.cuh"
#include "beam_moe_div.cuh"

#include <cuda_fp4.h>
#include <cuda_fp8.h>

namespace beam {
namespace {

constexpr uint64_t kMinDrainNs = 1000000000ull;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Row scale s = amax / 2688 of a BF16 row of nvec 8-element chunks (all lanes return it).
__device__ __forceinline__ float nvfp4_row_scale(const uint4* src, int nvec, int lane) {
  float amax = 0.f;
  for (int c = lane; c < nvec; c += 32) {
    const uint4 v = src[c];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[i])), fabsf(bf16_hi(w[i]))));
  }
  amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
  return amax / 2688.0f;
}

// One 16-element block (chunks c0, c1 of 8 BF16 values) with row scale s: returns its 8 code
// bytes and sets its E4M3 block-scale code.
__device__ __forceinline__ uint2 nvfp4_block(const uint4 c0, const uint4 c1, float s,
                                             uint8_t& bs) {
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
  float v[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_lo(w[i]);
    v[2 * i + 1] = bf16_hi(w[i]);
  }
  float mb = 0.f;
#pragma unroll
  for (int i = 0; i < 16; ++i) mb = fmaxf(mb, fabsf(v[i]));
  uint8_t code = 0;
  if (s > 0.f) {
    float t = mb / s;
    t = t / 6.0f;
    code = static_cast<uint8_t>(__nv_cvt_float_to_fp8(t, __NV_SATFINITE, __NV_E4M3));
  }
  bs = code;
  const __half_raw hr = __nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(code), __NV_E4M3);
  const float den = s * __half2float(__half(hr));
  if (!(den > 0.f)) return make_uint2(0u, 0u);
  // the quotients x / den correctly rounded: div_rn_by with one reciprocal per block, or the
  // division itself for a block scale outside its range
  float q[16];
  if (div_rn_by_applies(den)) {
    const float rden = __frcp_rn(den);
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = div_rn_by(v[i], den, rden);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) q[i] = v[i] / den;
  }
  uint32_t p[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t b =
        __nv_cvt_float2_to_fp4x2(make_float2(q[2 * i], q[2 * i + 1]), __NV_E2M1, cudaRoundNearest);
    p[i >> 2] |= b << (8 * (i & 3));
  }
  return make_uint2(p[0], p[1]);
}

// The four block scales of a 64-element K step, held by lanes 4u .. 4u + 3 (block 4u + i in
// lane 4u + i), packed into one word for lane 4u (byte i = block i).  All 32 lanes take part.
__device__ __forceinline__ uint32_t gather_step_scales(uint8_t bs) {
  const uint32_t b = bs;
  return b | (__shfl_down_sync(0xffffffffu, b, 1) << 8) |
         (__shfl_down_sync(0xffffffffu, b, 2) << 16) | (__shfl_down_sync(0xffffffffu, b, 3) << 24);
}

// Inclusive scan of one int per thread over a block of 256 threads.
__device__ __forceinline__ int block_scan256(int v, int* warp_tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_tot[warp] = v;
  __syncthreads();
  int base = 0;
  for (int w = 0; w < warp; ++w) base += warp_tot[w];
  __syncthreads();
  return v + base;
}

// ------------------------------------------------------------------ quantisers

// One warp per output row of [groups, rows_out, cols]; rows_out = 2 * rows when interleaving.
__global__ void __launch_bounds__(256) nvfp4_weights_kernel(const __nv_bfloat16* __restrict__ a,
                                                            const __nv_bfloat16* __restrict__ b,
                                                            int64_t groups, int rows, int cols,
                                                            uint8_t* __restrict__ codes,
                                                            uint8_t* __restrict__ sf,
                                                            float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int rows_out = b ? 2 * rows : rows;
  const int64_t o = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (o >= groups * rows_out) return;
  const int64_t g = o / rows_out;
  const int p = static_cast<int>(o - g * rows_out);
  const __nv_bfloat16* src;
  if (b) {
    const int c = p >> 7, w = p & 127;
    src = (w < 64 ? a : b) + (g * rows + 64 * c + (w & 63)) * static_cast<int64_t>(cols);
  } else {
    src = a + (g * rows + p) * static_cast<int64_t>(cols);
  }
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  const float s = nvfp4_row_scale(s4, cols / 8, lane);
  if (lane == 0) scale[o] = s;
  uint2* dst = reinterpret_cast<uint2*>(codes + o * (cols / 2));
  uint8_t* atoms = sf + (o >> 7) * (static_cast<int64_t>(cols) / 16) * 128;
  const int r = static_cast<int>(o & 127);
  for (int j = lane; j < cols / 16; j += 32) {
    uint8_t bs;
    dst[j] = nvfp4_block(s4[2 * j], s4[2 * j + 1], s, bs);
    atoms[nvfp4_sf_offset(r, j)] = bs;
  }
}

// Four warps per token, two tokens per CTA: the token row is quantised once (each warp a
// quarter of its 16-element blocks, after the four warps have combined their quarters' maxima
// into the row scale) and its codes, block scales and row scale written to each of its top_k
// rows.  The block scales of a row belong to its m-tile: m-tiles are numbered expert by
// expert, ceil(cnt[e] / 128) each.  (One warp per token left the SMs a third occupied.)
constexpr int kPermWarpsPerToken = 4;
constexpr int kPermTokensPerCta = 8 / kPermWarpsPerToken;

__global__ void __launch_bounds__(256) nvfp4_permute_kernel(const Fp4PermuteArgs a) {
  __shared__ int tile_off[kMaxE];
  __shared__ int warp_tot[8];
  __shared__ float part_max[8];
  const int e_t = threadIdx.x;
  const int c = e_t < a.E ? a.cnt[e_t] : 0;
  const int m = (c + kBM - 1) / kBM;
  const int incl = block_scan256(m, warp_tot);
  if (e_t < a.E) tile_off[e_t] = incl - m;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int part = warp % kPermWarpsPerToken;
  const int t = blockIdx.x * kPermTokensPerCta + warp / kPermWarpsPerToken;
  const bool live = t < a.T;
  const uint4* src = reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(live ? t : 0) * a.d);
  {
    const int per = a.d / 8 / kPermWarpsPerToken;  // 8-element chunks per warp (d % 256 == 0)
    float amax = 0.f;
    if (live)
      for (int ch = part * per + lane; ch < (part + 1) * per; ch += 32) {
        const uint4 v = src[ch];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(w[q])), fabsf(bf16_hi(w[q]))));
      }
    amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
    if (lane == 0) part_max[warp] = amax;
  }
  __syncthreads();  // tile_off and the quarters' maxima
  if (!live) return;
  const int w0 = warp - part;
  const float amax = fmaxf(fmaxf(part_max[w0], part_max[w0 + 1]),
                           fmaxf(part_max[w0 + 2], part_max[w0 + 3]));
  const float s = amax / 2688.0f;  // the row scale, as nvfp4_row_scale forms it

  int row = -1, tile = 0, rin = 0;  // rin: the slot's row inside its m-tile
  if (lane < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + lane;
    const int e = a.idx[slot];
    const int r = e >= 0 && e < a.E ? slot_rank(a.bits, a.base, a.words, e, t) : -1;
    if (r >= 0) {
      row = a.off[e] + r;
      if (row >= a.off[e + 1]) row = -1;
      tile = tile_off[e] + r / kBM;
      rin = r & (kBM - 1);
    }
    if (part == 0) {
      if (row < 0) record_status(a.status, kDevAssert, kWherePermute);
      a.rowmap[slot] = row;
      if (row >= 0) a.xs[row] = s;
    }
  }
  int rows[kMaxTopK], rins[kMaxTopK];
  uint8_t* atoms[kMaxTopK];
  const int64_t group_bytes = static_cast<int64_t>(a.d) / kF4KElems * kF4SfaBytes;
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, row, j);
    rins[j] = __shfl_sync(0xffffffffu, rin, j);
    const int tj = __shfl_sync(0xffffffffu, tile, j);
    atoms[j] = a.xsf + tj * group_bytes;
  }
  const int nb = a.d / 16 / kPermWarpsPerToken;  // 16-element blocks per warp (a multiple of 4)
  for (int jb0 = part * nb; jb0 < (part + 1) * nb; jb0 += 32) {
    const int jb = jb0 + lane;
    const bool act = jb < (part + 1) * nb;
    uint8_t bs = 0;
    uint2 q = make_uint2(0u, 0u);
    if (act) q = nvfp4_block(src[2 * jb], src[2 * jb + 1], s, bs);
    const uint32_t step = gather_step_scales(bs);
    if (act) {
#pragma unroll
      for (int j = 0; j < kMaxTopK; ++j) {
        if (j < a.k && rows[j] >= 0) {
          reinterpret_cast<uint2*>(a.xq + static_cast<size_t>(rows[j]) * (a.d / 2))[jb] = q;
          // the row's whole 16 bytes, its word in every position: a token's k rows lie in
          // k different m-tiles, and single bytes there left the sectors partly written
          if ((lane & 3) == 0)
            *reinterpret_cast<uint4*>(atoms[j] + (nvfp4_sfa_offset(rins[j], jb) & ~size_t{15})) =
                make_uint4(step, step, step, step);
        }
      }
    }
  }
}

// Rows of an m-tile quantised into the tile's block-scale atoms: 16 CTAs per m-tile, each
// taking 8 of its 128 rows, a warp per row (a CTA per tile alone leaves most SMs idle when the
// tiles are few and the rows long, as in the dense MLP).
constexpr int kActRowsPerCta = 8;
constexpr int kActCtasPerTile = kBM / kActRowsPerCta;

__global__ void __launch_bounds__(256) nvfp4_act_kernel(const Fp4ActArgs a) {
  const int mt = static_cast<int>(blockIdx.x / kActCtasPerTile);
  if (mt >= *a.mt_count) return;
  const MTile tile = a.mtiles[mt];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = static_cast<int>(blockIdx.x % kActCtasPerTile) * kActRowsPerCta + warp;
  if (r >= tile.nrows) return;  // uniform over the warp
  uint8_t* atoms = a.sf + static_cast<int64_t>(mt) * (a.cols / kF4KElems) * kF4SfaBytes;
  const int64_t row = tile.row0 + r;
  const uint4* src = reinterpret_cast<const uint4*>(a.x + row * a.cols);
  const float s = nvfp4_row_scale(src, a.cols / 8, lane);
  if (lane == 0) a.s[row] = s;
  uint2* dst = reinterpret_cast<uint2*>(a.q + row * (a.cols / 2));
  for (int jb = lane; jb < a.cols / 16; jb += 32) {
    uint8_t bs;
    dst[jb] = nvfp4_block(src[2 * jb], src[2 * jb + 1], s, bs);
    atoms[nvfp4_sfa_offset(r, jb)] = bs;
  }
}

// ------------------------------------------------------------------ block-scaled GEMM

// 1-D bulk copy global -> shared completing on mbarrier `bar` (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// Shared-memory descriptor of 32 rows x 16 bytes, rows contiguous, no swizzle (K-major
// interleaved layout: 8-row core matrices 128 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sf(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  desc |= static_cast<uint64_t>(128u >> 4) << 16;  // leading offset (one 16-byte column here)
  desc |= static_cast<uint64_t>(128u >> 4) << 32;  // stride between 8-row core matrices
  desc |= static_cast<uint64_t>(1u) << 46;
  return desc;  // layout type 0: no swizzle
}

// Shared-memory descriptor of 128 rows x 32 bytes, no swizzle: row L's first 16 bytes at
// 16 L, its second 16 bytes 2 KB further (8-row core matrices 128 bytes apart, the two 16-byte
// columns 2048 bytes apart).
__device__ __forceinline__ uint64_t smem_desc_sf_pair(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  desc |= static_cast<uint64_t>(2048u >> 4) << 16;  // leading offset: the second 16-byte column
  desc |= static_cast<uint64_t>(128u >> 4) << 32;   // stride between 8-row core matrices
  desc |= static_cast<uint64_t>(1u) << 46;
  return desc;  // layout type 0: no swizzle
}

// 128 TMEM lanes x 256 bits (8 columns) from shared memory: lane L gets row L, its first 16
// bytes in columns 0..3 and its second in columns 4..7.
__device__ __forceinline__ void tmem_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// 32 TMEM lanes x 128 bits from shared memory, repeated into all four lane quarters.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[tmem] (+)= (A . B^T) with E2M1 operands and E4M3 scales per 16 elements of K taken from
// TMEM (sfa: A's rows, sfb: B's rows); K = 64 per instruction.
__device__ __forceinline__ void umma_nvfp4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;"
      "\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Block-scaled instruction descriptor: A and B E2M1 (bits 7..9 and 10..12 = 1), both K-major,
// N >> 3 in 17..22, scale type UE4M3 (bit 23 = 0), M >> 4 in 24..28, scale-factor ids 0.
__host__ __device__ constexpr uint32_t umma_idesc_nvfp4(int M, int N) {
  return (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }

// v[j] *= sa * s[j] for 32 consecutive columns (s 16-byte aligned, the same across the warp).
__device__ __forceinline__ void scale32(uint32_t (&v)[32], float sa, const float* s) {
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 s4 = reinterpret_cast<const float4*>(s)[q];
    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) v[4 * q + i] = __float_as_uint(__uint_as_float(v[4 * q + i]) * sa * sv[i]);
  }
}

constexpr uint32_t kF4TmemCols = 512;
// Block scales of stage s in TMEM: A's at column 256 + 32 s (16 columns), B's 16 further.
constexpr uint32_t kF4SfCol = 256, kF4SfStageCols = 32;
static_assert(kF4SfCol + kF4SfStageCols * kF4Stages <= kF4TmemCols, "scale columns fit in TMEM");

template <bool kSwiGLU>
__global__ void __launch_bounds__(kF4Threads, 1)
    expert_gemm_nvfp4_kernel(const __grid_constant__ ATensorMaps tmA,
                             const __grid_constant__ CUtensorMap tmB, const Fp4GemmArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (sbase - raw);
  // [kF4Stages x (A 16 KB | B 16 KB | SFA 8 KB | SFB 2 KB)][barriers][TMEM address][abort flag]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kF4Stages * kF4StageBytes);
  constexpr int kBarFull = 0, kBarEmpty = kF4Stages, kBarTFull = 2 * kF4Stages,
                kBarTEmpty = kBarTFull + 2, kBarDrain = kBarTEmpty + 2,
                kBarSReady = kBarDrain + 1, kBarCopyDrain = kBarSReady + kF4Stages,
                kNumBars = kBarCopyDrain + 1;
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < kF4Stages; ++s) {
      mbar_init(bar(kBarFull + s), 1);
      mbar_init(bar(kBarEmpty + s), 1);
      mbar_init(bar(kBarSReady + s), 1);
    }
    mbar_init(bar(kBarCopyDrain), 1);
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
    tma_prefetch_desc(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), kF4TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int64_t sfa_group = static_cast<int64_t>(a.k_blocks) * kF4SfaBytes;  // per 128 rows
  const int64_t sfb_group = static_cast<int64_t>(a.k_blocks) * kF4SfBytes;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0, filled = 0, last_parity = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        int mt, n;
        band_decode_tile(a.mtiles, t, n_tiles, mt, n);
        const MTile m = a.mtiles[mt];
        const int brow = m.e * a.b_rows_per_expert + n * kF4N;
        const int a_box = a_box_for_rows(m.nrows);
        const uint32_t a_bytes = static_cast<uint32_t>(a_box_rows(a_box)) * 128;
        const uint8_t* sfa = a.a_sf + mt * sfa_group;
        const uint8_t* sfb = a.b_sf + (brow / kF4N) * sfb_group;
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kBarEmpty + stage), phase ^ 1u, abort_flag, limit, a.status,
                                 kWhereProducerEmpty)) {
            ok = false;
            break;
          }
          const uint32_t sA = sbase + stage * kF4StageBytes;
          const uint32_t sB = sA + kF4StageA;
          const uint32_t sS = sB + kF4StageB;
          const uint32_t fb = bar(kBarFull + stage);
          mbar_arrive_expect_tx(fb, a_bytes + kF4StageB + kF4SfaBytes + kF4SfBytes);
          tma_load_2d(sA, &tmA.m[a_box], fb, kb * 128, m.row0);
          tma_load_2d(sB, &tmB, fb, kb * 128, brow);
          bulk_load(sS, sfa + kb * kF4SfaBytes, kF4SfaBytes, fb);
          bulk_load(sS + kF4SfaBytes, sfb + kb * kF4SfBytes, kF4SfBytes, fb);
          filled |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == kF4Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      int no_abort = 0;
      for (int s = 0; s < kF4Stages; ++s)
        if ((filled >> s) & 1u)
          mbar_wait_bounded(bar(kBarFull + s), (last_parity >> s) & 1u, &no_abort, drain_limit,
                            a.status, kWhereDrain);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ scale copies
    // One thread copies each stage's block scales into the stage's own TMEM columns as soon as
    // the stage has landed and signals the MMA thread through a commit.  The stage's columns
    // are free again by then: the stage was refilled only after the MMAs that read them
    // completed.  Issued from a thread of their own, the copies run beside the MMAs instead of
    // between them.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kBarFull + stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sS = sbase + stage * kF4StageBytes + kF4StageA + kF4StageB;
          const uint32_t sfa_t = tmem_base + kF4SfCol + kF4SfStageCols * stage;
          const uint32_t sfb_t = sfa_t + 16u;
#pragma unroll
          for (int p = 0; p < 2; ++p)
            tmem_cp_sf_pair(sfa_t + 8u * p, smem_desc_sf_pair(sS + 4096u * p));
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            tmem_cp_sf(sfb_t + 4u * ks, smem_desc_sf(sS + kF4SfaBytes + 512u * ks));
          umma_commit(bar(kBarSReady + stage));
          if (++stage == kF4Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      int no_abort = 0;
      umma_commit(bar(kBarCopyDrain));
      mbar_wait_bounded(bar(kBarCopyDrain), 0, &no_abort, drain_limit, a.status, kWhereDrain);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_nvfp4(kBM, kF4N);
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        if (!mbar_wait_bounded(bar(kBarTEmpty + acc), acc_phase ^ 1u, abort_flag, limit, a.status,
                               kWhereMmaTmemEmpty))
          break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kF4N);
        for (int kb = 0; kb < a.k_blocks; ++kb) {
          if (!mbar_wait_bounded(bar(kBarFull + stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull) ||
              !mbar_wait_bounded(bar(kBarSReady + stage), phase, abort_flag, limit, a.status,
                                 kWhereMmaFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = sbase + stage * kF4StageBytes;
          const uint64_t adesc = smem_desc_k_sw128(sA);
          const uint64_t bdesc = smem_desc_k_sw128(sA + kF4StageA);
          const uint32_t sa_t = tmem_base + kF4SfCol + kF4SfStageCols * stage;
          const uint32_t sb_t = sa_t + 16u;
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)  // 64 E2M1 elements = 32 bytes of K: +2 in addr >> 4
            umma_nvfp4(d_tmem, adesc + 2u * ks, bdesc + 2u * ks, idesc, sa_t + 4u * ks,
                       sb_t + 4u * ks, (kb | ks) != 0 ? 1u : 0u);
          umma_commit(bar(kBarEmpty + stage));
          if (++stage == kF4Stages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(bar(kBarTFull + acc));
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      int no_abort = 0;
      umma_commit(bar(kBarDrain));
      mbar_wait_bounded(bar(kBarDrain), 0, &no_abort, drain_limit, a.status, kWhereDrain);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;  // M = 128: accumulator row r in TMEM lane r
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
      ok = mbar_wait_bounded(bar(kBarTFull + acc), acc_phase, abort_flag, limit, a.status,
                             kWhereEpiTmemFull);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();

      const uint32_t tb = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                          static_cast<uint32_t>(acc * kF4N);
      const bool valid = row < m.nrows;
      const float sa = valid ? a.a_scale[m.row0 + row] : 0.f;
      const float* sb = a.b_scale + static_cast<int64_t>(m.e) * a.b_rows_per_expert + n * kF4N;
      if (kSwiGLU) {
        __nv_bfloat16* dst = a.out + static_cast<int64_t>(m.row0 + (valid ? row : 0)) * a.out_ld +
                             n * (kF4N / 2);
#pragma unroll 1
        for (int c = 0; c < kF4N / 2; c += 32) {
          uint32_t g[32], u[32];
          tmem_ld32_sync(tb + c, g);
          tmem_ld32_sync(tb + kF4N / 2 + c, u);
          scale32(g, sa, sb + c);
          scale32(u, sa, sb + kF4N / 2 + c);
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
        __nv_bfloat16* dst = a.out + static_cast<int64_t>(m.row0 + (valid ? row : 0)) * a.out_ld +
                             n * kF4N;
#pragma unroll 1
        for (int c = 0; c < kF4N; c += 32) {
          uint32_t y[32];
          tmem_ld32_sync(tb + c, y);
          scale32(y, sa, sb + c);
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
    tmem_dealloc(tmem_base, kF4TmemCols);
  }
}

}  // namespace

cudaError_t prepare_gemm_nvfp4_kernels() {
  const void* kernels[] = {reinterpret_cast<const void*>(expert_gemm_nvfp4_kernel<true>),
                           reinterpret_cast<const void*>(expert_gemm_nvfp4_kernel<false>)};
  for (const void* k : kernels) {
    const cudaError_t e =
        cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, kF4SmemBytes);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_gemm_nvfp4(bool swiglu, const ATensorMaps& tmA, const CUtensorMap& tmB,
                              const Fp4GemmArgs& a, int grid, cudaStream_t s) {
  if (swiglu)
    expert_gemm_nvfp4_kernel<true><<<grid, kF4Threads, kF4SmemBytes, s>>>(tmA, tmB, a);
  else
    expert_gemm_nvfp4_kernel<false><<<grid, kF4Threads, kF4SmemBytes, s>>>(tmA, tmB, a);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_weights(const __nv_bfloat16* a, const __nv_bfloat16* b, int64_t groups,
                                 int rows, int cols, uint8_t* codes, uint8_t* sf, float* scale,
                                 cudaStream_t s) {
  const int64_t out_rows = groups * (b ? 2 * rows : rows);
  if (out_rows <= 0) return cudaSuccess;
  const int64_t blocks = (out_rows + 7) / 8;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  nvfp4_weights_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a, b, groups, rows, cols,
                                                                     codes, sf, scale);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_permute(const Fp4PermuteArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  nvfp4_permute_kernel<<<(a.T + kPermTokensPerCta - 1) / kPermTokensPerCta, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_act(const Fp4ActArgs& a, cudaStream_t s) {
  if (a.mt_cap <= 0) return cudaSuccess;
  const int64_t blocks = static_cast<int64_t>(a.mt_cap) * kActCtasPerTile;
  if (blocks > 0x7fffffff) return cudaErrorInvalidValue;
  nvfp4_act_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
