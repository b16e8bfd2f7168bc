// NVFP4 expert weights: shared constants, kernel arguments and launchers.
//
// Format (E2M1 codes, an E4M3 scale per 16 elements along K, an FP32 scale per row; the
// pages name NVFP4 checkpoints without a scale format -- news article "Reflection lança o
// Beam", section "Onde o Beam economiza ..."):
//   s = fl32(amax / 2688),  bs_b = e4m3(fl32(fl32(m_b / s) / 6)),
//   q_j = e2m1(fl32(x_j / fl32(s * bs_b)))
// Codes are packed two per byte, element 2i in the low nibble of byte i.  Block scales are
// stored in 512-byte atoms, one per 128 rows x 64 K elements: row r (0..127) and block j
// (0..3) of an atom sit at byte (r % 32) * 16 + (r / 32) * 4 + j, so that one
// tcgen05.cp.32x128b.warpx4 puts row r's four scales in TMEM lane r.  A 128-row group of a
// matrix keeps its atoms in K order: atom (row group g, K block b) at byte
// (g * K / 64 + b) * 512.
#pragma once
#include "beam_moe_internal.cuh"

namespace beam {

constexpr int kF4N = 128;                   // UMMA N (weight rows per tile); UMMA M = kBM
constexpr int kF4KElems = 256;              // K elements per stage: one 128-byte code row
constexpr int kF4Stages = 5;
constexpr int kF4StageA = kBM * 128;        // 16 KB of A codes
constexpr int kF4StageB = kF4N * 128;       // 16 KB of B codes
constexpr int kF4SfBytes = 2048;            // B block scales of 128 rows x 256 K elements
constexpr int kF4SfaBytes = 8192;           // A block scales of the same, laid out as below
constexpr int kF4StageBytes = kF4StageA + kF4StageB + kF4SfaBytes + kF4SfBytes;  // 42 KB
constexpr int kF4Threads = 224;  // warp 0 loads, 1 MMA, 2..5 epilogue, 6 scale copies
constexpr int kF4SmemBytes = kF4Stages * kF4StageBytes + 1024 /*barriers*/ + 1024 /*align*/;

// Byte offset of the scale of (row r of a 128-row group, 16-element block j) from the start of
// the group's atoms.
__host__ __device__ constexpr size_t nvfp4_sf_offset(int r, int j) {
  return static_cast<size_t>(j >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (j & 3);
}

// The A operand's (token rows') block scales are kept in the layout tcgen05.cp.128x256b
// reads: per 128-row group and 256-element K stage 8 KB, per 64-element K step a 2 KB block of
// 128 rows x 16 bytes in which row r's four scales sit at byte r * 16 + (r / 32) * 4.  The
// MMA reads A's scales of TMEM lane r from column r / 32 of the K step's four (lane quarter q
// reads column q), so the other 12 bytes of a row are never read by it: the permute fills them
// with copies of the same four (whole 16-byte stores), the activation quantiser leaves them
// unwritten.  One copy
// brings two K steps (two blocks, 2 KB apart): two copies a stage where one
// 32x128b.warpx4 copy per K step took four.  Groups of 128 rows keep their stages in K order.
__host__ __device__ constexpr size_t nvfp4_sfa_offset(int r, int j) {
  return static_cast<size_t>(j >> 4) * kF4SfaBytes + ((j >> 2) & 3) * 2048 + r * 16 +
         (r >> 5) * 4 + (j & 3);
}

struct Fp4GemmArgs {
  const MTile* mtiles;
  const int32_t* mt_count;
  __nv_bfloat16* out;      // GEMM1: act [R, I]; GEMM2: Y [R, d]
  uint32_t* status;
  uint64_t wait_limit_ns;
  int64_t out_ld;          // elements per output row
  int n_tiles_n;           // tiles along N per m-tile
  int k_blocks;            // K / kF4KElems
  int b_rows_per_expert;   // weight rows of one expert (2I interleaved gate|up, or d)
  const uint8_t* a_sf;     // block scales of the A rows (nvfp4_sfa_offset), one group per m-tile
  const uint8_t* b_sf;     // block-scale atoms of the weight rows
  const float* a_scale;    // [R] row scales of A
  const float* b_scale;    // [E * b_rows_per_expert] row scales of the weights
};

struct Fp4PermuteArgs {
  const __nv_bfloat16* h;  // [T, d]
  const int32_t* idx;      // [T, k]
  const uint32_t* bits;    // [E, words] token bitmap
  const int32_t* base;     // [E, words] its per-expert prefix counts
  int words;
  const int32_t* cnt;      // [E]
  const int32_t* off;      // [E + 1]
  int32_t* rowmap;         // [T, k] out
  uint8_t* xq;             // [R, d / 2] out: codes
  uint8_t* xsf;            // out: block scales (nvfp4_sfa_offset), one 128-row group per m-tile
  float* xs;               // [R] out: row scales
  uint32_t* status;
  int T, d, k, E;
};

struct Fp4ActArgs {
  const __nv_bfloat16* x;  // [R, cols] (the SwiGLU activation)
  const MTile* mtiles;
  const int32_t* mt_count;
  uint8_t* q;              // [R, cols / 2] out
  uint8_t* sf;             // out: block scales (nvfp4_sfa_offset), one 128-row group per m-tile
  float* s;                // [R] out
  int cols;
  int mt_cap;
};

// a [groups, rows, cols] BF16; with b (same shape) the output rows interleave a and b in
// 64-row chunks: output row 128c + w is a's row 64c + w (w < 64) or b's row 64c + w - 64.
cudaError_t launch_nvfp4_weights(const __nv_bfloat16* a, const __nv_bfloat16* b, int64_t groups,
                                 int rows, int cols, uint8_t* codes, uint8_t* sf, float* scale,
                                 cudaStream_t s);
cudaError_t launch_nvfp4_permute(const Fp4PermuteArgs& a, cudaStream_t s);
cudaError_t launch_nvfp4_act(const Fp4ActArgs& a, cudaStream_t s);
cudaError_t launch_gemm_nvfp4(bool swiglu, const ATensorMaps& tmA, const CUtensorMap& tmB,
                              const Fp4GemmArgs& a, int grid, cudaStream_t s);
cudaError_t prepare_gemm_nvfp4_kernels();

}  // namespace beam
