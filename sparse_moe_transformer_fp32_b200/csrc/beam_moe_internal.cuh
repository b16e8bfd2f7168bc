// Internal declarations of the Beam MoE CUDA path: constants, workspace layout,
// kernel argument blocks and the sm_100a inline-PTX wrappers (mbarrier, TMA,
// tcgen05) the expert GEMMs are built from.
#pragma once

#include <cuda.h>  // CUtensorMap (type only; the driver is reached through the runtime)
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace beam {

// ------------------------------------------------------------------ constants

constexpr int kBM = 128;        // rows (token slots) per expert tile = UMMA M
constexpr int kBK = 64;         // K elements per pipeline stage: one 128-byte swizzle row of BF16
constexpr int kUmmaK = 16;      // K of one tcgen05.mma kind::f16
constexpr int kStages = 4;      // shared-memory ring depth
constexpr int kN1Half = 128;    // gate (and up) columns per GEMM1 tile -> UMMA N = 256
constexpr int kN2 = 256;        // output columns per GEMM2 tile -> UMMA N = 256
constexpr int kUmmaN = 256;
constexpr int kBand = 8;        // m-tiles per raster band (L2 reuse of weight tiles)
constexpr int kPairMinRowsPerExpert = 256;  // calls at or above this mean use SM-pair GEMMs
constexpr int kSwapMaxRows = 32;   // m-tiles with at most this many rows may run weights-as-M
constexpr int kGemmThreads = 192;  // warp 0 TMA, warp 1 MMA, warps 2..5 epilogue
constexpr int kTmemCols = 512;     // two 256-column FP32 accumulators

constexpr int kStageABytes = kBM * kBK * 2;        // 16 KB
constexpr int kStageBBytes = kUmmaN * kBK * 2;     // 32 KB
constexpr int kStageBytes = kStageABytes + kStageBBytes;
constexpr int kGemmSmemBytes = kStages * kStageBytes + 1024 /*barriers*/ + 1024 /*align*/;

// router GEMM tiling (FP32 FFMA)
constexpr int kRM = 128, kRN = 128, kRK = 16, kRThreads = 256, kRBStages = 3;

constexpr int kRouterSlots = 2 * 148;  // resident router blocks on a 148-SM B200

constexpr int kMaxTopK = 8;
constexpr int kMaxE = 256;
constexpr int kMaxGroups = 32;
constexpr int kMaxD = 8192;

// device status codes (word 0 of the workspace)
enum : uint32_t {
  kDevOk = 0,
  kDevTimeout = 1,
  kDevAssert = 2,
};
// where a device error was detected (word 1)
enum : uint32_t {
  kWhereProducerEmpty = 1,
  kWhereMmaFull = 2,
  kWhereMmaTmemEmpty = 3,
  kWhereEpiTmemFull = 4,
  kWhereDrain = 5,
  kWherePermute = 6,
  kWhereCombine = 7,
  kWhereSelect = 8,
  kWhereDispatch = 9,
};

// Four views of the same row-major A operand (Xp or act) whose TMA boxes are 16, 32, 64 and
// 128 rows high: a tile loads only as many rows as it has (rounded up to the next box).
constexpr int kNumABoxes = 4;
struct ATensorMaps {
  CUtensorMap m[kNumABoxes];
};
__host__ __device__ constexpr int a_box_rows(int box) { return 16 << box; }
__host__ __device__ constexpr int a_box_for_rows(int nrows) {
  return nrows <= 16 ? 0 : nrows <= 32 ? 1 : nrows <= 64 ? 2 : 3;
}

struct MTile {
  int32_t e;      // expert
  int32_t row0;   // first row in the expert-contiguous buffers
  int32_t nrows;  // valid rows, 1..kBM
  int32_t band;   // raster band holding this m-tile: (first m-tile << 4) | m-tiles (1..15)
};
constexpr int kBandLenBits = 4;
static_assert(2 * kBand - 1 < (1 << kBandLenBits), "a band's length must fit its field");

// Raster bands group the m-tiles whose tiles run back to back, slice-major, so that the CTAs
// working at the same time share weight slices (and A rows) through L2.  A band holds whole
// experts: the experts of at most kBand m-tiles whose first m-tile falls in the same block of
// kBand m-tiles (so up to 2 kBand - 1 m-tiles); an expert with more m-tiles is cut into bands
// of kBand.  An expert therefore never straddles two bands unless it must, and its weight
// slices are streamed from HBM once per band.
__host__ __device__ constexpr int32_t pack_band(int start, int len) {
  return (start << kBandLenBits) | len;
}

// Tile t of a launch whose m-tiles carry bands: m-tile mt and N slice n.  The tiles of a band
// are contiguous in t, so the band of tile t is the band of m-tile t / n_tiles.
__device__ __forceinline__ void band_decode_tile(const MTile* mtiles, int t, int n_tiles, int& mt,
                                                 int& n) {
  const int32_t b = mtiles[t / n_tiles].band;
  const int start = b >> kBandLenBits, len = b & ((1 << kBandLenBits) - 1);
  const int r = t - start * n_tiles;
  n = r / len;
  mt = start + (r - n * len);
}

// ------------------------------------------------------------------ kernel arguments

struct RouterGemmArgs {
  const __nv_bfloat16* h;  // [T, d]
  const float* WT;         // [d, E] (transposed router weight)
  float* part;             // [S, T, E]
  int32_t* zero_counts;    // [E] zeroed by block (0,0,0), or null
  int T, d, E, kchunk;
};

// The token bitmap of a dispatch: bit (t % 32) of word bits[e * words + t / 32] is set when token
// t chose expert e (words = ceil(T / 32) per expert).  Its per-expert prefix counts give every
// (token, expert) slot its rank among the expert's rows in ascending token order, so the row
// layout of the expert-contiguous buffers does not depend on the order in which CTAs run.
struct SelectArgs {
  const float* part;  // [S, T, E]
  const float* bias;  // [E]
  float* logits_out;  // [T, E] or null
  int32_t* idx;       // [T, k]
  float* w;           // [T, k]
  int32_t* cnt;       // [E] or null (no dispatch); zeroed before the call
  uint32_t* bits;     // [E, words] token bitmap (dispatch only); zeroed before the call
  int words;
  uint32_t* status;
  int S, T, E, G, Gk, k;
  float scale;
  int norm;
};

struct DispatchArgs {
  const int32_t* cnt;    // [E]
  const uint32_t* bits;  // [E, words] token bitmap
  int32_t* base;         // [E, words] out: set bits of the expert's earlier words
  int32_t* off;          // [E + 1]
  int32_t* mt_count;     // [1] number of m-tiles
  MTile* mtiles;         // [capacity]
  int E, words;
  int tile_rows;         // rows per m-tile: 128 (one SM) or 256 (an SM pair)
};

struct PermuteArgs {
  const __nv_bfloat16* h;  // [T, d]
  const int32_t* idx;      // [T, k]
  const uint32_t* bits;    // [E, words] token bitmap
  const int32_t* base;     // [E, words] its per-expert prefix counts
  int words;
  const int32_t* off;      // [E + 1]
  int32_t* rowmap;         // [T, k] out: row of slot (t, j) in the expert-contiguous buffers
  __nv_bfloat16* xp;       // [R, d] out (BF16 path), or null
  uint8_t* xq;             // [R, d] out: E4M3 codes (FP8 path), or null
  float* xs;               // [R] out: row scales (FP8 path)
  uint32_t* status;
  int T, d, k, E;
};

struct GemmArgs {
  const MTile* mtiles;
  const int32_t* mt_count;
  __nv_bfloat16* out;      // GEMM1: act [R, I]; GEMM2: Y [R, d]
  uint32_t* status;
  uint64_t wait_limit_ns;
  int64_t out_ld;          // elements per output row
  int n_tiles_n;           // tiles along N per m-tile
  int k_blocks;            // K / kBK
  int b_rows_per_expert;   // rows of one expert in the 2-D weight view (I or d)
  int swap_max_rows;       // m-tiles with at most this many rows run weights-as-M (0: none)
  // FP8 instances only: D = acc * a_scale[A row] * b_scale[B row] (b_scale1: the up slice)
  const float* a_scale;
  const float* b_scale0;
  const float* b_scale1;
};

struct CombineArgs {
  const __nv_bfloat16* y;  // [R, d]
  const int32_t* rowmap;   // [T, k]
  const float* w;          // [T, k]
  __nv_bfloat16* out;      // [T, d] (layer)
  // block form
  const float* x;          // [T, d]
  const float* g_post;     // [d]
  float* x_out;            // [T, d]
  float eps, coef_x, coef_f;
  uint32_t* status;
  int T, d, k, R;
};

struct PreNormArgs {
  const float* x;       // [T, d]
  const float* g_pre;   // [d]
  __nv_bfloat16* h;     // [T, d]
  float eps;
  int T, d;
};

// ---- expert parallelism (ep.cu): P ranks, rank p owning experts p*E/P .. (p+1)*E/P - 1

constexpr int kMaxEpRanks = 64;

struct EpCountArgs {
  const int32_t* idx;  // [T, k] local routing
  int32_t* cnt;        // [E] out (zeroed before the call)
  uint32_t* bits;      // [E, words] out: token bitmap (zeroed before the call)
  int words;
  uint32_t* status;
  int T, k, E;
};

struct EpOffsetsArgs {
  const int32_t* all;     // [P, E] slot counts of every rank
  const uint32_t* bits;   // [E, words] local token bitmap
  int32_t* base;          // [E, words] out: its per-expert prefix counts
  int64_t* row_off;       // [E] out: row of this rank's first slot of e on e's owner
  int words, P, E, rank;
};

struct EpPushArgs {
  const __nv_bfloat16* h;  // [T, d] local tokens
  const int32_t* idx;      // [T, k]
  const uint32_t* bits;
  const int32_t* base;
  int words;
  const int64_t* row_off;  // [E]
  int32_t* slot_row;       // [T, k] out: row on the owner (-1: not sent)
  int32_t* slot_owner;     // [T, k] out: owner rank
  __nv_bfloat16* xrecv[kMaxEpRanks];  // receive buffers [recv_cap, d] of every rank
  int64_t recv_cap;
  uint32_t* status;
  int T, d, k, E, P;
};

struct EpCombineArgs {
  const int32_t* slot_row;
  const int32_t* slot_owner;
  const float* w;                            // [T, k]
  const __nv_bfloat16* yrecv[kMaxEpRanks];   // expert outputs [recv_cap, d] of every rank
  __nv_bfloat16* out;                        // [T, d]
  int64_t recv_cap;
  uint32_t* status;
  int T, d, k, P;
};

// ------------------------------------------------------------------ launchers (one per kernel)

cudaError_t launch_ep_count(const EpCountArgs& a, cudaStream_t s);
cudaError_t launch_ep_offsets(const EpOffsetsArgs& a, cudaStream_t s);
cudaError_t launch_ep_push(const EpPushArgs& a, cudaStream_t s);
cudaError_t launch_ep_local_counts(const int32_t* all, int P, int E, int rank, int64_t recv_cap,
                                   int32_t* cnt_local, uint32_t* status, cudaStream_t s);
cudaError_t launch_ep_combine(const EpCombineArgs& a, cudaStream_t s);

cudaError_t launch_router_transpose(const float* W, float* WT, int E, int d, cudaStream_t s);
cudaError_t launch_router_gemm(const RouterGemmArgs& a, int S, cudaStream_t s);
cudaError_t launch_router_select(const SelectArgs& a, cudaStream_t s);
cudaError_t launch_dispatch_scan(const DispatchArgs& a, cudaStream_t s);
cudaError_t launch_permute(const PermuteArgs& a, cudaStream_t s);
cudaError_t launch_gemm_gate_up(const ATensorMaps& tmA, const CUtensorMap& tmG,
                                const CUtensorMap& tmU, const GemmArgs& a, int grid,
                                cudaStream_t s, bool fp8 = false);
cudaError_t launch_gemm_down(const ATensorMaps& tmA, const CUtensorMap& tmD, const GemmArgs& a,
                             int grid, cudaStream_t s, bool fp8 = false);
cudaError_t launch_quantize_rows(const __nv_bfloat16* x, int64_t rows, int cols, uint8_t* q,
                                 float* scale, cudaStream_t s);
cudaError_t launch_gemm_gate_up_2sm(const ATensorMaps& tmA, const CUtensorMap& tmG,
                                    const CUtensorMap& tmU, const GemmArgs& a, int grid,
                                    cudaStream_t s);
cudaError_t launch_gemm_down_2sm(const ATensorMaps& tmA, const CUtensorMap& tmD,
                                 const GemmArgs& a, int grid, cudaStream_t s);
cudaError_t prepare_gemm_2sm_kernels();
int max_pair_grid(int sms);
cudaError_t launch_combine(const CombineArgs& a, cudaStream_t s);
cudaError_t launch_combine_block(const CombineArgs& a, cudaStream_t s);
cudaError_t launch_prenorm(const PreNormArgs& a, cudaStream_t s);
cudaError_t launch_dense_tiles(int T, MTile* mtiles, int32_t* mt_count, cudaStream_t s);
cudaError_t launch_bias_update(const int32_t* cnt, float* bias, int E, float mean, float gamma,
                               cudaStream_t s);
cudaError_t prepare_gemm_kernels();  // opt-in shared memory sizes (once per device)
cudaError_t prepare_router_kernels();

// ------------------------------------------------------------------ device helpers

#ifdef __CUDACC__

__device__ __forceinline__ void record_status(uint32_t* status, uint32_t code, uint32_t where) {
  if (status && atomicCAS(status, 0u, code) == 0u) {
    status[1] = where;
    status[2] = blockIdx.x;
  }
}

// Rank of token t among the rows of expert e (ascending token order), from the dispatch's token
// bitmap and its prefix counts; -1 when t did not choose e.
__device__ __forceinline__ int slot_rank(const uint32_t* bits, const int32_t* base, int words,
                                         int e, int t) {
  const size_t i = static_cast<size_t>(e) * words + (t >> 5);
  const uint32_t w = bits[i];
  const uint32_t b = 1u << (t & 31);
  if (!(w & b)) return -1;
  return base[i] + __popc(w & (b - 1u));
}

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// As mbar_try_wait, letting the hardware park the thread until the phase completes or about
// hint_ns nanoseconds pass.
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Waits for the phase of parity `parity` of barrier `bar` to complete.  Gives up when the
// CTA-wide abort flag is raised, or after limit_ns, in which case it raises the flag and
// records a timeout.  A limit of 0 gives up at the first check that finds the phase open.
// After a few polls the thread is parked by the hardware between checks (suspend hint), so
// long waits -- the epilogue's for a whole K loop -- issue few instructions.
// Returns true when the phase completed.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int* abort_flag, uint64_t limit_ns,
                                                  uint32_t* status, uint32_t where) {
  const int spins = limit_ns == 0 ? 1 : 32;
#pragma unroll 1
  for (int i = 0; i < spins; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
#pragma unroll 1
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait_hint(bar, parity, 1000u)) return true;
    if ((it & 7u) == 0u) {
      if (*abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        record_status(status, kDevTimeout, where);
        return false;
      }
    }
  }
}

// ---- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled load of a box at (x = inner coordinate, y = outer coordinate) into shared memory,
// completing on mbarrier `bar` (complete_tx).  x is always a multiple of 64 elements here.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* m, uint32_t bar,
                                            int32_t x, int32_t y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

// ---- tcgen05

__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, BF16 x BF16 -> FP32, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, E4M3 x E4M3 -> FP32, issued by one thread.
__device__ __forceinline__ void umma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued before has completed.
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
      : "memory");
}

// 32 lanes x 32 consecutive FP32 columns, loaded and waited for in one statement so that no
// use of the destination registers can be scheduled before the load completes.  Thread i of
// the warp gets TMEM lane (lane base + i), i.e. accumulator row (lane base + i).
__device__ __forceinline__ void tmem_ld32_sync(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
      " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
      " [%32];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// 32 lanes x 16 consecutive FP32 columns (load and wait in one statement, as above).
__device__ __forceinline__ void tmem_ld16_sync(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32"
      " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major operand tile written by TMA with 128-byte
// swizzle: rows of 128 bytes, 8-row atoms of 1024 bytes stacked along M/N.
//   start address >> 4 in bits 0..13, leading byte offset (16 B, unused by swizzled
//   K-major) in 16..29, stride byte offset 1024 B >> 4 in 32..45, version 1 in 46..47,
//   layout type 2 (128-byte swizzle) in 61..63.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(uint32_t saddr) {
  uint64_t desc = 0;
  desc |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  desc |= static_cast<uint64_t>(1u) << 16;
  desc |= static_cast<uint64_t>(1024u >> 4) << 32;
  desc |= static_cast<uint64_t>(1u) << 46;
  desc |= static_cast<uint64_t>(2u) << 61;
  return desc;
}

// Instruction descriptor, kind::f16: D FP32 (bits 4..5 = 1), A BF16 (7..9 = 1), B BF16
// (10..12 = 1), both K-major (bits 15, 16 = 0), N >> 3 in 17..22, M >> 4 in 24..28.
__host__ __device__ constexpr uint32_t umma_idesc_bf16_f32(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}

// Instruction descriptor, kind::f8f6f4: D FP32 (bits 4..5 = 1), A and B E4M3 (format 0 in
// bits 7..9 and 10..12), both K-major, N >> 3 in 17..22, M >> 4 in 24..28.
__host__ __device__ constexpr uint32_t umma_idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

#endif  // __CUDACC__

}  // namespace beam
