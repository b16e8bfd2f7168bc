// C ABI of the Beam MoE layer (declared in include/beam_moe.h): argument checks, workspace
// layout, TMA tensor maps, kernel launch sequence, device status, launch counting and timing.
#include "beam_moe.h"
#include "beam_moe_internal.cuh"
#include "beam_moe_router.cuh"
#include "beam_moe_nvfp4.cuh"

#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <vector>

namespace {

using namespace beam;

std::atomic<uint64_t> g_wait_limit_ns{4000000000ull};
std::atomic<uint64_t> g_launches{0};
std::atomic<int> g_sm_pairs{0};
thread_local char g_last_cuda_error[256] = "";

// ------------------------------------------------------------------ kernel ids and timing

enum KernelId {
  kKRouterGemm = 0,
  kKRouterSelect,
  kKDispatchScan,
  kKPermute,
  kKGemmGateUp,
  kKGemmDown,
  kKCombine,
  kKCombineBlock,
  kKPreNorm,
  kKRouterTranspose,
  kKDenseTiles,
  kKBiasUpdate,
  kKQuantize,
  kKQuantizeNvfp4,
  kKEpCount,
  kKEpOffsets,
  kKEpPush,
  kKEpLocalCounts,
  kKEpCombine,
  kNumKernels
};
const char* const kKernelNames[kNumKernels] = {
    "router_gemm", "router_select", "dispatch_scan", "permute", "expert_gemm_gate_up",
    "expert_gemm_down", "combine", "combine_block", "prenorm", "router_transpose", "dense_tiles",
    "bias_update", "quantize_e4m3", "quantize_nvfp4", "ep_count", "ep_offsets", "ep_push",
    "ep_local_counts", "ep_combine"};

struct Profiler {
  std::mutex mu;
  bool on = false;
  struct Rec {
    int id;
    cudaEvent_t a, b;
  };
  std::vector<Rec> pending;
  std::vector<cudaEvent_t> pool;
  int64_t launches[kNumKernels] = {};
  double ms[kNumKernels] = {};

  cudaEvent_t take() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
};
Profiler g_prof;

struct ProfScope {
  int id;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  ProfScope(int id_, cudaStream_t s_) : id(id_), s(s_) {
    std::lock_guard<std::mutex> lk(g_prof.mu);
    if (!g_prof.on) return;
    a = g_prof.take();
    cudaEventRecord(a, s);
  }
  ~ProfScope() {
    if (!a) return;
    std::lock_guard<std::mutex> lk(g_prof.mu);
    cudaEvent_t b = g_prof.take();
    cudaEventRecord(b, s);
    g_prof.pending.push_back({id, a, b});
  }
};

beam_status cuda_fail(cudaError_t e) {
  std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return BEAM_ERR_CUDA;
}

#define BEAM_LAUNCH(id, stream, call)                 \
  do {                                                \
    cudaError_t err_;                                 \
    {                                                 \
      ProfScope ps_(id, stream);                      \
      err_ = (call);                                  \
    }                                                 \
    if (err_ != cudaSuccess) return cuda_fail(err_);  \
    g_launches.fetch_add(1, std::memory_order_relaxed); \
  } while (0)

// ------------------------------------------------------------------ shapes and workspace

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

beam_status check_shape(const beam_moe_shape* s) {
  if (!s) return BEAM_ERR_INVALID_ARG;
  if (s->T < 0 || s->d <= 0 || s->E <= 0 || s->n_group <= 0 || s->topk_group <= 0 ||
      s->top_k <= 0 || s->I <= 0)
    return BEAM_ERR_INVALID_ARG;
  if (!std::isfinite(s->routed_scaling_factor)) return BEAM_ERR_INVALID_ARG;
  if (s->d % 256 != 0 || s->d > kMaxD) return BEAM_ERR_UNSUPPORTED;
  if (s->I % 128 != 0 || s->I > 65536) return BEAM_ERR_UNSUPPORTED;
  if (s->E > kMaxE || s->E % 4 != 0 || s->E % s->n_group != 0 || s->n_group > kMaxGroups)
    return BEAM_ERR_UNSUPPORTED;
  if (s->topk_group > s->n_group || s->top_k > kMaxTopK) return BEAM_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->top_k) > static_cast<int64_t>(s->topk_group) * (s->E / s->n_group))
    return BEAM_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(s->T) * s->top_k >= (int64_t(1) << 31)) return BEAM_ERR_UNSUPPORTED;
  return BEAM_OK;
}

struct Layout {
  size_t status, cnt, bits, off, mt_count, mtiles, base, rowmap, idx, w, wt, part, h, xp, act, y,
      total;
  size_t zero_bytes = 0;             // status, counts and token bitmap: cleared at each call
  int words = 0;                     // token bitmap words per expert, ceil(T / 32)
  size_t xs = 0, act8 = 0, as = 0;  // FP8 path: row scales of Xp, E4M3 act, act row scales
  size_t xsf = 0, asf = 0;           // NVFP4 path: block scales of Xp and of the act
  int S, kchunk;
  int64_t R, mt_cap;
};

// Router split-K factor S from a simple cost model: the FFMA time of the waves of
// (token tile, expert tile, K chunk) blocks over the resident router blocks of a 148-SM B200,
// plus the traffic of writing and re-reading S partial logit arrays and the selection kernel's
// latency of adding them (one round of loads per four splits).  K chunks are a multiple of the
// router's K step; at most max_s splits.
int router_split(const beam_moe_shape& s, int max_s) {
  const int64_t kblocks = s.d / kRK;
  if (s.T <= kRouterSmallT) {  // 32-token tiles: a fixed split, a few K tiles per block
    int S = kRouterSmallSplit < max_s ? kRouterSmallSplit : max_s;
    while (S > 1 && kblocks / S < 4) S /= 2;
    return S;
  }
  const int64_t tiles = ceil_div(s.T, kRM) * ceil_div(s.E, kRN);
  const double block_flops_per_k = 2.0 * kRM * kRN;
  const double slot_rate = 70e12 / kRouterSlots;  // FP32 FLOP/s per resident block
  const double hbm = 6.5e12;
  int best = 1;
  double best_t = 1e30;
  for (int S = 1; S <= max_s && S <= kblocks; ++S) {
    const int64_t per = ceil_div(kblocks, S);
    const int64_t Sx = ceil_div(kblocks, per);
    if (Sx != S) continue;
    const double waves = static_cast<double>(ceil_div(tiles * S, kRouterSlots));
    const double t = waves * per * kRK * block_flops_per_k / slot_rate +
                     static_cast<double>(S) * s.T * s.E * 8.0 / hbm +
                     static_cast<double>(ceil_div(S, 4)) * 0.8e-6;
    if (t < best_t * 0.97) {  // a larger split must win clearly
      best_t = t;
      best = S;
    }
  }
  return best;
}

Layout plan(const beam_moe_shape& s) {
  Layout L{};
  const int64_t T = s.T, R = T * s.top_k;
  L.R = R;
  const int64_t kblocks = s.d / kRK;
  const int S = router_split(s, 64);
  L.kchunk = static_cast<int>(ceil_div(kblocks, S) * kRK);
  L.S = static_cast<int>(ceil_div(s.d, L.kchunk));
  L.mt_cap = ceil_div(R, kBM) + s.E;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  L.words = static_cast<int>(ceil_div(T, 32));
  const size_t bitmap_bytes = sizeof(uint32_t) * static_cast<size_t>(s.E) * L.words;
  L.status = take(256);
  L.cnt = take(sizeof(int32_t) * s.E);
  L.bits = take(bitmap_bytes);
  L.zero_bytes = L.bits + bitmap_bytes;  // status, counts and bitmap are contiguous from 0
  L.off = take(sizeof(int32_t) * (s.E + 1));
  L.mt_count = take(16);
  L.mtiles = take(sizeof(MTile) * L.mt_cap);
  L.base = take(bitmap_bytes);
  L.rowmap = take(sizeof(int32_t) * R);
  L.idx = take(sizeof(int32_t) * R);
  L.w = take(sizeof(float) * R);
  L.wt = take(sizeof(float) * static_cast<size_t>(s.E) * s.d);
  L.part = take(sizeof(float) * static_cast<size_t>(L.S) * T * s.E);
  L.h = take(sizeof(__nv_bfloat16) * T * s.d);
  L.xp = take(sizeof(__nv_bfloat16) * R * s.d);
  L.act = take(sizeof(__nv_bfloat16) * R * s.I);
  L.y = take(sizeof(__nv_bfloat16) * R * s.d);
  L.total = o;
  return L;
}

// FP8 path: the BF16 layout (whose Xp region holds the E4M3 rows, half its size) plus the row
// scales of Xp, the E4M3 activation and its row scales.
Layout plan_fp8(const beam_moe_shape& s) {
  Layout L = plan(s);
  size_t o = L.total;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  L.xs = take(sizeof(float) * L.R);
  L.act8 = take(static_cast<size_t>(L.R) * s.I);
  L.as = take(sizeof(float) * L.R);
  L.total = o;
  return L;
}

// NVFP4 path: the BF16 layout (whose Xp region holds the code rows, a quarter of its size)
// plus the row scales and block-scale atoms of Xp, the activation's codes, atoms and scales.
// Atoms are kept per m-tile (one 128-row group each): mt_cap groups of K / 16 x 128 bytes.
Layout plan_nvfp4(const beam_moe_shape& s) {
  Layout L = plan(s);
  size_t o = L.total;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  const size_t groups = static_cast<size_t>(L.mt_cap);
  L.xs = take(sizeof(float) * L.R);
  L.xsf = take(groups * (s.d / kF4KElems) * kF4SfaBytes);
  L.act8 = take(static_cast<size_t>(L.R) * (s.I / 2));
  L.asf = take(groups * (s.I / kF4KElems) * kF4SfaBytes);
  L.as = take(sizeof(float) * L.R);
  L.total = o;
  return L;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

beam_status check_ws(const Layout& L, void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < L.total)
    return BEAM_ERR_WORKSPACE;
  return BEAM_OK;
}

// ------------------------------------------------------------------ TMA tensor maps

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D view [outer, inner] (inner contiguous) of BF16 (elem_bytes 2) or E4M3 (1) elements, box
// [box_outer rows, 128 bytes] with 128-byte swizzle; rows past `outer` read as zeros.
beam_status make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint32_t box_outer, int elem_bytes = 2) {
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * elem_bytes};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / elem_bytes), box_outer};
  const cuuint32_t es[2] = {1, 1};
  const CUtensorMapDataType dt =
      elem_bytes == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "cuTensorMapEncodeTiled: %d",
                  static_cast<int>(r));
    return BEAM_ERR_CUDA;
  }
  return BEAM_OK;
}

// ------------------------------------------------------------------ per-device state

struct DeviceInfo {
  int sms = 0;
  int pair_grid = 0;  // CTAs of co-resident SM-pair clusters
  bool prepared = false;
};

beam_status device_info(DeviceInfo** out) {
  static DeviceInfo info[64];
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return BEAM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  DeviceInfo& d = info[dev];
  if (!d.prepared) {
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e);
    e = prepare_gemm_kernels();
    if (e != cudaSuccess) return cuda_fail(e);
    e = prepare_router_kernels();
    if (e != cudaSuccess) return cuda_fail(e);
    e = prepare_gemm_2sm_kernels();
    if (e != cudaSuccess) return cuda_fail(e);
    e = prepare_gemm_nvfp4_kernels();
    if (e != cudaSuccess) return cuda_fail(e);
    d.pair_grid = max_pair_grid(d.sms);
    d.prepared = true;
  }
  *out = &d;
  return BEAM_OK;
}

// ------------------------------------------------------------------ launch sequences

// Router: logits partials, then selection (+ counts and ranks when dispatching).
beam_status run_router(const beam_moe_shape& s, const Layout& L, const __nv_bfloat16* h,
                       const float* router_w, const float* bias, int32_t* idx, float* w,
                       float* logits_out, bool dispatch, void* ws, cudaStream_t st) {
  RouterGemmArgs ga{};
  ga.h = h;
  ga.WT = at<float>(ws, L.wt);
  ga.part = at<float>(ws, L.part);
  ga.zero_counts = nullptr;
  ga.T = s.T;
  ga.d = s.d;
  ga.E = s.E;
  ga.kchunk = L.kchunk;
  // the status words reflect the latest call: cleared before the first kernel runs, together
  // with the dispatch's counts and token bitmap
  cudaError_t e = cudaMemsetAsync(at<uint32_t>(ws, L.status), 0, dispatch ? L.zero_bytes : 16, st);
  if (e != cudaSuccess) return cuda_fail(e);
  if (s.T <= kRouterSmallT) {  // reads W_r as stored
    BEAM_LAUNCH(kKRouterGemm, st, launch_router_gemm_small(ga, router_w, L.S, st));
  } else {
    BEAM_LAUNCH(kKRouterTranspose, st,
                launch_router_transpose(router_w, at<float>(ws, L.wt), s.E, s.d, st));
    BEAM_LAUNCH(kKRouterGemm, st, launch_router_gemm(ga, L.S, st));
  }

  SelectArgs sa{};
  sa.part = ga.part;
  sa.bias = bias;
  sa.logits_out = logits_out;
  sa.idx = idx;
  sa.w = w;
  sa.cnt = dispatch ? at<int32_t>(ws, L.cnt) : nullptr;
  sa.bits = dispatch ? at<uint32_t>(ws, L.bits) : nullptr;
  sa.words = L.words;
  sa.status = at<uint32_t>(ws, L.status);
  sa.S = L.S;
  sa.T = s.T;
  sa.E = s.E;
  sa.G = s.n_group;
  sa.Gk = s.topk_group;
  sa.k = s.top_k;
  sa.scale = s.routed_scaling_factor;
  sa.norm = s.norm_topk_prob ? 1 : 0;
  BEAM_LAUNCH(kKRouterSelect, st, launch_router_select(sa, st));
  return BEAM_OK;
}

// Row scales of E4M3 expert weights (gate and up [E * I], down [E * d]); see beam_moe_forward_fp8.
struct Fp8Scales {
  const float* gate;
  const float* up;
  const float* down;
};

// Dispatch, the two expert GEMMs; leaves Y and rowmap in the workspace.  With f8 the weights
// are E4M3 codes: the permute writes E4M3 rows of Xp with their scales, and the activation is
// quantised between the two GEMMs.
beam_status run_experts(const beam_moe_shape& s, const Layout& L, const DeviceInfo& dev,
                        const __nv_bfloat16* h, const int32_t* idx, const void* w_gate,
                        const void* w_up, const void* w_down, void* ws, cudaStream_t st,
                        const Fp8Scales* f8 = nullptr) {
  uint32_t* status = at<uint32_t>(ws, L.status);
  // With SM pairs enabled, calls averaging at least 256 rows per expert run their expert GEMMs
  // on SM pairs (cta_group::2, 256-row tiles): half the operand bytes per SM for the same tensor
  // work, but 256-row tiles pad more rows.
  const bool pairs = !f8 && g_sm_pairs.load(std::memory_order_relaxed) != 0 &&
                     L.R >= static_cast<int64_t>(kPairMinRowsPerExpert) * s.E &&
                     dev.pair_grid >= 2;
  DispatchArgs da{};
  da.cnt = at<int32_t>(ws, L.cnt);
  da.bits = at<uint32_t>(ws, L.bits);
  da.base = at<int32_t>(ws, L.base);
  da.off = at<int32_t>(ws, L.off);
  da.mt_count = at<int32_t>(ws, L.mt_count);
  da.mtiles = at<MTile>(ws, L.mtiles);
  da.E = s.E;
  da.words = L.words;
  da.tile_rows = pairs ? 2 * kBM : kBM;
  BEAM_LAUNCH(kKDispatchScan, st, launch_dispatch_scan(da, st));

  PermuteArgs pa{};
  pa.h = h;
  pa.idx = idx;
  pa.bits = da.bits;
  pa.base = da.base;
  pa.words = L.words;
  pa.off = da.off;
  pa.rowmap = at<int32_t>(ws, L.rowmap);
  pa.xp = f8 ? nullptr : at<__nv_bfloat16>(ws, L.xp);
  pa.xq = f8 ? at<uint8_t>(ws, L.xp) : nullptr;
  pa.xs = f8 ? at<float>(ws, L.xs) : nullptr;
  pa.status = status;
  pa.T = s.T;
  pa.d = s.d;
  pa.k = s.top_k;
  pa.E = s.E;
  BEAM_LAUNCH(kKPermute, st, launch_permute(pa, st));

  const uint64_t R = static_cast<uint64_t>(L.R);
  ATensorMaps tm_xp, tm_act;
  CUtensorMap tm_g, tm_u, tm_d;
  beam_status b;
  const int eb = f8 ? 1 : 2;  // bytes per element of the GEMM operands
  const void* a1 = at<void>(ws, L.xp);
  const void* a2 = at<void>(ws, f8 ? L.act8 : L.act);
  for (int i = 0; i < kNumABoxes; ++i) {
    if ((b = make_map(&tm_xp.m[i], a1, s.d, R, a_box_rows(i), eb)) != BEAM_OK) return b;
    if ((b = make_map(&tm_act.m[i], a2, s.I, R, a_box_rows(i), eb)) != BEAM_OK) return b;
  }
  const uint64_t EI = static_cast<uint64_t>(s.E) * s.I, Ed = static_cast<uint64_t>(s.E) * s.d;
  if ((b = make_map(&tm_g, w_gate, s.d, EI, kN1Half, eb)) != BEAM_OK) return b;
  if ((b = make_map(&tm_u, w_up, s.d, EI, kN1Half, eb)) != BEAM_OK) return b;
  if ((b = make_map(&tm_d, w_down, s.I, Ed, kN2, eb)) != BEAM_OK) return b;
  const int k_elems = 128 / eb;  // K elements per 128-byte pipeline stage

  const uint64_t limit = g_wait_limit_ns.load(std::memory_order_relaxed);
  GemmArgs g1{};
  g1.mtiles = da.mtiles;
  g1.mt_count = da.mt_count;
  g1.out = at<__nv_bfloat16>(ws, L.act);
  g1.status = status;
  g1.wait_limit_ns = limit;
  g1.out_ld = s.I;
  g1.n_tiles_n = s.I / kN1Half;
  g1.k_blocks = s.d / k_elems;
  g1.b_rows_per_expert = s.I;
  if (f8) {
    g1.a_scale = pa.xs;
    g1.b_scale0 = f8->gate;
    g1.b_scale1 = f8->up;
  }
  // Weights-as-M tiles pay off only when nearly every tile is tiny (decode-sized calls, a few
  // rows per expert); with larger tiles in the mix they measured slower.
  g1.swap_max_rows = L.R <= 8 * static_cast<int64_t>(s.E) ? kSwapMaxRows : 0;
  const int64_t max_tiles1 = L.mt_cap * g1.n_tiles_n;
  if (pairs) {
    g1.swap_max_rows = 0;
    const int64_t want = 2 * max_tiles1;
    const int grid = static_cast<int>(want < dev.pair_grid ? want : dev.pair_grid) & ~1;
    BEAM_LAUNCH(kKGemmGateUp, st, launch_gemm_gate_up_2sm(tm_xp, tm_g, tm_u, g1, grid, st));
  } else {
    const int grid1 = static_cast<int>(max_tiles1 < dev.sms ? max_tiles1 : dev.sms);
    BEAM_LAUNCH(kKGemmGateUp, st,
                launch_gemm_gate_up(tm_xp, tm_g, tm_u, g1, grid1, st, f8 != nullptr));
  }
  if (f8)
    BEAM_LAUNCH(kKQuantize, st,
                launch_quantize_rows(at<__nv_bfloat16>(ws, L.act), L.R, s.I,
                                     at<uint8_t>(ws, L.act8), at<float>(ws, L.as), st));

  GemmArgs g2 = g1;
  g2.out = at<__nv_bfloat16>(ws, L.y);
  g2.out_ld = s.d;
  g2.n_tiles_n = s.d / kN2;
  g2.k_blocks = s.I / k_elems;
  g2.b_rows_per_expert = s.d;
  if (f8) {
    g2.a_scale = at<float>(ws, L.as);
    g2.b_scale0 = f8->down;
    g2.b_scale1 = nullptr;
  }
  const int64_t max_tiles2 = L.mt_cap * g2.n_tiles_n;
  if (pairs) {
    CUtensorMap tm_d_half;  // each SM of a pair loads 128 of the tile's 256 weight rows
    if ((b = make_map(&tm_d_half, w_down, s.I, static_cast<uint64_t>(s.E) * s.d, kBM)) != BEAM_OK)
      return b;
    const int64_t want = 2 * max_tiles2;
    const int grid = static_cast<int>(want < dev.pair_grid ? want : dev.pair_grid) & ~1;
    BEAM_LAUNCH(kKGemmDown, st, launch_gemm_down_2sm(tm_act, tm_d_half, g2, grid, st));
  } else {
    const int grid2 = static_cast<int>(max_tiles2 < dev.sms ? max_tiles2 : dev.sms);
    BEAM_LAUNCH(kKGemmDown, st, launch_gemm_down(tm_act, tm_d, g2, grid2, st, f8 != nullptr));
  }
  return BEAM_OK;
}

// NVFP4 expert weights as produced by beam_moe_quantize_nvfp4: gate and up interleaved in
// 64-row chunks ([E, 2I] rows of d / 2 code bytes) and down ([E, d] rows of I / 2 bytes), each
// with its block-scale atoms and row scales.
struct Nvfp4Weights {
  const void* gu_codes;
  const void* gu_sf;
  const float* gu_scale;
  const void* d_codes;
  const void* d_sf;
  const float* d_scale;
};

// Dispatch and the two NVFP4 expert GEMMs; leaves Y and rowmap in the workspace.
beam_status run_experts_nvfp4(const beam_moe_shape& s, const Layout& L, const DeviceInfo& dev,
                              const __nv_bfloat16* h, const int32_t* idx, const Nvfp4Weights& w4,
                              void* ws, cudaStream_t st) {
  uint32_t* status = at<uint32_t>(ws, L.status);
  DispatchArgs da{};
  da.cnt = at<int32_t>(ws, L.cnt);
  da.bits = at<uint32_t>(ws, L.bits);
  da.base = at<int32_t>(ws, L.base);
  da.off = at<int32_t>(ws, L.off);
  da.mt_count = at<int32_t>(ws, L.mt_count);
  da.mtiles = at<MTile>(ws, L.mtiles);
  da.E = s.E;
  da.words = L.words;
  da.tile_rows = kBM;
  BEAM_LAUNCH(kKDispatchScan, st, launch_dispatch_scan(da, st));

  Fp4PermuteArgs pa{};
  pa.h = h;
  pa.idx = idx;
  pa.bits = da.bits;
  pa.base = da.base;
  pa.words = L.words;
  pa.cnt = da.cnt;
  pa.off = da.off;
  pa.rowmap = at<int32_t>(ws, L.rowmap);
  pa.xq = at<uint8_t>(ws, L.xp);
  pa.xsf = at<uint8_t>(ws, L.xsf);
  pa.xs = at<float>(ws, L.xs);
  pa.status = status;
  pa.T = s.T;
  pa.d = s.d;
  pa.k = s.top_k;
  pa.E = s.E;
  BEAM_LAUNCH(kKPermute, st, launch_nvfp4_permute(pa, st));

  const uint64_t R = static_cast<uint64_t>(L.R);
  ATensorMaps tm_x, tm_a;
  CUtensorMap tm_gu, tm_d;
  beam_status b;
  for (int i = 0; i < kNumABoxes; ++i) {
    if ((b = make_map(&tm_x.m[i], pa.xq, s.d / 2, R, a_box_rows(i), 1)) != BEAM_OK) return b;
    if ((b = make_map(&tm_a.m[i], at<void>(ws, L.act8), s.I / 2, R, a_box_rows(i), 1)) != BEAM_OK)
      return b;
  }
  const uint64_t E2I = static_cast<uint64_t>(s.E) * 2 * s.I, Ed = static_cast<uint64_t>(s.E) * s.d;
  if ((b = make_map(&tm_gu, w4.gu_codes, s.d / 2, E2I, kF4N, 1)) != BEAM_OK) return b;
  if ((b = make_map(&tm_d, w4.d_codes, s.I / 2, Ed, kF4N, 1)) != BEAM_OK) return b;

  Fp4GemmArgs g1{};
  g1.mtiles = da.mtiles;
  g1.mt_count = da.mt_count;
  g1.out = at<__nv_bfloat16>(ws, L.act);
  g1.status = status;
  g1.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  g1.out_ld = s.I;
  g1.n_tiles_n = 2 * s.I / kF4N;
  g1.k_blocks = s.d / kF4KElems;
  g1.b_rows_per_expert = 2 * s.I;
  g1.a_sf = pa.xsf;
  g1.b_sf = static_cast<const uint8_t*>(w4.gu_sf);
  g1.a_scale = pa.xs;
  g1.b_scale = w4.gu_scale;
  const int64_t max_tiles1 = L.mt_cap * g1.n_tiles_n;
  const int grid1 = static_cast<int>(max_tiles1 < dev.sms ? max_tiles1 : dev.sms);
  BEAM_LAUNCH(kKGemmGateUp, st, launch_gemm_nvfp4(true, tm_x, tm_gu, g1, grid1, st));

  Fp4ActArgs qa{};
  qa.x = g1.out;
  qa.mtiles = da.mtiles;
  qa.mt_count = da.mt_count;
  qa.q = at<uint8_t>(ws, L.act8);
  qa.sf = at<uint8_t>(ws, L.asf);
  qa.s = at<float>(ws, L.as);
  qa.cols = s.I;
  qa.mt_cap = static_cast<int>(L.mt_cap);
  BEAM_LAUNCH(kKQuantizeNvfp4, st, launch_nvfp4_act(qa, st));

  Fp4GemmArgs g2 = g1;
  g2.out = at<__nv_bfloat16>(ws, L.y);
  g2.out_ld = s.d;
  g2.n_tiles_n = s.d / kF4N;
  g2.k_blocks = s.I / kF4KElems;
  g2.b_rows_per_expert = s.d;
  g2.a_sf = qa.sf;
  g2.b_sf = static_cast<const uint8_t*>(w4.d_sf);
  g2.a_scale = qa.s;
  g2.b_scale = w4.d_scale;
  const int64_t max_tiles2 = L.mt_cap * g2.n_tiles_n;
  const int grid2 = static_cast<int>(max_tiles2 < dev.sms ? max_tiles2 : dev.sms);
  BEAM_LAUNCH(kKGemmDown, st, launch_gemm_nvfp4(false, tm_a, tm_d, g2, grid2, st));
  return BEAM_OK;
}

bool any_misaligned(std::initializer_list<const void*> ps) {
  for (const void* p : ps)
    if (!p || !aligned16(p)) return true;
  return false;
}

// ------------------------------------------------------------------ router without a workspace
//
// Scratch for beam_moe_route_static: one array per GPU, defined at file scope, so that the
// entry point needs neither a caller workspace nor any allocation.  Host code may not use the
// array's name as a device address (on the host it names a shadow variable); the device
// address is obtained once per device with cudaGetSymbolAddress and kept in static_scratch.
// Sized for the largest route plan with T <= kStaticRouteMaxTokens at any supported d and E:
// status words, per-expert counters, the transposed router weight (<= 256 x 8192 FP32) and
// up to 16 split-K partial logit arrays of T x 256 FP32.
constexpr int kStaticRouteMaxTokens = 512;
constexpr size_t kStaticRouteScratchBytes = (size_t(16) << 20) + 8192;
static __device__ __align__(256) unsigned char g_static_route_scratch[kStaticRouteScratchBytes];

// Offsets of the route-only plan inside the static scratch (status first, as in a workspace).
Layout plan_route_static(const beam_moe_shape& s) {
  Layout L{};
  L.R = static_cast<int64_t>(s.T) * s.top_k;
  const int64_t kblocks = s.d / kRK;
  const int S = router_split(s, 16);  // the static scratch holds 16 partial arrays
  L.kchunk = static_cast<int>(ceil_div(kblocks, S) * kRK);
  L.S = static_cast<int>(ceil_div(s.d, L.kchunk));
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 256);
    return r;
  };
  L.status = take(256);
  L.cnt = take(sizeof(int32_t) * s.E);
  L.wt = take(sizeof(float) * static_cast<size_t>(s.E) * s.d);
  L.part = take(sizeof(float) * static_cast<size_t>(L.S) * s.T * s.E);
  L.total = o;
  return L;
}

// Device address of this GPU's copy of the static scratch, looked up on first use per device.
beam_status static_scratch(void** out) {
  static void* addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= 64) return BEAM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_route_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    addr[dev] = p;
  }
  *out = addr[dev];
  return BEAM_OK;
}

// ------------------------------------------------------------------ dense SwiGLU MLP

beam_status check_dense_shape(const beam_dense_shape* s) {
  if (!s) return BEAM_ERR_INVALID_ARG;
  if (s->T < 0 || s->d <= 0 || s->I <= 0) return BEAM_ERR_INVALID_ARG;
  if (s->d % 256 != 0 || s->d > kMaxD || s->I % 128 != 0 || s->I > (1 << 20))
    return BEAM_ERR_UNSUPPORTED;
  return BEAM_OK;
}

struct DenseLayout {
  size_t status, mt_count, mtiles, act, total;
  size_t hq = 0, hs = 0, act8 = 0, as = 0;  // E4M3 form: quantised rows and their scales
  size_t hsf = 0, asf = 0;                    // NVFP4 form: block scales per m-tile
  int64_t mt_cap;
};

DenseLayout plan_dense(const beam_dense_shape& s) {
  DenseLayout L{};
  L.mt_cap = ceil_div(s.T, kBM);
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  L.status = take(256);
  L.mt_count = take(16);
  L.mtiles = take(sizeof(MTile) * L.mt_cap);
  L.act = take(sizeof(__nv_bfloat16) * static_cast<size_t>(s.T) * s.I);
  L.total = o;
  return L;
}

// E4M3 dense MLP: the BF16 layout plus the quantised token rows, the quantised activation and
// their row scales.
DenseLayout plan_dense_fp8(const beam_dense_shape& s) {
  DenseLayout L = plan_dense(s);
  size_t o = L.total;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  L.hq = take(static_cast<size_t>(s.T) * s.d);
  L.hs = take(sizeof(float) * s.T);
  L.act8 = take(static_cast<size_t>(s.T) * s.I);
  L.as = take(sizeof(float) * s.T);
  L.total = o;
  return L;
}

// NVFP4 dense MLP: the BF16 layout plus the token rows' codes, row scales and block-scale atoms,
// and the same for the activation (atoms per 128-row m-tile).
DenseLayout plan_dense_nvfp4(const beam_dense_shape& s) {
  DenseLayout L = plan_dense(s);
  size_t o = L.total;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  const size_t groups = static_cast<size_t>(L.mt_cap);
  L.hq = take(static_cast<size_t>(s.T) * (s.d / 2));
  L.hs = take(sizeof(float) * s.T);
  L.hsf = take(groups * (s.d / kF4KElems) * kF4SfaBytes);
  L.act8 = take(static_cast<size_t>(s.T) * (s.I / 2));
  L.as = take(sizeof(float) * s.T);
  L.asf = take(groups * (s.I / kF4KElems) * kF4SfaBytes);
  L.total = o;
  return L;
}

// ------------------------------------------------------------------ entry-point bodies
//
// The BF16 and E4M3 forms of each entry point share one body; f8 (non-null) carries the row
// scales of E4M3 expert weights.

bool misaligned_fp8(const Fp8Scales* f8) {
  return f8 && any_misaligned({f8->gate, f8->up, f8->down});
}

beam_status forward_impl(const beam_moe_shape* shape, const void* hidden, const float* router_w,
                         const float* bias, const void* w_gate, const void* w_up,
                         const void* w_down, void* out, int32_t* topk_idx, float* topk_w,
                         void* ws, size_t ws_bytes, beam_stream stream, const Fp8Scales* f8) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (any_misaligned({hidden, router_w, w_gate, w_up, w_down, out}) || misaligned_fp8(f8) ||
      !bias || (topk_idx && !aligned16(topk_idx)) || (topk_w && !aligned16(topk_w)))
    return BEAM_ERR_INVALID_ARG;
  const Layout L = f8 ? plan_fp8(*shape) : plan(*shape);
  if ((b = check_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.idx);
  float* w = topk_w ? topk_w : at<float>(ws, L.w);
  const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(hidden);
  if ((b = run_router(*shape, L, h, router_w, bias, idx, w, nullptr, true, ws, st)) != BEAM_OK)
    return b;
  if ((b = run_experts(*shape, L, *dev, h, idx, w_gate, w_up, w_down, ws, st, f8)) != BEAM_OK)
    return b;
  CombineArgs ca{};
  ca.y = at<__nv_bfloat16>(ws, L.y);
  ca.rowmap = at<int32_t>(ws, L.rowmap);
  ca.w = w;
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.status = at<uint32_t>(ws, L.status);
  ca.T = shape->T;
  ca.d = shape->d;
  ca.k = shape->top_k;
  ca.R = static_cast<int>(L.R);
  BEAM_LAUNCH(kKCombine, st, launch_combine(ca, st));
  return BEAM_OK;
}

beam_status forward_nvfp4_impl(const beam_moe_shape* shape, const void* hidden,
                               const float* router_w, const float* bias, const Nvfp4Weights& w4,
                               void* out, int32_t* topk_idx, float* topk_w, void* ws,
                               size_t ws_bytes, beam_stream stream) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->I % kF4KElems != 0) return BEAM_ERR_UNSUPPORTED;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (any_misaligned({hidden, router_w, w4.gu_codes, w4.gu_sf, w4.gu_scale, w4.d_codes, w4.d_sf,
                      w4.d_scale, out}) ||
      !bias || (topk_idx && !aligned16(topk_idx)) || (topk_w && !aligned16(topk_w)))
    return BEAM_ERR_INVALID_ARG;
  const Layout L = plan_nvfp4(*shape);
  if ((b = check_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.idx);
  float* w = topk_w ? topk_w : at<float>(ws, L.w);
  const __nv_bfloat16* h = static_cast<const __nv_bfloat16*>(hidden);
  if ((b = run_router(*shape, L, h, router_w, bias, idx, w, nullptr, true, ws, st)) != BEAM_OK)
    return b;
  if ((b = run_experts_nvfp4(*shape, L, *dev, h, idx, w4, ws, st)) != BEAM_OK) return b;
  CombineArgs ca{};
  ca.y = at<__nv_bfloat16>(ws, L.y);
  ca.rowmap = at<int32_t>(ws, L.rowmap);
  ca.w = w;
  ca.out = static_cast<__nv_bfloat16*>(out);
  ca.status = at<uint32_t>(ws, L.status);
  ca.T = shape->T;
  ca.d = shape->d;
  ca.k = shape->top_k;
  ca.R = static_cast<int>(L.R);
  BEAM_LAUNCH(kKCombine, st, launch_combine(ca, st));
  return BEAM_OK;
}

beam_status block_impl(const beam_moe_shape* shape, const float* x, const float* g_pre,
                       const float* g_post, float eps, int32_t k_resid, const float* router_w,
                       const float* bias, const void* w_gate, const void* w_up,
                       const void* w_down, float* x_out, int32_t* topk_idx, float* topk_w,
                       void* ws, size_t ws_bytes, beam_stream stream, const Fp8Scales* f8,
                       const Nvfp4Weights* w4 = nullptr) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (w4 && shape->I % kF4KElems != 0) return BEAM_ERR_UNSUPPORTED;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  // with w4, w_gate / w_up / w_down carry its gate|up codes, gate|up block scales, down codes
  if (any_misaligned({x, g_pre, g_post, router_w, w_gate, w_up, w_down, x_out}) ||
      misaligned_fp8(f8) || (w4 && any_misaligned({w4->gu_scale, w4->d_sf, w4->d_scale})) ||
      !bias || (topk_idx && !aligned16(topk_idx)) || (topk_w && !aligned16(topk_w)))
    return BEAM_ERR_INVALID_ARG;
  if (!(eps > 0.f) || !std::isfinite(eps) || k_resid < 1) return BEAM_ERR_INVALID_ARG;
  if (x_out != x) {  // in place or disjoint
    const char* a0 = reinterpret_cast<const char*>(x);
    const char* b0 = reinterpret_cast<const char*>(x_out);
    const size_t n = sizeof(float) * static_cast<size_t>(shape->T) * shape->d;
    if (a0 < b0 + n && b0 < a0 + n) return BEAM_ERR_INVALID_ARG;
  }
  const Layout L = w4 ? plan_nvfp4(*shape) : f8 ? plan_fp8(*shape) : plan(*shape);
  if ((b = check_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  PreNormArgs pn{};
  pn.x = x;
  pn.g_pre = g_pre;
  pn.h = at<__nv_bfloat16>(ws, L.h);
  pn.eps = eps;
  pn.T = shape->T;
  pn.d = shape->d;
  BEAM_LAUNCH(kKPreNorm, st, launch_prenorm(pn, st));

  int32_t* idx = topk_idx ? topk_idx : at<int32_t>(ws, L.idx);
  float* w = topk_w ? topk_w : at<float>(ws, L.w);
  if ((b = run_router(*shape, L, pn.h, router_w, bias, idx, w, nullptr, true, ws, st)) != BEAM_OK)
    return b;
  b = w4 ? run_experts_nvfp4(*shape, L, *dev, pn.h, idx, *w4, ws, st)
         : run_experts(*shape, L, *dev, pn.h, idx, w_gate, w_up, w_down, ws, st, f8);
  if (b != BEAM_OK) return b;
  const double kk = static_cast<double>(k_resid);
  CombineArgs ca{};
  ca.y = at<__nv_bfloat16>(ws, L.y);
  ca.rowmap = at<int32_t>(ws, L.rowmap);
  ca.w = w;
  ca.x = x;
  ca.g_post = g_post;
  ca.x_out = x_out;
  ca.eps = eps;
  ca.coef_x = static_cast<float>(std::sqrt((kk - 1.0) / kk));
  ca.coef_f = static_cast<float>(1.0 / std::sqrt(kk));
  ca.status = at<uint32_t>(ws, L.status);
  ca.T = shape->T;
  ca.d = shape->d;
  ca.k = shape->top_k;
  ca.R = static_cast<int>(L.R);
  BEAM_LAUNCH(kKCombineBlock, st, launch_combine_block(ca, st));
  return BEAM_OK;
}

// Dense SwiGLU MLP: one "expert" holding every token.  The E4M3 form quantises the token rows
// and the activation per row, as the MoE path does.
// Dense SwiGLU MLP on NVFP4 weights: 128-row tiles of consecutive tokens; the token rows are
// quantised into their tile's atoms by the activation quantiser, then the two block-scaled GEMMs
// run with the activation quantised between them.
beam_status dense_nvfp4_impl(const beam_dense_shape* shape, const void* hidden,
                             const Nvfp4Weights& w4, void* out, void* ws, size_t ws_bytes,
                             beam_stream stream) {
  beam_status b = check_dense_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->I % kF4KElems != 0) return BEAM_ERR_UNSUPPORTED;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (any_misaligned({hidden, w4.gu_codes, w4.gu_sf, w4.gu_scale, w4.d_codes, w4.d_sf,
                      w4.d_scale, out}))
    return BEAM_ERR_INVALID_ARG;
  const DenseLayout L = plan_dense_nvfp4(*shape);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < L.total)
    return BEAM_ERR_WORKSPACE;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const beam_dense_shape& s = *shape;
  uint32_t* status = at<uint32_t>(ws, L.status);
  cudaError_t e = cudaMemsetAsync(status, 0, 16, st);
  if (e != cudaSuccess) return cuda_fail(e);
  MTile* mtiles = at<MTile>(ws, L.mtiles);
  int32_t* mt_count = at<int32_t>(ws, L.mt_count);
  BEAM_LAUNCH(kKDenseTiles, st, launch_dense_tiles(s.T, mtiles, mt_count, st));

  Fp4ActArgs qh{};
  qh.x = static_cast<const __nv_bfloat16*>(hidden);
  qh.mtiles = mtiles;
  qh.mt_count = mt_count;
  qh.q = at<uint8_t>(ws, L.hq);
  qh.sf = at<uint8_t>(ws, L.hsf);
  qh.s = at<float>(ws, L.hs);
  qh.cols = s.d;
  qh.mt_cap = static_cast<int>(L.mt_cap);
  BEAM_LAUNCH(kKQuantizeNvfp4, st, launch_nvfp4_act(qh, st));

  ATensorMaps tm_h, tm_a;
  CUtensorMap tm_gu, tm_d;
  for (int i = 0; i < kNumABoxes; ++i) {
    if ((b = make_map(&tm_h.m[i], qh.q, s.d / 2, s.T, a_box_rows(i), 1)) != BEAM_OK) return b;
    if ((b = make_map(&tm_a.m[i], at<void>(ws, L.act8), s.I / 2, s.T, a_box_rows(i), 1)) !=
        BEAM_OK)
      return b;
  }
  if ((b = make_map(&tm_gu, w4.gu_codes, s.d / 2, 2 * static_cast<uint64_t>(s.I), kF4N, 1)) !=
      BEAM_OK)
    return b;
  if ((b = make_map(&tm_d, w4.d_codes, s.I / 2, s.d, kF4N, 1)) != BEAM_OK) return b;

  Fp4GemmArgs g1{};
  g1.mtiles = mtiles;
  g1.mt_count = mt_count;
  g1.out = at<__nv_bfloat16>(ws, L.act);
  g1.status = status;
  g1.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  g1.out_ld = s.I;
  g1.n_tiles_n = 2 * s.I / kF4N;
  g1.k_blocks = s.d / kF4KElems;
  g1.b_rows_per_expert = 2 * s.I;
  g1.a_sf = qh.sf;
  g1.b_sf = static_cast<const uint8_t*>(w4.gu_sf);
  g1.a_scale = qh.s;
  g1.b_scale = w4.gu_scale;
  const int64_t t1 = L.mt_cap * g1.n_tiles_n;
  BEAM_LAUNCH(kKGemmGateUp, st,
              launch_gemm_nvfp4(true, tm_h, tm_gu, g1,
                                static_cast<int>(t1 < dev->sms ? t1 : dev->sms), st));

  Fp4ActArgs qa = qh;
  qa.x = g1.out;
  qa.q = at<uint8_t>(ws, L.act8);
  qa.sf = at<uint8_t>(ws, L.asf);
  qa.s = at<float>(ws, L.as);
  qa.cols = s.I;
  BEAM_LAUNCH(kKQuantizeNvfp4, st, launch_nvfp4_act(qa, st));

  Fp4GemmArgs g2 = g1;
  g2.out = static_cast<__nv_bfloat16*>(out);
  g2.out_ld = s.d;
  g2.n_tiles_n = s.d / kF4N;
  g2.k_blocks = s.I / kF4KElems;
  g2.b_rows_per_expert = s.d;
  g2.a_sf = qa.sf;
  g2.b_sf = static_cast<const uint8_t*>(w4.d_sf);
  g2.a_scale = qa.s;
  g2.b_scale = w4.d_scale;
  const int64_t t2 = L.mt_cap * g2.n_tiles_n;
  BEAM_LAUNCH(kKGemmDown, st,
              launch_gemm_nvfp4(false, tm_a, tm_d, g2,
                                static_cast<int>(t2 < dev->sms ? t2 : dev->sms), st));
  return BEAM_OK;
}

beam_status dense_impl(const beam_dense_shape* shape, const void* hidden, const void* w_gate,
                       const void* w_up, const void* w_down, void* out, void* ws,
                       size_t ws_bytes, beam_stream stream, const Fp8Scales* f8) {
  beam_status b = check_dense_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (any_misaligned({hidden, w_gate, w_up, w_down, out}) || misaligned_fp8(f8))
    return BEAM_ERR_INVALID_ARG;
  const DenseLayout L = f8 ? plan_dense_fp8(*shape) : plan_dense(*shape);
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < L.total)
    return BEAM_ERR_WORKSPACE;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const beam_dense_shape& s = *shape;
  uint32_t* status = at<uint32_t>(ws, L.status);
  cudaError_t e = cudaMemsetAsync(status, 0, 16, st);
  if (e != cudaSuccess) return cuda_fail(e);
  MTile* mtiles = at<MTile>(ws, L.mtiles);
  int32_t* mt_count = at<int32_t>(ws, L.mt_count);
  BEAM_LAUNCH(kKDenseTiles, st, launch_dense_tiles(s.T, mtiles, mt_count, st));

  void* act = at<void>(ws, L.act);
  const void* a1 = hidden;
  const void* a2 = act;
  if (f8) {
    BEAM_LAUNCH(kKQuantize, st,
                launch_quantize_rows(static_cast<const __nv_bfloat16*>(hidden), s.T, s.d,
                                     at<uint8_t>(ws, L.hq), at<float>(ws, L.hs), st));
    a1 = at<void>(ws, L.hq);
    a2 = at<void>(ws, L.act8);
  }
  const int eb = f8 ? 1 : 2;
  const int k_elems = 128 / eb;
  ATensorMaps tm_h, tm_act;
  CUtensorMap tm_g, tm_u, tm_d;
  for (int i = 0; i < kNumABoxes; ++i) {
    if ((b = make_map(&tm_h.m[i], a1, s.d, s.T, a_box_rows(i), eb)) != BEAM_OK) return b;
    if ((b = make_map(&tm_act.m[i], a2, s.I, s.T, a_box_rows(i), eb)) != BEAM_OK) return b;
  }
  if ((b = make_map(&tm_g, w_gate, s.d, s.I, kN1Half, eb)) != BEAM_OK) return b;
  if ((b = make_map(&tm_u, w_up, s.d, s.I, kN1Half, eb)) != BEAM_OK) return b;
  if ((b = make_map(&tm_d, w_down, s.I, s.d, kN2, eb)) != BEAM_OK) return b;

  GemmArgs g1{};
  g1.mtiles = mtiles;
  g1.mt_count = mt_count;
  g1.out = static_cast<__nv_bfloat16*>(act);
  g1.status = status;
  g1.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  g1.out_ld = s.I;
  g1.n_tiles_n = s.I / kN1Half;
  g1.k_blocks = s.d / k_elems;
  g1.b_rows_per_expert = s.I;
  g1.swap_max_rows = 0;
  if (f8) {
    g1.a_scale = at<float>(ws, L.hs);
    g1.b_scale0 = f8->gate;
    g1.b_scale1 = f8->up;
  }
  const int64_t t1 = L.mt_cap * g1.n_tiles_n;
  BEAM_LAUNCH(kKGemmGateUp, st,
              launch_gemm_gate_up(tm_h, tm_g, tm_u, g1,
                                  static_cast<int>(t1 < dev->sms ? t1 : dev->sms), st,
                                  f8 != nullptr));
  if (f8)
    BEAM_LAUNCH(kKQuantize, st,
                launch_quantize_rows(static_cast<const __nv_bfloat16*>(act), s.T, s.I,
                                     at<uint8_t>(ws, L.act8), at<float>(ws, L.as), st));
  GemmArgs g2 = g1;
  g2.out = static_cast<__nv_bfloat16*>(out);
  g2.out_ld = s.d;
  g2.n_tiles_n = s.d / kN2;
  g2.k_blocks = s.I / k_elems;
  g2.b_rows_per_expert = s.d;
  if (f8) {
    g2.a_scale = at<float>(ws, L.as);
    g2.b_scale0 = f8->down;
    g2.b_scale1 = nullptr;
  }
  const int64_t t2 = L.mt_cap * g2.n_tiles_n;
  BEAM_LAUNCH(kKGemmDown, st,
              launch_gemm_down(tm_act, tm_d, g2,
                               static_cast<int>(t2 < dev->sms ? t2 : dev->sms), st,
                               f8 != nullptr));
  return BEAM_OK;
}

// ------------------------------------------------------------------ expert parallelism
//
// P ranks, rank p owning experts p * E / P .. (p + 1) * E / P - 1 (see ep.cu for the steps and
// the row layout).  The workspace of a rank holds its dispatch state (counts, token bitmap and
// its prefix counts, each slot's owner and row) and its expert side (the m-tiles over the
// received rows and the SwiGLU activation); the receive buffers of token rows and expert
// outputs are the caller's, since peers write and read them.

struct EpLayout {
  size_t status, cnt, bits, zero_bytes, base, row_off, slot_row, slot_owner, cnt_local, off,
      mt_count, mtiles, act, total;
  int words;
  int64_t mt_cap;
};

beam_status check_ep(const beam_moe_shape* s, int P, int64_t recv_cap) {
  beam_status b = check_shape(s);
  if (b != BEAM_OK) return b;
  if (P < 1 || P > kMaxEpRanks || s->E % P != 0) return BEAM_ERR_UNSUPPORTED;
  if (recv_cap < 1 || recv_cap >= (int64_t(1) << 31)) return BEAM_ERR_INVALID_ARG;
  return BEAM_OK;
}

EpLayout plan_ep(const beam_moe_shape& s, int P, int64_t recv_cap) {
  EpLayout L{};
  const int64_t R = static_cast<int64_t>(s.T) * s.top_k;
  const int ep = s.E / P;
  L.words = static_cast<int>(ceil_div(s.T > 0 ? s.T : 1, 32));
  L.mt_cap = ceil_div(recv_cap, kBM) + ep;
  const size_t bitmap_bytes = sizeof(uint32_t) * static_cast<size_t>(s.E) * L.words;
  size_t o = 0;
  auto take = [&](size_t bytes) {
    const size_t r = o;
    o = align_up(o + (bytes ? bytes : 1), 1024);
    return r;
  };
  L.status = take(256);
  L.cnt = take(sizeof(int32_t) * s.E);
  L.bits = take(bitmap_bytes);
  L.zero_bytes = L.bits + bitmap_bytes;
  L.base = take(bitmap_bytes);
  L.row_off = take(sizeof(int64_t) * s.E);
  L.slot_row = take(sizeof(int32_t) * R);
  L.slot_owner = take(sizeof(int32_t) * R);
  L.cnt_local = take(sizeof(int32_t) * ep);
  L.off = take(sizeof(int32_t) * (ep + 1));
  L.mt_count = take(16);
  L.mtiles = take(sizeof(MTile) * L.mt_cap);
  L.act = take(sizeof(__nv_bfloat16) * static_cast<size_t>(recv_cap) * s.I);
  L.total = o;
  return L;
}

beam_status check_ep_ws(const EpLayout& L, void* ws, size_t ws_bytes) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < L.total)
    return BEAM_ERR_WORKSPACE;
  return BEAM_OK;
}

}  // namespace

extern "C" {

int beam_moe_abi_version(void) { return 1; }

beam_status beam_moe_route_static(const beam_moe_shape* shape, const void* hidden,
                                  const float* router_w, const float* bias, int32_t* topk_idx,
                                  float* topk_w, float* logits_out, beam_stream stream) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (any_misaligned({hidden, router_w, topk_idx, topk_w}) || !bias ||
      (logits_out && !aligned16(logits_out)))
    return BEAM_ERR_INVALID_ARG;
  if (shape->T > kStaticRouteMaxTokens) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                  "beam_moe_route_static: T = %d exceeds the static-scratch limit of %d tokens",
                  shape->T, kStaticRouteMaxTokens);
    return BEAM_ERR_UNSUPPORTED;
  }
  const Layout L = plan_route_static(*shape);
  if (L.total > kStaticRouteScratchBytes) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                  "beam_moe_route_static: needs %zu bytes of scratch, the static array holds %zu",
                  L.total, kStaticRouteScratchBytes);
    return BEAM_ERR_UNSUPPORTED;
  }
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  void* scratch = nullptr;
  if ((b = static_scratch(&scratch)) != BEAM_OK) return b;
  return run_router(*shape, L, static_cast<const __nv_bfloat16*>(hidden), router_w, bias, topk_idx,
                    topk_w, logits_out, false, scratch, reinterpret_cast<cudaStream_t>(stream));
}

size_t beam_moe_workspace_size(const beam_moe_shape* shape) {
  if (check_shape(shape) != BEAM_OK) return 0;
  return plan(*shape).total;
}

const char* beam_status_string(beam_status s) {
  switch (s) {
    case BEAM_OK: return "BEAM_OK";
    case BEAM_ERR_INVALID_ARG: return "BEAM_ERR_INVALID_ARG";
    case BEAM_ERR_UNSUPPORTED: return "BEAM_ERR_UNSUPPORTED";
    case BEAM_ERR_WORKSPACE: return "BEAM_ERR_WORKSPACE";
    case BEAM_ERR_CUDA: return "BEAM_ERR_CUDA";
    case BEAM_ERR_TIMEOUT: return "BEAM_ERR_TIMEOUT";
    case BEAM_ERR_DEVICE_ASSERT: return "BEAM_ERR_DEVICE_ASSERT";
  }
  return "BEAM_ERR_UNKNOWN";
}

const char* beam_moe_last_cuda_error(void) { return g_last_cuda_error; }

void beam_moe_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }
void beam_moe_set_sm_pairs(int enable) { g_sm_pairs.store(enable ? 1 : 0); }
int beam_moe_get_sm_pairs(void) { return g_sm_pairs.load(); }
uint64_t beam_moe_get_wait_limit_ns(void) { return g_wait_limit_ns.load(); }
uint64_t beam_moe_launch_count(void) { return g_launches.load(); }

beam_status beam_moe_route(const beam_moe_shape* shape, const void* hidden, const float* router_w,
                           const float* bias, int32_t* topk_idx, float* topk_w, float* logits_out,
                           void* ws, size_t ws_bytes, beam_stream stream) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (any_misaligned({hidden, router_w, topk_idx, topk_w}) || !bias ||
      (logits_out && !aligned16(logits_out)))
    return BEAM_ERR_INVALID_ARG;
  const Layout L = plan(*shape);
  if ((b = check_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return run_router(*shape, L, static_cast<const __nv_bfloat16*>(hidden), router_w, bias, topk_idx,
                    topk_w, logits_out, false, ws, st);
}


size_t beam_moe_fp8_workspace_size(const beam_moe_shape* shape) {
  if (check_shape(shape) != BEAM_OK) return 0;
  return plan_fp8(*shape).total;
}

beam_status beam_moe_quantize_e4m3(const void* x, int64_t rows, int32_t cols, void* q,
                                   float* scale, beam_stream stream) {
  if (rows < 0 || cols <= 0 || cols % 16 != 0) return BEAM_ERR_INVALID_ARG;
  if (rows == 0) return BEAM_OK;
  if (any_misaligned({x, q}) || !scale) return BEAM_ERR_INVALID_ARG;
  const uintptr_t xb = reinterpret_cast<uintptr_t>(x), qb = reinterpret_cast<uintptr_t>(q);
  const uint64_t xbytes = static_cast<uint64_t>(rows) * cols * 2;
  if (qb < xb + xbytes && xb < qb + static_cast<uint64_t>(rows) * cols)
    return BEAM_ERR_INVALID_ARG;  // the codes may not overwrite the input
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  BEAM_LAUNCH(kKQuantize, st,
              launch_quantize_rows(static_cast<const __nv_bfloat16*>(x), rows, cols,
                                   static_cast<uint8_t*>(q), scale, st));
  return BEAM_OK;
}



size_t beam_moe_nvfp4_workspace_size(const beam_moe_shape* shape) {
  if (check_shape(shape) != BEAM_OK || shape->I % kF4KElems != 0) return 0;
  return plan_nvfp4(*shape).total;
}

beam_status beam_moe_quantize_nvfp4(const void* a, const void* b, int64_t groups, int32_t rows,
                                    int32_t cols, void* codes, void* block_scales,
                                    float* row_scales, beam_stream stream) {
  if (groups < 0 || rows <= 0 || cols <= 0 || cols % kF4KElems != 0 ||
      rows % (b ? 64 : 128) != 0)
    return BEAM_ERR_INVALID_ARG;
  if (groups == 0) return BEAM_OK;
  if (any_misaligned({a, codes, block_scales, row_scales}) || (b && !aligned16(b)))
    return BEAM_ERR_INVALID_ARG;
  const uint64_t in_bytes = static_cast<uint64_t>(groups) * rows * cols * 2;
  const uint64_t out_rows = static_cast<uint64_t>(groups) * (b ? 2 * rows : rows);
  const uint64_t outs[3][2] = {{reinterpret_cast<uintptr_t>(codes), out_rows * (cols / 2)},
                               {reinterpret_cast<uintptr_t>(block_scales), out_rows * (cols / 16)},
                               {reinterpret_cast<uintptr_t>(row_scales), out_rows * 4}};
  for (const void* in : {a, b}) {
    if (!in) continue;
    const uint64_t ib = reinterpret_cast<uintptr_t>(in);
    for (const auto& o : outs)
      if (o[0] < ib + in_bytes && ib < o[0] + o[1]) return BEAM_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  BEAM_LAUNCH(kKQuantizeNvfp4, st,
              launch_nvfp4_weights(static_cast<const __nv_bfloat16*>(a),
                                   static_cast<const __nv_bfloat16*>(b), groups, rows, cols,
                                   static_cast<uint8_t*>(codes),
                                   static_cast<uint8_t*>(block_scales), row_scales, st));
  return BEAM_OK;
}

beam_status beam_moe_forward_nvfp4(const beam_moe_shape* shape, const void* hidden,
                                   const float* router_w, const float* bias,
                                   const void* gate_up_codes, const void* gate_up_block_scales,
                                   const float* gate_up_scales, const void* down_codes,
                                   const void* down_block_scales, const float* down_scales,
                                   void* out, int32_t* topk_idx, float* topk_w, void* ws,
                                   size_t ws_bytes, beam_stream stream) {
  const Nvfp4Weights w4{gate_up_codes, gate_up_block_scales, gate_up_scales,
                        down_codes,    down_block_scales,    down_scales};
  return forward_nvfp4_impl(shape, hidden, router_w, bias, w4, out, topk_idx, topk_w, ws,
                            ws_bytes, stream);
}

beam_status beam_moe_forward(const beam_moe_shape* shape, const void* hidden, const float* router_w,
                             const float* bias, const void* w_gate, const void* w_up,
                             const void* w_down, void* out, int32_t* topk_idx, float* topk_w,
                             void* ws, size_t ws_bytes, beam_stream stream) {
  return forward_impl(shape, hidden, router_w, bias, w_gate, w_up, w_down, out, topk_idx, topk_w,
                      ws, ws_bytes, stream, nullptr);
}

beam_status beam_moe_forward_fp8(const beam_moe_shape* shape, const void* hidden,
                                 const float* router_w, const float* bias, const void* w_gate,
                                 const float* gate_scale, const void* w_up, const float* up_scale,
                                 const void* w_down, const float* down_scale, void* out,
                                 int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                                 beam_stream stream) {
  const Fp8Scales f8{gate_scale, up_scale, down_scale};
  return forward_impl(shape, hidden, router_w, bias, w_gate, w_up, w_down, out, topk_idx, topk_w,
                      ws, ws_bytes, stream, &f8);
}

beam_status beam_moe_block_nvfp4(const beam_moe_shape* shape, const float* x, const float* g_pre,
                                 const float* g_post, float eps, int32_t k_resid,
                                 const float* router_w, const float* bias,
                                 const void* gate_up_codes, const void* gate_up_block_scales,
                                 const float* gate_up_scales, const void* down_codes,
                                 const void* down_block_scales, const float* down_scales,
                                 float* x_out, int32_t* topk_idx, float* topk_w, void* ws,
                                 size_t ws_bytes, beam_stream stream) {
  const Nvfp4Weights w4{gate_up_codes, gate_up_block_scales, gate_up_scales,
                        down_codes,    down_block_scales,    down_scales};
  return block_impl(shape, x, g_pre, g_post, eps, k_resid, router_w, bias, gate_up_codes,
                    gate_up_block_scales, down_codes, x_out, topk_idx, topk_w, ws, ws_bytes,
                    stream, nullptr, &w4);
}

size_t beam_dense_nvfp4_workspace_size(const beam_dense_shape* shape) {
  if (check_dense_shape(shape) != BEAM_OK || shape->I % kF4KElems != 0) return 0;
  return plan_dense_nvfp4(*shape).total;
}

beam_status beam_dense_forward_nvfp4(const beam_dense_shape* shape, const void* hidden,
                                     const void* gate_up_codes, const void* gate_up_block_scales,
                                     const float* gate_up_scales, const void* down_codes,
                                     const void* down_block_scales, const float* down_scales,
                                     void* out, void* ws, size_t ws_bytes, beam_stream stream) {
  const Nvfp4Weights w4{gate_up_codes, gate_up_block_scales, gate_up_scales,
                        down_codes,    down_block_scales,    down_scales};
  return dense_nvfp4_impl(shape, hidden, w4, out, ws, ws_bytes, stream);
}

beam_status beam_moe_block(const beam_moe_shape* shape, const float* x, const float* g_pre,
                           const float* g_post, float eps, int32_t k_resid, const float* router_w,
                           const float* bias, const void* w_gate, const void* w_up,
                           const void* w_down, float* x_out, int32_t* topk_idx, float* topk_w,
                           void* ws, size_t ws_bytes, beam_stream stream) {
  return block_impl(shape, x, g_pre, g_post, eps, k_resid, router_w, bias, w_gate, w_up, w_down,
                    x_out, topk_idx, topk_w, ws, ws_bytes, stream, nullptr);
}

beam_status beam_moe_block_fp8(const beam_moe_shape* shape, const float* x, const float* g_pre,
                               const float* g_post, float eps, int32_t k_resid,
                               const float* router_w, const float* bias, const void* w_gate,
                               const float* gate_scale, const void* w_up, const float* up_scale,
                               const void* w_down, const float* down_scale, float* x_out,
                               int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                               beam_stream stream) {
  const Fp8Scales f8{gate_scale, up_scale, down_scale};
  return block_impl(shape, x, g_pre, g_post, eps, k_resid, router_w, bias, w_gate, w_up, w_down,
                    x_out, topk_idx, topk_w, ws, ws_bytes, stream, &f8);
}

beam_status beam_dense_forward(const beam_dense_shape* shape, const void* hidden,
                               const void* w_gate, const void* w_up, const void* w_down,
                               void* out, void* ws, size_t ws_bytes, beam_stream stream) {
  return dense_impl(shape, hidden, w_gate, w_up, w_down, out, ws, ws_bytes, stream, nullptr);
}

size_t beam_dense_fp8_workspace_size(const beam_dense_shape* shape) {
  if (check_dense_shape(shape) != BEAM_OK) return 0;
  return plan_dense_fp8(*shape).total;
}

beam_status beam_dense_forward_fp8(const beam_dense_shape* shape, const void* hidden,
                                   const void* w_gate, const float* gate_scale, const void* w_up,
                                   const float* up_scale, const void* w_down,
                                   const float* down_scale, void* out, void* ws, size_t ws_bytes,
                                   beam_stream stream) {
  const Fp8Scales f8{gate_scale, up_scale, down_scale};
  return dense_impl(shape, hidden, w_gate, w_up, w_down, out, ws, ws_bytes, stream, &f8);
}

size_t beam_dense_workspace_size(const beam_dense_shape* shape) {
  if (check_dense_shape(shape) != BEAM_OK) return 0;
  return plan_dense(*shape).total;
}


beam_status beam_moe_bias_update(const beam_moe_shape* shape, const void* ws, float* bias,
                                 float gamma, beam_stream stream) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (shape->T == 0) return BEAM_OK;  // nothing to read or write
  if (!ws || !bias || !std::isfinite(gamma)) return BEAM_ERR_INVALID_ARG;
  const Layout L = plan(*shape);
  const float mean = static_cast<float>(static_cast<double>(L.R) / shape->E);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  BEAM_LAUNCH(kKBiasUpdate, st,
              launch_bias_update(reinterpret_cast<const int32_t*>(static_cast<const char*>(ws) + L.cnt),
                                 bias, shape->E, mean, gamma, st));
  return BEAM_OK;
}

beam_status beam_moe_sync_status(void* ws, beam_stream stream) {
  if (!ws) return BEAM_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e);
  uint32_t words[4] = {0, 0, 0, 0};
  e = cudaMemcpy(words, ws, sizeof words, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  if (words[0] == kDevOk) return BEAM_OK;
  std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error,
                "device status %u at site %u, block %u", words[0], words[1], words[2]);
  e = cudaMemset(ws, 0, sizeof words);
  if (e != cudaSuccess) return cuda_fail(e);
  return words[0] == kDevTimeout ? BEAM_ERR_TIMEOUT : BEAM_ERR_DEVICE_ASSERT;
}

beam_status beam_moe_expert_counts(const beam_moe_shape* shape, const void* ws,
                                   int32_t* counts_host, beam_stream stream) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (!ws || !counts_host) return BEAM_ERR_INVALID_ARG;
  const Layout L = plan(*shape);
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpy(counts_host, static_cast<const char*>(ws) + L.cnt, sizeof(int32_t) * shape->E,
                 cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  return BEAM_OK;
}

beam_status beam_moe_slot_rows(const beam_moe_shape* shape, const void* ws, int32_t* rows_host,
                               beam_stream stream) {
  beam_status b = check_shape(shape);
  if (b != BEAM_OK) return b;
  if (!ws || !rows_host) return BEAM_ERR_INVALID_ARG;
  if (shape->T == 0) return BEAM_OK;
  const Layout L = plan(*shape);
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaMemcpy(rows_host, static_cast<const char*>(ws) + L.rowmap,
                 sizeof(int32_t) * static_cast<size_t>(L.R), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e);
  return BEAM_OK;
}

void beam_moe_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  g_prof.on = on != 0;
}

void beam_moe_profile_reset(void) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  for (auto& r : g_prof.pending) {
    cudaEventSynchronize(r.b);
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.pending.clear();
  for (int i = 0; i < kNumKernels; ++i) {
    g_prof.launches[i] = 0;
    g_prof.ms[i] = 0.0;
  }
}

int beam_moe_kernel_count(void) { return kNumKernels; }

const char* beam_moe_kernel_name(int id) {
  return id >= 0 && id < kNumKernels ? kKernelNames[id] : "";
}

beam_status beam_moe_profile_read(int id, int64_t* launches, double* total_ms) {
  if (id < 0 || id >= kNumKernels || !launches || !total_ms) return BEAM_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lk(g_prof.mu);
  for (auto& r : g_prof.pending) {
    cudaError_t e = cudaEventSynchronize(r.b);
    if (e != cudaSuccess) return cuda_fail(e);
    float ms = 0.f;
    e = cudaEventElapsedTime(&ms, r.a, r.b);
    if (e != cudaSuccess) return cuda_fail(e);
    g_prof.launches[r.id] += 1;
    g_prof.ms[r.id] += ms;
    g_prof.pool.push_back(r.a);
    g_prof.pool.push_back(r.b);
  }
  g_prof.pending.clear();
  *launches = g_prof.launches[id];
  *total_ms = g_prof.ms[id];
  return BEAM_OK;
}

// ------------------------------------------------------------------ expert parallelism

size_t beam_moe_ep_workspace_size(const beam_moe_shape* shape, int32_t P, int64_t recv_rows_max) {
  if (check_ep(shape, P, recv_rows_max) != BEAM_OK) return 0;
  return plan_ep(*shape, P, recv_rows_max).total;
}

beam_status beam_moe_enable_peer_access(int32_t peer_device) {
  int cur = 0, n = 0;
  if (cudaGetDevice(&cur) != cudaSuccess || cudaGetDeviceCount(&n) != cudaSuccess)
    return BEAM_ERR_CUDA;
  if (peer_device < 0 || peer_device >= n) return BEAM_ERR_INVALID_ARG;
  if (peer_device == cur) return BEAM_OK;
  int can = 0;
  if (cudaDeviceCanAccessPeer(&can, cur, peer_device) != cudaSuccess) return BEAM_ERR_CUDA;
  if (!can) return BEAM_ERR_UNSUPPORTED;
  const cudaError_t e = cudaDeviceEnablePeerAccess(peer_device, 0);
  if (e == cudaErrorPeerAccessAlreadyEnabled) {
    cudaGetLastError();  // the call also left this error as the last one: clear it
    return BEAM_OK;
  }
  return e == cudaSuccess ? BEAM_OK : BEAM_ERR_CUDA;
}

beam_status beam_moe_ep_plan(int32_t P, int32_t E, const int32_t* all_counts, int32_t rank,
                             int64_t* recv_rows, int64_t* send_rows, int64_t* recv_from) {
  if (P < 1 || P > kMaxEpRanks || E < 1 || E % P != 0 || rank < 0 || rank >= P || !all_counts)
    return BEAM_ERR_INVALID_ARG;
  const int ep = E / P;
  for (int i = 0; i < P * E; ++i)
    if (all_counts[i] < 0) return BEAM_ERR_INVALID_ARG;
  int64_t recv = 0;
  for (int q = 0; q < P; ++q) {
    int64_t to_q = 0, from_q = 0;
    for (int e = q * ep; e < (q + 1) * ep; ++e) to_q += all_counts[static_cast<size_t>(rank) * E + e];
    for (int e = rank * ep; e < (rank + 1) * ep; ++e) from_q += all_counts[static_cast<size_t>(q) * E + e];
    if (send_rows) send_rows[q] = to_q;
    if (recv_from) recv_from[q] = from_q;
    recv += from_q;
  }
  if (recv_rows) *recv_rows = recv;
  return BEAM_OK;
}

beam_status beam_moe_ep_count(const beam_moe_shape* shape, int32_t P, const int32_t* topk_idx,
                              int32_t* counts, int64_t recv_rows_max, void* ws, size_t ws_bytes,
                              beam_stream stream) {
  beam_status b = check_ep(shape, P, recv_rows_max);
  if (b != BEAM_OK) return b;
  if (!counts || !aligned16(counts) || (shape->T > 0 && (!topk_idx || !aligned16(topk_idx))))
    return BEAM_ERR_INVALID_ARG;
  const EpLayout L = plan_ep(*shape, P, recv_rows_max);
  if ((b = check_ep_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(ws, 0, L.zero_bytes, st);
  if (e != cudaSuccess) return cuda_fail(e);
  EpCountArgs a{};
  a.idx = topk_idx;
  a.cnt = at<int32_t>(ws, L.cnt);
  a.bits = at<uint32_t>(ws, L.bits);
  a.words = L.words;
  a.status = at<uint32_t>(ws, L.status);
  a.T = shape->T;
  a.k = shape->top_k;
  a.E = shape->E;
  if (shape->T > 0) BEAM_LAUNCH(kKEpCount, st, launch_ep_count(a, st));
  e = cudaMemcpyAsync(counts, a.cnt, sizeof(int32_t) * shape->E, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return cuda_fail(e);
  return BEAM_OK;
}

beam_status beam_moe_ep_dispatch(const beam_moe_shape* shape, int32_t P, int32_t rank,
                                 const void* hidden, const int32_t* topk_idx,
                                 const int32_t* all_counts, void* const* xrecv_peers,
                                 int64_t recv_rows_max, void* ws, size_t ws_bytes,
                                 beam_stream stream) {
  beam_status b = check_ep(shape, P, recv_rows_max);
  if (b != BEAM_OK) return b;
  if (rank < 0 || rank >= P || !xrecv_peers) return BEAM_ERR_INVALID_ARG;
  if (shape->T == 0) return BEAM_OK;  // nothing to send
  if (any_misaligned({hidden, topk_idx, all_counts})) return BEAM_ERR_INVALID_ARG;
  for (int q = 0; q < P; ++q)
    if (!xrecv_peers[q] || !aligned16(xrecv_peers[q])) return BEAM_ERR_INVALID_ARG;
  const EpLayout L = plan_ep(*shape, P, recv_rows_max);
  if ((b = check_ep_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  EpOffsetsArgs oa{};
  oa.all = all_counts;
  oa.bits = at<uint32_t>(ws, L.bits);
  oa.base = at<int32_t>(ws, L.base);
  oa.row_off = at<int64_t>(ws, L.row_off);
  oa.words = L.words;
  oa.P = P;
  oa.E = shape->E;
  oa.rank = rank;
  BEAM_LAUNCH(kKEpOffsets, st, launch_ep_offsets(oa, st));
  EpPushArgs pa{};
  pa.h = static_cast<const __nv_bfloat16*>(hidden);
  pa.idx = topk_idx;
  pa.bits = oa.bits;
  pa.base = oa.base;
  pa.words = L.words;
  pa.row_off = oa.row_off;
  pa.slot_row = at<int32_t>(ws, L.slot_row);
  pa.slot_owner = at<int32_t>(ws, L.slot_owner);
  for (int q = 0; q < P; ++q) pa.xrecv[q] = static_cast<__nv_bfloat16*>(xrecv_peers[q]);
  pa.recv_cap = recv_rows_max;
  pa.status = at<uint32_t>(ws, L.status);
  pa.T = shape->T;
  pa.d = shape->d;
  pa.k = shape->top_k;
  pa.E = shape->E;
  pa.P = P;
  BEAM_LAUNCH(kKEpPush, st, launch_ep_push(pa, st));
  return BEAM_OK;
}

beam_status beam_moe_ep_experts(const beam_moe_shape* shape, int32_t P, int32_t rank,
                                int64_t T_total, const int32_t* all_counts, const void* w_gate,
                                const void* w_up, const void* w_down, const void* xrecv,
                                void* yrecv, int64_t recv_rows_max, void* ws, size_t ws_bytes,
                                beam_stream stream) {
  beam_status b = check_ep(shape, P, recv_rows_max);
  if (b != BEAM_OK) return b;
  if (rank < 0 || rank >= P || T_total < 0) return BEAM_ERR_INVALID_ARG;
  if (any_misaligned({all_counts, w_gate, w_up, w_down, xrecv, yrecv})) return BEAM_ERR_INVALID_ARG;
  const EpLayout L = plan_ep(*shape, P, recv_rows_max);
  if ((b = check_ep_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  DeviceInfo* dev;
  if ((b = device_info(&dev)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int ep = shape->E / P;
  uint32_t* status = at<uint32_t>(ws, L.status);
  BEAM_LAUNCH(kKEpLocalCounts, st,
              launch_ep_local_counts(all_counts, P, shape->E, rank, recv_rows_max,
                                     at<int32_t>(ws, L.cnt_local), status, st));
  DispatchArgs da{};
  da.cnt = at<int32_t>(ws, L.cnt_local);
  da.bits = nullptr;  // the received rows are already in place: no bitmap ranks to form
  da.base = nullptr;
  da.off = at<int32_t>(ws, L.off);
  da.mt_count = at<int32_t>(ws, L.mt_count);
  da.mtiles = at<MTile>(ws, L.mtiles);
  da.E = ep;
  da.words = 0;
  da.tile_rows = kBM;
  BEAM_LAUNCH(kKDispatchScan, st, launch_dispatch_scan(da, st));

  const uint64_t R = static_cast<uint64_t>(recv_rows_max);
  ATensorMaps tm_x, tm_act;
  CUtensorMap tm_g, tm_u, tm_d;
  void* act = at<void>(ws, L.act);
  for (int i = 0; i < kNumABoxes; ++i) {
    if ((b = make_map(&tm_x.m[i], xrecv, shape->d, R, a_box_rows(i))) != BEAM_OK) return b;
    if ((b = make_map(&tm_act.m[i], act, shape->I, R, a_box_rows(i))) != BEAM_OK) return b;
  }
  const uint64_t EI = static_cast<uint64_t>(ep) * shape->I, Ed = static_cast<uint64_t>(ep) * shape->d;
  if ((b = make_map(&tm_g, w_gate, shape->d, EI, kN1Half)) != BEAM_OK) return b;
  if ((b = make_map(&tm_u, w_up, shape->d, EI, kN1Half)) != BEAM_OK) return b;
  if ((b = make_map(&tm_d, w_down, shape->I, Ed, kN2)) != BEAM_OK) return b;
  GemmArgs g1{};
  g1.mtiles = da.mtiles;
  g1.mt_count = da.mt_count;
  g1.out = static_cast<__nv_bfloat16*>(act);
  g1.status = status;
  g1.wait_limit_ns = g_wait_limit_ns.load(std::memory_order_relaxed);
  g1.out_ld = shape->I;
  g1.n_tiles_n = shape->I / kN1Half;
  g1.k_blocks = shape->d / kBK;
  g1.b_rows_per_expert = shape->I;
  // the single-GPU forward's choice for the whole batch, so that every tile is computed alike
  g1.swap_max_rows = T_total * shape->top_k <= 8 * static_cast<int64_t>(shape->E) ? kSwapMaxRows : 0;
  const int64_t max1 = L.mt_cap * g1.n_tiles_n;
  BEAM_LAUNCH(kKGemmGateUp, st,
              launch_gemm_gate_up(tm_x, tm_g, tm_u, g1, static_cast<int>(max1 < dev->sms ? max1 : dev->sms), st));
  GemmArgs g2 = g1;
  g2.out = static_cast<__nv_bfloat16*>(yrecv);
  g2.out_ld = shape->d;
  g2.n_tiles_n = shape->d / kN2;
  g2.k_blocks = shape->I / kBK;
  g2.b_rows_per_expert = shape->d;
  const int64_t max2 = L.mt_cap * g2.n_tiles_n;
  BEAM_LAUNCH(kKGemmDown, st,
              launch_gemm_down(tm_act, tm_d, g2, static_cast<int>(max2 < dev->sms ? max2 : dev->sms), st));
  return BEAM_OK;
}

beam_status beam_moe_ep_combine(const beam_moe_shape* shape, int32_t P, const float* topk_w,
                                const void* const* yrecv_peers, int64_t recv_rows_max, void* out,
                                void* ws, size_t ws_bytes, beam_stream stream) {
  beam_status b = check_ep(shape, P, recv_rows_max);
  if (b != BEAM_OK) return b;
  if (!yrecv_peers) return BEAM_ERR_INVALID_ARG;
  if (shape->T == 0) return BEAM_OK;
  if (any_misaligned({topk_w, out})) return BEAM_ERR_INVALID_ARG;
  for (int q = 0; q < P; ++q)
    if (!yrecv_peers[q] || !aligned16(yrecv_peers[q])) return BEAM_ERR_INVALID_ARG;
  const EpLayout L = plan_ep(*shape, P, recv_rows_max);
  if ((b = check_ep_ws(L, ws, ws_bytes)) != BEAM_OK) return b;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  EpCombineArgs a{};
  a.slot_row = at<int32_t>(ws, L.slot_row);
  a.slot_owner = at<int32_t>(ws, L.slot_owner);
  a.w = topk_w;
  for (int q = 0; q < P; ++q) a.yrecv[q] = static_cast<const __nv_bfloat16*>(yrecv_peers[q]);
  a.out = static_cast<__nv_bfloat16*>(out);
  a.recv_cap = recv_rows_max;
  a.status = at<uint32_t>(ws, L.status);
  a.T = shape->T;
  a.d = shape->d;
  a.k = shape->top_k;
  a.P = P;
  BEAM_LAUNCH(kKEpCombine, st, launch_ep_combine(a, st));
  return BEAM_OK;
}

}  // extern "C"
