// Expert parallelism: the layer's experts split over P GPUs in contiguous blocks of E / P
// ("Use HF Transformers" cookbook, section Parallelism: with ep_size = 8 each GPU holds 32 of the
// 256 experts and tokens travel to the GPU that holds their experts).
//
// Every rank routes its own tokens, then (one call per step, stream-ordered):
//   count     per-expert slot counts and the token bitmap of its slots        (local)
//   [counts of all ranks gathered by the caller: all[P, E]]
//   dispatch  each slot's row on the owner of its expert; the token row is written straight
//             into the owner's receive buffer (a peer store over NVLink when the owner is
//             another GPU)
//   [barrier: every rank's rows have landed]
//   experts   the grouped GEMMs over the received rows (owner-local)
//   [barrier: every owner's Y rows are complete]
//   combine   each token's k expert outputs read back from their owners' Y buffers (peer
//             loads) and summed with the routing weights in ascending expert order
//
// Row layout on owner q: its experts in ascending order; inside expert e the rows of rank 0,
// then rank 1, ..., each rank's in ascending local token order.  With ranks' tokens numbered
// rank-major this is the single-GPU layout of the same global batch restricted to q's experts,
// so every m-tile (and hence every Y row) is the one a single GPU computes, and the combine's
// fixed order makes the output bit-identical to the single-GPU forward with the same routing.
#include "beam_moe_internal.cuh"

namespace beam {
namespace {

// Per-slot counts and the token bitmap (bit t of expert e's row) of the local routing.
__global__ void __launch_bounds__(256) ep_count_kernel(const EpCountArgs a) {
  const int64_t slot = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (slot >= static_cast<int64_t>(a.T) * a.k) return;
  const int t = static_cast<int>(slot / a.k);
  const int e = a.idx[slot];
  if (e < 0 || e >= a.E) {
    record_status(a.status, kDevAssert, kWhereDispatch);
    return;
  }
  atomicAdd(a.cnt + e, 1);
  atomicOr(a.bits + static_cast<size_t>(e) * a.words + (t >> 5), 1u << (t & 31));
}

// A warp per expert e (all E): the row on e's owner where this rank's first slot of e lands,
//   row_off[e] = sum_{owner's experts e' < e} sum_p all[p][e'] + sum_{p < rank} all[p][e],
// and the exclusive prefix counts of e's row of the local token bitmap.
__global__ void __launch_bounds__(256) ep_offsets_kernel(const EpOffsetsArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= a.E) return;  // uniform over the warp
  const int ep = a.E / a.P;
  const int first = (e / ep) * ep;
  int64_t before = 0;
  for (int i = lane; i < (e - first) * a.P; i += 32) {
    const int ee = first + i / a.P, p = i % a.P;
    before += a.all[static_cast<size_t>(p) * a.E + ee];
  }
  for (int p = lane; p < a.rank; p += 32) before += a.all[static_cast<size_t>(p) * a.E + e];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) before += __shfl_xor_sync(0xffffffffu, before, off);
  if (lane == 0) a.row_off[e] = before;
  const uint32_t* bits = a.bits + static_cast<size_t>(e) * a.words;
  int32_t* base = a.base + static_cast<size_t>(e) * a.words;
  int run = 0;
  for (int w0 = 0; w0 < a.words; w0 += 32) {
    const int w = w0 + lane;
    const int n = w < a.words ? __popc(bits[w]) : 0;
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

constexpr uint64_t kPushWaitNs = 4000000000ull;  // bound of a row copy's wait for its load

// 1-D bulk copy global -> shared completing on mbarrier `bar` (16-byte aligned, bytes % 16 == 0).
__device__ __forceinline__ void bulk_load_row(uint32_t dst, const void* src, uint32_t bytes,
                                              uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(dst),
      "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(bar)
      : "memory");
}

// 1-D bulk copy shared -> global (local or a peer's memory) in the thread's bulk group.
__device__ __forceinline__ void bulk_store_row(void* dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
                   reinterpret_cast<uint64_t>(dst)),
               "r"(src), "r"(bytes)
               : "memory");
}

// A CTA of one warp per token: lanes below top_k find their slots' owners and rows; lane 0 reads
// the token row into shared memory with one bulk copy and writes it to each owner's receive
// buffer with bulk stores (peer memory for other GPUs), then waits until those writes are done
// and fences them, so that they are visible to the owners before this kernel completes.  A row
// beyond the owner's receive capacity is recorded and skipped.
__global__ void __launch_bounds__(32) ep_push_kernel(const EpPushArgs a) {
  extern __shared__ __align__(128) uint8_t row_sh[];
  __shared__ __align__(8) uint64_t bar_sh;
  const int lane = threadIdx.x;
  const int t = blockIdx.x;
  const int ep = a.E / a.P;
  int row = -1, owner = 0;
  if (lane < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + lane;
    const int e = a.idx[slot];
    const int r = e >= 0 && e < a.E ? slot_rank(a.bits, a.base, a.words, e, t) : -1;
    if (r >= 0) {
      const int64_t rr = a.row_off[e] + r;
      if (rr < a.recv_cap) {
        row = static_cast<int>(rr);
        owner = e / ep;
      }
    }
    if (row < 0) record_status(a.status, kDevAssert, kWhereDispatch);
    a.slot_row[slot] = row;
    a.slot_owner[slot] = owner;
  }
  int rows[kMaxTopK], owners[kMaxTopK];
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, row, j);
    owners[j] = __shfl_sync(0xffffffffu, owner, j);
  }
  if (lane != 0) return;
  const uint32_t bar = smem_u32(&bar_sh);
  const uint32_t bytes = static_cast<uint32_t>(a.d) * 2u;
  mbar_init(bar, 1);
  fence_mbarrier_init();
  mbar_arrive_expect_tx(bar, bytes);
  bulk_load_row(smem_u32(row_sh), a.h + static_cast<size_t>(t) * a.d, bytes, bar);
  int abort_flag = 0;
  if (!mbar_wait_bounded(bar, 0, &abort_flag, kPushWaitNs, a.status, kWhereDispatch)) {
    int no_abort = 0;  // the load must land before this CTA's shared memory is released
    mbar_wait_bounded(bar, 0, &no_abort, 1000000000ull, a.status, kWhereDispatch);
    return;
  }
#pragma unroll
  for (int j = 0; j < kMaxTopK; ++j)
    if (j < a.k && rows[j] >= 0)
      bulk_store_row(a.xrecv[owners[j]] + static_cast<size_t>(rows[j]) * a.d, smem_u32(row_sh),
                     bytes);
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // the writes are complete
  asm volatile("fence.proxy.async.global;" ::: "memory");
  __threadfence_system();
}

// Rows of this rank's experts received from all ranks, cnt_local[el] = sum_p all[p][rank*ep+el],
// cut so that their total stays within the receive capacity (the dispatch skipped, and
// recorded, every row beyond it).
__global__ void __launch_bounds__(32) ep_local_counts_kernel(const int32_t* all, int P, int E,
                                                            int rank, int64_t recv_cap,
                                                            int32_t* cnt_local, uint32_t* status) {
  // One warp: lane l sums experts l, l + 32, ... over the ranks; a warp scan gives each expert's
  // uncut prefix S.  The cut count is min(c, max(0, cap - S)), which is what cutting the experts
  // one after another in ascending order gives.
  const int lane = threadIdx.x;
  const int ep = E / P;
  int64_t run = 0;
  bool over = false;
  for (int el0 = 0; el0 < ep; el0 += 32) {
    const int el = el0 + lane;
    int64_t c = 0;
    if (el < ep)
      for (int p = 0; p < P; ++p) c += all[static_cast<size_t>(p) * E + rank * ep + el];
    int64_t incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int64_t o = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += o;
    }
    const int64_t before = run + incl - c;
    const int64_t room = recv_cap - before;
    const int64_t cut = c < room ? c : (room > 0 ? room : 0);
    if (cut != c) over = true;
    if (el < ep) cnt_local[el] = static_cast<int32_t>(cut);
    run += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (__any_sync(0xffffffffu, over) && lane == 0) record_status(status, kDevAssert, kWhereDispatch);
}

// out[t] = sum_j w[t, j] * Y_owner(j)[row(j)], j in slot (ascending expert) order, FP32 FMAs:
// the arithmetic of the single-GPU combine, with each expert output read from its owner.
constexpr int kEpCThreads = 128;  // a CTA per 128 16-byte pieces of a token's row

__global__ void __launch_bounds__(kEpCThreads) ep_combine_kernel(const EpCombineArgs a) {
  __shared__ const __nv_bfloat16* src[kMaxTopK];
  __shared__ float wsh[kMaxTopK];
  const int nvec = a.d / 8;
  const int chunks = (nvec + kEpCThreads - 1) / kEpCThreads;
  const int t = blockIdx.x / chunks;
  const int chunk = blockIdx.x % chunks;
  if (threadIdx.x < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + threadIdx.x;
    const int r = a.slot_row[slot];
    const int q = a.slot_owner[slot];
    const bool sent = r >= 0 && r < a.recv_cap && q >= 0 && q < a.P;
    if (!sent && chunk == 0) record_status(a.status, kDevAssert, kWhereCombine);
    // a slot that was not sent adds nothing
    src[threadIdx.x] = sent ? a.yrecv[q] + static_cast<size_t>(r) * a.d : nullptr;
    wsh[threadIdx.x] = a.w[slot];
  }
  __syncthreads();
  uint4* out = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.d);
  const int c = chunk * kEpCThreads + threadIdx.x;
  if (c < nvec) {
    uint4 v[kMaxTopK];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j)
      if (j < a.k && src[j]) v[j] = reinterpret_cast<const uint4*>(src[j])[c];
    float acc[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) acc[q] = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k && src[j]) {
        const uint32_t wv[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] = fmaf(wsh[j], __uint_as_float(wv[q] << 16), acc[2 * q]);
          acc[2 * q + 1] = fmaf(wsh[j], __uint_as_float(wv[q] & 0xffff0000u), acc[2 * q + 1]);
        }
      }
    }
    uint32_t p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
      p[q] = *reinterpret_cast<uint32_t*>(&b);
    }
    out[c] = make_uint4(p[0], p[1], p[2], p[3]);
  }
}

}  // namespace

cudaError_t launch_ep_count(const EpCountArgs& a, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(a.T) * a.k;
  if (n == 0) return cudaSuccess;
  ep_count_kernel<<<static_cast<unsigned>((n + 255) / 256), 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_offsets(const EpOffsetsArgs& a, cudaStream_t s) {
  ep_offsets_kernel<<<(a.E + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_push(const EpPushArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  ep_push_kernel<<<a.T, 32, static_cast<size_t>(a.d) * 2, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_local_counts(const int32_t* all, int P, int E, int rank, int64_t recv_cap,
                                   int32_t* cnt_local, uint32_t* status, cudaStream_t s) {
  ep_local_counts_kernel<<<1, 32, 0, s>>>(all, P, E, rank, recv_cap, cnt_local, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const EpCombineArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  const unsigned chunks = static_cast<unsigned>((a.d / 8 + kEpCThreads - 1) / kEpCThreads);
  ep_combine_kernel<<<static_cast<unsigned>(a.T) * chunks, kEpCThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
