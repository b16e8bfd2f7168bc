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

// One warp per token: each slot's owner and row, then the token row written to each of its
// top_k destinations (local or peer receive buffers, 16-byte stores).  A row beyond the
// owner's receive capacity is recorded and skipped.
__global__ void __launch_bounds__(256) ep_push_kernel(const EpPushArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= a.T) return;
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
  const uint4* src = reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(t) * a.d);
  const int nvec = a.d / 8;
  for (int c = lane; c < nvec; c += 32) {
    const uint4 v = src[c];
#pragma unroll
    for (int j = 0; j < kMaxTopK; ++j) {
      if (j < a.k && rows[j] >= 0)
        reinterpret_cast<uint4*>(a.xrecv[owners[j]] + static_cast<size_t>(rows[j]) * a.d)[c] = v;
    }
  }
  // the rows written into other GPUs' memory are visible to them before this kernel completes
  __threadfence_system();
}

// Rows of this rank's experts received from all ranks, cnt_local[el] = sum_p all[p][rank*ep+el],
// cut so that their total stays within the receive capacity (the dispatch skipped, and
// recorded, every row beyond it).
__global__ void ep_local_counts_kernel(const int32_t* all, int P, int E, int rank,
                                       int64_t recv_cap, int32_t* cnt_local, uint32_t* status) {
  if (threadIdx.x != 0) return;
  const int ep = E / P;
  int64_t total = 0;
  for (int el = 0; el < ep; ++el) {
    int64_t c = 0;
    for (int p = 0; p < P; ++p) c += all[static_cast<size_t>(p) * E + rank * ep + el];
    if (total + c > recv_cap) {
      record_status(status, kDevAssert, kWhereDispatch);
      c = recv_cap - total;
    }
    cnt_local[el] = static_cast<int32_t>(c);
    total += c;
  }
}

// out[t] = sum_j w[t, j] * Y_owner(j)[row(j)], j in slot (ascending expert) order, FP32 FMAs:
// the arithmetic of the single-GPU combine, with each expert output read from its owner.
constexpr int kEpCThreads = 128;

__global__ void __launch_bounds__(kEpCThreads) ep_combine_kernel(const EpCombineArgs a) {
  __shared__ const __nv_bfloat16* src[kMaxTopK];
  __shared__ float wsh[kMaxTopK];
  const int t = blockIdx.x;
  if (threadIdx.x < a.k) {
    const size_t slot = static_cast<size_t>(t) * a.k + threadIdx.x;
    const int r = a.slot_row[slot];
    const int q = a.slot_owner[slot];
    const __nv_bfloat16* p = nullptr;  // a slot that was not sent adds nothing
    if (r < 0 || r >= a.recv_cap || q < 0 || q >= a.P)
      record_status(a.status, kDevAssert, kWhereCombine);
    else
      p = a.yrecv[q] + static_cast<size_t>(r) * a.d;
    src[threadIdx.x] = p;
    wsh[threadIdx.x] = a.w[slot];
  }
  __syncthreads();
  const int nvec = a.d / 8;
  uint4* out = reinterpret_cast<uint4*>(a.out + static_cast<size_t>(t) * a.d);
  for (int c = threadIdx.x; c < nvec; c += kEpCThreads) {
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
  ep_push_kernel<<<(a.T + 7) / 8, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_ep_local_counts(const int32_t* all, int P, int E, int rank, int64_t recv_cap,
                                   int32_t* cnt_local, uint32_t* status, cudaStream_t s) {
  ep_local_counts_kernel<<<1, 32, 0, s>>>(all, P, E, rank, recv_cap, cnt_local, status);
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const EpCombineArgs& a, cudaStream_t s) {
  if (a.T == 0) return cudaSuccess;
  ep_combine_kernel<<<a.T, kEpCThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace beam
