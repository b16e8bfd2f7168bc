// Router launch shapes shared by the router kernels and the workspace planner.
#pragma once
#include "beam_moe_internal.cuh"

namespace beam {

// Batches of at most this many tokens run the 32-token router GEMM tile and the one-token
// selection form; their split-K count is kRouterSmallSplit.
constexpr int kRouterSmallT = 64;
constexpr int kRouterSmallSplit = 64;
constexpr int kSelSmallT = 1024;  // batches up to this size take the one-token selection form

// The router GEMM of a batch of at most kRouterSmallT tokens, reading W_r [E, d] as stored
// (the large-batch form reads the transposed copy that launch_router_transpose writes).
cudaError_t launch_router_gemm_small(const RouterGemmArgs& a, const float* W, int S,
                                     cudaStream_t s);

}  // namespace beam
