// Router launch shapes shared by the router kernels and the workspace planner.
#pragma once

namespace beam {

// Batches of at most this many tokens run the 32-token router GEMM tile and the one-token
// selection form; their split-K count is kRouterSmallSplit.
constexpr int kRouterSmallT = 64;
constexpr int kRouterSmallSplit = 64;
constexpr int kSelSmallT = 1024;  // batches up to this size take the one-token selection form

}  // namespace beam
