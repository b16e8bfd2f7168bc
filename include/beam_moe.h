/*
 * beam_moe.h -- C ABI of the B200 (sm_100a) forward pass of one Beam sparse-MoE layer.
 *
 * The layer (Transformers model doc "Beam", Overview, "Sparse MoE" bullet, and
 * BeamConfig; archdb fact sheet "Beam-1.0-501B-A23B", expert-groups entry; news
 * article "Reflection lança o Beam", section "Onde o Beam economiza ..."):
 *
 *   logits  = h . W_r^T                      FP32 router weights, FP32 logits
 *   s       = sigmoid(logits)                FP32
 *   sb      = s + bias                       bias chooses experts, never weighs them
 *   gs_g    = top1(sb in g) + top2(sb in g)  groups are contiguous runs of E/n_group experts
 *   keep the topk_group groups of largest gs, then the top_k experts of largest sb
 *   among them (ties: lower group / expert index wins)
 *   w       = routed_scaling_factor * s / sum(s over chosen)   (norm_topk_prob)
 *   y_e     = W_down,e . ( silu(W_gate,e . h) * (W_up,e . h) )  SwiGLU in FP32, BF16 weights
 *   out     = sum_j w_j y_{e_j}                no shared expert
 *
 * and its block form (Overview, "Sandwich norms with depth-scaled residuals"; archdb
 * residual-design entry): h = RMSNorm(x) * g_pre (FP32, then BF16), the layer above,
 * o = RMSNorm(out) * g_post, x' = x * sqrt((k-1)/k) + o / sqrt(k).
 *
 * Conventions shared by every entry point
 *  - All tensor pointers are DEVICE pointers on the current CUDA device, owned by the
 *    caller, row-major and dense.  The library allocates no device memory: scratch space
 *    is the caller's workspace `ws` of at least beam_moe_workspace_size() bytes, aligned
 *    to 256 bytes.  Tensor pointers must be 16-byte aligned.
 *  - Calls are asynchronous on `stream` (NULL = legacy default stream).  Argument errors
 *    are returned before anything is launched; a failed launch returns BEAM_ERR_CUDA.
 *    Errors found on the device (a bounded wait that ran out, a failed index check)
 *    are recorded in a status word inside `ws` and read by beam_moe_sync_status().
 *  - One workspace serves one call at a time: calls that share a workspace must be
 *    ordered on one stream.
 *  - The first call on each device sets the GEMM kernels' shared-memory limits (make it
 *    outside any stream capture); this per-device set-up lasts for the process and does not
 *    survive cudaDeviceReset, so reset a device only when done with the library on it.
 *  - Outputs topk_idx [T, top_k] list the chosen experts in ascending id order; topk_w
 *    [T, top_k] holds their weights in the same order; the combine sums in that order,
 *    so results are deterministic run to run.
 *  - Supported shapes: d % 256 == 0, d <= 8192, I % 128 == 0, 1 <= E <= 256,
 *    E % 4 == 0, E % n_group == 0, n_group <= 32, 1 <= topk_group <= n_group, 1 <= top_k <= 8,
 *    top_k <= topk_group * E / n_group, T >= 0, T * top_k < 2^31; the NVFP4 entry points
 *    also need I % 256 == 0.  Others return BEAM_ERR_UNSUPPORTED.  T == 0 is a no-op that
 *    reads no pointer (they may be NULL).
 *  - Expert weights come in three forms with the same entry-point structure: BF16
 *    (beam_moe_forward / _block, beam_dense_forward), E4M3 with FP32 row scales (the _fp8
 *    forms) and NVFP4 with E4M3 block scales and FP32 row scales (the _nvfp4 forms).
 */
#ifndef BEAM_MOE_H_
#define BEAM_MOE_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BEAM_API __attribute__((visibility("default")))
#else
#define BEAM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BEAM_OK = 0,
  BEAM_ERR_INVALID_ARG = 1,    /* NULL / misaligned pointer, bad scalar */
  BEAM_ERR_UNSUPPORTED = 2,    /* shape outside the supported set */
  BEAM_ERR_WORKSPACE = 3,      /* ws NULL, misaligned or smaller than required */
  BEAM_ERR_CUDA = 4,           /* a CUDA runtime / driver call failed */
  BEAM_ERR_TIMEOUT = 5,        /* a device-side bounded wait ran out (read by sync_status) */
  BEAM_ERR_DEVICE_ASSERT = 6   /* a device-side index check failed (read by sync_status) */
} beam_status;

/* Layer configuration; field names follow BeamConfig. */
typedef struct {
  int32_t T;                    /* tokens in this call */
  int32_t d;                    /* hidden_size (5120 for Beam) */
  int32_t E;                    /* num_experts (256) */
  int32_t n_group;              /* n_group (8) */
  int32_t topk_group;           /* topk_group (4) */
  int32_t top_k;                /* num_experts_per_tok (8) */
  int32_t I;                    /* moe_intermediate_size (2560) */
  float routed_scaling_factor;  /* 2.5 */
  int32_t norm_topk_prob;       /* nonzero: weights normalised to sum 1 before scaling */
} beam_moe_shape;

/* Same type as cudaStream_t. */
typedef struct CUstream_st* beam_stream;

/* Bytes of workspace the given shape needs for route, forward or block (the maximum of
 * the three); 0 if the shape is unsupported or NULL. */
BEAM_API size_t beam_moe_workspace_size(const beam_moe_shape* shape);

/* Router only: logits, sigmoid, bias, group-limited top-k, weights.
 *   hidden     BF16 [T, d]
 *   router_w   FP32 [E, d]
 *   bias       FP32 [E]
 *   topk_idx   INT32 [T, top_k] out, ascending expert id per token
 *   topk_w     FP32 [T, top_k] out, weights aligned with topk_idx (sum = scale if normalised)
 *   logits_out FP32 [T, E] out (the raw router logits), or NULL
 * Cites: "Beam" model doc, Overview ("Sparse MoE" bullet, FP32 routing) and Notes
 * ("output_router_logits=True still returns the router logits"). */
BEAM_API beam_status beam_moe_route(const beam_moe_shape* shape, const void* hidden, const float* router_w,
                           const float* bias, int32_t* topk_idx, float* topk_w, float* logits_out,
                           void* ws, size_t ws_bytes, beam_stream stream);

/* Router only, like beam_moe_route, for callers that cannot allocate device memory and have
 * no workspace to pass: for example a serving engine that has handed all device memory to its
 * own pool, or a host process that forbids device allocation (and the device-wide
 * synchronisation cudaMalloc / cudaFree may cause) on its request path.  The pages have no
 * counterpart to this entry point; it exists only for such callers.
 *
 * Scratch space is one static array of 16 MiB + 8 KiB in this library's device image; every
 * GPU that loads the library holds a copy until the process exits.  It bounds T to at most
 * 512 tokens (any supported d and E); larger T returns BEAM_ERR_UNSUPPORTED with the reason in
 * beam_moe_last_cuda_error().  Nothing is allocated: the first call on each device looks up
 * the array's device address (cudaGetSymbolAddress), so make that first call before any
 * stream capture.  All calls share the array and it keeps the last call's contents (each call
 * clears what must start at zero): calls that overlap on the GPU -- on different streams, or
 * from different host threads -- race on it and must be serialised by the caller.
 * Arguments, layouts and outputs are those of beam_moe_route.  With no workspace there is no
 * status word to read back: the one device-side check of the router (a token left with fewer
 * than top_k candidate experts, which a supported shape with finite logits never produces)
 * shows only in its outputs, whose missing entries are expert 0 with weight 0.  The cached
 * array address belongs to the device's current context: cudaDeviceReset invalidates it (as it
 * does the library's other per-device set-up), so reset a device only when done with it. */
BEAM_API beam_status beam_moe_route_static(const beam_moe_shape* shape, const void* hidden,
                                           const float* router_w, const float* bias,
                                           int32_t* topk_idx, float* topk_w, float* logits_out,
                                           beam_stream stream);

/* Whole MoE layer forward.
 *   hidden           BF16 [T, d]
 *   router_w, bias   as for beam_moe_route
 *   w_gate, w_up     BF16 [E, I, d]  (per expert nn.Linear weight: out x in)
 *   w_down           BF16 [E, d, I]
 *   out              BF16 [T, d] out
 *   topk_idx, topk_w optional outputs (NULL: kept inside ws)
 * Cites: "Beam" model doc, Overview ("Sparse MoE" bullet; SwiGLU in FP32) and BeamConfig
 * (moe_intermediate_size, num_experts_per_tok, routed_scaling_factor). */
BEAM_API beam_status beam_moe_forward(const beam_moe_shape* shape, const void* hidden, const float* router_w,
                             const float* bias, const void* w_gate, const void* w_up,
                             const void* w_down, void* out, int32_t* topk_idx, float* topk_w,
                             void* ws, size_t ws_bytes, beam_stream stream);

/* ---- FP8 (E4M3) expert weights
 *
 * The pages name FP8 and NVFP4 checkpoints of the model (news article "Reflection lança o
 * Beam", section "Onde o Beam economiza ..."; review page "обзор модели «Бим»", weights and
 * vLLM-recipe entries) but no scale format.  This path reads the plainest one the tensor cores
 * take directly: E4M3 codes with one FP32 scale per row, s = fl32(amax / 448) and
 * q = e4m3(fl32(x / s)) rounded to nearest even, saturating to +-448 (an all-zero row has
 * s = 0 and zero codes).  Weights are quantised per output channel, activations per token
 * row: the token rows entering the gate/up GEMM and the SwiGLU activation (after its BF16
 * rounding) entering the down GEMM.  Each GEMM multiplies codes on the tensor cores with FP32
 * accumulation and applies both row scales in its epilogue.  Routing is unchanged. */

/* Row-wise E4M3 quantisation of a BF16 matrix x [rows, cols] (row-major) into codes q
 * [rows, cols] (uint8) and scales scale [rows] (FP32), on `stream`.  Used once per model to
 * convert the expert weights: w_gate and w_up as [E * I, d], w_down as [E * d, I].
 * cols must be a positive multiple of 16; x and q 16-byte aligned and not overlapping.
 * Returns BEAM_ERR_INVALID_ARG otherwise; rows == 0 is a no-op. */
BEAM_API beam_status beam_moe_quantize_e4m3(const void* x, int64_t rows, int32_t cols, void* q,
                                            float* scale, beam_stream stream);

/* Workspace bytes for beam_moe_forward_fp8 (0 for an unsupported shape). */
BEAM_API size_t beam_moe_fp8_workspace_size(const beam_moe_shape* shape);

/* beam_moe_forward with E4M3 expert weights.
 *   w_gate, w_up     E4M3 [E, I, d] with row scales gate_scale, up_scale FP32 [E * I]
 *   w_down           E4M3 [E, d, I] with row scales down_scale FP32 [E * d]
 *   (as written by beam_moe_quantize_e4m3); every other argument as for beam_moe_forward,
 *   with ws sized by beam_moe_fp8_workspace_size.  Scale arrays must be 16-byte aligned. */
BEAM_API beam_status beam_moe_forward_fp8(const beam_moe_shape* shape, const void* hidden,
                                          const float* router_w, const float* bias,
                                          const void* w_gate, const float* gate_scale,
                                          const void* w_up, const float* up_scale,
                                          const void* w_down, const float* down_scale, void* out,
                                          int32_t* topk_idx, float* topk_w, void* ws,
                                          size_t ws_bytes, beam_stream stream);

/* beam_moe_block with E4M3 expert weights (codes and row scales as for beam_moe_forward_fp8);
 * every other argument as for beam_moe_block, with ws sized by beam_moe_fp8_workspace_size. */
BEAM_API beam_status beam_moe_block_fp8(const beam_moe_shape* shape, const float* x,
                                        const float* g_pre, const float* g_post, float eps,
                                        int32_t k_resid, const float* router_w, const float* bias,
                                        const void* w_gate, const float* gate_scale,
                                        const void* w_up, const float* up_scale,
                                        const void* w_down, const float* down_scale,
                                        float* x_out, int32_t* topk_idx, float* topk_w, void* ws,
                                        size_t ws_bytes, beam_stream stream);

/* ---- NVFP4 expert weights
 *
 * The other checkpoint format the pages name (same passages as the FP8 section, no scale
 * format given).  This path reads it as E2M1 codes (magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6)
 * with two scales: an E4M3 scale per block of 16 consecutive elements of a row, and an FP32
 * scale per row.  With amax the row's largest magnitude and m_b the block's:
 *   s = fl32(amax / 2688),  bs_b = e4m3(fl32(fl32(m_b / s) / 6)),
 *   q_j = e2m1(fl32(x_j / fl32(s * value(bs_b))))
 * rounded to nearest even and saturating; a block whose scale is 0 gets zero codes.  Weights are
 * quantised per output channel.  Token rows and the SwiGLU activation (after its BF16 rounding)
 * are quantised per row the same way.  Each GEMM runs tcgen05 block-scaled MMAs
 * (kind::mxf4nvf4, scales applied by the tensor cores, FP32 accumulation) and applies both row
 * scales in its epilogue.  Routing is unchanged.
 *
 * Storage: codes two per byte, element 2i in the low nibble of byte i.  Block scales in
 * 512-byte atoms covering 128 rows x 64 elements: the scale of row r (0..127) and block j
 * (0..3) of an atom is byte (r % 32) * 16 + (r / 32) * 4 + j, and the atoms of one 128-row
 * group follow each other in K order (atom (group g, K block b) at byte (g * K / 64 + b) * 512).
 * This is the layout the tensor cores read scales in. */

/* Converts BF16 weights to NVFP4 on `stream` (once per model).
 *   a        BF16 [groups, rows, cols] (row-major)
 *   b        NULL, or a second BF16 [groups, rows, cols]: the output then holds 2 * rows rows
 *            per group, interleaving a and b in 64-row chunks (row 128c + w is a's row 64c + w
 *            for w < 64, b's row 64c + w - 64 otherwise).  Pass w_gate and w_up [E, I, d] this
 *            way for beam_moe_forward_nvfp4.  w_down [E, d, I] is passed alone (b = NULL).
 *   codes         out: uint8 [groups * out_rows, cols / 2]
 *   block_scales  out: E4M3 atoms, groups * out_rows * cols / 16 bytes
 *   row_scales    out: FP32 [groups * out_rows]
 * Requires cols a positive multiple of 256, rows a positive multiple of 64 (with b) or 128
 * (without), every pointer 16-byte aligned, and no output overlapping an input; otherwise
 * BEAM_ERR_INVALID_ARG.  groups == 0 is a no-op. */
BEAM_API beam_status beam_moe_quantize_nvfp4(const void* a, const void* b, int64_t groups,
                                             int32_t rows, int32_t cols, void* codes,
                                             void* block_scales, float* row_scales,
                                             beam_stream stream);

/* Workspace bytes for beam_moe_forward_nvfp4 (0 for an unsupported shape; I must be a multiple
 * of 256 besides the layer's shape rules). */
BEAM_API size_t beam_moe_nvfp4_workspace_size(const beam_moe_shape* shape);

/* beam_moe_forward with NVFP4 expert weights as written by beam_moe_quantize_nvfp4:
 *   gate_up_*   w_gate and w_up interleaved: codes [E * 2I, d / 2], atoms, row scales [E * 2I]
 *   down_*      w_down: codes [E * d, I / 2], atoms, row scales [E * d]
 * Every other argument as for beam_moe_forward, with ws sized by
 * beam_moe_nvfp4_workspace_size.  All weight and scale pointers must be 16-byte aligned. */
BEAM_API beam_status beam_moe_forward_nvfp4(const beam_moe_shape* shape, const void* hidden,
                                            const float* router_w, const float* bias,
                                            const void* gate_up_codes,
                                            const void* gate_up_block_scales,
                                            const float* gate_up_scales, const void* down_codes,
                                            const void* down_block_scales,
                                            const float* down_scales, void* out,
                                            int32_t* topk_idx, float* topk_w, void* ws,
                                            size_t ws_bytes, beam_stream stream);

/* beam_moe_block with NVFP4 expert weights (as for beam_moe_forward_nvfp4); every other
 * argument as for beam_moe_block, with ws sized by beam_moe_nvfp4_workspace_size. */
BEAM_API beam_status beam_moe_block_nvfp4(const beam_moe_shape* shape, const float* x,
                                          const float* g_pre, const float* g_post, float eps,
                                          int32_t k_resid, const float* router_w,
                                          const float* bias, const void* gate_up_codes,
                                          const void* gate_up_block_scales,
                                          const float* gate_up_scales, const void* down_codes,
                                          const void* down_block_scales,
                                          const float* down_scales, float* x_out,
                                          int32_t* topk_idx, float* topk_w, void* ws,
                                          size_t ws_bytes, beam_stream stream);

/* MoE block: x' = x * sqrt((k_resid-1)/k_resid) + RMSNorm(MoE(bf16(RMSNorm(x) g_pre))) g_post
 *                 / sqrt(k_resid), RMSNorm(v) = v / sqrt(mean(v^2) + eps), all FP32.
 *   x       FP32 [T, d] residual stream in
 *   g_pre, g_post FP32 [d]
 *   eps     > 0 (rms_norm_eps, 1e-6 for Beam)
 *   k_resid >= 1: index of this contribution in the residual stream (embedding = 1)
 *   x_out   FP32 [T, d] out; may equal x (in place), must not otherwise overlap it
 * Cites: "Beam" model doc, Overview ("Sandwich norms with depth-scaled residuals");
 * archdb "Beam-1.0-501B-A23B", residual-design entry (FP32 residual accumulation). */
BEAM_API beam_status beam_moe_block(const beam_moe_shape* shape, const float* x, const float* g_pre,
                           const float* g_post, float eps, int32_t k_resid, const float* router_w,
                           const float* bias, const void* w_gate, const void* w_up,
                           const void* w_down, float* x_out, int32_t* topk_idx, float* topk_w,
                           void* ws, size_t ws_bytes, beam_stream stream);

/* Dense SwiGLU MLP of Beam's first three decoder layers: out = W_down (silu(W_gate h) * (W_up h)),
 * BF16 weights, FP32 accumulation and activation, BF16 output; no routing.
 *   hidden  BF16 [T, d];  w_gate, w_up BF16 [I, d];  w_down BF16 [d, I];  out BF16 [T, d]
 * Runs the same tensor-core GEMMs as the experts, with every token in one group.  Shapes:
 * d % 256 == 0, d <= 8192, I % 128 == 0, 0 <= T < 2^31.
 * Cites: "Beam" model doc, Overview ("The first 3 layers use a dense SwiGLU MLP") and
 * BeamConfig (intermediate_size = 20480, hidden_act = silu). */
typedef struct {
  int32_t T;  /* tokens */
  int32_t d;  /* hidden_size */
  int32_t I;  /* intermediate_size */
} beam_dense_shape;

BEAM_API size_t beam_dense_workspace_size(const beam_dense_shape* shape);
BEAM_API beam_status beam_dense_forward(const beam_dense_shape* shape, const void* hidden,
                                        const void* w_gate, const void* w_up, const void* w_down,
                                        void* out, void* ws, size_t ws_bytes, beam_stream stream);

/* Workspace bytes for beam_dense_forward_fp8 (0 for an unsupported shape). */
BEAM_API size_t beam_dense_fp8_workspace_size(const beam_dense_shape* shape);

/* beam_dense_forward with E4M3 weights: w_gate, w_up E4M3 [I, d] with row scales gate_scale,
 * up_scale FP32 [I]; w_down E4M3 [d, I] with row scales down_scale FP32 [d] (as written by
 * beam_moe_quantize_e4m3; scale arrays 16-byte aligned).  The token rows and the SwiGLU
 * activation are quantised per row as in beam_moe_forward_fp8. */
BEAM_API beam_status beam_dense_forward_fp8(const beam_dense_shape* shape, const void* hidden,
                                            const void* w_gate, const float* gate_scale,
                                            const void* w_up, const float* up_scale,
                                            const void* w_down, const float* down_scale,
                                            void* out, void* ws, size_t ws_bytes,
                                            beam_stream stream);

/* Workspace bytes for beam_dense_forward_nvfp4 (0 for an unsupported shape; I must be a
 * multiple of 256). */
BEAM_API size_t beam_dense_nvfp4_workspace_size(const beam_dense_shape* shape);

/* beam_dense_forward with NVFP4 weights written by beam_moe_quantize_nvfp4 with groups = 1:
 * gate_up_* from (w_gate, w_up) interleaved (codes [2I, d / 2], atoms, row scales [2I]),
 * down_* from w_down (codes [d, I / 2], atoms, row scales [d]); all 16-byte aligned.  The token
 * rows and the SwiGLU activation are quantised per row as in beam_moe_forward_nvfp4. */
BEAM_API beam_status beam_dense_forward_nvfp4(const beam_dense_shape* shape, const void* hidden,
                                              const void* gate_up_codes,
                                              const void* gate_up_block_scales,
                                              const float* gate_up_scales,
                                              const void* down_codes,
                                              const void* down_block_scales,
                                              const float* down_scales, void* out, void* ws,
                                              size_t ws_bytes, beam_stream stream);

/* Selection-bias update from the expert loads of the last beam_moe_forward / beam_moe_block
 * call made with `ws` (same shape):  bias[e] += gamma * sign(mean_load - load[e]), sign(0) = 0,
 * mean_load = T * top_k / E.  Under-loaded experts gain bias, over-loaded ones lose it; the
 * caller supplies gamma from its (e.g. cosine-decayed) schedule.
 * Cites: archdb "Beam-1.0-501B-A23B", load-balancing entry (auxiliary-loss-free bias with
 * cosine-decayed bias updates); news article "Reflection lança o Beam" (router follows
 * DeepSeek-V3's scheme); "Beam" model doc, Notes (no auxiliary loss). */
BEAM_API beam_status beam_moe_bias_update(const beam_moe_shape* shape, const void* ws,
                                          float* bias, float gamma, beam_stream stream);

/* ---- expert parallelism: the layer's experts over P GPUs ----
 *
 * Cites: cookbook "Use HF Transformers", section Parallelism (ep_size = 8: each GPU holds 32
 * of the 256 experts, and tokens are sent to the GPU that holds their experts); the device
 * count divides 256 (news article "Reflection lança o Beam", section "O que os benchmarks
 * mostram e como rodar o modelo").
 *
 * Rank p of P owns experts p*E/P .. (p+1)*E/P - 1 (E % P == 0, P <= 64) and routes its own
 * T_p tokens (for example with beam_moe_route).  One layer step on every rank, in this order
 * and on one stream per rank:
 *   1. beam_moe_ep_count     local slot counts [E] -> `counts` (device)
 *   2. the caller gathers every rank's counts into all_counts [P, E] (device, rank-major),
 *      for instance with an NCCL all-gather
 *   3. beam_moe_ep_dispatch  writes each token row into the receive buffer of the owner of
 *      each of its experts (a peer store when the owner is another GPU)
 *   4. the caller waits until every rank's step 3 has completed (a barrier ordered on the
 *      stream, e.g. an NCCL all-reduce of one word)
 *   5. beam_moe_ep_experts   the grouped GEMMs over the received rows -> yrecv
 *   6. the caller waits until every rank's step 5 has completed
 *   7. beam_moe_ep_combine   each token's k expert outputs read from their owners' yrecv
 *      and summed with topk_w in ascending expert order -> out [T_p, d] BF16
 * Every rank holds two caller-owned receive buffers of recv_rows_max rows, xrecv and yrecv
 * (BF16 [recv_rows_max, d]), and passes the device addresses of all ranks' buffers (their
 * peer mappings on this GPU) as host arrays of P pointers.  A rank's receive rows are its
 * experts in ascending order, each expert's rows from rank 0, 1, ... in turn, each rank's in
 * ascending token order: with tokens numbered rank-major this is the single-GPU layout of the
 * whole batch, so the result equals beam_moe_forward on the concatenated tokens with the same
 * routing bit for bit.  Rows beyond recv_rows_max are not sent and are recorded as
 * BEAM_ERR_DEVICE_ASSERT (size the buffers with beam_moe_ep_plan).  The same `shape` (T = this
 * rank's tokens) and workspace serve the four calls of a step; beam_moe_sync_status(ws) reads
 * the step's device status. */

/* Lets kernels on the calling thread's current device read and write memory of device
 * `peer_device` (cudaDeviceEnablePeerAccess), as the dispatch and combine kernels do with the
 * other ranks' receive buffers when those live on other GPUs of the node.  Already enabled, or
 * peer_device the current device: BEAM_OK.  BEAM_ERR_UNSUPPORTED when the two devices cannot
 * access each other; BEAM_ERR_INVALID_ARG for a device index out of range.  Per process and
 * device, undone by a device reset. */
BEAM_API beam_status beam_moe_enable_peer_access(int32_t peer_device);

/* Workspace bytes of one rank (0 if the arguments are unsupported). */
BEAM_API size_t beam_moe_ep_workspace_size(const beam_moe_shape* shape, int32_t P,
                                           int64_t recv_rows_max);

/* Host-only exchange sizes from the gathered counts all_counts [P, E] (HOST array): rows this
 * rank receives in total (*recv_rows), rows it sends to each rank (send_rows [P]) and rows it
 * receives from each rank (recv_from [P]).  Any output may be NULL.  Touches no GPU. */
BEAM_API beam_status beam_moe_ep_plan(int32_t P, int32_t E, const int32_t* all_counts,
                                      int32_t rank, int64_t* recv_rows, int64_t* send_rows,
                                      int64_t* recv_from);

/* Step 1: per-expert slot counts of this rank's routing topk_idx [T, top_k] -> counts [E]
 * (device INT32, always written; zeros when T = 0).  Clears the step's status word. */
BEAM_API beam_status beam_moe_ep_count(const beam_moe_shape* shape, int32_t P,
                                       const int32_t* topk_idx, int32_t* counts,
                                       int64_t recv_rows_max, void* ws, size_t ws_bytes,
                                       beam_stream stream);

/* Step 3: hidden [T, d] BF16 rows to the owners' receive buffers xrecv_peers[q] (host array
 * of P device pointers, this rank's own buffer at index `rank`). */
BEAM_API beam_status beam_moe_ep_dispatch(const beam_moe_shape* shape, int32_t P, int32_t rank,
                                          const void* hidden, const int32_t* topk_idx,
                                          const int32_t* all_counts, void* const* xrecv_peers,
                                          int64_t recv_rows_max, void* ws, size_t ws_bytes,
                                          beam_stream stream);

/* Step 5: the SwiGLU experts of this rank over its received rows.  w_gate, w_up [E/P, I, d],
 * w_down [E/P, d, I] BF16 are this rank's experts; xrecv and yrecv are this rank's receive
 * buffers; T_total is the tokens of all ranks together (it selects the same tile forms as a
 * single-GPU call of that size). */
BEAM_API beam_status beam_moe_ep_experts(const beam_moe_shape* shape, int32_t P, int32_t rank,
                                         int64_t T_total, const int32_t* all_counts,
                                         const void* w_gate, const void* w_up, const void* w_down,
                                         const void* xrecv, void* yrecv, int64_t recv_rows_max,
                                         void* ws, size_t ws_bytes, beam_stream stream);

/* Step 7: out [T, d] BF16 = sum_j topk_w[t, j] * y(slot j), the expert outputs read from
 * yrecv_peers[owner] (host array of P device pointers). */
BEAM_API beam_status beam_moe_ep_combine(const beam_moe_shape* shape, int32_t P,
                                         const float* topk_w, const void* const* yrecv_peers,
                                         int64_t recv_rows_max, void* out, void* ws,
                                         size_t ws_bytes, beam_stream stream);

/* Synchronises `stream`, reads and clears the device status word kept in `ws`, and
 * returns BEAM_OK, BEAM_ERR_TIMEOUT or BEAM_ERR_DEVICE_ASSERT (or BEAM_ERR_CUDA if the
 * stream itself reports an error).  `ws` must have been used with a call of this shape
 * family (the status word sits at offset 0 of every workspace). */
BEAM_API beam_status beam_moe_sync_status(void* ws, beam_stream stream);

/* Human-readable name of a status code (static storage). */
BEAM_API const char* beam_status_string(beam_status status);

/* Text of the last CUDA error seen by this library on the calling thread, or "". */
BEAM_API const char* beam_moe_last_cuda_error(void);

/* Per-expert token counts of the last forward/block call that used `ws` (synchronises
 * `stream` and copies E int32 values to the HOST buffer counts_host). */
BEAM_API beam_status beam_moe_expert_counts(const beam_moe_shape* shape, const void* ws,
                                   int32_t* counts_host, beam_stream stream);

/* Row of every (token, slot) pair in the expert-contiguous buffers of the last forward/block
 * call that used `ws` (synchronises `stream` and copies T * top_k int32 values, slot order as
 * topk_idx, to the HOST buffer rows_host).  Expert e owns rows off[e] .. off[e+1]-1, where
 * off is the exclusive prefix sum of the per-expert counts over ascending e, and inside them
 * its tokens sit in ascending token order: the layout is a function of the routing alone. */
BEAM_API beam_status beam_moe_slot_rows(const beam_moe_shape* shape, const void* ws,
                                        int32_t* rows_host, beam_stream stream);

/* ---- diagnostics (process-wide settings) ---- */

/* Limit, in nanoseconds, of every device-side wait in the expert GEMM kernels; after it
 * the kernel records BEAM_ERR_TIMEOUT, drains its own copies, frees its tensor memory and
 * returns.  Default 4e9 (4 s).  Applies to launches made after the call. */
BEAM_API void beam_moe_set_wait_limit_ns(uint64_t ns);
BEAM_API uint64_t beam_moe_get_wait_limit_ns(void);

/* Expert GEMMs on SM pairs (tcgen05 cta_group::2, 256-row tiles; one cluster of two CTAs
 * per tile) for beam_moe_forward / beam_moe_block calls averaging at least 256 rows per
 * expert.  Off by default: on a power-capped B200 those calls are bound by tensor throughput,
 * and 256-row tiles add padded rows, so the single-SM 128-row kernel measured faster.  The
 * setting applies to calls made after it. */
BEAM_API void beam_moe_set_sm_pairs(int enable);
BEAM_API int beam_moe_get_sm_pairs(void);

/* Total kernels this library has launched in this process. */
BEAM_API uint64_t beam_moe_launch_count(void);

/* Kernel timing: when enabled, every launch is bracketed by CUDA events on its stream.
 * beam_moe_profile_read() synchronises those events and returns, for kernel `id`
 * (0 <= id < beam_moe_kernel_count()), its launches and total milliseconds since the last
 * reset; beam_moe_profile_reset() clears the counters. */
BEAM_API void beam_moe_profile_enable(int on);
BEAM_API void beam_moe_profile_reset(void);
BEAM_API int beam_moe_kernel_count(void);
BEAM_API const char* beam_moe_kernel_name(int id);
BEAM_API beam_status beam_moe_profile_read(int id, int64_t* launches, double* total_ms);

/* ABI version of this header (bumped on any incompatible change). */
BEAM_API int beam_moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BEAM_MOE_H_ */
