/*
 * moe.h - C ABI of the B200 (sm_100a) DeepSeek-V3-style Mixture-of-Experts
 * layer forward pass.
 *
 * The layer (pages "DeepSeek-V3.2-Exp - Expert scores" and "DeepSeek-V3.2-Exp
 * - Weighted expert sum"; the MoE class on the hackaday page "time to jump
 * right in and swim with the big fish"):
 *
 *   z      = x . W_r^T                        fp32 router logits   (moe_gate)
 *   s      = sigmoid(z) | softmax(z)          unbiased scores
 *   b      = s + bias                         selection-only bias
 *   groups = top-topk_groups of n_groups contiguous expert blocks, scored by
 *            the sum of their top-2 b (with a bias) or their max b (without)
 *   idx    = top-k of b outside the dropped groups, descending b
 *   w      = s[idx] (/ sum, for sigmoid) * route_scale
 *   counts = bincount(idx), offsets = exclusive scan    (moe_dispatch)
 *   E_e(x) = w2_e (silu(w1_e x) * (w3_e x))   SwiGLU     (moe_experts_grouped)
 *   y[t]   = sum_j w[t,j] E_{idx[t,j]}(x[t]) + S(x[t])  (moe_combine)
 *            accumulated in fp32, cast back to the activation dtype once.
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major
 *     and contiguous, 16-byte aligned. "act" means the activation dtype of the
 *     config (fp32 or bf16): x, the router weight, all expert weights, the
 *     intermediates and y use it. The selection bias and the routing weights
 *     are always fp32; expert indices and all counts/offsets are int32.
 *   - Weights are stored [out, in]: W_r [E, D], w1/w3 [E, I, D], w2 [E, D, I],
 *     shared ws1/ws3 [I_s, D], ws2 [D, I_s] (I_s = shared_inter).
 *   - The library allocates no device memory. Scratch comes from the caller's
 *     workspace `ws` of at least moe_workspace_size() bytes, which must be
 *     zeroed once by moe_workspace_init() after allocation. A workspace may be
 *     reused by any sequence of calls on one stream; calls that share a
 *     workspace must not run concurrently.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream) of the device
 *     that holds the call's workspace (moe_gate_noalloc: x). Every call is
 *     asynchronous on it and never synchronises the host, except
 *     moe_check_error. moe_gate, moe_dispatch, moe_experts_grouped,
 *     moe_combine and moe_forward neither allocate, synchronise nor query
 *     the stream, so they can be captured into a CUDA graph and replayed
 *     with new data written into the same buffers.
 *   - Argument checks are synchronous: a bad config, size or pointer returns
 *     MOE_ERR_INVALID_ARG / MOE_ERR_UNSUPPORTED / MOE_ERR_WORKSPACE before
 *     anything is launched. A failed launch returns MOE_ERR_CUDA.
 *   - Conditions only the device can see (an expert index outside [0, E)
 *     handed to moe_dispatch, a pipeline wait that exceeded its time limit)
 *     set a sticky error word in the workspace; the offending element is
 *     skipped, nothing is written out of bounds. moe_check_error() reads and
 *     clears it.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, bad size or config */
  MOE_ERR_UNSUPPORTED = -2,  /* a valid config this library does not run   */
  MOE_ERR_WORKSPACE = -3,    /* workspace missing or smaller than required  */
  MOE_ERR_CUDA = -4,         /* a CUDA runtime call or launch failed         */
  MOE_ERR_DEVICE_CHECK = -5, /* a device-side check failed (bad index)       */
  MOE_ERR_TIMEOUT = -6       /* a device pipeline wait hit its time limit    */
} moe_status;

typedef enum { MOE_DT_F32 = 0, MOE_DT_BF16 = 1 } moe_dtype;
typedef enum { MOE_SCORE_SIGMOID = 0, MOE_SCORE_SOFTMAX = 1 } moe_score;

/* Layer shape, mirroring the Gate/MoE constructor arguments on the pages:
 * dim, n_routed_experts, n_expert_groups, n_limited_groups,
 * n_activated_experts, moe_inter_dim, n_shared_experts * moe_inter_dim,
 * score_func, route_scale, and whether the selection bias exists.
 * Limits: 1 <= n_routed <= 1024; n_groups divides n_routed, n_groups <= 64 and
 * the group width n_routed/n_groups is a power of two <= 32 or a multiple of
 * 32; 1 <= topk_groups <= n_groups; 1 <= topk <= min(32, topk_groups *
 * n_routed / n_groups); group width >= 2 when has_bias and n_groups > 1;
 * dim, moe_inter, shared_inter multiples of 8 (bf16) / 4 (fp32);
 * shared_inter may be 0 (no shared expert). */
typedef struct {
  int32_t dim;
  int32_t n_routed;
  int32_t n_groups;
  int32_t topk_groups;
  int32_t topk;
  int32_t moe_inter;
  int32_t shared_inter;
  int32_t score;       /* moe_score */
  float route_scale;
  int32_t has_bias;    /* 0 or 1 */
  int32_t dtype;       /* moe_dtype */
} moe_config;

/* Bytes of workspace every call below needs for T tokens (T >= 1). */
MOE_API moe_status moe_workspace_size(const moe_config* cfg, int64_t T, size_t* bytes);

/* Zero the workspace header (the sticky error word). Call once after
 * allocating the workspace, before any other call that uses it. */
MOE_API moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Router (page "Expert scores", Gate.forward): fp32 logits from x [T, D] (act)
 * and W_r [E, D] (act), scores, bias (fp32 [E], ignored unless has_bias;
 * may be NULL only then), group limit, top-k.
 * Out: weights [T, k] fp32 and idx [T, k] int32, each token's picks ordered
 * by descending biased score, ties to the lower expert index. */
MOE_API moe_status moe_gate(const moe_config* cfg, int64_t T, const void* x, const void* w_router,
                    const float* bias, float* weights, int32_t* idx,
                    void* ws, size_t ws_bytes, void* stream);

/* Dispatch (page "Weighted expert sum": bincount, then each expert's rows in
 * row-major order of idx): counts [E], offsets [E+1] (exclusive scan,
 * offsets[E] = number of valid pairs), src [T*k] (token of each permuted
 * row), pos [T*k] (permuted row of pair (t, j), -1 for an invalid index), and
 * x_perm [T*k, D] (act), x's rows in expert-contiguous order, ascending token
 * within an expert. x_perm may be NULL (and x with it): then only counts,
 * offsets, src and pos are written, for moe_experts_grouped_gather, which
 * reads x's rows through src. An index outside [0, E) sets
 * MOE_ERR_DEVICE_CHECK in the error word and its pair is dropped. */
MOE_API moe_status moe_dispatch(const moe_config* cfg, int64_t T, const int32_t* idx, const void* x,
                        int32_t* counts, int32_t* offsets, int32_t* src, int32_t* pos,
                        void* x_perm, void* ws, size_t ws_bytes, void* stream);

/* Experts (each Expert(dim, moe_inter_dim) and the shared MLP of width
 * n_shared_experts * moe_inter_dim; SwiGLU body): for every expert e, rows
 * [offsets[e], offsets[e+1]) of x_perm [T*k, D] go through expert e into
 * y_perm [T*k, D] (act); x [T, D] goes through the shared MLP into s [T, D]
 * (act). h = silu(w1 x) * (w3 x) is formed in fp32 and rounded to act before
 * w2. x, ws1, ws3, ws2 and s may be NULL when shared_inter == 0. Rows of
 * y_perm at or past offsets[E] are not written. */
MOE_API moe_status moe_experts_grouped(const moe_config* cfg, int64_t T, const void* x_perm,
                               const int32_t* offsets, const void* w1, const void* w3,
                               const void* w2, const void* x, const void* ws1,
                               const void* ws3, const void* ws2, void* y_perm, void* s,
                               void* ws, size_t ws_bytes, void* stream);

/* moe_experts_grouped without the expert-contiguous copy of x: row p of the
 * expert order is token src[p] of x [T, D] (src and offsets as moe_dispatch
 * writes them), read straight from x by the expert GEMM (TMA gather of four
 * token rows per copy on the tensor-core path). Same outputs as
 * moe_experts_grouped on x_perm; x is required. This is how moe_forward runs
 * the experts. Returns MOE_ERR_UNSUPPORTED for a bf16 layer while the
 * CTA-pair expert kernel is selected (it reads only x_perm). */
MOE_API moe_status moe_experts_grouped_gather(const moe_config* cfg, int64_t T, const void* x,
                                              const int32_t* src, const int32_t* offsets,
                                              const void* w1, const void* w3, const void* w2,
                                              const void* ws1, const void* ws3, const void* ws2,
                                              void* y_perm, void* s, void* ws, size_t ws_bytes,
                                              void* stream);

/* Combine (page "Weighted expert sum": y_routed = sum_i G_i E_i, accumulated
 * in float32 and cast back at the end; then the shared expert added):
 * y[t] = act( sum_j weights[t,j] * y_perm[pos[t,j]] + s[t] ), fp32 sum over
 * j = 0..k-1 then s. Pairs with pos < 0 are skipped; s may be NULL. */
MOE_API moe_status moe_combine(const moe_config* cfg, int64_t T, const void* y_perm,
                       const int32_t* pos, const float* weights, const void* s, void* y,
                       void* ws, size_t ws_bytes, void* stream);

/* The whole layer (MoE.forward): gate, dispatch, experts and combine chained
 * on `stream` with no host synchronisation. y [T, D] (act). weights_out
 * [T, k] and idx_out [T, k] may be NULL; when given they receive the routing.
 * For batches of at most 16 routed rows per expert on average (T * k <=
 * 16 * n_routed: decode) and for fp32 layers, the experts read the routed
 * token rows straight from x (as moe_experts_grouped_gather does) and no
 * permuted copy of x is made. Larger bf16 batches, and the CTA-pair expert
 * kernel, read an expert-contiguous copy that dispatch writes into the
 * workspace's y_perm region (free until the down-projection writes it): on
 * B200 the copy is the faster of the two for 128-row tiles. On the default
 * one-CTA tensor-core kernel the up-projection is launched as a programmatic
 * dependent of the dispatch's last kernel (cudaLaunchKernelEx with
 * programmatic stream serialization): its CTAs start, and take any shared-
 * expert tiles, while that kernel finishes, and wait for it (griddepcontrol)
 * before their first routed tile. The down-projection is in turn a
 * programmatic dependent of the up-projection: its CTAs start as the
 * up-projection's finish, prefetch their first weight tiles into L2 and wait
 * for h. Every kernel of the chain waits for its predecessor before it reads
 * what that grid wrote, so results do not depend on the overlap. */
MOE_API moe_status moe_forward(const moe_config* cfg, int64_t T, const void* x, const void* w_router,
                       const float* bias, const void* w1, const void* w3, const void* w2,
                       const void* ws1, const void* ws3, const void* ws2, void* y,
                       float* weights_out, int32_t* idx_out, void* ws, size_t ws_bytes,
                       void* stream);

/* Expert parallelism (the MoE class on the hackaday page and DeepseekV3MoE on
 * the thataiguy page: rank r of world_size holds the contiguous block of
 * experts [r E / world_size, (r + 1) E / world_size); every rank routes all
 * tokens and runs only its own experts, and one all_reduce sums the ranks'
 * outputs. The V3.2 listing on page "Weighted expert sum" adds the shared MLP
 * into y before that all_reduce, so each rank also holds a slice of the
 * shared MLP's inner width; the slices' outputs add up to the whole MLP.)
 *
 * One rank's share of the layer: the gate over all E experts (W_r and bias
 * whole), dispatch, the grouped experts for this rank's block [expert_begin,
 * expert_end) only, and its shared slice, combined into y_partial [T, D]
 * fp32 -- sum_j w[t,j] E_{idx[t,j]}(x[t]) over the pairs routed into the
 * block, plus the slice's output -- not rounded. w1, w3 [n_local, I, D] and
 * w2 [n_local, D, I] hold the block's experts (n_local = expert_end -
 * expert_begin, first expert first); ws1, ws3 [shared_local, D] and ws2
 * [D, shared_local] the rank's slice of the shared MLP (contiguous copies of
 * rows of ws1 / ws3 and columns of ws2; NULL when shared_local == 0). The
 * caller sums y_partial over the ranks in fp32 (an all_reduce) and casts the
 * sum once with moe_cast_output. Workspace as for moe_forward. Requires
 * 0 <= expert_begin < expert_end <= n_routed and 0 <= shared_local <=
 * shared_inter (a multiple of 8 for bf16, 4 for fp32); MOE_ERR_UNSUPPORTED
 * for a bf16 layer while the CTA-pair expert kernel is selected. */
MOE_API moe_status moe_forward_ep(const moe_config* cfg, int64_t T, int32_t expert_begin,
                                  int32_t expert_end, int32_t shared_local, const void* x,
                                  const void* w_router, const float* bias, const void* w1,
                                  const void* w3, const void* w2, const void* ws1, const void* ws3,
                                  const void* ws2, float* y_partial, float* weights_out,
                                  int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/* y [T, D] (act) = y_sum [T, D] (fp32) rounded once: the last step of an
 * expert-parallel layer, after the ranks' y_partial have been summed. */
MOE_API moe_status moe_cast_output(const moe_config* cfg, int64_t T, const float* y_sum, void* y,
                                   void* stream);

/* FP8 expert weights. The page "DeepSeek-V3.2-Exp - Expert scores" says the
 * block's other linears are FP8 and gives no layout; this library's layout:
 * e4m3 values (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; finite
 * values up to 448), one fp32 scale per 128 x 128 block of each [out, in]
 * matrix, a power of two: the smallest 2^s with the block's largest magnitude
 * <= 448 * 2^s, and s >= -127 (so that every scale is one UE8M0 byte, the
 * form the tensor core's block scaling reads; a block below 448 * 2^-127
 * keeps 2^-127). A weight is q * scale. moe_quantize_fp8 produces the layout
 * from bf16 or fp32 weights. Scales are row-major over the blocks:
 * w1_scale / w3_scale [E, I/128, D/128], w2_scale [E, D/128, I/128],
 * ws1_scale / ws3_scale [I_s/128, D/128], ws2_scale [D/128, I_s/128]. */
typedef struct {
  const void* w1;           /* e4m3 [E, I, D] */
  const void* w3;           /* e4m3 [E, I, D] */
  const void* w2;           /* e4m3 [E, D, I] */
  const float* w1_scale;
  const float* w3_scale;
  const float* w2_scale;
  const void* ws1;          /* shared MLP, e4m3 [I_s, D]; NULL when shared_inter == 0 */
  const void* ws3;          /* e4m3 [I_s, D] */
  const void* ws2;          /* e4m3 [D, I_s] */
  const float* ws1_scale;
  const float* ws3_scale;
  const float* ws2_scale;
} moe_fp8_weights;

/* Quantize a [rows, cols] matrix a (the config's activation dtype) to e4m3
 * with one power-of-two scale per block_rows x 128 block (block_rows = 128
 * for weights, 1 for rows of activations): scales [ceil(rows/block_rows),
 * cols/128] fp32, q [rows, cols] e4m3 bytes. Each value is rounded to the
 * nearest e4m3 value, ties to even. cols must be a multiple of 128. Stacked
 * expert weights [E, N, K] quantize as [E*N, K] when N is a multiple of 128. */
MOE_API moe_status moe_quantize_fp8(const moe_config* cfg, const void* a, int64_t rows,
                                    int64_t cols, int32_t block_rows, void* q, float* scales,
                                    void* stream);

/* Bytes of workspace moe_forward_fp8 needs for T tokens; MOE_ERR_UNSUPPORTED
 * unless the layer is bf16 with dim, moe_inter and shared_inter multiples of
 * 128 and at most 8192. */
MOE_API moe_status moe_workspace_size_fp8(const moe_config* cfg, int64_t T, size_t* bytes);

/* The whole layer with FP8 expert weights: the router as in moe_forward (bf16
 * W_r applied in fp32), then x quantized per 1 x 128 block of each row to
 * e4m3 (as the weights, one power-of-two scale per block), the routed and
 * shared SwiGLU experts on the e4m3 tensor cores (kind::mxf8f6f4 block
 * scaling: each product scaled by the weight's and the row's block scales
 * inside the tensor core, one fp32 accumulation over K), h = silu(w1 x) *
 * (w3 x) quantized the same way
 * before w2, each expert's output rounded to bf16, and the combine as in
 * moe_forward. Workspace of moe_workspace_size_fp8() bytes, initialised by
 * moe_workspace_init(). bf16 layers only.
 * Two forms of the expert GEMMs compute the same sums (see
 * moe_select_fp8_kernel): for batches of at most 16 rows per expert on
 * average, the weights on the MMA's M side and up to 32 tokens of an expert on
 * its N side (each weight tile streamed once per 32 tokens); above that, 128
 * token rows on M and 256 weight rows on N, the routed rows' codes written in
 * expert order by the row quantization. */
MOE_API moe_status moe_forward_fp8(const moe_config* cfg, int64_t T, const void* x,
                                   const void* w_router, const float* bias,
                                   const moe_fp8_weights* w, void* y, float* weights_out,
                                   int32_t* idx_out, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read and clear the workspace's error word. Returns
 * MOE_OK, MOE_ERR_DEVICE_CHECK or MOE_ERR_TIMEOUT (or MOE_ERR_CUDA). */
MOE_API moe_status moe_check_error(void* ws, void* stream);

/* Static text for a status code. */
MOE_API const char* moe_status_string(moe_status st);

/* Number of kernels moe_forward launches for T tokens of this config with the
 * expert kernel currently selected (moe_select_expert_kernel), for
 * accounting: router 2, dispatch 3 (1 for a batch of at most 4096 (token,
 * slot) pairs over at most 512 experts that reads the token rows from x),
 * the two expert GEMMs (plus one kernel that writes their per-expert A maps
 * on the default one-CTA tensor-core kernel), combine 1: 7 for the
 * DeepSeek-V3 decode batch, 9 for its prefill batch. */
MOE_API int32_t moe_forward_launch_count(const moe_config* cfg, int64_t T);

/* moe_gate without a workspace. The pages have no counterpart of this call:
 * it exists for callers that cannot allocate device memory or hand out a
 * workspace -- for instance a plugin inside a host framework that owns every
 * byte of device memory through its own pool, or a latency-critical serving
 * loop where cudaMalloc is off limits because it can synchronise the device.
 * Same arguments and results as moe_gate, minus ws / ws_bytes: the router's
 * split-k partial sums go to a 4 MiB scratch array built into the library
 * (1,048,576 floats; every GPU that loads the library holds it until the
 * process exits). Limit: T * n_routed <= 1,048,576 (T <= 4096 at 256
 * experts); larger shapes return MOE_ERR_UNSUPPORTED and launch nothing. The
 * call allocates no device memory itself. The first call on each device looks
 * up the scratch's device address (cudaGetSymbolAddress) and caches it; under
 * CUDA's lazy module loading (the default) that first call may also be what
 * loads the library's device code onto the device, which reserves the array
 * and can synchronise. A latency-critical loop should therefore make one call
 * (or one moe_gate_noalloc_check_error) on each device before it starts, and
 * before any stream capture. All calls share the one array and it keeps the
 * last call's partial sums (each call overwrites every element it reads);
 * calls whose work overlaps on the GPU, on different streams or host threads,
 * race on it and must be serialised by the caller.
 * Failures the device sees: a router pipeline wait that runs out sets the
 * timeout bit of an error word built into the library beside the array (one
 * per device, shared by every call on that device). While that bit is set,
 * calls write no weights and no indices (the partial sums may be stale);
 * moe_gate_noalloc_check_error reads and clears it. */
MOE_API moe_status moe_gate_noalloc(const moe_config* cfg, int64_t T, const void* x,
                                    const void* w_router, const float* bias, float* weights,
                                    int32_t* idx, void* stream);

/* Read and clear the built-in error word of moe_gate_noalloc on the device
 * that holds `x` (any device pointer of that device): synchronises `stream`,
 * returns MOE_ERR_TIMEOUT if a call's router pipeline wait ran out since the
 * last read, else MOE_OK (or MOE_ERR_CUDA / MOE_ERR_INVALID_ARG). Allocates
 * no device memory. The pages have no counterpart. */
MOE_API moe_status moe_gate_noalloc_check_error(const void* x, void* stream);

/* Per-kernel timing of moe_forward, for measurement (off by default).
 * moe_stage_timing_begin(max_calls) creates max_calls * 9 CUDA events (no
 * device memory) and arms the next max_calls moe_forward calls to record one
 * event on their stream before their first kernel and one after each of their
 * moe_forward_launch_count() kernels. moe_stage_timing_end(ms, n) disarms,
 * waits for the recorded events and writes to ms[i] the total milliseconds
 * kernel i (launch order: router logits, router select, dispatch rank,
 * dispatch scan, dispatch positions -- with the per-expert map kernel before
 * it, when there is one --, experts up, experts down, combine) took over the
 * recorded calls, for i < n <= 8; it returns the number of calls recorded, or
 * a negative moe_status. A recorded call launches its up-projection as an
 * ordinary launch (not as a programmatic dependent of the dispatch), so that
 * each interval holds one kernel. Single-threaded use only. */
MOE_API moe_status moe_stage_timing_begin(int32_t max_calls);
MOE_API int32_t moe_stage_timing_end(float* ms, int32_t n);

/* moe_stage_timing_begin, recording only one moe_forward call in `every`
 * (calls 0, every, 2*every, ... after arming), so that a timed loop carries
 * the events of a few calls instead of all (each event recorded between two
 * kernels costs the stream a little time). every >= 1. */
MOE_API moe_status moe_stage_timing_begin_every(int32_t max_calls, int32_t every);

/* Which kernels run the GEMMs of a bf16 layer, process-wide (for checks and
 * measurement; nothing switches on its own):
 *   AUTO (default)  tensor cores: router logits, and the grouped expert GEMM
 *                   with one CTA per 128-row tile;
 *   TCGEN05         tensor cores, expert GEMM always with one CTA per tile;
 *   TCGEN05_PAIR    tensor cores, expert GEMM always on CTA pairs;
 *   SIMT            the CUDA-core kernels that fp32 layers always use, for
 *                   both the router logits and the expert GEMMs: a slow,
 *                   independent cross-check of the tensor-core kernels.
 * Returns MOE_ERR_INVALID_ARG for other values. */
enum {
  MOE_EXPERT_KERNEL_AUTO = 0,
  MOE_EXPERT_KERNEL_SIMT = 1,
  MOE_EXPERT_KERNEL_TCGEN05 = 2,
  MOE_EXPERT_KERNEL_TCGEN05_PAIR = 3
};
MOE_API moe_status moe_select_expert_kernel(int32_t which);

/* Which form runs the expert GEMMs of moe_forward_fp8, process-wide (for
 * checks and measurement):
 *   AUTO (default)  by the batch: tokens on N for at most 16 (token, slot)
 *                   rows per expert on average, tokens on M above;
 *   TOKENS_ON_N     weights on the MMA's M side, up to 32 tokens on N;
 *   TOKENS_ON_M     128 token rows on M, 256 weight rows on N.
 * Both give the same results up to the order of the fp32 sums. Returns
 * MOE_ERR_INVALID_ARG for other values. */
enum {
  MOE_FP8_KERNEL_AUTO = 0,
  MOE_FP8_KERNEL_TOKENS_ON_N = 1,
  MOE_FP8_KERNEL_TOKENS_ON_M = 2
};
MOE_API moe_status moe_select_fp8_kernel(int32_t which);

/* The form moe_forward_fp8 runs for T tokens of this config under the current
 * selection (AUTO resolved by the batch): MOE_FP8_KERNEL_TOKENS_ON_N or
 * MOE_FP8_KERNEL_TOKENS_ON_M; -1 if the config or T is invalid. Host only. */
MOE_API int32_t moe_fp8_kernel_for(const moe_config* cfg, int64_t T);

/* Test hook for the failure path of the tensor-core pipelines, process-wide,
 * off by default; the pages have no counterpart. While enabled, one kernel
 * has its first CTA wait, before it issues anything, on a barrier phase that
 * nothing completes:
 *   1  the up-projection of every bf16 layer on the one-CTA tensor-core
 *      kernel, and of every FP8 layer in either form (the rows of that
 *      CTA's tiles are not written);
 *   2  the tensor-core router logits of every bf16 layer (that CTA's partial
 *      sums are not written).
 * The wait runs out after its 1 s limit; the launch then takes the abort
 * path every timed-out wait takes (drain the copies in flight, free TMEM,
 * return) and sets the timeout bit of the call's error word, so the next
 * moe_check_error() (moe_gate_noalloc_check_error() for moe_gate_noalloc)
 * returns MOE_ERR_TIMEOUT. 0 disables it; other values return
 * MOE_ERR_INVALID_ARG. */
MOE_API moe_status moe_debug_stall_pipeline(int32_t enable);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
