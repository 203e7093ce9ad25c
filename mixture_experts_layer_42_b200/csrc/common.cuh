// Internal helpers shared by the kernels of the MoE layer library.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/moe.h"

namespace moe {

// Bits of the sticky device error word (first 4 bytes of the workspace).
enum : uint32_t {
  ERRBIT_BAD_INDEX = 1u,   // an expert index outside [0, E)
  ERRBIT_TIMEOUT = 2u,     // a pipeline wait hit its time limit
};

// Alignment of every workspace region (bytes).
constexpr size_t kWsAlign = 256;

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

template <typename T>
__host__ __device__ inline T ceil_div(T a, T b) { return (a + b - 1) / b; }

// Tokens per dispatch chunk (the unit of the stable counting sort).
constexpr int kDispatchChunkTokens = 64;
// Batches up to this many (token, slot) pairs over at most this many experts,
// without a permuted copy of x, are dispatched by one kernel (one CTA).
constexpr int kDispatchSmallPairs = 4096;
constexpr int kDispatchSmallExperts = 512;

// Router GEMM tile: 128 tokens x 64 experts, 32-deep k slices.
constexpr int kRouterBM = 128;
constexpr int kRouterBN = 64;
constexpr int kRouterBK = 32;

struct WsLayout {
  size_t header;        // error word
  size_t router_part;   // [splits, T, E] fp32
  size_t chunk_hist;    // [n_chunks, E] int32
  size_t pos_local;     // [T * k] int32, ranks within a dispatch chunk
  size_t weights;       // [T, k] fp32
  size_t idx;           // [T, k] int32
  size_t counts;        // [E] int32
  size_t offsets;       // [E + 1] int32
  size_t src;           // [T * k] int32
  size_t pos;           // [T * k] int32
  size_t y_perm;        // [T * k, D] act; moe_forward on the CTA-pair kernel
                        // first holds the expert-contiguous copy of x here
  size_t s;             // [T, D] act
  size_t h;             // [T * k, I] act
  size_t hs;            // [T, I_s] act
  size_t row_maps;      // [2, E] TMA maps (128 B): A rows of each expert (up, down),
                        // then the tile counters of the up and down launches, 64 B apart
  size_t total;
  int router_splits;
  int n_chunks;
};

inline int act_bytes(const moe_config& c) { return c.dtype == MOE_DT_BF16 ? 2 : 4; }

// Scale block edge of the FP8 expert weights and activations.
constexpr int kFp8Block = 128;

// Extra workspace regions of moe_forward_fp8, after the common layout.
// (Activation scales are stored with their row stride, K/128, rounded up to
// a multiple of 4 floats: see fp8_scale_stride.)
struct Fp8Layout {
  size_t xq, xs;        // quantized x [T, D] e4m3, its scales [T, D/128] fp32
  size_t xs_perm;       // x's scales in expert order [T*k, D/128]
  size_t xq_perm;       // x's codes in expert order [T*k, D] (token-on-M form)
  size_t hq, hs;        // quantized h [T*k, I], scales [T*k, I/128]
  size_t hsq, hss;      // the shared MLP's h [T, I_s], scales [T, I_s/128]
  size_t total;
};
inline int fp8_stride_host(int K) { return ((K / kFp8Block) + 3) & ~3; }

// CTAs the router GEMM aims for (two per SM of a 148-SM B200).
constexpr int kRouterTargetCtas = 296;

// Number of k splits of the router GEMM for T tokens: enough CTAs to reach
// the target, at most 32 splits, each split at least 4 k slices deep. Depends
// only on the shape, so the workspace size is a pure function of it.
inline int router_splits(const moe_config& c, int64_t T) {
  int64_t tiles = ceil_div<int64_t>(T, kRouterBM) * ceil_div<int64_t>(c.n_routed, kRouterBN);
  int64_t want = (kRouterTargetCtas + tiles - 1) / tiles;
  int64_t kslices = ceil_div<int64_t>(c.dim, kRouterBK);
  int64_t maxs = kslices / 4 > 0 ? kslices / 4 : 1;
  if (want > 32) want = 32;
  if (want > maxs) want = maxs;
  if (want < 1) want = 1;
  return (int)want;
}

inline WsLayout ws_layout(const moe_config& c, int64_t T);

inline Fp8Layout fp8_layout(const moe_config& c, int64_t T, size_t base) {
  Fp8Layout L{};
  const int64_t k = c.topk, D = c.dim, I = c.moe_inter, Is = c.shared_inter;
  size_t off = base;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + (bytes ? bytes : 1), kWsAlign);
    return o;
  };
  L.xq = take((size_t)T * D);
  L.xs = take((size_t)T * fp8_stride_host((int)D) * 4);
  L.xs_perm = take((size_t)T * k * fp8_stride_host((int)D) * 4);
  L.xq_perm = take((size_t)T * k * D);
  L.hq = take((size_t)T * k * I);
  L.hs = take((size_t)T * k * fp8_stride_host((int)I) * 4);
  L.hsq = take((size_t)T * (Is > 0 ? Is : 1));
  L.hss = take((size_t)T * (Is > 0 ? fp8_stride_host((int)Is) : 1) * 4);
  L.total = off;
  return L;
}

inline WsLayout ws_layout(const moe_config& c, int64_t T) {
  WsLayout L{};
  const int64_t E = c.n_routed, k = c.topk, D = c.dim, I = c.moe_inter, Is = c.shared_inter;
  const int64_t ab = act_bytes(c);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + (bytes ? bytes : 1), kWsAlign);
    return o;
  };
  L.router_splits = router_splits(c, T);
  L.n_chunks = (int)ceil_div<int64_t>(T, kDispatchChunkTokens);
  L.header = take(kWsAlign);
  L.router_part = take((size_t)L.router_splits * T * E * 4);
  L.chunk_hist = take((size_t)L.n_chunks * E * 4);
  L.pos_local = take((size_t)T * k * 4);
  L.weights = take((size_t)T * k * 4);
  L.idx = take((size_t)T * k * 4);
  L.counts = take((size_t)E * 4);
  L.offsets = take((size_t)(E + 1) * 4);
  L.src = take((size_t)T * k * 4);
  L.pos = take((size_t)T * k * 4);
  L.y_perm = take((size_t)T * k * D * ab);
  L.s = take((size_t)T * D * ab);
  L.h = take((size_t)T * k * I * ab);
  L.hs = take((size_t)T * (Is > 0 ? Is : 1) * ab);
  L.row_maps = take((size_t)2 * E * 128 + 128);
  L.total = off;
  return L;
}

// ---------------------------------------------------------------- device

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bit) {
  if (err) atomicOr(err, bit);
}

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// 16-byte vector of activations: 8 bf16 or 4 fp32.
template <typename T> struct Vec16;
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  uint4 raw;
  __device__ __forceinline__ void to_float(float* f) const {
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(p[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
  __device__ __forceinline__ void from_float(const float* f) {
    __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&raw);
#pragma unroll
    for (int i = 0; i < 4; ++i) p[i] = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
  }
};
template <> struct Vec16<float> {
  static constexpr int N = 4;
  uint4 raw;
  __device__ __forceinline__ void to_float(float* f) const {
    f[0] = __uint_as_float(raw.x);
    f[1] = __uint_as_float(raw.y);
    f[2] = __uint_as_float(raw.z);
    f[3] = __uint_as_float(raw.w);
  }
  __device__ __forceinline__ void from_float(const float* f) {
    raw = make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                     __float_as_uint(f[3]));
  }
};

// ---------------------------------------------------------------- launchers

// Operands of one grouped expert launch ([0] routed experts, [1] shared MLP).
struct GroupedArgs {
  const void* a[2];     // A rows: [0] x_perm / h (or x, see a_rows), [1] x / hs
  // UP only: when set, row p of the routed A is row a_rows[p] of a[0] (x
  // gathered by the dispatch's src), instead of row p of an expert-contiguous copy
  const int32_t* a_rows;
  const void* b1[2];    // w1 / w2 stacked [E, N, K]; shared ws1 / ws2 [N_s, K_s]
  const void* b3[2];    // w3 / ws3 (UP only)
  void* out[2];         // [0] h / y_perm, [1] hs / s
  int n[2];             // output columns per group kind
  int kdim[2];          // reduction depth per group kind
  const int32_t* offsets;
  int E;
  int64_t t_shared;     // rows of the shared group (0: none)
};

// Records the next per-kernel timing event on `st` when moe_forward runs with
// stage timing on (see moe_stage_timing_begin); a no-op otherwise. Every
// launcher calls it right after each kernel it launches.
// A launch on `st`, as a programmatic dependent of the kernel before it in the
// stream when `pdl` (it may start once that kernel's CTAs have all executed
// griddepcontrol.launch_dependents, and must griddepcontrol.wait before it
// reads that kernel's output), else an ordinary launch.
template <typename... Params, typename... Args>
inline cudaError_t launch_pdl(bool pdl, void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                            cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = pdl ? attr : nullptr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

void stage_mark(cudaStream_t st);
// Whether the small kernels of a forward may be launched as programmatic
// dependents of the kernel before them (not while the stage timer records
// events between the launches).
bool pdl_ok();
// Whether the stage timer is recording the current forward call.
bool stage_timing_active();

// Router: logits (tensor cores for bf16 unless `simt`, else CUDA cores) into
// `part` with at most `splits` k splits, then selection into weights / idx.
// With `hold_on_timeout`, the selection writes nothing while the timeout bit
// of `err` is set (moe_gate_noalloc: its partial sums may then be stale).
cudaError_t launch_router(const moe_config& c, int64_t T, const void* x, const void* w_router,
                          const float* bias, float* weights, int32_t* idx, float* part,
                          int splits, bool simt, int num_sms, uint32_t* err, cudaStream_t st,
                          bool hold_on_timeout = false);
int router_tc_splits(const moe_config& c, int64_t T, int max_splits, int num_sms);
cudaError_t launch_router_logits_tc(const moe_config& c, int64_t T, const void* x,
                                    const void* w_router, float* part, int splits, uint32_t* err,
                                    cudaStream_t st, int* splits_used);
// Built-in router scratch (moe_gate_noalloc): its size in floats, and the
// device addresses of the scratch and of its error word on the current device.
size_t gate_scratch_floats();
cudaError_t gate_scratch_current_device(float** scratch, uint32_t** err);

// x_perm may be null: then only counts, offsets, src and pos are written (by
// one kernel for a small batch, dispatch_small_ok).
cudaError_t launch_dispatch(const moe_config& c, int64_t T, const int32_t* idx, const void* x,
                            int32_t* counts, int32_t* offsets, int32_t* src, int32_t* pos,
                            void* x_perm, int32_t* chunk_hist, int32_t* pos_local, int n_chunks,
                            uint32_t* err, cudaStream_t st);
// The dispatch in its two halves: the sort (counts, offsets, each pair's
// rank within its chunk), then the placement (pos, src and, when x_perm is
// given, the permuted copy of x). The placement lets a programmatic dependent
// launch start at once (it must wait for the grid before reading src or x_perm).
cudaError_t launch_dispatch_sort(const moe_config& c, int64_t T, const int32_t* idx,
                                 int32_t* counts, int32_t* offsets, int32_t* chunk_hist,
                                 int32_t* pos_local, int n_chunks, uint32_t* err, cudaStream_t st);
struct DispatchPlace {
  const moe_config* c;
  int64_t T;
  const int32_t* idx;
  const void* x;
  const int32_t* chunk_hist;
  const int32_t* pos_local;
  int32_t* pos;
  int32_t* src;
  void* x_perm;
};
cudaError_t launch_dispatch_place(const DispatchPlace& p, cudaStream_t st);
// The whole dispatch of a small batch (dispatch_small_ok) in one launch:
// counts, offsets, pos and src, the same values as the three-kernel path.
bool dispatch_small_ok(const moe_config& c, int64_t T, const void* x_perm);
cudaError_t launch_dispatch_small(const moe_config& c, int64_t T, const int32_t* idx,
                                  int32_t* counts, int32_t* offsets, int32_t* pos, int32_t* src,
                                  uint32_t* err, cudaStream_t st);
cudaError_t launch_combine(const moe_config& c, int64_t T, const void* y_perm, const int32_t* pos,
                           const float* weights, const void* s, void* y, cudaStream_t st);
// Expert parallelism: one rank's fp32 share of y (pairs routed to its
// n_local experts, whose offsets start at offsets_local, plus its slice of
// the shared MLP in s), and the final cast of the summed shares.
cudaError_t launch_combine_partial(const moe_config& c, int64_t T, const void* y_perm,
                                   const int32_t* pos, const float* weights, const void* s,
                                   const int32_t* offsets_local, int n_local, float* y32,
                                   cudaStream_t st);
cudaError_t launch_cast(const moe_config& c, int64_t T, const float* y32, void* y, cudaStream_t st);

// FP8 expert weights (moe_forward_fp8): e4m3 values and the fp32 scales of
// their 128 x 128 blocks.
struct Fp8Weights {
  const uint8_t *w1, *w3, *w2, *ws1, *ws3, *ws2;
  const float *s1, *s3, *s2, *ss1, *ss3, *ss2;
};
// Activation rows [R, K] (act) to e4m3 with one scale per 1 x 128 block;
// the scales' row stride is sstride floats (<= 0: K/128).
// With pos (T * k row positions) and scale_perm, each block's scale is also
// written to its row's permuted rows (the up-projection's routed row order),
// and with q_perm ([T * k, K]) its codes too.
cudaError_t launch_quant_rows(const moe_config& c, const void* a, int64_t R, int K, uint8_t* q,
                              float* scale, int sstride, cudaStream_t st,
                              const int32_t* pos = nullptr, float* scale_perm = nullptr,
                              uint8_t* q_perm = nullptr);
// A matrix [R, C] (bf16 or fp32) to e4m3 with one scale per 128 x 128 block.
cudaError_t launch_quant_blocks(bool bf16, const void* a, int64_t R, int C, uint8_t* q,
                                float* scale, cudaStream_t st);
// The FP8 expert GEMMs (gemm_fp8.cu): UP from the quantized x (routed rows
// through src, their scales already in expert order in xs_perm) into the
// quantized h, DOWN from it into y_perm and s (act).
cudaError_t launch_grouped_fp8(const moe_config& c, int64_t T, const Fp8Weights& w,
                               const uint8_t* xq, const float* xs, float* xs_perm,
                               const int32_t* src, const int32_t* offsets, uint8_t* hq, float* hsc,
                               uint8_t* hsq, float* hss, void* y_perm, void* s, uint32_t* err,
                               int num_sms, cudaStream_t st);
// The same GEMMs with 128 token rows on the MMA's M side (gemm_fp8m.cu), for
// batches with many rows per expert: UP reads the routed rows' codes in
// expert order from xq_perm (scales xs_perm) and the shared MLP's from xq.
// row_maps: the per-expert maps launch_row_maps(fp8 = true) wrote over xq_perm
// and hq (an expert's last tile then reads zeros past its rows), or null.
cudaError_t launch_grouped_fp8m(const moe_config& c, int64_t T, const Fp8Weights& w,
                                const uint8_t* xq, const float* xs, const uint8_t* xq_perm,
                                const float* xs_perm, const int32_t* offsets, uint8_t* hq,
                                float* hsc, uint8_t* hsq, float* hss, void* y_perm, void* s,
                                const void* row_maps, uint32_t* err, int num_sms, cudaStream_t st);
cudaError_t launch_grouped_simt(const moe_config& c, int64_t T, bool up, const GroupedArgs& g,
                                cudaStream_t st);
// Grouped tensor-core expert GEMM kernels (launch_grouped_tc `kind`).
enum { TC_ROWS = 0, TC_PAIR = 1 };
// Test hook (moe_debug_stall_pipeline): which kernel's first CTA lets its
// first pipeline wait run out -- STALL_EXPERTS_UP the one-CTA up-projection,
// STALL_ROUTER the tensor-core router logits.
enum { STALL_NONE = 0, STALL_EXPERTS_UP = 1, STALL_ROUTER = 2 };
void set_pipeline_stall(int which);
int pipeline_stall();
// UP with src set (one-CTA kernel): the routed A rows are gathered from the
// token rows gx [gT, k0] through src (a0 unused). row_maps: the per-expert A
// maps written by launch_row_maps (null: none); tile_ctr: UP's tile counter.
cudaError_t launch_grouped_tc(bool up, int kind, int64_t Tk, int64_t T_sh, int E, const void* a0,
                              const void* a1, const void* b1_0, const void* b3_0, const void* b1_1,
                              const void* b3_1, int n0, int k0, int n1, int k1, void* out0,
                              void* out1, const int32_t* offsets, const void* gx,
                              const int32_t* src, int64_t gT, const void* row_maps, int* tile_ctr,
                              uint32_t* err, int num_sms, cudaStream_t st, bool pdl);
// Before the one-CTA expert GEMMs: per-expert copies of the down-projection's
// A map over h [Tk, I] (at maps + E) and, when a_up is given, of the
// up-projection's over a_up [Tk, D] (at maps), each with its row extent cut
// at the expert's end; zeroes the up-projection's tile counter. Reads only
// the offsets (a_up's rows need not be written yet). fp8: maps over e4m3
// rows for the FP8 token-on-M kernel (128-row boxes for every expert).
cudaError_t launch_row_maps(const void* h, int64_t Tk, int I, const void* a_up, int D,
                            const int32_t* offsets, int E, void* maps, int* up_tile_ctr,
                            cudaStream_t st, bool fp8 = false);

}  // namespace moe
