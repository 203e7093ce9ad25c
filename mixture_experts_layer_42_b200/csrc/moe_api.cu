// C ABI of the MoE layer library: argument checks, workspace carving and the
// launch sequence of each entry point (declared in include/moe.h).
#include "common.cuh"

#include <cmath>
#include <cstring>
#include <vector>

namespace moe {

namespace {

// Which kernel runs the expert GEMMs of a bf16 layer (see moe_select_expert_kernel).
int g_expert_kernel = MOE_EXPERT_KERNEL_AUTO;
// Which form runs the FP8 expert GEMMs (see moe_select_fp8_kernel).
int g_fp8_kernel = MOE_FP8_KERNEL_AUTO;

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int v) { return v > 0 && (v & (v - 1)) == 0; }

moe_status check_config(const moe_config* c, int64_t T) {
  if (!c || T < 1) return MOE_ERR_INVALID_ARG;
  if (c->dtype != MOE_DT_F32 && c->dtype != MOE_DT_BF16) return MOE_ERR_INVALID_ARG;
  if (c->score != MOE_SCORE_SIGMOID && c->score != MOE_SCORE_SOFTMAX) return MOE_ERR_INVALID_ARG;
  if (c->has_bias != 0 && c->has_bias != 1) return MOE_ERR_INVALID_ARG;
  if (!std::isfinite(c->route_scale)) return MOE_ERR_INVALID_ARG;
  const int E = c->n_routed, G = c->n_groups;
  if (E < 1 || G < 1 || c->topk < 1 || c->topk_groups < 1) return MOE_ERR_INVALID_ARG;
  if (E % G != 0 || c->topk_groups > G) return MOE_ERR_INVALID_ARG;
  const int per = E / G;
  if (c->topk > c->topk_groups * per) return MOE_ERR_INVALID_ARG;   // -inf never picked
  if (c->has_bias && G > 1 && per < 2) return MOE_ERR_INVALID_ARG;  // top-2 group score
  if (c->dim < 1 || c->moe_inter < 1 || c->shared_inter < 0) return MOE_ERR_INVALID_ARG;
  const int q = c->dtype == MOE_DT_BF16 ? 8 : 4;  // 16-byte rows
  if (c->dim % q || c->moe_inter % q || c->shared_inter % q) return MOE_ERR_INVALID_ARG;
  if (E > 1024 || G > 64 || c->topk > 32) return MOE_ERR_UNSUPPORTED;
  if (G > 1 && !((per <= 32 && is_pow2(per)) || per % 32 == 0)) return MOE_ERR_UNSUPPORTED;
  if (T * c->topk > (int64_t)INT32_MAX) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

moe_status check_ws(const moe_config& c, int64_t T, void* ws, size_t ws_bytes, WsLayout* L) {
  *L = ws_layout(c, T);
  if (!ws) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < L->total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<uint8_t*>(ws) + off);
}

int num_sms_current() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// Make this thread's current device the one the caller's work lives on: the
// device of `ptr` (a device buffer of the call), else the stream's device.
// The library carries its own copy of the CUDA runtime, whose current device
// does not follow the caller's runtime. The pointer query comes first
// because asking a stream for its device invalidates a CUDA graph capture
// in progress on that stream, which would keep moe_forward out of graphs.
moe_status bind_device(cudaStream_t s, const void* ptr) {
  int dev = -1;
  if (ptr) {
    cudaPointerAttributes pa;
    if (cudaPointerGetAttributes(&pa, ptr) != cudaSuccess) return MOE_ERR_INVALID_ARG;
    if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged)
      return MOE_ERR_INVALID_ARG;
    dev = pa.device;
  } else if (s) {
    if (cudaStreamGetDevice(s, &dev) != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    return MOE_ERR_INVALID_ARG;
  }
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return MOE_ERR_CUDA;
  if (cur != dev && cudaSetDevice(dev) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

// The expert GEMMs. The routed A rows come from x_perm (an expert-contiguous
// copy of x) or, when x_perm is null, are gathered from x through src. With
// `place`, the dispatch's placement (pos, src, the copy) is launched here,
// after the row maps (which need only the offsets) and right before the
// up-projection. With `dependent_up` (moe_forward), the up-projection is
// launched as a programmatic dependent of the kernel before it (the placement,
// or the row-map kernel after a one-kernel dispatch): its launch and setup
// overlap that kernel's tail, and it waits for that grid before it reads
// anything the dispatch wrote.
moe_status run_experts(const moe_config& c, int64_t T, const void* x_perm, const int32_t* src,
                       const int32_t* offsets, const void* w1, const void* w3, const void* w2,
                       const void* x, const void* ws1, const void* ws3, const void* ws2,
                       void* y_perm, void* s, void* h, void* hs, void* row_maps, uint32_t* err,
                       cudaStream_t st, const DispatchPlace* place = nullptr,
                       bool dependent_up = false) {
  const int64_t Tk = T * c.topk;
  const bool sh = c.shared_inter > 0;
  const bool tc = c.dtype == MOE_DT_BF16 && g_expert_kernel != MOE_EXPERT_KERNEL_SIMT;
  if (tc) {
    // One CTA per 128-row tile unless CTA pairs are asked for: measured on
    // the same GPU, the pairs' 256-row tiles pad enough extra rows at the
    // DeepSeek-V3 prefill shape to lose to single CTAs under the power cap.
    const int kind = g_expert_kernel == MOE_EXPERT_KERNEL_TCGEN05_PAIR ? TC_PAIR : TC_ROWS;
    if (kind == TC_PAIR && x_perm == nullptr) return MOE_ERR_UNSUPPORTED;
    // tile counters of the up and down launches, after the 2 x E row maps
    int* ctr = reinterpret_cast<int*>(static_cast<uint8_t*>(row_maps) + (size_t)2 * c.n_routed * 128);
    void* maps_down = static_cast<uint8_t*>(row_maps) + (size_t)c.n_routed * 128;
    cudaError_t e = cudaSuccess;
    if (kind == TC_ROWS) {
      // one small launch before both GEMMs: each expert's A maps with the row
      // extent cut at its end (the down-projection's over h, and the
      // up-projection's over x_perm unless it gathers from x), and the
      // up-projection's tile counter reset
      e = launch_row_maps(h, Tk, c.moe_inter, x_perm, c.dim, offsets, c.n_routed, row_maps, ctr, st);
      if (e != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (place != nullptr && launch_dispatch_place(*place, st) != cudaSuccess)
      return MOE_ERR_CUDA;
    // a small batch's dispatch ran in one kernel before the row maps: close
    // the timer's dispatch interval here (it then holds the row-map kernel)
    if (place == nullptr && dependent_up) stage_mark(st);
    // (not while the stage timer records events between the launches)
    const bool pdl = (place != nullptr || dependent_up) && kind == TC_ROWS && !stage_timing_active();
    e = launch_grouped_tc(true, kind, Tk, sh ? T : 0, c.n_routed, x_perm, x, w1, w3, ws1, ws3,
                          c.moe_inter, c.dim, c.shared_inter, c.dim, h, hs, offsets, x,
                          x_perm ? nullptr : src, T, kind == TC_ROWS ? row_maps : nullptr, ctr, err,
                          num_sms_current(), st, pdl);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
    // the down-projection as a programmatic dependent of the up-projection:
    // it prefetches its first weight tiles while the up-projection finishes
    e = launch_grouped_tc(false, kind, Tk, sh ? T : 0, c.n_routed, h, hs, w2, nullptr, ws2, nullptr,
                          c.dim, c.moe_inter, c.dim, c.shared_inter, y_perm, s, offsets, nullptr,
                          nullptr, 0, kind == TC_ROWS ? maps_down : nullptr, nullptr, err,
                          num_sms_current(), st, kind == TC_ROWS && !stage_timing_active());
    return cuda_status(e);
  }
  if (place != nullptr && launch_dispatch_place(*place, st) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (place == nullptr && dependent_up) stage_mark(st);
  GroupedArgs g;
  memset(&g, 0, sizeof(g));
  g.offsets = offsets;
  g.E = c.n_routed;
  g.t_shared = sh ? T : 0;
  g.a[0] = x_perm ? x_perm : x; g.a[1] = x;
  g.a_rows = x_perm ? nullptr : src;
  g.b1[0] = w1; g.b1[1] = ws1;
  g.b3[0] = w3; g.b3[1] = ws3;
  g.out[0] = h; g.out[1] = hs;
  g.n[0] = c.moe_inter; g.n[1] = c.shared_inter;
  g.kdim[0] = c.dim; g.kdim[1] = c.dim;
  cudaError_t e = launch_grouped_simt(c, T, true, g, st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  g.a[0] = h; g.a[1] = hs;
  g.a_rows = nullptr;
  g.b1[0] = w2; g.b1[1] = ws2;
  g.b3[0] = nullptr; g.b3[1] = nullptr;
  g.out[0] = y_perm; g.out[1] = s;
  g.n[0] = c.dim; g.n[1] = c.dim;
  g.kdim[0] = c.moe_inter; g.kdim[1] = c.shared_inter;
  return cuda_status(launch_grouped_simt(c, T, false, g, st));
}

// Per-kernel timing of moe_forward (moe_stage_timing_begin / _end).
struct StageTiming {
  bool on = false;        // armed by moe_stage_timing_begin
  bool in_forward = false;
  int max_calls = 0;
  int calls = 0;          // moe_forward calls recorded
  int every = 1;          // record one moe_forward call in `every`
  int seen = 0;           // moe_forward calls since begin
  int marks = 0;          // events recorded in the current call
  int per_call = 0;       // events per call (kernels + 1)
  std::vector<cudaEvent_t> ev;
};
StageTiming g_timing;

// Arms the per-kernel events for one forward call when stage timing is on
// (one call in `every`); counts the call if all its events were recorded.
struct TimedCall {
  explicit TimedCall(cudaStream_t s) {
    StageTiming& T = g_timing;
    T.in_forward = T.on && T.calls < T.max_calls && T.seen % T.every == 0;
    if (T.on) ++T.seen;
    if (T.in_forward) T.marks = 0;
    stage = s;
  }
  void start();
  ~TimedCall() {
    StageTiming& T = g_timing;
    if (T.in_forward) {
      if (T.marks == T.per_call) ++T.calls;
      T.in_forward = false;
    }
  }
  cudaStream_t stage;
};

// Average rows per expert up to which moe_forward gathers the up-projection's
// rows from x instead of copying them. Measured at the DeepSeek-V3 shape: the
// two take the same time at 16 rows per expert (T = 512), and the copy is
// faster above (T = 1024: 2.99 vs 3.51 ms per step; T = 2048: 3.56 vs 4.91),
// where experts run multi-row or 128-row tiles whose gathers bound the stage
// rate.
constexpr int64_t kGatherRows = 16;

// Average rows per expert above which moe_forward_fp8 runs its expert GEMMs
// with the tokens on the MMA's M side (the crossover measured at the
// DeepSeek-V3 shape: the two forms take the same time at 16 rows per expert,
// the token-on-N form is faster below, the token-on-M form above).
constexpr int64_t kFp8TokensOnMRows = 16;

// Whether moe_forward_fp8 runs the token-on-M form for T tokens (the
// selection, or AUTO's rule by the average rows per expert).
bool fp8_tokens_on_m(const moe_config& c, int64_t T) {
  return g_fp8_kernel == MOE_FP8_KERNEL_TOKENS_ON_M ||
         (g_fp8_kernel == MOE_FP8_KERNEL_AUTO && T * (int64_t)c.topk > kFp8TokensOnMRows * c.n_routed);
}

bool fp8_shapes_ok(const moe_config& c) {
  const int B = kFp8Block;
  if (c.dtype != MOE_DT_BF16) return false;
  if (c.dim % B || c.moe_inter % B || c.shared_inter % B) return false;
  return c.dim / B <= 64 && c.moe_inter / B <= 64 && c.shared_inter / B <= 64;
}

}  // namespace

bool stage_timing_active() { return g_timing.on && g_timing.in_forward; }

bool pdl_ok() { return !stage_timing_active(); }

void stage_mark(cudaStream_t st) {
  StageTiming& T = g_timing;
  if (!T.on || !T.in_forward || T.marks >= T.per_call) return;
  cudaEventRecord(T.ev[(size_t)T.calls * T.per_call + T.marks], st);
  ++T.marks;
}

namespace {
void TimedCall::start() { stage_mark(stage); }
}  // namespace

}  // namespace moe

using namespace moe;

extern "C" {

moe_status moe_workspace_size(const moe_config* cfg, int64_t T, size_t* bytes) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  *bytes = ws_layout(*cfg, T).total;
  return MOE_OK;
}

moe_status moe_workspace_init(void* ws, size_t ws_bytes, void* stream) {
  if (!ws || ws_bytes < kWsAlign || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  moe_status st = bind_device((cudaStream_t)stream, ws);
  if (st != MOE_OK) return st;
  return cuda_status(cudaMemsetAsync(ws, 0, kWsAlign, (cudaStream_t)stream));
}

moe_status moe_gate(const moe_config* cfg, int64_t T, const void* x, const void* w_router,
                    const float* bias, float* weights, int32_t* idx, void* ws, size_t ws_bytes,
                    void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(weights) || !aligned16(idx))
    return MOE_ERR_INVALID_ARG;
  if (cfg->has_bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((st = check_ws(*cfg, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = bind_device((cudaStream_t)stream, ws)) != MOE_OK) return st;
  return cuda_status(launch_router(*cfg, T, x, w_router, bias, weights, idx,
                                   at<float>(ws, L.router_part), L.router_splits,
                                   g_expert_kernel == MOE_EXPERT_KERNEL_SIMT, num_sms_current(),
                                   at<uint32_t>(ws, L.header), (cudaStream_t)stream));
}

moe_status moe_dispatch(const moe_config* cfg, int64_t T, const int32_t* idx, const void* x,
                        int32_t* counts, int32_t* offsets, int32_t* src, int32_t* pos,
                        void* x_perm, void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(idx) || !aligned16(counts) || !aligned16(offsets) || !aligned16(src) ||
      !aligned16(pos))
    return MOE_ERR_INVALID_ARG;
  if (x_perm && (!aligned16(x_perm) || !aligned16(x))) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((st = check_ws(*cfg, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = bind_device((cudaStream_t)stream, ws)) != MOE_OK) return st;
  return cuda_status(launch_dispatch(*cfg, T, idx, x, counts, offsets, src, pos, x_perm,
                                     at<int32_t>(ws, L.chunk_hist), at<int32_t>(ws, L.pos_local),
                                     L.n_chunks, at<uint32_t>(ws, L.header), (cudaStream_t)stream));
}

moe_status moe_experts_grouped(const moe_config* cfg, int64_t T, const void* x_perm,
                               const int32_t* offsets, const void* w1, const void* w3,
                               const void* w2, const void* x, const void* ws1, const void* ws3,
                               const void* ws2, void* y_perm, void* s, void* ws, size_t ws_bytes,
                               void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(x_perm) || !aligned16(offsets) || !aligned16(w1) || !aligned16(w3) ||
      !aligned16(w2) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if (cfg->shared_inter > 0 && (!aligned16(x) || !aligned16(ws1) || !aligned16(ws3) ||
                                !aligned16(ws2) || !aligned16(s)))
    return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((st = check_ws(*cfg, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = bind_device((cudaStream_t)stream, ws)) != MOE_OK) return st;
  return run_experts(*cfg, T, x_perm, nullptr, offsets, w1, w3, w2, x, ws1, ws3, ws2, y_perm, s,
                     at<void>(ws, L.h), at<void>(ws, L.hs), at<void>(ws, L.row_maps),
                     at<uint32_t>(ws, L.header), (cudaStream_t)stream);
}

moe_status moe_experts_grouped_gather(const moe_config* cfg, int64_t T, const void* x,
                                      const int32_t* src, const int32_t* offsets, const void* w1,
                                      const void* w3, const void* w2, const void* ws1,
                                      const void* ws3, const void* ws2, void* y_perm, void* s,
                                      void* ws, size_t ws_bytes, void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(src) || !aligned16(offsets) || !aligned16(w1) ||
      !aligned16(w3) || !aligned16(w2) || !aligned16(y_perm))
    return MOE_ERR_INVALID_ARG;
  if (cfg->shared_inter > 0 && (!aligned16(ws1) || !aligned16(ws3) || !aligned16(ws2) ||
                                !aligned16(s)))
    return MOE_ERR_INVALID_ARG;
  if (cfg->dtype == MOE_DT_BF16 && g_expert_kernel == MOE_EXPERT_KERNEL_TCGEN05_PAIR)
    return MOE_ERR_UNSUPPORTED;
  WsLayout L;
  if ((st = check_ws(*cfg, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = bind_device((cudaStream_t)stream, ws)) != MOE_OK) return st;
  return run_experts(*cfg, T, nullptr, src, offsets, w1, w3, w2, x, ws1, ws3, ws2, y_perm, s,
                     at<void>(ws, L.h), at<void>(ws, L.hs), at<void>(ws, L.row_maps),
                     at<uint32_t>(ws, L.header), (cudaStream_t)stream);
}

moe_status moe_combine(const moe_config* cfg, int64_t T, const void* y_perm, const int32_t* pos,
                       const float* weights, const void* s, void* y, void* ws, size_t ws_bytes,
                       void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(y_perm) || !aligned16(pos) || !aligned16(weights) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  if (s && !aligned16(s)) return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((st = check_ws(*cfg, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  if ((st = bind_device((cudaStream_t)stream, ws)) != MOE_OK) return st;
  return cuda_status(launch_combine(*cfg, T, y_perm, pos, weights, s, y, (cudaStream_t)stream));
}

moe_status moe_forward(const moe_config* cfg, int64_t T, const void* x, const void* w_router,
                       const float* bias, const void* w1, const void* w3, const void* w2,
                       const void* ws1, const void* ws3, const void* ws2, void* y,
                       float* weights_out, int32_t* idx_out, void* ws, size_t ws_bytes,
                       void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w1) || !aligned16(w3) ||
      !aligned16(w2) || !aligned16(y))
    return MOE_ERR_INVALID_ARG;
  if (c.has_bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  if (c.shared_inter > 0 && (!aligned16(ws1) || !aligned16(ws3) || !aligned16(ws2)))
    return MOE_ERR_INVALID_ARG;
  if ((weights_out && !aligned16(weights_out)) || (idx_out && !aligned16(idx_out)))
    return MOE_ERR_INVALID_ARG;
  WsLayout L;
  if ((st = check_ws(c, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = bind_device(s, ws)) != MOE_OK) return st;
  TimedCall timed(s);
  timed.start();
  float* weights = weights_out ? weights_out : at<float>(ws, L.weights);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
  uint32_t* err = at<uint32_t>(ws, L.header);
  if (launch_router(c, T, x, w_router, bias, weights, idx, at<float>(ws, L.router_part),
                    L.router_splits, g_expert_kernel == MOE_EXPERT_KERNEL_SIMT, num_sms_current(),
                    err, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* pos = at<int32_t>(ws, L.pos);
  int32_t* src = at<int32_t>(ws, L.src);
  // The routed token rows reach the up-projection either straight from x
  // through src (tile::gather4, four rows per copy) or from an
  // expert-contiguous copy made by the dispatch (one tile copy per stage).
  // Measured on B200 at the DeepSeek-V3 shape: with 128-row tiles the 32
  // gathers per stage bound the up-projection by the TMA's copy rate (10.9
  // against 4.8 ms at T = 8192), while batches of at most kGatherRows rows per
  // expert on average (decode) run their few rows as swapped tiles and gather
  // 4 to 16 rows per stage at no cost. So batches that average more rows per expert, and
  // the CTA-pair option, take the copy; it lives in y_perm's space, which is
  // free until the down-projection writes it.
  const bool big = T * (int64_t)c.topk > (int64_t)kGatherRows * c.n_routed;
  const bool copy_rows = c.dtype == MOE_DT_BF16 &&
                         (g_expert_kernel == MOE_EXPERT_KERNEL_TCGEN05_PAIR || big);
  void* x_perm = copy_rows ? at<void>(ws, L.y_perm) : nullptr;
  // a small batch without the copy: the whole dispatch in one kernel (the
  // timer's rank interval; its scan interval stays empty)
  const bool small = dispatch_small_ok(c, T, x_perm);
  if (small) {
    if (launch_dispatch_small(c, T, idx, at<int32_t>(ws, L.counts), offsets, pos, src, err, s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    stage_mark(s);
    stage_mark(s);
  } else if (launch_dispatch_sort(c, T, idx, at<int32_t>(ws, L.counts), offsets,
                                  at<int32_t>(ws, L.chunk_hist), at<int32_t>(ws, L.pos_local),
                                  L.n_chunks, err, s) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  const DispatchPlace place{&c, T, idx, x, at<int32_t>(ws, L.chunk_hist),
                            at<int32_t>(ws, L.pos_local), pos, src, x_perm};
  const bool sh = c.shared_inter > 0;
  void* sbuf = sh ? at<void>(ws, L.s) : nullptr;
  st = run_experts(c, T, x_perm, src, offsets, w1, w3, w2, x, ws1, ws3, ws2,
                   at<void>(ws, L.y_perm), sbuf, at<void>(ws, L.h), at<void>(ws, L.hs),
                   at<void>(ws, L.row_maps), err, s, small ? nullptr : &place, true);
  if (st != MOE_OK) return st;
  return cuda_status(launch_combine(c, T, at<void>(ws, L.y_perm), pos, weights, sbuf, y, s));
}

moe_status moe_forward_ep(const moe_config* cfg, int64_t T, int32_t expert_begin,
                          int32_t expert_end, int32_t shared_local, const void* x,
                          const void* w_router, const float* bias, const void* w1, const void* w3,
                          const void* w2, const void* ws1, const void* ws3, const void* ws2,
                          float* y_partial, float* weights_out, int32_t* idx_out, void* ws,
                          size_t ws_bytes, void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (expert_begin < 0 || expert_end <= expert_begin || expert_end > c.n_routed)
    return MOE_ERR_INVALID_ARG;
  const int q = c.dtype == MOE_DT_BF16 ? 8 : 4;
  if (shared_local < 0 || shared_local > c.shared_inter || shared_local % q) return MOE_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(w1) || !aligned16(w3) ||
      !aligned16(w2) || !aligned16(y_partial))
    return MOE_ERR_INVALID_ARG;
  if (c.has_bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  if (shared_local > 0 && (!aligned16(ws1) || !aligned16(ws3) || !aligned16(ws2)))
    return MOE_ERR_INVALID_ARG;
  if ((weights_out && !aligned16(weights_out)) || (idx_out && !aligned16(idx_out)))
    return MOE_ERR_INVALID_ARG;
  if (c.dtype == MOE_DT_BF16 && g_expert_kernel == MOE_EXPERT_KERNEL_TCGEN05_PAIR)
    return MOE_ERR_UNSUPPORTED;
  WsLayout L;
  if ((st = check_ws(c, T, ws, ws_bytes, &L)) != MOE_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = bind_device(s, ws)) != MOE_OK) return st;
  float* weights = weights_out ? weights_out : at<float>(ws, L.weights);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
  uint32_t* err = at<uint32_t>(ws, L.header);
  // this rank's experts are a contiguous run of the expert order: the
  // grouped GEMMs see them as a layer of n_local experts whose offsets start
  // at expert_begin's, and the shared MLP as one of width shared_local
  moe_config lc = c;
  lc.n_routed = expert_end - expert_begin;
  lc.shared_inter = shared_local;
  // every rank routes every token over all experts (the gate is replicated)
  if (launch_router(c, T, x, w_router, bias, weights, idx, at<float>(ws, L.router_part),
                    L.router_splits, g_expert_kernel == MOE_EXPERT_KERNEL_SIMT, num_sms_current(),
                    err, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* pos = at<int32_t>(ws, L.pos);
  int32_t* src = at<int32_t>(ws, L.src);
  // gathered rows or a permuted copy, by the same rule as moe_forward
  const bool big = T * (int64_t)c.topk > (int64_t)kGatherRows * c.n_routed;
  void* x_perm = (c.dtype == MOE_DT_BF16 && big) ? at<void>(ws, L.y_perm) : nullptr;
  // a small batch without the copy: the whole dispatch in one kernel (the
  // timer's rank interval; its scan interval stays empty)
  const bool small = dispatch_small_ok(c, T, x_perm);
  if (small) {
    if (launch_dispatch_small(c, T, idx, at<int32_t>(ws, L.counts), offsets, pos, src, err, s) !=
        cudaSuccess)
      return MOE_ERR_CUDA;
    stage_mark(s);
    stage_mark(s);
  } else if (launch_dispatch_sort(c, T, idx, at<int32_t>(ws, L.counts), offsets,
                                  at<int32_t>(ws, L.chunk_hist), at<int32_t>(ws, L.pos_local),
                                  L.n_chunks, err, s) != cudaSuccess) {
    return MOE_ERR_CUDA;
  }
  const DispatchPlace place{&c, T, idx, x, at<int32_t>(ws, L.chunk_hist),
                            at<int32_t>(ws, L.pos_local), pos, src, x_perm};
  const int32_t* off_local = offsets + expert_begin;
  void* sbuf = shared_local > 0 ? at<void>(ws, L.s) : nullptr;
  st = run_experts(lc, T, x_perm, src, off_local, w1, w3, w2, x, ws1, ws3, ws2,
                   at<void>(ws, L.y_perm), sbuf, at<void>(ws, L.h), at<void>(ws, L.hs),
                   at<void>(ws, L.row_maps), err, s, small ? nullptr : &place, true);
  if (st != MOE_OK) return st;
  return cuda_status(launch_combine_partial(c, T, at<void>(ws, L.y_perm), pos, weights, sbuf,
                                            off_local, lc.n_routed, y_partial, s));
}

moe_status moe_cast_output(const moe_config* cfg, int64_t T, const float* y_sum, void* y,
                           void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(y_sum) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if ((st = bind_device((cudaStream_t)stream, y)) != MOE_OK) return st;
  return cuda_status(launch_cast(*cfg, T, y_sum, y, (cudaStream_t)stream));
}

moe_status moe_quantize_fp8(const moe_config* cfg, const void* a, int64_t rows, int64_t cols,
                            int32_t block_rows, void* q, float* scales, void* stream) {
  if (!cfg || (cfg->dtype != MOE_DT_BF16 && cfg->dtype != MOE_DT_F32)) return MOE_ERR_INVALID_ARG;
  if (rows < 1 || cols < kFp8Block || cols % kFp8Block || cols > INT32_MAX) return MOE_ERR_INVALID_ARG;
  if (block_rows != 1 && block_rows != kFp8Block) return MOE_ERR_INVALID_ARG;
  if (!aligned16(a) || !aligned16(q) || !aligned16(scales)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  moe_status st = bind_device(s, a);
  if (st != MOE_OK) return st;
  if (block_rows == 1)
    return cuda_status(launch_quant_rows(*cfg, a, rows, (int)cols, static_cast<uint8_t*>(q), scales, 0, s));
  return cuda_status(launch_quant_blocks(cfg->dtype == MOE_DT_BF16, a, rows, (int)cols,
                                         static_cast<uint8_t*>(q), scales, s));
}

moe_status moe_workspace_size_fp8(const moe_config* cfg, int64_t T, size_t* bytes) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!bytes) return MOE_ERR_INVALID_ARG;
  if (!fp8_shapes_ok(*cfg)) return MOE_ERR_UNSUPPORTED;
  *bytes = fp8_layout(*cfg, T, ws_layout(*cfg, T).total).total;
  return MOE_OK;
}

moe_status moe_forward_fp8(const moe_config* cfg, int64_t T, const void* x, const void* w_router,
                           const float* bias, const moe_fp8_weights* w, void* y,
                           float* weights_out, int32_t* idx_out, void* ws, size_t ws_bytes,
                           void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (!fp8_shapes_ok(c)) return MOE_ERR_UNSUPPORTED;
  if (!w || !aligned16(x) || !aligned16(w_router) || !aligned16(y)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w->w1) || !aligned16(w->w3) || !aligned16(w->w2) || !aligned16(w->w1_scale) ||
      !aligned16(w->w3_scale) || !aligned16(w->w2_scale))
    return MOE_ERR_INVALID_ARG;
  if (c.shared_inter > 0 &&
      (!aligned16(w->ws1) || !aligned16(w->ws3) || !aligned16(w->ws2) ||
       !aligned16(w->ws1_scale) || !aligned16(w->ws3_scale) || !aligned16(w->ws2_scale)))
    return MOE_ERR_INVALID_ARG;
  if (c.has_bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  if ((weights_out && !aligned16(weights_out)) || (idx_out && !aligned16(idx_out)))
    return MOE_ERR_INVALID_ARG;
  WsLayout L = ws_layout(c, T);
  const Fp8Layout F = fp8_layout(c, T, L.total);
  if (!ws) return MOE_ERR_WORKSPACE;
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  if (ws_bytes < F.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = bind_device(s, ws)) != MOE_OK) return st;
  TimedCall timed(s);
  timed.start();
  float* weights = weights_out ? weights_out : at<float>(ws, L.weights);
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
  uint32_t* err = at<uint32_t>(ws, L.header);
  if (launch_router(c, T, x, w_router, bias, weights, idx, at<float>(ws, L.router_part),
                    L.router_splits, g_expert_kernel == MOE_EXPERT_KERNEL_SIMT, num_sms_current(),
                    err, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  int32_t* pos = at<int32_t>(ws, L.pos);
  int32_t* src = at<int32_t>(ws, L.src);
  if (launch_dispatch(c, T, idx, x, at<int32_t>(ws, L.counts), offsets, src, pos, nullptr,
                      at<int32_t>(ws, L.chunk_hist), at<int32_t>(ws, L.pos_local), L.n_chunks, err,
                      s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // x to e4m3 once per step, each block's scale also to the routed pairs'
  // permuted rows, and for the token-on-M form their codes too (its kernel
  // is timed with the up-projection)
  const bool on_m = fp8_tokens_on_m(c, T);
  uint8_t* xq = at<uint8_t>(ws, F.xq);
  float* xs = at<float>(ws, F.xs);
  uint8_t* xq_perm = on_m ? at<uint8_t>(ws, F.xq_perm) : nullptr;
  void* row_maps = at<void>(ws, L.row_maps);
  if (on_m) {
    // per-expert maps over the routed rows of x and h (the tile counter the
    // kernel also zeroes is not used on this path)
    int* ctr = reinterpret_cast<int*>(static_cast<uint8_t*>(row_maps) + (size_t)2 * c.n_routed * 128);
    if (launch_row_maps(at<uint8_t>(ws, F.hq), T * c.topk, c.moe_inter, xq_perm, c.dim, offsets,
                        c.n_routed, row_maps, ctr, s, true) != cudaSuccess)
      return MOE_ERR_CUDA;
  }
  if (launch_quant_rows(c, x, T, c.dim, xq, xs, fp8_stride_host(c.dim), s, pos,
                        at<float>(ws, F.xs_perm), xq_perm) != cudaSuccess)
    return MOE_ERR_CUDA;
  Fp8Weights fw{static_cast<const uint8_t*>(w->w1), static_cast<const uint8_t*>(w->w3),
                static_cast<const uint8_t*>(w->w2), static_cast<const uint8_t*>(w->ws1),
                static_cast<const uint8_t*>(w->ws3), static_cast<const uint8_t*>(w->ws2),
                w->w1_scale, w->w3_scale, w->w2_scale, w->ws1_scale, w->ws3_scale, w->ws2_scale};
  const bool sh = c.shared_inter > 0;
  void* sbuf = sh ? at<void>(ws, L.s) : nullptr;
  const cudaError_t ge =
      on_m ? launch_grouped_fp8m(c, T, fw, xq, xs, xq_perm, at<float>(ws, F.xs_perm), offsets,
                                 at<uint8_t>(ws, F.hq), at<float>(ws, F.hs), at<uint8_t>(ws, F.hsq),
                                 at<float>(ws, F.hss), at<void>(ws, L.y_perm), sbuf, row_maps, err,
                                 num_sms_current(), s)
           : launch_grouped_fp8(c, T, fw, xq, xs, at<float>(ws, F.xs_perm), src, offsets,
                                at<uint8_t>(ws, F.hq), at<float>(ws, F.hs), at<uint8_t>(ws, F.hsq),
                                at<float>(ws, F.hss), at<void>(ws, L.y_perm), sbuf, err,
                                num_sms_current(), s);
  if (ge != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_combine(c, T, at<void>(ws, L.y_perm), pos, weights, sbuf, y, s));
}

moe_status moe_check_error(void* ws, void* stream) {
  if (!ws || !aligned16(ws)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  moe_status st = bind_device(s, ws);
  if (st != MOE_OK) return st;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, ws, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(word), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (word & ERRBIT_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (word & ERRBIT_BAD_INDEX) return MOE_ERR_DEVICE_CHECK;
  return MOE_OK;
}

const char* moe_status_string(moe_status st) {
  switch (st) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing or too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_DEVICE_CHECK: return "device-side check failed (expert index out of range)";
    case MOE_ERR_TIMEOUT: return "device pipeline wait timed out";
  }
  return "unknown status";
}

int32_t moe_forward_launch_count(const moe_config* cfg, int64_t T) {
  if (check_config(cfg, T) != MOE_OK) return -1;
  // router: logits + select; dispatch: rank + scan + positions, or one kernel
  // for a small batch without the row copy (the rule of moe_forward);
  // experts: up + down, with one kernel that writes the per-expert A maps
  // when the one-CTA tensor-core kernel runs; combine
  const moe_config& c = *cfg;
  const bool row_maps = c.dtype == MOE_DT_BF16 && (g_expert_kernel == MOE_EXPERT_KERNEL_AUTO ||
                                                   g_expert_kernel == MOE_EXPERT_KERNEL_TCGEN05);
  const bool copy_rows = c.dtype == MOE_DT_BF16 &&
                         (g_expert_kernel == MOE_EXPERT_KERNEL_TCGEN05_PAIR ||
                          T * (int64_t)c.topk > (int64_t)kGatherRows * c.n_routed);
  const bool small = T * (int64_t)c.topk <= kDispatchSmallPairs &&
                     c.n_routed <= kDispatchSmallExperts && !copy_rows;
  return 2 + (small ? 1 : 3) + 2 + (row_maps ? 1 : 0) + 1;
}

moe_status moe_gate_noalloc(const moe_config* cfg, int64_t T, const void* x, const void* w_router,
                            const float* bias, float* weights, int32_t* idx, void* stream) {
  moe_status st = check_config(cfg, T);
  if (st != MOE_OK) return st;
  if (!aligned16(x) || !aligned16(w_router) || !aligned16(weights) || !aligned16(idx))
    return MOE_ERR_INVALID_ARG;
  if (cfg->has_bias && !aligned16(bias)) return MOE_ERR_INVALID_ARG;
  const int64_t per_split = T * (int64_t)cfg->n_routed;  // floats of one split's partials
  if (per_split > (int64_t)gate_scratch_floats()) return MOE_ERR_UNSUPPORTED;
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = bind_device(s, x)) != MOE_OK) return st;
  float* scratch = nullptr;
  uint32_t* err = nullptr;
  if (gate_scratch_current_device(&scratch, &err) != cudaSuccess) return MOE_ERR_CUDA;
  int splits = router_splits(*cfg, T);
  const int64_t fit = (int64_t)gate_scratch_floats() / per_split;
  if (splits > fit) splits = (int)fit;
  // a router wait that runs out sets the timeout bit of the built-in error
  // word; the selection then writes no routing until the word is cleared
  return cuda_status(launch_router(*cfg, T, x, w_router, bias, weights, idx, scratch, splits,
                                   g_expert_kernel == MOE_EXPERT_KERNEL_SIMT, num_sms_current(),
                                   err, s, /*hold_on_timeout=*/true));
}

moe_status moe_gate_noalloc_check_error(const void* x, void* stream) {
  cudaStream_t s = (cudaStream_t)stream;
  moe_status st = bind_device(s, x);
  if (st != MOE_OK) return st;
  float* scratch = nullptr;
  uint32_t* err = nullptr;
  if (gate_scratch_current_device(&scratch, &err) != cudaSuccess) return MOE_ERR_CUDA;
  uint32_t word = 0;
  if (cudaMemcpyAsync(&word, err, sizeof(word), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (cudaMemsetAsync(err, 0, sizeof(word), s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  return (word & ERRBIT_TIMEOUT) ? MOE_ERR_TIMEOUT : MOE_OK;
}

moe_status moe_stage_timing_begin(int32_t max_calls) {
  return moe_stage_timing_begin_every(max_calls, 1);
}
moe_status moe_stage_timing_begin_every(int32_t max_calls, int32_t every) {
  StageTiming& T = g_timing;
  if (max_calls < 1 || max_calls > 4096 || every < 1) return MOE_ERR_INVALID_ARG;
  for (cudaEvent_t e : T.ev) cudaEventDestroy(e);
  T.ev.clear();
  T.per_call = 2 + 3 + 2 + 1 + 1;
  T.ev.resize((size_t)max_calls * T.per_call, nullptr);
  for (auto& e : T.ev)
    if (cudaEventCreate(&e) != cudaSuccess) return MOE_ERR_CUDA;
  T.max_calls = max_calls;
  T.calls = 0;
  T.every = every;
  T.seen = 0;
  T.on = true;
  return MOE_OK;
}

int32_t moe_stage_timing_end(float* ms, int32_t n) {
  StageTiming& T = g_timing;
  if (!T.on) return MOE_ERR_INVALID_ARG;
  T.on = false;
  const int kernels = T.per_call - 1;
  if (!ms || n < 1 || n > kernels) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n; ++i) ms[i] = 0.f;
  for (int c = 0; c < T.calls; ++c) {
    for (int i = 0; i < n; ++i) {
      cudaEvent_t a = T.ev[(size_t)c * T.per_call + i], b = T.ev[(size_t)c * T.per_call + i + 1];
      if (cudaEventSynchronize(b) != cudaSuccess) return MOE_ERR_CUDA;
      float t = 0.f;
      if (cudaEventElapsedTime(&t, a, b) != cudaSuccess) return MOE_ERR_CUDA;
      ms[i] += t;
    }
  }
  return T.calls;
}

moe_status moe_debug_stall_pipeline(int32_t enable) {
  if (enable != STALL_NONE && enable != STALL_EXPERTS_UP && enable != STALL_ROUTER)
    return MOE_ERR_INVALID_ARG;
  set_pipeline_stall(enable);
  return MOE_OK;
}

moe_status moe_select_expert_kernel(int32_t which) {
  if (which != MOE_EXPERT_KERNEL_AUTO && which != MOE_EXPERT_KERNEL_SIMT &&
      which != MOE_EXPERT_KERNEL_TCGEN05 && which != MOE_EXPERT_KERNEL_TCGEN05_PAIR)
    return MOE_ERR_INVALID_ARG;
  g_expert_kernel = which;
  return MOE_OK;
}

int32_t moe_fp8_kernel_for(const moe_config* cfg, int64_t T) {
  if (check_config(cfg, T) != MOE_OK) return -1;
  return fp8_tokens_on_m(*cfg, T) ? MOE_FP8_KERNEL_TOKENS_ON_M : MOE_FP8_KERNEL_TOKENS_ON_N;
}

moe_status moe_select_fp8_kernel(int32_t which) {
  if (which != MOE_FP8_KERNEL_AUTO && which != MOE_FP8_KERNEL_TOKENS_ON_N &&
      which != MOE_FP8_KERNEL_TOKENS_ON_M)
    return MOE_ERR_INVALID_ARG;
  g_fp8_kernel = which;
  return MOE_OK;
}

}  // extern "C"
