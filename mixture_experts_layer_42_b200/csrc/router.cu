// Router of the MoE layer (page "DeepSeek-V3.2-Exp - Expert scores",
// Gate.forward): fp32 logits z = x . W_r^T, softmax or sigmoid scores, the
// selection-only bias, group-limited top-k and the routing weights.
//
// Two kernels:
//   router_logits_kernel  SIMT GEMM [T, D] x [E, D]^T, split over k. The
//                         bf16 x bf16 products are exact in fp32; they are
//                         summed in fp32 over 64-deep chunks and each chunk is
//                         added into an fp64 accumulator, so the only rounding
//                         that matters is the final cast of each split's sum
//                         to fp32 (near-ties in routing depend on this).
//   router_select_kernel  8 tokens per CTA: the CTA sums the splits (fp64,
//                         fixed order) into shared memory, then one warp per
//                         token applies the score function, bias, group limit
//                         and top-k with shuffle reductions and writes idx /
//                         weights.
#include "common.cuh"

#include <float.h>

#include <mutex>

namespace moe {

namespace {

constexpr int RBM = kRouterBM, RBN = kRouterBN, RBK = kRouterBK;
constexpr int RTHREADS = 256;
constexpr int RTM = 8, RTN = 4;         // per-thread micro tile (tokens x experts)
constexpr int RAPAD = 4;                // smem padding of the transposed tiles

template <typename T>
__device__ __forceinline__ void load_vec(const T* base, int64_t rows, int64_t ld, int64_t row,
                                         int k0, int kend, float* out) {
  constexpr int VE = 16 / sizeof(T);
  if (row < rows && k0 + VE <= kend) {
    Vec16<T> v;
    v.raw = *reinterpret_cast<const uint4*>(base + row * ld + k0);
    v.to_float(out);
  } else {
#pragma unroll
    for (int q = 0; q < VE; ++q) {
      int k = k0 + q;
      out[q] = (row < rows && k < kend) ? to_f32(base[row * ld + k]) : 0.f;
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(RTHREADS)
router_logits_kernel(const T* __restrict__ x, const T* __restrict__ w, int64_t T_tok, int E,
                     int D, int k_per_split, float* __restrict__ part) {
  constexpr int VE = 16 / sizeof(T);
  constexpr int A_VECS = RBM * RBK / VE / RTHREADS;   // vectors of x per thread per slice
  constexpr int B_VECS = RBN * RBK / VE / RTHREADS;   // vectors of W_r per thread per slice
  constexpr int VPR = RBK / VE;                       // vectors per tile row
  __shared__ __align__(16) float As[RBK][RBM + RAPAD];
  __shared__ __align__(16) float Bs[RBK][RBN + RAPAD];

  const int tid = threadIdx.x;
  const int tn = tid % 16, tm = tid / 16;
  const int64_t m0 = (int64_t)blockIdx.x * RBM;
  const int n0 = blockIdx.y * RBN;
  const int split = blockIdx.z;
  const int kbeg = split * k_per_split;
  const int kend = min(D, kbeg + k_per_split);

  double acc64[RTM][RTN];
  float acc[RTM][RTN];
#pragma unroll
  for (int i = 0; i < RTM; ++i)
#pragma unroll
    for (int j = 0; j < RTN; ++j) { acc64[i][j] = 0.0; acc[i][j] = 0.f; }

  float ra[A_VECS][VE], rb[B_VECS][VE];
  auto gload = [&](int kt) {
#pragma unroll
    for (int i = 0; i < A_VECS; ++i) {
      int v = tid + i * RTHREADS;
      load_vec<T>(x, T_tok, D, m0 + v / VPR, kt + (v % VPR) * VE, kend, ra[i]);
    }
#pragma unroll
    for (int i = 0; i < B_VECS; ++i) {
      int v = tid + i * RTHREADS;
      load_vec<T>(w, E, D, n0 + v / VPR, kt + (v % VPR) * VE, kend, rb[i]);
    }
  };
  auto sstore = [&]() {
#pragma unroll
    for (int i = 0; i < A_VECS; ++i) {
      int v = tid + i * RTHREADS;
#pragma unroll
      for (int q = 0; q < VE; ++q) As[(v % VPR) * VE + q][v / VPR] = ra[i][q];
    }
#pragma unroll
    for (int i = 0; i < B_VECS; ++i) {
      int v = tid + i * RTHREADS;
#pragma unroll
      for (int q = 0; q < VE; ++q) Bs[(v % VPR) * VE + q][v / VPR] = rb[i][q];
    }
  };

  int slice = 0;
  if (kbeg < kend) gload(kbeg);
  for (int kt = kbeg; kt < kend; kt += RBK, ++slice) {
    __syncthreads();
    sstore();
    __syncthreads();
    if (kt + RBK < kend) gload(kt + RBK);
#pragma unroll 8
    for (int kk = 0; kk < RBK; ++kk) {
      float a[RTM], b[RTN];
      float4 a0 = *reinterpret_cast<const float4*>(&As[kk][tm * RTM]);
      float4 a1 = *reinterpret_cast<const float4*>(&As[kk][tm * RTM + 4]);
      float4 b0 = *reinterpret_cast<const float4*>(&Bs[kk][tn * RTN]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w;
      a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      b[0] = b0.x; b[1] = b0.y; b[2] = b0.z; b[3] = b0.w;
#pragma unroll
      for (int i = 0; i < RTM; ++i)
#pragma unroll
        for (int j = 0; j < RTN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (slice & 1) {  // every 64 products: move the fp32 chunk sums into fp64
#pragma unroll
      for (int i = 0; i < RTM; ++i)
#pragma unroll
        for (int j = 0; j < RTN; ++j) { acc64[i][j] += (double)acc[i][j]; acc[i][j] = 0.f; }
    }
  }
#pragma unroll
  for (int i = 0; i < RTM; ++i)
#pragma unroll
    for (int j = 0; j < RTN; ++j) acc64[i][j] += (double)acc[i][j];

  float* out = part + (int64_t)split * T_tok * E;
#pragma unroll
  for (int i = 0; i < RTM; ++i) {
    int64_t t = m0 + tm * RTM + i;
    if (t >= T_tok) continue;
#pragma unroll
    for (int j = 0; j < RTN; ++j) {
      int e = n0 + tn * RTN + j;
      if (e < E) out[t * E + e] = (float)acc64[i][j];
    }
  }
}

// (value, index) ordering of every top-k here: larger value first, equal
// values go to the lower index.
__device__ __forceinline__ bool better(float v, int i, float bv, int bi) {
  return v > bv || (v == bv && i < bi);
}

__device__ __forceinline__ void top2_merge(float& m1, float& m2, float p1, float p2) {
  float hi = fmaxf(m1, p1), lo = fminf(m1, p1);
  m2 = fmaxf(lo, fmaxf(m2, p2));
  m1 = hi;
}

struct SelectArgs {
  const float* part;
  int splits;
  const float* bias;
  int64_t T;
  int E, G, TG, k;
  int sigmoid;
  float route_scale;
  float* weights;
  int32_t* idx;
  // when set: write nothing while its timeout bit is set (the logits may be
  // partial)
  const uint32_t* hold_on_timeout;
};

// Values per lane VPL = ceil(E / 32); expert e lives in lane e % 32, slot e / 32.
template <int VPL>
__global__ void __launch_bounds__(256) router_select_kernel(const SelectArgs a) {
  extern __shared__ float z_s[];  // [8][E] logits of this CTA's tokens
  __shared__ float gsc_s[8][64];
  // launched as a programmatic dependent of the logits kernel: the dispatch
  // after it may start; the logits (and the error word) are read after the
  // logits grid completes
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (a.hold_on_timeout && (*a.hold_on_timeout & ERRBIT_TIMEOUT)) return;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int E = a.E;
  const int64_t t0 = (int64_t)blockIdx.x * 8;

  // 1. logits: the CTA sums the k splits of its (up to) 8 tokens together --
  //    each split's rows are one contiguous block of 8*E floats, and thread
  //    i owns elements i + 256 q, q < VPL -- in fp64, in split order, with
  //    one fp32 rounding, into shared memory. All VPL loads of a split are in
  //    flight together.
  {
    const int64_t rows = a.T - t0 < 8 ? a.T - t0 : 8;
    const int n = (int)(rows * E);
    const int64_t stride = a.T * E;
    const float* base = a.part + t0 * E;
    double s[VPL];
#pragma unroll
    for (int q = 0; q < VPL; ++q) s[q] = 0.0;
#pragma unroll 4
    for (int sp = 0; sp < a.splits; ++sp) {
      float p[VPL];
#pragma unroll
      for (int q = 0; q < VPL; ++q) {
        const int i = threadIdx.x + 256 * q;
        p[q] = i < n ? base[sp * stride + i] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < VPL; ++q) s[q] += (double)p[q];
    }
#pragma unroll
    for (int q = 0; q < VPL; ++q) {
      const int i = threadIdx.x + 256 * q;
      if (i < n) z_s[i] = (float)s[q];
    }
  }
  __syncthreads();
  const int64_t t = t0 + warp;
  if (t >= a.T) return;
  float z[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const int e = v * 32 + lane;
    z[v] = (e < E) ? z_s[warp * E + e] : -INFINITY;
  }

  // 2. scores (unbiased) and 3. selection scores
  float s[VPL], b[VPL];
  if (a.sigmoid) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) s[v] = (v * 32 + lane < E) ? 1.0f / (1.0f + expf(-z[v])) : 0.f;
  } else {
    float m = -INFINITY;
#pragma unroll
    for (int v = 0; v < VPL; ++v) m = fmaxf(m, z[v]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = 0.f;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      s[v] = (v * 32 + lane < E) ? expf(z[v] - m) : 0.f;
      sum += s[v];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
#pragma unroll
    for (int v = 0; v < VPL; ++v) s[v] = s[v] / sum;
  }
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    int e = v * 32 + lane;
    b[v] = (e < E) ? (a.bias ? s[v] + a.bias[e] : s[v]) : -INFINITY;
  }

  // 4. group limit: score each contiguous block of E/G experts by its top-2
  //    sum (bias present) or its max, keep the best TG groups
  uint64_t keep = ~0ull;
  if (a.G > 1) {
    const int per = E / a.G;
    const bool use_top2 = a.bias != nullptr;
    if (per <= 32) {
      // groups sit inside one slot, on aligned runs of `per` lanes
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        float m1 = b[v], m2 = -INFINITY;
        for (int o = 1; o < per; o <<= 1) {
          float p1 = __shfl_xor_sync(0xffffffffu, m1, o);
          float p2 = __shfl_xor_sync(0xffffffffu, m2, o);
          top2_merge(m1, m2, p1, p2);
        }
        int g = v * (32 / per) + lane / per;
        if (lane % per == 0 && g < a.G) gsc_s[warp][g] = use_top2 ? m1 + m2 : m1;
      }
    } else {
      // each group spans per/32 whole slots
      const int spg = per / 32;
      for (int g = 0; g < a.G; ++g) {
        float m1 = -INFINITY, m2 = -INFINITY;
#pragma unroll
        for (int v = 0; v < VPL; ++v)
          if (v / spg == g) top2_merge(m1, m2, b[v], -INFINITY);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          float p1 = __shfl_xor_sync(0xffffffffu, m1, o);
          float p2 = __shfl_xor_sync(0xffffffffu, m2, o);
          top2_merge(m1, m2, p1, p2);
        }
        if (lane == 0) gsc_s[warp][g] = use_top2 ? m1 + m2 : m1;
      }
    }
    __syncwarp();
    float g0 = lane < a.G ? gsc_s[warp][lane] : -INFINITY;
    float g1 = lane + 32 < a.G ? gsc_s[warp][lane + 32] : -INFINITY;
    keep = 0;
    for (int r = 0; r < a.TG; ++r) {
      float bv = -INFINITY;
      int bi = INT32_MAX;
      if (lane < a.G && !((keep >> lane) & 1ull)) { bv = g0; bi = lane; }
      if (lane + 32 < a.G && !((keep >> (lane + 32)) & 1ull) && better(g1, lane + 32, bv, bi)) {
        bv = g1; bi = lane + 32;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        float pv = __shfl_xor_sync(0xffffffffu, bv, o);
        int pi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (better(pv, pi, bv, bi)) { bv = pv; bi = pi; }
      }
      keep |= 1ull << bi;
    }
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int e = v * 32 + lane;
      if (e < E && !((keep >> (e / per)) & 1ull)) b[v] = -INFINITY;
    }
  }

  // 5. expert top-k over the kept groups, descending, ties to the lower index
  uint32_t taken = 0;
  int my_idx = -1;
  float my_s = 0.f;
  for (int j = 0; j < a.k; ++j) {
    float bv = -INFINITY, bs = 0.f;
    int bi = INT32_MAX;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      int e = v * 32 + lane;
      if (e < E && !((taken >> v) & 1u) && better(b[v], e, bv, bi)) { bv = b[v]; bi = e; bs = s[v]; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      float pv = __shfl_xor_sync(0xffffffffu, bv, o);
      int pi = __shfl_xor_sync(0xffffffffu, bi, o);
      float ps = __shfl_xor_sync(0xffffffffu, bs, o);
      if (better(pv, pi, bv, bi)) { bv = pv; bi = pi; bs = ps; }
    }
    if (lane == (bi & 31)) taken |= 1u << (bi >> 5);
    if (lane == j) { my_idx = bi; my_s = bs; }
  }

  // 6. weights: unbiased scores, renormalised over the picks for sigmoid
  float w = my_s;
  if (a.sigmoid) {
    float sum = lane < a.k ? my_s : 0.f;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    w = my_s / sum;
  }
  w *= a.route_scale;
  if (lane < a.k) {
    a.idx[t * a.k + lane] = my_idx;
    a.weights[t * a.k + lane] = w;
  }
}

}  // namespace

cudaError_t launch_router(const moe_config& c, int64_t T, const void* x, const void* w_router,
                          const float* bias, float* weights, int32_t* idx, float* part,
                          int splits, bool simt, int num_sms, uint32_t* err_word,
                          cudaStream_t st, bool hold_on_timeout) {
  const int E = c.n_routed, D = c.dim;
  cudaError_t err;
  if (c.dtype == MOE_DT_BF16 && !simt) {
    int used = 0;
    err = launch_router_logits_tc(c, T, x, w_router, part, router_tc_splits(c, T, splits, num_sms),
                                  err_word, st, &used);
    if (err != cudaSuccess) return err;
    splits = used;
  } else {
    const int kps = ceil_div(ceil_div(D, splits), RBK) * RBK;
    splits = ceil_div(D, kps);
    dim3 grid((unsigned)ceil_div<int64_t>(T, RBM), (unsigned)ceil_div(E, RBN), (unsigned)splits);
    if (c.dtype == MOE_DT_BF16)
      router_logits_kernel<__nv_bfloat16><<<grid, RTHREADS, 0, st>>>(
          (const __nv_bfloat16*)x, (const __nv_bfloat16*)w_router, T, E, D, kps, part);
    else
      router_logits_kernel<float><<<grid, RTHREADS, 0, st>>>((const float*)x,
                                                              (const float*)w_router, T, E, D, kps,
                                                              part);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  stage_mark(st);

  SelectArgs a;
  a.part = part;
  a.splits = splits;
  a.bias = c.has_bias ? bias : nullptr;
  a.T = T;
  a.E = E;
  a.G = c.n_groups;
  a.TG = c.topk_groups;
  a.k = c.topk;
  a.sigmoid = c.score == MOE_SCORE_SIGMOID;
  a.route_scale = c.route_scale;
  a.weights = weights;
  a.idx = idx;
  a.hold_on_timeout = hold_on_timeout ? err_word : nullptr;
  unsigned blocks = (unsigned)ceil_div<int64_t>(T, 8);
  int vpl = ceil_div(E, 32);
  const size_t zs = (size_t)8 * E * sizeof(float);
  void (*k)(const SelectArgs) = vpl <= 1    ? router_select_kernel<1>
                                : vpl <= 2  ? router_select_kernel<2>
                                : vpl <= 4  ? router_select_kernel<4>
                                : vpl <= 8  ? router_select_kernel<8>
                                : vpl <= 16 ? router_select_kernel<16>
                                            : router_select_kernel<32>;
  err = launch_pdl(pdl_ok(), k, dim3(blocks), dim3(256), zs, st, a);
  stage_mark(st);
  if (err != cudaSuccess) return err;
  return cudaGetLastError();
}

// ---------------------------------------------------------------- built-in scratch
//
// moe_gate_noalloc runs the router with its split-k partial sums in this
// file-scope device array instead of a caller workspace, for callers that
// cannot allocate device memory, and keeps its sticky error word (the timeout
// bit of a router pipeline wait that ran out) in a file-scope word beside it.
// Every GPU that loads the library holds both (4 MiB) until the process
// exits. Host code must not pass `g_gate_scratch` or `g_gate_err` itself to a
// kernel: on the host those names are only stand-ins; the device addresses
// come from cudaGetSymbolAddress, taken once per device.

namespace {
constexpr size_t kGateScratchFloats = size_t(1) << 20;
static __device__ __align__(256) float g_gate_scratch[kGateScratchFloats];
static __device__ __align__(16) uint32_t g_gate_err;

constexpr int kMaxDevices = 64;
std::mutex g_gate_scratch_mu;
float* g_gate_scratch_addr[kMaxDevices] = {};
uint32_t* g_gate_err_addr[kMaxDevices] = {};
}  // namespace

size_t gate_scratch_floats() { return kGateScratchFloats; }

// Device addresses of the built-in scratch and of its error word on the
// current device; looked up on the first call for each device (with that
// device current) and cached.
cudaError_t gate_scratch_current_device(float** scratch, uint32_t** err) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_gate_scratch_mu);
  if (!g_gate_scratch_addr[dev]) {
    float* ptr = nullptr;
    uint32_t* eptr = nullptr;
    e = cudaGetSymbolAddress((void**)&ptr, g_gate_scratch);
    if (e != cudaSuccess) return e;
    e = cudaGetSymbolAddress((void**)&eptr, g_gate_err);
    if (e != cudaSuccess) return e;
    g_gate_err_addr[dev] = eptr;
    g_gate_scratch_addr[dev] = ptr;
  }
  *scratch = g_gate_scratch_addr[dev];
  *err = g_gate_err_addr[dev];
  return cudaSuccess;
}

}  // namespace moe
