// Grouped SwiGLU expert GEMMs on the CUDA cores (fp32 FMA).
//
// The experts of the layer (each Expert(dim, moe_inter_dim) plus the shared
// MLP; SwiGLU body E(x) = w2 (silu(w1 x) * (w3 x))) as two grouped launches:
//   UP:   h[r, n] = silu(sum_k A[r,k] w1[e,n,k]) * (sum_k A[r,k] w3[e,n,k])
//   DOWN: out[r, n] = sum_k h[r,k] w2[e,n,k]
// Group e owns rows [offsets[e], offsets[e+1]) of A (for UP, either an
// expert-contiguous copy of the token rows or the token rows themselves read
// through the dispatch's src); a last group, the shared expert, owns all T
// rows of its own A. Tiles of 64 rows x 64 columns; each
// CTA finds its group from the device offsets (no host round trip).
//
// This path serves the fp32 layer (tensor cores have no full-precision fp32
// product) and is a cross-check of the tensor-core kernel for bf16.
#include "common.cuh"

namespace moe {

namespace {

constexpr int SBM = 64, SBN = 64, SBK = 16, SPAD = 4;

__device__ __forceinline__ float silu_f(float u) { return u / (1.0f + expf(-u)); }

template <typename T, bool UP>
__global__ void __launch_bounds__(256) grouped_simt_kernel(const GroupedArgs g) {
  __shared__ int32_t P[1025];
  __shared__ int32_t wsum[8];
  __shared__ __align__(16) float As[SBK][SBM + SPAD];
  __shared__ __align__(16) float B1s[SBK][SBN + SPAD];
  __shared__ __align__(16) float B3s[UP ? SBK : 1][SBN + SPAD];
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int E = g.E;

  // m-tiles per expert and their exclusive prefix P[0..E]
  int loc[4], lsum = 0;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    int e = tid * 4 + u;
    loc[u] = e < E ? ceil_div(g.offsets[e + 1] - g.offsets[e], SBM) : 0;
    lsum += loc[u];
  }
  int incl = lsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int p = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += p;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  int wbase = 0;
  for (int w = 0; w < warp; ++w) wbase += wsum[w];
  int run = wbase + incl - lsum;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    int e = tid * 4 + u;
    if (e < E) P[e] = run;
    run += loc[u];
    if (e == E - 1) P[E] = run;
  }
  __syncthreads();

  const int mi = blockIdx.x;
  int kind, e = 0;
  int64_t row0, rows;
  if (mi < P[E]) {
    kind = 0;
    int lo = 0, hi = E;  // last e with P[e] <= mi
    while (hi - lo > 1) {
      int mid = (lo + hi) / 2;
      if (P[mid] <= mi) lo = mid; else hi = mid;
    }
    e = lo;
    const int m = mi - P[e];
    row0 = (int64_t)g.offsets[e] + (int64_t)m * SBM;
    rows = g.offsets[e + 1] - row0;
    if (rows > SBM) rows = SBM;
  } else {
    kind = 1;
    row0 = (int64_t)(mi - P[E]) * SBM;
    if (row0 >= g.t_shared) return;
    rows = g.t_shared - row0;
    if (rows > SBM) rows = SBM;
  }
  const int N = g.n[kind], K = g.kdim[kind];
  const int n0 = blockIdx.y * SBN;
  if (n0 >= N) return;
  const T* A = (const T*)g.a[kind];
  // row of A that holds row r of this group (gathered rows for routed UP)
  const int32_t* a_rows = (UP && kind == 0) ? g.a_rows : nullptr;
  auto arow = [&](int64_t r) -> int64_t { return a_rows ? (int64_t)a_rows[r] : r; };
  const T* B1 = (const T*)g.b1[kind] + (int64_t)e * N * K;
  const T* B3 = UP ? (const T*)g.b3[kind] + (int64_t)e * N * K : nullptr;
  T* out = (T*)g.out[kind];

  const int tm = tid / 16, tn = tid % 16;
  float acc1[4][4], acc3[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) { acc1[i][j] = 0.f; acc3[i][j] = 0.f; }

  for (int k0 = 0; k0 < K; k0 += SBK) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int i = tid + 256 * r;
      const int rr = i / SBK, kk = i % SBK;
      const int k = k0 + kk;
      As[kk][rr] = (rr < rows && k < K) ? to_f32(A[arow(row0 + rr) * K + k]) : 0.f;
      const int n = n0 + rr;
      B1s[kk][rr] = (n < N && k < K) ? to_f32(B1[(int64_t)n * K + k]) : 0.f;
      if (UP) B3s[kk][rr] = (n < N && k < K) ? to_f32(B3[(int64_t)n * K + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SBK; ++kk) {
      float4 av = *reinterpret_cast<const float4*>(&As[kk][tm * 4]);
      float4 bv = *reinterpret_cast<const float4*>(&B1s[kk][tn * 4]);
      float a[4] = {av.x, av.y, av.z, av.w}, b[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc1[i][j] = fmaf(a[i], b[j], acc1[i][j]);
      if (UP) {
        float4 cv = *reinterpret_cast<const float4*>(&B3s[kk][tn * 4]);
        float c[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc3[i][j] = fmaf(a[i], c[j], acc3[i][j]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int rr = tm * 4 + i;
    if (rr >= rows) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tn * 4 + j;
      if (n >= N) continue;
      const float v = UP ? silu_f(acc1[i][j]) * acc3[i][j] : acc1[i][j];
      out[(row0 + rr) * N + n] = from_f32<T>(v);
    }
  }
}

}  // namespace

cudaError_t launch_grouped_simt(const moe_config& c, int64_t T, bool up, const GroupedArgs& g,
                                cudaStream_t st) {
  const int64_t Tk = T * c.topk;
  const int64_t slots = ceil_div<int64_t>(Tk, SBM) + c.n_routed + ceil_div<int64_t>(g.t_shared, SBM);
  const int nmax = g.t_shared > 0 ? (g.n[0] > g.n[1] ? g.n[0] : g.n[1]) : g.n[0];
  dim3 grid((unsigned)slots, (unsigned)ceil_div(nmax, SBN));
  if (c.dtype == MOE_DT_BF16) {
    if (up) grouped_simt_kernel<__nv_bfloat16, true><<<grid, 256, 0, st>>>(g);
    else grouped_simt_kernel<__nv_bfloat16, false><<<grid, 256, 0, st>>>(g);
  } else {
    if (up) grouped_simt_kernel<float, true><<<grid, 256, 0, st>>>(g);
    else grouped_simt_kernel<float, false><<<grid, 256, 0, st>>>(g);
  }
  stage_mark(st);
  return cudaGetLastError();
}

}  // namespace moe
