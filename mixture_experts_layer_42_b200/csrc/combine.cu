// Weighted combine of the MoE layer (page "DeepSeek-V3.2-Exp - Weighted
// expert sum": y_routed = sum_i G_i E_i, accumulated in float32 and cast back
// at the end, then the shared expert added to every token).
//
// One thread per 16-byte column slice of one token: gathers the k expert
// output rows of the token from y_perm (through pos), scales by the routing
// weights, adds the shared-expert row, all in fp32, and rounds once.
#include "common.cuh"

namespace moe {

namespace {

template <typename T>
__global__ void __launch_bounds__(256)
combine_kernel(const T* __restrict__ y_perm, const int32_t* __restrict__ pos,
               const float* __restrict__ weights, const T* __restrict__ s, int k, int D,
               T* __restrict__ y) {
  __shared__ int32_t p_s[32];
  __shared__ float w_s[32];
  // a programmatic dependent of the down-projection: its outputs are read
  // after that grid completes
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    p_s[threadIdx.x] = pos[t * k + threadIdx.x];
    w_s[threadIdx.x] = weights[t * k + threadIdx.x];
  }
  __syncthreads();
  constexpr int VE = 16 / sizeof(T);
  const int v = blockIdx.y * blockDim.x + threadIdx.x;
  if (v >= D / VE) return;
  float acc[VE];
#pragma unroll
  for (int q = 0; q < VE; ++q) acc[q] = 0.f;
  // the token's rows, 8 at a time: all loads issued before the first add
  // (more bytes in flight per thread), then added in slot order
  for (int j0 = 0; j0 < k; j0 += 8) {
    uint4 raw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int p = j0 + u < k ? p_s[j0 + u] : -1;
      raw[u] = p >= 0 ? reinterpret_cast<const uint4*>(y_perm + (int64_t)p * D)[v]
                      : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (j0 + u >= k || p_s[j0 + u] < 0) continue;
      Vec16<T> r;
      r.raw = raw[u];
      float f[VE];
      r.to_float(f);
      const float w = w_s[j0 + u];
#pragma unroll
      for (int q = 0; q < VE; ++q) acc[q] = fmaf(w, f[q], acc[q]);
    }
  }
  if (s) {
    Vec16<T> r;
    r.raw = reinterpret_cast<const uint4*>(s + t * D)[v];
    float f[VE];
    r.to_float(f);
#pragma unroll
    for (int q = 0; q < VE; ++q) acc[q] += f[q];
  }
  Vec16<T> o;
  o.from_float(acc);
  reinterpret_cast<uint4*>(y + t * D)[v] = o.raw;
}

// One expert-parallel rank's share of y, before the sum over ranks: the same
// gather-scale-accumulate as combine_kernel over the pairs whose permuted row
// lies in this rank's expert block [offsets[0], offsets[n_local]) (the
// offsets pointer starts at the block's first expert), plus this rank's slice
// of the shared MLP, left in fp32 (the sum over ranks is taken in fp32 and
// cast once by cast_kernel).
template <typename T>
__global__ void __launch_bounds__(256)
combine_partial_kernel(const T* __restrict__ y_perm, const int32_t* __restrict__ pos,
                       const float* __restrict__ weights, const T* __restrict__ s,
                       const int32_t* __restrict__ offsets_local, int n_local, int k, int D,
                       float* __restrict__ y) {
  __shared__ int32_t p_s[32];
  __shared__ float w_s[32];
  asm volatile("griddepcontrol.wait;" ::: "memory");   // as combine_kernel
  const int64_t t = blockIdx.x;
  if (threadIdx.x < k) {
    const int lo = offsets_local[0], hi = offsets_local[n_local];
    const int p = pos[t * k + threadIdx.x];
    p_s[threadIdx.x] = (p >= lo && p < hi) ? p : -1;
    w_s[threadIdx.x] = weights[t * k + threadIdx.x];
  }
  __syncthreads();
  constexpr int VE = 16 / sizeof(T);
  const int v = blockIdx.y * blockDim.x + threadIdx.x;
  if (v >= D / VE) return;
  float acc[VE];
#pragma unroll
  for (int q = 0; q < VE; ++q) acc[q] = 0.f;
  for (int j = 0; j < k; ++j) {
    const int p = p_s[j];
    if (p < 0) continue;
    Vec16<T> r;
    r.raw = reinterpret_cast<const uint4*>(y_perm + (int64_t)p * D)[v];
    float f[VE];
    r.to_float(f);
    const float w = w_s[j];
#pragma unroll
    for (int q = 0; q < VE; ++q) acc[q] = fmaf(w, f[q], acc[q]);
  }
  if (s) {
    Vec16<T> r;
    r.raw = reinterpret_cast<const uint4*>(s + t * D)[v];
    float f[VE];
    r.to_float(f);
#pragma unroll
    for (int q = 0; q < VE; ++q) acc[q] += f[q];
  }
  float4* out = reinterpret_cast<float4*>(y + t * D + (int64_t)v * VE);
#pragma unroll
  for (int q = 0; q < VE; q += 4) out[q / 4] = make_float4(acc[q], acc[q + 1], acc[q + 2], acc[q + 3]);
}

// y = act(y32), one rounding per element; one 16-byte output vector per
// thread (8 bf16 or 4 fp32 elements).
template <typename T>
__global__ void __launch_bounds__(256) cast_kernel(const float* __restrict__ y32, int64_t nvec,
                                                   T* __restrict__ y) {
  constexpr int VE = 16 / sizeof(T);
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nvec) return;
  float f[VE];
#pragma unroll
  for (int q = 0; q < VE; q += 4) {
    const float4 a = reinterpret_cast<const float4*>(y32 + i * VE)[q / 4];
    f[q] = a.x; f[q + 1] = a.y; f[q + 2] = a.z; f[q + 3] = a.w;
  }
  Vec16<T> o;
  o.from_float(f);
  reinterpret_cast<uint4*>(y)[i] = o.raw;
}

}  // namespace

cudaError_t launch_combine_partial(const moe_config& c, int64_t T, const void* y_perm,
                                   const int32_t* pos, const float* weights, const void* s,
                                   const int32_t* offsets_local, int n_local, float* y32,
                                   cudaStream_t st) {
  const int D = c.dim, k = c.topk;
  const int nvec = D * act_bytes(c) / 16;
  dim3 grid((unsigned)T, (unsigned)ceil_div(nvec, 256));
  if (c.dtype == MOE_DT_BF16)
    return launch_pdl(pdl_ok(), combine_partial_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                      (const __nv_bfloat16*)y_perm, pos, weights, (const __nv_bfloat16*)s,
                      offsets_local, n_local, k, D, y32);
  return launch_pdl(pdl_ok(), combine_partial_kernel<float>, grid, dim3(256), 0, st,
                    (const float*)y_perm, pos, weights, (const float*)s, offsets_local, n_local, k,
                    D, y32);
}

cudaError_t launch_cast(const moe_config& c, int64_t T, const float* y32, void* y, cudaStream_t st) {
  // dim is a multiple of 16 bytes of act (checked with the config)
  const int64_t nvec = T * c.dim * act_bytes(c) / 16;
  const unsigned blocks = (unsigned)ceil_div<int64_t>(nvec, 256);
  if (c.dtype == MOE_DT_BF16)
    cast_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(y32, nvec, (__nv_bfloat16*)y);
  else
    cast_kernel<float><<<blocks, 256, 0, st>>>(y32, nvec, (float*)y);
  return cudaGetLastError();
}

cudaError_t launch_combine(const moe_config& c, int64_t T, const void* y_perm, const int32_t* pos,
                           const float* weights, const void* s, void* y, cudaStream_t st) {
  const int D = c.dim, k = c.topk;
  const int nvec = D * act_bytes(c) / 16;
  dim3 grid((unsigned)T, (unsigned)ceil_div(nvec, 256));
  cudaError_t e;
  if (c.dtype == MOE_DT_BF16)
    e = launch_pdl(pdl_ok(), combine_kernel<__nv_bfloat16>, grid, dim3(256), 0, st,
                   (const __nv_bfloat16*)y_perm, pos, weights, (const __nv_bfloat16*)s, k, D,
                   (__nv_bfloat16*)y);
  else
    e = launch_pdl(pdl_ok(), combine_kernel<float>, grid, dim3(256), 0, st, (const float*)y_perm,
                   pos, weights, (const float*)s, k, D, (float*)y);
  stage_mark(st);
  return e;
}

}  // namespace moe
