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
  Vec16<T> o;
  o.from_float(acc);
  reinterpret_cast<uint4*>(y + t * D)[v] = o.raw;
}

}  // namespace

cudaError_t launch_combine(const moe_config& c, int64_t T, const void* y_perm, const int32_t* pos,
                           const float* weights, const void* s, void* y, cudaStream_t st) {
  const int D = c.dim, k = c.topk;
  const int nvec = D * act_bytes(c) / 16;
  dim3 grid((unsigned)T, (unsigned)ceil_div(nvec, 256));
  if (c.dtype == MOE_DT_BF16)
    combine_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        (const __nv_bfloat16*)y_perm, pos, weights, (const __nv_bfloat16*)s, k, D, (__nv_bfloat16*)y);
  else
    combine_kernel<float><<<grid, 256, 0, st>>>((const float*)y_perm, pos, weights, (const float*)s,
                                                k, D, (float*)y);
  stage_mark(st);
  return cudaGetLastError();
}

}  // namespace moe
