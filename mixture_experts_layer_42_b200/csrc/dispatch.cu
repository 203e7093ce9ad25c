// Dispatch of the MoE layer (page "DeepSeek-V3.2-Exp - Weighted expert sum",
// MoE.forward: a bincount of the chosen indices, then, for each expert in
// ascending order, the rows routed to it in row-major order of idx).
//
// This builds the same order without a host round trip: a stable counting
// sort of the T*k (token, slot) pairs by expert.
//   dispatch_rank_kernel    one CTA per chunk of 64 tokens: per-warp ranks
//                           with __match_any_sync, then ranks within the chunk
//                           and the chunk's histogram.
//   dispatch_scan_kernel    one CTA: per-expert exclusive scan over chunks,
//                           counts, and the exclusive scan over experts
//                           (offsets).
//   dispatch_pos_kernel     grid over the T*k pairs: final positions (pos)
//                           and the token of every permuted row (src). The
//                           layer's expert GEMMs read x through src, so no
//                           permuted copy of x is made.
//   dispatch_scatter_kernel (only when a permuted copy is asked for) grid over
//                           (row slices, tokens): pos, src, and the copy of
//                           x[t] into its k permuted rows with 16-byte loads
//                           and stores (x is read once).
//   dispatch_small_kernel   small batches without a copy: all of the above in
//                           one CTA (one launch instead of three).
#include "common.cuh"

namespace moe {

namespace {

constexpr int DWARPS = 8;
constexpr int DMAX_ROUNDS = kDispatchChunkTokens * 32 / DWARPS / 32;  // k <= 32

__global__ void __launch_bounds__(DWARPS * 32)
dispatch_rank_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E,
                     int32_t* __restrict__ pos_local, int32_t* __restrict__ chunk_hist,
                     uint32_t* err) {
  extern __shared__ int32_t hist[];  // [DWARPS][E]
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < DWARPS * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();

  const int64_t q0 = (int64_t)blockIdx.x * kDispatchChunkTokens * k;
  const int64_t q1 = min((int64_t)(blockIdx.x + 1) * kDispatchChunkTokens, T) * k;
  const int64_t per_warp = ceil_div<int64_t>(ceil_div<int64_t>(q1 - q0, DWARPS), 32) * 32;
  const int64_t wq0 = q0 + warp * per_warp;
  const int rounds = (int)(per_warp / 32);
  const uint32_t lt_mask = (1u << lane) - 1u;

  int32_t rank[DMAX_ROUNDS];
  int32_t ex[DMAX_ROUNDS];
#pragma unroll
  for (int r = 0; r < DMAX_ROUNDS; ++r) {
    rank[r] = -1;
    ex[r] = -1;
    if (r >= rounds) continue;
    const int64_t q = wq0 + (int64_t)r * 32 + lane;
    int e = -2;  // past the chunk
    if (q < q1) {
      e = idx[q];
      if (e < 0 || e >= E) {
        set_error(err, ERRBIT_BAD_INDEX);
        e = -1;
      }
    }
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    int base = 0;
    if (e >= 0) base = hist[warp * E + e];
    __syncwarp();
    if (e >= 0) {
      if ((__ffs(same) - 1) == lane) hist[warp * E + e] = base + __popc(same);
      rank[r] = base + __popc(same & lt_mask);
      ex[r] = e;
    }
    __syncwarp();
  }
  __syncthreads();
  // exclusive scan over the warps of this chunk, per expert
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
#pragma unroll
    for (int w = 0; w < DWARPS; ++w) {
      int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    chunk_hist[(int64_t)blockIdx.x * E + e] = run;
  }
  __syncthreads();
#pragma unroll
  for (int r = 0; r < DMAX_ROUNDS; ++r) {
    if (r >= rounds) continue;
    const int64_t q = wq0 + (int64_t)r * 32 + lane;
    if (q < q1) pos_local[q] = ex[r] >= 0 ? rank[r] + hist[warp * E + ex[r]] : -1;
  }
}

__global__ void __launch_bounds__(1024)
dispatch_scan_kernel(int32_t* __restrict__ chunk_hist, int n_chunks, int E,
                     int32_t* __restrict__ counts, int32_t* __restrict__ offsets) {
  __shared__ int32_t wsum[32];
  const int e = threadIdx.x;  // E <= 1024
  int run = 0;
  if (e < E) {
    int c = 0;
    // 8 independent loads in flight per step
    for (; c + 8 <= n_chunks; c += 8) {
      int v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = chunk_hist[(int64_t)(c + u) * E + e];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        chunk_hist[(int64_t)(c + u) * E + e] = run;
        run += v[u];
      }
    }
    for (; c < n_chunks; ++c) {
      int v = chunk_hist[(int64_t)c * E + e];
      chunk_hist[(int64_t)c * E + e] = run;
      run += v;
    }
    counts[e] = run;
  }
  // exclusive scan of the counts over experts
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int p = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += p;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int p = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += p;
    }
    wsum[lane] = vi - v;
  }
  __syncthreads();
  const int excl = incl - run + wsum[warp];
  if (e < E) offsets[e] = excl;
  if (e == E - 1) offsets[E] = excl + run;
  __syncthreads();
  if (e < E)
    for (int c = 0; c < n_chunks; ++c) chunk_hist[(int64_t)c * E + e] += excl;
}

__global__ void __launch_bounds__(256)
dispatch_pos_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ pos_local,
                    const int32_t* __restrict__ chunk_base, int64_t Tk, int k, int E,
                    int32_t* __restrict__ pos, int32_t* __restrict__ src) {
  // a programmatic dependent launch (the up-projection) may start now; it
  // waits for this grid before it reads src
  asm volatile("griddepcontrol.launch_dependents;");
  const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (q >= Tk) return;
  const int64_t t = q / k;
  const int pl = pos_local[q];
  int p = -1;
  if (pl >= 0) p = chunk_base[(t / kDispatchChunkTokens) * E + idx[q]] + pl;
  pos[q] = p;
  if (p >= 0) src[p] = (int32_t)t;
}

// Grid (token, 4 KB slice of the row). Lets a programmatic dependent launch
// (the up-projection) start as soon as its last wave is running.
template <typename T>
__global__ void __launch_bounds__(256)
dispatch_scatter_kernel(const int32_t* __restrict__ idx, const int32_t* __restrict__ pos_local,
                        const int32_t* __restrict__ chunk_base, int k, int E, int D,
                        const T* __restrict__ x, int32_t* __restrict__ pos,
                        int32_t* __restrict__ src, T* __restrict__ x_perm) {
  asm volatile("griddepcontrol.launch_dependents;");
  __shared__ int32_t dst[32];
  const int64_t t = blockIdx.x;
  const int64_t chunk = t / kDispatchChunkTokens;
  if (threadIdx.x < k) {
    const int64_t q = t * k + threadIdx.x;
    const int pl = pos_local[q];
    int p = -1;
    if (pl >= 0) p = chunk_base[chunk * E + idx[q]] + pl;
    dst[threadIdx.x] = p;
    if (blockIdx.y == 0) {
      pos[q] = p;
      if (p >= 0) src[p] = (int32_t)t;
    }
  }
  __syncthreads();
  constexpr int VE = 16 / sizeof(T);
  const int nvec = D / VE;
  const int v = blockIdx.y * blockDim.x + threadIdx.x;
  if (v >= nvec) return;
  const uint4 val = reinterpret_cast<const uint4*>(x + t * D)[v];
  for (int j = 0; j < k; ++j) {
    const int p = dst[j];
    if (p >= 0) reinterpret_cast<uint4*>(x_perm + (int64_t)p * D)[v] = val;
  }
}

// Small batches (T*k <= kDispatchSmallPairs, E <= kDispatchSmallExperts, no
// permuted copy): the whole stable counting sort in one CTA of SW warps, the
// steps of the three kernels above in one launch. Warp w ranks the pairs
// [w * per_warp, (w + 1) * per_warp) in rounds of 32 (ranks within the warp
// by __match_any_sync, in pair order), an exclusive scan over the warps per
// expert and one over the experts give each pair its row.
constexpr int SW = 16;
__global__ void __launch_bounds__(SW * 32)
dispatch_small_kernel(const int32_t* __restrict__ idx, int64_t T, int k, int E,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      int32_t* __restrict__ pos, int32_t* __restrict__ src, uint32_t* err) {
  extern __shared__ int32_t hist[];  // [SW][E], then the expert offsets [E + 1]
  int32_t* eoff = hist + SW * E;
  __shared__ int32_t wsum[SW];
  // a programmatic dependent of the selection: the kernel after it may
  // launch now; idx is read after the selection's grid completes
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int i = threadIdx.x; i < SW * E; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const int64_t n = T * k;
  const int per_warp = (int)ceil_div<int64_t>(ceil_div<int64_t>(n, SW), 32) * 32;
  const int rounds = per_warp / 32;
  const uint32_t lt_mask = (1u << lane) - 1u;
  int rank[kDispatchSmallPairs / SW / 32];
  int ex[kDispatchSmallPairs / SW / 32];
#pragma unroll
  for (int r = 0; r < kDispatchSmallPairs / SW / 32; ++r) {
    rank[r] = -1;
    ex[r] = -1;
    if (r >= rounds) continue;
    const int64_t q = (int64_t)warp * per_warp + r * 32 + lane;
    int e = -2;  // past the pairs
    if (q < n) {
      e = idx[q];
      if (e < 0 || e >= E) {
        set_error(err, ERRBIT_BAD_INDEX);
        e = -1;
      }
    }
    const uint32_t same = __match_any_sync(0xffffffffu, e);
    int base = 0;
    if (e >= 0) base = hist[warp * E + e];
    __syncwarp();
    if (e >= 0) {
      if ((__ffs(same) - 1) == lane) hist[warp * E + e] = base + __popc(same);
      rank[r] = base + __popc(same & lt_mask);
      ex[r] = e;
    }
    __syncwarp();
  }
  __syncthreads();
  // per expert: exclusive scan over the warps, the count; then the exclusive
  // scan of the counts over the experts (E <= blockDim.x)
  const int e = threadIdx.x;
  int run = 0;
  if (e < E) {
#pragma unroll
    for (int w = 0; w < SW; ++w) {
      const int c = hist[w * E + e];
      hist[w * E + e] = run;
      run += c;
    }
    counts[e] = run;
  }
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int p = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += p;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int v = lane < SW ? wsum[lane] : 0;
    int vi = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int p = __shfl_up_sync(0xffffffffu, vi, o);
      if (lane >= o) vi += p;
    }
    if (lane < SW) wsum[lane] = vi - v;
  }
  __syncthreads();
  const int excl = incl - run + wsum[warp];
  if (e < E) {
    offsets[e] = excl;
    eoff[e] = excl;
  }
  if (e == E - 1) offsets[E] = excl + run;
  __syncthreads();
#pragma unroll
  for (int r = 0; r < kDispatchSmallPairs / SW / 32; ++r) {
    if (r >= rounds) continue;
    const int64_t q = (int64_t)warp * per_warp + r * 32 + lane;
    if (q >= n) continue;
    int p = -1;
    if (ex[r] >= 0) p = eoff[ex[r]] + hist[warp * E + ex[r]] + rank[r];
    pos[q] = p;
    if (p >= 0) src[p] = (int32_t)(q / k);
  }
}

}  // namespace

cudaError_t launch_dispatch_sort(const moe_config& c, int64_t T, const int32_t* idx,
                                 int32_t* counts, int32_t* offsets, int32_t* chunk_hist,
                                 int32_t* pos_local, int n_chunks, uint32_t* err, cudaStream_t st) {
  const int E = c.n_routed, k = c.topk;
  size_t smem = (size_t)DWARPS * E * sizeof(int32_t);
  dispatch_rank_kernel<<<n_chunks, DWARPS * 32, smem, st>>>(idx, T, k, E, pos_local, chunk_hist,
                                                           err);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  stage_mark(st);
  dispatch_scan_kernel<<<1, 1024, 0, st>>>(chunk_hist, n_chunks, E, counts, offsets);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  stage_mark(st);
  return cudaSuccess;
}

cudaError_t launch_dispatch_place(const DispatchPlace& p, cudaStream_t st) {
  const moe_config& c = *p.c;
  const int E = c.n_routed, k = c.topk, D = c.dim;
  if (p.x_perm == nullptr) {
    const int64_t Tk = p.T * k;
    dispatch_pos_kernel<<<(unsigned)ceil_div<int64_t>(Tk, 256), 256, 0, st>>>(
        p.idx, p.pos_local, p.chunk_hist, Tk, k, E, p.pos, p.src);
    stage_mark(st);
    return cudaGetLastError();
  }
  const int ab = act_bytes(c);
  const int nvec = D * ab / 16;
  dim3 grid((unsigned)p.T, (unsigned)ceil_div(nvec, 256));
  if (c.dtype == MOE_DT_BF16)
    dispatch_scatter_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(
        p.idx, p.pos_local, p.chunk_hist, k, E, D, (const __nv_bfloat16*)p.x, p.pos, p.src,
        (__nv_bfloat16*)p.x_perm);
  else
    dispatch_scatter_kernel<float><<<grid, 256, 0, st>>>(p.idx, p.pos_local, p.chunk_hist, k, E, D,
                                                         (const float*)p.x, p.pos, p.src,
                                                         (float*)p.x_perm);
  stage_mark(st);
  return cudaGetLastError();
}

bool dispatch_small_ok(const moe_config& c, int64_t T, const void* x_perm) {
  return x_perm == nullptr && T * c.topk <= kDispatchSmallPairs && c.n_routed <= kDispatchSmallExperts;
}

cudaError_t launch_dispatch_small(const moe_config& c, int64_t T, const int32_t* idx,
                                  int32_t* counts, int32_t* offsets, int32_t* pos, int32_t* src,
                                  uint32_t* err, cudaStream_t st) {
  const size_t smem = ((size_t)SW * c.n_routed + c.n_routed + 1) * sizeof(int32_t);
  return launch_pdl(pdl_ok(), dispatch_small_kernel, dim3(1), dim3(SW * 32), smem, st, idx, T,
                    c.topk, c.n_routed, counts, offsets, pos, src, err);
}

cudaError_t launch_dispatch(const moe_config& c, int64_t T, const int32_t* idx, const void* x,
                            int32_t* counts, int32_t* offsets, int32_t* src, int32_t* pos,
                            void* x_perm, int32_t* chunk_hist, int32_t* pos_local, int n_chunks,
                            uint32_t* err, cudaStream_t st) {
  if (dispatch_small_ok(c, T, x_perm)) {
    cudaError_t e = launch_dispatch_small(c, T, idx, counts, offsets, pos, src, err, st);
    for (int m = 0; m < 3; ++m) stage_mark(st);   // the timer's three dispatch intervals
    return e;
  }
  cudaError_t e =
      launch_dispatch_sort(c, T, idx, counts, offsets, chunk_hist, pos_local, n_chunks, err, st);
  if (e != cudaSuccess) return e;
  DispatchPlace p{&c, T, idx, x, chunk_hist, pos_local, pos, src, x_perm};
  return launch_dispatch_place(p, st);
}

}  // namespace moe
