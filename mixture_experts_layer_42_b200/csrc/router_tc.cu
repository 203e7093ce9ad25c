// Router logits of a bf16 layer on the tensor cores (page "DeepSeek-V3.2-Exp
// - Expert scores": z = x . W_r^T applied in float32).
//
// bf16 x bf16 products are exact in fp32; what must stay exact enough for
// routing (near-ties at 1e-6) is the summation over D = 7168. So each 64-deep
// k-block is accumulated by the tensor core into a fresh fp32 TMEM
// accumulator (4 MMAs, 64 products per sum), and the epilogue warps add every
// k-block's sums with Kahan's compensated summation in fp32 (sum plus a
// running correction): its error stays within a few ulps of the sum however
// many chunks are added, without fp64 work, at 4 additions per value (done
// two values at a time with the packed f32x2 adds of sm_100, each lane
// rounded exactly as a scalar add would be).
// The tensor core therefore never sums more than 64 products, and the result
// carries one fp32 rounding per split.
//
// Tile: 128 tokens x 64 experts; grid (token tiles, expert tiles, k splits).
// 192 threads: warp 0 TMA (x and W_r tiles, 128-byte swizzle, 4-stage ring),
// warp 1 tcgen05.mma (M128 N64 K16) into eight rotating 64-column TMEM
// buffers (each k-block's sums wait there for the epilogue, so the MMA runs
// up to eight k-blocks ahead), warps 2-5 tcgen05.ld + compensated accumulation, then the split's
// partial logits are written as fp32 [split, T, E]. Waits are bounded as in
// the expert GEMM kernel.
#include "tc_common.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int RM = 128, RN = 64, RK = 64, RSTAGES = 4;
constexpr int RA = RM * RK * 2;        // 16 KB x tile
constexpr int RB = RN * RK * 2;        // 8 KB W_r tile
constexpr int RSTAGE = RA + RB;
constexpr int RNBUF = 8;               // TMEM chunk buffers between the MMA and the epilogue
constexpr uint32_t RTMEM = RNBUF * RN; // 512 columns
constexpr size_t RSMEM = 1024 + (size_t)RSTAGES * RSTAGE + 256;
constexpr uint32_t RIDESC = idesc_bf16(RM, RN);

// Two fp32 lanes in one 64-bit register, for the packed (f32x2) adds of the
// compensated summation: each lane is rounded to nearest like a scalar add.
__device__ __forceinline__ uint64_t pack2(uint32_t lo, uint32_t hi) {
  uint64_t v;
  asm("mov.b64 %0, {%1, %2};" : "=l"(v) : "r"(lo), "r"(hi));
  return v;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ float2 unpack2(uint64_t v) {
  uint32_t lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(lo), "=r"(hi) : "l"(v));
  return make_float2(__uint_as_float(lo), __uint_as_float(hi));
}

struct RouterTcArgs {
  CUtensorMap tmx;   // x [T, D]
  CUtensorMap tmw;   // W_r [E, D]
  float* part;       // [splits, T, E]
  int64_t T;
  int E;
  int kb_total;
  int kb_per_split;
  // Test hook (moe_debug_stall_pipeline): the first CTA's MMA thread first
  // waits on a barrier phase that nothing completes, so that wait runs out
  // (1 s) and the launch takes its abort path.
  int stall;
  uint32_t* err;
};

__global__ void __launch_bounds__(192, 1) router_tc_kernel(const __grid_constant__ RouterTcArgs g) {
  // the selection, a programmatic dependent of this kernel, may launch now
  // (it waits for this grid before it reads the logits)
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + RSTAGES * RSTAGE);
  uint64_t* empty = full + RSTAGES;
  uint64_t* tfull = empty + RSTAGES;
  uint64_t* tempty = tfull + RNBUF;
  uint64_t* drain = tempty + RNBUF;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int m0 = blockIdx.x * RM;
  const int n0 = blockIdx.y * RN;
  const int split = blockIdx.z;
  const int kb0 = split * g.kb_per_split;
  const int kb1 = min(g.kb_total, kb0 + g.kb_per_split);
  const int nkb = kb1 - kb0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < RSTAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < RNBUF; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 128); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(RTMEM));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int kb = kb0; kb < kb1; ++kb) {
        if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, g.err)) { ok = false; break; }
        uint8_t* sa = tiles + s * RSTAGE;
        mbar_expect_tx(&full[s], RSTAGE);
        tma_load_2d(sa, &g.tmx, &full[s], kb * RK, m0);
        tma_load_2d(sa + RA, &g.tmw, &full[s], kb * RK, n0);
        ++issued;
        if (++s == RSTAGES) { s = 0; ph ^= 1; }
      }
      if (!ok)
        for (int j = 0; j < RSTAGES; ++j) {
          const int n = issued / RSTAGES + (j < issued % RSTAGES ? 1 : 0);
          if (n > 0) mbar_drain(&full[j], (uint32_t)((n - 1) & 1));
        }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      // test hook: the drain barrier is committed only after the loop
      const bool first = blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0;
      const bool ok = !(g.stall && first && !mbar_wait(drain, 0, abort_flag, g.err));
      for (int i = 0; ok && i < nkb; ++i) {
        const int b = i % RNBUF;
        const uint32_t use = (uint32_t)(i / RNBUF);
        if (!mbar_wait(&tempty[b], (use & 1) ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        if (!mbar_wait(&full[s], ph, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(tiles + s * RSTAGE);
        const uint32_t b0 = a0 + RA;
        const uint32_t d = tmem_base + (uint32_t)(b * RN);
#pragma unroll
        for (int kk = 0; kk < RK / 16; ++kk)
          tc_mma(d, sdesc(a0 + kk * 32), sdesc(b0 + kk * 32), RIDESC, kk != 0 ? 1u : 0u);
        tc_commit(&empty[s]);
        tc_commit(&tfull[b]);
        if (++s == RSTAGES) { s = 0; ph ^= 1; }
      }
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    // Kahan sums of the 64 expert columns, two columns per packed register
    uint64_t hi[RN / 2], lo[RN / 2];
#pragma unroll
    for (int j = 0; j < RN / 2; ++j) hi[j] = lo[j] = 0ull;
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
      const int b = i % RNBUF;
      const uint32_t use = (uint32_t)(i / RNBUF);
      int w = 1;
      if (lane == 0) w = mbar_wait(&tfull[b], use & 1, abort_flag, g.err) ? 1 : 0;
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w) { ok = false; break; }
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * RN);
      uint32_t r[RN];
      tmem_ld16(tb + 0, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
      tmem_ld16(tb + 16, *reinterpret_cast<uint32_t(*)[16]>(&r[16]));
      tmem_ld16(tb + 32, *reinterpret_cast<uint32_t(*)[16]>(&r[32]));
      tmem_ld16(tb + 48, *reinterpret_cast<uint32_t(*)[16]>(&r[48]));
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(&tempty[b]);
#pragma unroll
      for (int j = 0; j < RN / 2; ++j) {  // Kahan: hi = running sum, lo = -(lost low part)
        const uint64_t y = sub2(pack2(r[2 * j], r[2 * j + 1]), lo[j]);
        const uint64_t t = add2(hi[j], y);
        lo[j] = sub2(sub2(t, hi[j]), y);
        hi[j] = t;
      }
    }
    const int64_t t = (int64_t)m0 + row;
    if (ok && t < g.T) {
      float* out = g.part + ((int64_t)split * g.T + t) * g.E + n0;
      const int nvalid = min(RN, g.E - n0);
      if (nvalid == RN && (g.E & 3) == 0) {
#pragma unroll
        for (int j = 0; j < RN / 2; j += 2) {
          const float2 a = unpack2(sub2(hi[j], lo[j])), b = unpack2(sub2(hi[j + 1], lo[j + 1]));
          *reinterpret_cast<float4*>(out + 2 * j) = make_float4(a.x, a.y, b.x, b.y);
        }
      } else {
#pragma unroll
        for (int j = 0; j < RN / 2; ++j) {
          const float2 a = unpack2(sub2(hi[j], lo[j]));
          if (2 * j < nvalid) out[2 * j] = a.x;
          if (2 * j + 1 < nvalid) out[2 * j + 1] = a.y;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(RTMEM));
  }
}

}  // namespace

// Splits of the k range for T tokens: about 32 CTAs for small batches --
// the partial sums of every split are written out and summed again by the
// select kernel, so more splits cost more than they hide -- at most
// `max_splits`, at least 8 k-blocks per split.
int router_tc_splits(const moe_config& c, int64_t T, int max_splits, int num_sms) {
  (void)num_sms;
  const int64_t tiles = ceil_div<int64_t>(T, RM) * ceil_div<int64_t>(c.n_routed, RN);
  const int kbt = ceil_div(c.dim, RK);
  int64_t s = ceil_div<int64_t>(32, tiles);
  if (s > kbt / 8) s = kbt / 8;
  if (s > max_splits) s = max_splits;
  if (s < 1) s = 1;
  return (int)s;
}

cudaError_t launch_router_logits_tc(const moe_config& c, int64_t T, const void* x,
                                    const void* w_router, float* part, int splits, uint32_t* err,
                                    cudaStream_t st, int* splits_used) {
  RouterTcArgs g;
  memset(&g, 0, sizeof(g));
  if (!map_2d(&g.tmx, x, (uint64_t)T, (uint64_t)c.dim, RM)) return cudaErrorInvalidValue;
  if (!map_2d(&g.tmw, w_router, (uint64_t)c.n_routed, (uint64_t)c.dim, RN))
    return cudaErrorInvalidValue;
  g.part = part;
  g.T = T;
  g.E = c.n_routed;
  g.kb_total = ceil_div(c.dim, RK);
  g.kb_per_split = ceil_div(g.kb_total, splits);
  g.stall = pipeline_stall() == STALL_ROUTER ? 1 : 0;
  g.err = err;
  const int used = ceil_div(g.kb_total, g.kb_per_split);  // every split gets >= 1 k-block
  *splits_used = used;
  dim3 grid((unsigned)ceil_div<int64_t>(T, RM), (unsigned)ceil_div(c.n_routed, RN), (unsigned)used);
  cudaError_t e = cudaFuncSetAttribute(router_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)RSMEM);
  if (e != cudaSuccess) return e;
  router_tc_kernel<<<grid, 192, RSMEM, st>>>(g);
  return cudaGetLastError();
}

}  // namespace moe
