// Grouped SwiGLU expert GEMMs on the 5th-generation tensor cores (sm_100a).
//
// The experts of the layer (each Expert(dim, moe_inter_dim) and the shared
// MLP of width n_shared_experts * moe_inter_dim; SwiGLU body
// E(x) = w2 (silu(w1 x) * (w3 x))) as two persistent grouped launches:
//   UP:   h[r, f]  = silu(A[r,:] . w1[e,f,:]) * (A[r,:] . w3[e,f,:])   (bf16 out)
//   DOWN: out[r,n] = h[r,:] . w2[e,n,:]                                (bf16 out)
// Group e owns rows [offsets[e], offsets[e+1]) of the expert-contiguous A;
// the shared expert is one more group that owns all T rows of its own A.
//
// One CTA per SM, 192 threads, warp-specialised:
//   warp 0      TMA producer: A tile 128x64 and B tile 256x64 (bf16, 128-byte
//               swizzle) per stage into a 4-stage shared-memory ring.
//   warp 1      MMA issuer: tcgen05.mma kind::f16, M=128 N=256 K=16, fp32
//               accumulator in TMEM (two 256-column buffers so the epilogue of
//               one tile overlaps the main loop of the next).
//   warps 2-5   epilogue: tcgen05.ld of the accumulator rows (TMEM lane =
//               tile row), silu(a)*b for UP, rounding to bf16, masked stores.
// For UP the N=256 B tile stacks 128 rows of w1 over the same 128 rows of w3,
// so accumulator columns j and 128+j hold a and b of the same feature.
//
// Tiles are enumerated from the device offsets (no host round trip): expert
// by expert, n-tile outer and m-tile inner so that CTAs running at the same
// time share weight tiles and A rows in L2. Every pipeline wait is bounded
// (1 s); on expiry the kernel raises the timeout bit of the error word, drains
// what it has in flight, frees TMEM and returns.
#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {

struct TcArgs {
  CUtensorMap tmA[2];   // [0] routed A rows, [1] shared A rows; 2D {K, rows}
  CUtensorMap tmB1[2];  // w1 (UP) / w2 (DOWN) as 3D {K, N, E}; shared: E = 1
  CUtensorMap tmB3[2];  // w3 / ws3 (UP only)
  void* out[2];
  int n_out[2];         // output columns: UP I / I_s, DOWN D / D
  int kdim[2];          // reduction depth: UP D / D, DOWN I / I_s
  const int32_t* offsets;
  int E;
  int t_shared;         // rows of the shared group (0: none)
  uint32_t* err;
};

namespace {

constexpr int BM = 128;
constexpr int BK = 64;                     // one 128-byte swizzled row of bf16
constexpr int BN = 256;                    // MMA N
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BK * 2;        // 16 KB
constexpr int B_TILE = BN * BK * 2;        // 32 KB
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;   // 1 s
constexpr uint64_t DRAIN_LIMIT_NS = 20000000ull;    // 20 ms
constexpr int MAX_E = 1024;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + 2 * (MAX_E + 1) * 4;

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, N = 256, M = 128.
constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                           ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `bar` with the given parity. Gives up when another
// role has raised the abort flag, or after WAIT_LIMIT_NS (then raises it).
__device__ __noinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                       uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer() - t0 > WAIT_LIMIT_NS) {
      *abort_flag = 1;
      set_error(err, ERRBIT_TIMEOUT);
      return false;
    }
  }
}

// Bounded wait used only while draining after an abort.
__device__ __noinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait(bar, parity))
    if (globaltimer() - t0 > DRAIN_LIMIT_NS) return;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(IDESC), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct Tile {
  int kind;   // 0 routed, 1 shared
  int e;      // expert (0 for shared)
  int row0;   // first A row
  int rows;   // valid rows (<= BM)
  int n0;     // first output column
};

struct Sched {
  const int32_t* P;    // smem: m-tile prefix over experts [E + 1]
  const int32_t* off;  // smem: offsets [E + 1]
  int E, nt0, nt1, mt_sh, routed, total, t_shared, bn_out;
};

__device__ __forceinline__ Tile decode(const Sched& S, int i) {
  Tile t;
  if (i < S.routed) {
    const int q = i / S.nt0;
    int lo = 0, hi = S.E;  // the e with P[e] <= q < P[e+1]
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (S.P[mid] <= q) lo = mid; else hi = mid;
    }
    const int e = lo;
    const int mt = S.P[e + 1] - S.P[e];
    const int l = i - S.nt0 * S.P[e];
    const int nt = l / mt, m = l % mt;
    t.kind = 0;
    t.e = e;
    t.row0 = S.off[e] + m * BM;
    t.rows = min(BM, S.off[e + 1] - t.row0);
    t.n0 = nt * S.bn_out;
  } else {
    const int l = i - S.routed;
    const int nt = l / S.mt_sh, m = l % S.mt_sh;
    t.kind = 1;
    t.e = 0;
    t.row0 = m * BM;
    t.rows = min(BM, S.t_shared - t.row0);
    t.n0 = nt * S.bn_out;
  }
  return t;
}

__device__ __forceinline__ float silu_fast(float u) { return u / (1.0f + __expf(-u)); }

template <bool UP>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_tc_kernel(const __grid_constant__ TcArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* tiles = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* P = reinterpret_cast<int32_t*>(tiles + STAGES * STAGE_BYTES + 256);
  int32_t* off = P + MAX_E + 1;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int E = g.E;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
      for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 128); }
      mbar_init(drain, 1);
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // m-tiles per expert and their exclusive prefix
    const int per = (E + 31) / 32;
    int lsum = 0;
    for (int u = 0; u < per; ++u) {
      const int e = lane * per + u;
      if (e < E) {
        const int o0 = g.offsets[e], o1 = g.offsets[e + 1];
        off[e] = o0;
        if (e == E - 1) off[E] = o1;
        lsum += (o1 - o0 + BM - 1) / BM;
      }
    }
    int incl = lsum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int p = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += p;
    }
    int run = incl - lsum;
    for (int u = 0; u < per; ++u) {
      const int e = lane * per + u;
      if (e < E) {
        P[e] = run;
        run += (g.offsets[e + 1] - g.offsets[e] + BM - 1) / BM;
      }
    }
    if (lane == 31) P[E] = incl;
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  Sched S;
  S.P = P;
  S.off = off;
  S.E = E;
  S.bn_out = UP ? BN / 2 : BN;
  S.nt0 = (g.n_out[0] + S.bn_out - 1) / S.bn_out;
  S.nt1 = g.t_shared > 0 ? (g.n_out[1] + S.bn_out - 1) / S.bn_out : 0;
  S.mt_sh = (g.t_shared + BM - 1) / BM;
  S.t_shared = g.t_shared;
  S.routed = S.nt0 * P[E];
  S.total = S.routed + S.nt1 * S.mt_sh;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < S.total; i += gridDim.x) {
        const Tile t = decode(S, i);
        const int kb_n = (g.kdim[t.kind] + BK - 1) / BK;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, g.err)) { ok = false; break; }
          uint8_t* sa = tiles + s * STAGE_BYTES;
          uint8_t* sb = sa + A_TILE;
          mbar_expect_tx(&full[s], STAGE_BYTES);
          tma_load_2d(sa, &g.tmA[t.kind], &full[s], kb * BK, t.row0);
          if (UP) {
            tma_load_3d(sb, &g.tmB1[t.kind], &full[s], kb * BK, t.n0, t.e);
            tma_load_3d(sb + B_TILE / 2, &g.tmB3[t.kind], &full[s], kb * BK, t.n0, t.e);
          } else {
            tma_load_3d(sb, &g.tmB1[t.kind], &full[s], kb * BK, t.n0, t.e);
          }
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      if (!ok) {
        // let every copy still in flight land before the CTA exits
        for (int j = 0; j < STAGES; ++j) {
          const int n = issued / STAGES + (j < issued % STAGES ? 1 : 0);
          if (n > 0) mbar_drain(&full[j], (uint32_t)((n - 1) & 1));
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0, lt = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = blockIdx.x; ok && i < S.total; i += gridDim.x, ++lt) {
        const Tile t = decode(S, i);
        const int kb_n = (g.kdim[t.kind] + BK - 1) / BK;
        const int acc = lt & 1;
        const uint32_t use = (uint32_t)(lt >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(tiles + s * STAGE_BYTES);
          const uint32_t b0 = a0 + A_TILE;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma(d, sdesc(a0 + kk * 32), sdesc(b0 + kk * 32), (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);
      }
      // all MMAs issued by this thread complete before TMEM is released
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;           // TMEM lanes 32*quad .. 32*quad+31
    const int row = quad * 32 + lane;
    int lt = 0;
    for (int i = blockIdx.x; i < S.total; i += gridDim.x, ++lt) {
      const Tile t = decode(S, i);
      const int acc = lt & 1;
      const uint32_t use = (uint32_t)(lt >> 1);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], use & 1, abort_flag, g.err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      const bool valid = row < t.rows;
      const int n_out = g.n_out[t.kind];
      __nv_bfloat16* out =
          reinterpret_cast<__nv_bfloat16*>(g.out[t.kind]) + (int64_t)(t.row0 + row) * n_out + t.n0;
      if (UP) {
#pragma unroll 1
        for (int j = 0; j < BN / 2; j += 16) {
          uint32_t ra[16], rb[16];
          tmem_ld16(tb + j, ra);
          tmem_ld16(tb + BN / 2 + j, rb);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float h0 = silu_fast(__uint_as_float(ra[2 * q])) * __uint_as_float(rb[2 * q]);
            const float h1 =
                silu_fast(__uint_as_float(ra[2 * q + 1])) * __uint_as_float(rb[2 * q + 1]);
            __nv_bfloat162 v = __floats2bfloat162_rn(h0, h1);
            pk[q] = *reinterpret_cast<uint32_t*>(&v);
          }
          if (valid) {
            if (t.n0 + j + 8 <= n_out)
              *reinterpret_cast<uint4*>(out + j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (t.n0 + j + 16 <= n_out)
              *reinterpret_cast<uint4*>(out + j + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
#pragma unroll 1
        for (int j = 0; j < BN; j += 16) {
          uint32_t ra[16];
          tmem_ld16(tb + j, ra);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            __nv_bfloat162 v =
                __floats2bfloat162_rn(__uint_as_float(ra[2 * q]), __uint_as_float(ra[2 * q + 1]));
            pk[q] = *reinterpret_cast<uint32_t*>(&v);
          }
          if (valid) {
            if (t.n0 + j + 8 <= n_out)
              *reinterpret_cast<uint4*>(out + j) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (t.n0 + j + 16 <= n_out)
              *reinterpret_cast<uint4*>(out + j + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 map over a row-major [rows, K] matrix, box 64 (K) x 128 rows.
bool map_rows(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {BK, BM};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map over stacked weights [E, N, K], box 64 (K) x box_n x 1.
bool map_weights(CUtensorMap* m, const void* ptr, uint64_t E, uint64_t N, uint64_t K,
                 uint32_t box_n) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {K, N, E};
  cuuint64_t strides[2] = {K * 2, N * K * 2};
  cuuint32_t box[3] = {BK, box_n, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

// A: routed rows [Tk, K0] and shared rows [T, K1]; B1/B3 stacked [E, N0, K0]
// and shared [N1, K1]; outputs [Tk, N0] and [T, N1].
cudaError_t launch_grouped_tc(bool up, int64_t Tk, int64_t T_sh, int E, const void* a0,
                              const void* a1, const void* b1_0, const void* b3_0, const void* b1_1,
                              const void* b3_1, int n0, int k0, int n1, int k1, void* out0,
                              void* out1, const int32_t* offsets, uint32_t* err, int num_sms,
                              cudaStream_t st) {
  TcArgs g;
  memset(&g, 0, sizeof(g));
  const uint32_t box_n = up ? BN / 2 : BN;
  const bool has_sh = T_sh > 0;
  if (!map_rows(&g.tmA[0], a0, (uint64_t)Tk, (uint64_t)k0)) return cudaErrorInvalidValue;
  if (!map_weights(&g.tmB1[0], b1_0, (uint64_t)E, (uint64_t)n0, (uint64_t)k0, box_n))
    return cudaErrorInvalidValue;
  if (up && !map_weights(&g.tmB3[0], b3_0, (uint64_t)E, (uint64_t)n0, (uint64_t)k0, box_n))
    return cudaErrorInvalidValue;
  if (has_sh) {
    if (!map_rows(&g.tmA[1], a1, (uint64_t)T_sh, (uint64_t)k1)) return cudaErrorInvalidValue;
    if (!map_weights(&g.tmB1[1], b1_1, 1, (uint64_t)n1, (uint64_t)k1, box_n))
      return cudaErrorInvalidValue;
    if (up && !map_weights(&g.tmB3[1], b3_1, 1, (uint64_t)n1, (uint64_t)k1, box_n))
      return cudaErrorInvalidValue;
  } else {
    g.tmA[1] = g.tmA[0];
    g.tmB1[1] = g.tmB1[0];
    g.tmB3[1] = g.tmB3[0];
  }
  if (!up) g.tmB3[0] = g.tmB1[0], g.tmB3[1] = g.tmB1[1];
  g.out[0] = out0;
  g.out[1] = has_sh ? out1 : out0;
  g.n_out[0] = n0;
  g.n_out[1] = has_sh ? n1 : n0;
  g.kdim[0] = k0;
  g.kdim[1] = has_sh ? k1 : k0;
  g.offsets = offsets;
  g.E = E;
  g.t_shared = has_sh ? (int)T_sh : 0;
  g.err = err;

  const int bn_out = up ? BN / 2 : BN;
  const int64_t nt0 = (n0 + bn_out - 1) / bn_out;
  const int64_t bound = nt0 * ((Tk + BM - 1) / BM + E) +
                        (has_sh ? (int64_t)((n1 + bn_out - 1) / bn_out) * ((T_sh + BM - 1) / BM) : 0);
  const int grid = (int)(bound < num_sms ? bound : num_sms);
  if (grid <= 0) {
    stage_mark(st);
    return cudaSuccess;
  }
  cudaError_t e;
  if (up) {
    e = cudaFuncSetAttribute(grouped_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    grouped_tc_kernel<true><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(g);
  } else {
    e = cudaFuncSetAttribute(grouped_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    grouped_tc_kernel<false><<<grid, NUM_THREADS, SMEM_BYTES, st>>>(g);
  }
  stage_mark(st);
  return cudaGetLastError();
}

}  // namespace moe
