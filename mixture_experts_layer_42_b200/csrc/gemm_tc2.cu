// Grouped SwiGLU expert GEMMs on CTA pairs (tcgen05 cta_group::2), for
// batches with many rows per expert (prefill).
//
// Same layer math and tile order as the one-CTA kernel (gemm_tc.cu), with a
// tile of up to 256 rows computed by a cluster of two CTAs on neighbouring
// SMs:
//   * each CTA's TMA warp loads its share of A and its 128-row half of the
//     N=256 B tile into its own 6-stage ring (UP: rank r loads rows
//     [n0 + 64 r, n0 + 64 r + 64) of w1 and the same rows of w3, so every
//     half holds a and b of the same 64 features; DOWN: rank r loads output
//     columns [n0 + 128 r, n0 + 128 r + 128)). Both CTAs' copies signal the
//     leader's (rank 0) "full" barrier; no load is multicast.
//   * the leader's MMA thread issues tcgen05.mma.cta_group::2 K=16, N=256:
//       - M=256 while more than 128 rows of the tile are valid: each CTA
//         holds 128 A rows and its TMEM lane l = tile row 128 r + l, with
//         columns 0-255 = the N columns;
//       - M=128 for an expert's last chunk of at most 128 rows (its padding is
//         then that of 128-row tiles): each CTA holds 64 A rows; TMEM lanes
//         0-63 hold those rows against N columns 0-127 (the leader's B half),
//         lanes 64-127 the same rows against N columns 128-255, both in TMEM
//         columns 0-127.
//     M=128 on a pair runs at nearly the M=256 rate per FLOP (unlike M=64 on
//     one CTA, which runs at half rate). Commits are multicast to both CTAs.
//   * each CTA's epilogue warps drain their own TMEM lanes (silu(a)*b for UP)
//     and arrive on the leader's accumulator-free barrier.
// Per CTA a stage is 32 KB instead of 48 KB for the same MMA work, so six
// stages fit, and each B byte is read once per 256 rows instead of 128.
#include "tc_common.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int PBM = 256;                   // rows per pair tile
constexpr int HBM = 128;                   // rows per CTA
constexpr int BK = 64;
constexpr int BN = 256;                    // MMA N
constexpr int HBN = 128;                   // B rows per CTA
constexpr int STAGES = 6;
constexpr int A_HALF = HBM * BK * 2;       // 16 KB
constexpr int B_HALF = HBN * BK * 2;       // 16 KB
constexpr int STAGE_BYTES = A_HALF + B_HALF;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_E = 1024;
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + 2 * (MAX_E + 1) * 4;
constexpr uint32_t IDESC = idesc_bf16(PBM, BN);       // full chunk: 256 rows
constexpr uint32_t IDESC_TAIL = idesc_bf16(HBM, BN);  // last chunk of <= 128 rows
constexpr int A_TAIL = HBM / 2 * BK * 2;              // 8 KB: 64 A rows per CTA

struct Tile {
  int kind, e, row0, rows, n0;
};

struct Sched {
  const int32_t* P;
  const int32_t* off;
  int E, nt0, nt1, mt_sh, routed, total, t_shared, bn_out;
};

__device__ __forceinline__ Tile decode(const Sched& S, int i) {
  Tile t;
  if (i < S.routed) {
    const int q = i / S.nt0;
    int lo = 0, hi = S.E;
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
    t.row0 = S.off[e] + m * PBM;
    t.rows = min(PBM, S.off[e + 1] - t.row0);
    t.n0 = nt * S.bn_out;
  } else {
    const int l = i - S.routed;
    const int nt = l / S.mt_sh, m = l % S.mt_sh;
    t.kind = 1;
    t.e = 0;
    t.row0 = m * PBM;
    t.rows = min(PBM, S.t_shared - t.row0);
    t.n0 = nt * S.bn_out;
  }
  return t;
}

__device__ __forceinline__ float silu_fast(float u) { return u / (1.0f + __expf(-u)); }

template <bool UP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NUM_THREADS, 1)
    grouped_tc2_kernel(const __grid_constant__ TcArgs g) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
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
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int E = g.E;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
      // tempty: one arrive per epilogue warp of both CTAs (used on the leader)
      for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 8); }
      mbar_init(drain, 1);
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    const int per = (E + 31) / 32;
    int lsum = 0;
    for (int u = 0; u < per; ++u) {
      const int e = lane * per + u;
      if (e < E) {
        const int o0 = g.offsets[e], o1 = g.offsets[e + 1];
        off[e] = o0;
        if (e == E - 1) off[E] = o1;
        lsum += (o1 - o0 + PBM - 1) / PBM;
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
        run += (g.offsets[e + 1] - g.offsets[e] + PBM - 1) / PBM;
      }
    }
    if (lane == 31) P[E] = incl;
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  Sched S;
  S.P = P;
  S.off = off;
  S.E = E;
  S.bn_out = UP ? BN / 2 : BN;
  S.nt0 = (g.n_out[0] + S.bn_out - 1) / S.bn_out;
  S.nt1 = g.t_shared > 0 ? (g.n_out[1] + S.bn_out - 1) / S.bn_out : 0;
  S.mt_sh = (g.t_shared + PBM - 1) / PBM;
  S.t_shared = g.t_shared;
  S.routed = S.nt0 * P[E];
  S.total = S.routed + S.nt1 * S.mt_sh;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer (both CTAs)
    if (lane == 0) {
      int s = 0, issued = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = pair; ok && i < S.total; i += npairs) {
        const Tile t = decode(S, i);
        const int kb_n = (g.kdim[t.kind] + BK - 1) / BK;
        const bool tail = t.rows <= HBM;
        const CUtensorMap* ta = tail ? &g.tmA64[t.kind] : &g.tmA[t.kind];
        const int arow = t.row0 + (int)rank * (tail ? HBM / 2 : HBM);
        const uint32_t tx = 2u * (uint32_t)((tail ? A_TAIL : A_HALF) + B_HALF);
        // UP: w1 and w3 rows [n0 + 64 r, +64); DOWN: output columns [n0 + 128 r, +128)
        const int brow = UP ? t.n0 + (int)rank * (HBN / 2) : t.n0 + (int)rank * HBN;
        const int b13 = UP ? g.b13[t.kind] : 0;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&empty[s], ph ^ 1, abort_flag, g.err)) { ok = false; break; }
          uint8_t* sa = tiles + s * STAGE_BYTES;
          const uint32_t fb = mapa(smem_u32(&full[s]), 0);
          if (leader) mbar_expect_tx(&full[s], tx);
          tma2_load_2d(sa, ta, fb, kb * BK, arow);
          if (!UP) {
            tma2_load_3d(sa + A_HALF, &g.tmB1[t.kind], fb, kb * BK, brow, t.e);
          } else if (b13 != 0) {
            tma2_load_4d(sa + A_HALF, &g.tmB13[t.kind], fb, kb * BK, brow, t.e, 0);
          } else {
            tma2_load_3d(sa + A_HALF, &g.tmB1[t.kind], fb, kb * BK, brow, t.e);
            tma2_load_3d(sa + A_HALF + B_HALF / 2, &g.tmB3[t.kind], fb, kb * BK, brow, t.e);
          }
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
      }
      if (!ok && leader)
        for (int j = 0; j < STAGES; ++j) {
          const int n = issued / STAGES + (j < issued % STAGES ? 1 : 0);
          if (n > 0) mbar_drain(&full[j], (uint32_t)((n - 1) & 1));
        }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader)
    if (leader && lane == 0) {
      int s = 0, lt = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int i = pair; ok && i < S.total; i += npairs, ++lt) {
        const Tile t = decode(S, i);
        const int kb_n = (g.kdim[t.kind] + BK - 1) / BK;
        const uint32_t idesc = t.rows <= HBM ? IDESC_TAIL : IDESC;
        const int acc = lt & 1;
        const uint32_t use = (uint32_t)(lt >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(tiles + s * STAGE_BYTES);
          const uint32_t b0 = a0 + A_HALF;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_pair(d, sdesc(a0 + kk * 32), sdesc(b0 + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
          commit_pair(&empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        commit_pair(&tfull[acc]);
      }
      commit_pair(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t tempty_leader0 = mapa(smem_u32(&tempty[0]), 0);
    const uint32_t tempty_leader1 = mapa(smem_u32(&tempty[1]), 0);
    int lt = 0;
    for (int i = pair; i < S.total; i += npairs, ++lt) {
      const Tile t = decode(S, i);
      const int acc = lt & 1;
      const uint32_t use = (uint32_t)(lt >> 1);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], use & 1, abort_flag, g.err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(acc * BN);
      const bool tail = t.rows <= HBM;
      // tile row held by this lane, and the first N column of its TMEM column 0
      const int my_row = tail ? (int)rank * (HBM / 2) + (row & (HBM / 2 - 1)) : (int)rank * HBM + row;
      const int ncol0 = tail ? (row / (HBM / 2)) * (BN / 2) : 0;
      const int ncols = tail ? BN / 2 : BN;  // TMEM columns holding this lane's results (DOWN)
      const bool valid = my_row < t.rows;
      const int n_out = g.n_out[t.kind];
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out[t.kind]) +
                           (int64_t)(t.row0 + my_row) * n_out + t.n0;
      if (UP) {
        // every 128 N columns hold 64 features: 64 w1 rows, then the same 64
        // w3 rows (b13 = 2: w3 first). Full chunk: 128 features in TMEM
        // columns 0-255; tail: this lane's 64 features in columns 0-127.
        const int ca = g.b13[t.kind] == 2 ? BN / 4 : 0;
        const int cb = BN / 4 - ca;
        const int nfeat = tail ? BN / 4 : BN / 2;
        const int f0 = ncol0 / 2;
#pragma unroll 1
        for (int u = 0; u < nfeat; u += 16) {
          const int f = f0 + u;                       // feature offset from n0
          const int col = (u / (BN / 4)) * (BN / 2) + (u % (BN / 4));
          uint32_t ra[16], rb[16];
          tmem_ld16(tb + col + ca, ra);
          tmem_ld16(tb + col + cb, rb);
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
            if (t.n0 + f + 8 <= n_out)
              *reinterpret_cast<uint4*>(out + f) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (t.n0 + f + 16 <= n_out)
              *reinterpret_cast<uint4*>(out + f + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      } else {
#pragma unroll 1
        for (int c = 0; c < ncols; c += 16) {
          uint32_t ra[16];
          tmem_ld16(tb + c, ra);
          tmem_wait_ld();
          uint32_t pk[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            __nv_bfloat162 v =
                __floats2bfloat162_rn(__uint_as_float(ra[2 * q]), __uint_as_float(ra[2 * q + 1]));
            pk[q] = *reinterpret_cast<uint32_t*>(&v);
          }
          const int n = ncol0 + c;
          if (valid) {
            if (t.n0 + n + 8 <= n_out)
              *reinterpret_cast<uint4*>(out + n) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            if (t.n0 + n + 16 <= n_out)
              *reinterpret_cast<uint4*>(out + n + 8) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no remote arrive or MMA into this CTA is still pending
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(TMEM_COLS));
  }
}

}  // namespace

namespace tc {

// Launch the pair kernel on `pairs` clusters of two CTAs.
cudaError_t launch_grouped_tc2(bool up, const TcArgs& g, int pairs, cudaStream_t st) {
  cudaError_t e;
  if (up) {
    e = cudaFuncSetAttribute(grouped_tc2_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    grouped_tc2_kernel<true><<<2 * pairs, NUM_THREADS, SMEM_BYTES, st>>>(g);
  } else {
    e = cudaFuncSetAttribute(grouped_tc2_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    grouped_tc2_kernel<false><<<2 * pairs, NUM_THREADS, SMEM_BYTES, st>>>(g);
  }
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace moe
