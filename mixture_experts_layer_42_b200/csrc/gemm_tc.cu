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
// For UP the N=256 B tile stacks 128 rows of w1 over the same 128 rows of w3
// (one 4D TMA box over both tensors when their distance allows, else two
// boxes), so accumulator columns j and 128+j hold a and b of the same feature.
//
// The up-projection's routed A rows come either from an expert-contiguous
// copy of x (one tile load per stage) or straight from x through the
// dispatch's src (tile::gather4: each lane of the TMA warp brings 4 rows, 32
// copies per 128-row stage). The gathers bound a 128-row stage by the TMA's
// copy rate, so the layer gathers only for decode-sized batches, whose
// experts run one swapped tile of a few rows (see below).
//
// An expert's last, partial m-tile loads its A rows through a copy of the A
// tensor map whose row extent ends at the expert's last row (one per expert,
// written by build_row_maps_kernel before the launch): TMA fills the rows
// past it with zeros instead of the next expert's rows. Gathered rows past
// the expert get an out-of-range row and read zeros too. The results are the
// same (those rows are never stored), but zero operands draw less power, and
// under the board's power cap that buys clock.
//
// Tiles are enumerated from the device offsets (no host round trip): expert
// by expert, n-tile outer and m-tile inner so that CTAs running at the same
// time share weight tiles and A rows in L2. The up-projection hands tiles out
// in that order from a launch-wide counter (the TMA thread claims one and
// passes its index to the MMA and epilogue warps through a small mbarrier
// queue), which keeps the CTAs that share data starting together; the
// down-projection assigns them round-robin by CTA. Every pipeline wait is bounded
// (1 s); on expiry the kernel raises the timeout bit of the error word, drains
// what it has in flight, frees TMEM and returns.
#include "fp8_common.cuh"

namespace moe {

namespace {

using namespace tc;

constexpr int BM = 128;
constexpr int BK = 64;                     // one 128-byte swizzled row of bf16
constexpr int BN = 256;                    // MMA N
constexpr int STAGES = 4;
constexpr int A_TILE = BM * BK * 2;        // 16 KB
constexpr int B_TILE = BN * BK * 2;        // 32 KB
constexpr int STAGE_BYTES = A_TILE + B_TILE;
constexpr int NUM_THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr int MAX_E = 1024;
constexpr int TQ = 4;                      // tile queue depth (dynamic schedule)
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 256 + 2 * (MAX_E + 1) * 4;

constexpr uint32_t IDESC = tc::idesc_bf16(BM, BN);

struct Tile {
  int kind;   // 0 routed, 1 shared
  int e;      // expert (0 for shared)
  int row0;   // first A row
  int rows;   // valid rows (<= BM)
  int n0;     // first output column
  bool only;  // the expert's only m-tile
};

struct Sched {
  const int32_t* P;    // smem: m-tile prefix over experts [E + 1]
  const int32_t* off;  // smem: offsets [E + 1]
  int E, nt0, nt1, mt_sh, routed, total, t_shared, bn_out;
};

// Tile i: the shared expert's tiles first, then the routed experts' tiles.
__device__ __forceinline__ Tile decode(const Sched& S, int i) {
  Tile t;
  const int n_sh = S.total - S.routed;
  if (i >= n_sh) {
    i -= n_sh;
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
    t.only = mt == 1;
  } else {
    const int l = i;
    const int nt = l / S.mt_sh, m = l % S.mt_sh;
    t.kind = 1;
    t.e = 0;
    t.row0 = m * BM;
    t.rows = min(BM, S.t_shared - t.row0);
    t.n0 = nt * S.bn_out;
    t.only = false;
  }
  return t;
}

// Slot and phase parity of the shared-memory tile queue, kept by each role
// that reads or writes it.
struct TileQueue {
  int q = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void advance() {
    if (++q == TQ) { q = 0; ph ^= 1; }
  }
};

// The tile of an expert with at most SWAP_ROWS rows (its only tile; routed,
// row maps built) runs with the operands swapped: the 128 weight rows of each
// half of the B tile are the MMA's M side and the tile's r token rows,
// rounded up to r16, its N side. The token box of that expert's row map is
// r16 rows high, so the stage carries r16 token rows instead of 128, and the
// MMAs do r16 columns of work instead of 128 padded rows. At decode batch
// sizes (a few rows per expert) this removes most of the tensor work and its
// power, and the SM clock rises under the power cap (2.33 -> 2.17 ms per V3
// decode step). Experts with several m-tiles keep the plain form for their
// last tile: their m-tiles stream the same weight tiles side by side and
// share them in L2, which holds only while every m-tile runs at the same pace
// (a swapped tile drifts out of step and re-reads its weights from HBM).
// Single tiles of more than SWAP_ROWS rows also stay plain: swapping them
// measured slower at prefill.
constexpr int SWAP_ROWS = 64;
__device__ __forceinline__ bool swap_tail(const Tile& t, const TcArgs& g) {
  return t.kind == 0 && t.only && t.rows <= SWAP_ROWS && (g.row_maps != nullptr || g.src != nullptr);
}
__device__ __forceinline__ int tail_n(int rows) { return (rows + 15) & ~15; }

__device__ __forceinline__ float silu_fast(float u) { return u / (1.0f + __expf(-u)); }

template <bool UP>
__global__ void __launch_bounds__(NUM_THREADS, 1) grouped_tc_kernel(const __grid_constant__ TcArgs g) {
  // DOWN: the combine after it may launch now (it waits for this grid
  // before it reads the outputs). UP lets the down-projection launch only
  // after its own prologue (below), once it has waited for its predecessors.
  if (!UP) asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* tiles = base;
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + STAGES * STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* qfull = drain + 1;            // tile queue: index written
  uint64_t* qempty = qfull + TQ;          //             index read by the MMA and 4 epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(qempty + TQ);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* tq = reinterpret_cast<volatile int*>(tmem_slot + 2);  // [TQ] tile indices
  int32_t* P = reinterpret_cast<int32_t*>(tiles + STAGES * STAGE_BYTES + 256);
  int32_t* off = P + MAX_E + 1;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int E = g.E;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
      for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 128); }
      for (int q = 0; q < TQ; ++q) { mbar_init(&qfull[q], 1); mbar_init(&qempty[q], 1 + 4); }
      mbar_init(drain, 1);
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // UP, launched as a programmatic dependent of the kernel before it (the
    // dispatch or the row-map kernel), may be running before that one
    // completes: it waits for it before anything it wrote is read (the
    // offsets here; src, the row maps and the tile counter after the
    // __syncthreads below). The wait returns at once for an ordinary launch.
    // DOWN, a programmatic dependent of the up-projection, reads here only
    // what was complete before that grid let it launch (the offsets; later
    // the row maps); it waits for h in its producer, after prefetching its
    // first weight tiles.
    if (UP) asm volatile("griddepcontrol.wait;" ::: "memory");
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
  // UP: every thread of the CTA is past the wait for the kernels before it,
  // so a dependent down-projection may read what they wrote (the offsets,
  // the row maps) before it waits for this grid
  if (UP) asm volatile("griddepcontrol.launch_dependents;");

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
    // Lane 0 claims tiles, waits for free stages and loads B (and A, when A
    // is loaded by tile). When the routed A rows are gathered from the token
    // rows, every lane brings 4 of the tile's rows per stage (tile::gather4):
    // lane l rows 4l..4l+3.
    int s = 0, issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    TileQueue Q;
    const bool dyn = g.tile_ctr != nullptr;
    if (!UP) {
      // the first tile's leading weight k-blocks into L2 while the
      // up-projection finishes, then wait for it (h)
      if (lane == 0 && (int)blockIdx.x < S.total) {
        const Tile t0 = decode(S, blockIdx.x);
        const int kb_n = (g.kdim[t0.kind] + BK - 1) / BK;
        const int n_pf = min(kb_n, DOWN_PREFETCH_KB_BYTES / B_TILE);
        for (int kb = 0; kb < n_pf; ++kb) tma_prefetch_3d(&g.tmB1[t0.kind], kb * BK, t0.n0, t0.e);
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    // the next tile is claimed a few k-blocks before the current one ends,
    // so the atomic's round trip overlaps the current tile's loads
    int next = 0;
    if (lane == 0) next = dyn ? atomicAdd(g.tile_ctr, 1) : (int)blockIdx.x;
    next = __shfl_sync(0xffffffffu, next, 0);
    for (;;) {
      const int i = next;
      if (dyn) {
        // hand the tile's index to the MMA and epilogue warps
        int w = 1;
        if (lane == 0) {
          w = mbar_wait(&qempty[Q.q], Q.ph ^ 1, abort_flag, g.err) ? 1 : 0;
          if (w) {
            tq[Q.q] = i;
            mbar_arrive(&qfull[Q.q]);
          }
        }
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        Q.advance();
      } else {
        next = i + (int)gridDim.x;
      }
      if (i >= S.total) break;
      const Tile t = decode(S, i);
      const int kb_n = (g.kdim[t.kind] + BK - 1) / BK;
      const int kb_claim = kb_n > 4 ? kb_n - 4 : 0;
      const bool swap = swap_tail(t, g);
      // an expert's last, partial tile reads zeros past its rows, not the
      // next expert's; a swapped tile's box is only tail_n(rows) rows high
      const CUtensorMap* ta = &g.tmA[t.kind];
      uint32_t tx = STAGE_BYTES;
      if (swap) tx = (uint32_t)(tail_n(t.rows) * BK * 2 + B_TILE);
      const bool gath = UP && t.kind == 0 && g.src != nullptr;
      int gr0 = 0, gr1 = 0, gr2 = 0, gr3 = 0, n_g = 0;
      if (gath) {
        // this lane's four rows: their tokens, or the out-of-range row gT
        // (zeros) past the expert's end
        n_g = (swap ? tail_n(t.rows) : BM) / 4;
        const int r = 4 * lane;
        gr0 = r + 0 < t.rows ? g.src[t.row0 + r + 0] : g.gT;
        gr1 = r + 1 < t.rows ? g.src[t.row0 + r + 1] : g.gT;
        gr2 = r + 2 < t.rows ? g.src[t.row0 + r + 2] : g.gT;
        gr3 = r + 3 < t.rows ? g.src[t.row0 + r + 3] : g.gT;
      } else if (t.kind == 0 && t.rows < BM && g.row_maps != nullptr) {
        ta = g.row_maps + t.e;
        if (lane == 0) tmap_acquire(ta);
      }
      for (int kb = 0; kb < kb_n; ++kb) {
        int w = 1;
        if (lane == 0) {
          if (dyn && kb == kb_claim) next = atomicAdd(g.tile_ctr, 1);
          w = mbar_wait(&empty[s], ph ^ 1, abort_flag, g.err) ? 1 : 0;
        }
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        uint8_t* sa = tiles + s * STAGE_BYTES;
        uint8_t* sb = sa + A_TILE;
        if (lane == 0) {
          mbar_expect_tx(&full[s], tx);
          if (!gath) tma_load_2d(sa, ta, &full[s], kb * BK, t.row0);
          if (UP && g.b13[t.kind]) {
            tma_load_4d(sb, &g.tmB13[t.kind], &full[s], kb * BK, t.n0, t.e, 0);
          } else if (UP) {
            tma_load_3d(sb, &g.tmB1[t.kind], &full[s], kb * BK, t.n0, t.e);
            tma_load_3d(sb + B_TILE / 2, &g.tmB3[t.kind], &full[s], kb * BK, t.n0, t.e);
          } else {
            tma_load_3d(sb, &g.tmB1[t.kind], &full[s], kb * BK, t.n0, t.e);
          }
        }
        __syncwarp();
        if (gath && lane < n_g)
          tma_gather4(sa + lane * (4 * BK * 2), &g.tmG, &full[s], kb * BK, gr0, gr1, gr2, gr3);
        ++issued;
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      if (dyn) next = __shfl_sync(0xffffffffu, next, 0);
    }
    if (!ok && lane == 0) {
      // let every copy still in flight land before the CTA exits
      for (int j = 0; j < STAGES; ++j) {
        const int n = issued / STAGES + (j < issued % STAGES ? 1 : 0);
        if (n > 0) mbar_drain(&full[j], (uint32_t)((n - 1) & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      TileQueue Q;
      // test hook: a wait that runs out (the drain barrier is committed only
      // after the tile loop), before any MMA is issued
      if (g.stall && blockIdx.x == 0 && !mbar_wait(drain, 0, abort_flag, g.err)) ok = false;
      for (int lt = 0; ok; ++lt) {
        int i;
        if (g.tile_ctr != nullptr) {
          if (!mbar_wait(&qfull[Q.q], Q.ph, abort_flag, g.err)) break;
          i = tq[Q.q];
          mbar_arrive(&qempty[Q.q]);
          Q.advance();
        } else {
          i = blockIdx.x + lt * gridDim.x;
        }
        if (i >= S.total) break;
        const Tile t = decode(S, i);
        const int kb_n = (g.kdim[t.kind] + BK - 1) / BK;
        const int acc = lt & 1;
        const uint32_t use = (uint32_t)(lt >> 1);
        if (!mbar_wait(&tempty[acc], (use & 1) ^ 1, abort_flag, g.err)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(acc * BN);
        const bool swap = swap_tail(t, g);
        // swapped tail: w1 (UP) or w2 rows 0-127 (DOWN) into TMEM columns
        // [0, r16), w3 or w2 rows 128-255 into [128, 128 + r16)
        const uint32_t idesc_t = idesc_bf16(BM, tail_n(t.rows));
        const uint32_t w_lo = (UP && g.b13[t.kind] == 2) ? B_TILE / 2 : 0, w_hi = B_TILE / 2 - w_lo;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(tiles + s * STAGE_BYTES);
          const uint32_t b0 = a0 + A_TILE;
          if (swap) {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk) {
              const uint32_t acc_flag = (kb | kk) != 0 ? 1u : 0u;
              tc_mma(d, sdesc(b0 + w_lo + kk * 32), sdesc(a0 + kk * 32), idesc_t, acc_flag);
              tc_mma(d + BN / 2, sdesc(b0 + w_hi + kk * 32), sdesc(a0 + kk * 32), idesc_t, acc_flag);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < BK / 16; ++kk)
              tc_mma(d, sdesc(a0 + kk * 32), sdesc(b0 + kk * 32), IDESC, (kb | kk) != 0 ? 1u : 0u);
          }
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
    TileQueue Q;
    for (int lt = 0;; ++lt) {
      int i;
      if (g.tile_ctr != nullptr) {
        int w = 1;
        i = 0;
        if (lane == 0) {
          w = mbar_wait(&qfull[Q.q], Q.ph, abort_flag, g.err) ? 1 : 0;
          if (w) {
            i = tq[Q.q];
            mbar_arrive(&qempty[Q.q]);
          }
        }
        w = __shfl_sync(0xffffffffu, w, 0);
        i = __shfl_sync(0xffffffffu, i, 0);
        if (!w) break;
        Q.advance();
      } else {
        i = blockIdx.x + lt * gridDim.x;
      }
      if (i >= S.total) break;
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
      if (swap_tail(t, g)) {
        // TMEM lane = output feature, column = token row of the tile
        const int rn = tail_n(t.rows);
        __nv_bfloat16* base = reinterpret_cast<__nv_bfloat16*>(g.out[t.kind]) + (int64_t)t.row0 * n_out;
        if (UP) {
          const int f = t.n0 + row;            // this lane's feature
#pragma unroll 1
          for (int j = 0; j < rn; j += 16) {
            uint32_t ra[16], rb[16];
            tmem_ld16(tb + j, ra);
            tmem_ld16(tb + BN / 2 + j, rb);
            tmem_wait_ld();
            if (f < n_out) {
#pragma unroll
              for (int q = 0; q < 16; ++q)
                if (j + q < t.rows)
                  base[(int64_t)(j + q) * n_out + f] = __float2bfloat16_rn(
                      silu_fast(__uint_as_float(ra[q])) * __uint_as_float(rb[q]));
            }
          }
        } else {
#pragma unroll 1
          for (int half = 0; half < 2; ++half) {
            const int f = t.n0 + half * (BN / 2) + row;
#pragma unroll 1
            for (int j = 0; j < rn; j += 16) {
              uint32_t ra[16];
              tmem_ld16(tb + half * (BN / 2) + j, ra);
              tmem_wait_ld();
              if (f < n_out) {
#pragma unroll
                for (int q = 0; q < 16; ++q)
                  if (j + q < t.rows)
                    base[(int64_t)(j + q) * n_out + f] = __float2bfloat16_rn(__uint_as_float(ra[q]));
              }
            }
          }
        }
      } else if (UP) {
        // accumulator columns of w1 (a) and w3 (b): w3 first when its tile
        // came first in the paired load
        const uint32_t ca = g.b13[t.kind] == 2 ? BN / 2 : 0, cb = BN / 2 - ca;
#pragma unroll 1
        for (int j = 0; j < BN / 2; j += 16) {
          uint32_t ra[16], rb[16];
          tmem_ld16(tb + ca + j, ra);
          tmem_ld16(tb + cb + j, rb);
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

// Per-expert copies of an A map with the row extent cut at the expert's end:
// one warp per expert edits a copy in shared memory and publishes it to
// global memory with a release fence for the tensor-map proxy. blockIdx.y
// selects the map: 0 the down-projection's (rows of h), 1 the
// up-projection's (rows of the expert-contiguous copy of x; not launched when
// the up-projection gathers its rows from x).
struct RowMapArgs {
  CUtensorMap base[2];
  CUtensorMap* maps[2];
};

__global__ void __launch_bounds__(256) build_row_maps_kernel(const __grid_constant__ RowMapArgs a,
                                                             const int32_t* __restrict__ offsets,
                                                             int E, int* tile_ctr, int swap_boxes) {
  // the up-projection, a programmatic dependent of this kernel when the
  // dispatch ran before it, may start now (it waits for this grid before its
  // routed tiles); this kernel is itself a programmatic dependent of the
  // dispatch, whose offsets it reads after that grid completes
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ __align__(128) CUtensorMap sm[8];
  const int w = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int which = blockIdx.y;
  if (blockIdx.x == 0 && which == 0 && threadIdx.x == 0) *tile_ctr = 0;  // the up-projection's queue restarts
  const int e = blockIdx.x * 8 + w;
  if (e >= E) return;  // whole warps
  reinterpret_cast<uint32_t*>(&sm[w])[lane] = reinterpret_cast<const uint32_t*>(&a.base[which])[lane];
  __syncwarp();
  if (lane == 0) {
    const int end = offsets[e + 1];
    // an expert with at most SWAP_ROWS rows: its only tile runs swapped, with
    // a token box of tail_n(rows) rows; other experts keep BM-row boxes (all
    // of them do for the FP8 kernel, which swaps no tile)
    const int tail = swap_boxes && end - offsets[e] <= SWAP_ROWS ? end - offsets[e] : 0;
    asm volatile("tensormap.replace.tile.global_dim.shared::cta.b1024.b32 [%0], 1, %1;" ::"r"(
                     smem_u32(&sm[w])),
                 "r"(end > 0 ? end : 1)
                 : "memory");
    if (tail > 0)
      asm volatile("tensormap.replace.tile.box_dim.shared::cta.b1024.b32 [%0], 1, %1;" ::"r"(
                       smem_u32(&sm[w])),
                   "r"(tail_n(tail))
                   : "memory");
  }
  __syncwarp();
  asm volatile(
      "tensormap.cp_fenceproxy.global.shared::cta.tensormap::generic.release.gpu.sync.aligned [%0], "
      "[%1], 128;" ::"l"(a.maps[which] + e),
      "r"(smem_u32(&sm[w]))
      : "memory");
}

}  // namespace


// Test hook state (moe_debug_stall_pipeline).
static int g_stall = STALL_NONE;
void set_pipeline_stall(int which) { g_stall = which; }
int pipeline_stall() { return g_stall; }

cudaError_t launch_row_maps(const void* h, int64_t Tk, int I, const void* a_up, int D,
                            const int32_t* offsets, int E, void* maps, int* up_tile_ctr,
                            cudaStream_t st, bool fp8) {
  RowMapArgs a;
  memset(&a, 0, sizeof(a));
  // bf16 rows (box 64 x 128) for the one-CTA kernel, e4m3 rows (box
  // 128 x 128) for the FP8 token-on-M kernel
  auto map = [&](CUtensorMap* m, const void* p, int K) {
    return fp8 ? fp8::map_u8_tile(m, p, (uint64_t)Tk, (uint64_t)K, BM)
               : tc::map_2d(m, p, (uint64_t)Tk, (uint64_t)K, BM);
  };
  if (!map(&a.base[0], h, I)) return cudaErrorInvalidValue;
  a.maps[0] = static_cast<CUtensorMap*>(maps) + E;
  if (a_up != nullptr) {
    if (!map(&a.base[1], a_up, D)) return cudaErrorInvalidValue;
    a.maps[1] = static_cast<CUtensorMap*>(maps);
  }
  dim3 grid((unsigned)((E + 7) / 8), a_up != nullptr ? 2u : 1u);
  return launch_pdl(pdl_ok(), build_row_maps_kernel, grid, dim3(256), 0, st, a, offsets, E, up_tile_ctr,
                    fp8 ? 0 : 1);
}

// A: routed rows [Tk, K0] (or, for UP, the token rows gx [gT, K0] gathered
// through src) and shared rows [T_sh, K1]; B1/B3 stacked [E, N0, K0] and
// shared [N1, K1]; outputs [Tk, N0] and [T_sh, N1]. `kind` picks the kernel:
// TC_ROWS this one (128-row tiles), TC_PAIR the CTA-pair kernel (256-row
// tiles, gemm_tc2.cu; no gathering, row maps or tile counter).
cudaError_t launch_grouped_tc(bool up, int kind, int64_t Tk, int64_t T_sh, int E, const void* a0,
                              const void* a1, const void* b1_0, const void* b3_0, const void* b1_1,
                              const void* b3_1, int n0, int k0, int n1, int k1, void* out0,
                              void* out1, const int32_t* offsets, const void* gx,
                              const int32_t* src, int64_t gT, const void* row_maps, int* tile_ctr,
                              uint32_t* err, int num_sms, cudaStream_t st, bool pdl) {
  TcArgs g;
  memset(&g, 0, sizeof(g));
  const bool pair = kind == TC_PAIR;
  const bool gather = up && !pair && src != nullptr;
  if (!gather && a0 == nullptr) return cudaErrorInvalidValue;
  // Weight rows per TMA box: one CTA loads all 256 MMA rows of B (UP: 128 w1
  // + 128 w3); in a pair each CTA loads 128 (UP: 64 w1 + 64 w3).
  const uint32_t box_n = up ? (pair ? BN / 4 : BN / 2) : (pair ? BN / 2 : BN);
  const uint32_t box_a = BM;
  const bool has_sh = T_sh > 0;
  if (gather) {
    if (!tc::map_gather(&g.tmG, gx, (uint64_t)gT, (uint64_t)k0)) return cudaErrorInvalidValue;
    g.src = src;
    g.gT = (int)gT;
  } else {
    if (!tc::map_2d(&g.tmA[0], a0, (uint64_t)Tk, (uint64_t)k0, box_a)) return cudaErrorInvalidValue;
    if (pair && !tc::map_2d(&g.tmA64[0], a0, (uint64_t)Tk, (uint64_t)k0, box_a / 2))
      return cudaErrorInvalidValue;
  }
  if (!tc::map_3d(&g.tmB1[0], b1_0, (uint64_t)E, (uint64_t)n0, (uint64_t)k0, box_n))
    return cudaErrorInvalidValue;
  if (up && !tc::map_3d(&g.tmB3[0], b3_0, (uint64_t)E, (uint64_t)n0, (uint64_t)k0, box_n))
    return cudaErrorInvalidValue;
  if (has_sh) {
    if (!tc::map_2d(&g.tmA[1], a1, (uint64_t)T_sh, (uint64_t)k1, box_a)) return cudaErrorInvalidValue;
    if (pair && !tc::map_2d(&g.tmA64[1], a1, (uint64_t)T_sh, (uint64_t)k1, box_a / 2))
      return cudaErrorInvalidValue;
    if (!tc::map_3d(&g.tmB1[1], b1_1, 1, (uint64_t)n1, (uint64_t)k1, box_n))
      return cudaErrorInvalidValue;
    if (up && !tc::map_3d(&g.tmB3[1], b3_1, 1, (uint64_t)n1, (uint64_t)k1, box_n))
      return cudaErrorInvalidValue;
  } else {
    g.tmA[1] = g.tmA[0];
    g.tmA64[1] = g.tmA64[0];
    g.tmB1[1] = g.tmB1[0];
    g.tmB3[1] = g.tmB3[0];
  }
  if (!up) g.tmB3[0] = g.tmB1[0], g.tmB3[1] = g.tmB1[1];
  // UP: w1 and w3 tiles in one TMA box when the two tensors can be described
  // by one map
  if (up) {
    g.b13[0] = tc::map_pair_4d(&g.tmB13[0], b1_0, b3_0, (uint64_t)E, (uint64_t)n0, (uint64_t)k0,
                               box_n);
    if (has_sh)
      g.b13[1] = tc::map_pair_4d(&g.tmB13[1], b1_1, b3_1, 1, (uint64_t)n1, (uint64_t)k1, box_n);
    else
      g.b13[1] = g.b13[0], g.tmB13[1] = g.tmB13[0];
  }
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

  // upper bound on the tiles (the exact count depends on the device offsets)
  const int bm = pair ? 2 * BM : BM;
  const int bn_out = up ? BN / 2 : BN;
  const int64_t nt0 = (n0 + bn_out - 1) / bn_out;
  const int64_t bound = nt0 * ((Tk + bm - 1) / bm + E) +
                        (has_sh ? (int64_t)((n1 + bn_out - 1) / bn_out) * ((T_sh + bm - 1) / bm) : 0);
  cudaError_t e;
  if (pair) {
    const int pairs = (int)(bound < num_sms / 2 ? bound : num_sms / 2);
    if (pairs <= 0) {
      stage_mark(st);
      return cudaSuccess;
    }
    e = launch_grouped_tc2(up, g, pairs, st);
    stage_mark(st);
    return e;
  }
  const int grid = (int)(bound < num_sms ? bound : num_sms);
  if (grid <= 0) {
    stage_mark(st);
    return cudaSuccess;
  }
  if (E > 0) {
    // per-expert A maps (built before the launch; not needed when gathering)
    g.row_maps = gather ? nullptr : static_cast<const CUtensorMap*>(row_maps);
    // Tiles in order from a counter for the up-projection: its long tiles
    // (K = D) keep the CTAs that share weight and A tiles in step, where
    // round-robin lets them drift apart and re-read from HBM (UP read 1.15x
    // its algorithmic DRAM bytes at prefill). The down-projection's tiles
    // (K = I) are short enough that the hand-off costs more than it saves.
    g.tile_ctr = up ? tile_ctr : nullptr;
    g.stall = up && g_stall == STALL_EXPERTS_UP ? 1 : 0;
  }
  if (up) {
    e = cudaFuncSetAttribute(grouped_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = launch_pdl(pdl, grouped_tc_kernel<true>, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, st, g);
    if (e != cudaSuccess) return e;
  } else {
    e = cudaFuncSetAttribute(grouped_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    e = launch_pdl(pdl, grouped_tc_kernel<false>, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES, st, g);
    if (e != cudaSuccess) return e;
  }
  stage_mark(st);
  return cudaGetLastError();
}

}  // namespace moe
