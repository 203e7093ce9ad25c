// Grouped SwiGLU expert GEMMs with FP8 (e4m3) block-scaled weights and
// activations, on the 5th-generation tensor cores (tcgen05.mma
// kind::mxf8f6f4 with block scaling: the tensor core applies the scales).
//
// The pages say only that the block's other linears are FP8 ("Expert
// scores", dtype note). The layout here is this library's: e4m3 values, one
// power-of-two fp32 scale per 128 x 128 block of a weight matrix [out, in]
// and per 1 x 128 block of a row of activations (the smallest scale that
// keeps the block within 448, and at least 2^-127, so that every scale is one
// UE8M0 byte). x is quantized once per step (quant_rows
// kernel); h = silu(w1 x) * (w3 x) is quantized by the up-projection's
// epilogue; each expert's output is bf16, as on the bf16 path.
//
// Tiles put the weights on the MMA's M side (MMAs of 128 rows: one scale
// block; two per stage, UP's w1 and w3 rows or 256 of DOWN's w2 rows) and up
// to NT = 32 tokens of one expert on its N side, so a decode batch (a few
// tokens per expert) does little MMA work while it streams the active
// experts' weights at half the bytes of bf16. (Batches with more rows per
// expert run the token-on-M form of gemm_fp8m.cu.) Every MMA is block-scaled: per
// 32-deep slice of K it multiplies each weight row by its UE8M0 scale and each
// token by its own, so one fp32 TMEM accumulator sums the whole K,
//   sum[f, t] = sum_kb s_w(e, f/128, kb) s_x(t, kb) sum_{k in kb} q_w[f, k] q_x[t, k]
// (a lane of TMEM is a weight row f, a column a token t), and the epilogue
// reads it once per tile. The producer writes each stage's scale bytes to
// shared memory (the weight block's byte in all 128 rows, each token's byte
// in its row) and the MMA thread copies them to TMEM (tcgen05.cp
// 32x128b.warpx4) before that stage's MMAs.
//
// One CTA per SM, 192 threads: warp 0 TMA (weights by tile, token rows by
// tile::gather4 from the routed rows' tokens or the rows themselves; rows
// past a tile's tokens read zeros), warp 1 MMA, warps 2-5 epilogue. Waits are
// bounded as in the bf16 kernel (1 s, then the abort path).
#include "fp8_common.cuh"

namespace moe {

namespace {

using namespace tc;
using namespace fp8;

constexpr int NT = 32;                         // tokens per tile at most (MMA N)
constexpr int A_BYTES = NT * QB;               // 4 KB of token rows
constexpr int W_BYTES = QB * QB;               // 16 KB per weight tile
// Stages: UP carries the w1 and w3 tiles (36 KB, 5 stages), DOWN one w2 tile
// (20 KB, 9 stages), so both keep ~160-180 KB of weights in flight per SM.
// A stage holds KPS k-blocks: per k-block the tile's token rows and its two
// 128-row weight tiles (UP: w1 and w3; DOWN: two consecutive blocks of w2's
// rows, so a DOWN tile covers 256 output features).
template <bool UP> struct Ring {
  static constexpr int KPS = 1;   // 128-deep k-blocks per stage
  static constexpr int STAGES = 5;
  static constexpr int BYTES = KPS * (A_BYTES + 2 * W_BYTES);
};
// Output features per tile: UP 128 (the w1 rows, with the w3 rows beside
// them), DOWN 256.
template <bool UP> struct TileN {
  static constexpr int BN = UP ? QB : 2 * QB;
};
constexpr int RING_BYTES = 9 * (A_BYTES + W_BYTES);  // the larger of the two rings (184 KB)
static_assert(Ring<true>::STAGES * Ring<true>::BYTES <= RING_BYTES, "UP ring");
static_assert(Ring<false>::STAGES * Ring<false>::BYTES <= RING_BYTES, "DOWN ring");
constexpr int NTHREADS = 192;
constexpr uint32_t FTMEM = 256;
constexpr int MAXE = 1024;
constexpr int MAX_KB = 64;                     // k-blocks per tile (K <= 8192)
// TMEM columns: two accumulator buffers (the epilogue drains one tile while
// the next accumulates), each 2 x NT columns for UP (w1 rows | w3 rows) and
// NT for DOWN, from column 0; then SF_SLOTS slots of scale factors, one per
// group of up to four k-blocks of a tile: 4 columns for the weight rows'
// (SFA; w1 and w3 each for UP) and 4 for the tokens' (SFB; only the first is
// read at N = 32). Byte j of each 32-bit TMEM word holds k-block 4g + j's
// scale; the MMA picks it with the instruction's scale-factor IDs.
constexpr int ACC_COLS = 2 * NT;
constexpr int SF_COL0 = 2 * ACC_COLS;
// A slot is rewritten SF_SLOTS groups later, at least SF_SLOTS k-blocks on:
// by then the MMAs that read it are complete (the MMA thread has passed the
// full barrier of a stage the producer refilled after their commit), as long
// as SF_SLOTS exceeds either ring's stages.
constexpr int SF_SLOTS = 10;
template <bool UP> struct SfCols {
  static constexpr int PER_SLOT = 12;
};
static_assert(SF_COL0 + SF_SLOTS * 12 <= (int)FTMEM, "TMEM columns");
static_assert(SF_SLOTS > 5, "scale-factor slots outlive the ring");
// Per stage in shared memory, the scale-factor bytes the MMA thread copies to
// TMEM (tcgen05.cp 32x128b.warpx4) when the stage starts a group: 512 bytes
// each for SFA (w1), SFA (w3, UP) and SFB, row r = TMEM lane r of each of the
// four sub-partitions.
constexpr int SF_BYTES = 512;
constexpr int SC_SLOT = NT * MAX_KB * 4;      // one tile's token scales (8 KB)
// alignment slack, stages, the stages' scale-factor bytes, barriers (512), P
// and off, 16 bytes to align the scale slots, the two scale slots, the
// per-warp maxima
constexpr size_t FSMEM = 1024 + (size_t)RING_BYTES + 9 * 2 * SF_BYTES + 512 +
                         2 * (MAXE + 1) * 4 + 16 + 2 * (size_t)SC_SLOT + 4 * NT * 4;
static_assert(5 * 3 * SF_BYTES <= 9 * 2 * SF_BYTES, "UP scale-factor bytes");

struct Fp8Args {
  // token rows (uint8 [rows, K], box 128 x 1, for tile::gather4): [0] routed
  // (UP: the quantized x, read by token through src; DOWN: the quantized h
  // in expert order), [1] the shared MLP's (UP: quantized x; DOWN: its h)
  CUtensorMap tmA[2];
  // the same tensors for tile loads of NT contiguous rows: every A but the
  // routed UP's, whose rows are gathered by token
  CUtensorMap tmAt[2];
  CUtensorMap tmW1[2];   // weights [E, N, K] uint8, box 128 x 128 x 1: w1 (UP) / w2 (DOWN); shared E = 1
  CUtensorMap tmW3[2];   // w3 / ws3 (UP)
  const float* ws1[2];   // weight scales [E, N/128, K/128] of tmW1
  const float* ws3[2];   // of tmW3
  // scales of the A rows [rows, K/128], in the A rows' order: routed UP the
  // quantized x's scales in expert order (quant_rows_kernel writes them
  // through pos), so that a tile's are one contiguous run the producer copies
  // in bulk
  const float* asc[2];
  const int32_t* src;    // routed UP: the token of each expert-order row
  int a_rows[2];         // rows of the A tensors (an out-of-range row reads zeros)
  void* out[2];          // UP: quantized h [rows, N] uint8; DOWN: bf16 [rows, N]
  float* out_scale[2];   // UP: h's scales [rows, N/128]
  int n_out[2];
  int kdim[2];
  const int32_t* offsets;
  int E;
  int t_shared;
  // Test hook (moe_debug_stall_pipeline): CTA 0's MMA thread first waits on
  // a barrier phase that nothing completes, so that wait runs out (1 s)
  // before anything is issued, and the launch takes its abort path.
  int stall;
  uint32_t* err;
};

struct Tile {
  int kind, e, row0, rows, n0;
};

struct Sched {
  const int32_t* P;
  const int32_t* off;
  int E, nb0, nb1, ch_sh, routed, total, t_shared, bn;
};

// Tile i. `hint` is the expert of the caller's previous routed tile: a thread
// visits its tiles in increasing order, so the expert only moves forward (a
// few steps from the hint instead of a binary search per tile).
__device__ __forceinline__ Tile decode(const Sched& S, int i, int& hint) {
  Tile t;
  if (i < S.routed) {
    const int q = i / S.nb0;
    int e = hint;
    while (S.P[e + 1] <= q) ++e;
    hint = e;
    const int mt = S.P[e + 1] - S.P[e];
    const int l = i - S.nb0 * S.P[e];
    const int nb = l / mt, c = l % mt;
    t.kind = 0;
    t.e = e;
    t.row0 = S.off[e] + c * NT;
    t.rows = min(NT, S.off[e + 1] - t.row0);
    t.n0 = nb * S.bn;
  } else {
    const int l = i - S.routed;
    const int nb = l / S.ch_sh, c = l % S.ch_sh;
    t.kind = 1;
    t.e = 0;
    t.row0 = c * NT;
    t.rows = min(NT, S.t_shared - t.row0);
    t.n0 = nb * S.bn;
  }
  return t;
}


template <bool UP>
__global__ void __launch_bounds__(NTHREADS, 1) grouped_fp8_kernel(const __grid_constant__ Fp8Args g) {
  // DOWN: the combine after it may launch now (it waits for this grid
  // before it reads the outputs). UP lets the down-projection launch only
  // after its own prologue (below), once it has waited for its predecessors.
  if (!UP) asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  constexpr int FSTAGES = Ring<UP>::STAGES;
  constexpr int FSTAGE = Ring<UP>::BYTES;
  constexpr int SF_STAGE = 3 * SF_BYTES;   // SFA (first weight tile), SFA (second), SFB
  uint8_t* sfs = tiles + RING_BYTES;                  // [FSTAGES][SF_STAGE]
  uint64_t* full = reinterpret_cast<uint64_t*>(sfs + 9 * 2 * SF_BYTES);
  uint64_t* empty = full + FSTAGES;
  uint64_t* tfull = empty + FSTAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint64_t* sfull = drain + 1;            // token-scale slots, copied in by the producer
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sfull + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* P = reinterpret_cast<int32_t*>(sfs + 9 * 2 * SF_BYTES + 512);
  int32_t* off = P + MAXE + 1;
  // [2][rows][K/128] the token scales of a tile (two slots, copied in bulk
  // a tile ahead), then [4][NT] per-warp maxima
  float* tsc = reinterpret_cast<float*>(off + MAXE + 1 + 2);  // 16-byte aligned
  float* red = tsc + 2 * NT * MAX_KB;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int E = g.E;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < FSTAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
      for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 128); }
      for (int b = 0; b < 2; ++b) mbar_init(&sfull[b], 1);
      mbar_init(drain, 1);
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // UP, a programmatic dependent of the row quantization: wait for it
    // before anything it or the kernels before it wrote is read (the offsets
    // here; src, the scales and x's codes after the __syncthreads below).
    // DOWN, a programmatic dependent of the up-projection, reads here only
    // what was complete before that grid let it launch (the offsets); it
    // waits for h in its producer, after prefetching its first weight tiles.
    if (UP) asm volatile("griddepcontrol.wait;" ::: "memory");
    // token chunks per expert and their exclusive prefix
    const int per = (E + 31) / 32;
    int lsum = 0;
    for (int u = 0; u < per; ++u) {
      const int e = lane * per + u;
      if (e < E) {
        const int o0 = g.offsets[e], o1 = g.offsets[e + 1];
        off[e] = o0;
        if (e == E - 1) off[E] = o1;
        lsum += (o1 - o0 + NT - 1) / NT;
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
        run += (g.offsets[e + 1] - g.offsets[e] + NT - 1) / NT;
      }
    }
    if (lane == 31) P[E] = incl;
    __syncwarp();
  } else if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(FTMEM));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // UP: every thread of the CTA is past the wait for the kernels before it,
  // so a dependent down-projection may read what they wrote (the offsets)
  // before it waits for this grid
  if (UP) asm volatile("griddepcontrol.launch_dependents;");

  Sched S;
  S.P = P;
  S.off = off;
  S.E = E;
  S.bn = TileN<UP>::BN;
  S.nb0 = (g.n_out[0] + S.bn - 1) / S.bn;
  S.nb1 = g.t_shared > 0 ? (g.n_out[1] + S.bn - 1) / S.bn : 0;
  S.ch_sh = (g.t_shared + NT - 1) / NT;
  S.t_shared = g.t_shared;
  S.routed = S.nb0 * P[E];
  S.total = S.routed + S.nb1 * S.ch_sh;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Lane 0: barriers, the weight tiles and a contiguous tile's token rows;
    // lanes 0..NT/4-1 gather 4 token rows each (routed UP). Every lane writes
    // its row of each stage's scale-factor bytes: the weight block's scale
    // (the same for all 128 weight rows of the tile) and its token's.
    int s = 0, issued = 0, scopies = 0;
    int hint = 0, hint_next = 0, hint_w = 0;  // experts of the last tile decoded: this, next, scales
    uint32_t ph = 0;
    bool ok = true;
    // the weight-block scales of a tile, k-blocks lane and lane + 32 (1.0 past
    // its k-blocks and for a missing second block), loaded a tile ahead
    float nw[4];
    auto load_wscales = [&](const Tile& tt) {
      const int kbn = g.kdim[tt.kind] / QB;
      const int nbw = g.n_out[tt.kind] / QB;
      const bool two_t = UP || tt.n0 + QB < g.n_out[tt.kind];
      const float* pw1 = g.ws1[tt.kind] + ((int64_t)tt.e * nbw + tt.n0 / QB) * kbn;
      const float* pw3 = UP ? g.ws3[tt.kind] + ((int64_t)tt.e * nbw + tt.n0 / QB) * kbn : pw1 + kbn;
      nw[0] = lane < kbn ? __ldg(pw1 + lane) : 1.f;
      nw[1] = lane + 32 < kbn ? __ldg(pw1 + lane + 32) : 1.f;
      nw[2] = two_t && lane < kbn ? __ldg(pw3 + lane) : 1.f;
      nw[3] = two_t && lane + 32 < kbn ? __ldg(pw3 + lane + 32) : 1.f;
    };
    if ((int)blockIdx.x < S.total) load_wscales(decode(S, blockIdx.x, hint_w));
    if (!UP) {
      // the first tile's leading weight k-blocks into L2 while the
      // up-projection finishes, then wait for it (h and its scales)
      if (lane == 0 && (int)blockIdx.x < S.total) {
        int h0 = 0;
        const Tile t0 = decode(S, blockIdx.x, h0);
        const int kb_n = g.kdim[t0.kind] / QB;
        const bool two0 = t0.n0 + QB < g.n_out[t0.kind];
        const int n_pf = min(kb_n, DOWN_PREFETCH_KB_BYTES / (2 * W_BYTES));
        for (int kb = 0; kb < n_pf; ++kb) {
          tma_prefetch_3d(&g.tmW1[t0.kind], kb * QB, t0.n0, t0.e);
          if (two0) tma_prefetch_3d(&g.tmW1[t0.kind], kb * QB, t0.n0 + QB, t0.e);
        }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    if (lane == 0 && (int)blockIdx.x < S.total) {   // the first tile's token scales
      int h0 = 0;
      const Tile t0 = decode(S, blockIdx.x, h0);
      const int kbp = scale_stride(g.kdim[t0.kind]);
      const uint32_t bytes = (uint32_t)(t0.rows * kbp * 4);
      mbar_expect_tx(&sfull[0], bytes);
      bulk_load(tsc, g.asc[t0.kind] + (int64_t)t0.row0 * kbp, bytes, &sfull[0]);
      ++scopies;
    }
    for (int i = blockIdx.x, lt = 0; i < S.total; i += gridDim.x, ++lt) {
      const Tile t = decode(S, i, hint);
      const int kb_n = g.kdim[t.kind] / QB;
      const int kbp = scale_stride(g.kdim[t.kind]);
      const int slot = lt & 1;
      // the second weight tile: UP w3's rows, DOWN the next 128 rows of w2
      // (none in a DOWN tile at the end of an odd number of row blocks)
      const bool two = UP || t.n0 + QB < g.n_out[t.kind];
      // the tile's weight scales as UE8M0 bytes (loaded a tile ahead), then
      // the next tile's loads
      const uint32_t w1a = ue8m0(nw[0]), w1b = ue8m0(nw[1]), w3a = ue8m0(nw[2]), w3b = ue8m0(nw[3]);
      if (i + (int)gridDim.x < S.total) load_wscales(decode(S, i + gridDim.x, hint_w));
      // this tile's token scales (copied a tile ahead), then the next tile's
      // copy into the other slot (its last reader, the previous tile's loop
      // below, is done: the warp has synchronised since)
      {
        int w = 1;
        if (lane == 0) w = mbar_wait(&sfull[slot], (uint32_t)(lt >> 1) & 1, abort_flag, g.err) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
      }
      if (lane == 0 && i + (int)gridDim.x < S.total) {
        const Tile tn = decode(S, i + gridDim.x, hint_next);
        const int kbpn = scale_stride(g.kdim[tn.kind]);
        const uint32_t bytes = (uint32_t)(tn.rows * kbpn * 4);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_expect_tx(&sfull[slot ^ 1], bytes);
        bulk_load(tsc + (slot ^ 1) * NT * MAX_KB, g.asc[tn.kind] + (int64_t)tn.row0 * kbpn, bytes,
                  &sfull[slot ^ 1]);
        ++scopies;
      }
      const float* ts = tsc + slot * NT * MAX_KB;   // [t.rows][kbp]
      // routed UP rows are tokens scattered over x: gathered four at a time;
      // the others (expert-ordered h, token rows) are contiguous: one tile
      // load of NT rows (rows past a tile's tokens are multiplied and not
      // stored; past the tensor's end they read zeros)
      const bool gath = UP && t.kind == 0;
      // token rows brought in per k-block: a gathered tile only its rows,
      // rounded up to 4 (the MMA's other token columns read whatever the
      // stage held; their sums are not stored), a tile load all NT
      const int a_rows_ld = gath ? ((t.rows + 3) & ~3) : NT;
      constexpr int KPS = Ring<UP>::KPS;
      int r[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int j = 4 * lane + q;
        const int row = t.row0 + j;
        int a = g.a_rows[t.kind];                        // out of range: zeros
        if (j < t.rows) a = (UP && t.kind == 0 && g.src != nullptr) ? g.src[row] : row;
        r[q] = a;
      }
      for (int kb = 0; kb < kb_n; kb += KPS) {
        const int nk = kb_n - kb < KPS ? kb_n - kb : KPS;   // k-blocks in this stage
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty[s], ph ^ 1, abort_flag, g.err) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        if ((kb & 3) == 0) {
          // a group's first stage: the scale factors of k-blocks kb .. kb + 3,
          // byte j for kb + j (bytes past the tile's k-blocks are not read).
          // The stage's previous MMAs, and the copies to TMEM before them, are
          // complete: empty[s] came from their commit.
          uint8_t* sf = sfs + s * SF_STAGE;
          uint32_t p1 = 0, p3 = 0, pt = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = kb + j;
            p1 |= __shfl_sync(0xffffffffu, k < 32 ? w1a : w1b, k & 31) << (8 * j);
            p3 |= __shfl_sync(0xffffffffu, k < 32 ? w3a : w3b, k & 31) << (8 * j);
            pt |= (lane < t.rows && k < kb_n ? ue8m0(ts[lane * kbp + k]) : 127u) << (8 * j);
          }
          *reinterpret_cast<uint4*>(sf + lane * 16) = make_uint4(p1, p1, p1, p1);
          *reinterpret_cast<uint4*>(sf + SF_BYTES + lane * 16) = make_uint4(p3, p3, p3, p3);
          *reinterpret_cast<uint4*>(sf + 2 * SF_BYTES + lane * 16) = make_uint4(pt, 0u, 0u, 0u);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        // stage layout: the KPS token tiles, then per k-block its weight tile(s)
        uint8_t* sa = tiles + s * FSTAGE;
        if (lane == 0) {
          mbar_expect_tx(&full[s], (uint32_t)(nk * (a_rows_ld * QB + (two ? 2 : 1) * W_BYTES)));
          for (int q = 0; q < nk; ++q) {
            uint8_t* sw = sa + KPS * A_BYTES + q * 2 * W_BYTES;
            tma_load_3d(sw, &g.tmW1[t.kind], &full[s], (kb + q) * QB, t.n0, t.e);
            if (UP) tma_load_3d(sw + W_BYTES, &g.tmW3[t.kind], &full[s], (kb + q) * QB, t.n0, t.e);
            else if (two) tma_load_3d(sw + W_BYTES, &g.tmW1[t.kind], &full[s], (kb + q) * QB, t.n0 + QB, t.e);
            if (!gath) tma_load_2d(sa + q * A_BYTES, &g.tmAt[t.kind], &full[s], (kb + q) * QB, t.row0);
          }
        }
        __syncwarp();
        if (gath && lane < a_rows_ld / 4)
          tma_gather4(sa + lane * (4 * QB), &g.tmA[t.kind], &full[s], kb * QB, r[0], r[1], r[2], r[3]);
        ++issued;
        if (++s == FSTAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
    }
    if (!ok && lane == 0) {
      for (int j = 0; j < FSTAGES; ++j) {
        const int n = issued / FSTAGES + (j < issued % FSTAGES ? 1 : 0);
        if (n > 0) mbar_drain(&full[j], (uint32_t)((n - 1) & 1));
      }
      for (int j = 0; j < 2; ++j) {
        const int n = scopies / 2 + (j < scopies % 2 ? 1 : 0);
        if (n > 0) mbar_drain(&sfull[j], (uint32_t)((n - 1) & 1));
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    // Per group of four stages: the scale factors to TMEM (tcgen05.cp,
    // ordered before the MMAs this thread issues after it); per stage four
    // K = 32 block-scaled MMAs per weight tile (two tiles: UP w1 and w3, DOWN
    // two row blocks of w2) into the tile's accumulator, which sums the whole
    // K, reading byte kb % 4 of the scale words; one commit per tile hands it
    // to the epilogue.
    if (lane == 0) {
      int s = 0, groups = 0, hint = 0;
      uint32_t ph = 0, tsa = 0;
      bool ok = true;
      // test hook: a wait that runs out (the drain barrier is committed only
      // after the tile loop), before any MMA is issued
      if (g.stall && blockIdx.x == 0 && !mbar_wait(drain, 0, abort_flag, g.err)) ok = false;
      for (int i = blockIdx.x, lt = 0; ok && i < S.total; i += gridDim.x, ++lt) {
        const Tile t = decode(S, i, hint);
        const int kb_n = g.kdim[t.kind] / QB;
        const bool two = UP || t.n0 + QB < g.n_out[t.kind];
        const int b = lt & 1;
        if (!mbar_wait(&tempty[b], ((uint32_t)(lt >> 1) & 1) ^ 1, abort_flag, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base + (uint32_t)(b * ACC_COLS);
        constexpr int KPS = Ring<UP>::KPS;
        for (int kb = 0; kb < kb_n; kb += KPS) {
          const int nk = kb_n - kb < KPS ? kb_n - kb : KPS;
          if (!mbar_wait(&full[s], ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(tiles + s * FSTAGE);
          if ((kb & 3) == 0) {
            const uint32_t sf0 = smem_u32(sfs + s * SF_STAGE);
            tsa = tmem_base + (uint32_t)(SF_COL0 + (groups % SF_SLOTS) * SfCols<UP>::PER_SLOT);
            ++groups;
            tmem_cp_sf(tsa, sdesc_sf(sf0));
            if (two) tmem_cp_sf(tsa + 4, sdesc_sf(sf0 + SF_BYTES));
            tmem_cp_sf(tsa + 8, sdesc_sf(sf0 + 2 * SF_BYTES));
          }
          for (int q = 0; q < nk; ++q) {
            const uint32_t aq = a0 + q * A_BYTES;
            const uint32_t wq = a0 + KPS * A_BYTES + q * 2 * W_BYTES;
            // byte j = (kb + q) % 4 of the words: in the instruction
            // descriptor and, as the byte address, in the top two bits of the
            // TMEM addresses
            const uint32_t j = (uint32_t)((kb + q) & 3);
            const uint32_t idesc = idesc_mx_e4m3(QB, NT, j);
            const uint32_t sfa1 = tsa | (j << 30), sfa3 = (tsa + 4) | (j << 30);
            const uint32_t sfb = (tsa + 8) | (j << 30);
#pragma unroll
            for (int kk = 0; kk < QB / 32; ++kk) {
              const uint32_t acc = (kb + q > 0 || kk > 0) ? 1u : 0u;
              mma_mx(d, sdesc(wq + kk * 32), sdesc(aq + kk * 32), idesc, sfa1, sfb, acc);
              if (two) mma_mx(d + NT, sdesc(wq + W_BYTES + kk * 32), sdesc(aq + kk * 32), idesc, sfa3,
                              sfb, acc);
            }
          }
          tc_commit(&empty[s]);
          if (++s == FSTAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit(&tfull[b]);
      }
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // The tile's fp32 sums (scales already applied by the tensor core): a
    // TMEM lane is a weight row f, a column a token.
    const int quad = warp & 3;
    int hint = 0;
    const int f = quad * 32 + lane;      // this thread's weight row (TMEM lane) in the tile
    const int et = threadIdx.x - 64;     // 0..127 among the epilogue threads
    for (int i = blockIdx.x, lt = 0; i < S.total; i += gridDim.x, ++lt) {
      const Tile t = decode(S, i, hint);
      const bool two = UP || t.n0 + QB < g.n_out[t.kind];
      const int b = lt & 1;
      bool ok;
      {
        int w = 1;
        if (lane == 0) w = mbar_wait(&tfull[b], (uint32_t)(lt >> 1) & 1, abort_flag, g.err) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, w, 0) != 0;
      }
      float sa[NT], sb[NT];
      if (ok) {
        tc_fence_after();
        const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16) + (uint32_t)(b * ACC_COLS);
        uint32_t r0[16], r1[16];
        tmem_ld16(tb, r0);
        tmem_ld16(tb + 16, r1);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; ++j) { sa[j] = __uint_as_float(r0[j]); sa[16 + j] = __uint_as_float(r1[j]); }
        if (two) {
          tmem_ld16(tb + NT, r0);
          tmem_ld16(tb + NT + 16, r1);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j) { sb[j] = __uint_as_float(r0[j]); sb[16 + j] = __uint_as_float(r1[j]); }
        }
        tc_fence_before();
        mbar_arrive(&tempty[b]);
      }
      // one decision for all four warps: stop if any of them gave up
      if (epi_sync_any(!ok)) break;
      if (UP) {
        // h = silu(a) * b, quantized per token over this tile's 128 features
        // (one 1 x 128 block of h's row)
        uint8_t* hq = reinterpret_cast<uint8_t*>(g.out[t.kind]);
        float* hs = g.out_scale[t.kind];
        const int nbh = scale_stride(g.n_out[t.kind]);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const float h = silu_f(sa[j]) * sb[j];
          sa[j] = h;
          float m = fabsf(h);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
          if (lane == 0) red[quad * NT + j] = m;
        }
        asm volatile("bar.sync 1, 128;" ::: "memory");
#pragma unroll
        for (int j = 0; j < NT; ++j) {   // unrolled: sa stays in registers
          if (j < t.rows) {
            const float amax = fmaxf(fmaxf(red[j], red[NT + j]), fmaxf(red[2 * NT + j], red[3 * NT + j]));
            const int se = block_exp(amax);
            const int64_t row = t.row0 + j;
            hq[row * g.n_out[t.kind] + t.n0 + f] = to_e4m3(ldexpf(sa[j], -se));
            if (et == 0) hs[row * nbh + t.n0 / QB] = ldexpf(1.f, se);
          }
        }
      } else {
        // the tile's two row blocks: features n0 + f and n0 + 128 + f
        __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(g.out[t.kind]);
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          if (j < t.rows) {
            __nv_bfloat16* o = out + (int64_t)(t.row0 + j) * g.n_out[t.kind] + t.n0 + f;
            o[0] = __float2bfloat16_rn(sa[j]);
            if (two) o[QB] = __float2bfloat16_rn(sb[j]);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"(FTMEM));
  }
}

// Rows [R, K] (act) to e4m3 with one power-of-two scale per 1 x 128 block:
// one warp per two blocks of a row, a half-warp per block, 8 elements (one or
// two 16-byte loads, one 8-byte store of codes) per lane.
// With pos, each block's scale is also written to the k permuted rows of its
// row's (token, slot) pairs (scale_perm, for the up-projection's routed rows;
// pairs with pos < 0 are skipped), and with q_perm its codes too (the
// token-on-M up-projection reads its routed rows from there).
template <typename T>
__global__ void __launch_bounds__(256) quant_rows_kernel(const T* __restrict__ a, int64_t R, int K,
                                                         uint8_t* __restrict__ q,
                                                         float* __restrict__ scale, int sstride,
                                                         const int32_t* __restrict__ pos, int k,
                                                         float* __restrict__ scale_perm,
                                                         uint8_t* __restrict__ q_perm) {
  // a programmatic dependent of the dispatch (pos): the up-projection after
  // it may launch now; pos is read after the dispatch's grid completes
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int kbn = K / QB;
  const int pairs = (kbn + 1) / 2;     // block pairs per row
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) / 32;
  const int lane = threadIdx.x % 32;
  if (w >= R * pairs) return;          // whole warps
  const int64_t r = w / pairs;
  const int kb = (int)(w % pairs) * 2 + (lane >> 4);   // this half-warp's block
  const int sl = lane & 15;                            // elements 8 sl .. 8 sl + 7 of it
  const bool active = kb < kbn;                        // the second block of an odd row end: none
  float v[8];
  if (active) {
    const T* p = a + r * K + kb * QB + sl * 8;
    Vec16<T> x0;
    x0.raw = reinterpret_cast<const uint4*>(p)[0];
    x0.to_float(v);
    if (Vec16<T>::N == 4) {
      Vec16<T> x1;
      x1.raw = reinterpret_cast<const uint4*>(p)[1];
      x1.to_float(v + 4);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = 0.f;
  }
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[i]));
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));  // within the half
  const int se = block_exp(m);
  uint32_t c0 = 0, c1 = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c0 |= (uint32_t)to_e4m3(ldexpf(v[i], -se)) << (8 * i);
    c1 |= (uint32_t)to_e4m3(ldexpf(v[4 + i], -se)) << (8 * i);
  }
  const uint2 codes = make_uint2(c0, c1);
  const float sc = ldexpf(1.f, se);
  if (active) {
    reinterpret_cast<uint2*>(q + r * K + kb * QB)[sl] = codes;
    if (sl == 0) scale[r * sstride + kb] = sc;
  }
  if (pos != nullptr) {
    const int p = lane < k ? pos[r * k + lane] : -1;   // k <= 32
    for (int j = 0; j < k; ++j) {
      const int pj = __shfl_sync(0xffffffffu, p, j);
      if (pj >= 0 && active) {
        if (sl == 0 && scale_perm != nullptr) scale_perm[(int64_t)pj * sstride + kb] = sc;
        if (q_perm != nullptr) reinterpret_cast<uint2*>(q_perm + (int64_t)pj * K + kb * QB)[sl] = codes;
      }
    }
  }
}

// A bf16 / fp32 matrix [R, C] to e4m3 with one power-of-two scale per
// 128 x 128 block (the weights' layout): one CTA per block, 256 threads.
template <typename T>
__global__ void __launch_bounds__(256) quant_blocks_kernel(const T* __restrict__ a, int64_t R, int C,
                                                           uint8_t* __restrict__ q,
                                                           float* __restrict__ scale) {
  __shared__ float wmax[8];
  const int64_t br = blockIdx.y;
  const int bc = blockIdx.x;
  const int nbc = C / QB;
  const int64_t r0 = br * QB;
  const int rows = (int)(R - r0 < QB ? R - r0 : QB);
  float m = 0.f;
  for (int i = threadIdx.x; i < rows * QB; i += 256) {
    const int rr = i / QB, cc = i % QB;
    m = fmaxf(m, fabsf(to_f32(a[(r0 + rr) * C + bc * QB + cc])));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (threadIdx.x % 32 == 0) wmax[threadIdx.x / 32] = m;
  __syncthreads();
  m = wmax[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) m = fmaxf(m, wmax[w]);
  const int se = block_exp(m);
  for (int i = threadIdx.x; i < rows * QB; i += 256) {
    const int rr = i / QB, cc = i % QB;
    const int64_t o = (r0 + rr) * C + bc * QB + cc;
    q[o] = to_e4m3(ldexpf(to_f32(a[o]), -se));  // exact: a power-of-two step, no overflow
  }
  if (threadIdx.x == 0) scale[br * nbc + bc] = ldexpf(1.f, se);
}

}  // namespace

namespace fp8 {

bool map_u8_rows(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K};
  cuuint32_t box[2] = {QB, 1};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_u8_tile(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K};
  cuuint32_t box[2] = {QB, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_u8_weights(CUtensorMap* m, const void* ptr, uint64_t E, uint64_t N, uint64_t K) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {K, N, E};
  cuuint64_t strides[2] = {K, N * K};
  cuuint32_t box[3] = {QB, QB, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace fp8

cudaError_t launch_quant_rows(const moe_config& c, const void* a, int64_t R, int K, uint8_t* q,
                              float* scale, int sstride, cudaStream_t st, const int32_t* pos,
                              float* scale_perm, uint8_t* q_perm) {
  const int64_t warps = R * ((K / QB + 1) / 2);
  if (warps == 0) return cudaSuccess;
  if (sstride <= 0) sstride = K / QB;
  const unsigned blocks = (unsigned)ceil_div<int64_t>(warps * 32, 256);
  if (c.dtype == MOE_DT_BF16)
    return launch_pdl(pdl_ok(), quant_rows_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, st,
                      (const __nv_bfloat16*)a, R, K, q, scale, sstride, pos, c.topk, scale_perm, q_perm);
  return launch_pdl(pdl_ok(), quant_rows_kernel<float>, dim3(blocks), dim3(256), 0, st,
                    (const float*)a, R, K, q, scale, sstride, pos, c.topk, scale_perm, q_perm);
}

int fp8_scale_stride(int K) { return scale_stride(K); }

cudaError_t launch_quant_blocks(bool bf16, const void* a, int64_t R, int C, uint8_t* q,
                                float* scale, cudaStream_t st) {
  dim3 grid((unsigned)(C / QB), (unsigned)ceil_div<int64_t>(R, QB));
  if (bf16)
    quant_blocks_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>((const __nv_bfloat16*)a, R, C, q, scale);
  else
    quant_blocks_kernel<float><<<grid, 256, 0, st>>>((const float*)a, R, C, q, scale);
  return cudaGetLastError();
}

// The FP8 expert GEMMs of one layer: UP reads the quantized x (routed rows
// by token through src, shared rows directly) and writes the quantized h and
// hs; DOWN reads them and writes y_perm and s (bf16).
cudaError_t launch_grouped_fp8(const moe_config& c, int64_t T, const Fp8Weights& w,
                               const uint8_t* xq, const float* xs, float* xs_perm,
                               const int32_t* src, const int32_t* offsets, uint8_t* hq, float* hsc,
                               uint8_t* hsq, float* hss, void* y_perm, void* s, uint32_t* err,
                               int num_sms, cudaStream_t st) {
  const int E = c.n_routed, D = c.dim, I = c.moe_inter, Is = c.shared_inter;
  const int64_t Tk = T * c.topk;
  const bool sh = Is > 0;
  cudaError_t e;
  for (int pass = 0; pass < 2; ++pass) {
    const bool up = pass == 0;
    Fp8Args g;
    memset(&g, 0, sizeof(g));
    const int n0 = up ? I : D, k0 = up ? D : I, n1 = up ? Is : D, k1 = up ? D : Is;
    if (up) {
      if (!map_u8_rows(&g.tmA[0], xq, (uint64_t)T, (uint64_t)D)) return cudaErrorInvalidValue;
      g.a_rows[0] = (int)T;
      g.asc[0] = xs_perm;
      g.src = src;
      if (!map_u8_weights(&g.tmW1[0], w.w1, E, I, D)) return cudaErrorInvalidValue;
      if (!map_u8_weights(&g.tmW3[0], w.w3, E, I, D)) return cudaErrorInvalidValue;
      g.ws1[0] = w.s1;
      g.ws3[0] = w.s3;
      g.out[0] = hq;
      g.out_scale[0] = hsc;
      if (sh) {
        g.tmA[1] = g.tmA[0];
        g.a_rows[1] = (int)T;
        g.asc[1] = xs;
        if (!map_u8_weights(&g.tmW1[1], w.ws1, 1, Is, D)) return cudaErrorInvalidValue;
        if (!map_u8_weights(&g.tmW3[1], w.ws3, 1, Is, D)) return cudaErrorInvalidValue;
        g.ws1[1] = w.ss1;
        g.ws3[1] = w.ss3;
        g.out[1] = hsq;
        g.out_scale[1] = hss;
      }
    } else {
      if (!map_u8_rows(&g.tmA[0], hq, (uint64_t)Tk, (uint64_t)I)) return cudaErrorInvalidValue;
      g.a_rows[0] = (int)Tk;
      g.asc[0] = hsc;
      if (!map_u8_weights(&g.tmW1[0], w.w2, E, D, I)) return cudaErrorInvalidValue;
      g.ws1[0] = w.s2;
      g.out[0] = y_perm;
      if (sh) {
        if (!map_u8_rows(&g.tmA[1], hsq, (uint64_t)T, (uint64_t)Is)) return cudaErrorInvalidValue;
        g.a_rows[1] = (int)T;
        g.asc[1] = hss;
        if (!map_u8_weights(&g.tmW1[1], w.ws2, 1, D, Is)) return cudaErrorInvalidValue;
        g.ws1[1] = w.ss2;
        g.out[1] = s;
      }
    }
    // tile-load maps of the A tensors (boxes of NT rows)
    {
      const void* a0p = up ? (const void*)xq : (const void*)hq;
      const uint64_t r0 = up ? (uint64_t)T : (uint64_t)Tk, kk0 = up ? (uint64_t)D : (uint64_t)I;
      if (!map_u8_tile(&g.tmAt[0], a0p, r0, kk0, NT)) return cudaErrorInvalidValue;
      if (sh) {
        const void* a1p = up ? (const void*)xq : (const void*)hsq;
        const uint64_t kk1 = up ? (uint64_t)D : (uint64_t)Is;
        if (!map_u8_tile(&g.tmAt[1], a1p, (uint64_t)T, kk1, NT)) return cudaErrorInvalidValue;
      } else {
        g.tmAt[1] = g.tmAt[0];
      }
    }
    if (!sh) {  // no shared group: its maps are never used, keep them valid
      g.tmA[1] = g.tmA[0];
      g.tmW1[1] = g.tmW1[0];
      g.tmW3[1] = g.tmW3[0];
    }
    if (!up) {  // DOWN reads one weight tile per stage
      g.tmW3[0] = g.tmW1[0];
      g.tmW3[1] = g.tmW1[1];
    }
    g.n_out[0] = n0;
    g.n_out[1] = sh ? n1 : n0;
    g.kdim[0] = k0;
    g.kdim[1] = sh ? k1 : k0;
    g.offsets = offsets;
    g.E = E;
    g.t_shared = sh ? (int)T : 0;
    g.err = err;
    g.stall = up && pipeline_stall() == STALL_EXPERTS_UP ? 1 : 0;
    const int bn = up ? TileN<true>::BN : TileN<false>::BN;   // output features per tile
    const int64_t bound = (int64_t)((n0 + bn - 1) / bn) * ((Tk + NT - 1) / NT + E) +
                          (sh ? (int64_t)((n1 + bn - 1) / bn) * ((T + NT - 1) / NT) : 0);
    const int grid = (int)(bound < num_sms ? bound : num_sms);
    if (grid > 0) {
      if (up) {
        e = cudaFuncSetAttribute(grouped_fp8_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)FSMEM);
        if (e != cudaSuccess) return e;
        // a programmatic dependent of the row quantization
        e = launch_pdl(pdl_ok(), grouped_fp8_kernel<true>, dim3(grid), dim3(NTHREADS), FSMEM, st, g);
        if (e != cudaSuccess) return e;
      } else {
        e = cudaFuncSetAttribute(grouped_fp8_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)FSMEM);
        if (e != cudaSuccess) return e;
        // a programmatic dependent of the up-projection
        e = launch_pdl(pdl_ok(), grouped_fp8_kernel<false>, dim3(grid), dim3(NTHREADS), FSMEM, st, g);
        if (e != cudaSuccess) return e;
      }
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    stage_mark(st);
  }
  return cudaSuccess;
}

}  // namespace moe
