// Grouped SwiGLU expert GEMMs with FP8 (e4m3) block-scaled weights for large
// batches: 128 token rows of one expert on the MMA's M side, 256 weight rows
// on its N side (UP: 128 rows of w1 over the same 128 rows of w3; DOWN: 256
// rows of w2), 128-deep k-blocks (one scale block) per pipeline stage.
//
// The form follows from the layout (one scale per 1 x 128 block of an
// activation row, one per 128 x 128 block of a weight matrix): per 32-deep
// slice of K the block-scaled MMA multiplies each row of A (a token) by its
// own UE8M0 scale and each row of B (a weight row) by its block's, so one
// fp32 TMEM accumulator sums the whole K,
//   acc[t, f] = sum_kb s_x(t, kb) s_w(e, f/128, kb) sum_{k in kb} q_x[t, k] q_w[f, k].
// At prefill the experts have hundreds of rows each, and this form does the
// MMA work of the batch at full tile size; the token-on-N form
// (gemm_fp8.cu) streams the weights once per 32 tokens instead and suits
// decode batches.
//
// The routed up-projection reads x's codes in expert order (written by the
// row quantization kernel straight to each (token, slot) pair's row, so
// there is no separate dispatch copy); the rows of a tile past its expert's
// rows are multiplied and not stored. The scales come from the rows' fp32
// scale arrays: the producer packs each group of four k-blocks' UE8M0 bytes
// into the shared-memory image that tcgen05.cp 32x128b.warpx4 moves to TMEM
// (token row m at lane m % 32, column m / 32; byte j = k-block 4g + j,
// picked by the MMA's scale-factor IDs), and the weight blocks' bytes into
// the 256 weight rows' columns.
//
// One CTA per SM, 320 threads: warp 0 TMA producer and scale images, warp 1
// MMA issuer (tcgen05.mma kind::mxf8f6f4.block_scale, M = 128, N = 256,
// K = 32), warps 2-9 epilogue. TMEM holds one 256-column accumulator and the
// scale-factor slots; the epilogue frees the accumulator as soon as it has
// read it into registers (128 values per thread: two threads per row), so
// the next tile's MMAs wait only for the TMEM reads. UP forms h = silu(a) b,
// one 1 x 128 block per row and tile, and quantizes it (the two threads of a
// row exchange their halves' maxima); DOWN rounds to bf16. Every pipeline
// wait is bounded (1 s, then the abort path of the other tensor-core
// kernels).
#include "fp8_common.cuh"

namespace moe {

namespace {

using namespace tc;
using namespace fp8;

constexpr int BM = 128;                            // token rows per tile (MMA M)
constexpr int BN = 256;                            // weight rows per tile (MMA N)
constexpr int STAGES = 4;
constexpr int A_TILE = BM * QB;                    // 16 KB of token rows
constexpr int W_TILE = QB * QB;                    // 16 KB, one 128 x 128 weight block
constexpr int STAGE_BYTES = A_TILE + 2 * W_TILE;   // 48 KB
constexpr int EPI_WARPS = 8;
constexpr int NTHREADS = 64 + 32 * EPI_WARPS;
constexpr uint32_t TMEM_COLS = 512;
// TMEM: the accumulator in columns [0, BN); from SF_COL0 the scale-factor
// slots, one per group of up to four k-blocks: 4 columns for the 128 token
// rows (SFA), 8 for the 256 weight rows (SFB). A slot is rewritten SF_SLOTS
// groups later, at least SF_SLOTS k-blocks on, when the MMAs that read it
// are complete (the MMA thread has since passed the full barrier of a stage
// the producer refilled after their commit), as SF_SLOTS exceeds STAGES.
constexpr int SF_COL0 = BN;
constexpr int SF_SLOT_COLS = 12;
constexpr int SF_SLOTS = 16;
static_assert(SF_COL0 + SF_SLOTS * SF_SLOT_COLS <= (int)TMEM_COLS, "TMEM columns");
static_assert(SF_SLOTS > STAGES, "scale-factor slots outlive the ring");
// Per stage in shared memory, the images the MMA thread copies to TMEM when
// the stage starts a group: SFA, SFB of the first weight block, SFB of the
// second (512 bytes each: 32 rows of 16 bytes).
constexpr int SF_BYTES = 512;
constexpr int SF_STAGE = 3 * SF_BYTES;
constexpr int MAXE = 1024;
// DOWN's output staging, per epilogue warp: 32 rows x 16 bf16 columns
constexpr int STAGE_WARP_BYTES = 32 * 32;
// Shared memory from the 1024-byte aligned base: the stages, the scale
// images, the output staging (16-byte accesses: every offset up to here is a
// multiple of 16), the row maxima of the two halves, barriers, P and off.
constexpr int OFF_SFS = STAGES * STAGE_BYTES;
constexpr int OFF_STAGE = OFF_SFS + STAGES * SF_STAGE;
constexpr int OFF_RED = OFF_STAGE + EPI_WARPS * STAGE_WARP_BYTES;
constexpr int OFF_BAR = OFF_RED + 2 * BM * 4;
constexpr int OFF_P = OFF_BAR + 256;
constexpr size_t SMEM_BYTES = 1024 + (size_t)OFF_P + 2 * (MAXE + 1) * 4;
static_assert(OFF_SFS % 16 == 0 && OFF_STAGE % 16 == 0 && OFF_BAR % 8 == 0, "shared memory alignment");
static_assert(SMEM_BYTES <= 232448, "shared memory per block");

struct Fp8mArgs {
  // token rows [rows, K] e4m3, box 128 x 128: [0] routed (UP: x's codes in
  // expert order; DOWN: h in expert order), [1] the shared MLP's (UP: x;
  // DOWN: its h)
  CUtensorMap tmA[2];
  CUtensorMap tmW1[2];   // weights [E, N, K] e4m3, box 128 x 128 x 1: w1 (UP) / w2 (DOWN); shared E = 1
  CUtensorMap tmW3[2];   // w3 / ws3 (UP)
  const float* ws1[2];   // weight scales [E, N/128, K/128] of tmW1
  const float* ws3[2];   // of tmW3
  const float* asc[2];   // the A rows' scales [rows, scale_stride(K)], in the A rows' order
  // [E] copies of tmA[0] whose row extent ends at each expert's last row
  // (written before the launch): an expert's last, partial tile reads zeros
  // past its rows, which cost less power than the next expert's codes; null:
  // tmA[0]
  const CUtensorMap* row_maps;
  void* out[2];          // UP: quantized h [rows, N] e4m3; DOWN: bf16 [rows, N]
  float* out_scale[2];   // UP: h's scales [rows, scale_stride(N)]
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
  int E, nb0, nb1, mt_sh, routed, total, t_shared, bn;
};

// Tile i: routed tiles expert by expert (n-tile outer, m-tile inner, so the
// CTAs running side by side share the expert's weight tiles and rows in
// L2), then the shared MLP's. `hint` is the expert of the caller's previous
// routed tile (a role visits its tiles in increasing order).
__device__ __forceinline__ Tile decode(const Sched& S, int i, int& hint) {
  Tile t;
  if (i < S.routed) {
    const int q = i / S.nb0;
    int e = hint;
    while (S.P[e + 1] <= q) ++e;
    hint = e;
    const int mt = S.P[e + 1] - S.P[e];
    const int l = i - S.nb0 * S.P[e];
    const int nb = l / mt, m = l % mt;
    t.kind = 0;
    t.e = e;
    t.row0 = S.off[e] + m * BM;
    t.rows = min(BM, S.off[e + 1] - t.row0);
    t.n0 = nb * S.bn;
  } else {
    const int l = i - S.routed;
    const int nb = l / S.mt_sh, m = l % S.mt_sh;
    t.kind = 1;
    t.e = 0;
    t.row0 = m * BM;
    t.rows = min(BM, S.t_shared - t.row0);
    t.n0 = nb * S.bn;
  }
  return t;
}

// Named barrier 1 over the eight epilogue warps that ORs a flag across them
// (every warp takes the same abort decision).
__device__ __forceinline__ bool epi8_sync_any(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag), "n"(32 * EPI_WARPS)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ void epi8_sync() {
  asm volatile("bar.sync 2, %0;" ::"n"(32 * EPI_WARPS) : "memory");
}

// Four k-blocks' scales of one row as UE8M0 bytes, k-block kb + j in byte j.
__device__ __forceinline__ uint32_t pack_scales(const float4& v) {
  return ue8m0(v.x) | (ue8m0(v.y) << 8) | (ue8m0(v.z) << 16) | (ue8m0(v.w) << 24);
}

template <bool UP>
__global__ void __launch_bounds__(NTHREADS, 1) grouped_fp8m_kernel(const __grid_constant__ Fp8mArgs g) {
  // DOWN: the combine after it may launch now (it waits for this grid
  // before it reads the outputs). UP lets the down-projection launch only
  // after its own prologue (below), once it has waited for its predecessors.
  if (!UP) asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* sfs = tiles + OFF_SFS;                              // [STAGES][SF_STAGE]
  uint8_t* stage = tiles + OFF_STAGE;                          // [EPI_WARPS][STAGE_WARP_BYTES]
  float* red = reinterpret_cast<float*>(tiles + OFF_RED);      // [2][BM] row maxima of the halves
  uint64_t* full = reinterpret_cast<uint64_t*>(tiles + OFF_BAR);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 1;
  uint64_t* drain = tempty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* P = reinterpret_cast<int32_t*>(tiles + OFF_P);
  int32_t* off = P + MAXE + 1;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int E = g.E;

  if (warp == 0) {
    if (lane == 0) {
      for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
      mbar_init(tfull, 1);
      mbar_init(tempty, 32 * EPI_WARPS);
      mbar_init(drain, 1);
      *abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    // UP, a programmatic dependent of the row quantization: wait for it
    // before anything it or the kernels before it wrote is read (the offsets
    // here; the codes and scales after the __syncthreads below). DOWN, a
    // programmatic dependent of the up-projection, reads here only what was
    // complete before that grid let it launch (the offsets); it waits for h
    // in its producer, after prefetching its first weight tiles.
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
  // so a dependent down-projection may read what they wrote (the offsets)
  // before it waits for this grid
  if (UP) asm volatile("griddepcontrol.launch_dependents;");

  Sched S;
  S.P = P;
  S.off = off;
  S.E = E;
  S.bn = UP ? QB : BN;   // output features per tile: UP 128 of h, DOWN 256
  S.nb0 = (g.n_out[0] + S.bn - 1) / S.bn;
  S.nb1 = g.t_shared > 0 ? (g.n_out[1] + S.bn - 1) / S.bn : 0;
  S.mt_sh = (g.t_shared + BM - 1) / BM;
  S.t_shared = g.t_shared;
  S.routed = S.nb0 * P[E];
  S.total = S.routed + S.nb1 * S.mt_sh;

  if (warp == 0) {
    // ---------------------------------------------------------------- TMA producer
    // Lane 0: barriers and the tile loads. Every lane: its row of each
    // group's scale images -- SFA words c = 0..3 for token rows lane + 32c,
    // SFB the weight blocks' bytes (the same in all rows). The scales are
    // loaded a group ahead (the next tile's first group and its weight
    // blocks' scales during the current tile's last group), after the
    // stage's copies are issued, so the producer does not wait on them.
    int s = 0, issued = 0, hint = 0, hint_n = 0;
    uint32_t ph = 0;
    bool ok = true;
    float4 nx[4];   // token scales of the next group: rows lane + 32c, four k-blocks
    float nw[4];    // weight-block scales of the next tile: w1 (or w2) and the second block, k-blocks lane, lane + 32
    auto load_group = [&](const Tile& t, int kb) {
      const int kbp = scale_stride(g.kdim[t.kind]);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int r = lane + 32 * c;
        if (r < t.rows)
          nx[c] = __ldg(reinterpret_cast<const float4*>(g.asc[t.kind] + (int64_t)(t.row0 + r) * kbp + kb));
      }
    };
    auto load_wscales = [&](const Tile& t) {
      const int kb_n = g.kdim[t.kind] / QB;
      const int nbw = g.n_out[t.kind] / QB;
      const bool two = UP || t.n0 + QB < g.n_out[t.kind];
      const float* pw1 = g.ws1[t.kind] + ((int64_t)t.e * nbw + t.n0 / QB) * kb_n;
      const float* pw3 = UP ? g.ws3[t.kind] + ((int64_t)t.e * nbw + t.n0 / QB) * kb_n : pw1 + kb_n;
      nw[0] = lane < kb_n ? __ldg(pw1 + lane) : 1.f;
      nw[1] = lane + 32 < kb_n ? __ldg(pw1 + lane + 32) : 1.f;
      nw[2] = two && lane < kb_n ? __ldg(pw3 + lane) : 1.f;
      nw[3] = two && lane + 32 < kb_n ? __ldg(pw3 + lane + 32) : 1.f;
    };
    int i = blockIdx.x;
    Tile t{};
    if (i < S.total) t = decode(S, i, hint);
    if (!UP) {
      // the first tile's leading weight k-blocks into L2 while the
      // up-projection finishes, then wait for it (h and its scales)
      if (lane == 0 && i < S.total) {
        const int kb_n = g.kdim[t.kind] / QB;
        const bool two0 = t.n0 + QB < g.n_out[t.kind];
        const int n_pf = min(kb_n, DOWN_PREFETCH_KB_BYTES / (2 * W_TILE));
        for (int kb = 0; kb < n_pf; ++kb) {
          tma_prefetch_3d(&g.tmW1[t.kind], kb * QB, t.n0, t.e);
          if (two0) tma_prefetch_3d(&g.tmW1[t.kind], kb * QB, t.n0 + QB, t.e);
        }
      }
      asm volatile("griddepcontrol.wait;" ::: "memory");
    }
    if (i < S.total) {
      load_group(t, 0);
      load_wscales(t);
    }
    for (; i < S.total; i += gridDim.x) {
      const int kb_n = g.kdim[t.kind] / QB;
      const bool two = UP || t.n0 + QB < g.n_out[t.kind];
      const int in = i + (int)gridDim.x;
      Tile tn{};
      if (in < S.total) tn = decode(S, in, hint_n);
      // this tile's weight-block scales as UE8M0 bytes (1.0 = byte 127 past
      // its k-blocks and for a missing second block)
      const uint32_t w1a = ue8m0(nw[0]), w1b = ue8m0(nw[1]), w3a = ue8m0(nw[2]), w3b = ue8m0(nw[3]);
      const uint32_t tx = (uint32_t)(A_TILE + (two ? 2 : 1) * W_TILE);
      const CUtensorMap* ta = &g.tmA[t.kind];
      if (t.kind == 0 && t.rows < BM && g.row_maps != nullptr) {
        ta = g.row_maps + t.e;
        if (lane == 0) tmap_acquire(ta);
      }
      for (int kb = 0; kb < kb_n; ++kb) {
        int w = 1;
        if (lane == 0) w = mbar_wait(&empty[s], ph ^ 1, abort_flag, g.err) ? 1 : 0;
        if (!__shfl_sync(0xffffffffu, w, 0)) { ok = false; break; }
        const bool gstart = (kb & 3) == 0;
        if (gstart) {
          // a group's first stage: the images of k-blocks kb .. kb + 3 (bytes
          // past the tile's k-blocks are not read). The stage's previous
          // MMAs, and the copies to TMEM before them, are complete: empty[s]
          // came from their commit.
          uint8_t* sf = sfs + s * SF_STAGE;
          uint32_t p1 = 0, p3 = 0;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int k = kb + j;
            p1 |= __shfl_sync(0xffffffffu, k < 32 ? w1a : w1b, k & 31) << (8 * j);
            p3 |= __shfl_sync(0xffffffffu, k < 32 ? w3a : w3b, k & 31) << (8 * j);
          }
          uint32_t wa[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) wa[c] = lane + 32 * c < t.rows ? pack_scales(nx[c]) : 0x7F7F7F7Fu;
          *reinterpret_cast<uint4*>(sf + lane * 16) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
          *reinterpret_cast<uint4*>(sf + SF_BYTES + lane * 16) = make_uint4(p1, p1, p1, p1);
          *reinterpret_cast<uint4*>(sf + 2 * SF_BYTES + lane * 16) = make_uint4(p3, p3, p3, p3);
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0) {
          uint8_t* sa = tiles + s * STAGE_BYTES;
          uint8_t* sb = sa + A_TILE;
          mbar_expect_tx(&full[s], tx);
          tma_load_2d(sa, ta, &full[s], kb * QB, t.row0);
          tma_load_3d(sb, &g.tmW1[t.kind], &full[s], kb * QB, t.n0, t.e);
          if (UP) tma_load_3d(sb + W_TILE, &g.tmW3[t.kind], &full[s], kb * QB, t.n0, t.e);
          else if (two) tma_load_3d(sb + W_TILE, &g.tmW1[t.kind], &full[s], kb * QB, t.n0 + QB, t.e);
        }
        __syncwarp();
        if (gstart) {
          // the next group's scales: this tile's, or the next tile's first
          // (with the next tile's weight-block scales)
          if (kb + 4 < kb_n) {
            load_group(t, kb + 4);
          } else if (in < S.total) {
            load_group(tn, 0);
            load_wscales(tn);
          }
        }
        ++issued;
        if (++s == STAGES) { s = 0; ph ^= 1; }
      }
      if (!ok) break;
      t = tn;
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
    // Per group of four stages the scale images to TMEM (tcgen05.cp, ordered
    // before the MMAs this thread issues after it); per stage four K = 32
    // block-scaled MMAs into the accumulator, which sums the whole K, reading
    // byte kb % 4 of the scale words; one commit per tile hands it to the
    // epilogue.
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
        // the epilogue has read the previous tile's accumulator
        if (!mbar_wait(tempty, ((uint32_t)lt & 1) ^ 1, abort_flag, g.err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d = tmem_base;
        for (int kb = 0; kb < kb_n; ++kb) {
          if (!mbar_wait(&full[s], ph, abort_flag, g.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(tiles + s * STAGE_BYTES);
          const uint32_t b0 = a0 + A_TILE;
          if ((kb & 3) == 0) {
            const uint32_t sf0 = smem_u32(sfs + s * SF_STAGE);
            tsa = tmem_base + (uint32_t)(SF_COL0 + (groups % SF_SLOTS) * SF_SLOT_COLS);
            ++groups;
            tmem_cp_sf(tsa, sdesc_sf(sf0));
            tmem_cp_sf(tsa + 4, sdesc_sf(sf0 + SF_BYTES));
            if (two) tmem_cp_sf(tsa + 8, sdesc_sf(sf0 + 2 * SF_BYTES));
          }
          // byte j = kb % 4 of the scale words: in the instruction descriptor
          // and, as the byte address, in the top two bits of the TMEM addresses
          const uint32_t j = (uint32_t)(kb & 3);
          const uint32_t idesc = idesc_mx_e4m3(BM, two ? BN : BN / 2, j);
          const uint32_t sfa = tsa | (j << 30), sfb = (tsa + 4) | (j << 30);
#pragma unroll
          for (int kk = 0; kk < QB / 32; ++kk)
            mma_mx(d, sdesc(a0 + kk * 32), sdesc(b0 + kk * 32), idesc, sfa, sfb, (kb | kk) != 0 ? 1u : 0u);
          tc_commit(&empty[s]);
          if (++s == STAGES) { s = 0; ph ^= 1; }
        }
        if (!ok) break;
        tc_commit(tfull);
      }
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    // A TMEM lane is a token row of the tile, a column a weight row. Two
    // threads per row: half 0 the first half of the row's columns (UP: h
    // features 0-63 of the tile, from a in columns 0-63 and b in 128-191;
    // DOWN: outputs 0-127), half 1 the second.
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;
    const int row = quad * 32 + lane;
    int hint = 0;
    for (int i = blockIdx.x, lt = 0; i < S.total; i += gridDim.x, ++lt) {
      const Tile t = decode(S, i, hint);
      const bool two = UP || t.n0 + QB < g.n_out[t.kind];
      bool ok;
      {
        int w = 1;
        if (lane == 0) w = mbar_wait(tfull, (uint32_t)lt & 1, abort_flag, g.err) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, w, 0) != 0;
      }
      // the row's 128 accumulator values (UP: a and b of this thread's 64
      // features, all loads in flight under one wait; DOWN: its 128
      // outputs); the accumulator is released before any other arithmetic,
      // so the next tile's MMAs wait only for these reads
      uint32_t u[128];
      if (ok) {
        tc_fence_after();
        const uint32_t tb = tmem_base + ((uint32_t)(quad * 32) << 16);
        if (UP) {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            tmem_ld16(tb + half * 64 + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&u[q * 16]));
            tmem_ld16(tb + QB + half * 64 + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&u[64 + q * 16]));
          }
          tmem_wait_ld();
        } else if (half == 0 || two) {
          // in two rounds of 64, each rounded to bf16 pairs at once (u[0..63]
          // then holds the row's 128 outputs as pairs)
#pragma unroll
          for (int hr = 0; hr < 2; ++hr) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
              tmem_ld16(tb + half * QB + hr * 64 + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&u[64 + q * 16]));
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(u[64 + 2 * j]),
                                                        __uint_as_float(u[64 + 2 * j + 1]));
              u[hr * 32 + j] = *reinterpret_cast<uint32_t*>(&b2);
            }
          }
        }
        tc_fence_before();
        mbar_arrive(tempty);
      }
      // one decision for all eight warps: stop if any of them gave up
      if (epi8_sync_any(!ok)) break;
      const int n_out = g.n_out[t.kind];
      if (UP) {
        // h = silu(a) * b (in place of a); the row's 1 x 128 block of h
        // takes the larger of the two halves' maxima
        float m = 0.f;
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          const float h = silu_f(__uint_as_float(u[j])) * __uint_as_float(u[64 + j]);
          u[j] = __float_as_uint(h);
          m = fmaxf(m, fabsf(h));
        }
        red[half * BM + row] = m;
        epi8_sync();
        const float amax = fmaxf(red[row], red[BM + row]);
        const int se = block_exp(amax);
        // 2^-se, exact (finite amax keeps se <= 120), so h * 2^-se rounds
        // exactly as the scaling of the oracle does
        const float p2 = __int_as_float((127 - se) << 23);
        if (row < t.rows) {
          uint8_t* hq = reinterpret_cast<uint8_t*>(g.out[t.kind]) + (int64_t)(t.row0 + row) * n_out +
                        t.n0 + half * 64;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t wd[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int j = q * 16 + c * 4;
              wd[c] = (uint32_t)to_e4m3(__uint_as_float(u[j]) * p2) |
                      ((uint32_t)to_e4m3(__uint_as_float(u[j + 1]) * p2) << 8) |
                      ((uint32_t)to_e4m3(__uint_as_float(u[j + 2]) * p2) << 16) |
                      ((uint32_t)to_e4m3(__uint_as_float(u[j + 3]) * p2) << 24);
            }
            *reinterpret_cast<uint4*>(hq + q * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
          }
          if (half == 0)
            g.out_scale[t.kind][(int64_t)(t.row0 + row) * scale_stride(n_out) + t.n0 / QB] = ldexpf(1.f, se);
        }
      } else if (half == 0 || two) {
        // bf16 outputs staged through this warp's 1 KB buffer, 16 columns at
        // a time: lane l writes its row's 32 bytes, then each store
        // instruction writes 16 rows x 32 bytes (whole sectors) instead of
        // 32 rows x 16 bytes. The 16-byte chunk c of row r sits at
        // c ^ ((r >> 2) & 1), which keeps both phases free of bank conflicts.
        uint8_t* buf = stage + (warp - 2) * STAGE_WARP_BYTES;
        __nv_bfloat16* ob = reinterpret_cast<__nv_bfloat16*>(g.out[t.kind]) + (int64_t)t.row0 * n_out +
                            t.n0 + half * QB;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int j = q * 8 + c * 4;
            *reinterpret_cast<uint4*>(buf + lane * 32 + ((c ^ ((lane >> 2) & 1)) * 16)) =
                make_uint4(u[j], u[j + 1], u[j + 2], u[j + 3]);
          }
          __syncwarp();
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int r = 16 * k2 + (lane >> 1), c = lane & 1;
            const uint4 val = *reinterpret_cast<const uint4*>(buf + r * 32 + ((c ^ ((r >> 2) & 1)) * 16));
            if (quad * 32 + r < t.rows)
              *reinterpret_cast<uint4*>(ob + (int64_t)(quad * 32 + r) * n_out + q * 16 + c * 8) = val;
          }
          __syncwarp();
        }
      }
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

}  // namespace

// The FP8 expert GEMMs of one layer in the token-on-M form: UP reads x's
// codes in expert order (xq_perm, scales xs_perm) and x itself for the shared
// MLP, and writes the quantized h and hs; DOWN reads them and writes y_perm
// and s (bf16).
cudaError_t launch_grouped_fp8m(const moe_config& c, int64_t T, const Fp8Weights& w,
                                const uint8_t* xq, const float* xs, const uint8_t* xq_perm,
                                const float* xs_perm, const int32_t* offsets, uint8_t* hq,
                                float* hsc, uint8_t* hsq, float* hss, void* y_perm, void* s,
                                const void* row_maps, uint32_t* err, int num_sms, cudaStream_t st) {
  const int E = c.n_routed, D = c.dim, I = c.moe_inter, Is = c.shared_inter;
  const int64_t Tk = T * c.topk;
  const bool sh = Is > 0;
  cudaError_t e;
  for (int pass = 0; pass < 2; ++pass) {
    const bool up = pass == 0;
    Fp8mArgs g;
    memset(&g, 0, sizeof(g));
    const int n0 = up ? I : D, k0 = up ? D : I, n1 = up ? Is : D, k1 = up ? D : Is;
    if (up) {
      if (!map_u8_tile(&g.tmA[0], xq_perm, (uint64_t)Tk, (uint64_t)D, BM)) return cudaErrorInvalidValue;
      g.asc[0] = xs_perm;
      if (!map_u8_weights(&g.tmW1[0], w.w1, E, I, D)) return cudaErrorInvalidValue;
      if (!map_u8_weights(&g.tmW3[0], w.w3, E, I, D)) return cudaErrorInvalidValue;
      g.ws1[0] = w.s1;
      g.ws3[0] = w.s3;
      g.out[0] = hq;
      g.out_scale[0] = hsc;
      if (sh) {
        if (!map_u8_tile(&g.tmA[1], xq, (uint64_t)T, (uint64_t)D, BM)) return cudaErrorInvalidValue;
        g.asc[1] = xs;
        if (!map_u8_weights(&g.tmW1[1], w.ws1, 1, Is, D)) return cudaErrorInvalidValue;
        if (!map_u8_weights(&g.tmW3[1], w.ws3, 1, Is, D)) return cudaErrorInvalidValue;
        g.ws1[1] = w.ss1;
        g.ws3[1] = w.ss3;
        g.out[1] = hsq;
        g.out_scale[1] = hss;
      }
    } else {
      if (!map_u8_tile(&g.tmA[0], hq, (uint64_t)Tk, (uint64_t)I, BM)) return cudaErrorInvalidValue;
      g.asc[0] = hsc;
      if (!map_u8_weights(&g.tmW1[0], w.w2, E, D, I)) return cudaErrorInvalidValue;
      g.ws1[0] = w.s2;
      g.out[0] = y_perm;
      if (sh) {
        if (!map_u8_tile(&g.tmA[1], hsq, (uint64_t)T, (uint64_t)Is, BM)) return cudaErrorInvalidValue;
        g.asc[1] = hss;
        if (!map_u8_weights(&g.tmW1[1], w.ws2, 1, D, Is)) return cudaErrorInvalidValue;
        g.ws1[1] = w.ss2;
        g.out[1] = s;
      }
    }
    if (!sh) {  // no shared group: its maps are never used, keep them valid
      g.tmA[1] = g.tmA[0];
      g.tmW1[1] = g.tmW1[0];
      g.tmW3[1] = g.tmW3[0];
    }
    if (!up) {  // DOWN reads w2 only
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
    // UP's maps over xq_perm first, then DOWN's over hq
    g.row_maps = row_maps ? static_cast<const CUtensorMap*>(row_maps) + (up ? 0 : E) : nullptr;
    const int bn = up ? QB : BN;   // output features per tile
    const int64_t bound = (int64_t)((n0 + bn - 1) / bn) * ((Tk + BM - 1) / BM + E) +
                          (sh ? (int64_t)((n1 + bn - 1) / bn) * ((T + BM - 1) / BM) : 0);
    const int grid = (int)(bound < num_sms ? bound : num_sms);
    if (grid > 0) {
      if (up) {
        e = cudaFuncSetAttribute(grouped_fp8m_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        // a programmatic dependent of the row quantization
        e = launch_pdl(pdl_ok(), grouped_fp8m_kernel<true>, dim3(grid), dim3(NTHREADS), SMEM_BYTES, st, g);
        if (e != cudaSuccess) return e;
      } else {
        e = cudaFuncSetAttribute(grouped_fp8m_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        // a programmatic dependent of the up-projection
        e = launch_pdl(pdl_ok(), grouped_fp8m_kernel<false>, dim3(grid), dim3(NTHREADS), SMEM_BYTES, st, g);
        if (e != cudaSuccess) return e;
      }
      if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    stage_mark(st);
  }
  return cudaSuccess;
}

}  // namespace moe
