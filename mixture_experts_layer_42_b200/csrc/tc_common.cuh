// Device helpers for the sm_100a tensor-core kernels: shared-memory
// addresses, mbarriers with bounded waits, TMA tiled loads, tcgen05 MMA /
// commit / TMEM loads and fences, UMMA shared-memory and instruction
// descriptors, and host-side TMA tensor-map encoding.
#pragma once

#include "common.cuh"

#include <cuda.h>
#include <cudaTypedefs.h>

namespace moe {
namespace tc {

constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;   // 1 s: no legitimate wait comes close
constexpr uint64_t DRAIN_LIMIT_NS = 20000000ull;    // 20 ms, only while draining after an abort

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

// try_wait that lets the thread sleep in hardware for up to ~1 us while the
// phase is still pending, instead of spinning on the issue slots the other
// warps of its SM sub-partition need.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(1000u)
      : "memory");
  return ok != 0;
}

// Slow path of mbar_wait: poll with sleeping try_waits, giving up when
// another role has raised the abort flag or after WAIT_LIMIT_NS (then raises
// it); both are checked every 64 polls.
static __device__ __noinline__ bool mbar_wait_slow(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort_flag, uint32_t* err) {
  const uint64_t t0 = globaltimer();
  for (uint32_t n = 1;; ++n) {
    if (mbar_try_wait_sleep(bar, parity)) return true;
    if ((n & 63) == 0) {
      if (*abort_flag) return false;
      if (globaltimer() - t0 > WAIT_LIMIT_NS) {
        *abort_flag = 1;
        set_error(err, ERRBIT_TIMEOUT);
        return false;
      }
    }
  }
}

// Wait for the phase of `bar` with the given parity (bounded, see
// mbar_wait_slow). The first try is inline: on the pipeline's critical path
// the phase has usually completed already.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  return mbar_wait_slow(bar, parity, abort_flag, err);
}

// Bounded wait used only while draining after an abort.
static __device__ __noinline__ void mbar_drain(uint64_t* bar, uint32_t parity) {
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

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0,
                                            int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

// One box of a 3D tensor into L2 only (no shared-memory destination, no
// barrier): the down-projection's first weight tiles, fetched while the
// up-projection before it finishes.
__device__ __forceinline__ void tma_prefetch_3d(const CUtensorMap* tm, int c0, int c1, int c2) {
  asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(tm), "r"(c0),
               "r"(c1), "r"(c2)
               : "memory");
}

// k-blocks of a down-projection CTA's first tile prefetched into L2 before
// it waits for the up-projection (256 KB per CTA, ~38 MB over the GPU).
constexpr int DOWN_PREFETCH_KB_BYTES = 256 * 1024;

// Four rows of a 2D tensor (a map whose box is 64 elements x 1 row) into
// shared memory as one 4-row, 512-byte piece of a 128-byte-swizzled tile: row
// coordinates r0..r3 may be anything (an out-of-range row reads zeros), the
// column coordinate c0 selects the 64-element slice. The swizzle follows the
// destination address, so `dst` at a 512-byte offset inside a 1024-byte-
// aligned tile gives the same bytes as one tile load of those rows.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* tm, uint64_t* bar, int c0,
                                            int r0, int r1, int r2, int r3) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(smem_u32(bar)), "r"(c0), "r"(r0), "r"(r1), "r"(r2), "r"(r3)
      : "memory");
}

// Contiguous bytes (a multiple of 16, both addresses 16-byte aligned) from
// global to shared memory, completing on an mbarrier (non-tensor bulk copy).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Make a tensor map written to global memory through the generic proxy
// (tensormap.cp_fenceproxy ... release) visible to this thread's TMA loads.
__device__ __forceinline__ void tmap_acquire(const void* map) {
  asm volatile("fence.proxy.tensormap::generic.acquire.gpu [%0], 128;" ::"l"(map) : "memory");
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
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
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

// ---------------------------------------------------------------- CTA pairs
// (cluster of two CTAs running tcgen05 cta_group::2 MMAs)

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Address of the same shared-memory location in CTA `cta` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t cta) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(cta));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// TMA load into this CTA's shared memory whose completion is counted on the
// mbarrier at `bar` (a shared::cluster address, here the leader's).
__device__ __forceinline__ void tma2_load_2d(void* dst, const CUtensorMap* tm, uint32_t bar, int c0,
                                             int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma2_load_3d(void* dst, const CUtensorMap* tm, uint32_t bar, int c0,
                                             int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ void tma2_load_4d(void* dst, const CUtensorMap* tm, uint32_t bar, int c0,
                                             int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
      "l"(tm), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}

__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the mbarrier at the same offset in both CTAs of the pair once
// every MMA issued so far by this thread has completed.
__device__ __forceinline__ void commit_pair(uint64_t* bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
      "[%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar)
               : "memory");
}

// kind::f16 instruction descriptor: fp32 accumulator, bf16 A and B, both
// K-major, the given M and N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Operands of one grouped expert launch on the tensor cores: [0] routed
// experts (A rows expert-contiguous, B stacked per expert), [1] the shared MLP.
// Named barrier 1 over the four epilogue warps that also ORs a flag across
// them, so that every warp takes the same abort decision before the next
// barrier (a warp that left alone would leave the others waiting).
__device__ __forceinline__ bool epi_sync_any(bool flag) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "barrier.cta.red.or.pred q, 1, 128, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)flag)
      : "memory");
  return r != 0;
}

struct TcArgs {
  CUtensorMap tmA[2];   // [0] routed A rows, [1] shared A rows; 2D {K, rows}
  CUtensorMap tmA64[2]; // the same with 64-row boxes (CTA-pair tail chunks)
  CUtensorMap tmB1[2];  // w1 (UP) / w2 (DOWN) as 3D {K, N, E}; shared: E = 1
  CUtensorMap tmB3[2];  // w3 / ws3 (UP only)
  // UP only: w1 and w3 as one 4D map {K, N, E, 2} whose last stride is the
  // distance between the two tensors, so one TMA box brings the w1 tile and
  // the w3 tile; b13 = 0 when unavailable, 1 when w1 is the lower address
  // (smem: w1 rows, then w3 rows), 2 when w3 is (smem: w3 rows, then w1).
  // Boxes hold 128 rows of each for one CTA, 64 for a CTA pair.
  CUtensorMap tmB13[2];
  int b13[2];
  // UP, one-CTA kernel: when `src` is set, the routed A rows are not read
  // from an expert-contiguous copy but gathered from the token rows x [gT, K]
  // through tmG (box 64 x 1 row, tile::gather4): row p of the expert order is
  // token src[p]; rows past an expert's end are given the out-of-range row gT
  // and read as zeros.
  CUtensorMap tmG;
  const int32_t* src;
  int gT;
  void* out[2];
  int n_out[2];         // output columns: UP I / I_s, DOWN D / D
  int kdim[2];          // reduction depth: UP D / D, DOWN I / I_s
  const int32_t* offsets;
  // One-CTA kernel: [E] copies of tmA[0] whose row extent ends at the
  // expert's last row (offsets[e + 1]), so that a tile reaching past it reads
  // zeros there (written by build_row_maps_kernel before the launch); null
  // when the routed A rows are gathered or the maps are not built.
  const CUtensorMap* row_maps;
  // One-CTA kernel: the launch's tile counter (zeroed by build_row_maps_kernel
  // before it); CTAs take tiles from it in order instead of round-robin by
  // CTA index. Null: round-robin.
  int* tile_ctr;
  // Test hook (moe_debug_stall_pipeline): CTA 0's MMA thread first waits on
  // a barrier phase that nothing completes, so that wait runs out (1 s)
  // before anything is issued, and the launch takes its abort path.
  int stall;
  int E;
  int t_shared;         // rows of the shared group (0: none)
  uint32_t* err;
};

// Launch the CTA-pair grouped GEMM (gemm_tc2.cu) on `pairs` clusters.
cudaError_t launch_grouped_tc2(bool up, const TcArgs& g, int pairs, cudaStream_t st);


// Host: TMA tensor-map encoder from the driver, without linking libcuda.
PFN_cuTensorMapEncodeTiled_v12000 encode_fn();

// 2D bf16 map over a row-major [rows, K] matrix, box 64 (K) x box_rows,
// 128-byte swizzle, zero fill out of bounds.
bool map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K, uint32_t box_rows);

// 2D bf16 map over a row-major [rows, K] matrix for tile::gather4 loads: box
// 64 (K) x 1 row, 128-byte swizzle, zero fill out of bounds.
bool map_gather(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K);

// 3D bf16 map over stacked matrices [E, N, K], box 64 (K) x box_n x 1.
bool map_3d(CUtensorMap* m, const void* ptr, uint64_t E, uint64_t N, uint64_t K, uint32_t box_n);

// 4D bf16 map over two same-shaped stacks [E, N, K] at p and q, box
// 64 x box_n x 1 x 2 (the p tile then the q tile, or q then p when q is the
// lower address). Returns 0 if the pair cannot be described (equal pointers,
// or a distance TMA cannot stride), else 1 (p first) or 2 (q first).
int map_pair_4d(CUtensorMap* m, const void* p, const void* q, uint64_t E, uint64_t N, uint64_t K,
                uint32_t box_n);

}  // namespace tc

using tc::launch_grouped_tc2;
using tc::TcArgs;

}  // namespace moe
