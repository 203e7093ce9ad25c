// Device helpers shared by the two FP8 (e4m3, block-scaled) expert GEMM
// kernels: the token-on-N form for small batches (gemm_fp8.cu) and the
// token-on-M form for large ones (gemm_fp8m.cu). Both read the same layout:
// e4m3 values, one power-of-two scale per 128 x 128 block of a weight matrix
// [out, in] and per 1 x 128 block of an activation row, every scale one
// UE8M0 byte (2^-127 .. 2^127); the tensor core applies the scales
// (tcgen05.mma kind::mxf8f6f4 with block scaling, one scale vector per 32 K).
#pragma once

#include "tc_common.cuh"

#include <cuda_fp8.h>

namespace moe {
namespace fp8 {

using namespace tc;

constexpr int QB = 128;   // scale block edge; K per pipeline stage

// kind::mxf8f6f4 block-scaled instruction descriptor: e4m3 A and B, both
// K-major, fp32 accumulator, UE8M0 scale factors (bit 23), byte `sf` of A's
// and B's TMEM scale words (bits 29-30 and 4-5), M x N.
__host__ __device__ constexpr uint32_t idesc_mx_e4m3(int M, int N, uint32_t sf) {
  return (sf << 4) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
         (sf << 29);
}

// D[M x N] (+)= (A * 2^SFA) (B * 2^SFB)^T over K = 32: one UE8M0 scale per row
// of A and per row of B (tcgen05 block scaling, one scale vector per 32 K).
__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
      : "memory");
}

// Shared-memory descriptor of a 32 x 16-byte matrix, no swizzle, rows 16
// bytes apart (8-row core matrices 128 bytes apart): the source of a
// tcgen05.cp 32x128b.
__device__ __forceinline__ uint64_t sdesc_sf(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFF) >> 4) | ((uint64_t)(128 >> 4) << 16) |
         ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}

// TMEM lanes 32w + r (w = 0..3) <- shared row r (16 bytes), r = 0..31.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// The UE8M0 byte of a power-of-two scale 2^s, -127 <= s <= 127: the biased
// exponent field of its fp32 encoding (2^-127 is the subnormal with a zero
// exponent field, which is UE8M0's code 0).
__device__ __forceinline__ uint32_t ue8m0(float scale) {
  return (__float_as_uint(scale) >> 23) & 0xFFu;
}

// Row stride, in floats, of the activation scales inside the layer: K/128
// rounded up to a multiple of 4, so every row starts 16-byte aligned and a
// tile's rows can be copied in one bulk copy.
__host__ __device__ __forceinline__ int scale_stride(int K) { return ((K / QB) + 3) & ~3; }

// Smallest s with amax <= 448 * 2^s (0 for amax == 0), and at least -127,
// the smallest scale UE8M0 encodes (blocks whose largest magnitude is below
// 448 * 2^-127 keep that scale): amax = m 2^e with 0.5 <= m < 1, so s = e - 9,
// plus one when 2m > 1.75.
__device__ __forceinline__ int block_exp(float amax) {
  if (!(amax > 0.f)) return 0;
  int e;
  const float m = frexpf(amax, &e);
  const int s = e - 9 + (2.f * m > 1.75f ? 1 : 0);
  return s < -127 ? -127 : s;
}

// (Values are brought into range with ldexpf(v, -s): the reciprocal 2^-s of
// a tiny block's scale would overflow fp32, the scaled value does not.)
__device__ __forceinline__ uint8_t to_e4m3(float v) {
  return (uint8_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float silu_f(float u) { return u / (1.0f + __expf(-u)); }

// Host: TMA maps over e4m3 tensors (128-byte swizzle, zero fill out of
// bounds). Rows [rows, K] with a 128 x 1 box (tile::gather4 loads); rows
// [rows, K] with a 128 x box_rows box (tile loads); stacked weights [E, N, K]
// with a 128 x 128 x 1 box.
bool map_u8_rows(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K);
bool map_u8_tile(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K, uint32_t box_rows);
bool map_u8_weights(CUtensorMap* m, const void* ptr, uint64_t E, uint64_t N, uint64_t K);

}  // namespace fp8
}  // namespace moe
