// Host side of the tensor-core helpers: TMA tensor-map encoding.
#include "tc_common.cuh"

namespace moe {
namespace tc {

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

bool map_2d(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {K, rows};
  cuuint64_t strides[1] = {K * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool map_gather(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t K) {
  return map_2d(m, ptr, rows, K, 1);
}

bool map_3d(CUtensorMap* m, const void* ptr, uint64_t E, uint64_t N, uint64_t K, uint32_t box_n) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {K, N, E};
  cuuint64_t strides[2] = {K * 2, N * K * 2};
  cuuint32_t box[3] = {64, box_n, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int map_pair_4d(CUtensorMap* m, const void* p, const void* q, uint64_t E, uint64_t N, uint64_t K,
                uint32_t box_n) {
  auto fn = encode_fn();
  if (!fn || !p || !q || p == q) return 0;
  const uintptr_t a = reinterpret_cast<uintptr_t>(p), b = reinterpret_cast<uintptr_t>(q);
  const uintptr_t lo = a < b ? a : b, dist = a < b ? b - a : a - b;
  if (dist % 16 != 0 || dist >= (uintptr_t(1) << 40) || dist < E * N * K * 2) return 0;
  cuuint64_t dims[4] = {K, N, E, 2};
  cuuint64_t strides[3] = {K * 2, N * K * 2, (cuuint64_t)dist};
  cuuint32_t box[4] = {64, box_n, 1, 2};
  cuuint32_t es[4] = {1, 1, 1, 1};
  if (fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, reinterpret_cast<void*>(lo), dims, strides, box, es,
         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return 0;
  return a < b ? 1 : 2;
}

}  // namespace tc
}  // namespace moe
