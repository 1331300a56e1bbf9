// Host-side TMA tensor-map builders shared by the grouped GEMM passes (gemm_common.cuh).
#include <cstdlib>
#include <mutex>

#include "gemm_common.cuh"

namespace moe {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

}  // namespace

bool make_row_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                  uint32_t box_rows) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {static_cast<cuuint32_t>(kBK), box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_row_maps(RowMaps* maps, const void* ptr, uint64_t inner, uint64_t rows) {
  for (int i = 0; i < kNumBoxHeights; ++i)
    if (!make_row_map(&maps->m[i], ptr, inner, rows, static_cast<uint32_t>(kNMax >> i)))
      return false;
  return true;
}

bool make_weight_map(CUtensorMap* m, const void* ptr, uint64_t n_feat, uint64_t rows,
                     uint32_t blocks) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[3] = {64, rows, n_feat / 64};
  cuuint64_t strides[2] = {n_feat * 2, 128};
  cuuint32_t box[3] = {64, static_cast<cuuint32_t>(kBK), blocks};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_f32_tile_map(CUtensorMap* m, void* ptr, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 4};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, ptr, dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_u8_tile_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                      uint32_t box_inner, uint32_t box_rows) {
  auto enc = get_encode_fn();
  if (enc == nullptr) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

uint64_t wait_budget_ns() {
  static uint64_t budget = [] {
    const char* s = std::getenv("MOE_WAIT_BUDGET_NS");
    if (s != nullptr && *s) return static_cast<uint64_t>(std::strtoull(s, nullptr, 10));
    return static_cast<uint64_t>(2000000000ull);  // 2 s
  }();
  return budget;
}

}  // namespace moe
