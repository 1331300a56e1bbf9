// Internal launchers behind the C ABI (moe_b200.h). Arguments are validated by api.cu.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "moe_b200.h"

namespace moe {

// Flat routing slots handled by one warp in the permutation kernels.
constexpr int kChunk = 512;
constexpr int kWarpsPerTile = 8;
constexpr int kTile = kChunk * kWarpsPerTile;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline int64_t permute_num_chunks(int64_t F) { return ceil_div(F, kChunk); }

// Number of SMs of the current device (cached per device).
int num_sms();

moe_status launch_permute(const void* x, const int32_t* topk_ids, int64_t S, int64_t H, int32_t K,
                          int32_t E, void* x_perm, int32_t* counts, int32_t* cu_seqlens,
                          int32_t* row_id_map, int32_t* perm_src, double* maxvio,
                          int32_t* max_count, int32_t* chunk_counts, int32_t* d_status,
                          cudaStream_t stream);

moe_status launch_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, double* maxvio,
                         int32_t* max_count, cudaStream_t stream);

moe_status launch_combine(const void* y, const int32_t* row_id_map, const float* route_w,
                          int64_t S, int64_t H, int32_t K, void* out, cudaStream_t stream);

// One pass of the grouped FFN. dual: h = SwiGLU pass (w0 = gate, w1 = up, act = x_perm,
// out = h); otherwise the down pass (w0 = down, act = h, out = y).
moe_status launch_ffn_pass(bool dual, const void* act, const void* w0, const void* w1,
                           const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp, int32_t E,
                           void* out, int32_t* d_status, cudaStream_t stream);

}  // namespace moe
