// Internal launchers behind the C ABI (moe_b200.h). Arguments are validated by api.cu.
#pragma once
#include <cstddef>
#include <cstdint>
#include <mutex>
#include <utility>

#include <cuda_runtime.h>

#include "moe_b200.h"

namespace moe {

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// The permutation's metadata (counts, cu_seqlens, stable ranks) is computed by one
// thread-block cluster, with no workspace, for routing tables of up to kClusterMaxSlots flat
// slots and for any table with more experts than the cooperative kernel's shared-memory
// histograms hold; larger tables go to a cooperative grid over all SMs that keeps per-chunk
// counts in the caller's workspace. (Measured on B200: the cluster kernel takes 10 us at 8K
// slots and 29 us at 128K, the cooperative one 29-35 us over that range and 33 us at 512K,
// where the cluster kernel's 16 SMs need 80 us.)
#ifndef MOE_CLUSTER_MAX_SLOTS
#define MOE_CLUSTER_MAX_SLOTS (int64_t{1} << 17)
#endif
constexpr int64_t kClusterMaxSlots = MOE_CLUSTER_MAX_SLOTS;
constexpr int kCoopMaxExperts = 1024;
constexpr int kChunkSlots = 512;  // flat slots per warp (one chunk) in the cooperative kernel
constexpr int kWarpsPerTile = 8;

inline bool permute_uses_cluster(int64_t F, int32_t E) {
  return F <= kClusterMaxSlots || E > kCoopMaxExperts;
}

inline int64_t permute_num_chunks(int64_t F) { return ceil_div(F, kChunkSlots); }

// Number of SMs of the current device (cached per device).
int num_sms();

// Process-unique id of the CUDA context current on the calling thread, 0 when there is none
// yet (the runtime creates the primary context lazily, at the first call that needs it).
// Kernel attributes and device-symbol addresses belong to one context: a second context on
// the same device, or the primary context re-created after cudaDeviceReset, gets a new id
// even where the driver reuses the old handle value.
uint64_t current_context_id();

// A small thread-safe map from context id to a pointer-sized value: what a one-time set-up
// produced in that context. Ids that do not fit (more than kSlots contexts) are not cached,
// so their set-up simply runs again on every call.
class ContextCache {
 public:
  static constexpr int kSlots = 64;
  bool find(uint64_t ctx, void** value);
  void put(uint64_t ctx, void* value);

 private:
  std::mutex mu_;
  uint64_t ids_[kSlots] = {};
  void* values_[kSlots] = {};
  int n_ = 0;
};

// Sets `kernel`'s dynamic shared-memory limit to `bytes`, once per context (cached in `done`).
bool set_smem_optin(const void* kernel, int bytes, ContextCache& done);

// Launch `kernel` as a programmatic dependent launch: it may be scheduled while the previous
// kernel in the stream finishes, and waits for it (griddepcontrol.wait) before touching data
// that kernel produces. Falls back to an ordinary launch if the attribute is refused.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = 0;
    err = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  }
  return err;
}

// chunk_counts: the workspace (used by the cooperative path only; may be null otherwise).
moe_status launch_permute(const void* x, const int32_t* topk_ids, int64_t S, int64_t H, int32_t K,
                          int32_t E, void* x_perm, int32_t* counts, int32_t* cu_seqlens,
                          int32_t* row_id_map, int32_t* perm_src, double* maxvio,
                          int32_t* max_count, int32_t* chunk_counts, int32_t* d_status,
                          cudaStream_t stream);

moe_status launch_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, double* maxvio,
                         int32_t* max_count, cudaStream_t stream);

// Routing [S, K+n_shared]: the token's K routed slots, then experts E .. E+n_shared-1 with
// weight 1 (shared experts).
moe_status launch_append_shared(const int32_t* ids, const float* w, int64_t S, int32_t K,
                                int32_t E, int32_t n_shared, int32_t* ids_out, float* w_out,
                                cudaStream_t stream);

// route_w == nullptr: unit weights (the permutation's backward).
moe_status launch_combine(const void* y, const int32_t* row_id_map, const float* route_w,
                          int64_t S, int64_t H, int32_t K, void* out, cudaStream_t stream);

moe_status launch_combine_backward(const void* grad_out, const void* y, const int32_t* row_id_map,
                                   const float* route_w, int64_t S, int64_t H, int32_t K,
                                   void* grad_y, float* grad_w, cudaStream_t stream);

// One pass of the grouped FFN. dual: h = SwiGLU pass (w0 = gate, w1 = up, act = x_perm,
// out = h; gate_pre/up_pre non-null also stores the bf16 pre-activations); otherwise the down
// pass (w0 = down, act = h, out = y; gate_pre/up_pre must be null).
moe_status launch_ffn_pass(bool dual, const void* act, const void* w0, const void* w1,
                           const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp, int32_t E,
                           void* out, void* gate_pre, void* up_pre, int32_t* d_status,
                           cudaStream_t stream);

// The SwiGLU pass with its token rows gathered from the token-major x [S, H] (row r of the
// expert-grouped order is token perm_src[r] / K): h, and gate_pre/up_pre when non-null, as
// launch_ffn_pass(dual) on x_perm would produce them, without x_perm.
moe_status launch_ffn_up_gate_gather(const void* x, const int32_t* perm_src, int64_t S, int32_t K,
                                     const void* w_gate, const void* w_up,
                                     const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                     int32_t E, void* h, void* gate_pre, void* up_pre,
                                     int32_t* d_status, cudaStream_t stream);

// Backward of the down projection fused with the SwiGLU backward: from grad_y [M,H] and the
// saved pre-activations [M,H'], d_gate and d_up [M,H'] (bf16).
moe_status launch_ffn_down_backward(const void* grad_y, const void* w_down, const void* gate_pre,
                                    const void* up_pre, const int32_t* cu_seqlens, int64_t M,
                                    int64_t H, int64_t Hp, int32_t E, void* d_gate, void* d_up,
                                    int32_t* d_status, cudaStream_t stream);

// Backward of the up and gate projections to the input rows:
// grad_x_perm = d_gate W_gate^T + d_up W_up^T (bf16 [M,H]).
moe_status launch_ffn_up_gate_backward(const void* d_gate, const void* d_up, const void* w_gate,
                                       const void* w_up, const int32_t* cu_seqlens, int64_t M,
                                       int64_t H, int64_t Hp, int32_t E, void* grad_x_perm,
                                       int32_t* d_status, cudaStream_t stream);

// Weight gradients (fp32, written or added into): grad_w_gate = x^T d_gate, grad_w_up =
// x^T d_up ([E,H,H']), grad_w_down = h^T grad_y ([E,H',H]), sums over each expert's rows.
moe_status launch_ffn_weight_grad(const void* x_perm, const void* h, const void* d_gate,
                                  const void* d_up, const void* grad_y, const int32_t* cu_seqlens,
                                  int64_t M, int64_t H, int64_t Hp, int32_t E, float* grad_w_gate,
                                  float* grad_w_up, float* grad_w_down, bool accumulate,
                                  int32_t* d_status, cudaStream_t stream);

// MXFP8 (E4M3 elements, E8M0 scales per 32 elements along the reduction dimension; layouts in
// grouped_ffn_mx.cu). Weights [E][R][C] bf16 -> q [E][R][C] and chunked scales
// [E][C/128][R/128][512]; R and C multiples of 128.
moe_status launch_mx_quantize_weights(const void* w, int32_t E, int64_t R, int64_t C, void* q,
                                      void* sf, cudaStream_t stream);

// x [S][H] bf16 -> x_q [S*K][H] E4M3 and x_sf [S*K][H/32] at the rows of row_id_map.
moe_status launch_mx_permute_quantize(const void* x, int64_t S, int64_t H, int32_t K,
                                      const int32_t* row_id_map, void* xq, void* xsf,
                                      cudaStream_t stream);

// One MXFP8 pass. dual: h_q/h_sf = SwiGLU pass (w0 = gate, w1 = up, act = x_q/x_sf);
// otherwise y (bf16) = down pass (w0 = down, act = h_q/h_sf, out_sf unused).
moe_status launch_mx_ffn_pass(bool dual, const void* act_q, const void* act_sf, const void* w0_q,
                              const void* w0_sf, const void* w1_q, const void* w1_sf,
                              const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                              int32_t E, void* out, void* out_sf, int32_t* d_status,
                              cudaStream_t stream);

}  // namespace moe
