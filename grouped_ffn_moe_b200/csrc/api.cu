// C ABI entry points (include/moe_b200.h): argument validation, workspace sizing, launch.
// Nothing here allocates device memory or synchronises the host.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "internal.h"

namespace moe {

int num_sms() {
  static std::atomic<int> cache[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64) {
    const int v = cache[dev].load(std::memory_order_relaxed);
    if (v > 0) return v;
  }
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
    n = 148;
  if (dev < 64) cache[dev].store(n, std::memory_order_relaxed);
  return n;
}

namespace {

using PfnCtxGetCurrent = CUresult (*)(CUcontext*);
using PfnCtxGetId = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

}  // namespace

uint64_t current_context_id() {
  static const PfnCtxGetCurrent get_current = driver_fn<PfnCtxGetCurrent>("cuCtxGetCurrent");
  static const PfnCtxGetId get_id = driver_fn<PfnCtxGetId>("cuCtxGetId");
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return static_cast<uint64_t>(id) + 1;  // 0 stays "no context"
}

bool ContextCache::find(uint64_t ctx, void** value) {
  if (ctx == 0) return false;
  std::lock_guard<std::mutex> lock(mu_);
  for (int i = 0; i < n_; ++i)
    if (ids_[i] == ctx) {
      *value = values_[i];
      return true;
    }
  return false;
}

void ContextCache::put(uint64_t ctx, void* value) {
  if (ctx == 0) return;
  std::lock_guard<std::mutex> lock(mu_);
  for (int i = 0; i < n_; ++i)
    if (ids_[i] == ctx) {
      values_[i] = value;
      return;
    }
  if (n_ < kSlots) {
    ids_[n_] = ctx;
    values_[n_] = value;
    ++n_;
  }
}

bool set_smem_optin(const void* kernel, int bytes, ContextCache& done) {
  void* v = nullptr;
  if (done.find(current_context_id(), &v)) return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess)
    return false;
  done.put(current_context_id(), reinterpret_cast<void*>(uintptr_t{1}));  // context exists now
  return true;
}

namespace {

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr int64_t kMaxRows = (int64_t{1} << 31) - 1;

}  // namespace
}  // namespace moe

using moe::aligned;

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARGUMENT: return "invalid argument";
    case MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_BAD_ROUTING: return "expert id outside [0, E)";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    case MOE_ERR_BAD_ROUTING | MOE_ERR_DEVICE_TIMEOUT:
      return "expert id outside [0, E); device wait timed out";
    default: return "unknown status";
  }
}

int32_t moe_abi_version(void) { return (1 << 16) | 2; }

size_t moe_permute_workspace_bytes(int64_t S, int32_t K, int32_t E) {
  if (S <= 0 || K <= 0 || E <= 0) return 0;
  if (moe::permute_uses_cluster(S * K, E)) return 0;  // metadata in one cluster's shared memory
  const int64_t nchunk = moe::permute_num_chunks(S * K);
  const size_t bytes = sizeof(int32_t) * static_cast<size_t>(nchunk) * static_cast<size_t>(E);
  return (bytes + 255) & ~static_cast<size_t>(255);
}

moe_status moe_permute(const void* x, const int32_t* topk_ids, int64_t S, int64_t H, int32_t K,
                       int32_t E, void* x_perm, int32_t* counts, int32_t* cu_seqlens,
                       int32_t* row_id_map, int32_t* perm_src, double* maxvio, int32_t* max_count,
                       void* workspace, size_t workspace_bytes, int32_t* d_status,
                       void* cuda_stream) {
  if (S < 0 || K < 1 || E < 1 || K > E) return MOE_ERR_INVALID_ARGUMENT;
  if (E > MOE_MAX_EXPERTS) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!counts || !cu_seqlens) return MOE_ERR_INVALID_ARGUMENT;
  if (S > 0 && (!row_id_map || !topk_ids)) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned(counts, 4) || !aligned(cu_seqlens, 4) || !aligned(row_id_map, 4) ||
      !aligned(topk_ids, 4) || !aligned(perm_src, 4) || !aligned(max_count, 4) ||
      !aligned(maxvio, 8) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  if (x_perm != nullptr) {
    if ((S > 0 && x == nullptr) || H <= 0) return MOE_ERR_INVALID_ARGUMENT;
    if (H % 8 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(x, 16) || !aligned(x_perm, 16)) return MOE_ERR_INVALID_ARGUMENT;
  }
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if (S == 0) {
    // Nothing routed: zero counts and offsets; maxvio is undefined (T_bar = 0) -> NaN.
    if (cudaMemsetAsync(counts, 0, sizeof(int32_t) * E, stream) != cudaSuccess ||
        cudaMemsetAsync(cu_seqlens, 0, sizeof(int32_t) * (E + 1), stream) != cudaSuccess ||
        (max_count && cudaMemsetAsync(max_count, 0, sizeof(int32_t), stream) != cudaSuccess) ||
        (maxvio && cudaMemsetAsync(maxvio, 0xFF, sizeof(double), stream) != cudaSuccess))
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  const size_t need = moe_permute_workspace_bytes(S, K, E);
  if (need > 0 && (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 16)))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_permute(x, topk_ids, S, H, K, E, x_perm, counts, cu_seqlens, row_id_map,
                             perm_src, maxvio, max_count, static_cast<int32_t*>(workspace),
                             d_status, stream);
}

namespace {

moe_status check_ffn_shapes(int64_t M, int64_t H, int64_t Hp, int32_t E) {
  if (M < 0 || H <= 0 || Hp <= 0 || E < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (E > MOE_MAX_FFN_EXPERTS || M > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (H % 128 != 0 || Hp % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(E) * H > moe::kMaxRows || static_cast<int64_t>(E) * Hp > moe::kMaxRows)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  return MOE_OK;
}

bool ok_ptr16(const void* p) { return p != nullptr && aligned(p, 16); }

}  // namespace

moe_status moe_grouped_ffn_up_gate(const void* x_perm, const void* w_gate, const void* w_up,
                                   const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                   int32_t E, void* h_scratch, int32_t* d_status,
                                   void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  // no rows: nothing is read or written (row buffers may be NULL)
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(x_perm) || !ok_ptr16(w_gate) || !ok_ptr16(w_up) || !ok_ptr16(h_scratch) ||
      cu_seqlens == nullptr || !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_pass(true, x_perm, w_gate, w_up, cu_seqlens, M, H, Hp, E, h_scratch,
                              nullptr, nullptr, d_status, static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_down(const void* h_scratch, const void* w_down,
                                const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                int32_t E, void* y, int32_t* d_status, void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(h_scratch) || !ok_ptr16(w_down) || !ok_ptr16(y) || cu_seqlens == nullptr ||
      !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_pass(false, h_scratch, w_down, nullptr, cu_seqlens, M, H, Hp, E, y,
                              nullptr, nullptr, d_status, static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn(const void* x_perm, const void* w_gate, const void* w_up,
                           const void* w_down, const int32_t* cu_seqlens, int64_t M, int64_t H,
                           int64_t Hp, int32_t E, void* h_scratch, void* y, int32_t* d_status,
                           void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  // validate both passes before launching either
  if (!ok_ptr16(x_perm) || !ok_ptr16(w_gate) || !ok_ptr16(w_up) || !ok_ptr16(w_down) ||
      !ok_ptr16(h_scratch) || !ok_ptr16(y) || cu_seqlens == nullptr || !aligned(cu_seqlens, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  const moe_status s1 = moe_grouped_ffn_up_gate(x_perm, w_gate, w_up, cu_seqlens, M, H, Hp, E,
                                                h_scratch, d_status, cuda_stream);
  if (s1 != MOE_OK) return s1;
  return moe_grouped_ffn_down(h_scratch, w_down, cu_seqlens, M, H, Hp, E, y, d_status,
                              cuda_stream);
}

moe_status moe_grouped_ffn_up_gate_gather(const void* x, const int32_t* perm_src, int64_t S,
                                          int32_t K, const void* w_gate, const void* w_up,
                                          const int32_t* cu_seqlens, int64_t H, int64_t Hp,
                                          int32_t E, void* h_scratch, void* gate_pre,
                                          void* up_pre, int32_t* d_status, void* cuda_stream) {
  if (S < 0 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int64_t M = S * K;
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if ((gate_pre == nullptr) != (up_pre == nullptr)) return MOE_ERR_INVALID_ARGUMENT;
  if (!ok_ptr16(x) || perm_src == nullptr || !aligned(perm_src, 4) || !ok_ptr16(w_gate) ||
      !ok_ptr16(w_up) || !ok_ptr16(h_scratch) || !aligned(gate_pre, 16) ||
      !aligned(up_pre, 16) || cu_seqlens == nullptr || !aligned(cu_seqlens, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_up_gate_gather(x, perm_src, S, K, w_gate, w_up, cu_seqlens, M, H, Hp, E,
                                        h_scratch, gate_pre, up_pre, d_status,
                                        static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_gather(const void* x, const int32_t* perm_src, int64_t S, int32_t K,
                                  const void* w_gate, const void* w_up, const void* w_down,
                                  const int32_t* cu_seqlens, int64_t H, int64_t Hp, int32_t E,
                                  void* h_scratch, void* y, int32_t* d_status,
                                  void* cuda_stream) {
  if (S < 0 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  const int64_t M = S * K;
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  // validate both passes before launching either
  if (!ok_ptr16(x) || perm_src == nullptr || !aligned(perm_src, 4) || !ok_ptr16(w_gate) ||
      !ok_ptr16(w_up) || !ok_ptr16(w_down) || !ok_ptr16(h_scratch) || !ok_ptr16(y) ||
      cu_seqlens == nullptr || !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  const moe_status s1 =
      moe_grouped_ffn_up_gate_gather(x, perm_src, S, K, w_gate, w_up, cu_seqlens, H, Hp, E,
                                     h_scratch, nullptr, nullptr, d_status, cuda_stream);
  if (s1 != MOE_OK) return s1;
  return moe_grouped_ffn_down(h_scratch, w_down, cu_seqlens, M, H, Hp, E, y, d_status,
                              cuda_stream);
}

moe_status moe_grouped_ffn_up_gate_train(const void* x_perm, const void* w_gate,
                                         const void* w_up, const int32_t* cu_seqlens, int64_t M,
                                         int64_t H, int64_t Hp, int32_t E, void* h_scratch,
                                         void* gate_pre, void* up_pre, int32_t* d_status,
                                         void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(x_perm) || !ok_ptr16(w_gate) || !ok_ptr16(w_up) || !ok_ptr16(h_scratch) ||
      !ok_ptr16(gate_pre) || !ok_ptr16(up_pre) || cu_seqlens == nullptr ||
      !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_pass(true, x_perm, w_gate, w_up, cu_seqlens, M, H, Hp, E, h_scratch,
                              gate_pre, up_pre, d_status, static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_down_backward(const void* grad_y, const void* w_down,
                                         const void* gate_pre, const void* up_pre,
                                         const int32_t* cu_seqlens, int64_t M, int64_t H,
                                         int64_t Hp, int32_t E, void* d_gate, void* d_up,
                                         int32_t* d_status, void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(grad_y) || !ok_ptr16(w_down) || !ok_ptr16(gate_pre) || !ok_ptr16(up_pre) ||
      !ok_ptr16(d_gate) || !ok_ptr16(d_up) || cu_seqlens == nullptr || !aligned(cu_seqlens, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_down_backward(grad_y, w_down, gate_pre, up_pre, cu_seqlens, M, H, Hp, E,
                                       d_gate, d_up, d_status,
                                       static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_up_gate_backward(const void* d_gate, const void* d_up,
                                            const void* w_gate, const void* w_up,
                                            const int32_t* cu_seqlens, int64_t M, int64_t H,
                                            int64_t Hp, int32_t E, void* grad_x_perm,
                                            int32_t* d_status, void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(d_gate) || !ok_ptr16(d_up) || !ok_ptr16(w_gate) || !ok_ptr16(w_up) ||
      !ok_ptr16(grad_x_perm) || cu_seqlens == nullptr || !aligned(cu_seqlens, 4) ||
      !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_up_gate_backward(d_gate, d_up, w_gate, w_up, cu_seqlens, M, H, Hp, E,
                                          grad_x_perm, d_status,
                                          static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_weight_grad(const void* x_perm, const void* h, const void* d_gate,
                                       const void* d_up, const void* grad_y,
                                       const int32_t* cu_seqlens, int64_t M, int64_t H,
                                       int64_t Hp, int32_t E, float* grad_w_gate,
                                       float* grad_w_up, float* grad_w_down, int32_t accumulate,
                                       int32_t* d_status, void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (accumulate != 0 && accumulate != 1) return MOE_ERR_INVALID_ARGUMENT;
  if (!ok_ptr16(grad_w_gate) || !ok_ptr16(grad_w_up) || !ok_ptr16(grad_w_down) ||
      cu_seqlens == nullptr || !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  if (M == 0) {
    // no rows: every expert's gradient is zero
    if (accumulate) return MOE_OK;
    const size_t n = static_cast<size_t>(E) * H * Hp * sizeof(float);
    if (cudaMemsetAsync(grad_w_gate, 0, n, stream) != cudaSuccess ||
        cudaMemsetAsync(grad_w_up, 0, n, stream) != cudaSuccess ||
        cudaMemsetAsync(grad_w_down, 0, n, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  if (!ok_ptr16(x_perm) || !ok_ptr16(h) || !ok_ptr16(d_gate) || !ok_ptr16(d_up) ||
      !ok_ptr16(grad_y))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_ffn_weight_grad(x_perm, h, d_gate, d_up, grad_y, cu_seqlens, M, H, Hp, E,
                                     grad_w_gate, grad_w_up, grad_w_down, accumulate != 0,
                                     d_status, stream);
}

moe_status moe_grouped_ffn_backward(const void* x_perm, const void* h, const void* gate_pre,
                                    const void* up_pre, const void* w_gate, const void* w_up,
                                    const void* w_down, const int32_t* cu_seqlens, int64_t M,
                                    int64_t H, int64_t Hp, int32_t E, const void* grad_y,
                                    void* d_gate, void* d_up, void* grad_x_perm,
                                    float* grad_w_gate, float* grad_w_up, float* grad_w_down,
                                    int32_t accumulate, int32_t* d_status, void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  // validate all three passes before launching any
  if (accumulate != 0 && accumulate != 1) return MOE_ERR_INVALID_ARGUMENT;
  if (!ok_ptr16(grad_w_gate) || !ok_ptr16(grad_w_up) || !ok_ptr16(grad_w_down) ||
      cu_seqlens == nullptr || !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  if (M > 0 && (!ok_ptr16(x_perm) || !ok_ptr16(h) || !ok_ptr16(gate_pre) || !ok_ptr16(up_pre) ||
                !ok_ptr16(w_gate) || !ok_ptr16(w_up) || !ok_ptr16(w_down) ||
                !ok_ptr16(grad_y) || !ok_ptr16(d_gate) || !ok_ptr16(d_up) ||
                !ok_ptr16(grad_x_perm)))
    return MOE_ERR_INVALID_ARGUMENT;
  if (M > 0) {
    moe_status s = moe_grouped_ffn_down_backward(grad_y, w_down, gate_pre, up_pre, cu_seqlens, M,
                                                 H, Hp, E, d_gate, d_up, d_status, cuda_stream);
    if (s != MOE_OK) return s;
    s = moe_grouped_ffn_up_gate_backward(d_gate, d_up, w_gate, w_up, cu_seqlens, M, H, Hp, E,
                                         grad_x_perm, d_status, cuda_stream);
    if (s != MOE_OK) return s;
  }
  return moe_grouped_ffn_weight_grad(x_perm, h, d_gate, d_up, grad_y, cu_seqlens, M, H, Hp, E,
                                     grad_w_gate, grad_w_up, grad_w_down, accumulate, d_status,
                                     cuda_stream);
}

moe_status moe_unpermute_combine(const void* y, const int32_t* row_id_map, const float* route_w,
                                 int64_t S, int64_t H, int32_t K, void* out, void* cuda_stream) {
  if (S < 0 || H <= 0 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (H % 8 != 0 || S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (S == 0) return MOE_OK;
  if (!y || !row_id_map || !route_w || !out) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned(y, 16) || !aligned(out, 16) || !aligned(row_id_map, 4) || !aligned(route_w, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_combine(y, row_id_map, route_w, S, H, K, out,
                             static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_combine_backward(const void* grad_out, const void* y, const int32_t* row_id_map,
                                const float* route_w, int64_t S, int64_t H, int32_t K,
                                void* grad_y, float* grad_w, void* cuda_stream) {
  if (S < 0 || H <= 0 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (H % 8 != 0 || S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (S == 0) return MOE_OK;
  if (!grad_out || !row_id_map || !route_w || !grad_y || (grad_w && !y))
    return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned(grad_out, 16) || !aligned(grad_y, 16) || !aligned(y, 16) ||
      !aligned(row_id_map, 4) || !aligned(route_w, 4) || !aligned(grad_w, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_combine_backward(grad_out, grad_w != nullptr ? y : nullptr, row_id_map,
                                      route_w, S, H, K, grad_y, grad_w,
                                      static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_permute_backward(const void* grad_x_perm, const int32_t* row_id_map, int64_t S,
                                int64_t H, int32_t K, void* grad_x, void* cuda_stream) {
  if (S < 0 || H <= 0 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (H % 8 != 0 || S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (S == 0) return MOE_OK;
  if (!grad_x_perm || !row_id_map || !grad_x) return MOE_ERR_INVALID_ARGUMENT;
  if (!aligned(grad_x_perm, 16) || !aligned(grad_x, 16) || !aligned(row_id_map, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_combine(grad_x_perm, row_id_map, nullptr, S, H, K, grad_x,
                             static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_append_shared(const int32_t* topk_ids, const float* route_w, int64_t S, int32_t K,
                             int32_t E, int32_t n_shared, int32_t* ids_out, float* w_out,
                             void* cuda_stream) {
  if (S < 0 || K < 1 || E < 1 || n_shared < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (static_cast<int64_t>(E) + n_shared > MOE_MAX_EXPERTS ||
      S * (static_cast<int64_t>(K) + n_shared) > moe::kMaxRows)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  if (S == 0) return MOE_OK;
  if (!topk_ids || !route_w || !ids_out || !w_out || !aligned(topk_ids, 4) ||
      !aligned(route_w, 4) || !aligned(ids_out, 4) || !aligned(w_out, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_append_shared(topk_ids, route_w, S, K, E, n_shared, ids_out, w_out,
                                   static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, double* maxvio,
                      int32_t* max_count, void* cuda_stream) {
  if (E < 1 || S < 1 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (!counts || !maxvio || !aligned(counts, 4) || !aligned(maxvio, 8) || !aligned(max_count, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_maxvio(counts, E, S, K, maxvio, max_count,
                            static_cast<cudaStream_t>(cuda_stream));
}


// ----------------------------------------------------------------------------- MXFP8

size_t moe_mx_weight_scale_bytes(int32_t E, int64_t R, int64_t C) {
  if (E <= 0 || R <= 0 || C <= 0 || R % 128 != 0 || C % 128 != 0) return 0;
  return static_cast<size_t>(E) * static_cast<size_t>(R / 32) * static_cast<size_t>(C);
}

moe_status moe_mx_quantize_weights(const void* w, int32_t E, int64_t R, int64_t C, void* w_q,
                                   void* w_sf, void* cuda_stream) {
  if (E < 1 || R <= 0 || C <= 0) return MOE_ERR_INVALID_ARGUMENT;
  if (R % 128 != 0 || C % 128 != 0) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (static_cast<int64_t>(E) * R > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!ok_ptr16(w) || !ok_ptr16(w_q) || !ok_ptr16(w_sf)) return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_mx_quantize_weights(w, E, R, C, w_q, w_sf,
                                         static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_mx_permute_quantize(const void* x, const int32_t* row_id_map, int64_t S, int64_t H,
                                   int32_t K, void* x_q, void* x_sf, void* cuda_stream) {
  if (S < 0 || H <= 0 || K < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (H % 128 != 0 || S * K > moe::kMaxRows) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (S == 0) return MOE_OK;
  if (!ok_ptr16(x) || !ok_ptr16(x_q) || !ok_ptr16(x_sf) || row_id_map == nullptr ||
      !aligned(row_id_map, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_mx_permute_quantize(x, S, H, K, row_id_map, x_q, x_sf,
                                         static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_up_gate_mxfp8(const void* x_q, const void* x_sf, const void* w_gate_q,
                                         const void* w_gate_sf, const void* w_up_q,
                                         const void* w_up_sf, const int32_t* cu_seqlens, int64_t M,
                                         int64_t H, int64_t Hp, int32_t E, void* h_q, void* h_sf,
                                         int32_t* d_status, void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(x_q) || !ok_ptr16(x_sf) || !ok_ptr16(w_gate_q) || !ok_ptr16(w_gate_sf) ||
      !ok_ptr16(w_up_q) || !ok_ptr16(w_up_sf) || !ok_ptr16(h_q) || !ok_ptr16(h_sf) ||
      cu_seqlens == nullptr || !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_mx_ffn_pass(true, x_q, x_sf, w_gate_q, w_gate_sf, w_up_q, w_up_sf,
                                 cu_seqlens, M, H, Hp, E, h_q, h_sf, d_status,
                                 static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_down_mxfp8(const void* h_q, const void* h_sf, const void* w_down_q,
                                      const void* w_down_sf, const int32_t* cu_seqlens, int64_t M,
                                      int64_t H, int64_t Hp, int32_t E, void* y, int32_t* d_status,
                                      void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(h_q) || !ok_ptr16(h_sf) || !ok_ptr16(w_down_q) || !ok_ptr16(w_down_sf) ||
      !ok_ptr16(y) || cu_seqlens == nullptr || !aligned(cu_seqlens, 4) || !aligned(d_status, 4))
    return MOE_ERR_INVALID_ARGUMENT;
  return moe::launch_mx_ffn_pass(false, h_q, h_sf, w_down_q, w_down_sf, nullptr, nullptr,
                                 cu_seqlens, M, H, Hp, E, y, nullptr, d_status,
                                 static_cast<cudaStream_t>(cuda_stream));
}

moe_status moe_grouped_ffn_mxfp8(const void* x_q, const void* x_sf, const void* w_gate_q,
                                 const void* w_gate_sf, const void* w_up_q, const void* w_up_sf,
                                 const void* w_down_q, const void* w_down_sf,
                                 const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                 int32_t E, void* h_q, void* h_sf, void* y, int32_t* d_status,
                                 void* cuda_stream) {
  const moe_status st = check_ffn_shapes(M, H, Hp, E);
  if (st != MOE_OK) return st;
  if (M == 0) return MOE_OK;
  if (!ok_ptr16(w_down_q) || !ok_ptr16(w_down_sf) || !ok_ptr16(y))
    return MOE_ERR_INVALID_ARGUMENT;
  const moe_status s1 = moe_grouped_ffn_up_gate_mxfp8(x_q, x_sf, w_gate_q, w_gate_sf, w_up_q,
                                                      w_up_sf, cu_seqlens, M, H, Hp, E, h_q, h_sf,
                                                      d_status, cuda_stream);
  if (s1 != MOE_OK) return s1;
  return moe_grouped_ffn_down_mxfp8(h_q, h_sf, w_down_q, w_down_sf, cu_seqlens, M, H, Hp, E, y,
                                    d_status, cuda_stream);
}

}  // extern "C"
