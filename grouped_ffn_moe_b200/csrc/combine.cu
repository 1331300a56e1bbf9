// Unpermute-combine: restore token order, scale by route weight, sum the K results.
//
// "Distributed expert parallelism" (open-llm-engineering), lifecycle step 8 (restore the
// original token indexes, multiply by route weights, sum the k results per token) and
// "Duplicate route accumulation" (add, never assign). MoonEP README, "combine fwd": bf16
// expert outputs in, bf16 token-major output, fp32 route weights.
//
//   out[t] = bf16( sum_{k ascending} w[t,k] * float(y[row_id_map[t*K+k]]) )
//
// One warp per (token, row slice of 32*U 16-byte vectors): each lane owns U = 4 vectors (8
// bf16 each) and keeps their fp32 sums in registers; the K source rows are loaded four slots
// at a time (16 loads in flight per lane) before the fixed-order FMAs consume them. Slicing
// the rows keeps every SM busy when there are few tokens.
#include <algorithm>
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"

#ifndef MOE_COMBINE_U
#define MOE_COMBINE_U 4      // 16-byte vectors per lane per pass
#endif
#ifndef MOE_COMBINE_SLOTS
#define MOE_COMBINE_SLOTS 4  // route slots whose loads are issued together
#endif

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void fma_bf16x8(float (&acc)[8], const uint4& v, float w) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    acc[2 * i] = fmaf(w, __uint_as_float(u[i] << 16), acc[2 * i]);
    acc[2 * i + 1] = fmaf(w, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
  }
}

__device__ __forceinline__ uint4 pack_bf16x8(const float (&acc)[8]) {
  uint32_t u[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t lo = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i]));
    const uint32_t hi = __bfloat16_as_ushort(__float2bfloat16_rn(acc[2 * i + 1]));
    u[i] = lo | (hi << 16);
  }
  return make_uint4(u[0], u[1], u[2], u[3]);
}

template <int U, int kSlots>
__global__ void __launch_bounds__(256) combine_kernel(const uint4* __restrict__ y,
                                                      const int32_t* __restrict__ row_id_map,
                                                      const float* __restrict__ route_w, int64_t S,
                                                      int64_t nvec, int32_t K,
                                                      uint4* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  griddep_wait();  // y and row_id_map come from earlier kernels in the stream
  griddep_launch_dependents();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t npass = (nvec + 32 * U - 1) / (32 * U);
  const int64_t items = S * npass;
  // the slot table of an item (lane k: row and weight of slot k), loaded one item ahead so
  // that its latency overlaps the previous item's row loads
  auto slot_of = [&](int64_t it, int32_t& row, float& wt) {
    row = -1;
    wt = 0.0f;
    if (it < items && lane < K) {
      const int64_t t = it / npass;
      row = row_id_map[t * K + lane];
      wt = route_w != nullptr ? route_w[t * K + lane] : 1.0f;
    }
  };
  int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  int32_t next_row;
  float next_w;
  slot_of(it, next_row, next_w);
  for (; it < items; it += nwarps) {
    const int64_t t = it / npass;
    const int64_t v0 = (it - t * npass) * (32 * U);
    const int32_t my_row = next_row;
    const float my_w = next_w;
    slot_of(it + nwarps, next_row, next_w);
    {
      float acc[U][8];
#pragma unroll
      for (int j = 0; j < U; ++j)
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[j][i] = 0.0f;
      for (int k0 = 0; k0 < K; k0 += kSlots) {
        uint4 r[kSlots][U];
        int32_t rows[kSlots];
        float ws[kSlots];
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
          const int k = k0 + s;
          if (K <= 32) {
            rows[s] = __shfl_sync(kFull, my_row, k & 31);
            ws[s] = __shfl_sync(kFull, my_w, k & 31);
          } else {
            rows[s] = (k < K) ? row_id_map[t * K + k] : -1;
            ws[s] = (k < K) ? (route_w != nullptr ? route_w[t * K + k] : 1.0f) : 0.0f;
          }
          if (k >= K) rows[s] = -1;
#pragma unroll
          for (int j = 0; j < U; ++j) {
            const int64_t v = v0 + j * 32 + lane;
            r[s][j] = (rows[s] >= 0 && v < nvec)
                          ? __ldg(y + static_cast<int64_t>(rows[s]) * nvec + v)
                          : make_uint4(0, 0, 0, 0);
          }
        }
#pragma unroll
        for (int s = 0; s < kSlots; ++s) {
          if (rows[s] < 0) continue;
#pragma unroll
          for (int j = 0; j < U; ++j) fma_bf16x8(acc[j], r[s][j], ws[s]);
        }
      }
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int64_t v = v0 + j * 32 + lane;
        if (v < nvec) out[t * nvec + v] = pack_bf16x8(acc[j]);
      }
    }
  }
}

// w * g rounded once to bf16, as the exact product would be: the fp32 product is taken
// rounded toward zero and its last bit set when inexact (rounding to odd, Boldo and
// Melquiond, "Emulation of FMA and correctly rounded sums: proved algorithms using rounding
// to odd"); with 24 >= 8 + 2 significand bits the bf16 round-to-nearest of that value equals
// the round-to-nearest of the exact product. The residual fmaf(w, g, -p) is exact.
__device__ __forceinline__ float mul_round_odd(float w, float g) {
  const float p = __fmul_rz(w, g);
  const float e = fmaf(w, g, -p);
  return (e != 0.0f) ? __uint_as_float(__float_as_uint(p) | 1u) : p;
}

// Backward of the combine (MoonEP README, "combine bwd": the output gradient goes back to the
// expert-grouped rows along the saved plan), for every token t and slot k:
//   grad_y[r(t,k)] = bf16(w[t,k] * grad_out[t])   (one rounding of the exact product)
//   grad_w[t,k]    = <grad_out[t], y[r(t,k)]>      (fp32, fixed summation order)
// One CTA of 8 warps per token: warp i takes the i-th eighth of the row's 16-byte vectors,
// and the slots go in groups of kBwdSlots whose rows' loads are in flight together. The dot
// product is summed per lane in vector order, then over the lanes by a fixed butterfly, then
// over the 8 warps in warp order through shared memory: deterministic. HBM traffic: grad_out
// once (re-read per slot group from L1/L2), y and grad_y once each.
constexpr int kBwdSlots = 4;
constexpr int kBwdWarps = 8;

__global__ void __launch_bounds__(32 * kBwdWarps) combine_backward_kernel(
    const uint4* __restrict__ grad_out, const uint4* __restrict__ y,
    const int32_t* __restrict__ row_id_map, const float* __restrict__ route_w, int64_t S,
    int64_t nvec, int32_t K, uint4* __restrict__ grad_y, float* __restrict__ grad_w) {
  __shared__ float s_dot[kBwdWarps][kBwdSlots];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  griddep_wait();
  griddep_launch_dependents();
  const int64_t per_warp = (nvec + kBwdWarps - 1) / kBwdWarps;
  const int64_t vb = min(static_cast<int64_t>(warp) * per_warp, nvec);
  const int64_t ve = min(vb + per_warp, nvec);
  for (int64_t t = blockIdx.x; t < S; t += gridDim.x) {
    const uint4* g = grad_out + t * nvec;
    for (int k0 = 0; k0 < K; k0 += kBwdSlots) {
      int32_t rows[kBwdSlots];
      float ws[kBwdSlots], dot[kBwdSlots];
#pragma unroll
      for (int s = 0; s < kBwdSlots; ++s) {
        const int k = k0 + s;
        rows[s] = k < K ? row_id_map[t * K + k] : -1;
        ws[s] = k < K ? route_w[t * K + k] : 0.0f;
        dot[s] = 0.0f;
      }
      for (int64_t v = vb + lane; v < ve; v += 32) {
        const uint4 gv = __ldg(g + v);
        uint4 yv[kBwdSlots];
#pragma unroll
        for (int s = 0; s < kBwdSlots; ++s)
          yv[s] = (rows[s] >= 0 && y != nullptr)
                      ? __ldg(y + static_cast<int64_t>(rows[s]) * nvec + v)
                      : make_uint4(0, 0, 0, 0);
        float gf[8];
        const uint32_t gu[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          gf[2 * i] = __uint_as_float(gu[i] << 16);
          gf[2 * i + 1] = __uint_as_float(gu[i] & 0xFFFF0000u);
        }
#pragma unroll
        for (int s = 0; s < kBwdSlots; ++s) {
          if (rows[s] < 0) continue;
          float sc[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) sc[i] = mul_round_odd(ws[s], gf[i]);
          grad_y[static_cast<int64_t>(rows[s]) * nvec + v] = pack_bf16x8(sc);
          const uint32_t yu[4] = {yv[s].x, yv[s].y, yv[s].z, yv[s].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            dot[s] = fmaf(gf[2 * i], __uint_as_float(yu[i] << 16), dot[s]);
            dot[s] = fmaf(gf[2 * i + 1], __uint_as_float(yu[i] & 0xFFFF0000u), dot[s]);
          }
        }
      }
      if (grad_w != nullptr) {
#pragma unroll
        for (int s = 0; s < kBwdSlots; ++s) {
#pragma unroll
          for (int d = 16; d > 0; d >>= 1) dot[s] += __shfl_xor_sync(kFull, dot[s], d);
        }
        if (lane == 0)
#pragma unroll
          for (int s = 0; s < kBwdSlots; ++s) s_dot[warp][s] = dot[s];
        __syncthreads();
        if (threadIdx.x < kBwdSlots && k0 + static_cast<int>(threadIdx.x) < K) {
          float sum = 0.0f;
          for (int i = 0; i < kBwdWarps; ++i) sum += s_dot[i][threadIdx.x];
          grad_w[t * K + k0 + threadIdx.x] = sum;
        }
        __syncthreads();  // s_dot is rewritten by the next slot group
      }
    }
  }
}

ContextCache g_combine_blocks;

// Resident 256-thread blocks of the combine kernel per SM (queried once per context).
int combine_blocks_per_sm() {
  void* v = nullptr;
  if (g_combine_blocks.find(current_context_id(), &v))
    return static_cast<int>(reinterpret_cast<intptr_t>(v));
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(
          &n, combine_kernel<MOE_COMBINE_U, MOE_COMBINE_SLOTS>, 256, 0) != cudaSuccess || n < 1) {
    (void)cudaGetLastError();
    n = 1;
  }
  g_combine_blocks.put(current_context_id(), reinterpret_cast<void*>(static_cast<intptr_t>(n)));
  return n;
}

}  // namespace

moe_status launch_combine_backward(const void* grad_out, const void* y, const int32_t* row_id_map,
                                   const float* route_w, int64_t S, int64_t H, int32_t K,
                                   void* grad_y, float* grad_w, cudaStream_t stream) {
  const int64_t nvec = H / 8;
  const int64_t blocks = std::min<int64_t>(S, static_cast<int64_t>(num_sms()) * 8);
  const cudaError_t err = launch_dependent(
      combine_backward_kernel, dim3(static_cast<unsigned>(blocks)), dim3(32 * kBwdWarps), 0,
      stream,
      static_cast<const uint4*>(grad_out), static_cast<const uint4*>(y), row_id_map, route_w, S,
      nvec, K, static_cast<uint4*>(grad_y), grad_w);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_combine(const void* y, const int32_t* row_id_map, const float* route_w,
                          int64_t S, int64_t H, int32_t K, void* out, cudaStream_t stream) {
  const int64_t nvec = H / 8;
  const int64_t items = S * ceil_div(nvec, 32 * MOE_COMBINE_U);
  // one resident wave of blocks: every warp strides over several items, loading each next
  // item's slot table while the current item's rows are in flight
  const int64_t blocks = std::min<int64_t>(
      ceil_div(items, 8), static_cast<int64_t>(num_sms()) * combine_blocks_per_sm());
  const cudaError_t err = launch_dependent(
      combine_kernel<MOE_COMBINE_U, MOE_COMBINE_SLOTS>, dim3(static_cast<unsigned>(blocks)),
      dim3(256), 0, stream, static_cast<const uint4*>(y), row_id_map, route_w, S, nvec, K,
      static_cast<uint4*>(out));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
