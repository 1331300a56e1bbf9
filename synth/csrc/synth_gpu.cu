// Seeded synthetic inputs for the MoE layer: device twin of synth_host.c.
//
// Fills large bf16 tensors (token activations, expert weights) on the GPU with
// the same counter-based SplitMix64 stream and Box-Muller cosine branch as the
// host generator, so that a weight tensor of tens of GB is made in milliseconds
// and any slice of it can be re-made on the host. No floating-point contraction
// (built with --fmad=false), so the device performs the same IEEE operations as
// the host; the only possible difference is the last ulp of log/cos, which moves
// a bf16 value only when a double lands within one ulp of a rounding boundary.
#include <cstdint>
#include <cuda_runtime.h>

namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ULL;
constexpr double kTwoPi = 6.283185307179586;

__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

__device__ __forceinline__ double unit_open(uint64_t r) {
  return ((double)(r >> 12) + 0.5) * 0x1p-52;
}

__device__ __forceinline__ uint16_t float_to_bf16_rne(float f) {
  uint32_t b = __float_as_uint(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

__global__ void normal_bf16_kernel(uint64_t key, uint64_t offset, int64_t n, double scale,
                                   uint16_t* __restrict__ out) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride) {
    const uint64_t j = offset + (uint64_t)i;
    const double u1 = unit_open(mix64(key + (2ULL * j + 1ULL) * kGamma));
    const double u2 = unit_open(mix64(key + (2ULL * j + 2ULL) * kGamma));
    const double v = sqrt(-2.0 * log(u1)) * cos(kTwoPi * u2) * scale;
    out[i] = float_to_bf16_rne((float)v);
  }
}

}  // namespace

extern "C" int synth_normal_bf16_gpu(uint64_t seed, uint64_t tag, uint64_t offset, int64_t n,
                                     double scale, void* out, void* stream) {
  if (n <= 0) return 0;
  if (out == nullptr) return 1;
  const uint64_t key = mix64(seed * kGamma + tag);
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 32) blocks = 148 * 32;
  normal_bf16_kernel<<<blocks, 256, 0, (cudaStream_t)stream>>>(key, offset, n, scale,
                                                               (uint16_t*)out);
  return cudaGetLastError() == cudaSuccess ? 0 : 3;
}
