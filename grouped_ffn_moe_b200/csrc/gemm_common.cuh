// Pieces shared by the grouped expert GEMM kernels (forward passes in grouped_ffn.cu,
// backward passes in grouped_ffn_bwd.cu): tile constants, the token-row tensor maps, the
// work-unit decomposition over expert-contiguous rows, and the host-side tensor-map builders.
//
// Experts own contiguous row blocks [cu[e], cu[e+1]) of the activation matrices (MoonEP
// README, "Integration": cu_seqlens selects each expert's rows of one contiguous tensor).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "internal.h"
#include "ptx.cuh"

namespace moe {

constexpr int kBM = 128;                       // output rows per tile (UMMA M)
constexpr int kBK = 64;                        // reduction elements per stage (128 bytes)
constexpr int kNMax = 256;                     // tokens per unit (UMMA N max)
constexpr int kABytes = kBM * kBK * 2;         // 16 KB: one 128 x 64 bf16 operand tile
constexpr int kAHalfBytes = 64 * kBK * 2;      // 8 KB: 64 MN-contiguous elements x 64 k
constexpr int kRowBytes = kBK * 2;             // one 64-element row of a K-major tile
constexpr int kNumBoxHeights = 5;              // token boxes of 256, 128, 64, 32, 16 rows
constexpr int kEpiGroups = 2;                  // epilogue warp groups, alternating chunks
constexpr int kEpiThreads = 128 * kEpiGroups;
constexpr int kThreads = 64 + kEpiThreads;     // TMA warp, MMA warp, epilogue warps
constexpr int kOutChunk = 32;                  // TMEM columns per epilogue chunk
constexpr int kOutBytes = kOutChunk * kBM * 2; // 8 KB bf16 staging buffer per group
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kAccCols = 256;
// After a time-out, waits for this CTA's own copies and MMAs to land use this fixed bound
// (not the caller's budget, which may be tiny), so that nothing is in flight at exit.
constexpr uint64_t kDrainBudgetNs = 200000000ull;

// Token-row tensor maps of one activation matrix, box heights 256, 128, 64, 32, 16 rows: a
// unit's N rows (a multiple of 16) load as the binary decomposition of N, i.e. at most five
// boxes and no row beyond the 16-row rounding.
struct RowMaps {
  CUtensorMap m[kNumBoxHeights];
};

// A unit of a token-chunked pass: expert e, feature block fb, rows [row0, row0 + nrows).
struct Unit {
  int e, fb, row0, nrows, ntc;
};

// Unit u -> (expert, feature block, token rows). s_ustart[e] is the first unit of expert e;
// an expert's rows are cut into ntc balanced chunks of at most kNMaxU rows (multiples of 16).
template <int kNMaxU = kNMax>
__device__ __forceinline__ Unit decode_unit(int u, const int32_t* s_ustart, const int32_t* s_cu,
                                            int E) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (s_ustart[mid] <= u) lo = mid; else hi = mid - 1;
  }
  Unit U;
  U.e = lo;
  const int local = u - s_ustart[lo];
  const int cnt = s_cu[lo + 1] - s_cu[lo];
  const int ntc = (cnt + kNMaxU - 1) / kNMaxU;
  U.ntc = ntc;
  U.fb = local / ntc;
  const int tc = local - U.fb * ntc;
  const int cs = (((cnt + ntc - 1) / ntc) + 15) & ~15;  // balanced chunks, multiple of 16
  const int r0 = tc * cs;
  U.row0 = s_cu[lo] + r0;
  U.nrows = min(cnt - r0, cs);
  return U;
}

__device__ __forceinline__ uint8_t* align_1024(uint8_t* p) {
  const uint32_t a = smem_u32(p);
  return p + ((1024u - (a & 1023u)) & 1023u);
}

// Block prologue, called by all kNT threads of the block: s_cu = cu_seqlens clamped to
// [0, M] (so that no row outside [0, M) is ever addressed), s_ustart[e] = first unit of
// expert e with ceil(rows / nmax) * nfb units per non-empty expert, s_ustart[E] = total
// units. s_scan holds kNT / 32 ints.
template <int kNT = kThreads>
__device__ __forceinline__ void unit_starts(const int32_t* cu, int64_t M, int E, int nfb,
                                            int nmax, int32_t* s_cu, int32_t* s_ustart,
                                            int32_t* s_scan) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  for (int e = tid; e <= E; e += kNT) {
    int64_t v = cu[e];
    v = v < 0 ? 0 : (v > M ? M : v);
    s_cu[e] = static_cast<int32_t>(v);
  }
  __syncthreads();
  const int per = (E + kNT - 1) / kNT;  // <= 4 for E <= 1024
  const int beg = min(tid * per, E), end = min(beg + per, E);
  int local = 0;
  for (int e = beg; e < end; ++e) {
    const int cnt = s_cu[e + 1] - s_cu[e];
    const int units = cnt > 0 ? ((cnt + nmax - 1) / nmax) * nfb : 0;
    s_ustart[e] = units;
    local += units;
  }
  int incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, d);
    if (lane >= d) incl += n;
  }
  if (lane == 31) s_scan[warp] = incl;
  __syncthreads();
  int off = 0;
  for (int w = 0; w < warp; ++w) off += s_scan[w];
  int run = off + incl - local;
  for (int e = beg; e < end; ++e) {
    const int units = s_ustart[e];
    s_ustart[e] = run;
    run += units;
  }
  if (tid == kNT - 1) s_ustart[E] = off + incl;
}

// ----------------------------------------------------------------------------- host side
// (tensor_maps.cu)

// Token rows of a row-major bf16 matrix [rows, inner], box (64 x box_rows), 128-byte swizzle:
// a K-major operand tile whose rows are tokens (or weight rows).
bool make_row_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                  uint32_t box_rows);
// The five token-row maps (256 ... 16 rows) of one activation matrix.
bool make_row_maps(RowMaps* maps, const void* ptr, uint64_t inner, uint64_t rows);
// A row-major bf16 matrix [rows][n_feat] viewed as (64 features, rows, n_feat / 64) with a
// (64 x 64 x blocks) box: an MN-major operand tile of 64 * blocks features x 64 rows, laid
// out as `blocks` 8 KB 64-feature slices, 128-byte swizzle.
bool make_weight_map(CUtensorMap* m, const void* ptr, uint64_t n_feat, uint64_t rows,
                     uint32_t blocks = 2);
// A row-major fp32 matrix [rows][inner] with a (box_inner x box_rows) box, 128-byte swizzle
// (box_inner * 4 must be 128): the staging layout of a TMA store or reduce-add.
bool make_f32_tile_map(CUtensorMap* m, void* ptr, uint64_t inner, uint64_t rows,
                       uint32_t box_inner, uint32_t box_rows);
// Bound, in nanoseconds, of every pipeline wait in the GEMM kernels (MOE_WAIT_BUDGET_NS).
uint64_t wait_budget_ns();

}  // namespace moe
