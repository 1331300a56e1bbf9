// Route permutation into expert-contiguous order, and the row copy that goes with it.
//
// Follows "Distributed expert parallelism" (open-llm-engineering): "The
// dispatch-compute-combine lifecycle" steps 2-3 (copy every token k times, sort the copies
// by expert) and "Token permutation and metadata" (expert-contiguous rows plus the map that
// reverses them). The order inside an expert is the flat slot order f = t*K + k, which
// makes the permutation a stable counting sort and the output independent of scheduling.
//
// Two launches, no host synchronisation, no atomics on data. The metadata kernel is one
// cooperative launch (all CTAs co-resident, grid-wide syncs between its phases):
//   A  per chunk of 512 slots (64 up to 65536 slots; one warp, the chunk's ids prefetched
//      into registers): per-expert counts with __match_any_sync
//   B  per expert (one warp): exclusive scan over chunks -> chunk bases, counts
//   C  exclusive scan of counts -> cu_seqlens (+ max count, maxvio); every warp replays its
//      chunk with per-expert cursors -> row_id_map, perm_src
// then permute_rows (one warp per token and 1024-element row slice: read once in 16-byte
// vectors, written to the token's K rows) runs as a programmatic dependent launch. The metadata phases also exist as
// three ordinary launches ("staged", MOE_PERMUTE_KERNEL=staged); both give identical results.
#include <cooperative_groups.h>

#include <algorithm>
#include <cstdlib>
#include <cstring>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void flag_status(int32_t* d_status, int32_t bit) {
  if (d_status != nullptr) atomicOr(d_status, bit);
}

// chunk_counts[e * nchunk + c] = #{f in chunk c : ids[f] == e}. Warp w of block b owns
// chunk b*8 + w. Ids outside [0, E) are not counted and set MOE_ERR_BAD_ROUTING.
__global__ void __launch_bounds__(256) route_hist_kernel(const int32_t* __restrict__ ids,
                                                         int64_t F, int32_t E, int64_t nchunk,
                                                         int32_t chunk,
                                                         int32_t* __restrict__ chunk_counts,
                                                         int32_t* d_status) {
  extern __shared__ int32_t s_hist[];  // [8][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < kWarpsPerTile * E; i += blockDim.x) s_hist[i] = 0;
  __syncthreads();
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile + warp;
  int32_t* hist = s_hist + warp * E;
  if (c < nchunk) {
    bool bad = false;
    for (int step = 0; step < chunk / 32; ++step) {
      const int64_t f0 = c * chunk + step * 32;
      if (f0 >= F) break;  // warp-uniform
      const int64_t f = f0 + lane;
      const int32_t e = (f < F) ? ids[f] : -1;
      const bool ok = (f < F) && e >= 0 && e < E;
      bad |= (f < F) && !ok;
      const unsigned peers = __match_any_sync(kFull, ok ? e : -1);
      if (ok && lane == __ffs(peers) - 1) hist[e] += __popc(peers);
      __syncwarp();
    }
    if (__any_sync(kFull, bad) && lane == 0) flag_status(d_status, MOE_ERR_BAD_ROUTING);
  }
  __syncthreads();
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile;
  for (int j = threadIdx.x; j < kWarpsPerTile * E; j += blockDim.x) {
    const int e = j / kWarpsPerTile, w = j % kWarpsPerTile;
    if (c0 + w < nchunk) chunk_counts[static_cast<int64_t>(e) * nchunk + c0 + w] = s_hist[w * E + e];
  }
}

// In place exclusive scan of one expert's chunk counts by one warp; returns the total. The
// values of eight 32-chunk steps are loaded before they are scanned (loads in flight).
__device__ __forceinline__ int32_t scan_chunk_row(int32_t* row, int64_t nchunk, int lane) {
  constexpr int kB = 8;
  int32_t carry = 0;
  for (int64_t base = 0; base < nchunk; base += 32 * kB) {
    int32_t v[kB];
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      const int64_t i = base + u * 32 + lane;
      v[u] = (i < nchunk) ? row[i] : 0;
    }
#pragma unroll
    for (int u = 0; u < kB; ++u) {
      if (base + u * 32 >= nchunk) break;  // warp-uniform
      const int64_t i = base + u * 32 + lane;
      int32_t incl = v[u];
#pragma unroll
      for (int d = 1; d < 32; d <<= 1) {
        const int32_t n = __shfl_up_sync(kFull, incl, d);
        if (lane >= d) incl += n;
      }
      if (i < nchunk) row[i] = carry + incl - v[u];
      carry += __shfl_sync(kFull, incl, 31);
    }
  }
  return carry;
}

// In place: chunk_counts[e][c] -> sum_{c' < c} chunk_counts[e][c']; counts[e] = total.
__global__ void __launch_bounds__(256) route_scan_kernel(int32_t* __restrict__ chunk_counts,
                                                         int64_t nchunk, int32_t E,
                                                         int32_t* __restrict__ counts) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e >= E) return;
  int32_t* row = chunk_counts + static_cast<int64_t>(e) * nchunk;
  const int32_t carry = scan_chunk_row(row, nchunk, lane);
  if (lane == 0) counts[e] = carry;
}

// maxvio = ((double)mc * E) / ((double)S * K) - 1, every operation rounded once (no FMA).
__device__ __forceinline__ double maxvio_expr(int32_t mc, int32_t E, int64_t S, int32_t K) {
  const double num = __dmul_rn(static_cast<double>(mc), static_cast<double>(E));
  const double den = __dmul_rn(static_cast<double>(S), static_cast<double>(K));
  return __dsub_rn(__ddiv_rn(num, den), 1.0);
}

// Exclusive scan of counts (E <= 1024, 4 per thread) into s_cu[0..E]; returns the max count
// in *s_max. Whole block (256 threads).
__device__ void block_scan_counts(const int32_t* __restrict__ counts, int32_t E, int32_t* s_cu,
                                  int32_t* s_tmp /*[16]*/, int32_t* s_max) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t v[4];
  int32_t local = 0, lmax = 0;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = tid * 4 + j;
    v[j] = (e < E) ? counts[e] : 0;
    local += v[j];
    lmax = max(lmax, v[j]);
  }
  int32_t incl = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t n = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += n;
  }
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) lmax = max(lmax, __shfl_xor_sync(kFull, lmax, d));
  if (lane == 31) s_tmp[warp] = incl;
  if (lane == 0) s_tmp[8 + warp] = lmax;
  __syncthreads();
  int32_t woff = 0;
  for (int w = 0; w < warp; ++w) woff += s_tmp[w];
  int32_t run = woff + incl - local;
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int e = tid * 4 + j;
    if (e < E) s_cu[e] = run;
    run += v[j];
  }
  if (tid == blockDim.x - 1) s_cu[E] = woff + incl;
  if (tid == 0) {
    int32_t m = 0;
    for (int w = 0; w < 8; ++w) m = max(m, s_tmp[8 + w]);
    *s_max = m;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(256) route_rank_kernel(
    const int32_t* __restrict__ ids, int64_t F, int64_t S, int32_t K, int32_t E, int64_t nchunk,
    int32_t chunk, const int32_t* __restrict__ chunk_base, const int32_t* __restrict__ counts,
    int32_t* __restrict__ cu_seqlens, int32_t* __restrict__ row_id_map,
    int32_t* __restrict__ perm_src, double* maxvio, int32_t* max_count) {
  extern __shared__ int32_t smem[];
  int32_t* s_cu = smem;                 // [E+1]
  int32_t* s_cursor = smem + (E + 1);   // [8][E]
  __shared__ int32_t s_tmp[16];
  __shared__ int32_t s_max;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  block_scan_counts(counts, E, s_cu, s_tmp, &s_max);
  if (blockIdx.x == 0) {
    for (int e = tid; e <= E; e += blockDim.x) cu_seqlens[e] = s_cu[e];
    if (tid == 0) {
      if (max_count != nullptr) *max_count = s_max;
      if (maxvio != nullptr) *maxvio = maxvio_expr(s_max, E, S, K);
    }
  }
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile;
  for (int j = tid; j < kWarpsPerTile * E; j += blockDim.x) {
    const int e = j / kWarpsPerTile, w = j % kWarpsPerTile;
    if (c0 + w < nchunk)
      s_cursor[w * E + e] = s_cu[e] + chunk_base[static_cast<int64_t>(e) * nchunk + c0 + w];
  }
  __syncthreads();

  const int64_t c = c0 + warp;
  if (c >= nchunk) return;
  int32_t* cur = s_cursor + warp * E;
  for (int step = 0; step < chunk / 32; ++step) {
    const int64_t f0 = c * chunk + step * 32;
    if (f0 >= F) break;  // warp-uniform
    const int64_t f = f0 + lane;
    const int32_t e = (f < F) ? ids[f] : -1;
    const bool ok = (f < F) && e >= 0 && e < E;
    const unsigned peers = __match_any_sync(kFull, ok ? e : -1);
    int32_t row = -1;
    if (ok) row = cur[e] + __popc(peers & ((1u << lane) - 1u));
    __syncwarp();
    if (ok && lane == __ffs(peers) - 1) cur[e] += __popc(peers);
    __syncwarp();
    if (f < F) {
      row_id_map[f] = row;
      if (perm_src != nullptr && ok) perm_src[row] = static_cast<int32_t>(f);
    }
  }
}

// One warp per (token, row slice of 32*U 16-byte vectors): the slice is read once and written
// to the token's K destination rows. Slicing the rows keeps every SM busy when there are few
// tokens (S = 1024 tokens of 7168 features are 7168 work items, not 1024).
template <int U>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ x, int64_t S,
                                                           int64_t nvec, int32_t K,
                                                           const int32_t* __restrict__ row_id_map,
                                                           uint4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  griddep_wait();  // row_id_map comes from the metadata kernel
  griddep_launch_dependents();
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t npass = (nvec + 32 * U - 1) / (32 * U);
  const int64_t items = S * npass;
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       it < items; it += nwarps) {
    const int64_t t = it / npass;
    const int64_t v0 = (it - t * npass) * (32 * U);
    const int32_t my_row = (lane < K) ? row_id_map[t * K + lane] : -1;
    const uint4* src = x + t * nvec;
    uint4 r[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t v = v0 + j * 32 + lane;
      if (v < nvec) r[j] = __ldg(src + v);
    }
    for (int k = 0; k < K; ++k) {
      const int32_t row = (K <= 32) ? __shfl_sync(kFull, my_row, k) : row_id_map[t * K + k];
      if (row < 0) continue;
      uint4* dst = x_perm + static_cast<int64_t>(row) * nvec;
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const int64_t v = v0 + j * 32 + lane;
        if (v < nvec) dst[v] = r[j];
      }
    }
  }
}

__global__ void maxvio_kernel(const int32_t* __restrict__ counts, int32_t E, int64_t S, int32_t K,
                              double* maxvio, int32_t* max_count) {
  __shared__ int32_t s_w[32];
  int32_t m = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) m = max(m, counts[e]);
#pragma unroll
  for (int d = 16; d > 0; d >>= 1) m = max(m, __shfl_xor_sync(kFull, m, d));
  if ((threadIdx.x & 31) == 0) s_w[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    int32_t mc = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) mc = max(mc, s_w[w]);
    if (max_count != nullptr) *max_count = mc;
    *maxvio = maxvio_expr(mc, E, S, K);
  }
}

// ----------------------------------------------------------------------------- fused kernel

struct PermuteArgs {
  const int32_t* ids;
  int64_t S, F, nchunk;
  int32_t K, E;
  int32_t chunk;  // slots per chunk (permute_chunk_slots)
  int32_t* chunk_counts;
  int32_t* counts;
  int32_t* cu_seqlens;
  int32_t* row_id_map;
  int32_t* perm_src;
  double* maxvio;
  int32_t* max_count;
  int32_t* d_status;
};

__device__ __forceinline__ void load_chunk_ids(const PermuteArgs& a, int64_t c, int lane,
                                               int32_t (&idr)[kChunkMax / 32]) {
#pragma unroll
  for (int j = 0; j < kChunkMax / 32; ++j) {
    const int64_t f = c * a.chunk + j * 32 + lane;
    idr[j] = (j < a.chunk / 32 && f < a.F) ? __ldg(a.ids + f) : -1;
  }
}

__global__ void __launch_bounds__(256) permute_fused_kernel(const PermuteArgs a) {
  namespace cg = cooperative_groups;
  cg::grid_group grid = cg::this_grid();
  extern __shared__ __align__(128) uint8_t fsmem[];
  int32_t* s_tab = reinterpret_cast<int32_t*>(fsmem);  // [8][E]
  int32_t* s_cu = s_tab + kWarpsPerTile * a.E;         // [E+1]
  __shared__ int32_t s_tmp[16];
  __shared__ int32_t s_max;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = a.E;
  const int64_t wstride = static_cast<int64_t>(gridDim.x) * kWarpsPerTile;

  griddep_wait();  // the routing table may come from the previous kernel in the stream

  // A: chunk histograms -> chunk_counts[e][c]
  for (int64_t cb = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile; cb < a.nchunk; cb += wstride) {
    int32_t* hist = s_tab + warp * E;
    for (int i = lane; i < E; i += 32) hist[i] = 0;
    __syncwarp();
    const int64_t c = cb + warp;
    if (c < a.nchunk) {
      int32_t idr[kChunkMax / 32];
      load_chunk_ids(a, c, lane, idr);
      bool bad = false;
#pragma unroll
      for (int j = 0; j < kChunkMax / 32; ++j) {
        if (j >= a.chunk / 32) break;  // uniform
        const int64_t f = c * a.chunk + j * 32 + lane;
        const int32_t e = idr[j];
        const bool ok = f < a.F && e >= 0 && e < E;
        bad |= (f < a.F) && !ok;
        const unsigned peers = __match_any_sync(kFull, ok ? e : -1);
        if (ok && lane == __ffs(peers) - 1) hist[e] += __popc(peers);
        __syncwarp();
      }
      if (__any_sync(kFull, bad) && lane == 0) flag_status(a.d_status, MOE_ERR_BAD_ROUTING);
    }
    __syncthreads();
    for (int j = threadIdx.x; j < kWarpsPerTile * E; j += blockDim.x) {
      const int e = j / kWarpsPerTile, w = j % kWarpsPerTile;
      if (cb + w < a.nchunk)
        a.chunk_counts[static_cast<int64_t>(e) * a.nchunk + cb + w] = s_tab[w * E + e];
    }
    __syncthreads();
  }
  grid.sync();

  // B: per-expert exclusive scan over chunks
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile + warp; e < E; e += wstride) {
    const int32_t carry = scan_chunk_row(a.chunk_counts + e * a.nchunk, a.nchunk, lane);
    if (lane == 0) a.counts[e] = carry;
  }
  grid.sync();

  // C: cu_seqlens, maxvio; stable ranks
  block_scan_counts(a.counts, E, s_cu, s_tmp, &s_max);
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) a.cu_seqlens[e] = s_cu[e];
    if (threadIdx.x == 0) {
      if (a.max_count != nullptr) *a.max_count = s_max;
      if (a.maxvio != nullptr) *a.maxvio = maxvio_expr(s_max, E, a.S, a.K);
    }
  }
  for (int64_t cb = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile; cb < a.nchunk; cb += wstride) {
    for (int j = threadIdx.x; j < kWarpsPerTile * E; j += blockDim.x) {
      const int e = j / kWarpsPerTile, w = j % kWarpsPerTile;
      if (cb + w < a.nchunk)
        s_tab[w * E + e] = s_cu[e] + a.chunk_counts[static_cast<int64_t>(e) * a.nchunk + cb + w];
    }
    __syncthreads();
    const int64_t c = cb + warp;
    if (c < a.nchunk) {
      int32_t* cur = s_tab + warp * E;
      int32_t idr[kChunkMax / 32];
      load_chunk_ids(a, c, lane, idr);
#pragma unroll
      for (int j = 0; j < kChunkMax / 32; ++j) {
        if (j >= a.chunk / 32) break;  // uniform
        const int64_t f = c * a.chunk + j * 32 + lane;
        const int32_t e = idr[j];
        const bool ok = f < a.F && e >= 0 && e < E;
        const unsigned peers = __match_any_sync(kFull, ok ? e : -1);
        int32_t row = -1;
        if (ok) row = cur[e] + __popc(peers & ((1u << lane) - 1u));
        __syncwarp();
        if (ok && lane == __ffs(peers) - 1) cur[e] += __popc(peers);
        __syncwarp();
        if (f < a.F) {
          a.row_id_map[f] = row;
          if (a.perm_src != nullptr && ok) a.perm_src[row] = static_cast<int32_t>(f);
        }
      }
    }
    __syncthreads();
  }
  // rows are copied by permute_rows_kernel, launched right after as a dependent grid
  griddep_launch_dependents();
}

size_t fused_smem_bytes(int32_t E) {
  return sizeof(int32_t) * (static_cast<size_t>(kWarpsPerTile) * E + E + 1);
}

// Co-resident CTAs per SM of the fused kernel at the largest shared-memory size (cached).
int fused_blocks_per_sm() {
  static std::once_flag once;
  static int blocks = 0;
  std::call_once(once, [] {
    const size_t smem = fused_smem_bytes(MOE_MAX_EXPERTS);
    if (cudaFuncSetAttribute(permute_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, permute_fused_kernel, 256, smem) ==
        cudaSuccess)
      blocks = n;
  });
  return blocks;
}

bool use_staged_permute() {
  static const bool staged = [] {
    const char* s = std::getenv("MOE_PERMUTE_KERNEL");
    return s != nullptr && std::strcmp(s, "staged") == 0;
  }();
  return staged;
}

// Row copy as a programmatic dependent launch of the metadata kernel before it.
cudaError_t launch_rows(const void* x, int64_t S, int64_t H, int32_t K, const int32_t* row_id_map,
                        void* x_perm, cudaStream_t stream) {
  const int64_t nvec = H / 8;
  const int64_t items = S * ceil_div(nvec, 32 * 4);
  const int64_t blocks = std::min<int64_t>(ceil_div(items, 8), static_cast<int64_t>(num_sms()) * 8);
  return launch_dependent(permute_rows_kernel<4>, dim3(static_cast<unsigned>(blocks)), dim3(256),
                          0, stream, static_cast<const uint4*>(x), S, nvec, K, row_id_map,
                          static_cast<uint4*>(x_perm));
}

}  // namespace

moe_status launch_permute(const void* x, const int32_t* topk_ids, int64_t S, int64_t H, int32_t K,
                          int32_t E, void* x_perm, int32_t* counts, int32_t* cu_seqlens,
                          int32_t* row_id_map, int32_t* perm_src, double* maxvio,
                          int32_t* max_count, int32_t* chunk_counts, int32_t* d_status,
                          cudaStream_t stream) {
  const int64_t F = S * K;
  const int64_t nchunk = permute_num_chunks(F);
  const int32_t chunk = permute_chunk_slots(F);
  const int64_t tiles = ceil_div(nchunk, kWarpsPerTile);
  const int per_sm = use_staged_permute() ? 0 : fused_blocks_per_sm();
  if (per_sm > 0) {
    const int64_t want = std::max<int64_t>({tiles, ceil_div(E, kWarpsPerTile), 1});
    const int grid = static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(per_sm) * num_sms()));
    PermuteArgs pa{topk_ids, S, F, nchunk, K, E, chunk, chunk_counts, counts, cu_seqlens,
                   row_id_map, perm_src, maxvio, max_count, d_status};
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(256);
    cfg.dynamicSmemBytes = fused_smem_bytes(E);
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    if (cudaLaunchKernelEx(&cfg, permute_fused_kernel, pa) != cudaSuccess) {
      (void)cudaGetLastError();  // refused as a dependent launch: cooperative only
      cfg.numAttrs = 1;
      if (cudaLaunchKernelEx(&cfg, permute_fused_kernel, pa) != cudaSuccess) return MOE_ERR_CUDA;
    }
    if (x_perm != nullptr && launch_rows(x, S, H, K, row_id_map, x_perm, stream) != cudaSuccess)
      return MOE_ERR_CUDA;
    return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  // staged: three ordinary launches (E <= 1024: at most 32 KB and 37 KB of shared memory)
  const size_t hist_smem = sizeof(int32_t) * kWarpsPerTile * E;
  const size_t rank_smem = sizeof(int32_t) * (E + 1 + kWarpsPerTile * E);
  route_hist_kernel<<<static_cast<unsigned>(tiles), 256, hist_smem, stream>>>(
      topk_ids, F, E, nchunk, chunk, chunk_counts, d_status);
  route_scan_kernel<<<static_cast<unsigned>(ceil_div(E, 8)), 256, 0, stream>>>(chunk_counts,
                                                                             nchunk, E, counts);
  route_rank_kernel<<<static_cast<unsigned>(tiles), 256, rank_smem, stream>>>(
      topk_ids, F, S, K, E, nchunk, chunk, chunk_counts, counts, cu_seqlens, row_id_map, perm_src,
      maxvio, max_count);
  if (x_perm != nullptr && launch_rows(x, S, H, K, row_id_map, x_perm, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, double* maxvio,
                         int32_t* max_count, cudaStream_t stream) {
  maxvio_kernel<<<1, 256, 0, stream>>>(counts, E, S, K, maxvio, max_count);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ----------------------------------------------------------------------------- shared experts

namespace {

// Routing with n_shared always-on experts appended: slot K + j of every token is expert
// E + j with weight 1 (MoE(x) = SharedExpert(x) + sum_k w_k RoutedExpert_k(x), "Mixture of
// Kittens" digest, Step 1), so the shared expert's rows join the same grouped launches.
// One thread per output slot.
__global__ void append_shared_kernel(const int32_t* __restrict__ ids, const float* __restrict__ w,
                                     int64_t S, int32_t K, int32_t E, int32_t n_shared,
                                     int32_t* __restrict__ ids_out, float* __restrict__ w_out) {
  griddep_wait();
  griddep_launch_dependents();
  const int32_t K2 = K + n_shared;
  const int64_t total = S * K2;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = i / K2;
    const int32_t k = static_cast<int32_t>(i - t * K2);
    ids_out[i] = k < K ? ids[t * K + k] : E + (k - K);
    w_out[i] = k < K ? w[t * K + k] : 1.0f;
  }
}

}  // namespace

moe_status launch_append_shared(const int32_t* ids, const float* w, int64_t S, int32_t K,
                                int32_t E, int32_t n_shared, int32_t* ids_out, float* w_out,
                                cudaStream_t stream) {
  const int64_t total = S * (K + n_shared);
  const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), static_cast<int64_t>(num_sms()) * 8);
  const cudaError_t err =
      launch_dependent(append_shared_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0,
                       stream, ids, w, S, K, E, n_shared, ids_out, w_out);
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// ----------------------------------------------------------------------------- no-alloc entry

// Scratch of moe_permute_no_alloc, in the library's own device memory: every GPU that loads
// the library holds MOE_NO_ALLOC_SCRATCH_BYTES of it until the process exits. All calls on a
// device share it.
static __device__ __align__(256) int32_t g_permute_scratch[MOE_NO_ALLOC_SCRATCH_BYTES / 4];

namespace {

ContextCache g_scratch_addr;

// Device address of g_permute_scratch in the current CUDA context. The host-side name is
// only a stand-in, so the address is looked up (with the device current) the first time a
// context calls, and kept per context: another context on the same device, or the primary
// context re-created after cudaDeviceReset, gets its own lookup.
moe_status scratch_address(void** out) {
  void* p = nullptr;
  if (g_scratch_addr.find(current_context_id(), &p)) {
    *out = p;
    return MOE_OK;
  }
  if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr)
    return MOE_ERR_CUDA;
  g_scratch_addr.put(current_context_id(), p);  // the lookup made the context current
  *out = p;
  return MOE_OK;
}

}  // namespace
}  // namespace moe

extern "C" moe_status moe_permute_no_alloc(const void* x, const int32_t* topk_ids, int64_t S,
                                           int64_t H, int32_t K, int32_t E, void* x_perm,
                                           int32_t* counts, int32_t* cu_seqlens,
                                           int32_t* row_id_map, int32_t* perm_src, double* maxvio,
                                           int32_t* max_count, int32_t* d_status,
                                           void* cuda_stream) {
  if (S < 0 || K < 1 || E < 1) return MOE_ERR_INVALID_ARGUMENT;
  if (moe_permute_workspace_bytes(S, K, E) > MOE_NO_ALLOC_SCRATCH_BYTES)
    return MOE_ERR_UNSUPPORTED_SHAPE;
  void* scratch = nullptr;
  const moe_status st = moe::scratch_address(&scratch);
  if (st != MOE_OK) return st;
  // The kernels write every scratch entry they later read, so nothing is cleared first.
  return moe_permute(x, topk_ids, S, H, K, E, x_perm, counts, cu_seqlens, row_id_map, perm_src,
                     maxvio, max_count, scratch, MOE_NO_ALLOC_SCRATCH_BYTES, d_status,
                     cuda_stream);
}
