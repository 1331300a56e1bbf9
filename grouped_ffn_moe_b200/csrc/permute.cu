// Route permutation into expert-contiguous order, and the row copy that goes with it.
//
// Follows "Distributed expert parallelism" (open-llm-engineering): "The
// dispatch-compute-combine lifecycle" steps 2-3 (copy every token k times, sort the copies
// by expert) and "Token permutation and metadata" (expert-contiguous rows plus the map that
// reverses them). The order inside an expert is the flat slot order f = t*K + k, which
// makes the permutation a stable counting sort and the output independent of scheduling.
//
// Two launches, no host synchronisation, no atomics on data:
//
//   metadata  counts, cu_seqlens, maxvio and the stable ranks (row_id_map, perm_src). Up to
//             2^17 flat slots (and for any E above 1024) by one thread-block cluster: every
//             warp owns a contiguous run of slots, counts them per expert in its own shared
//             histogram (__match_any_sync finds the lanes holding the same expert), the CTA
//             scans its warps' counts, the CTAs exchange their totals through distributed
//             shared memory, and every warp replays its slots with per-expert cursors. No
//             grid-wide synchronisation, no workspace. Experts are handled 1024 at a time
//             (one per thread); E > 1024 takes several such windows. Larger tables use a
//             cooperative grid over all SMs (histogram, per-expert scan over chunks, replay,
//             with grid-wide syncs between) that keeps the per-chunk counts in the caller's
//             workspace.
//   rows      permute_rows: one warp per token and 1024-element row slice reads the slice
//             once in 16-byte vectors and writes it to the token's K rows. It is launched as a
//             programmatic dependent of the metadata kernel and loads its first slice of x
//             before waiting for the ranks, so the x read overlaps the metadata work.
#include <cooperative_groups.h>

#include <algorithm>

#include "internal.h"
#include "ptx.cuh"

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void flag_status(int32_t* d_status, int32_t bit) {
  if (d_status != nullptr) atomicOr(d_status, bit);
}

// maxvio = ((double)mc * E) / ((double)S * K) - 1, every operation rounded once (no FMA).
__device__ __forceinline__ double maxvio_expr(int32_t mc, int32_t E, int64_t S, int32_t K) {
  const double num = __dmul_rn(static_cast<double>(mc), static_cast<double>(E));
  const double den = __dmul_rn(static_cast<double>(S), static_cast<double>(K));
  return __dsub_rn(__ddiv_rn(num, den), 1.0);
}

// ----------------------------------------------------------------------------- cluster kernel

constexpr int kClWarps = 32;               // warps per CTA
constexpr int kClThreads = 32 * kClWarps;  // 1024: one expert of a window per thread
constexpr int kClWindow = kClThreads;      // experts per window
constexpr int kClRegSteps = 8;             // 32-slot steps per warp whose ids stay in registers
constexpr size_t kClSmemBytes = sizeof(int32_t) * (kClWarps + 1) * kClWindow;
#ifndef MOE_CLUSTER_CTAS
#define MOE_CLUSTER_CTAS 16
#endif
constexpr int kClMaxCtas = MOE_CLUSTER_CTAS;  // largest cluster tried (16: non-portable size)
static_assert(kClMaxCtas >= 1 && kClMaxCtas <= 16, "cluster size");

struct ClusterArgs {
  const int32_t* ids;
  int64_t S, F;
  int32_t K, E;
  int64_t per_warp;  // flat slots per warp, a multiple of 32
  int32_t* counts;
  int32_t* cu_seqlens;
  int32_t* row_id_map;
  int32_t* perm_src;
  double* maxvio;
  int32_t* max_count;
  int32_t* d_status;
};

// Exclusive prefix, sum and maximum of v over the 1024 threads of the CTA (the sum and the
// maximum are the same in every thread). s_w holds 66 ints.
__device__ __forceinline__ int32_t cta_scan(int32_t v, int32_t* s_w, int32_t* sum, int32_t* mx) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int32_t incl = v, m = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int32_t n = __shfl_up_sync(kFull, incl, d);
    if (lane >= d) incl += n;
    m = max(m, __shfl_xor_sync(kFull, m, d));
  }
  if (lane == 31) s_w[warp] = incl;
  if (lane == 0) s_w[32 + warp] = m;
  __syncthreads();
  if (warp == 0) {
    const int32_t wv = s_w[lane];
    int32_t wi = wv, wm = s_w[32 + lane];
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t n = __shfl_up_sync(kFull, wi, d);
      if (lane >= d) wi += n;
      wm = max(wm, __shfl_xor_sync(kFull, wm, d));
    }
    s_w[lane] = wi - wv;  // exclusive prefix of the warp sums
    if (lane == 31) s_w[64] = wi;
    if (lane == 0) s_w[65] = wm;
  }
  __syncthreads();
  const int32_t excl = s_w[warp] + incl - v;
  *sum = s_w[64];
  *mx = s_w[65];
  __syncthreads();  // s_w is reused by the next call
  return excl;
}

// One thread-block cluster. Warp g = rank * 32 + w owns flat slots [g * per_warp, ...).
// Per window of experts [e0, e0 + 1024):
//   A  every warp counts its slots per expert of the window (its own shared row, no atomics)
//   B  thread j scans expert e0+j over the CTA's 32 warps: the warps' offsets inside the CTA,
//      and the CTA's total, published in shared memory
//   C  (cluster barrier) thread j reads expert e0+j's totals of all CTAs (distributed shared
//      memory): the count, and the offset of this CTA (the CTAs before it); a CTA-wide scan
//      of the counts gives cu_seqlens; every warp's cursor = cu + CTA offset + warp offset
//   D  every warp replays its slots: row = cursor + number of earlier lanes with the same
//      expert; the group's first lane advances the cursor
// Slots of experts outside the window are skipped (taken in their own window); ids outside
// [0, E) get row -1 and set MOE_ERR_BAD_ROUTING.
__global__ void __launch_bounds__(kClThreads, 1) route_cluster_kernel(const ClusterArgs a) {
  extern __shared__ __align__(16) int32_t csm[];
  int32_t* hist = csm;                        // [kClWarps][kClWindow]
  int32_t* tot = csm + kClWarps * kClWindow;  // [kClWindow]
  __shared__ int32_t s_w[66];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t ncta = cluster_nctarank();
  int32_t* my = hist + warp * kClWindow;

  griddep_wait();  // ids (and x, read by the row copy) may come from the previous kernel
  griddep_launch_dependents();

  const int64_t g = static_cast<int64_t>(rank) * kClWarps + warp;
  const int64_t f_begin = min(g * a.per_warp, a.F);
  const int64_t f_end = min(f_begin + a.per_warp, a.F);
  const int nsteps = static_cast<int>((f_end - f_begin + 31) / 32);  // warp-uniform
  // ids of the warp's first kClRegSteps steps stay in registers; later steps are read in
  // batches of kClRegSteps (all loads of a batch in flight before its first use)
  int32_t idr[kClRegSteps];
  auto load_batch = [&](int j0, int32_t (&v)[kClRegSteps]) {
#pragma unroll
    for (int i = 0; i < kClRegSteps; ++i) {
      const int64_t f = f_begin + (j0 + i) * 32 + lane;
      v[i] = (j0 + i < nsteps && f < f_end) ? __ldg(a.ids + f) : -1;
    }
  };
  load_batch(0, idr);
  // body(j, f, e) for every step j of the warp's run, in order
  auto for_each_step = [&](auto&& body) {
    for (int j0 = 0; j0 < nsteps; j0 += kClRegSteps) {
      int32_t v[kClRegSteps];
      if (j0 == 0) {
#pragma unroll
        for (int i = 0; i < kClRegSteps; ++i) v[i] = idr[i];
      } else {
        load_batch(j0, v);
      }
#pragma unroll
      for (int i = 0; i < kClRegSteps; ++i)
        if (j0 + i < nsteps) body(f_begin + (j0 + i) * 32 + lane, v[i]);  // warp-uniform
    }
  };

  bool bad = false;
  int32_t carry = 0, run_max = 0;
  for (int32_t e0 = 0; e0 < a.E; e0 += kClWindow) {
    const int32_t ew = min(kClWindow, a.E - e0);
    for (int i = lane; i < ew; i += 32) my[i] = 0;
    __syncwarp();
    // A
    for_each_step([&](int64_t f, int32_t e) {
      if (e0 == 0) bad |= (f < f_end) && (e < 0 || e >= a.E);
      const bool in = (f < f_end) && e >= e0 && e < e0 + ew;
      const int32_t key = in ? e - e0 : -1;
      const unsigned peers = __match_any_sync(kFull, key);
      if (in && lane == __ffs(peers) - 1) my[key] += __popc(peers);
      __syncwarp();
    });
    __syncthreads();
    // B
    int32_t cta_total = 0;
    if (tid < ew) {
      for (int w = 0; w < kClWarps; ++w) {
        const int32_t c = hist[w * kClWindow + tid];
        hist[w * kClWindow + tid] = cta_total;
        cta_total += c;
      }
      tot[tid] = cta_total;
    }
    cluster_sync();  // every CTA's totals are visible cluster-wide
    // C
    int32_t base = 0, total = 0;
    if (tid < ew) {
      const uint32_t addr = smem_u32(tot + tid);
      int32_t v[16];  // all of the (at most 16) reads in flight before the sums
#pragma unroll
      for (uint32_t r = 0; r < 16; ++r) v[r] = r < ncta ? ld_shared_cluster(map_to_cta(addr, r)) : 0;
#pragma unroll
      for (uint32_t r = 0; r < 16; ++r) {
        base += r < rank ? v[r] : 0;
        total += v[r];
      }
    }
    cluster_arrive();  // this CTA is done reading the others' totals
    int32_t wsum = 0, wmax = 0;
    const int32_t excl = carry + cta_scan(total, s_w, &wsum, &wmax);
    if (tid < ew) {
      if (rank == 0) {
        a.counts[e0 + tid] = total;
        a.cu_seqlens[e0 + tid] = excl;
      }
      const int32_t cur0 = excl + base;
      for (int w = 0; w < kClWarps; ++w) hist[w * kClWindow + tid] += cur0;
    }
    carry += wsum;
    run_max = max(run_max, wmax);
    __syncthreads();
    // D
    for_each_step([&](int64_t f, int32_t e) {
      const bool in = (f < f_end) && e >= e0 && e < e0 + ew;
      const int32_t key = in ? e - e0 : -1;
      const unsigned peers = __match_any_sync(kFull, key);
      const int32_t row = in ? my[key] + __popc(peers & ((1u << lane) - 1u)) : -1;
      __syncwarp();
      if (in && lane == __ffs(peers) - 1) my[key] += __popc(peers);
      __syncwarp();
      if (in) {
        a.row_id_map[f] = row;
        if (a.perm_src != nullptr) a.perm_src[row] = static_cast<int32_t>(f);
      } else if (e0 == 0 && f < f_end && (e < 0 || e >= a.E)) {
        a.row_id_map[f] = -1;  // dropped slot
      }
    });
    cluster_wait();  // no CTA still reads this CTA's totals: they may be rewritten
    __syncthreads();
  }
  if (__any_sync(kFull, bad) && lane == 0) flag_status(a.d_status, MOE_ERR_BAD_ROUTING);
  if (rank == 0 && tid == 0) {
    a.cu_seqlens[a.E] = carry;
    if (a.max_count != nullptr) *a.max_count = run_max;
    if (a.maxvio != nullptr) *a.maxvio = maxvio_expr(run_max, a.E, a.S, a.K);
  }
}

// ----------------------------------------------------------------------------- cooperative kernel
// (routing tables above kClusterMaxSlots slots with E <= 1024)

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

struct PermuteArgs {
  const int32_t* ids;
  int64_t S, F, nchunk;
  int32_t K, E;
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
                                               int32_t (&idr)[kChunkSlots / 32]) {
#pragma unroll
  for (int j = 0; j < kChunkSlots / 32; ++j) {
    const int64_t f = c * kChunkSlots + j * 32 + lane;
    idr[j] = f < a.F ? __ldg(a.ids + f) : -1;
  }
}

// A: per-chunk histograms -> chunk_counts[e][c]; B: per-expert exclusive scan over chunks;
// C: cu_seqlens, maxvio, and every warp's replay of its chunk. Grid-wide syncs in between.
__global__ void __launch_bounds__(256) permute_coop_kernel(const PermuteArgs a) {
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

  griddep_wait();  // the routing table (and x) may come from the previous kernel
  griddep_launch_dependents();

  // A
  for (int64_t cb = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile; cb < a.nchunk; cb += wstride) {
    int32_t* hist = s_tab + warp * E;
    for (int i = lane; i < E; i += 32) hist[i] = 0;
    __syncwarp();
    const int64_t c = cb + warp;
    if (c < a.nchunk) {
      int32_t idr[kChunkSlots / 32];
      load_chunk_ids(a, c, lane, idr);
      bool bad = false;
#pragma unroll
      for (int j = 0; j < kChunkSlots / 32; ++j) {
        const int64_t f = c * kChunkSlots + j * 32 + lane;
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

  // B
  for (int64_t e = static_cast<int64_t>(blockIdx.x) * kWarpsPerTile + warp; e < E; e += wstride) {
    const int32_t carry = scan_chunk_row(a.chunk_counts + e * a.nchunk, a.nchunk, lane);
    if (lane == 0) a.counts[e] = carry;
  }
  grid.sync();

  // C
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
      int32_t idr[kChunkSlots / 32];
      load_chunk_ids(a, c, lane, idr);
#pragma unroll
      for (int j = 0; j < kChunkSlots / 32; ++j) {
        const int64_t f = c * kChunkSlots + j * 32 + lane;
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
}

size_t coop_smem_bytes(int32_t E) {
  return sizeof(int32_t) * (static_cast<size_t>(kWarpsPerTile) * E + E + 1);
}

// ----------------------------------------------------------------------------- row copy

// One warp per (token, row slice of 32*U 16-byte vectors): the slice is read once and written
// to the token's K destination rows. Slicing the rows keeps every SM busy when there are few
// tokens (S = 1024 tokens of 7168 features are 7168 work items, not 1024). The warp's first
// slice of x is loaded before the wait for the metadata kernel (x does not depend on it).
template <int U>
__global__ void __launch_bounds__(256) permute_rows_kernel(const uint4* __restrict__ x, int64_t S,
                                                           int64_t nvec, int32_t K,
                                                           const int32_t* __restrict__ row_id_map,
                                                           uint4* __restrict__ x_perm) {
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t npass = (nvec + 32 * U - 1) / (32 * U);
  const int64_t items = S * npass;
  const int64_t first = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
  uint4 r[U];
  auto load = [&](int64_t item) {
    const int64_t t = item / npass;
    const int64_t v0 = (item - t * npass) * (32 * U);
    const uint4* src = x + t * nvec;
#pragma unroll
    for (int j = 0; j < U; ++j) {
      const int64_t v = v0 + j * 32 + lane;
      if (v < nvec) r[j] = __ldg(src + v);
    }
  };
  if (first < items) load(first);
  griddep_wait();  // row_id_map comes from the metadata kernel
  griddep_launch_dependents();
  for (int64_t it = first; it < items; it += nwarps) {
    if (it != first) load(it);
    const int64_t t = it / npass;
    const int64_t v0 = (it - t * npass) * (32 * U);
    const int32_t my_row = (lane < K) ? row_id_map[t * K + lane] : -1;
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

// ----------------------------------------------------------------------------- host side

// Cluster size of the metadata kernel in the current context: the largest of 16, 8, 4, 2, 1
// CTAs that the device can co-schedule with the kernel's shared memory (cached per context).
ContextCache g_cluster_size;

int cluster_size() {
  void* v = nullptr;
  if (g_cluster_size.find(current_context_id(), &v))
    return static_cast<int>(reinterpret_cast<intptr_t>(v));
  if (cudaFuncSetAttribute(route_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kClSmemBytes)) != cudaSuccess ||
      cudaFuncSetAttribute(route_cluster_kernel,
                           cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  int best = 0;
  for (int c = kClMaxCtas; c >= 1 && best == 0; c >>= 1) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(c);
    cfg.blockDim = dim3(kClThreads);
    cfg.dynamicSmemBytes = kClSmemBytes;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = c;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, route_cluster_kernel, &cfg) == cudaSuccess && n > 0)
      best = c;
    else
      (void)cudaGetLastError();
  }
  g_cluster_size.put(current_context_id(), reinterpret_cast<void*>(static_cast<intptr_t>(best)));
  return best;
}

cudaError_t launch_cluster_metadata(const ClusterArgs& args_in, cudaStream_t stream) {
  const int c = cluster_size();
  if (c <= 0) return cudaErrorNotSupported;
  ClusterArgs args = args_in;
  const int64_t warps = static_cast<int64_t>(c) * kClWarps;
  args.per_warp = std::max<int64_t>(32, ceil_div(ceil_div(args.F, warps), 32) * 32);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(c);
  cfg.blockDim = dim3(kClThreads);
  cfg.dynamicSmemBytes = kClSmemBytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = c;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t err = cudaLaunchKernelEx(&cfg, route_cluster_kernel, args);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();
    cfg.numAttrs = 1;  // without the dependent-launch attribute
    err = cudaLaunchKernelEx(&cfg, route_cluster_kernel, args);
  }
  return err;
}

// Co-resident CTAs per SM of the cooperative kernel at E = 1024 (cached per context).
ContextCache g_coop_blocks;

int coop_blocks_per_sm() {
  void* v = nullptr;
  if (g_coop_blocks.find(current_context_id(), &v))
    return static_cast<int>(reinterpret_cast<intptr_t>(v));
  const size_t smem = coop_smem_bytes(kCoopMaxExperts);
  int n = 0;
  if (cudaFuncSetAttribute(permute_coop_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem)) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, permute_coop_kernel, 256, smem) !=
          cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  g_coop_blocks.put(current_context_id(), reinterpret_cast<void*>(static_cast<intptr_t>(n)));
  return n;
}

cudaError_t launch_coop_metadata(const PermuteArgs& pa, cudaStream_t stream) {
  const int per_sm = coop_blocks_per_sm();
  if (per_sm <= 0) return cudaErrorNotSupported;
  const int64_t tiles = ceil_div(pa.nchunk, kWarpsPerTile);
  const int64_t want = std::max<int64_t>({tiles, ceil_div(pa.E, kWarpsPerTile), 1});
  const int grid =
      static_cast<int>(std::min<int64_t>(want, static_cast<int64_t>(per_sm) * num_sms()));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = coop_smem_bytes(pa.E);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t err = cudaLaunchKernelEx(&cfg, permute_coop_kernel, pa);
  if (err != cudaSuccess) {
    (void)cudaGetLastError();  // refused as a dependent launch: cooperative only
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, permute_coop_kernel, pa);
  }
  return err;
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
  cudaError_t err;
  if (permute_uses_cluster(F, E)) {
    const ClusterArgs ca{topk_ids, S, F, K, E, 0, counts, cu_seqlens, row_id_map, perm_src,
                         maxvio, max_count, d_status};
    err = launch_cluster_metadata(ca, stream);
  } else {
    const PermuteArgs pa{topk_ids, S, F, permute_num_chunks(F), K, E, chunk_counts, counts,
                         cu_seqlens, row_id_map, perm_src, maxvio, max_count, d_status};
    err = launch_coop_metadata(pa, stream);
  }
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (x_perm != nullptr && launch_rows(x, S, H, K, row_id_map, x_perm, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, double* maxvio,
                         int32_t* max_count, cudaStream_t stream) {
  maxvio_kernel<<<1, 1024, 0, stream>>>(counts, E, S, K, maxvio, max_count);
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
