// Backward of the grouped expert SwiGLU FFN on tcgen05 tensor cores (sm_100a).
//
// The forward is Down(SwiGLU(Up x, Gate x)) per expert ("Mixture of Kittens" digest, Step 1)
// over the expert-contiguous rows that cu_seqlens selects (MoonEP README, "Integration");
// training keeps one fp32 gradient buffer per projection, laid out like the weights (MoonEP
// README, "Gradient buffers"). The chain rule of that forward, with g = x.W_gate and
// u = x.W_up saved as bf16 by the training forward and s = sigmoid(g):
//
//   down dgrad + SwiGLU backward (one kernel, grad_h never leaves TMEM):
//       grad_h = grad_y . W_down[e]^T
//       d_gate = bf16(grad_h * u * s * (1 + g (1 - s)))     d_up = bf16(grad_h * g * s)
//   up/gate dgrad (one accumulator over a reduction of length 2 H'):
//       grad_x_perm = bf16(d_gate . W_gate[e]^T + d_up . W_up[e]^T)
//   weight gradients (fp32, written or added into):
//       dW_gate[e] = x^T d_gate    dW_up[e] = x^T d_up    dW_down[e] = h^T grad_y
//
// The dgrad passes use the forward's swap-AB tiling: the tensor-core M side (128) runs over
// output features, the N side over up to 256 of an expert's tokens. Their weight tiles are
// K-major: W_down[e] is [H', H] and W_gate[e], W_up[e] are [H, H'], so for an output feature
// the reduction index is the contiguous one, and a 128-row x 64-column TMA box is the
// canonical K-major 128-byte-swizzled operand. The token tiles are K-major as in the forward.
//
// The weight-gradient pass reduces over an expert's tokens. Its unit is one 128 x 256 tile of
// one expert's gradient; both operands are MN-major (features contiguous in the activation
// rows), loaded by TMA as 64-feature x 64-token slices. The last 64-token block of an expert
// is cut at the next multiple of 16 tokens; the rows between the expert's end and that cut
// (the next expert's tokens) are zeroed in shared memory before the MMAs read them.
//
// Warp roles as in the forward (320 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA
// issuer, warps 2-9 two epilogue groups alternating 32-column chunks of the accumulator. Two
// accumulator stages of 256 TMEM columns let the epilogue of one unit overlap the next unit's
// MMAs. Every wait is bounded (globaltimer) and a time-out leaves MOE_ERR_DEVICE_TIMEOUT in
// d_status after the CTA has drained its own copies and MMAs.

#include "gemm_common.cuh"

namespace moe {
namespace {

constexpr int kBBytes = kNMax * kRowBytes;  // 32 KB: up to 256 token rows x 64 k (K-major)

// ----------------------------------------------------------------------------- dgrad passes

enum DgradMode : int { kDown = 0, kUpGate = 1 };

template <int kMode>
struct DCfg {
  static constexpr int kStageBytes = kABytes + kBBytes;  // 48 KB
  // kDown stages the pre-activations (two 8 KB tiles per epilogue group)
  static constexpr int kEpiBytes = kEpiGroups * kOutBytes * (kMode == kDown ? 2 : 1);
  static constexpr int kStages = kMode == kDown ? 3 : 4;
  static constexpr int kPipeBytes = kStages * kStageBytes;
  static constexpr int kOffEpi = kPipeBytes;
  static constexpr int kOffCu = kOffEpi + kEpiBytes;
  static constexpr int kOffUnits = kOffCu + 4 * (MOE_MAX_FFN_EXPERTS + 1);
  static constexpr int kOffBars = (kOffUnits + 4 * (MOE_MAX_FFN_EXPERTS + 1) + 7) & ~7;
  static constexpr int kNumBars = 2 * kStages + 2 * 2 + 1;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 64 + 1024;  // + alignment slack
};
static_assert(DCfg<kDown>::kSmemBytes <= 232448, "shared memory budget (down dgrad)");
static_assert(DCfg<kUpGate>::kSmemBytes <= 232448, "shared memory budget (up/gate dgrad)");

struct DgradArgs {
  const int32_t* cu;             // [E+1]
  __nv_bfloat16* out0;           // kDown: d_gate [M,H']; kUpGate: grad_x_perm [M,H]
  __nv_bfloat16* out1;           // kDown: d_up [M,H']
  const __nv_bfloat16* gate_pre; // kDown: [M,H']
  const __nv_bfloat16* up_pre;   // kDown: [M,H']
  int32_t* d_status;
  int64_t M;
  int32_t E;
  int32_t k_dim;   // reduction length of one operand pair: H (kDown) or H' (kUpGate)
  int32_t n_feat;  // output features per expert: H' (kDown) or H (kUpGate)
  uint64_t budget_ns;
};

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    dgrad_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                 const __grid_constant__ RowMaps tmB0, const __grid_constant__ RowMaps tmB1,
                 const DgradArgs args) {
  using C = DCfg<kMode>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* s_epi = smem + C::kOffEpi;
  int32_t* s_cu = reinterpret_cast<int32_t*>(smem + C::kOffCu);
  int32_t* s_ustart = reinterpret_cast<int32_t*>(smem + C::kOffUnits);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::kStages;
  uint64_t* tfull = bars + 2 * C::kStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  int32_t* s_scan = reinterpret_cast<int32_t*>(smem + C::kOffMisc + 8);  // [10]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  const int nfb = args.n_feat / kBM;
  const int KT = args.k_dim / kBK;                    // k blocks of one operand pair
  const int KTT = kMode == kUpGate ? 2 * KT : KT;     // k blocks of the whole reduction

  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiThreads / 32);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA0);
    if (kMode == kUpGate) tma_prefetch_map(&tmA1);
    for (int i = 0; i < kNumBoxHeights; ++i) {
      tma_prefetch_map(&tmB0.m[i]);
      if (kMode == kUpGate) tma_prefetch_map(&tmB1.m[i]);
    }
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  griddep_wait();
  griddep_launch_dependents();
  unit_starts(args.cu, args.M, E, nfb, kNMax, s_cu, s_ustart, s_scan);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_units = s_ustart[E];

  if (warp == 0) {
    // TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const Unit U = decode_unit<kNMax>(u, s_ustart, s_cu, E);
        if (U.nrows <= 0) continue;
        const int n = (U.nrows + 15) & ~15;
        const uint32_t bytes = kABytes + n * kRowBytes;
        const uint64_t pol_w = U.ntc > 1 ? pol_keep : pol_stream;
        const int wrow = U.e * args.n_feat + U.fb * kBM;  // first weight row of the tile
        for (int kt = 0; kt < KTT; ++kt) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, args.budget_ns)) break;
          uint8_t* st = smem + stage * C::kStageBytes;
          const bool second = kMode == kUpGate && kt >= KT;
          const int kx = (second ? kt - KT : kt) * kBK;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d_hint(st, second ? &tmA1 : &tmA0, &full[stage], kx, wrow, pol_w);
          const RowMaps& rb = second ? tmB1 : tmB0;
          uint8_t* sb = st + kABytes;
          int r = 0;
#pragma unroll
          for (int i = 0; i < kNumBoxHeights; ++i) {
            const int h = kNMax >> i;
            if (n & h) {
              tma_load_2d_hint(sb + r * kRowBytes, &rb.m[i], &full[stage], kx, U.row0 + r,
                               pol_keep);
              r += h;
            }
          }
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*s_abort) {
        volatile int dummy = 0;
        for (int s = 0; s < C::kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full[s], (issued_phase >> s) & 1u, &dummy, kDrainBudgetNs);
      }
    }
  } else if (warp == 1) {
    // MMA issuer: D[128 features x n tokens] += A(K-major) . B(K-major)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int astage = 0;
      uint32_t aphase = 0;
      bool issued_any = false;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const Unit U = decode_unit<kNMax>(u, s_ustart, s_cu, E);
        if (U.nrows <= 0) continue;
        const uint32_t n = static_cast<uint32_t>((U.nrows + 15) & ~15);
        const uint32_t idesc = idesc_bf16(128, n, 0, 0);
        if (!mbar_wait_bounded(&tempty[astage], aphase ^ 1u, s_abort, args.budget_ns)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + astage * kAccCols;
        bool ok = true;
        for (int kt = 0; kt < KTT; ++kt) {
          if (!mbar_wait_bounded(&full[stage], phase, s_abort, args.budget_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            umma_f16(d, smem_desc_sw128(a0 + kk * 32, 16, 1024),
                     smem_desc_sw128(b0 + kk * 32, 16, 1024), idesc, (kt | kk) != 0 ? 1u : 0u);
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[astage]);
        if (++astage == 2) {
          astage = 0;
          aphase ^= 1u;
        }
      }
      if (*s_abort && issued_any) {
        umma_commit(drain);
        volatile int dummy = 0;
        mbar_wait_bounded(drain, 0, &dummy, kDrainBudgetNs);
      }
    }
  } else {
    // Epilogue: group grp drains the 32-token chunks c with (c / 32) % 2 == grp; warp w reads
    // TMEM lanes 32*(w%4) .. +31, i.e. features f_local = 32*(w%4) + lane of the tile.
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int f_local = q * 32 + lane;
    const int gt = (tid - 64) & 127;
    const uint32_t bar_grp = 1 + grp, bar_all = 3;
    uint8_t* sa_bytes = s_epi + grp * kOutBytes * (kMode == kDown ? 2 : 1);
    uint8_t* sb_bytes = sa_bytes + kOutBytes;  // kDown only
    __nv_bfloat16* sa = reinterpret_cast<__nv_bfloat16*>(sa_bytes);
    __nv_bfloat16* sbuf = reinterpret_cast<__nv_bfloat16*>(sb_bytes);
    int astage = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const Unit U = decode_unit<kNMax>(u, s_ustart, s_cu, E);
      if (U.nrows <= 0) continue;
      const int f0 = U.fb * kBM;
      mbar_wait_bounded(&tfull[astage], aphase, s_abort, args.budget_ns);
      // every epilogue warp takes the same decision
      if (named_bar_red_or(bar_all, kEpiThreads, *s_abort != 0)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + astage * kAccCols;
      for (int c = grp * kOutChunk; c < U.nrows; c += kEpiGroups * kOutChunk) {
        __syncwarp();
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + c, r);
        if (kMode == kDown) {
          // the chunk's saved pre-activations, [32 tokens][128 features], 16-byte vectors
#pragma unroll
          for (int p = 0; p < (kOutChunk * kBM * 2 / 16) / 128; ++p) {
            const int vid = gt + 128 * p;
            const int j = vid >> 4, c16 = vid & 15;
            if (c + j < U.nrows) {
              const int64_t off = static_cast<int64_t>(U.row0 + c + j) * args.n_feat + f0 + c16 * 8;
              *reinterpret_cast<uint4*>(sa_bytes + j * (kBM * 2) + c16 * 16) =
                  __ldg(reinterpret_cast<const uint4*>(args.gate_pre + off));
              *reinterpret_cast<uint4*>(sb_bytes + j * (kBM * 2) + c16 * 16) =
                  __ldg(reinterpret_cast<const uint4*>(args.up_pre + off));
            }
          }
          named_bar_sync(bar_grp, 128);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            // token columns past the unit's rows hold stale staging data; they are computed
            // but never stored
            const float gh = __uint_as_float(r[j]);
            const float g = __bfloat162float(sa[j * kBM + f_local]);
            const float uu = __bfloat162float(sbuf[j * kBM + f_local]);
            const float sg = __fdividef(1.0f, 1.0f + __expf(-g));
            const float ghs = gh * sg;
            sa[j * kBM + f_local] = __float2bfloat16_rn(ghs * uu * (1.0f + g * (1.0f - sg)));
            sbuf[j * kBM + f_local] = __float2bfloat16_rn(ghs * g);
          }
        } else {
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) sa[j * kBM + f_local] = __float2bfloat16_rn(__uint_as_float(r[j]));
        }
        named_bar_sync(bar_grp, 128);
#pragma unroll
        for (int p = 0; p < (kOutChunk * kBM * 2 / 16) / 128; ++p) {
          const int vid = gt + 128 * p;
          const int j = vid >> 4, c16 = vid & 15;
          if (c + j < U.nrows) {
            const int64_t off = static_cast<int64_t>(U.row0 + c + j) * args.n_feat + f0 + c16 * 8;
            *reinterpret_cast<uint4*>(args.out0 + off) =
                *reinterpret_cast<const uint4*>(sa_bytes + j * (kBM * 2) + c16 * 16);
            if (kMode == kDown)
              *reinterpret_cast<uint4*>(args.out1 + off) =
                  *reinterpret_cast<const uint4*>(sb_bytes + j * (kBM * 2) + c16 * 16);
          }
        }
        named_bar_sync(bar_grp, 128);  // staging free for the group's next chunk
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[astage]);
      if (++astage == 2) {
        astage = 0;
        aphase ^= 1u;
      }
    }
  }

  __syncthreads();
  if (tid == 0 && *s_abort && args.d_status != nullptr) atomicOr(args.d_status, MOE_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------------------- weight gradients

constexpr int kWN = 256;                    // gradient columns per unit (UMMA N)
constexpr int kWKB = 64;                    // tokens per stage
constexpr int kWABytes = 2 * kAHalfBytes;   // 16 KB: 128 X features x 64 tokens (MN-major)
constexpr int kWBBytes = 4 * kAHalfBytes;   // 32 KB: 256 D features x 64 tokens (MN-major)
constexpr int kWStageBytes = kWABytes + kWBBytes;
// Default layout: four 48 KB stages (192 KB of operands in flight), one 4 KB staging tile
// per epilogue warp, expert offsets read from global memory. Measured against three stages
// with two tiles and a shared cu_seqlens copy: 0.67 against 0.77 ms at the medium layer.
#ifndef MOE_WGRAD_STAGES
#define MOE_WGRAD_STAGES 4
#endif
#ifndef MOE_WGRAD_EPI_TILES
#define MOE_WGRAD_EPI_TILES 1
#endif
#ifndef MOE_WGRAD_SMEM_CU
#define MOE_WGRAD_SMEM_CU 0
#endif
constexpr int kWStages = MOE_WGRAD_STAGES;
// epilogue staging: per epilogue warp kWEpiTiles 32 x 32 fp32 tiles (4 KB, 128-byte swizzle);
// a tile is refilled once the TMA store that last used it has read it
constexpr int kWEpiTiles = MOE_WGRAD_EPI_TILES;
constexpr int kWEpiTileBytes = 32 * 32 * 4;
constexpr int kWOffEpi = kWStages * kWStageBytes;
constexpr int kWOffCu = kWOffEpi + (kEpiThreads / 32) * kWEpiTiles * kWEpiTileBytes;
// expert row offsets: a shared copy of cu_seqlens, or (when the pipeline needs the room)
// two cached global loads per unit
constexpr int kWCuBytes = MOE_WGRAD_SMEM_CU ? 4 * (MOE_MAX_FFN_EXPERTS + 1) : 0;
constexpr int kWOffBars = (kWOffCu + kWCuBytes + 7) & ~7;
constexpr int kWNumBars = 2 * kWStages + 2 * 2 + 1;
constexpr int kWOffMisc = kWOffBars + 8 * kWNumBars;
constexpr int kWSmemBytes = kWOffMisc + 64 + 1024;
static_assert(kWSmemBytes <= 232448, "shared memory budget (weight gradients)");

constexpr int kWProblems = 3;  // gate, up, down

struct WgradProblem {
  float* out;    // [E][fx][fd] fp32
  int32_t fx;    // gradient rows = features of the X operand
  int32_t fd;    // gradient columns = features of the D operand
  int32_t mbs;      // fx / 128
  int32_t nbs;      // ceil(fd / 256)
  int32_t dblocks;  // 64-feature slices per D box: min(4, fd / 64)
};

struct WgradArgs {
  const int32_t* cu;
  int32_t* d_status;
  int64_t M;
  int32_t E;
  int32_t accumulate;
  uint64_t budget_ns;
  WgradProblem p[kWProblems];
  int32_t pstart[kWProblems + 1];  // first unit of each problem; pstart[3] = total
};

struct WgradMaps {
  CUtensorMap x[kWProblems];    // (64, M, fx/64), box (64, 64, 2)
  CUtensorMap d[kWProblems];    // (64, M, fd/64), box (64, 64, dblocks)
  CUtensorMap out[kWProblems];  // fp32 (fd, E * fx), box (32, 32), 128-byte swizzle
};

struct WUnit {
  int p, e, mb, nb;
};

// Rows [r0, r0 + T) of expert e, clamped to [0, M] (so no row outside [0, M) is addressed).
__device__ __forceinline__ void expert_span_global(const WgradArgs& a, int e, int& r0, int& T) {
  int64_t lo = __ldg(a.cu + e), hi = __ldg(a.cu + e + 1);
  lo = lo < 0 ? 0 : (lo > a.M ? a.M : lo);
  hi = hi < lo ? lo : (hi > a.M ? a.M : hi);
  r0 = static_cast<int>(lo);
  T = static_cast<int>(hi - lo);
}

__device__ __forceinline__ void expert_span(const WgradArgs& a, const int32_t* s_cu, int e,
                                            int& r0, int& T) {
  if (MOE_WGRAD_SMEM_CU) {
    r0 = s_cu[e];
    T = s_cu[e + 1] - r0;
  } else {
    expert_span_global(a, e, r0, T);
  }
}

__device__ __forceinline__ WUnit decode_wunit(int u, const WgradArgs& a) {
  WUnit w;
  w.p = u >= a.pstart[2] ? 2 : (u >= a.pstart[1] ? 1 : 0);
  const WgradProblem& P = a.p[w.p];
  const int per = P.mbs * P.nbs;
  const int local = u - a.pstart[w.p];
  w.e = local / per;
  const int rem = local - w.e * per;
  w.mb = rem / P.nbs;
  w.nb = rem - w.mb * P.nbs;
  return w;
}

__global__ void __launch_bounds__(kThreads, 1)
    wgrad_kernel(const __grid_constant__ WgradMaps maps, const __grid_constant__ WgradArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  int32_t* s_cu = reinterpret_cast<int32_t*>(smem + kWOffCu);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWOffBars);
  uint64_t* full = bars;
  uint64_t* empty = bars + kWStages;
  uint64_t* tfull = bars + 2 * kWStages;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + kWOffMisc);
  volatile int* s_abort = reinterpret_cast<volatile int*>(smem + kWOffMisc + 4);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  const int total_units = args.pstart[kWProblems];

  if (tid == 0) {
    for (int s = 0; s < kWStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiThreads / 32);
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    for (int p = 0; p < kWProblems; ++p) {
      tma_prefetch_map(&maps.x[p]);
      tma_prefetch_map(&maps.d[p]);
      tma_prefetch_map(&maps.out[p]);
    }
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  griddep_wait();
  griddep_launch_dependents();
  if (MOE_WGRAD_SMEM_CU)
    for (int e = tid; e <= E; e += kThreads) {
      int64_t v = args.cu[e];
      v = v < 0 ? 0 : (v > args.M ? args.M : v);
      s_cu[e] = static_cast<int32_t>(v);
    }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;

  if (warp == 0) {
    // TMA producer: per 64-token block, X^T slice (128 features) and D^T slice (256 features)
    if (lane == 0) {
      const uint64_t pol_keep = policy_evict_last();  // every tile of the expert re-reads them
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const WUnit W = decode_wunit(u, args);
        int r0, T;
        expert_span(args, s_cu, W.e, r0, T);
        const int nkb = (T + kWKB - 1) / kWKB;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, args.budget_ns)) break;
          uint8_t* st = smem + stage * kWStageBytes;
          mbar_arrive_expect_tx(&full[stage],
                                static_cast<uint32_t>(kWABytes + args.p[W.p].dblocks * kAHalfBytes));
          tma_load_3d_hint(st, &maps.x[W.p], &full[stage], 0, r0 + kb * kWKB, W.mb * 2, pol_keep);
          tma_load_3d_hint(st + kWABytes, &maps.d[W.p], &full[stage], 0, r0 + kb * kWKB, W.nb * 4,
                           pol_keep);
          issued_mask |= 1u << stage;
          issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kWStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (*s_abort) {
        volatile int dummy = 0;
        for (int s = 0; s < kWStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full[s], (issued_phase >> s) & 1u, &dummy, kDrainBudgetNs);
      }
    }
  } else if (warp == 1) {
    // MMA issuer (the whole warp: it zeroes the rows past an expert's end, lane 0 issues)
    int stage = 0;
    uint32_t phase = 0;
    int astage = 0;
    uint32_t aphase = 0;
    bool issued_any = false;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      if (__shfl_sync(0xffffffffu, *s_abort, 0)) break;  // lane 0's view: a uniform exit
      const WUnit W = decode_wunit(u, args);
      int r0, T;
      expert_span(args, s_cu, W.e, r0, T);
      if (T <= 0) continue;
      const int nkb = (T + kWKB - 1) / kWKB;
      const int fd = args.p[W.p].fd;
      const uint32_t n = static_cast<uint32_t>(min(kWN, fd - W.nb * kWN));  // 128 or 256
      const uint32_t idesc = idesc_bf16(128, n, 1, 1);
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&tempty[astage], aphase ^ 1u, s_abort, args.budget_ns);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const uint32_t d = tmem_base + astage * kAccCols;
      for (int kb = 0; kb < nkb; ++kb) {
        if (lane == 0) ok = mbar_wait_bounded(&full[stage], phase, s_abort, args.budget_ns);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + stage * kWStageBytes;
        const int valid = min(kWKB, T - kb * kWKB);
        const int kcut = (valid + 15) & ~15;
        if (valid < kcut) {
          // rows valid .. kcut-1 of every 64-feature slice belong to the next expert (or are
          // past the end of the matrix): zero them. A row is 128 contiguous bytes in the
          // swizzled layout, so this is independent of the swizzle pattern.
          const int rows = kcut - valid;
          for (int i = lane; i < 6 * rows * 8; i += 32) {
            const int slice = i / (rows * 8);
            const int rem = i - slice * rows * 8;
            const int row = valid + rem / 8, v16 = rem & 7;
            *reinterpret_cast<uint4*>(st + slice * kAHalfBytes + row * 128 + v16 * 16) =
                make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        __syncwarp();
        if (lane == 0) {
          tc_fence_after();
          const uint32_t a0 = smem_u32(st);
          const uint32_t b0 = a0 + kWABytes;
          for (int kk = 0; kk < kcut / 16; ++kk)
            umma_f16(d, smem_desc_sw128(a0 + kk * 2048, kAHalfBytes, 1024),
                     smem_desc_sw128(b0 + kk * 2048, kAHalfBytes, 1024), idesc,
                     (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&empty[stage]);
        }
        issued_any = true;
        __syncwarp();
        if (++stage == kWStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) umma_commit(&tfull[astage]);
      __syncwarp();
      if (++astage == 2) {
        astage = 0;
        aphase ^= 1u;
      }
    }
    if (*s_abort && issued_any && lane == 0) {
      umma_commit(drain);
      volatile int dummy = 0;
      mbar_wait_bounded(drain, 0, &dummy, kDrainBudgetNs);
    }
    __syncwarp();
  } else {
    // Epilogue: warp w owns gradient rows 32*(w%4) .. +31 of the tile (TMEM lanes); group
    // grp takes the 32-column chunks c with (c / 32) % 2 == grp. A chunk (32 rows x 32 fp32)
    // goes TMEM -> registers -> a 128-byte-swizzled shared tile (16-byte chunk j of row r at
    // position j ^ (r % 8), conflict-free) -> one TMA bulk store (or, when accumulating, a
    // TMA reduce-add: the fp32 addition happens at L2 and the prior values never reach the SM).
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;
    const uint32_t bar_all = 3;
    uint8_t* tiles = smem + kWOffEpi + (warp - 2) * kWEpiTiles * kWEpiTileBytes;
    int ci = 0;  // chunks this warp has staged; tile (ci % kWEpiTiles) is the next one to fill
    int astage = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const WUnit W = decode_wunit(u, args);
      const WgradProblem& P = args.p[W.p];
      int r0_unused, T;
      expert_span(args, s_cu, W.e, r0_unused, T);
      const int ncols = min(kWN, P.fd - W.nb * kWN);
      const int row0 = W.e * P.fx + W.mb * kBM + q * 32;  // first gradient row of this warp
      if (T <= 0) {
        // an expert without tokens: zero gradient (nothing to add when accumulating)
        if (!args.accumulate) {
          float* dst_row = P.out + static_cast<int64_t>(row0 + lane) * P.fd + W.nb * kWN;
          for (int c = grp * kOutChunk; c < ncols; c += kEpiGroups * kOutChunk)
#pragma unroll
            for (int v = 0; v < 8; ++v)
              *reinterpret_cast<float4*>(dst_row + c + 4 * v) = make_float4(0.f, 0.f, 0.f, 0.f);
        }
        continue;
      }
      mbar_wait_bounded(&tfull[astage], aphase, s_abort, args.budget_ns);
      // every epilogue warp takes the same decision
      if (named_bar_red_or(bar_all, kEpiThreads, *s_abort != 0)) break;
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + astage * kAccCols;
      for (int c = grp * kOutChunk; c < ncols; c += kEpiGroups * kOutChunk) {
        __syncwarp();
        uint32_t r[32];
        tmem_ld_32x32b_x32(tbase + c, r);
        // the tile about to be filled was stored kWEpiTiles chunks ago: that store must have
        // read it
        if (lane == 0) bulk_wait_group_read<kWEpiTiles - 1>();
        __syncwarp();
        tmem_ld_wait();
        uint8_t* tile = tiles + (ci % kWEpiTiles) * kWEpiTileBytes;
#pragma unroll
        for (int v = 0; v < 8; ++v)
          *reinterpret_cast<uint4*>(tile + lane * 128 + ((v ^ (lane & 7)) * 16)) =
              make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const int x = W.nb * kWN + c;
          if (args.accumulate)
            tma_reduce_add_2d(&maps.out[W.p], tile, x, row0);
          else
            tma_store_2d(&maps.out[W.p], tile, x, row0);
          bulk_commit_group();
        }
        ++ci;
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[astage]);
      if (++astage == 2) {
        astage = 0;
        aphase ^= 1u;
      }
    }
    if (lane == 0) bulk_wait_group<0>();  // this warp's stores complete before the CTA exits
    __syncwarp();
  }

  __syncthreads();
  if (tid == 0 && *s_abort && args.d_status != nullptr) atomicOr(args.d_status, MOE_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------------------- host side

template <typename Kernel>
bool ensure_smem(Kernel kernel, int bytes, ContextCache& done) {
  return set_smem_optin(reinterpret_cast<const void*>(kernel), bytes, done);
}

ContextCache g_smem_down, g_smem_upgate, g_smem_wgrad;

}  // namespace

moe_status launch_ffn_down_backward(const void* grad_y, const void* w_down, const void* gate_pre,
                                    const void* up_pre, const int32_t* cu_seqlens, int64_t M,
                                    int64_t H, int64_t Hp, int32_t E, void* d_gate, void* d_up,
                                    int32_t* d_status, cudaStream_t stream) {
  CUtensorMap m_wd;
  RowMaps m_gy;
  // W_down [E*H', H]: rows are output features, 128 per box, K (= H) contiguous
  if (!make_row_map(&m_wd, w_down, H, static_cast<uint64_t>(E) * Hp, kBM) ||
      !make_row_maps(&m_gy, grad_y, H, M) ||
      !ensure_smem(dgrad_kernel<kDown>, DCfg<kDown>::kSmemBytes, g_smem_down))
    return MOE_ERR_CUDA;
  const DgradArgs a{cu_seqlens,
                    static_cast<__nv_bfloat16*>(d_gate),
                    static_cast<__nv_bfloat16*>(d_up),
                    static_cast<const __nv_bfloat16*>(gate_pre),
                    static_cast<const __nv_bfloat16*>(up_pre),
                    d_status,
                    M,
                    E,
                    static_cast<int32_t>(H),
                    static_cast<int32_t>(Hp),
                    wait_budget_ns()};
  const cudaError_t err =
      launch_dependent(dgrad_kernel<kDown>, dim3(num_sms()), dim3(kThreads),
                       DCfg<kDown>::kSmemBytes, stream, m_wd, m_wd, m_gy, m_gy, a);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_ffn_up_gate_backward(const void* d_gate, const void* d_up, const void* w_gate,
                                       const void* w_up, const int32_t* cu_seqlens, int64_t M,
                                       int64_t H, int64_t Hp, int32_t E, void* grad_x_perm,
                                       int32_t* d_status, cudaStream_t stream) {
  CUtensorMap m_wg, m_wu;
  RowMaps m_dg, m_du;
  // W_gate, W_up [E*H, H']: rows are output features (of H), K (= H') contiguous
  if (!make_row_map(&m_wg, w_gate, Hp, static_cast<uint64_t>(E) * H, kBM) ||
      !make_row_map(&m_wu, w_up, Hp, static_cast<uint64_t>(E) * H, kBM) ||
      !make_row_maps(&m_dg, d_gate, Hp, M) || !make_row_maps(&m_du, d_up, Hp, M) ||
      !ensure_smem(dgrad_kernel<kUpGate>, DCfg<kUpGate>::kSmemBytes, g_smem_upgate))
    return MOE_ERR_CUDA;
  const DgradArgs a{cu_seqlens,
                    static_cast<__nv_bfloat16*>(grad_x_perm),
                    nullptr,
                    nullptr,
                    nullptr,
                    d_status,
                    M,
                    E,
                    static_cast<int32_t>(Hp),
                    static_cast<int32_t>(H),
                    wait_budget_ns()};
  const cudaError_t err =
      launch_dependent(dgrad_kernel<kUpGate>, dim3(num_sms()), dim3(kThreads),
                       DCfg<kUpGate>::kSmemBytes, stream, m_wg, m_wu, m_dg, m_du, a);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_ffn_weight_grad(const void* x_perm, const void* h, const void* d_gate,
                                  const void* d_up, const void* grad_y, const int32_t* cu_seqlens,
                                  int64_t M, int64_t H, int64_t Hp, int32_t E, float* grad_w_gate,
                                  float* grad_w_up, float* grad_w_down, bool accumulate,
                                  int32_t* d_status, cudaStream_t stream) {
  WgradMaps maps;
  // problem 0: x^T d_gate, 1: x^T d_up ([H, H']), 2: h^T grad_y ([H', H])
  const void* xs[kWProblems] = {x_perm, x_perm, h};
  const void* ds[kWProblems] = {d_gate, d_up, grad_y};
  float* outs[kWProblems] = {grad_w_gate, grad_w_up, grad_w_down};
  const int64_t fxs[kWProblems] = {H, H, Hp};
  const int64_t fds[kWProblems] = {Hp, Hp, H};
  WgradArgs a{};
  a.cu = cu_seqlens;
  a.d_status = d_status;
  a.M = M;
  a.E = E;
  a.accumulate = accumulate ? 1 : 0;
  a.budget_ns = wait_budget_ns();
  int64_t units = 0;
  for (int p = 0; p < kWProblems; ++p) {
    WgradProblem& P = a.p[p];
    P.dblocks = static_cast<int32_t>(fds[p] / 64 < 4 ? fds[p] / 64 : 4);
    if (!make_weight_map(&maps.x[p], xs[p], fxs[p], M, 2) ||
        !make_weight_map(&maps.d[p], ds[p], fds[p], M, static_cast<uint32_t>(P.dblocks)) ||
        !make_f32_tile_map(&maps.out[p], outs[p], fds[p], static_cast<uint64_t>(E) * fxs[p], 32,
                           32))
      return MOE_ERR_CUDA;
    P.out = outs[p];
    P.fx = static_cast<int32_t>(fxs[p]);
    P.fd = static_cast<int32_t>(fds[p]);
    P.mbs = static_cast<int32_t>(fxs[p] / kBM);
    P.nbs = static_cast<int32_t>(ceil_div(fds[p], kWN));
    a.pstart[p] = static_cast<int32_t>(units);
    units += static_cast<int64_t>(E) * P.mbs * P.nbs;
  }
  if (units > INT32_MAX) return MOE_ERR_UNSUPPORTED_SHAPE;
  a.pstart[kWProblems] = static_cast<int32_t>(units);
  if (!ensure_smem(wgrad_kernel, kWSmemBytes, g_smem_wgrad)) return MOE_ERR_CUDA;
  const cudaError_t err = launch_dependent(wgrad_kernel, dim3(num_sms()), dim3(kThreads),
                                           kWSmemBytes, stream, maps, a);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
