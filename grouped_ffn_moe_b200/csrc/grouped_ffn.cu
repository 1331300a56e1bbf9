// Grouped expert SwiGLU FFN on 5th-generation tensor cores (tcgen05 + TMEM + TMA), sm_100a.
//
// Computes, for every expert e and every row r of e's contiguous block
// [cu_seqlens[e], cu_seqlens[e+1]) ("Mixture of Kittens" digest, Step 1; MoonEP README,
// "Integration" and "Weight buffer": experts addressed by row index of one contiguous
// [E, H, H'] tensor per projection, cu_seqlens selects the rows):
//
//   pass 1 (SwiGLU): h[r] = bf16( silu(x[r] . W_gate[e]) * (x[r] . W_up[e]) )
//   pass 2:          y[r] = bf16( h[r] . W_down[e] )
//
// Design ("swap AB"): the tensor-core M side (128) runs over output features and the N side
// over an expert's tokens, D^T[f, tok] = sum_k W[e][k, f] * X[tok, k]. Expert sizes are
// ragged and often small (171 rows on average at S=8192, K=8, E=384); with tokens on N the
// MMA shape follows the expert exactly up to the next multiple of 16 (N = 16..256), where
// tokens on M would pad every expert to multiples of 128. The weight tile (A) is
// MN-major (features contiguous, as stored), the token tile (B) K-major; both are loaded
// by TMA with 128-byte swizzle, which is the canonical UMMA shared-memory layout.
//
// Work unit = (expert, 128-feature block, chunk of <= 256 of the expert's tokens). Units are
// enumerated expert-major, then feature block, then chunk, and a persistent grid of one CTA
// per SM strides over them: CTAs that run at the same time share the expert's token rows
// (and, for an expert split into chunks, its weight tile) through L2, so each weight byte
// crosses HBM about once, and a hot expert's chunks spread over all SMs.
//
// Warp roles (320 threads): warp 0 issues TMA loads into a kStages-deep shared-memory ring;
// warp 1 owns TMEM (alloc/dealloc) and issues the MMAs from one thread; warps 2-9 (two groups
// of four, alternating 32-token chunks) drain the fp32 accumulators with tcgen05.ld, apply
// SiLU*up (pass 1) and rounding, transpose through shared memory and store whole 16-byte
// vectors of the expert's rows only. For training, pass 1 also stores the pre-activations
// bf16(x.W_gate) and bf16(x.W_up) that the backward differentiates SwiGLU at.
// Every wait is bounded (globaltimer); on expiry the CTA records MOE_ERR_DEVICE_TIMEOUT,
// drains its own copies and MMAs with bounded waits, frees TMEM and exits.
#include "gemm_common.cuh"

namespace moe {
namespace {

#ifndef MOE_SWIGLU_NMAX
#define MOE_SWIGLU_NMAX 256                    // tokens per SwiGLU unit (128: two TMEM stages)
#endif

// Kernel modes.
//   kSwiGLU: A0 = W_gate, A1 = W_up on the same 128 features; h = silu(acc0) * acc1.
//   kSwiGLUGather: kSwiGLU whose token tile is gathered straight from the token-major x
//            (row r of the expert-grouped order is token perm_src[r] / K) by four extra
//            gather warps' 16-byte cp.async copies into the same swizzled layout: the
//            permutation's row copy x_perm is never materialised (the zero-copy fusion of the
//            MoonEP README, "Zero-copy"). Measured alternatives: one TMA tile::gather4 per four
//            rows (2.9x slower: the per-instruction cost set the pace) and cp.async from the
//            producer warp alone (2.9x slower: one warp keeps too few copies in flight).
//   kPair:   A0, A1 = two adjacent 128-feature blocks of one weight tensor sharing the token
//            tile (half the token-row traffic per feature); y = acc0 | acc1.
enum Mode : int { kSwiGLU = 0, kPair = 2, kSwiGLUGather = 3 };

template <int kMode>
struct Cfg {
  static constexpr bool kSwi = kMode == kSwiGLU || kMode == kSwiGLUGather;
  // gather: four more warps (10-13) copy the token rows
  static constexpr int kGatherWarps = kMode == kSwiGLUGather ? 4 : 0;
  static constexpr int kBlock = kThreads + 32 * kGatherWarps;
  static constexpr int kNumA = 2;
  static constexpr int kNMaxMode = kSwi ? MOE_SWIGLU_NMAX : kNMax;
  // accumulator stages: two when they fit in TMEM (N <= 128 tokens per unit)
  static constexpr int kAccStages = kNMaxMode <= 128 ? 2 : 1;
  static constexpr int kUpOff = kAccStages == 2 ? kNMaxMode : 256;  // up accumulator column
  static constexpr int kFeatPerUnit = kMode == kPair ? 2 * kBM : kBM;
  static constexpr int kStageBytes = kNumA * kABytes + kNMaxMode * kBK * 2;
  static constexpr int kStages = (192 * 1024) / kStageBytes;
  static constexpr int kPipeBytes = kStages * kStageBytes;
  static constexpr int kOffOut = kPipeBytes;
  static constexpr int kOffCu = kOffOut + kEpiGroups * kOutBytes;
  static constexpr int kOffUnits = kOffCu + 4 * (MOE_MAX_FFN_EXPERTS + 1);
  static constexpr int kOffBars = (kOffUnits + 4 * (MOE_MAX_FFN_EXPERTS + 1) + 7) & ~7;
  static constexpr int kNumBars = 2 * kStages + 2 * 2 + 1;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 128 + 1024;  // + alignment slack
};
static_assert(Cfg<kSwiGLU>::kSmemBytes <= 232448, "shared memory budget (SwiGLU)");
static_assert(Cfg<kSwiGLUGather>::kSmemBytes == Cfg<kSwiGLU>::kSmemBytes, "gather layout");
static_assert(Cfg<kPair>::kSmemBytes <= 232448, "shared memory budget (pair)");

struct FfnArgs {
  const int32_t* cu;     // [E+1]
  __nv_bfloat16* out;    // [M, n_feat]
  int32_t* d_status;
  int64_t M;
  int32_t E;
  int32_t k_dim;         // reduction length: H (pass 1) or H' (pass 2)
  int32_t n_feat;        // output features: H' (pass 1) or H (pass 2)
  uint64_t budget_ns;
  __nv_bfloat16* gate_pre;  // [M, H'] bf16(x.W_gate), pass 1 when training; else null
  __nv_bfloat16* up_pre;    // [M, H'] bf16(x.W_up), with gate_pre
  const int32_t* perm_src;  // kSwiGLUGather: [M] flat slot of each row; token = slot / route_k
  int32_t route_k;          // kSwiGLUGather: K
  const __nv_bfloat16* x;   // kSwiGLUGather: token-major [S, k_dim]
  int64_t S;                // kSwiGLUGather: rows of x
};

template <int kMode>
__global__ void __launch_bounds__(Cfg<kMode>::kBlock, 1)
    grouped_ffn_kernel(const __grid_constant__ CUtensorMap tmA0,
                       const __grid_constant__ CUtensorMap tmA1,
                       const __grid_constant__ RowMaps tmB, const FfnArgs args) {
  using C = Cfg<kMode>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_1024(smem_raw);
  uint8_t* s_out = smem + C::kOffOut;
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
  int32_t* s_scan = reinterpret_cast<int32_t*>(smem + C::kOffMisc + 8);  // [kBlock / 32]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = args.E;
  const int nfb = (args.n_feat + C::kFeatPerUnit - 1) / C::kFeatPerUnit;
  const int KT = args.k_dim / kBK;

  // ------------------------------------------------------------------ prologue
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // gather: the weight loads' arrive.expect_tx plus one cp.async arrival per gather lane
      mbar_init(&full[s], 1 + 32 * C::kGatherWarps);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&tfull[s], 1);
      mbar_init(&tempty[s], kEpiThreads / 32);  // one arrival per epilogue warp
    }
    mbar_init(drain, 1);
    *s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&tmA0);
    if (C::kSwi) tma_prefetch_map(&tmA1);
    if (kMode != kSwiGLUGather)  // gather mode reads no token-row map
      for (int i = 0; i < kNumBoxHeights; ++i) tma_prefetch_map(&tmB.m[i]);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  // everything above overlaps the previous kernel's tail (programmatic dependent launch);
  // cu_seqlens and the activations come from earlier kernels in the stream
  griddep_wait();
  griddep_launch_dependents();
  unit_starts<C::kBlock>(args.cu, args.M, E, nfb, C::kNMaxMode, s_cu, s_ustart, s_scan);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_units = s_ustart[E];

  // ------------------------------------------------------------------ roles
  if (kMode == kSwiGLUGather && warp >= 2 + kEpiThreads / 32) {
    // Gather warps g = 0..3. Per unit each lane loads the tokens of its 16 rows,
    // r = 16i + 4g + (lane >> 3), into registers (rows past the unit, up to the 16-row
    // rounding, repeat its last row; their MMA columns are never stored). Per stage, after
    // the slot is free, lane (8 * row-in-group + piece) copies 16-byte piece `piece` of its
    // row's 128-byte segment with cp.async into the 128-byte-swizzled K-major token tile
    // (piece c of row r at r*128 + ((c ^ (r % 8)) * 16)) and arrives when its copies land.
    const int g = warp - (2 + kEpiThreads / 32);
    const int piece = lane & 7;
    const int rsub = lane >> 3;
    int stage = 0;
    uint32_t phase = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < total_units && !stop; u += gridDim.x) {
      if (__shfl_sync(0xffffffffu, *s_abort, 0)) break;  // lane 0's view: a uniform exit
      const Unit U = decode_unit<C::kNMaxMode>(u, s_ustart, s_cu, E);
      if (U.nrows <= 0) continue;
      const int n = (U.nrows + 15) & ~15;
      int tok[C::kNMaxMode / 16];
#pragma unroll
      for (int i = 0; i < C::kNMaxMode / 16; ++i) {
        const int r = min(16 * i + 4 * g + rsub, U.nrows - 1);
        int64_t t = __ldg(args.perm_src + U.row0 + r) / args.route_k;
        t = t < 0 ? 0 : (t >= args.S ? args.S - 1 : t);  // any perm_src stays inside x
        tok[i] = static_cast<int32_t>(t);
      }
      for (int kt = 0; kt < KT; ++kt) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, args.budget_ns);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        const uint32_t sb = smem_u32(smem + stage * C::kStageBytes + C::kNumA * kABytes);
        const __nv_bfloat16* xk = args.x + kt * kBK + piece * 8;
#pragma unroll
        for (int i = 0; i < C::kNMaxMode / 16; ++i) {
          if (16 * i < n) {  // uniform
            const int r = 16 * i + 4 * g + rsub;
            cp_async_16(sb + r * kRowBytes + ((piece ^ (r & 7)) << 4),
                        xk + static_cast<int64_t>(tok[i]) * args.k_dim);
          }
        }
        cp_async_mbar_arrive_noinc(&full[stage]);
        if (++stage == C::kStages) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // own copies land before the CTA exits
  } else if (warp == 0) {
    // TMA producer
    if (lane == 0) {
      const uint64_t pol_stream = policy_evict_first();  // weights read by one unit only
      const uint64_t pol_keep = policy_evict_last();     // token rows (all feature blocks) and
                                                         // weights shared by an expert's chunks
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const Unit U = decode_unit<C::kNMaxMode>(u, s_ustart, s_cu, E);
        if (U.nrows <= 0) continue;
        const int n = (U.nrows + 15) & ~15;
        // gather: the token rows arrive by the gather warps' cp.async, not by TMA
        const uint32_t bytes = C::kNumA * kABytes + (kMode == kSwiGLUGather ? 0 : n * kRowBytes);
        const uint64_t pol_w = U.ntc > 1 ? pol_keep : pol_stream;
        const int fz = U.fb * (C::kFeatPerUnit / 64);  // 64-feature index of the first feature
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, args.budget_ns)) break;
          uint8_t* st = smem + stage * C::kStageBytes;
          const int ky = U.e * args.k_dim + kt * kBK;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_3d_hint(st, &tmA0, &full[stage], 0, ky, fz, pol_w);
          if (C::kSwi) tma_load_3d_hint(st + kABytes, &tmA1, &full[stage], 0, ky, fz, pol_w);
          // second block of a pair; past the last feature the box is zero-filled (not stored)
          if (kMode == kPair) tma_load_3d_hint(st + kABytes, &tmA0, &full[stage], 0, ky, fz + 2, pol_w);
          uint8_t* sb = st + C::kNumA * kABytes;
          int r = 0;
#pragma unroll
          for (int i = 0; i < kNumBoxHeights; ++i) {
            const int h = kNMax >> i;
            if (kMode != kSwiGLUGather && (n & h)) {
              tma_load_2d_hint(sb + r * kRowBytes, &tmB.m[i], &full[stage], kt * kBK, U.row0 + r,
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
        // let this CTA's own copies land before the CTA exits (bounded)
        volatile int dummy = 0;
        for (int s = 0; s < C::kStages; ++s)
          if (issued_mask & (1u << s))
            mbar_wait_bounded(&full[s], (issued_phase >> s) & 1u, &dummy, kDrainBudgetNs);
      }
    }
  } else if (warp == 1) {
    // MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int astage = 0;
      uint32_t aphase = 0;
      bool issued_any = false;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const Unit U = decode_unit<C::kNMaxMode>(u, s_ustart, s_cu, E);
        if (U.nrows <= 0) continue;
        const uint32_t n = static_cast<uint32_t>((U.nrows + 15) & ~15);
        const uint32_t idesc = idesc_bf16_m128_amn_bk(n);
        if (!mbar_wait_bounded(&tempty[astage], aphase ^ 1u, s_abort, args.budget_ns)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + astage * kAccCols;  // astage is 0 with one stage
        const uint32_t d1 = d0 + (C::kSwi ? C::kUpOff : kAccCols);
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_bounded(&full[stage], phase, s_abort, args.budget_ns)) {
            ok = false;
            break;
          }
          // gather: the token rows were written by cp.async (generic proxy)
          if (kMode == kSwiGLUGather) fence_proxy_async_smem();
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t a1 = a0 + kABytes;
          const uint32_t b0 = a0 + C::kNumA * kABytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(b0 + kk * 32, 16, 1024);
            const uint32_t acc = (kt | kk) != 0 ? 1u : 0u;
            umma_f16(d0, smem_desc_sw128(a0 + kk * 2048, kAHalfBytes, 1024), bdesc, idesc, acc);
            umma_f16(d1, smem_desc_sw128(a1 + kk * 2048, kAHalfBytes, 1024), bdesc, idesc, acc);
          }
          issued_any = true;
          umma_commit(&empty[stage]);  // frees the smem stage when these MMAs complete
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[astage]);  // accumulator ready for the epilogue
        if (++astage == C::kAccStages) {
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
    // Epilogue: warps 2..9 in two groups of four (warps 2-5 and 6-9); group g drains the
    // 32-token chunks c with (c / 32) % 2 == g. Warp w reads TMEM lanes 32*(w%4) .. +31, i.e.
    // 32 of the unit's 128 features, and within a group the four warps cover all 128. A warp
    // releases the accumulator as soon as its last chunk of the unit is in registers, so the
    // next unit's MMAs overlap that chunk's SwiGLU, conversion and stores.
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int f_local = q * 32 + lane;
    const int gt = (tid - 64) & 127;  // thread index inside the group
    const uint32_t bar_grp = 1 + grp, bar_all = 3;
    uint8_t* so_bytes = s_out + grp * kOutBytes;
    __nv_bfloat16* so = reinterpret_cast<__nv_bfloat16*>(so_bytes);
    int astage = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const Unit U = decode_unit<C::kNMaxMode>(u, s_ustart, s_cu, E);
      if (U.nrows <= 0) continue;
      mbar_wait_bounded(&tfull[astage], aphase, s_abort, args.budget_ns);
      // every epilogue warp takes the same decision
      if (named_bar_red_or(bar_all, kEpiThreads, *s_abort != 0)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + astage * kAccCols;
      bool released = false;
      const int nhalf = (kMode == kPair && U.fb * C::kFeatPerUnit + kBM < args.n_feat) ? 2 : 1;
      for (int c = grp * kOutChunk; c < U.nrows; c += kEpiGroups * kOutChunk) {
        const bool last_chunk = c + kEpiGroups * kOutChunk >= U.nrows;
        // kPair: two 128-feature halves per chunk; otherwise one
        for (int half = 0; half < nhalf; ++half) {
          const int f0 = U.fb * C::kFeatPerUnit + half * kBM;
          const bool last = last_chunk && half == nhalf - 1;
          __syncwarp();  // tcgen05.ld is .sync.aligned: whole warp, converged
          // staged chunk [32 tokens][128 features] -> rows of dst (row stride n_feat)
          auto store_chunk = [&](__nv_bfloat16* dst_base) {
            named_bar_sync(bar_grp, 128);
#pragma unroll
            for (int p = 0; p < (kOutChunk * kBM * 2 / 16) / 128; ++p) {
              const int vid = gt + 128 * p;
              const int j = vid >> 4, c16 = vid & 15;
              if (c + j < U.nrows) {
                const uint4 val =
                    *reinterpret_cast<const uint4*>(so_bytes + j * (kBM * 2) + c16 * 16);
                __nv_bfloat16* dst = dst_base +
                                     static_cast<int64_t>(U.row0 + c + j) * args.n_feat + f0 +
                                     c16 * 8;
                *reinterpret_cast<uint4*>(dst) = val;
              }
            }
            named_bar_sync(bar_grp, 128);  // staging buffer free for the group's next use
          };
          uint32_t r0[32], r1[32];
          tmem_ld_32x32b_x32(tbase + half * kAccCols + c, r0);
          if (C::kSwi) {
            tmem_ld_32x32b_x32(tbase + C::kUpOff + c, r1);
            tmem_ld_wait();
            if (last) {  // the unit's accumulator is all in registers: release it
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[astage]);
              released = true;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              // silu(g) * u = g / (1 + e^-g) * u (fast exp and divide; the result is rounded
              // to bf16, whose step is 2^16 times coarser than their error)
              const float g = __uint_as_float(r0[j]);
              const float hval = __fdividef(g, 1.0f + __expf(-g)) * __uint_as_float(r1[j]);
              so[j * kBM + f_local] = __float2bfloat16_rn(hval);
            }
          } else {
            tmem_ld_wait();
            if (last) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&tempty[astage]);
              released = true;
            }
#pragma unroll
            for (int j = 0; j < 32; ++j)
              so[j * kBM + f_local] = __float2bfloat16_rn(__uint_as_float(r0[j]));
          }
          store_chunk(args.out);
          if (C::kSwi && args.gate_pre != nullptr) {
            // training: the pre-activations, each rounded once from the fp32 accumulator
#pragma unroll
            for (int j = 0; j < 32; ++j)
              so[j * kBM + f_local] = __float2bfloat16_rn(__uint_as_float(r0[j]));
            store_chunk(args.gate_pre);
#pragma unroll
            for (int j = 0; j < 32; ++j)
              so[j * kBM + f_local] = __float2bfloat16_rn(__uint_as_float(r1[j]));
            store_chunk(args.up_pre);
          }
        }
      }
      if (!released) {  // this group had no chunk of the unit
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[astage]);
      }
      if (++astage == C::kAccStages) {
        astage = 0;
        aphase ^= 1u;
      }
    }
  }

  // ------------------------------------------------------------------ teardown
  __syncthreads();
  if (tid == 0 && *s_abort && args.d_status != nullptr) atomicOr(args.d_status, MOE_ERR_DEVICE_TIMEOUT);
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ----------------------------------------------------------------------------- host side

template <int kMode>
bool ensure_smem_attr() {
  static ContextCache done;
  return set_smem_optin(reinterpret_cast<const void*>(grouped_ffn_kernel<kMode>),
                        Cfg<kMode>::kSmemBytes, done);
}

}  // namespace

moe_status launch_ffn_up_gate_gather(const void* x, const int32_t* perm_src, int64_t S, int32_t K,
                                     const void* w_gate, const void* w_up,
                                     const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                                     int32_t E, void* h, void* gate_pre, void* up_pre,
                                     int32_t* d_status, cudaStream_t stream) {
  CUtensorMap m_wg, m_wu;
  RowMaps m_x = {};
  // token rows come by cp.async from x itself: the row-map table is unused in this mode
  if (!make_weight_map(&m_wg, w_gate, Hp, static_cast<uint64_t>(E) * H) ||
      !make_weight_map(&m_wu, w_up, Hp, static_cast<uint64_t>(E) * H) ||
      !ensure_smem_attr<kSwiGLUGather>())
    return MOE_ERR_CUDA;
  const FfnArgs a{cu_seqlens, static_cast<__nv_bfloat16*>(h), d_status, M, E,
                  static_cast<int32_t>(H), static_cast<int32_t>(Hp), wait_budget_ns(),
                  static_cast<__nv_bfloat16*>(gate_pre), static_cast<__nv_bfloat16*>(up_pre),
                  perm_src, K, static_cast<const __nv_bfloat16*>(x), S};
  const cudaError_t err =
      launch_dependent(grouped_ffn_kernel<kSwiGLUGather>, dim3(num_sms()),
                       dim3(Cfg<kSwiGLUGather>::kBlock),
                       Cfg<kSwiGLUGather>::kSmemBytes, stream, m_wg, m_wu, m_x, a);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_ffn_pass(bool dual, const void* act, const void* w0, const void* w1,
                           const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp, int32_t E,
                           void* out, void* gate_pre, void* up_pre, int32_t* d_status,
                           cudaStream_t stream) {
  const int grid = num_sms();
  if (dual) {
    CUtensorMap m_wg, m_wu;
    RowMaps m_x;
    if (!make_weight_map(&m_wg, w0, Hp, static_cast<uint64_t>(E) * H) ||
        !make_weight_map(&m_wu, w1, Hp, static_cast<uint64_t>(E) * H) ||
        !make_row_maps(&m_x, act, H, M) || !ensure_smem_attr<kSwiGLU>())
      return MOE_ERR_CUDA;
    const FfnArgs a{cu_seqlens, static_cast<__nv_bfloat16*>(out), d_status, M, E,
                    static_cast<int32_t>(H), static_cast<int32_t>(Hp), wait_budget_ns(),
                    static_cast<__nv_bfloat16*>(gate_pre), static_cast<__nv_bfloat16*>(up_pre),
                    nullptr, 1, nullptr, 0};
    const cudaError_t err =
        launch_dependent(grouped_ffn_kernel<kSwiGLU>, dim3(grid), dim3(kThreads),
                         Cfg<kSwiGLU>::kSmemBytes, stream, m_wg, m_wu, m_x, a);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  } else {
    CUtensorMap m_wd;
    RowMaps m_h;
    if (!make_weight_map(&m_wd, w0, H, static_cast<uint64_t>(E) * Hp) ||
        !make_row_maps(&m_h, act, Hp, M) || !ensure_smem_attr<kPair>())
      return MOE_ERR_CUDA;
    const FfnArgs a{cu_seqlens, static_cast<__nv_bfloat16*>(out), d_status, M, E,
                    static_cast<int32_t>(Hp), static_cast<int32_t>(H), wait_budget_ns(),
                    nullptr, nullptr, nullptr, 1, nullptr, 0};
    const cudaError_t err = launch_dependent(grouped_ffn_kernel<kPair>, dim3(grid),
                                             dim3(kThreads), Cfg<kPair>::kSmemBytes, stream,
                                             m_wd, m_wd, m_h, a);
    if (err != cudaSuccess) return MOE_ERR_CUDA;
  }
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
