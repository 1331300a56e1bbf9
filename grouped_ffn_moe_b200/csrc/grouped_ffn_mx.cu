// MXFP8 grouped expert SwiGLU FFN on block-scaled 5th-generation tensor cores, sm_100a.
//
// The computation of grouped_ffn.cu with its operands in MXFP8, the low-precision mode the
// "Mixture of Kittens" digest (Step 8) names for the expert GEMMs: FP8 E4M3 elements with one
// E8M0 power-of-two scale per 32 consecutive elements along the reduction dimension (OCP
// Microscaling Formats v1.0). Weights are quantised once ahead of time; activations are
// quantised where they are produced (x while it is permuted, h in the SwiGLU epilogue):
//
//   pass 1: h = silu(deq(x_q) . deq(Wg_q)) * (deq(x_q) . deq(Wu_q)), stored as MXFP8 along H'
//   pass 2: y = bf16(deq(h_q) . deq(Wd_q))
//
// Each MMA is tcgen05.mma kind::mxf8f6f4.block_scale (K = 32, one scale per operand row per
// instruction); the scales of a 128-k stage sit in tensor memory beside the accumulators,
// copied there from shared memory with tcgen05.cp.
//
// Layouts (bytes, row-major):
//   weights  q  [E][R][C] E4M3, as the bf16 weights (C features contiguous, R the reduction)
//            sf [E][C/128][R/128][512] E8M0: one 512-byte chunk per (128 features, 128 k), byte
//               (f % 32) * 16 + (f / 32) * 4 + kb for feature f (0..127) of the block and
//               32-element k block kb (0..3) of the 128 k. tcgen05.cp 32x128b.warpx4 moves a
//               chunk to 4 TMEM columns: 16-byte line l goes to lane l of every lane quarter,
//               so row f's scales land in column f / 32, byte kb -- where the block-scaled MMA
//               reads the scale of operand row f for its k block kb (the byte is selected by
//               bits 30-31 of the scale address and the sf_id fields of the descriptor).
//   activations q [M][D] E4M3, sf [M][D/32] E8M0 (D = H for x, H' for h). A scale warp
//               copies each stage's 4 bytes per token row into the same chunk order (4-byte
//               cp.async, completion counted on the stage's barrier).
//
// Tiles as in grouped_ffn.cu ("swap AB": M = 128 features, N = the unit's tokens), with units of
// at most 224 tokens so that the accumulators and the scales of every pipeline stage share the
// 512 TMEM columns: pass 1 keeps gate and up at columns 0 and 224, pass 2 double-buffers two
// 224-column accumulators; columns 448-511 hold 16 scale columns per stage.
//
// Warp roles (352 threads): warp 0 TMA (weight tiles, weight scales by bulk copy, token
// tiles), warp 1 TMEM owner and MMA issuer (tcgen05.cp of the stage's scales, then the MMAs),
// warps 2-9 epilogue, warp 10 activation scales. Every wait is bounded as in grouped_ffn.cu.
#include <cuda_fp8.h>

#include <algorithm>
#include <atomic>
#include <cstdlib>

#include "gemm_common.cuh"

namespace moe {

// Host-side builder (tensor_maps.cu): a row-major byte matrix [rows][inner] (E4M3 elements)
// with a (box_inner x box_rows) box, 128-byte swizzle (box_inner must be 128): the K-major token
// tiles and MN-major weight tiles of the MXFP8 passes.
bool make_u8_tile_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows,
                      uint32_t box_inner, uint32_t box_rows);

namespace {

constexpr int kMxBK = 128;                  // k elements (= bytes) per stage
constexpr int kMxN = 224;                   // tokens per unit
constexpr int kMxATile = kBM * kMxBK;       // 16 KB: 128 features x 128 k, E4M3
constexpr int kMxChunk = 512;               // scale bytes of 128 rows x 128 k
constexpr uint32_t kMxAccCols = kMxN;
constexpr uint32_t kMxSfCol = 2 * kMxN;     // first scale column (448)
constexpr uint32_t kMxSfStageCols = 16;     // SFA (4 per weight) at +0/+4, SFB (8) at +8
constexpr int kMxBoxes = 4;                 // token boxes of 128, 64, 32, 16 rows
constexpr int kMxScaleWarp = 2 + kEpiThreads / 32;

template <bool kSwi>
struct MxCfg {
  static constexpr int kNumA = kSwi ? 2 : 1;
  static constexpr int kAccStages = kSwi ? 1 : 2;
  static constexpr int kBlock = kThreads + 32;
  static constexpr int kOffB = kNumA * kMxATile;
  static constexpr int kOffSfa = kOffB + kMxN * kMxBK;
  static constexpr int kOffSfb = kOffSfa + kNumA * kMxChunk;
  static constexpr int kStageBytes = (kOffSfb + 2 * kMxChunk + 1023) & ~1023;
  static constexpr int kStages = kSwi ? 3 : 4;
  static constexpr int kPipeBytes = kStages * kStageBytes;
  static constexpr int kOffOut = kPipeBytes;
  static constexpr int kOffCu = kOffOut + kEpiGroups * kOutBytes;
  static constexpr int kOffUnits = kOffCu + 4 * (MOE_MAX_FFN_EXPERTS + 1);
  static constexpr int kOffBars = (kOffUnits + 4 * (MOE_MAX_FFN_EXPERTS + 1) + 7) & ~7;
  static constexpr int kNumBars = 2 * kStages + 2 * 2 + 1;
  static constexpr int kOffMisc = kOffBars + 8 * kNumBars;
  static constexpr int kSmemBytes = kOffMisc + 128 + 1024;  // + alignment slack
  static_assert(kMxSfCol + kStages * kMxSfStageCols <= kTmemCols, "TMEM columns");
  static_assert(kAccStages * kMxAccCols <= kMxSfCol && (kSwi ? 2 : 1) * kMxAccCols <= kMxSfCol,
                "accumulators below the scale columns");
  static_assert(kOffSfa % 16 == 0 && kOffSfb % 16 == 0, "bulk copies and tcgen05.cp: 16 B");
};
static_assert(MxCfg<true>::kSmemBytes <= 232448, "shared memory budget (MXFP8 SwiGLU)");
static_assert(MxCfg<false>::kSmemBytes <= 232448, "shared memory budget (MXFP8 down)");

struct MxRowMaps {
  CUtensorMap m[kMxBoxes];
};

struct MxArgs {
  const int32_t* cu;      // [E+1]
  const uint8_t* act_sf;  // [M][k_dim / 32]
  const uint8_t* w_sf0;   // [E][n_feat / 128][k_dim / 128][512]
  const uint8_t* w_sf1;   // pass 1: W_up's scales; else null
  void* out;              // pass 1: h_q [M][n_feat] E4M3; pass 2: y [M][n_feat] bf16
  uint8_t* out_sf;        // pass 1: h_sf [M][n_feat / 32]
  int32_t* d_status;
  int64_t M;
  int32_t E;
  int32_t k_dim;
  int32_t n_feat;
  uint64_t budget_ns;
};

// ----------------------------------------------------------------------------- PTX

// Shared-memory descriptor without swizzle (K-major core matrices of 8 rows x 16 bytes, rows
// 16 bytes apart; sbo_bytes between 8-row groups): the source of tcgen05.cp.
__device__ __forceinline__ uint64_t smem_desc_plain(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // version; layout bits 61-63 = 0: no swizzle
  return d;
}

// 32 rows x 128 bits from shared memory to TMEM lanes 0-31 of `taddr`'s 4 columns, repeated in
// the other three lane quarters (32-63, 64-95, 96-127).
__device__ __forceinline__ void tmem_cp_32x128b_warpx4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Block-scaled MMA descriptor: A and B E4M3 (format 0), A MN-major, B K-major, E8M0 scales,
// M = 128, N given; sf_id selects the scale byte (k block) in both scale columns.
//   bits 4-5 B sf_id; 7-9 A format; 10-12 B format; 15 A major; 16 B major; 17-22 N >> 3;
//   bit 23 scale format (1 = E8M0); 24-28 M >> 4; 29-30 A sf_id; bit 31 K = 32 (0).
__device__ __forceinline__ uint32_t idesc_mxf8_m128_amn_bk(uint32_t n, uint32_t sf_id) {
  return (sf_id << 4) | (1u << 15) | ((n >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24) |
         (sf_id << 29);
}

// D[tmem] (+)= (A * SFA) (B * SFB), E4M3 x E4M3 with E8M0 block scales read from TMEM.
__device__ __forceinline__ void umma_mxf8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::
          "r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// 4-byte asynchronous global -> shared copy (generic proxy, like cp_async_16).
__device__ __forceinline__ void cp_async_4(uint32_t smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_dst), "l"(gmem_src)
               : "memory");
}

// Contiguous global -> shared bulk copy (16-byte aligned addresses, size a multiple of 16),
// completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_load_hint(void* smem_dst, const void* src, uint32_t bytes,
                                               uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(smem_dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// ----------------------------------------------------------------------------- MX arithmetic

// Scale exponent of a block with maximum magnitude amax: floor(log2 amax) - 8 (8 = the
// exponent of E4M3's largest power of two, 256), at least -127; amax = 0 (or subnormal) gives
// -127. Read off the float's exponent field, so exact.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  const int e = static_cast<int>((__float_as_uint(amax) >> 23) & 0xFFu) - 127 - 8;
  return e < -127 ? -127 : e;
}

// 2^-sexp for sexp in [-127, 119] (a normal float, so scaling by it is exact).
__device__ __forceinline__ float mx_inv_scale(int sexp) {
  return __uint_as_float(static_cast<uint32_t>(127 - sexp) << 23);
}

// Two floats to E4M3, round to nearest even, magnitudes above 448 saturating; a in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float a, float b) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3));
}

__device__ __forceinline__ uint8_t e4m3(float a) {
  return static_cast<uint8_t>(__nv_cvt_float_to_fp8(a, __NV_SATFINITE, __NV_E4M3));
}

// ----------------------------------------------------------------------------- GEMM kernel

template <bool kSwi>
__global__ void __launch_bounds__(MxCfg<kSwi>::kBlock, 1)
    grouped_ffn_mx_kernel(const __grid_constant__ CUtensorMap tmA0,
                          const __grid_constant__ CUtensorMap tmA1,
                          const __grid_constant__ MxRowMaps tmB, const MxArgs args) {
  using C = MxCfg<kSwi>;
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
  const int nfb = args.n_feat / kBM;
  const int KT = args.k_dim / kMxBK;
  const int sf_row = args.k_dim / 32;  // activation scale bytes per row

  // ------------------------------------------------------------------ prologue
  if (tid == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      // the TMA lane's arrive.expect_tx + one cp.async arrival per scale-warp lane
      mbar_init(&full[s], 1 + 32);
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
    if (kSwi) tma_prefetch_map(&tmA1);
    for (int i = 0; i < kMxBoxes; ++i) tma_prefetch_map(&tmB.m[i]);
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, kTmemCols);
    tmem_relinquish();
  }
  griddep_wait();
  griddep_launch_dependents();
  unit_starts<C::kBlock>(args.cu, args.M, E, nfb, kMxN, s_cu, s_ustart, s_scan);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *s_tmem;
  const int total_units = s_ustart[E];

  // ------------------------------------------------------------------ roles
  if (warp == kMxScaleWarp) {
    // Activation scales: per stage, token i = lane + 32 j (j < 8, i < the unit's rows) copies
    // its 4 scale bytes (k blocks 4 kt .. 4 kt + 3) with a 4-byte cp.async to chunk i / 128,
    // line i % 32, word (i / 32) % 4; each lane then arrives on the stage's full barrier when
    // its copies land, so the copies overlap like the TMA loads (as deep as the stage ring).
    // Rows past the unit (up to the 16-row rounding) keep whatever the slot held: their MMA
    // columns are never stored.
    int stage = 0;
    uint32_t phase = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < total_units && !stop; u += gridDim.x) {
      if (__shfl_sync(0xffffffffu, *s_abort, 0)) break;  // lane 0's view: a uniform exit
      const Unit U = decode_unit<kMxN>(u, s_ustart, s_cu, E);
      if (U.nrows <= 0) continue;
      const uint8_t* base = args.act_sf + static_cast<int64_t>(U.row0) * sf_row;
      for (int kt = 0; kt < KT; ++kt) {
        int ok = 1;
        if (lane == 0) ok = mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, args.budget_ns);
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          stop = true;
          break;
        }
        const uint32_t sfb = smem_u32(smem + stage * C::kStageBytes + C::kOffSfb);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int i = lane + 32 * j;
          if (i < U.nrows)
            cp_async_4(sfb + (i >> 7) * kMxChunk + (i & 31) * 16 + ((i >> 5) & 3) * 4,
                       base + static_cast<int64_t>(i) * sf_row + kt * 4);
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
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_keep = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0, issued_phase = 0;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const Unit U = decode_unit<kMxN>(u, s_ustart, s_cu, E);
        if (U.nrows <= 0) continue;
        const int n = (U.nrows + 15) & ~15;
        const uint32_t bytes = C::kNumA * (kMxATile + kMxChunk) + n * kMxBK;
        const uint64_t pol_w = U.ntc > 1 ? pol_keep : pol_stream;
        const int64_t sf_off = (static_cast<int64_t>(U.e) * nfb + U.fb) * KT * kMxChunk;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, s_abort, args.budget_ns)) break;
          uint8_t* st = smem + stage * C::kStageBytes;
          const int ky = U.e * args.k_dim + kt * kMxBK;
          mbar_arrive_expect_tx(&full[stage], bytes);
          tma_load_2d_hint(st, &tmA0, &full[stage], U.fb * kBM, ky, pol_w);
          bulk_load_hint(st + C::kOffSfa, args.w_sf0 + sf_off + kt * kMxChunk, kMxChunk,
                         &full[stage], pol_w);
          if (kSwi) {
            tma_load_2d_hint(st + kMxATile, &tmA1, &full[stage], U.fb * kBM, ky, pol_w);
            bulk_load_hint(st + C::kOffSfa + kMxChunk, args.w_sf1 + sf_off + kt * kMxChunk,
                           kMxChunk, &full[stage], pol_w);
          }
          int r = 0;
#pragma unroll
          for (int i = 0; i < kMxBoxes; ++i) {
            const int h = 128 >> i;
            if (n & h) {
              tma_load_2d_hint(st + C::kOffB + r * kMxBK, &tmB.m[i], &full[stage], kt * kMxBK,
                               U.row0 + r, pol_keep);
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
    // MMA issuer: per stage, the scales to TMEM (tcgen05.cp runs before the MMAs issued after
    // it by this thread), then 4 MMAs of K = 32 per accumulator. A stage's scale columns are
    // rewritten only after its slot was refilled, i.e. after the MMAs that read them completed.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int astage = 0;
      uint32_t aphase = 0;
      bool issued_any = false;
      for (int u = blockIdx.x; u < total_units && !*s_abort; u += gridDim.x) {
        const Unit U = decode_unit<kMxN>(u, s_ustart, s_cu, E);
        if (U.nrows <= 0) continue;
        const uint32_t n = static_cast<uint32_t>((U.nrows + 15) & ~15);
        if (!mbar_wait_bounded(&tempty[astage], aphase ^ 1u, s_abort, args.budget_ns)) break;
        tc_fence_after();
        const uint32_t d0 = tmem_base + astage * kMxAccCols;  // astage is 0 in pass 1
        const uint32_t d1 = d0 + kMxAccCols;
        bool ok = true;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_bounded(&full[stage], phase, s_abort, args.budget_ns)) {
            ok = false;
            break;
          }
          fence_proxy_async_smem();  // the activation scales arrived by cp.async (generic proxy)
          tc_fence_after();
          const uint32_t st = smem_u32(smem + stage * C::kStageBytes);
          const uint32_t sf = tmem_base + kMxSfCol + stage * kMxSfStageCols;
          tmem_cp_32x128b_warpx4(sf, smem_desc_plain(st + C::kOffSfa, 16, 128));
          if (kSwi) tmem_cp_32x128b_warpx4(sf + 4, smem_desc_plain(st + C::kOffSfa + kMxChunk, 16, 128));
          tmem_cp_32x128b_warpx4(sf + 8, smem_desc_plain(st + C::kOffSfb, 16, 128));
          if (n > 128)
            tmem_cp_32x128b_warpx4(sf + 12, smem_desc_plain(st + C::kOffSfb + kMxChunk, 16, 128));
#pragma unroll
          for (uint32_t kk = 0; kk < kMxBK / 32; ++kk) {
            const uint64_t bdesc = smem_desc_sw128(st + C::kOffB + kk * 32, 16, 1024);
            const uint32_t idesc = idesc_mxf8_m128_amn_bk(n, kk);
            const uint32_t acc = (kt != 0 || kk != 0) ? 1u : 0u;
            umma_mxf8(d0, smem_desc_sw128(st + kk * 4096, kMxATile, 1024), bdesc, idesc,
                      sf | (kk << 30), (sf + 8) | (kk << 30), acc);
            if (kSwi)
              umma_mxf8(d1, smem_desc_sw128(st + kMxATile + kk * 4096, kMxATile, 1024), bdesc,
                        idesc, (sf + 4) | (kk << 30), (sf + 8) | (kk << 30), acc);
          }
          issued_any = true;
          umma_commit(&empty[stage]);
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&tfull[astage]);
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
    // Epilogue: warps 2..9, two groups alternating 32-token chunks; warp w drains TMEM lanes
    // 32 (w % 4) .. +31, i.e. one 32-feature block, which is one MXFP8 block of h.
    const int q = warp & 3;
    const int grp = (warp - 2) >> 2;
    const int f_local = q * 32 + lane;
    const int gt = (tid - 64) & 127;
    const uint32_t bar_grp = 1 + grp, bar_all = 3;
    uint8_t* so_bytes = s_out + grp * kOutBytes;
    int astage = 0;
    uint32_t aphase = 0;
    for (int u = blockIdx.x; u < total_units; u += gridDim.x) {
      const Unit U = decode_unit<kMxN>(u, s_ustart, s_cu, E);
      if (U.nrows <= 0) continue;
      mbar_wait_bounded(&tfull[astage], aphase, s_abort, args.budget_ns);
      if (named_bar_red_or(bar_all, kEpiThreads, *s_abort != 0)) break;
      tc_fence_after();
      const uint32_t tbase =
          tmem_base + (static_cast<uint32_t>(q * 32) << 16) + astage * kMxAccCols;
      const int f0 = U.fb * kBM;
      bool released = false;
      // release the accumulator once this warp's last chunk of the unit is in registers
      auto release_if_last = [&](int c) {
        if (c + kEpiGroups * kOutChunk >= U.nrows) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&tempty[astage]);
          released = true;
        }
      };
      for (int c = grp * kOutChunk; c < U.nrows; c += kEpiGroups * kOutChunk) {
        __syncwarp();
        uint32_t r0[32];
        tmem_ld_32x32b_x32(tbase + c, r0);
        if (kSwi) {
          uint32_t r1[32];
          tmem_ld_32x32b_x32(tbase + kMxAccCols + c, r1);
          tmem_ld_wait();
          release_if_last(c);
          uint32_t my_sf = 127;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const float g = __uint_as_float(r0[j]);
            const float hval = __fdividef(g, 1.0f + __expf(-g)) * __uint_as_float(r1[j]);
            // the block of token c + j: features f0 + 32 q .. +31, one per lane
            const uint32_t amax = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(hval)));
            const int sexp = mx_scale_exp(__uint_as_float(amax));
            so_bytes[j * kBM + f_local] = e4m3(hval * mx_inv_scale(sexp));
            if (lane == j) my_sf = static_cast<uint32_t>(sexp + 127);
          }
          named_bar_sync(bar_grp, 128);
          // [32 tokens][128 features] E4M3 -> 32 rows of h_q, 8 x 16 bytes each
#pragma unroll
          for (int p = 0; p < (kOutChunk * kBM / 16) / 128; ++p) {
            const int vid = gt + 128 * p;
            const int j = vid >> 3, c16 = vid & 7;
            if (c + j < U.nrows) {
              const uint4 val = *reinterpret_cast<const uint4*>(so_bytes + j * kBM + c16 * 16);
              uint8_t* dst = static_cast<uint8_t*>(args.out) +
                             static_cast<int64_t>(U.row0 + c + j) * args.n_feat + f0 + c16 * 16;
              *reinterpret_cast<uint4*>(dst) = val;
            }
          }
          if (c + lane < U.nrows)
            args.out_sf[static_cast<int64_t>(U.row0 + c + lane) * (args.n_feat / 32) + f0 / 32 +
                        q] = static_cast<uint8_t>(my_sf);
          named_bar_sync(bar_grp, 128);
        } else {
          tmem_ld_wait();
          release_if_last(c);
          __nv_bfloat16* so = reinterpret_cast<__nv_bfloat16*>(so_bytes);
#pragma unroll
          for (int j = 0; j < 32; ++j) so[j * kBM + f_local] = __float2bfloat16_rn(__uint_as_float(r0[j]));
          named_bar_sync(bar_grp, 128);
#pragma unroll
          for (int p = 0; p < (kOutChunk * kBM * 2 / 16) / 128; ++p) {
            const int vid = gt + 128 * p;
            const int j = vid >> 4, c16 = vid & 15;
            if (c + j < U.nrows) {
              const uint4 val = *reinterpret_cast<const uint4*>(so_bytes + j * (kBM * 2) + c16 * 16);
              __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(args.out) +
                                   static_cast<int64_t>(U.row0 + c + j) * args.n_feat + f0 +
                                   c16 * 8;
              *reinterpret_cast<uint4*>(dst) = val;
            }
          }
          named_bar_sync(bar_grp, 128);
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

// ----------------------------------------------------------------------------- quantisation

// Weights [E][R][C] bf16 -> E4M3 [E][R][C] and chunked E8M0 scales. One thread per (expert,
// 32-row block, column): the 32 elements of a block run down a column, so a warp reads and
// writes 32 neighbouring columns of each row.
__global__ void __launch_bounds__(256) mx_quantize_weight_kernel(const __nv_bfloat16* __restrict__ w,
                                                                 int64_t E, int64_t R, int64_t C,
                                                                 uint8_t* __restrict__ q,
                                                                 uint8_t* __restrict__ sf) {
  const int64_t nb = R / 32;
  const int64_t total = E * nb * C;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += stride) {
    const int64_t c = i % C;
    const int64_t rb = (i / C) % nb;
    const int64_t e = i / (C * nb);
    const int64_t off = (e * R + rb * 32) * C + c;
    float v[32];
    float amax = 0.0f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      v[r] = __bfloat162float(w[off + r * C]);
      amax = fmaxf(amax, fabsf(v[r]));
    }
    const int sexp = mx_scale_exp(amax);
    const float inv = mx_inv_scale(sexp);
#pragma unroll
    for (int r = 0; r < 32; ++r) q[off + r * C] = e4m3(v[r] * inv);
    const int64_t fb = c / 128, fl = c % 128, kt = rb / 4, kb = rb % 4;
    sf[((e * (C / 128) + fb) * (R / 128) + kt) * kMxChunk + (fl % 32) * 16 + (fl / 32) * 4 + kb] =
        static_cast<uint8_t>(sexp + 127);
  }
}

// Token rows x [S][H] bf16 -> their K expert-grouped copies in MXFP8 (x_q [M][H] E4M3, x_sf
// [M][H/32]): each token is quantised once and written to the rows row_id_map[t][k] (-1: not
// routed). One warp per (token, 256-element slice); lane l holds 8 elements, four lanes one
// 32-element block.
__global__ void __launch_bounds__(256) mx_permute_quantize_kernel(
    const uint4* __restrict__ x, int64_t S, int64_t H, int32_t K,
    const int32_t* __restrict__ row_id_map, uint8_t* __restrict__ xq, uint8_t* __restrict__ xsf) {
  const int lane = threadIdx.x & 31;
  griddep_wait();  // row_id_map comes from the metadata kernel
  griddep_launch_dependents();
  const int64_t M = S * K;
  const int64_t nvec = H / 8;
  const int64_t nslice = (nvec + 31) / 32;
  const int64_t items = S * nslice;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5);
       it < items; it += nwarps) {
    const int64_t t = it / nslice;
    const int64_t v = (it - t * nslice) * 32 + lane;
    const bool active = v < nvec;  // H % 32 == 0: whole four-lane groups are active or not
    float f[8];
    float amax = 0.0f;
    if (active) {
      const uint4 raw = __ldg(x + t * nvec + v);
      const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f[2 * j] = __uint_as_float(wds[j] << 16);
        f[2 * j + 1] = __uint_as_float(wds[j] & 0xFFFF0000u);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) f[j] = 0.0f;
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const int sexp = mx_scale_exp(amax);
    const float inv = mx_inv_scale(sexp);
    uint2 packed;
    packed.x = e4m3x2(f[0] * inv, f[1] * inv) | (e4m3x2(f[2] * inv, f[3] * inv) << 16);
    packed.y = e4m3x2(f[4] * inv, f[5] * inv) | (e4m3x2(f[6] * inv, f[7] * inv) << 16);
    const int32_t my_row = (lane < K) ? row_id_map[t * K + lane] : -1;
    for (int k = 0; k < K; ++k) {
      const int32_t row = (K <= 32) ? __shfl_sync(0xffffffffu, my_row, k) : row_id_map[t * K + k];
      if (row < 0 || row >= M || !active) continue;
      *reinterpret_cast<uint2*>(xq + static_cast<int64_t>(row) * H + v * 8) = packed;
      if ((lane & 3) == 0) xsf[static_cast<int64_t>(row) * (H / 32) + v / 4] = static_cast<uint8_t>(sexp + 127);
    }
  }
}

// The kernel's dynamic shared-memory opt-in, once per device.
template <bool kSwi>
bool ensure_mx_smem_attr() {
  static ContextCache done;
  return set_smem_optin(reinterpret_cast<const void*>(grouped_ffn_mx_kernel<kSwi>),
                        MxCfg<kSwi>::kSmemBytes, done);
}

bool make_mx_row_maps(MxRowMaps* maps, const void* ptr, uint64_t inner, uint64_t rows) {
  for (int i = 0; i < kMxBoxes; ++i)
    if (!make_u8_tile_map(&maps->m[i], ptr, inner, rows, kMxBK, static_cast<uint32_t>(128 >> i)))
      return false;
  return true;
}

}  // namespace

moe_status launch_mx_quantize_weights(const void* w, int32_t E, int64_t R, int64_t C, void* q,
                                      void* sf, cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(E) * (R / 32) * C;
  if (total == 0) return MOE_OK;
  const int64_t blocks = std::min<int64_t>(ceil_div(total, 256), static_cast<int64_t>(num_sms()) * 8);
  mx_quantize_weight_kernel<<<static_cast<unsigned>(blocks), 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(w), E, R, C, static_cast<uint8_t*>(q),
      static_cast<uint8_t*>(sf));
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_mx_permute_quantize(const void* x, int64_t S, int64_t H, int32_t K,
                                      const int32_t* row_id_map, void* xq, void* xsf,
                                      cudaStream_t stream) {
  const int64_t items = S * ceil_div(H / 8, 32);
  if (items == 0) return MOE_OK;
  const int64_t blocks = std::min<int64_t>(ceil_div(items, 8), static_cast<int64_t>(num_sms()) * 8);
  const cudaError_t err = launch_dependent(
      mx_permute_quantize_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
      static_cast<const uint4*>(x), S, H, K, row_id_map, static_cast<uint8_t*>(xq),
      static_cast<uint8_t*>(xsf));
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status launch_mx_ffn_pass(bool dual, const void* act_q, const void* act_sf, const void* w0_q,
                              const void* w0_sf, const void* w1_q, const void* w1_sf,
                              const int32_t* cu_seqlens, int64_t M, int64_t H, int64_t Hp,
                              int32_t E, void* out, void* out_sf, int32_t* d_status,
                              cudaStream_t stream) {
  const int64_t k_dim = dual ? H : Hp;
  const int64_t n_feat = dual ? Hp : H;
  CUtensorMap tmA0, tmA1;
  MxRowMaps tmB;
  if (!make_u8_tile_map(&tmA0, w0_q, n_feat, static_cast<uint64_t>(E) * k_dim, kBM, kMxBK) ||
      !make_u8_tile_map(&tmA1, dual ? w1_q : w0_q, n_feat, static_cast<uint64_t>(E) * k_dim, kBM,
                        kMxBK) ||
      !make_mx_row_maps(&tmB, act_q, k_dim, M))
    return MOE_ERR_CUDA;
  MxArgs args;
  args.cu = cu_seqlens;
  args.act_sf = static_cast<const uint8_t*>(act_sf);
  args.w_sf0 = static_cast<const uint8_t*>(w0_sf);
  args.w_sf1 = dual ? static_cast<const uint8_t*>(w1_sf) : nullptr;
  args.out = out;
  args.out_sf = dual ? static_cast<uint8_t*>(out_sf) : nullptr;
  args.d_status = d_status;
  args.M = M;
  args.E = E;
  args.k_dim = static_cast<int32_t>(k_dim);
  args.n_feat = static_cast<int32_t>(n_feat);
  args.budget_ns = wait_budget_ns();
  const int sms = num_sms();
  cudaError_t err;
  if (dual) {
    if (!ensure_mx_smem_attr<true>()) return MOE_ERR_CUDA;
    err = launch_dependent(grouped_ffn_mx_kernel<true>, dim3(sms), dim3(MxCfg<true>::kBlock),
                           MxCfg<true>::kSmemBytes, stream, tmA0, tmA1, tmB, args);
  } else {
    if (!ensure_mx_smem_attr<false>()) return MOE_ERR_CUDA;
    err = launch_dependent(grouped_ffn_mx_kernel<false>, dim3(sms), dim3(MxCfg<false>::kBlock),
                           MxCfg<false>::kSmemBytes, stream, tmA0, tmA1, tmB, args);
  }
  return err == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

}  // namespace moe
