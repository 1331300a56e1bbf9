// Plain C++ CPU oracle of the MoE layer's hot path: the forward (permutation, maxvio, grouped
// SwiGLU FFN, weighted combine), the backward of the two data-movement steps, and the MXFP8
// quantisation.
//
// TEST INFRASTRUCTURE ONLY: loaded by tests/ (through oracle/ref.py) to cross-check the
// numpy oracle; the product path never links or loads it, and it shares no code, header or
// helper with grouped_ffn_moe_b200/csrc. Everything is scalar loops in the order the pages
// state, in IEEE double with one final rounding per stored bf16 value. Compile without
// floating-point contraction (-ffp-contract=off) so that every product and sum is rounded
// on its own, as written.
//
// Pages followed:
//  * "Distributed expert parallelism", "The dispatch-compute-combine lifecycle" and "Token
//    permutation and metadata": a token's K copies are sorted by destination expert (expert
//    0's rows first), the metadata records where each copy went, and after the experts ran
//    each copy is scaled by its route weight and the token's K results are summed
//    ("Duplicate route accumulation": added, never overwritten).
//  * "Mixture of Kittens" digest, Step 1 (The Math): expert i computes
//    Down_i(SwiGLU(Up_i x, Gate_i x)), read as silu(x Wg) * (x Wu), silu(z) = z / (1 + e^-z).
//  * MoonEP README, "Integration" / "Weight buffer": one weight tensor per projection with
//    experts addressed by row index, rows of expert e at [cu[e], cu[e+1]).
//  * MoonEP README, "Performance": maxvio = max_e(T_e / T_bar) - 1, T_bar = S*K/E.
//
// Readings shared with the numpy oracle: rows of one expert keep flat-slot order
// f = t*K + k; cu has E+1 entries with cu[0] = 0; W_down is [E, H', H]; bf16 values are
// uint16 bit patterns rounded to nearest, ties to even.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

double bf16_to_double(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return static_cast<double>(f);
}

// Round a double once to bf16 (1 sign, 8 exponent, 7 fraction bits; fp32's exponent
// range), nearest with ties to even, by integer arithmetic on the double's fields.
uint16_t double_to_bf16(double v) {
  uint64_t d;
  std::memcpy(&d, &v, sizeof d);
  const uint16_t sign = static_cast<uint16_t>((d >> 63) << 15);
  const int exp = static_cast<int>((d >> 52) & 0x7FF);
  const uint64_t frac = d & ((uint64_t{1} << 52) - 1);
  if (exp == 0x7FF) return frac ? static_cast<uint16_t>(sign | 0x7FC0) : static_cast<uint16_t>(sign | 0x7F80);
  if (exp == 0 && frac == 0) return sign;
  // value = mant * 2^(e2 - 52) with mant the 53-bit significand (implicit bit made explicit)
  const uint64_t mant = exp ? (frac | (uint64_t{1} << 52)) : frac;
  const int e2 = (exp ? exp : 1) - 1023;
  // bf16 quantum at this magnitude: 2^(e_lead - 7) for normals (e_lead = exponent of the
  // leading bit), never finer than the subnormal quantum 2^-133
  int lead = 52;
  while (lead > 0 && !((mant >> lead) & 1)) --lead;
  const int e_lead = e2 - 52 + lead;
  int quantum = e_lead - 7;
  if (quantum < -133) quantum = -133;
  // q = mant * 2^(e2 - 52 - quantum), rounded to nearest even
  const int shift = quantum - (e2 - 52);  // > 0: bits to drop
  uint64_t q;
  if (shift <= 0) {
    q = mant << (-shift);  // exact (cannot happen for doubles below 2^128 with 8 kept bits)
  } else if (shift >= 64) {
    q = 0;
  } else {
    q = mant >> shift;
    const uint64_t rem = mant & ((uint64_t{1} << shift) - 1);
    const uint64_t half = uint64_t{1} << (shift - 1);
    if (rem > half || (rem == half && (q & 1))) ++q;
  }
  // value = q * 2^quantum; encode (q may have grown to 2^8 by the rounding carry)
  if (q == 0) return sign;
  int e = quantum;
  while (q >= 256) {  // renormalise to 8 significant bits (only after a carry: q == 256)
    q >>= 1;
    ++e;
  }
  if (q < 128) {  // subnormal: e == -133, stored fraction = q
    return static_cast<uint16_t>(sign | q);
  }
  // normal: value = (q / 128) * 2^(e + 7), biased exponent e + 7 + 127
  const int be = e + 7 + 127;
  if (be >= 255) return static_cast<uint16_t>(sign | 0x7F80);  // overflow to infinity
  return static_cast<uint16_t>(sign | (be << 7) | (q & 127));
}

double silu(double z) { return z / (1.0 + std::exp(-z)); }

}  // namespace

extern "C" {

// bf16 rounding of n doubles (exposed for the tests).
void ref_round_bf16(const double* v, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(v[i]);
}

// Counting sort of the flat slots f = t*K + k by expert id: counts, exclusive scan, then one
// pass in increasing f that hands each slot the next row of its expert. Returns 0, or -1
// (and writes nothing) when an id lies outside [0, E).
int ref_permute(const int32_t* topk_ids, int64_t S, int32_t K, int32_t E, int32_t* counts,
                int32_t* cu, int32_t* row_id_map, int32_t* perm_src) {
  const int64_t F = S * K;
  for (int64_t f = 0; f < F; ++f)
    if (topk_ids[f] < 0 || topk_ids[f] >= E) return -1;
  for (int32_t e = 0; e < E; ++e) counts[e] = 0;
  for (int64_t f = 0; f < F; ++f) counts[topk_ids[f]] += 1;
  cu[0] = 0;
  for (int32_t e = 0; e < E; ++e) cu[e + 1] = cu[e] + counts[e];
  std::vector<int32_t> next(cu, cu + E);
  for (int64_t f = 0; f < F; ++f) {
    const int32_t row = next[topk_ids[f]]++;
    row_id_map[f] = row;
    perm_src[row] = static_cast<int32_t>(f);
  }
  return 0;
}

// x_perm[row] = x[perm_src[row] / K], a copy of the token's bf16 row.
void ref_permute_rows(const uint16_t* x, const int32_t* perm_src, int64_t M, int32_t K,
                      int64_t H, uint16_t* x_perm) {
  for (int64_t r = 0; r < M; ++r) {
    const int64_t t = perm_src[r] / K;
    for (int64_t j = 0; j < H; ++j) x_perm[r * H + j] = x[t * H + j];
  }
}

// maxvio = (max_e counts[e]) * E / (S * K) - 1 in double: two exact products, one division,
// one subtraction. Writes the maximum count too.
double ref_maxvio(const int32_t* counts, int32_t E, int64_t S, int32_t K, int32_t* max_count) {
  int32_t mc = 0;
  for (int32_t e = 0; e < E; ++e)
    if (counts[e] > mc) mc = counts[e];
  *max_count = mc;
  const double num = static_cast<double>(mc) * static_cast<double>(E);
  const double den = static_cast<double>(S) * static_cast<double>(K);
  return num / den - 1.0;
}

// Expert FFN over expert-contiguous rows: for row r of expert e and output feature j,
//   g = sum_i x[r,i] Wg[e,i,j],  u = sum_i x[r,i] Wu[e,i,j]   (i ascending, double)
//   h[r,j] = bf16(silu(g) * u)
// then y[r,n] = bf16(sum_j h[r,j] Wd[e,j,n]) (j ascending). w_gate, w_up [E,H,Hp] and
// w_down [E,Hp,H], bf16 bits.
void ref_grouped_ffn(const uint16_t* x_perm, const uint16_t* w_gate, const uint16_t* w_up,
                     const uint16_t* w_down, const int32_t* cu, int32_t E, int64_t H,
                     int64_t Hp, uint16_t* h, uint16_t* y) {
  std::vector<double> xr(H), hr(Hp);
  for (int32_t e = 0; e < E; ++e) {
    const uint16_t* wg = w_gate + static_cast<int64_t>(e) * H * Hp;
    const uint16_t* wu = w_up + static_cast<int64_t>(e) * H * Hp;
    const uint16_t* wd = w_down + static_cast<int64_t>(e) * Hp * H;
    for (int64_t r = cu[e]; r < cu[e + 1]; ++r) {
      for (int64_t i = 0; i < H; ++i) xr[i] = bf16_to_double(x_perm[r * H + i]);
      for (int64_t j = 0; j < Hp; ++j) {
        double g = 0.0, u = 0.0;
        for (int64_t i = 0; i < H; ++i) {
          g += xr[i] * bf16_to_double(wg[i * Hp + j]);
          u += xr[i] * bf16_to_double(wu[i * Hp + j]);
        }
        h[r * Hp + j] = double_to_bf16(silu(g) * u);
        hr[j] = bf16_to_double(h[r * Hp + j]);
      }
      for (int64_t n = 0; n < H; ++n) {
        double acc = 0.0;
        for (int64_t j = 0; j < Hp; ++j) acc += hr[j] * bf16_to_double(wd[j * H + n]);
        y[r * H + n] = double_to_bf16(acc);
      }
    }
  }
}

// out[t] = bf16(sum over k ascending of w[t,k] * y[row_id_map[t*K+k]]) in double; the route
// weight is fp32, widened exactly.
void ref_combine(const uint16_t* y, const int32_t* row_id_map, const float* route_w, int64_t S,
                 int32_t K, int64_t H, uint16_t* out) {
  for (int64_t t = 0; t < S; ++t) {
    for (int64_t n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int32_t k = 0; k < K; ++k) {
        const int64_t r = row_id_map[t * K + k];
        acc += static_cast<double>(route_w[t * K + k]) * bf16_to_double(y[r * H + n]);
      }
      out[t * H + n] = double_to_bf16(acc);
    }
  }
}

// ---------------------------------------------------------------------------- backward
// MoonEP README, "API walkthrough": combine bwd re-dispatches the output gradient along the
// saved plan, dispatch bwd sums each token's K row gradients. With out[t] = sum_k w[t,k] *
// y[r(t,k)]:
//   grad_y[r(t,k)] = bf16(w[t,k] * grad_out[t])      grad_w[t,k] = <grad_out[t], y[r(t,k)]>
//   grad_x[t]      = bf16(sum over k ascending of grad_x_perm[r(t,k)])

// grad_w in double, summed over n ascending; rows no slot maps to are left as they are.
void ref_combine_backward(const uint16_t* grad_out, const uint16_t* y,
                          const int32_t* row_id_map, const float* route_w, int64_t S,
                          int32_t K, int64_t H, uint16_t* grad_y, double* grad_w) {
  for (int64_t t = 0; t < S; ++t) {
    for (int32_t k = 0; k < K; ++k) {
      const int64_t r = row_id_map[t * K + k];
      const double w = static_cast<double>(route_w[t * K + k]);
      double dot = 0.0;
      for (int64_t n = 0; n < H; ++n) {
        const double g = bf16_to_double(grad_out[t * H + n]);
        grad_y[r * H + n] = double_to_bf16(w * g);  // exact product, one rounding
        dot += g * bf16_to_double(y[r * H + n]);
      }
      grad_w[t * K + k] = dot;
    }
  }
}

void ref_permute_backward(const uint16_t* grad_x_perm, const int32_t* row_id_map, int64_t S,
                          int32_t K, int64_t H, uint16_t* grad_x) {
  for (int64_t t = 0; t < S; ++t)
    for (int64_t n = 0; n < H; ++n) {
      double acc = 0.0;
      for (int32_t k = 0; k < K; ++k)
        acc += bf16_to_double(grad_x_perm[static_cast<int64_t>(row_id_map[t * K + k]) * H + n]);
      grad_x[t * H + n] = double_to_bf16(acc);
    }
}

// ---------------------------------------------------------------------------- MXFP8
// OCP Microscaling (MX) v1.0, MXFP8: blocks of 32 consecutive elements share a power-of-two
// scale 2^s stored as E8M0, s = floor(log2(block max |v|)) - 8 (8 = the exponent of E4M3's
// largest power of two), s = -127 for an all-zero block; elements are v / 2^s rounded to
// E4M3 (nearest, ties to even; normal exponents -6..8 with 3 fraction bits, subnormal step
// 2^-9), saturating at 448.

// E4M3 rounding of one double, through frexp: a = m * 2^e, m in [0.5, 1), so the leading
// bit's exponent is e - 1 and the E4M3 quantum there is 2^(e - 1 - 3) (at least 2^-9).
static double e4m3_of(double v) {
  const double a = std::fabs(v);
  if (a == 0.0) return v;
  int e;
  std::frexp(a, &e);
  int quantum = e - 1 - 3;
  if (quantum < -9) quantum = -9;
  double q = std::ldexp(std::nearbyint(std::ldexp(a, -quantum)), quantum);
  if (q > 448.0) q = 448.0;
  return std::copysign(q, v);
}

void ref_e4m3_round(const double* v, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = e4m3_of(v[i]);
}

// Rows of length L (a multiple of 32) quantised along the row: q[r, j] (E4M3 values as
// doubles) and sexp[r, j / 32].
void ref_mx_quantize_rows(const double* v, int64_t rows, int64_t L, double* q, int32_t* sexp) {
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t b = 0; b < L / 32; ++b) {
      const double* blk = v + r * L + b * 32;
      double amax = 0.0;
      for (int i = 0; i < 32; ++i) amax = std::fmax(amax, std::fabs(blk[i]));
      int s = -127;
      if (amax > 0.0) {
        int e;
        std::frexp(amax, &e);
        s = (e - 1) - 8;
        if (s < -127) s = -127;
        if (s > 127) s = 127;
      }
      sexp[r * (L / 32) + b] = s;
      for (int i = 0; i < 32; ++i) q[r * L + b * 32 + i] = e4m3_of(std::ldexp(blk[i], -s));
    }
}

// ---------------------------------------------------------------------------- expert backward
// Chain rule of one expert's forward ("Mixture of Kittens" digest, Step 1, The Math) at the
// saved bf16 pre-activations g = bf16(x Wg), u = bf16(x Wu), with s = 1 / (1 + e^-g):
//   grad_h = grad_y Wd^T (not stored)
//   d_u = bf16(grad_h * g * s)      d_g = bf16(grad_h * u * s * (1 + g (1 - s)))
//   grad_x = bf16(d_g Wg^T + d_u Wu^T)                     (one rounding)
//   dWg = x^T d_g, dWu = x^T d_u, dWd = h^T grad_y          (double sums over the n rows)
// x [n,H], g, u, h [n,Hp], grad_y [n,H]; Wg, Wu [H,Hp], Wd [Hp,H]; bf16 bits.
void ref_expert_backward(const uint16_t* x, const uint16_t* g, const uint16_t* u,
                         const uint16_t* h, const uint16_t* grad_y, const uint16_t* wg,
                         const uint16_t* wu, const uint16_t* wd, int64_t n, int64_t H,
                         int64_t Hp, uint16_t* d_g, uint16_t* d_u, uint16_t* grad_x,
                         double* dwg, double* dwu, double* dwd) {
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t j = 0; j < Hp; ++j) {
      double gh = 0.0;
      for (int64_t m = 0; m < H; ++m)
        gh += bf16_to_double(grad_y[r * H + m]) * bf16_to_double(wd[j * H + m]);
      const double gv = bf16_to_double(g[r * Hp + j]);
      const double uv = bf16_to_double(u[r * Hp + j]);
      const double sg = 1.0 / (1.0 + std::exp(-gv));
      d_u[r * Hp + j] = double_to_bf16(gh * (gv * sg));
      d_g[r * Hp + j] = double_to_bf16(gh * uv * (sg * (1.0 + gv * (1.0 - sg))));
    }
    for (int64_t i = 0; i < H; ++i) {
      double acc = 0.0;
      for (int64_t j = 0; j < Hp; ++j)
        acc += bf16_to_double(d_g[r * Hp + j]) * bf16_to_double(wg[i * Hp + j]);
      for (int64_t j = 0; j < Hp; ++j)
        acc += bf16_to_double(d_u[r * Hp + j]) * bf16_to_double(wu[i * Hp + j]);
      grad_x[r * H + i] = double_to_bf16(acc);
    }
  }
  for (int64_t i = 0; i < H; ++i)
    for (int64_t j = 0; j < Hp; ++j) {
      double a = 0.0, b = 0.0;
      for (int64_t r = 0; r < n; ++r) {
        a += bf16_to_double(x[r * H + i]) * bf16_to_double(d_g[r * Hp + j]);
        b += bf16_to_double(x[r * H + i]) * bf16_to_double(d_u[r * Hp + j]);
      }
      dwg[i * Hp + j] = a;
      dwu[i * Hp + j] = b;
    }
  for (int64_t j = 0; j < Hp; ++j)
    for (int64_t m = 0; m < H; ++m) {
      double c = 0.0;
      for (int64_t r = 0; r < n; ++r)
        c += bf16_to_double(h[r * Hp + j]) * bf16_to_double(grad_y[r * H + m]);
      dwd[j * H + m] = c;
    }
}

// ---------------------------------------------------------------------------- MXFP8 expert
// One expert in MXFP8 ("Mixture of Kittens" digest, Step 8, MXFP8 mode; OCP MX v1.0): x
// quantised along H, the weights along their reduction dimension (Wg, Wu [H,Hp] along H; Wd
// [Hp,H] along Hp), h = silu(g) u from the dequantised operands quantised along Hp, and
// y = bf16(deq(h) deq(Wd)); products exact, sums in double. Outputs the h codes as E4M3
// values (doubles), their exponents, and y bits.
void ref_expert_ffn_mxfp8(const uint16_t* x, const uint16_t* wg, const uint16_t* wu,
                          const uint16_t* wd, int64_t n, int64_t H, int64_t Hp, double* hq,
                          int32_t* hs, uint16_t* y) {
  // weights: quantise column by column along the reduction (row) index
  auto quant_cols = [&](const uint16_t* w, int64_t R, int64_t C, std::vector<double>& deq) {
    deq.assign(static_cast<size_t>(R * C), 0.0);
    std::vector<double> col(R), q(R);
    std::vector<int32_t> sx(R / 32);
    for (int64_t c = 0; c < C; ++c) {
      for (int64_t r = 0; r < R; ++r) col[r] = bf16_to_double(w[r * C + c]);
      ref_mx_quantize_rows(col.data(), 1, R, q.data(), sx.data());
      for (int64_t r = 0; r < R; ++r) deq[r * C + c] = std::ldexp(q[r], sx[r / 32]);
    }
  };
  std::vector<double> g_deq, u_deq, d_deq;
  quant_cols(wg, H, Hp, g_deq);
  quant_cols(wu, H, Hp, u_deq);
  quant_cols(wd, Hp, H, d_deq);
  std::vector<double> xr(H), xq(H), hv(Hp);
  std::vector<int32_t> xs(H / 32);
  for (int64_t r = 0; r < n; ++r) {
    for (int64_t i = 0; i < H; ++i) xr[i] = bf16_to_double(x[r * H + i]);
    ref_mx_quantize_rows(xr.data(), 1, H, xq.data(), xs.data());
    for (int64_t i = 0; i < H; ++i) xr[i] = std::ldexp(xq[i], xs[i / 32]);
    for (int64_t j = 0; j < Hp; ++j) {
      double gg = 0.0, uu = 0.0;
      for (int64_t i = 0; i < H; ++i) {
        gg += xr[i] * g_deq[i * Hp + j];
        uu += xr[i] * u_deq[i * Hp + j];
      }
      hv[j] = silu(gg) * uu;
    }
    ref_mx_quantize_rows(hv.data(), 1, Hp, hq + r * Hp, hs + r * (Hp / 32));
    for (int64_t m = 0; m < H; ++m) {
      double acc = 0.0;
      for (int64_t j = 0; j < Hp; ++j)
        acc += std::ldexp(hq[r * Hp + j], hs[r * (Hp / 32) + j / 32]) * d_deq[j * H + m];
      y[r * H + m] = double_to_bf16(acc);
    }
  }
}

}  // extern "C"
