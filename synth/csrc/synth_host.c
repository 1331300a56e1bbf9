/*
 * Seeded synthetic inputs for the MoE layer: host implementation.
 *
 * This module holds none of the layer's arithmetic. It only draws numbers:
 *   - SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
 *     generators", OOPSLA 2014) used as a counter-based stream: the i-th value of
 *     stream (seed, tag) is the (i+1)-th output of SplitMix64 started at
 *     key(seed, tag) = mix64(seed * GAMMA + tag);
 *   - uniforms u = ((r >> 12) + 0.5) * 2^-52, strictly inside (0, 1);
 *   - normals by the cosine branch of Box-Muller, one pair of uniforms per value,
 *     evaluated in double, scaled, rounded to float (RN) and then to bf16 (RNE);
 *   - top-K expert routing by Efraimidis-Spirakis keys log(u)/p_e ("Weighted random
 *     sampling with a reservoir", IPL 2006) with an optional per-expert cap.
 *
 * The CUDA twin (synth_gpu.cu) evaluates the same formulas; both are compiled
 * without floating-point contraction so that the same operations are performed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL
#define TWO_PI 6.283185307179586

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t tag) { return mix64(seed * GAMMA + tag); }

static inline uint64_t draw64(uint64_t key, uint64_t i) { return mix64(key + (i + 1ULL) * GAMMA); }

static inline double unit_open(uint64_t r) { return ((double)(r >> 12) + 0.5) * 0x1p-52; }

static inline double normal_at(uint64_t key, uint64_t i) {
  double u1 = unit_open(draw64(key, 2ULL * i));
  double u2 = unit_open(draw64(key, 2ULL * i + 1ULL));
  return sqrt(-2.0 * log(u1)) * cos(TWO_PI * u2);
}

static inline uint16_t float_to_bf16_rne(float f) {
  uint32_t b;
  memcpy(&b, &f, 4);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return (uint16_t)(b >> 16);
}

uint64_t synth_draw64(uint64_t seed, uint64_t tag, uint64_t i) { return draw64(stream_key(seed, tag), i); }

void synth_uniform(uint64_t seed, uint64_t tag, uint64_t offset, int64_t n, double* out) {
  const uint64_t key = stream_key(seed, tag);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = unit_open(draw64(key, offset + (uint64_t)i));
}

void synth_normal_f64(uint64_t seed, uint64_t tag, uint64_t offset, int64_t n, double* out) {
  const uint64_t key = stream_key(seed, tag);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = normal_at(key, offset + (uint64_t)i);
}

void synth_normal_bf16(uint64_t seed, uint64_t tag, uint64_t offset, int64_t n, double scale,
                       uint16_t* out) {
  const uint64_t key = stream_key(seed, tag);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    double v = normal_at(key, offset + (uint64_t)i) * scale;
    out[i] = float_to_bf16_rne((float)v);
  }
}

/*
 * Top-K routing without replacement. For token t (in order 0..S-1) every expert e
 * whose running count is below `cap` (cap <= 0: no cap) gets the key
 * log(u[t,e]) / p_e with p_e = 1 except p_hot = w_hot; the K largest keys are the
 * token's experts, written in descending key order. If fewer than K experts are
 * below the cap, the cap is ignored for that token. Returns the hot expert's count.
 */
int64_t synth_route(uint64_t seed, uint64_t tag, int64_t S, int32_t K, int32_t E, int32_t hot_e,
                    double w_hot, int64_t cap, int32_t* ids) {
  const uint64_t key = stream_key(seed, tag);
  int64_t* count = (int64_t*)calloc((size_t)E, sizeof(int64_t));
  double* keys = (double*)malloc((size_t)E * sizeof(double));
  if (!count || !keys) {
    free(count);
    free(keys);
    return -1;
  }
  for (int64_t t = 0; t < S; ++t) {
    int32_t avail = 0;
    for (int32_t e = 0; e < E; ++e) {
      double u = unit_open(draw64(key, (uint64_t)t * (uint64_t)E + (uint64_t)e));
      double k = log(u);
      if (e == hot_e) k = k / w_hot;
      keys[e] = k;
      if (cap <= 0 || count[e] < cap) ++avail;
    }
    const int use_cap = (cap > 0 && avail >= K);
    for (int32_t j = 0; j < K; ++j) {
      int32_t best = -1;
      for (int32_t e = 0; e < E; ++e) {
        if (keys[e] == -INFINITY) continue; /* already taken */
        if (use_cap && count[e] >= cap) continue;
        if (best < 0 || keys[e] > keys[best]) best = e;
      }
      ids[t * K + j] = best;
      keys[best] = -INFINITY;
      count[best] += 1;
    }
  }
  int64_t hot = (hot_e >= 0 && hot_e < E) ? count[hot_e] : 0;
  free(count);
  free(keys);
  return hot;
}
