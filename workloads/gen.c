/*
 * Seeded synthetic Q/K/V generator for Token Sparse Attention prefill
 * workloads.
 *
 * This file holds no step of the attention method itself: it only draws
 * numbers. Both the CPU oracle (tests) and the CUDA path (tests, bench)
 * consume its output, so the two sides see the same bytes.
 *
 * Random numbers: SplitMix64 (Steele, Lea and Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014; finaliser constants as
 * published by Vigna), used counter-based: value n of stream (seed, id) is
 * mix(key + (n + 1) * GAMMA) with key = mix(mix(seed) ^ id * PHI2).
 * Normals: Box-Muller (cosine branch) on two uniforms in (0, 1].
 * bf16: round-to-nearest-even of the fp32 value (NaN kept quiet).
 *
 * Workload structure (shapes of the long-context prefill runs the pages
 * evaluate; the benchmark datasets themselves are not used):
 *   - Q [B,Hq,L,d], K and V [B,Hkv,L,d], all ~ N(0,1) in bf16.
 *   - Optional local band bias: per (b, kv head) a moving sum of iid N(0,1)
 *     vectors over a window of 2*half+1 positions, scaled to unit variance,
 *     mixed into Q and K as (x + a*u)/sqrt(1+a^2).  Q heads of one group
 *     share the same u as their K head.
 *   - Heavy keys: per (b, kv head) a set of distinct rows of K, drawn by a
 *     partial Fisher-Yates shuffle, multiplied by heavy_scale (fp32) and
 *     re-rounded to bf16.  Optional sink: row 0 of K multiplied by
 *     sink_scale instead (the sink multiplier replaces the heavy one).
 *   - heavy_count > 0 fixes the number of heavy rows; otherwise the count is
 *     ceil(frac * L) with frac drawn U[frac_lo, frac_hi] per (b, kv head)
 *     (frac_lo == frac_hi gives a fixed fraction).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ull
#define PHI2 0xD1B54A32D192ED03ull

enum { STREAM_Q = 1, STREAM_K = 2, STREAM_V = 3, STREAM_BAND = 4,
       STREAM_HEAVY = 5, STREAM_FRAC = 6 };

typedef struct {
  int32_t B, Hq, Hkv, L, d;
  uint64_t seed;
  int32_t heavy_count;
  double heavy_frac_lo, heavy_frac_hi;
  float heavy_scale;
  int32_t sink;
  float sink_scale;
  int32_t band_half;
  double band_a;
} tsagen_spec;

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t id) {
  return mix64(mix64(seed + GAMMA) ^ (id * PHI2));
}

/* Value n of the counter-based stream with the given key. */
static inline uint64_t draw(uint64_t key, uint64_t n) {
  return mix64(key + (n + 1) * GAMMA);
}

/* Uniform in (0, 1] from the top 53 bits. */
static inline double unit_open0(uint64_t x) {
  return (double)((x >> 11) + 1) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t n) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = unit_open0(draw(key, 2 * n));
  double u2 = unit_open0(draw(key, 2 * n + 1));
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline uint16_t f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* ---- exported helpers (also used by the tests to pin the generator) ---- */

uint64_t tsagen_mix64(uint64_t z) { return mix64(z); }

uint64_t tsagen_draw(uint64_t seed, uint32_t stream, uint64_t n) {
  return draw(stream_key(seed, stream), n);
}

double tsagen_normal(uint64_t seed, uint32_t stream, uint64_t n) {
  return normal_at(stream_key(seed, stream), n);
}

uint16_t tsagen_f32_to_bf16(float f) { return f32_to_bf16(f); }

static void fill_normal(uint64_t key, uint16_t* out, int64_t count) {
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < count; ++n) out[n] = f32_to_bf16((float)normal_at(key, (uint64_t)n));
}

/* Number of heavy rows for (b, g). */
static int32_t heavy_rows_count(const tsagen_spec* s, int b, int g) {
  if (s->heavy_count > 0) return s->heavy_count < s->L ? s->heavy_count : s->L;
  if (s->heavy_frac_hi <= 0.0) return 0;
  double frac = s->heavy_frac_lo;
  if (s->heavy_frac_hi > s->heavy_frac_lo) {
    uint64_t key = stream_key(s->seed, STREAM_FRAC);
    double u = unit_open0(draw(key, (uint64_t)b * (uint64_t)s->Hkv + (uint64_t)g));
    frac = s->heavy_frac_lo + (s->heavy_frac_hi - s->heavy_frac_lo) * u;
  }
  double c = ceil(frac * (double)s->L);
  if (c > s->L) c = s->L;
  return (int32_t)c;
}

/* Distinct heavy rows of (b, g) by partial Fisher-Yates over [0, L).
 * Writes at most cap rows; returns the count. */
int32_t tsagen_heavy_rows(const tsagen_spec* s, int32_t b, int32_t g, int32_t* rows, int32_t cap) {
  int32_t m = heavy_rows_count(s, b, g);
  if (m <= 0) return 0;
  int32_t L = s->L;
  int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (size_t)L);
  if (!perm) return -1;
  for (int32_t i = 0; i < L; ++i) perm[i] = i;
  uint64_t key = stream_key(s->seed, STREAM_HEAVY);
  uint64_t base = ((uint64_t)b * (uint64_t)s->Hkv + (uint64_t)g) << 32;
  for (int32_t i = 0; i < m; ++i) {
    uint64_t r = draw(key, base + (uint64_t)i);
    uint64_t span = (uint64_t)(L - i);
    int32_t j = i + (int32_t)(((unsigned __int128)r * span) >> 64);
    int32_t t = perm[i];
    perm[i] = perm[j];
    perm[j] = t;
  }
  int32_t n = m < cap ? m : cap;
  memcpy(rows, perm, sizeof(int32_t) * (size_t)n);
  free(perm);
  return m;
}

/* Local band bias for group (b, g): u_t = (1/sqrt(2h+1)) * sum_{|s-t|<=h} g_s. */
static int apply_band(const tsagen_spec* s, int b, int g, uint16_t* q, uint16_t* k) {
  const int64_t L = s->L, d = s->d, h = s->band_half;
  const int64_t span = L + 2 * h;
  const int G = s->Hq / s->Hkv;
  double* gv = (double*)malloc(sizeof(double) * (size_t)(span * d));
  double* u = (double*)malloc(sizeof(double) * (size_t)(L * d));
  if (!gv || !u) { free(gv); free(u); return -1; }
  uint64_t key = stream_key(s->seed, STREAM_BAND);
  uint64_t off = ((uint64_t)b * (uint64_t)s->Hkv + (uint64_t)g) * (uint64_t)(span * d);
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < span * d; ++n) gv[n] = normal_at(key, off + (uint64_t)n);
  const double norm = 1.0 / sqrt((double)(2 * h + 1));
#pragma omp parallel for schedule(static)
  for (int64_t dd = 0; dd < d; ++dd) {
    double acc = 0.0;
    for (int64_t t = 0; t < 2 * h + 1; ++t) acc += gv[t * d + dd];
    for (int64_t t = 0; t < L; ++t) {
      u[t * d + dd] = acc * norm;
      if (t + 1 < L) acc += gv[(t + 2 * h + 1) * d + dd] - gv[t * d + dd];
    }
  }
  const double a = s->band_a;
  const double inv = 1.0 / sqrt(1.0 + a * a);
  for (int hh = 0; hh < G; ++hh) {
    uint16_t* qh = q + ((int64_t)b * s->Hq + (int64_t)g * G + hh) * L * d;
#pragma omp parallel for schedule(static)
    for (int64_t n = 0; n < L * d; ++n)
      qh[n] = f32_to_bf16((float)(((double)bf16_to_f32(qh[n]) + a * u[n]) * inv));
  }
  uint16_t* kh = k + ((int64_t)b * s->Hkv + g) * L * d;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < L * d; ++n)
    kh[n] = f32_to_bf16((float)(((double)bf16_to_f32(kh[n]) + a * u[n]) * inv));
  free(gv);
  free(u);
  return 0;
}

static void scale_row(uint16_t* row, int64_t d, float mult) {
  for (int64_t i = 0; i < d; ++i) row[i] = f32_to_bf16(bf16_to_f32(row[i]) * mult);
}

/* Fill q, k, v (caller-owned, bf16 bit patterns). Returns 0 on success. */
int tsagen_generate(const tsagen_spec* s, uint16_t* q, uint16_t* k, uint16_t* v) {
  if (!s || s->B <= 0 || s->Hq <= 0 || s->Hkv <= 0 || s->L <= 0 || s->d <= 0) return -1;
  if (s->Hq % s->Hkv != 0) return -1;
  const int64_t L = s->L, d = s->d;
  fill_normal(stream_key(s->seed, STREAM_Q), q, (int64_t)s->B * s->Hq * L * d);
  fill_normal(stream_key(s->seed, STREAM_K), k, (int64_t)s->B * s->Hkv * L * d);
  fill_normal(stream_key(s->seed, STREAM_V), v, (int64_t)s->B * s->Hkv * L * d);
  for (int b = 0; b < s->B; ++b) {
    for (int g = 0; g < s->Hkv; ++g) {
      if (s->band_half > 0 && apply_band(s, b, g, q, k) != 0) return -2;
      uint16_t* kh = k + ((int64_t)b * s->Hkv + g) * L * d;
      int32_t m = heavy_rows_count(s, b, g);
      if (m > 0) {
        int32_t* rows = (int32_t*)malloc(sizeof(int32_t) * (size_t)m);
        if (!rows) return -2;
        tsagen_heavy_rows(s, b, g, rows, m);
        for (int32_t i = 0; i < m; ++i)
          if (!(s->sink && rows[i] == 0)) scale_row(kh + (int64_t)rows[i] * d, d, s->heavy_scale);
        free(rows);
      }
      if (s->sink) scale_row(kh, d, s->sink_scale);
    }
  }
  return 0;
}
