/*
 * synth.c — seeded synthetic inputs shared by the tests, the smoke check and the
 * benchmark.  It holds none of the NVFP4 arithmetic: only random numbers and the
 * bf16 rounding of what it generates.
 *
 * Generator (counter based, so any element can be produced independently):
 *   mix64(z)        : the splitmix64 output function (Steele, Lea, Flood 2014;
 *                     constants as published by S. Vigna):
 *                     z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                     z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31.
 *   key(seed, s)    = mix64(seed + (s + 1) * 0x9E3779B97F4A7C15)    (stream s)
 *   u64(seed, s, i) = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   unif(...)       = ((u64 >> 11) + 1) * 2^-53                      in (0, 1]
 *   normal(i)       = sqrt(-2 ln unif(2i)) * cos(2 pi unif(2i+1))    (Box-Muller)
 *   student_t3(i)   = z0 / sqrt((z1^2 + z2^2 + z3^2) / 3), z_j = normal(4i + j)
 * Values are formed in double, rounded to float, then to bf16 (nearest-even).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ull;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBull;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_key(uint64_t seed, uint64_t s) { return mix64(seed + (s + 1) * GOLDEN); }

static inline double unif(uint64_t key, uint64_t i) {
  uint64_t z = mix64(key + (i + 1) * GOLDEN);
  return (double)((z >> 11) + 1) * (1.0 / 9007199254740992.0);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = unif(key, 2 * i), u2 = unif(key, 2 * i + 1);
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline double t3_at(uint64_t key, uint64_t i) {
  double z0 = normal_at(key, 4 * i), z1 = normal_at(key, 4 * i + 1);
  double z2 = normal_at(key, 4 * i + 2), z3 = normal_at(key, 4 * i + 3);
  return z0 / sqrt((z1 * z1 + z2 * z2 + z3 * z3) / 3.0);
}

static inline uint16_t to_bf16(double v) {
  float f = (float)v;
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* i-th output (i = 0, 1, ...) of a plain splitmix64 generator whose state starts at `state`. */
uint64_t synth_splitmix64_at(uint64_t state, uint64_t i) { return mix64(state + (i + 1) * GOLDEN); }

uint64_t synth_u64(uint64_t seed, uint64_t stream, uint64_t i) {
  return mix64(stream_key(seed, stream) + (i + 1) * GOLDEN);
}

double synth_uniform(uint64_t seed, uint64_t stream, uint64_t i) {
  return unif(stream_key(seed, stream), i);
}

/* out[i] = bf16(mean + std * normal(first + i)), i < n */
void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, double mean,
                       double std, uint16_t* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = to_bf16(mean + std * normal_at(key, first + (uint64_t)i));
}

/* out[i] = float(mean + std * normal(first + i)) */
void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t first, int64_t n, double mean,
                      double std, float* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(mean + std * normal_at(key, first + (uint64_t)i));
}

/* Activation matrix [rows, cols] (row-major bf16):
 *   x[r, c] = bf16(scale * student_t3(r * cols + c) * (outlier(c) ? factor : 1))
 * `outlier` is a 0/1 byte per column. */
void synth_t3_matrix_bf16(uint64_t seed, uint64_t stream, int64_t rows, int64_t cols, double scale,
                          const uint8_t* outlier, double factor, uint16_t* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      double v = scale * t3_at(key, (uint64_t)(r * cols + c));
      if (outlier && outlier[c]) v *= factor;
      out[r * cols + c] = to_bf16(v);
    }
}

/* Matrix [rows, cols] of bf16(N(0,1)) with columns flagged in `outlier` scaled by factor. */
void synth_normal_matrix_bf16(uint64_t seed, uint64_t stream, int64_t rows, int64_t cols,
                              double std, const uint8_t* outlier, double factor, uint16_t* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < rows; ++r)
    for (int64_t c = 0; c < cols; ++c) {
      double v = std * normal_at(key, (uint64_t)(r * cols + c));
      if (outlier && outlier[c]) v *= factor;
      out[r * cols + c] = to_bf16(v);
    }
}

/* KV chunk [T][C] with C = heads * head_dim:
 *   out[t, c] = bf16(normal(first_token * C + t * C + c) + offset[c])   (offset may be NULL) */
void synth_kv_chunk_bf16(uint64_t seed, uint64_t stream, int64_t first_token, int64_t T, int64_t C,
                         const float* offset, uint16_t* out) {
  uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t)
    for (int64_t c = 0; c < C; ++c) {
      double v = normal_at(key, (uint64_t)((first_token + t) * C + c));
      if (offset) v += (double)offset[c];
      out[t * C + c] = to_bf16(v);
    }
}

/* The first `count` distinct values of floor(unif(i) * n), i = 0, 1, ... (count <= n). */
void synth_distinct_picks(uint64_t seed, uint64_t stream, int64_t n, int64_t count, int64_t* out) {
  uint64_t key = stream_key(seed, stream);
  int64_t got = 0;
  for (uint64_t i = 0; got < count; ++i) {
    int64_t v = (int64_t)(unif(key, i) * (double)n);
    if (v >= n) v = n - 1;
    int dup = 0;
    for (int64_t j = 0; j < got; ++j)
      if (out[j] == v) { dup = 1; break; }
    if (!dup) out[got++] = v;
  }
}
