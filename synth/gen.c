/*
 * Seeded synthetic inputs for split decode attention: a counter-based
 * generator, shared by the tests, the benchmark and the oracle's callers.
 *
 * This file holds no attention arithmetic.  It only turns (seed, tensor id,
 * element index) into a number, so any slice of any tensor can be rebuilt on
 * its own, in any order and on any number of threads, with identical bytes.
 *
 *   word(seed, id, i) = splitmix64_mix(key(seed, id) + (i + 1) * GOLDEN)
 *   key(seed, id)     = splitmix64_mix(seed * GOLDEN ^ (id << 32) ^ 0x5EED)
 *
 * splitmix64_mix is the output function of Steele, Lea and Flood's SplitMix64
 * (OOPSLA 2014), with the shift/multiply constants of Vigna's public-domain
 * reference.  A normal value is produced by the Box-Muller transform from two
 * consecutive words of pair p = i / 2 (cosine branch for even i, sine branch for
 * odd i), in double precision, then rounded to float32 (round to nearest even)
 * and, for bf16 tensors, rounded again to bf16 (round to nearest even on the
 * bit pattern).  The oracle never regenerates data: it reads the same host
 * bytes that are uploaded to the device, so libm rounding choices here cannot
 * affect parity.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint32_t id) {
  return mix64(seed * GOLDEN ^ ((uint64_t)id << 32) ^ 0x5EEDULL);
}

static inline uint64_t word_at(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * GOLDEN);
}

uint64_t synth_word(uint64_t seed, uint32_t id, uint64_t i) {
  return word_at(stream_key(seed, id), i);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  const uint64_t p = i >> 1;
  const uint64_t w1 = word_at(key, 2 * p);
  const uint64_t w2 = word_at(key, 2 * p + 1);
  const double u1 = (double)((w1 >> 11) + 1) * 0x1.0p-53; /* (0, 1] */
  const double u2 = (double)(w2 >> 11) * 0x1.0p-53;       /* [0, 1) */
  const double r = sqrt(-2.0 * log(u1));
  const double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

static inline float bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* n normal values for elements [start, start + n) of tensor (seed, id), as bf16 bits. */
void synth_normal_bf16(uint64_t seed, uint32_t id, uint64_t start, uint64_t n, uint16_t* out) {
  const uint64_t key = stream_key(seed, id);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)n; ++j) {
    out[j] = f32_to_bf16_rne((float)normal_at(key, start + (uint64_t)j));
  }
}

/* Same values, rounded only to float32. */
void synth_normal_f32(uint64_t seed, uint32_t id, uint64_t start, uint64_t n, float* out) {
  const uint64_t key = stream_key(seed, id);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < (int64_t)n; ++j) {
    out[j] = (float)normal_at(key, start + (uint64_t)j);
  }
}

/*
 * "Salient spikes": choose exactly n_spikes distinct rows of a [rows][dim] bf16
 * matrix with a seeded partial Fisher-Yates shuffle and multiply each chosen row
 * by `factor` (a power of two, so the product is exact in bf16 unless it
 * overflows).  Draw k picks j = k + (word(seed, id, stream*2^40 + k) mod (rows-k)).
 * The chosen row indices are written to `chosen` (length n_spikes) in draw order.
 * Returns 0 on success, -1 on bad arguments or allocation failure.
 */
int synth_spike_rows_bf16(uint64_t seed, uint32_t id, uint64_t stream, uint16_t* mat, int64_t rows,
                          int32_t dim, int64_t n_spikes, float factor, int64_t* chosen) {
  if (rows < 0 || dim <= 0 || n_spikes < 0 || n_spikes > rows) return -1;
  if (n_spikes == 0) return 0;
  int64_t* perm = (int64_t*)malloc(sizeof(int64_t) * (size_t)rows);
  if (!perm) return -1;
  for (int64_t r = 0; r < rows; ++r) perm[r] = r;
  const uint64_t key = stream_key(seed, id);
  for (int64_t k = 0; k < n_spikes; ++k) {
    const uint64_t w = word_at(key, (stream << 40) + (uint64_t)k);
    const int64_t j = k + (int64_t)(w % (uint64_t)(rows - k));
    const int64_t t = perm[k];
    perm[k] = perm[j];
    perm[j] = t;
    chosen[k] = perm[k];
  }
  free(perm);
  for (int64_t k = 0; k < n_spikes; ++k) {
    uint16_t* row = mat + chosen[k] * (int64_t)dim;
    for (int32_t d = 0; d < dim; ++d) row[d] = f32_to_bf16_rne(bf16_to_f32(row[d]) * factor);
  }
  return 0;
}
