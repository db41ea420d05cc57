/*
 * Seeded synthetic inputs for the group-quantised weight x activation product.
 *
 * This file holds NO arithmetic of the product itself: it only draws random
 * integers, normals and their fp16/bf16 encodings.  Both the CUDA path and the
 * CPU oracle consume what it writes; neither calls the other.
 *
 * Random numbers: a counter-based generator.  Each (seed, stream) pair gets a
 * key; word i of the stream is the SplitMix64 finaliser applied to
 * key + (i + 1) * golden-ratio increment (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  Every word is addressable on
 * its own, so any row of any tensor can be regenerated without the others.
 *
 * Distributions (the workloads of the single-user decode weight stream):
 *   q4 weights : 16 codes of 4-bit two's complement, uniform on [-8, 7];
 *                word n*(K/16) + k/16 holds 16 nibbles, nibble k%16 is element (n,k).
 *   q8 weights : uniform on [-127, 127]; word n*(K/2) + k/2, 32-bit half k%2,
 *                mapped by Lemire's multiply-shift h*255 >> 32 (bias < 6e-8).
 *   normals    : Box-Muller (cosine branch) in double precision on words 2i, 2i+1.
 *   scales     : fp16, round-to-nearest-even of |0.02 * z|.
 *   activations: bf16, round-to-nearest-even of z.
 *
 * Canonical (interchange) layout written here:
 *   q4: uint8 [N][K/2], element k in byte k/2, low nibble for even k.
 *   q8: int8  [N][K].
 *   scales: uint16 fp16 bits [N][K/32].
 *   x: uint16 bf16 bits [M][K].
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL
#define SYNTH_STREAM_MUL 0xD1B54A32D192ED03ULL

static inline uint64_t synth_mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix64((seed + 1) * SYNTH_GAMMA) ^ synth_mix64((stream + 1) * SYNTH_STREAM_MUL);
}

uint64_t synth_word(uint64_t key, uint64_t i) { return synth_mix64(key + (i + 1) * SYNTH_GAMMA); }

/* Uniform double in the open interval (0, 1) from the top 53 bits of a word. */
static inline double synth_unit(uint64_t w) { return ((double)(w >> 11) + 0.5) * 0x1p-53; }

double synth_normal(uint64_t key, uint64_t i) {
  double u1 = synth_unit(synth_word(key, 2 * i));
  double u2 = synth_unit(synth_word(key, 2 * i + 1));
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* Round a double to the nearest fp16 (ties to even), returning its bits.
 * Uses the default rounding mode of nearbyint (round-to-nearest-even). */
uint16_t synth_f64_to_f16(double d) {
  uint16_t sign = signbit(d) ? 0x8000 : 0;
  double a = fabs(d);
  if (isnan(d)) return (uint16_t)(sign | 0x7E00);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00);
  if (a < 0x1p-14) {
    /* subnormal range: value = m * 2^-24, m in [0, 1024] (1024 is the smallest normal) */
    double m = nearbyint(a * 0x1p24);
    return (uint16_t)(sign | (uint16_t)m);
  }
  int e;
  (void)frexp(a, &e); /* a = f * 2^e with f in [0.5, 1) */
  double m = nearbyint(ldexp(a, 11 - e)); /* significand in [1024, 2048] */
  int E = e - 1 + 15;
  if (m == 2048.0) {
    m = 1024.0;
    E += 1;
  }
  if (E >= 31) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | (E << 10) | ((int)m - 1024));
}

/* Round a double to the nearest bf16 (ties to even), returning its bits. */
uint16_t synth_f64_to_bf16(double d) {
  uint16_t sign = signbit(d) ? 0x8000 : 0;
  double a = fabs(d);
  if (isnan(d)) return (uint16_t)(sign | 0x7FC0);
  /* largest finite bf16 is (2 - 2^-7) * 2^127; halfway to 2^128 rounds up */
  if (a >= 0x1.FFp127) return (uint16_t)(sign | 0x7F80);
  if (a < 0x1p-126) {
    /* subnormal range: value = m * 2^-133, m in [0, 128] (128 is the smallest normal) */
    double m = nearbyint(a * 0x1p133);
    return (uint16_t)(sign | (uint16_t)m);
  }
  int e;
  (void)frexp(a, &e);
  double m = nearbyint(ldexp(a, 8 - e)); /* significand in [128, 256] */
  int E = e - 1 + 127;
  if (m == 256.0) {
    m = 128.0;
    E += 1;
  }
  if (E >= 255) return (uint16_t)(sign | 0x7F80);
  return (uint16_t)(sign | (E << 7) | ((int)m - 128));
}

/* Rows [row0, row0 + nrows) of a q4 tensor with K columns, canonical layout. */
int synth_q4(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, uint8_t* out) {
  if (K <= 0 || K % 32 != 0 || nrows < 0 || row0 < 0 || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  const int64_t words_per_row = K / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    uint8_t* dst = out + r * (K / 2);
    const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)words_per_row;
    for (int64_t w = 0; w < words_per_row; ++w) {
      uint64_t v = synth_word(key, base + (uint64_t)w);
      /* 16 nibbles; nibble j is element 16w + j; bytes hold (even, odd) pairs */
      for (int j = 0; j < 8; ++j) dst[w * 8 + j] = (uint8_t)((v >> (8 * j)) & 0xFF);
    }
  }
  return 0;
}

/* Rows [row0, row0 + nrows) of a q8 tensor with K columns, canonical layout. */
int synth_q8(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, int8_t* out) {
  if (K <= 0 || K % 32 != 0 || nrows < 0 || row0 < 0 || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  const int64_t words_per_row = K / 2;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    int8_t* dst = out + r * K;
    const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)words_per_row;
    for (int64_t w = 0; w < words_per_row; ++w) {
      uint64_t v = synth_word(key, base + (uint64_t)w);
      for (int j = 0; j < 2; ++j) {
        uint64_t h = (v >> (32 * j)) & 0xFFFFFFFFULL;
        dst[2 * w + j] = (int8_t)((int64_t)((h * 255ULL) >> 32) - 127);
      }
    }
  }
  return 0;
}

/* Rows [row0, row0 + nrows) of the fp16 group scales [N][K/32] = |std * z|. */
int synth_scales(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, double std,
                 uint16_t* out) {
  if (K <= 0 || K % 32 != 0 || nrows < 0 || row0 < 0 || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  const int64_t G = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r) {
    const uint64_t base = (uint64_t)(row0 + r) * (uint64_t)G;
    for (int64_t g = 0; g < G; ++g)
      out[r * G + g] = synth_f64_to_f16(fabs(std * synth_normal(key, base + (uint64_t)g)));
  }
  return 0;
}

/* count normals of a stream from index i0, rounded to bf16 (activations). */
int synth_bf16_normals(uint64_t seed, uint64_t stream, int64_t i0, int64_t count, uint16_t* out) {
  if (count < 0 || i0 < 0 || (!out && count > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = synth_f64_to_bf16(synth_normal(key, (uint64_t)(i0 + i)));
  return 0;
}

/* Raw normals in double (tests of the distribution). */
int synth_normals_f64(uint64_t seed, uint64_t stream, int64_t i0, int64_t count, double* out) {
  if (count < 0 || i0 < 0 || (!out && count > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i) out[i] = synth_normal(key, (uint64_t)(i0 + i));
  return 0;
}

/* Elementwise conversions exposed for tests. */
void synth_f64_to_f16_array(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_f64_to_f16(in[i]);
}
void synth_f64_to_bf16_array(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_f64_to_bf16(in[i]);
}
void synth_words(uint64_t seed, uint64_t stream, int64_t i0, int64_t count, uint64_t* out) {
  const uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i) out[i] = synth_word(key, (uint64_t)(i0 + i));
}
