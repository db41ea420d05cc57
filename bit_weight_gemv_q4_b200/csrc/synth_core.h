/*
 * Seeded synthetic inputs: the generator's definition, compiled for the host
 * (gcc or nvcc's host pass) and for the device from this one source, so that
 * both sides produce identical bits.  It holds no arithmetic of the quantised
 * product: only random integers, normals and their fp16 / bf16 encodings.
 *
 * Determinism across host and device: every floating-point step is a single
 * IEEE-754 double operation (+, -, *, / and sqrt, all correctly rounded on both
 * sides); logarithm and cosine are written out below as short series instead of
 * calling a math library, and the files that include this header are compiled
 * without floating-point contraction (-ffp-contract=off, -fmad=false).
 *
 * Random words: counter-based.  A (seed, stream) pair gives a key; word i of a
 * stream is the SplitMix64 finaliser of key + (i + 1) * 0x9E3779B97F4A7C15
 * (Steele, Lea & Flood, "Fast splittable pseudorandom number generators",
 * OOPSLA 2014).  Any word can be computed on its own.
 *
 * Distributions:
 *   q4: word n*(K/16) + k/16 holds 16 nibbles; nibble k % 16 is the 4-bit two's
 *       complement code of element (n, k), uniform on [-8, 7].
 *   q8: word n*(K/2) + k/2; 32-bit half k % 2, h, gives q = (h*255 >> 32) - 127,
 *       uniform on [-127, 127] (Lemire's multiply-shift; bias below 6e-8).
 *   normal i: Box-Muller, z = sqrt(-2 ln u1) cos(2 pi u2) with u1, u2 from
 *       words 2i and 2i+1, u = ((w >> 11) + 0.5) * 2^-53 in (0, 1).
 *   scales: fp16 round-to-nearest-even of |std * z|; activations: bf16
 *       round-to-nearest-even of z.
 */
#ifndef Q4_SYNTH_CORE_H
#define Q4_SYNTH_CORE_H

#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define SYNTH_HD __host__ __device__ __forceinline__
#else
#define SYNTH_HD static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL
#define SYNTH_STREAM_MUL 0xD1B54A32D192ED03ULL

SYNTH_HD uint64_t synth_mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

SYNTH_HD uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix64((seed + 1) * SYNTH_GAMMA) ^ synth_mix64((stream + 1) * SYNTH_STREAM_MUL);
}

SYNTH_HD uint64_t synth_word(uint64_t key, uint64_t i) { return synth_mix64(key + (i + 1) * SYNTH_GAMMA); }

SYNTH_HD uint64_t synth_dbits(double d) {
#ifdef __CUDA_ARCH__
  return (uint64_t)__double_as_longlong(d);
#else
  uint64_t b;
  memcpy(&b, &d, sizeof b);
  return b;
#endif
}

SYNTH_HD double synth_bitsd(uint64_t b) {
#ifdef __CUDA_ARCH__
  return __longlong_as_double((long long)b);
#else
  double d;
  memcpy(&d, &b, sizeof d);
  return d;
#endif
}

/* 2^n for -1022 <= n <= 1023, exactly. */
SYNTH_HD double synth_pow2(int n) { return synth_bitsd((uint64_t)(n + 1023) << 52); }

/* Round a non-negative double below 2^51 to the nearest integer, ties to even
 * (adding and removing 2^52 leaves no fraction bits in round-to-nearest). */
SYNTH_HD double synth_rint(double m) {
  const double big = 4503599627370496.0; /* 2^52 */
#ifdef __CUDA_ARCH__
  return __dsub_rn(__dadd_rn(m, big), big);
#else
  const double t = m + big;
  return t - big;
#endif
}

SYNTH_HD double synth_unit(uint64_t w) { return ((double)(w >> 11) + 0.5) * 0x1p-53; }

/* ln(u) for u in (0, 1]: u = m 2^e with m in [sqrt(1/2), sqrt(2)), and
 * ln m = 2 atanh(s), s = (m - 1)/(m + 1), |s| < 0.172, as an odd series. */
SYNTH_HD double synth_log(double u) {
  const uint64_t b = synth_dbits(u);
  int e = (int)((b >> 52) & 0x7FF) - 1023;
  double m = synth_bitsd((b & 0x000FFFFFFFFFFFFFULL) | 0x3FF0000000000000ULL); /* [1, 2) */
  if (m > 1.4142135623730951) {
    m = m * 0.5;
    e += 1;
  }
  const double s = (m - 1.0) / (m + 1.0);
  const double t = s * s;
  double p = 1.0 / 23.0;
  p = p * t + 1.0 / 21.0;
  p = p * t + 1.0 / 19.0;
  p = p * t + 1.0 / 17.0;
  p = p * t + 1.0 / 15.0;
  p = p * t + 1.0 / 13.0;
  p = p * t + 1.0 / 11.0;
  p = p * t + 1.0 / 9.0;
  p = p * t + 1.0 / 7.0;
  p = p * t + 1.0 / 5.0;
  p = p * t + 1.0 / 3.0;
  p = p * t + 1.0;
  return (double)e * 0.6931471805599453 + 2.0 * s * p;
}

/* sin and cos of theta in [0, pi/4] by their Taylor series. */
SYNTH_HD double synth_sin_small(double th) {
  const double t = th * th;
  double p = -1.0 / 355687428096000.0;   /* -1/17! */
  p = p * t + 1.0 / 1307674368000.0;     /* 1/15! */
  p = p * t - 1.0 / 6227020800.0;        /* 1/13! */
  p = p * t + 1.0 / 39916800.0;          /* 1/11! */
  p = p * t - 1.0 / 362880.0;            /* 1/9! */
  p = p * t + 1.0 / 5040.0;              /* 1/7! */
  p = p * t - 1.0 / 120.0;               /* 1/5! */
  p = p * t + 1.0 / 6.0;                 /* 1/3! */
  p = p * t;
  return th - th * p;
}

SYNTH_HD double synth_cos_small(double th) {
  const double t = th * th;
  double p = 1.0 / 6402373705728000.0;   /* 1/18! */
  p = p * t - 1.0 / 20922789888000.0;    /* 1/16! */
  p = p * t + 1.0 / 87178291200.0;       /* 1/14! */
  p = p * t - 1.0 / 479001600.0;         /* 1/12! */
  p = p * t + 1.0 / 3628800.0;           /* 1/10! */
  p = p * t - 1.0 / 40320.0;             /* 1/8! */
  p = p * t + 1.0 / 720.0;               /* 1/6! */
  p = p * t - 1.0 / 24.0;                /* 1/4! */
  p = p * t + 0.5;                       /* 1/2! */
  return 1.0 - t * p;
}

/* cos(2 pi u) for u in [0, 1): quadrant q = floor(4u), remainder r in [0, 1)
 * (both exact), angle (pi/2) r folded into [0, pi/4]. */
SYNTH_HD double synth_cos2pi(double u) {
  const double v = 4.0 * u;
  const int q = (int)v;
  const double r = v - (double)q;
  const double half_pi = 1.5707963267948966;
  double c, s;
  if (r <= 0.5) {
    const double th = r * half_pi;
    c = synth_cos_small(th);
    s = synth_sin_small(th);
  } else {
    const double th = (1.0 - r) * half_pi;
    c = synth_sin_small(th);
    s = synth_cos_small(th);
  }
  switch (q & 3) {
    case 0: return c;
    case 1: return -s;
    case 2: return -c;
    default: return s;
  }
}

SYNTH_HD double synth_normal(uint64_t key, uint64_t i) {
  const double u1 = synth_unit(synth_word(key, 2 * i));
  const double u2 = synth_unit(synth_word(key, 2 * i + 1));
#ifdef __CUDA_ARCH__
  const double r = __dsqrt_rn(-2.0 * synth_log(u1));
#else
  const double r = __builtin_sqrt(-2.0 * synth_log(u1));
#endif
  return r * synth_cos2pi(u2);
}

/* Nearest fp16 (ties to even), as bits. */
SYNTH_HD uint16_t synth_f64_to_f16(double d) {
  const uint64_t b = synth_dbits(d);
  const uint16_t sign = (uint16_t)((b >> 48) & 0x8000);
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFULL;
  if (mag > 0x7FF0000000000000ULL) return (uint16_t)(sign | 0x7E00); /* NaN */
  const double a = synth_bitsd(mag);
  if (a >= 65520.0) return (uint16_t)(sign | 0x7C00);
  if (a < 0x1p-14) return (uint16_t)(sign | (uint16_t)synth_rint(a * 0x1p24)); /* m * 2^-24, m <= 1024 */
  const int e = (int)((mag >> 52) & 0x7FF) - 1023;                          /* -14 .. 15 */
  double m = synth_rint(a * synth_pow2(10 - e));                             /* [1024, 2048] */
  int E = e + 15;
  if (m == 2048.0) {
    m = 1024.0;
    E += 1;
  }
  if (E >= 31) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | (E << 10) | ((int)m - 1024));
}

/* Nearest bf16 (ties to even), as bits. */
SYNTH_HD uint16_t synth_f64_to_bf16(double d) {
  const uint64_t b = synth_dbits(d);
  const uint16_t sign = (uint16_t)((b >> 48) & 0x8000);
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFULL;
  if (mag > 0x7FF0000000000000ULL) return (uint16_t)(sign | 0x7FC0);
  const double a = synth_bitsd(mag);
  if (a >= 0x1.FFp127) return (uint16_t)(sign | 0x7F80);
  if (a < 0x1p-126) return (uint16_t)(sign | (uint16_t)synth_rint(a * 0x1p133)); /* m * 2^-133, m <= 128 */
  const int e = (int)((mag >> 52) & 0x7FF) - 1023;                            /* -126 .. 127 */
  double m = synth_rint(a * synth_pow2(7 - e));                                 /* [128, 256] */
  int E = e + 127;
  if (m == 256.0) {
    m = 128.0;
    E += 1;
  }
  if (E >= 255) return (uint16_t)(sign | 0x7F80);
  return (uint16_t)(sign | (E << 7) | ((int)m - 128));
}

/* Element generators, addressed by position. */
SYNTH_HD uint8_t synth_q4_byte(uint64_t key, int64_t K, int64_t row, int64_t byte_in_row) {
  const uint64_t w = synth_word(key, (uint64_t)row * (uint64_t)(K / 16) + (uint64_t)(byte_in_row / 8));
  return (uint8_t)((w >> (8 * (byte_in_row % 8))) & 0xFF);
}

SYNTH_HD int8_t synth_q8_value(uint64_t key, int64_t K, int64_t row, int64_t k) {
  const uint64_t w = synth_word(key, (uint64_t)row * (uint64_t)(K / 2) + (uint64_t)(k / 2));
  const uint64_t h = (w >> (32 * (k % 2))) & 0xFFFFFFFFULL;
  return (int8_t)((int64_t)((h * 255ULL) >> 32) - 127);
}

SYNTH_HD uint16_t synth_scale_value(uint64_t key, int64_t G, int64_t row, int64_t g, double std) {
  const double z = synth_normal(key, (uint64_t)row * (uint64_t)G + (uint64_t)g);
  const double v = std * z;
  return synth_f64_to_f16(v < 0 ? -v : v);
}

/* NVFP4 block scale (E4M3 bits) of block b of a row: finite, positive, from
   0x28 (0.25) to 0x47 (3.75), uniform over the 32 byte values. */
SYNTH_HD uint8_t synth_e4m3_scale(uint64_t key, int64_t B, int64_t row, int64_t b) {
  const uint64_t w = synth_word(key, (uint64_t)row * (uint64_t)B + (uint64_t)b);
  return (uint8_t)(0x28 + (w >> 59));
}

#endif /* Q4_SYNTH_CORE_H */
