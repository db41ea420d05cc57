/*
 * CPU ORACLE -- test infrastructure only.
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may load
 * or call this file's library.  The product path never does: it has no CPU
 * fallback.  This file shares no code, header, table or helper with the CUDA
 * library; the two meet only at the canonical (interchange) input layout.
 *
 * What it computes: the group-quantised weight x activation product of
 * single-user decode.  The weight formats are 4-bit integers (jdon.com "Two
 * RTX 3090s, 105 tok/s", section "27 billion parameters into 24 GB": four bits
 * per parameter instead of sixteen) and 8-bit integers for the sensitive
 * projections and the output head (bs178.com llamAmpere post, "Why it is this
 * fast", part two).  The pages never give the bit layout or the group size, so
 * the plain reading below is taken:
 *
 *   W is N x K, stored as integers q[n][k] with one fp16 scale s[n][g] per
 *   group of 32 consecutive k (g = k / 32), symmetric (no zero point):
 *       w[n][k] = s[n][k/32] * q[n][k]          (exact in fp32)
 *   x is M x K bf16 (the 16-bit activations of "W4A16": jdon.com page, section
 *   "Schools of quantisation"), y is M x N:
 *       y[m][n] = sum_k w[n][k] * x[m][k]       accumulated in fp64
 *       B[m][n] = sum_k |w[n][k] * x[m][k]|     (the scale of the error bound)
 *
 * Every product w*x is exact in fp64 (at most 11+8+8 significant bits), so the
 * only rounding is the fp64 summation, |error| <= K * 2^-53 * B.
 *
 * Canonical layout read here:
 *   q4: uint8 [N][K/2], element k in byte k/2, low nibble for even k,
 *       4-bit two's complement (values -8..7).
 *   q8: int8 [N][K].
 *   s:  uint16 [N][K/32], IEEE 754 binary16 bits.
 *   x:  uint16 [M][K], bfloat16 bits (the upper half of an IEEE binary32).
 *   y, B: double [M][N].
 */
#include <math.h>
#include <stdint.h>

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_value(uint16_t h) {
  const int sign = (h >> 15) & 1;
  const int e = (h >> 10) & 0x1F;
  const int f = h & 0x3FF;
  double v;
  if (e == 0)
    v = ldexp((double)f, -24); /* zero / subnormal: f * 2^-14 * 2^-10 */
  else if (e == 31)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(1024 + f), e - 15 - 10);
  return sign ? -v : v;
}

/* bfloat16: 1 sign bit, 8 exponent bits (bias 127), 7 fraction bits. */
double oracle_bf16_value(uint16_t b) {
  const int sign = (b >> 15) & 1;
  const int e = (b >> 7) & 0xFF;
  const int f = b & 0x7F;
  double v;
  if (e == 0)
    v = ldexp((double)f, -126 - 7);
  else if (e == 255)
    v = f ? NAN : INFINITY;
  else
    v = ldexp((double)(128 + f), e - 127 - 7);
  return sign ? -v : v;
}

/* Element k of a canonical q4 row: 4-bit two's complement nibble. */
int oracle_q4_value(const uint8_t* row, int64_t k) {
  const int byte = row[k / 2];
  const int nib = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
  return nib >= 8 ? nib - 16 : nib;
}

/* Element k of a canonical q8 row. */
int oracle_q8_value(const int8_t* row, int64_t k) { return (int)row[k]; }

/* Dequantised weight w[n][k] as the fp32 product s * q (exact: an 11-bit
 * significand times an integer of at most 8 bits). */
float oracle_weight(int bits, const void* q, const uint16_t* s, int64_t K, int64_t n, int64_t k) {
  int qv;
  if (bits == 4)
    qv = oracle_q4_value((const uint8_t*)q + n * (K / 2), k);
  else
    qv = oracle_q8_value((const int8_t*)q + n * K, k);
  const float sv = (float)oracle_f16_value(s[n * (K / 32) + k / 32]);
  return sv * (float)qv;
}

/*
 * y[m][n] = sum_k w[n][k] x[m][k] and B[m][n] = sum_k |w[n][k] x[m][k]|, both
 * in fp64, in plain k order.  Returns 0, or -1 on a bad argument.
 */
int oracle_gemv(int bits, const void* q, const uint16_t* s, int64_t N, int64_t K, const uint16_t* x, int M,
                double* y, double* absacc) {
  /* N = 0 and K = 0 are valid: an empty output, or the empty sum 0 */
  if ((bits != 4 && bits != 8) || N < 0 || K < 0 || K % 32 != 0 || M < 1 || !y) return -1;
  if (N > 0 && K > 0 && (!q || !s || !x)) return -1;
#pragma omp parallel for schedule(dynamic, 16)
  for (int64_t n = 0; n < N; ++n) {
    for (int m = 0; m < M; ++m) {
      double acc = 0.0, aacc = 0.0;
      for (int64_t k = 0; k < K; ++k) {
        const double w = (double)oracle_weight(bits, q, s, K, n, k);
        const double xv = oracle_bf16_value(x[(int64_t)m * K + k]);
        acc += w * xv;
        aacc += fabs(w * xv);
      }
      y[(int64_t)m * N + n] = acc;
      if (absacc) absacc[(int64_t)m * N + n] = aacc;
    }
  }
  return 0;
}

/* Dense dequantised matrix W[n][k] as double (for tests that go through a
 * library matrix product). */
int oracle_dequantize(int bits, const void* q, const uint16_t* s, int64_t N, int64_t K, double* W) {
  if ((bits != 4 && bits != 8) || N < 0 || K < 0 || K % 32 != 0 || (N * K > 0 && (!q || !s || !W))) return -1;
  for (int64_t n = 0; n < N; ++n)
    for (int64_t k = 0; k < K; ++k) W[n * K + k] = (double)oracle_weight(bits, q, s, K, n, k);
  return 0;
}

/* Number of OpenMP threads a parallel region of this library uses. */
int oracle_threads(void) {
  int t = 1;
#pragma omp parallel
  {
#pragma omp single
    {
#ifdef _OPENMP
      extern int omp_get_num_threads(void);
      t = omp_get_num_threads();
#endif
    }
  }
  return t;
}
