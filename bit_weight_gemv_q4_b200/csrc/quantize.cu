// Offline quantiser: bf16 weights -> group-32 symmetric codes and fp16 scales
// in the canonical layout (the input of q4_pack_weights).  Round to nearest,
// no zero point; the pages leave the recipe open beyond naming 4-bit and 8-bit
// formats and saying that a quantiser's grouping and scale computation matter
// (jdon.com "Two RTX 3090s, 105 tok/s", section "Schools of quantisation").
//
// Every rounding step is fixed, so the host and the device versions produce
// the same bits: per group of 32 values w (fp32, exact from bf16)
//   s32 = max|w| / qmax                 (absmax; qmax 7 or 127, IEEE fp32 division)
//   s32 = w_m / -8                      (signed, q4 only; w_m the first value of
//                                        largest magnitude)
//   s16 = fp16(s32), nearest even, saturated to +-65504;  s = s16 as fp32
//   q   = 0 if s == 0, else clamp(nearest(w / s), lo, hi): the integer nearest
//         to the exact quotient, ties to even
// The host forms the quotient in fp64 (w has an 8-bit, s an 11-bit
// significand: a quotient above 1/2 that is not half-way lies >= 2^-21 from
// the half-way point, beyond fp64's rounding, so rint decides exactly).  The
// device takes a candidate from a reciprocal multiply (within one of the
// nearest integer) and settles it with the exact remainder w - q s (one FMA;
// exact by Sterbenz's lemma, as q s is within a factor 2 of w).
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <string>

#include "q4gemv.h"

namespace q4 {
void set_error(const std::string& msg);
}  // namespace q4

namespace {

int qfail(int code, const std::string& msg) {
  q4::set_error(msg);
  return code;
}

struct QRange {
  int lo, hi;
  float qmax;  // absmax divisor
};

bool quant_range(int bits, int mode, QRange* r) {
  if (bits == 4 && mode == Q4_QUANT_ABSMAX) {
    *r = {-7, 7, 7.f};
  } else if (bits == 4 && mode == Q4_QUANT_SIGNED_MAX) {
    *r = {-8, 7, 0.f};
  } else if (bits == 8 && mode == Q4_QUANT_ABSMAX) {
    *r = {-127, 127, 127.f};
  } else {
    return false;
  }
  return true;
}

int check(int bits, int mode, const void* w, int64_t N, int64_t K, const void* q, const void* s, const char* who,
          QRange* r) {
  if (!quant_range(bits, mode, r))
    return qfail(Q4_ERR_INVALID_ARG, std::string(who) + ": bits must be 4 or 8, mode absmax (or signed-max for 4)");
  if (N < 0 || K < 0 || K % 32 != 0 || K > (int64_t(1) << 30) || N > (int64_t(1) << 34))
    return qfail(Q4_ERR_SHAPE, std::string(who) + ": need N >= 0 and K a multiple of 32");
  if (N * K > 0 && (!w || !q || !s)) return qfail(Q4_ERR_INVALID_ARG, std::string(who) + ": null buffer");
  if ((reinterpret_cast<uintptr_t>(w) | reinterpret_cast<uintptr_t>(s)) & 1)
    return qfail(Q4_ERR_ALIGN, std::string(who) + ": weights and scales must be 2-byte aligned");
  return Q4_OK;
}

// ---------------------------------------------------------------- host
float bf16_to_float(uint16_t b) {
  const uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// fp32 -> fp16 bits, round to nearest even, saturated to +-65504 (finite input).
uint16_t float_to_half_sat(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  const uint32_t sign = (x >> 16) & 0x8000u;
  const uint32_t ax = x & 0x7FFFFFFFu;
  if (ax >= 0x477FF000u) return static_cast<uint16_t>(sign | 0x7BFFu);  // >= 65520 rounds past the largest
  const int e = static_cast<int>(ax >> 23);                               // biased fp32 exponent
  if (e >= 113) {                                                          // fp16 normal: >= 2^-14
    const uint32_t m = ax & 0x7FFFFFu;
    uint32_t h = (static_cast<uint32_t>(e - 112) << 10) | (m >> 13);
    const uint32_t rest = m & 0x1FFFu;
    if (rest > 0x1000u || (rest == 0x1000u && (h & 1u))) ++h;  // a carry moves into the exponent correctly
    return static_cast<uint16_t>(sign | h);
  }
  // fp16 subnormal: units of 2^-24; the value is mant * 2^(e - 150)
  const int sh = 126 - e;  // >= 14
  if (e == 0 || sh > 24) return static_cast<uint16_t>(sign);
  const uint32_t mant = (ax & 0x7FFFFFu) | 0x800000u;
  uint32_t h = mant >> sh;
  const uint32_t rest = mant & ((1u << sh) - 1u), half = 1u << (sh - 1);
  if (rest > half || (rest == half && (h & 1u))) ++h;
  return static_cast<uint16_t>(sign | h);
}

float half_to_float(uint16_t h) {
  const uint32_t sign = static_cast<uint32_t>(h & 0x8000u) << 16;
  const uint32_t e = (h >> 10) & 0x1Fu, m = h & 0x3FFu;
  float f;
  if (e == 0) {
    f = std::ldexp(static_cast<float>(m), -24);
  } else {
    const uint32_t u = ((e + 112) << 23) | (m << 13);
    std::memcpy(&f, &u, 4);
  }
  uint32_t u;
  std::memcpy(&u, &f, 4);
  u |= sign;
  std::memcpy(&f, &u, 4);
  return f;
}

void quantize_group_host(int bits, int mode, const QRange& r, const uint16_t* w, uint8_t* q_out_row, int64_t k0,
                         uint16_t* s_out) {
  float wf[32];
  for (int i = 0; i < 32; ++i) wf[i] = bf16_to_float(w[i]);
  float amax = std::fabs(wf[0]), wm = wf[0];
  for (int i = 1; i < 32; ++i) {
    const float a = std::fabs(wf[i]);
    if (a > amax) {  // strict: the first value of largest magnitude
      amax = a;
      wm = wf[i];
    }
  }
  const float s32 = mode == Q4_QUANT_ABSMAX ? amax / r.qmax : wm / -8.f;
  const uint16_t s16 = float_to_half_sat(s32);
  *s_out = s16;
  const float s = half_to_float(s16);
  for (int i = 0; i < 32; ++i) {
    int q = 0;
    if (s != 0.f) {
      double v = std::rint(static_cast<double>(wf[i]) / static_cast<double>(s));
      v = std::fmin(std::fmax(v, static_cast<double>(r.lo)), static_cast<double>(r.hi));
      q = static_cast<int>(v);
    }
    if (bits == 8) {
      reinterpret_cast<int8_t*>(q_out_row)[k0 + i] = static_cast<int8_t>(q);
    } else {
      uint8_t& byte = q_out_row[(k0 + i) / 2];
      const uint8_t nib = static_cast<uint8_t>(q & 0xF);
      byte = (i & 1) ? static_cast<uint8_t>((byte & 0x0F) | (nib << 4)) : static_cast<uint8_t>((byte & 0xF0) | nib);
    }
  }
}

// ---------------------------------------------------------------- device
constexpr int kQuantGroupsPerLane = 2;  // loads in flight per thread

// One group-part: a lane holds eight values of a group (four lanes per group).
// The lane finds the largest magnitude among its values (the first on ties),
// the four lanes combine theirs in lane order, the group's first lane writes
// the scale, and every lane its eight codes (q4: one 32-bit store, q8: one
// 64-bit store).  All 32 lanes run it (the shuffles need them); `live` lanes
// store.
__device__ __forceinline__ void quantize_part(int bits, int mode, int lo, int hi, float qmax, const uint4 v, bool live,
                                              int part, long long n, long long g, long long G, long long K,
                                              uint8_t* __restrict__ q_out, uint16_t* __restrict__ s_out) {
  const uint32_t words[4] = {v.x, v.y, v.z, v.w};
  float wf[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    wf[2 * i] = __uint_as_float(words[i] << 16);
    wf[2 * i + 1] = __uint_as_float(words[i] & 0xFFFF0000u);
  }
  float amax = fabsf(wf[0]), wm = wf[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    if (fabsf(wf[i]) > amax) {
      amax = fabsf(wf[i]);
      wm = wf[i];
    }
  }
  // combine the four lanes of the group: a later lane wins only if strictly larger
#pragma unroll
  for (int o = 1; o < 4; o <<= 1) {
    const float oa = __shfl_xor_sync(0xFFFFFFFFu, amax, o);
    const float ow = __shfl_xor_sync(0xFFFFFFFFu, wm, o);
    const int opart = part ^ o;
    if (oa > amax || (oa == amax && opart < part)) {
      amax = oa;
      wm = ow;
    }
  }
  if (!live) return;
  const float s32 = mode == Q4_QUANT_ABSMAX ? __fdiv_rn(amax, qmax) : __fdiv_rn(wm, -8.f);
  __half h = __float2half_rn(s32);
  if (__hisinf(h)) h = __float2half_rn(s32 > 0.f ? 65504.f : -65504.f);
  const float s = __half2float(h);
  if (part == 0) s_out[n * G + g] = __half_as_ushort(h);
  int q[8];
  // any reciprocal within a few ulp will do: the candidate it gives is within
  // one of the nearest integer, and the exact remainder settles the rest
  const float rcp = s != 0.f ? __fdividef(1.f, s) : 0.f;
  const float half = 0.5f * fabsf(s);
  const bool s_pos = s > 0.f;  // the quotient grows with w - q s when s > 0
  // adding 1.5 * 2^23 to a float below 2^22 in magnitude rounds it to an
  // integer (nearest, ties to even) held in the low mantissa bits, exactly
  constexpr float kMagic = 12582912.f;
  constexpr int kMagicBits = 0x4B400000;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    // candidate within one of the nearest integer, kept small
    const float x = fminf(fmaxf(wf[i] * rcp, static_cast<float>(lo - 1)), static_cast<float>(hi + 1));
    const float cm = x + kMagic;
    const float c = cm - kMagic;
    int ci = __float_as_int(cm) - kMagicBits;
    const float rem = fmaf(-c, s, wf[i]);  // exact: w - c s
    const float ar = fabsf(rem);
    const int step = ((rem > 0.f) == s_pos) ? 1 : -1;
    if (ar > half || (ar == half && (ci & 1))) ci += step;  // past half-way, or a tie to the even one
    q[i] = s != 0.f ? min(max(ci, lo), hi) : 0;
  }
  const long long base = n * K + 32 * g + 8 * part;
  if (bits == 8) {
    uint32_t lo4 = 0, hi4 = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      lo4 |= static_cast<uint32_t>(q[i] & 0xFF) << (8 * i);
      hi4 |= static_cast<uint32_t>(q[4 + i] & 0xFF) << (8 * i);
    }
    *reinterpret_cast<uint2*>(q_out + base) = make_uint2(lo4, hi4);
  } else {
    uint32_t nib = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) nib |= static_cast<uint32_t>(q[i] & 0xF) << (4 * i);
    *reinterpret_cast<uint32_t*>(q_out + base / 2) = nib;
  }
}

// Grid (ceil(4 G / 256), rows): thread t of the x dimension handles part
// t % 4 of group t / 4 of rows blockIdx.y, blockIdx.y + gridDim.y, ...; the
// loads of kQuantGroupsPerLane rows are issued together.  (32-bit index math:
// a 64-bit division per group would cost more than the quantisation.)
__global__ void quantize_kernel(int bits, int mode, int lo, int hi, float qmax, const uint16_t* __restrict__ w,
                                long long N, long long K, uint8_t* __restrict__ q_out, uint16_t* __restrict__ s_out) {
  const int G = static_cast<int>(K / 32);
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int g = t >> 2, part = t & 3;
  const bool in_row = g < G;
  for (long long n0 = blockIdx.y; n0 < N; n0 += static_cast<long long>(gridDim.y) * kQuantGroupsPerLane) {
    uint4 v[kQuantGroupsPerLane];
#pragma unroll
    for (int j = 0; j < kQuantGroupsPerLane; ++j) {
      const long long n = n0 + static_cast<long long>(j) * gridDim.y;
      v[j] = make_uint4(0, 0, 0, 0);
      if (in_row && n < N) v[j] = __ldcs(reinterpret_cast<const uint4*>(w + n * K + 32 * g + 8 * part));
    }
#pragma unroll
    for (int j = 0; j < kQuantGroupsPerLane; ++j) {
      const long long n = n0 + static_cast<long long>(j) * gridDim.y;
      if (n >= N) break;  // the same for the whole block
      quantize_part(bits, mode, lo, hi, qmax, v[j], in_row, part, n, g, G, K, q_out, s_out);
    }
  }
}

}  // namespace

extern "C" Q4_API int q4_quantize(int bits, int mode, const uint16_t* w_bf16, int64_t N, int64_t K, void* canon_q_out,
                                  uint16_t* scales_out) {
  QRange r;
  int rc = check(bits, mode, w_bf16, N, K, canon_q_out, scales_out, "q4_quantize", &r);
  if (rc) return rc;
  const int64_t G = K / 32;
  const int64_t row_bytes = bits == 4 ? K / 2 : K;
#pragma omp parallel for schedule(static)
  for (int64_t n = 0; n < N; ++n) {
    uint8_t* qrow = static_cast<uint8_t*>(canon_q_out) + n * row_bytes;
    for (int64_t g = 0; g < G; ++g)
      quantize_group_host(bits, mode, r, w_bf16 + n * K + 32 * g, qrow, 32 * g, scales_out + n * G + g);
  }
  return Q4_OK;
}

extern "C" Q4_API int q4_quantize_device(int bits, int mode, const uint16_t* w_bf16, int64_t N, int64_t K,
                                         void* canon_q_out, uint16_t* scales_out, void* stream) {
  QRange r;
  int rc = check(bits, mode, w_bf16, N, K, canon_q_out, scales_out, "q4_quantize_device", &r);
  if (rc) return rc;
  const long long groups = N * (K / 32);
  if (groups == 0) return Q4_OK;
  if (reinterpret_cast<uintptr_t>(w_bf16) % 16 || reinterpret_cast<uintptr_t>(canon_q_out) % 8)
    return qfail(Q4_ERR_ALIGN, "q4_quantize_device: weights must be 16-byte and codes 8-byte aligned");
  const int threads = 128;
  const long long G = K / 32;
  const long long passes = (N + kQuantGroupsPerLane - 1) / kQuantGroupsPerLane;  // rows handled together
  const dim3 grid(static_cast<unsigned>((4 * G + threads - 1) / threads),
                  static_cast<unsigned>(passes < 65535 ? passes : 65535));
  quantize_kernel<<<grid, threads, 0, static_cast<cudaStream_t>(stream)>>>(
      bits, mode, r.lo, r.hi, r.qmax, w_bf16, N, K, static_cast<uint8_t*>(canon_q_out), scales_out);
  const cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess)
    return qfail(Q4_ERR_CUDA, std::string("q4_quantize_device: launch: ") + cudaGetErrorString(err));
  return Q4_OK;
}
