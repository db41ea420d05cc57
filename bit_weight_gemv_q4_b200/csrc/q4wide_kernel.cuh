// q5 / q6 weights (symmetric, group 32, fp16 scales): the widths between q4
// and q8 that a mixed-precision recipe gives its sensitive tensors (the
// bs178.com llamAmpere post's "smarter bits", part two, upgrades some tensors
// to 5 and 6 bits).  The chunk is the q4 chunk (32 rows x 64 columns) with a
// plane of high bits after the low nibbles (layout in include/q4gemv.h):
// u = q + 16 (q5) or q + 32 (q6), low nibble u & 15 where q4 keeps its
// nibble, high bits u >> 4 in one 32-bit word per lane and half (q5) or two
// (q6), at positions chosen so that one shift of the word brings the high
// bits of a register pair to the mantissa bits the decode needs.
//
// Decode (exact): a register whose nibble sits at bits 0-3 of each half
// becomes the fp16 1024 + lo + 16 hi = 1024 + u, minus (1024 + offset) = q; one
// whose nibble sits at bits 4-7 becomes 1024 + 16 lo + 256 hi = 1024 + 16 u,
// then u - offset by one fp16 FMA (x 1/16 - (64 + offset)).  Every value is an
// integer below 2048, so fp16 holds it exactly.  The bf16 path (activations
// not fp16-exact) uses 128 + u.
#pragma once

#include <stdint.h>

#include "q4gemv_kernels.cuh"

namespace q4k {

template <int BITS>
struct Wide {
  static_assert(BITS == 5 || BITS == 6, "q5 or q6");
  static constexpr int kOffset = BITS == 5 ? 16 : 32;              // u = q + kOffset
  static constexpr int kHiBytes = BITS == 5 ? 256 : 512;           // the high-bit plane
  static constexpr int kScaleBase = kCodeBytes + kHiBytes;         // scales, q4 placement
  static constexpr int kChunkBytes = kScaleBase + 128;             // 1408 / 1664
  static constexpr uint32_t kMaskEven = BITS == 5 ? 0x00100010u : 0x00300030u;  // high bits at 4 (+1)
  static constexpr uint32_t kMaskOdd = BITS == 5 ? 0x01000100u : 0x03000300u;   // high bits at 8 (+1)
};

// Shift of the high-bit word that lines up register pair p (registers 2p and
// 2p + 1) of code word j: negative = left.
template <int BITS>
__host__ __device__ constexpr int wide_shift(int j, int p) {
  return BITS == 5 ? (j < 2 ? -4 + 2 * j + p : 4 + 2 * (j - 2) + p) : ((j & 1) ? 4 + 2 * p : -4 + 2 * p);
}

template <int S>
__device__ __forceinline__ uint32_t shift_by(uint32_t v) {
  if constexpr (S < 0)
    return v << (-S);
  else
    return v >> S;
}

// x | (y & m)
__device__ __forceinline__ uint32_t lop3_or_and(uint32_t x, uint32_t y, uint32_t m) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xF8;" : "=r"(d) : "r"(x), "r"(y), "r"(m));
  return d;
}

// fp16 pair constants of the decode
template <int BITS>
struct WideF16 {
  static constexpr uint32_t pair(uint32_t h) { return h | (h << 16); }
  // 1024 + offset: 0x6410 (1040) / 0x6420 (1056)
  static constexpr uint32_t kSubEven = pair(BITS == 5 ? 0x6410u : 0x6420u);
  // -(64 + offset): -80 = 0xD500, -96 = 0xD600
  static constexpr uint32_t kAddOdd = pair(BITS == 5 ? 0xD500u : 0xD600u);
};

// Code word w (code word j of the lane's half) and its two lined-up high-bit
// words hs0 (registers 0, 1) and hs1 (registers 2, 3) -> the four fp16 A
// registers holding q exactly.
template <int BITS>
__device__ __forceinline__ void dequant_wide_word_f16(uint32_t w, uint32_t hs0, uint32_t hs1, uint32_t (&a)[4]) {
  const uint32_t t = w >> 8;
  a[0] = f16x2_sub(lop3_or_and(lop3_and_or(w, kNibbleMask, kF16_1024), hs0, Wide<BITS>::kMaskEven),
                   WideF16<BITS>::kSubEven);
  a[1] = f16x2_fma(lop3_or_and(lop3_and_or(w, kNibbleMaskHi, kF16_1024), hs0, Wide<BITS>::kMaskOdd), kF16_1_16,
                   WideF16<BITS>::kAddOdd);
  a[2] = f16x2_sub(lop3_or_and(lop3_and_or(t, kNibbleMask, kF16_1024), hs1, Wide<BITS>::kMaskEven),
                   WideF16<BITS>::kSubEven);
  a[3] = f16x2_fma(lop3_or_and(lop3_and_or(t, kNibbleMaskHi, kF16_1024), hs1, Wide<BITS>::kMaskOdd), kF16_1_16,
                   WideF16<BITS>::kAddOdd);
}

// The same in bf16: every register's nibble brought to bits 0-3, its high
// bits to bit 4 (+1): 128 + u, minus (128 + offset).
template <int BITS>
__device__ __forceinline__ void dequant_wide_word_bf16(uint32_t w, uint32_t hs0, uint32_t hs1, uint32_t (&a)[4]) {
  constexpr uint32_t sub = (BITS == 5 ? 0x4310u : 0x4320u) * 0x10001u;  // bf16 pair 144 / 160
  a[0] = bf16x2_sub(lop3_or_and(lop3_and_or(w, kNibbleMask, kBf16_128), hs0, Wide<BITS>::kMaskEven), sub);
  a[1] = bf16x2_sub(lop3_or_and(lop3_and_or(w >> 4, kNibbleMask, kBf16_128), hs0 >> 4, Wide<BITS>::kMaskEven), sub);
  a[2] = bf16x2_sub(lop3_or_and(lop3_and_or(w >> 8, kNibbleMask, kBf16_128), hs1, Wide<BITS>::kMaskEven), sub);
  a[3] = bf16x2_sub(lop3_or_and(lop3_and_or(w >> 12, kNibbleMask, kBf16_128), hs1 >> 4, Wide<BITS>::kMaskEven), sub);
}

// The lined-up high-bit words of code word j (0..3) of half h: hi holds the
// lane's high-bit words (q5: .x = half 0, .y = half 1; q6: .x, .y = half 0,
// .z, .w = half 1, the second word of each for code words 2, 3).
template <int BITS, int H, int J>
__device__ __forceinline__ void wide_hi_words(const uint4& hi, uint32_t& hs0, uint32_t& hs1) {
  uint32_t word;
  if constexpr (BITS == 5)
    word = H ? hi.y : hi.x;
  else
    word = H ? (J >= 2 ? hi.w : hi.z) : (J >= 2 ? hi.y : hi.x);
  hs0 = shift_by<wide_shift<BITS>(J, 0)>(word);
  hs1 = shift_by<wide_shift<BITS>(J, 1)>(word);
}

template <int BITS, bool F16, int H, int J>
__device__ __forceinline__ void wide_registers(const uint4& w, const uint4& hi, uint32_t (&a)[4]) {
  uint32_t hs0, hs1;
  wide_hi_words<BITS, H, J>(hi, hs0, hs1);
  const uint32_t word = J == 0 ? w.x : J == 1 ? w.y : J == 2 ? w.z : w.w;
  if constexpr (F16)
    dequant_wide_word_f16<BITS>(word, hs0, hs1, a);
  else
    dequant_wide_word_bf16<BITS>(word, hs0, hs1, a);
}

// One q5 / q6 chunk's contribution to this lane's accumulators: as the q4
// chunk (two groups, per-group fp32 scale FMA), with the high bits merged
// into each register.  codes: the lane's 16 bytes of each half; hi: its
// high-bit words; scales: its 16 scale bytes (q4 placement).
template <int BITS, bool F16>
__device__ __forceinline__ void wide_chunk_mac(float (&acc)[2][4], const uint4 (&codes)[2], const uint4& hi,
                                               const uint4& scales, const uint4& xa, const uint4& xb) {
  const uint32_t sc[4] = {scales.x, scales.y, scales.z, scales.w};
#pragma unroll
  for (int G = 0; G < 2; ++G) {
    const uint4& xg = G ? xb : xa;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      float d[4];
      uint32_t a[4];
      if (h == 0) {
        if (G == 0) wide_registers<BITS, F16, 0, 0>(codes[0], hi, a); else wide_registers<BITS, F16, 0, 2>(codes[0], hi, a);
      } else {
        if (G == 0) wide_registers<BITS, F16, 1, 0>(codes[1], hi, a); else wide_registers<BITS, F16, 1, 2>(codes[1], hi, a);
      }
      mma_m16n8k16_first<F16>(d, a, xg.x, xg.y);
      if (h == 0) {
        if (G == 0) wide_registers<BITS, F16, 0, 1>(codes[0], hi, a); else wide_registers<BITS, F16, 0, 3>(codes[0], hi, a);
      } else {
        if (G == 0) wide_registers<BITS, F16, 1, 1>(codes[1], hi, a); else wide_registers<BITS, F16, 1, 3>(codes[1], hi, a);
      }
      mma_m16n8k16<F16>(d, a, xg.z, xg.w);
      const float2 s_r = half2_bits_to_float2(sc[2 * h]);       // row 16h + gi: groups 2c, 2c+1
      const float2 s_r8 = half2_bits_to_float2(sc[2 * h + 1]);  // row 16h + gi + 8
      const float sr = G ? s_r.y : s_r.x;
      const float sr8 = G ? s_r8.y : s_r8.x;
      acc[h][0] = fmaf(sr, d[0], acc[h][0]);
      acc[h][1] = fmaf(sr, d[1], acc[h][1]);
      acc[h][2] = fmaf(sr8, d[2], acc[h][2]);
      acc[h][3] = fmaf(sr8, d[3], acc[h][3]);
    }
  }
}

// The lane's high-bit words of a chunk in shared memory (q5: 8 bytes, q6: 16).
template <int BITS>
__device__ __forceinline__ uint4 wide_load_hi(uint32_t chunk, int lane) {
  if constexpr (BITS == 5) {
    const uint2 v = lds64(chunk + kCodeBytes + 8 * lane);
    return make_uint4(v.x, v.y, 0u, 0u);
  } else {
    return lds128(chunk + kCodeBytes + 16 * lane);
  }
}

// ----------------------------------------------------------------------------
// Device repack of q5 / q6 (canonical int8 [N][K], K % 64 == 0): one thread
// per 16-byte code slot writes the slot's low nibbles and its word(s) of high
// bits; thread (h = 0, ti even) writes the scale entries, as for q4.  Codes
// outside the width's range are packed modulo 2^BITS.
// ----------------------------------------------------------------------------
template <int BITS>
__global__ void pack_wide_kernel(const int8_t* q, const uint16_t* s, long long N, long long K, int T, int C,
                                 uint8_t* out) {
  constexpr int CB = Wide<BITS>::kChunkBytes;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * C * 64) return;
  const long long chunk = idx >> 6;
  const int h = static_cast<int>((idx >> 5) & 1);
  const int lane = static_cast<int>(idx & 31);
  const int gi = lane >> 2, ti = lane & 3;
  const long long t = chunk / C, c = chunk % C;
  uint32_t w[4] = {0u, 0u, 0u, 0u}, hw[2] = {0u, 0u};
  for (int j = 0; j < 4; ++j)
    for (int i = 0; i < 8; ++i) {
      const long long row = t * kTileRows + 16 * h + gi + 8 * (i & 1);
      const long long col = 64 * c + 32 * (j >> 1) + 8 * ti + 4 * (j & 1) + 2 * ((i >> 1) & 1) + (i >> 2);
      const int u = ((row < N ? q[row * K + col] : 0) + Wide<BITS>::kOffset) & ((1 << BITS) - 1);
      w[j] |= static_cast<uint32_t>(u & 15) << (4 * i);
      const int r = i & 3, e = i >> 2;
      const int pos = 16 * e + wide_shift<BITS>(j, r >> 1) + ((r & 1) ? 8 : 4);
      hw[BITS == 5 ? 0 : (j >> 1)] |= static_cast<uint32_t>(u >> 4) << pos;
    }
  uint8_t* dst = out + chunk * CB;
  *reinterpret_cast<uint4*>(dst + kHalfBytes * h + 16 * lane) = make_uint4(w[0], w[1], w[2], w[3]);
  if (BITS == 5)
    *reinterpret_cast<uint32_t*>(dst + kCodeBytes + 8 * lane + 4 * h) = hw[0];
  else
    *reinterpret_cast<uint2*>(dst + kCodeBytes + 16 * lane + 8 * h) = make_uint2(hw[0], hw[1]);
  if (h == 0 && ti == 0) {
    const long long G = K / 32;
    uint16_t v[8];
    for (int hh = 0; hh < 2; ++hh)
      for (int up = 0; up < 2; ++up)
        for (int g = 0; g < 2; ++g) {
          const long long row = t * kTileRows + 16 * hh + gi + 8 * up;
          v[4 * hh + 2 * up + g] = row < N ? s[row * G + 2 * c + g] : 0;
        }
    *reinterpret_cast<uint4*>(dst + Wide<BITS>::kScaleBase + 16 * gi) =
        make_uint4(v[0] | (static_cast<uint32_t>(v[1]) << 16), v[2] | (static_cast<uint32_t>(v[3]) << 16),
                   v[4] | (static_cast<uint32_t>(v[5]) << 16), v[6] | (static_cast<uint32_t>(v[7]) << 16));
  }
}

// Debug decoder: q through both register decodes (fp16 and bf16), written
// where they agree, -128 where they do not; scales copied.  One warp per chunk.
template <int BITS>
__global__ void unpack_wide_kernel(const uint8_t* packed, long long N, long long K, int T, int C, int8_t* q_out,
                                   uint16_t* s_out) {
  constexpr int CB = Wide<BITS>::kChunkBytes;
  const long long chunk = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (chunk >= static_cast<long long>(T) * C) return;
  const int lane = threadIdx.x & 31, gi = lane >> 2, ti = lane & 3;
  const long long t = chunk / C, c = chunk % C;
  const uint8_t* src = packed + chunk * CB;
  uint4 hi;
  if (BITS == 5) {
    const uint2 v = *reinterpret_cast<const uint2*>(src + kCodeBytes + 8 * lane);
    hi = make_uint4(v.x, v.y, 0u, 0u);
  } else {
    hi = *reinterpret_cast<const uint4*>(src + kCodeBytes + 16 * lane);
  }
  uint4 codes[2];
  codes[0] = *reinterpret_cast<const uint4*>(src + 16 * lane);
  codes[1] = *reinterpret_cast<const uint4*>(src + kHalfBytes + 16 * lane);
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      uint32_t af[4], ab[4];
      if (h == 0) {
        if (j == 0) { wide_registers<BITS, true, 0, 0>(codes[0], hi, af); wide_registers<BITS, false, 0, 0>(codes[0], hi, ab); }
        if (j == 1) { wide_registers<BITS, true, 0, 1>(codes[0], hi, af); wide_registers<BITS, false, 0, 1>(codes[0], hi, ab); }
        if (j == 2) { wide_registers<BITS, true, 0, 2>(codes[0], hi, af); wide_registers<BITS, false, 0, 2>(codes[0], hi, ab); }
        if (j == 3) { wide_registers<BITS, true, 0, 3>(codes[0], hi, af); wide_registers<BITS, false, 0, 3>(codes[0], hi, ab); }
      } else {
        if (j == 0) { wide_registers<BITS, true, 1, 0>(codes[1], hi, af); wide_registers<BITS, false, 1, 0>(codes[1], hi, ab); }
        if (j == 1) { wide_registers<BITS, true, 1, 1>(codes[1], hi, af); wide_registers<BITS, false, 1, 1>(codes[1], hi, ab); }
        if (j == 2) { wide_registers<BITS, true, 1, 2>(codes[1], hi, af); wide_registers<BITS, false, 1, 2>(codes[1], hi, ab); }
        if (j == 3) { wide_registers<BITS, true, 1, 3>(codes[1], hi, af); wide_registers<BITS, false, 1, 3>(codes[1], hi, ab); }
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int vf = f16_bits_to_int(static_cast<uint16_t>(af[r] >> (16 * e)));
          const int vb = static_cast<int>(__uint_as_float((ab[r] >> (16 * e)) << 16));
          const int i = r + 4 * e;
          const long long row = t * kTileRows + 16 * h + gi + 8 * (i & 1);
          const long long col = 64 * c + 32 * (j >> 1) + 8 * ti + 4 * (j & 1) + 2 * ((i >> 1) & 1) + (i >> 2);
          if (row < N) q_out[row * K + col] = static_cast<int8_t>(vf == vb ? vf : -128);
        }
    }
  if (ti == 0) {
    const long long G = K / 32;
    for (int hh = 0; hh < 2; ++hh)
      for (int up = 0; up < 2; ++up)
        for (int g = 0; g < 2; ++g) {
          const long long row = t * kTileRows + 16 * hh + gi + 8 * up;
          if (row < N)
            s_out[row * G + 2 * c + g] =
                *reinterpret_cast<const uint16_t*>(src + Wide<BITS>::kScaleBase + 16 * gi + 2 * (4 * hh + 2 * up + g));
        }
  }
}

}  // namespace q4k
