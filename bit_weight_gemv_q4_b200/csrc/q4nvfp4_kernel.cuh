// NVFP4 weights on the tensor-core path: FP4 E2M1 codes, one FP8 E4M3 scale
// per 16 values along K, one fp32 scale t per tensor,
//     w[n][k] = t * e4m3(s[n][k / 16]) * e2m1(c[n][k]).
// Blackwell converts a byte of two E2M1 codes, and a pair of E4M3 bytes, to an
// fp16 pair in one instruction each.  The product e2m1 * e4m3 has at most six
// significant bits and lies in [2^-10, 2688], so it is EXACT in fp16 (and in
// bf16): the decoded weight s * c, times an fp16 activation, is an exact
// product on the fp16 tensor-core path, accumulated in fp32 over the whole
// tile; t (and the activations' power-of-two scale) multiply the tile's sums
// once, at the end.
//
// Packed chunk (32 rows x 64 columns, 1152 bytes; the q4 chunk's geometry):
// bytes 512h + 16L + 4j + r (L = 4gi + ti, j = 2G + e) hold the two codes of
// tensor-core A register r of product e of group G for lane L: row
// 16h + gi + 8 (r & 1), columns 32G + 8ti + 4e + 2 (r >> 1) + {0, 1} (low
// nibble the lower column).  These are the columns of the q4 format's nibbles
// for the same register, so both formats use the same activation fragments.
// Bytes 1024 + 8 (2gi + b) + 4h + 2G + up hold the E4M3 scale of row
// 16h + gi + 8up, block 4c + 2G + b.  The 16 bytes after the last chunk hold t.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "q4gemv_kernels.cuh"

namespace q4k {

constexpr int kFmtNvfp4 = 16;           // format id of NVFP4 entries (the entry's `bits` field)
constexpr int kNvfp4TrailerBytes = 16;  // the tensor scale, after the chunks

// The four E2M1 pairs of a word -> four fp16 pairs: d[i] from byte i (low
// nibble -> low half).  The word is split into byte registers by one vector
// move, so the conversions read the bytes in place (no shifts).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t (&d)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
      : "r"(w));
}

// The two E4M3 pairs of a word -> two fp16 pairs: lo from bytes 0, 1, hi
// from bytes 2, 3 (the lower byte -> the low half).
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t& lo, uint32_t& hi) {
  asm("{\n\t.reg .b16 h0, h1;\n\t"
      "mov.b32 {h0, h1}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, h0;\n\t"
      "cvt.rn.f16x2.e4m3x2 %1, h1;\n\t}"
      : "=r"(lo), "=r"(hi)
      : "r"(w));
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, 0, %2;" : "=r"(d) : "r"(a), "r"(sel));
  return d;
}

// fp16 pair -> bf16 pair, for values exact in both (the bf16 fallback).
__device__ __forceinline__ uint32_t f16x2_to_bf16x2(uint32_t h2) {
  const float2 f = half2_bits_to_float2(h2);
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(f.y), "f"(f.x));
  return d;
}

// One chunk's contribution to this lane's accumulators, accumulated by the
// tensor cores themselves (no per-group scaling: the block scales are folded
// into the exact fp16 weights).  codes: this lane's 16 bytes of each half;
// sc: its 8 scale bytes (byte 4h + 2G + up).  F16: fp16 activations, else bf16
// (the weights are then converted to bf16, still exactly).
template <bool F16>
__device__ __forceinline__ void nvfp4_chunk_mac(float (&acc)[2][4], const uint4 (&codes)[2], uint2 sc,
                                                const uint4& xa, const uint4& xb) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4& w = codes[h];
    uint32_t s2[2];  // per group G: (row 16h + gi, row 16h + gi + 8)
    e4m3x4_to_f16x2(h ? sc.y : sc.x, s2[0], s2[1]);
#pragma unroll
    for (int G = 0; G < 2; ++G) {
      const uint32_t s_r = byte_perm(s2[G], 0x1010u), s_r8 = byte_perm(s2[G], 0x3232u);
      const uint4& xg = G ? xb : xa;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const uint32_t word = G ? (e ? w.w : w.z) : (e ? w.y : w.x);
        uint32_t a[4];
        e2m1x8_to_f16x2(word, a);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          a[r] = f16x2_mul(a[r], (r & 1) ? s_r8 : s_r);
          if constexpr (!F16) a[r] = f16x2_to_bf16x2(a[r]);
        }
        mma_m16n8k16<F16>(acc[h], a, e ? xg.z : xg.x, e ? xg.w : xg.y);
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Device repack: canonical codes [N][K/2] and E4M3 scales [N][K/16] -> packed
// chunks, one thread per 16-byte code slot (the host packer's placement).
// Thread 0 also writes the trailer.
// ----------------------------------------------------------------------------
__global__ void pack_nvfp4_kernel(const uint8_t* codes, const uint8_t* scales, float tscale, long long N,
                                  long long K, int T, int C, uint8_t* out) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long TC = static_cast<long long>(T) * C;
  if (idx == 0) {
    *reinterpret_cast<uint4*>(out + TC * Format<4>::kChunkBytes) = make_uint4(__float_as_uint(tscale), 0u, 0u, 0u);
  }
  if (idx >= TC * 64) return;
  const long long chunk = idx >> 6;
  const int h = static_cast<int>((idx >> 5) & 1);
  const int slot = static_cast<int>(idx & 31);
  const int gi = slot >> 2, ti = slot & 3;
  const long long t = chunk / C, c = chunk % C;
  uint32_t w[4];
  for (int j = 0; j < 4; ++j) {
    uint32_t word = 0;
    for (int r = 0; r < 4; ++r) {
      const long long row = t * kTileRows + 16 * h + gi + 8 * (r & 1);
      const long long col = 64 * c + 32 * (j >> 1) + 8 * ti + 4 * (j & 1) + 2 * (r >> 1);
      const uint32_t b = row < N ? codes[row * (K / 2) + col / 2] : 0u;
      word |= b << (8 * r);
    }
    w[j] = word;
  }
  uint8_t* dst = out + chunk * Format<4>::kChunkBytes;
  *reinterpret_cast<uint4*>(dst + kHalfBytes * h + 16 * slot) = make_uint4(w[0], w[1], w[2], w[3]);
  if (h == 0 && (ti & 1) == 0) {  // one thread per (gi, b): 8 scale bytes
    const int b = ti >> 1;
    const long long B = K / 16;
    uint32_t s[2] = {0u, 0u};
    for (int hh = 0; hh < 2; ++hh)
      for (int G = 0; G < 2; ++G)
        for (int up = 0; up < 2; ++up) {
          const long long row = t * kTileRows + 16 * hh + gi + 8 * up;
          const uint32_t v = row < N ? scales[row * B + 4 * c + 2 * G + b] : 0u;
          s[hh] |= v << (8 * (2 * G + up));
        }
    *reinterpret_cast<uint2*>(dst + kCodeBytes + 8 * (2 * gi + b)) = make_uint2(s[0], s[1]);
  }
}

// ----------------------------------------------------------------------------
// Device decode, for checking the in-register conversion: the weights the
// product kernel multiplies, w / t = e4m3 * e2m1 as the fp16 product the
// tensor cores see, widened to fp32 (exact), times t in fp32 (one rounding of
// the exact product), written to w_out [N][K].  One thread per 16-byte code
// slot, through the same register decode as nvfp4_chunk_mac.
// ----------------------------------------------------------------------------
__global__ void dequant_nvfp4_kernel(const uint8_t* packed, long long N, long long K, int T, int C, float* w_out) {
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long TC = static_cast<long long>(T) * C;
  if (idx >= TC * 64) return;
  const float t = *reinterpret_cast<const float*>(packed + TC * Format<4>::kChunkBytes);
  const long long chunk = idx >> 6;
  const int h = static_cast<int>((idx >> 5) & 1);
  const int slot = static_cast<int>(idx & 31);
  const int gi = slot >> 2, ti = slot & 3;
  const long long tt = chunk / C, c = chunk % C;
  const uint8_t* src = packed + chunk * Format<4>::kChunkBytes;
  const uint4 w = *reinterpret_cast<const uint4*>(src + kHalfBytes * h + 16 * slot);
  const uint2 sc = *reinterpret_cast<const uint2*>(src + kCodeBytes + 8 * (2 * gi + (ti >> 1)));
  uint32_t s2[2];
  e4m3x4_to_f16x2(h ? sc.y : sc.x, s2[0], s2[1]);
  for (int j = 0; j < 4; ++j) {
    const int G = j >> 1, e = j & 1;
    const uint32_t word = j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w;
    uint32_t c2[4];
    e2m1x8_to_f16x2(word, c2);
    for (int r = 0; r < 4; ++r) {
      const uint32_t sel = (r & 1) ? byte_perm(s2[G], 0x3232u) : byte_perm(s2[G], 0x1010u);
      const float2 v = half2_bits_to_float2(f16x2_mul(c2[r], sel));
      const long long row = tt * kTileRows + 16 * h + gi + 8 * (r & 1);
      const long long col = 64 * c + 32 * G + 8 * ti + 4 * e + 2 * (r >> 1);
      if (row < N) {
        w_out[row * K + col] = v.x * t;
        w_out[row * K + col + 1] = v.y * t;
      }
    }
  }
}

}  // namespace q4k
