// Offline repack of canonical group-quantised weights into the kernel-native
// chunk layout, and its exact inverse.  Host code, run once per tensor (the
// weights of a decode model are packed when they are loaded, not per token).
//
// The layout itself is specified in include/q4gemv.h; in short, the tensor is a
// sequence of 32-row x (64 or 32)-column chunks in memory order (tile, chunk),
// each chunk holding the tensor-core A fragments of one warp for its two
// 16-row halves, followed by the fp16 scales of its groups.  Streaming a tile
// is streaming one contiguous run.
#include <cstdint>
#include <cstring>
#include <string>

#include "q4gemv.h"

namespace q4 {
void set_error(const std::string& msg);
}  // namespace q4

namespace {

constexpr int kTileRows = 32;

struct Geometry {
  int bits;
  int64_t N, K, T, C, chunk_bytes, k_per_chunk;
};

bool geometry(int bits, int64_t N, int64_t K, Geometry* g) {
  if ((bits < 4 || bits > 6) && bits != 8) return false;
  if (N < 0 || K < 0 || K % 32 != 0 || ((bits == 5 || bits == 6) && K % 64 != 0)) return false;
  // keep every offset and index comfortably inside int64 / int32 tile counts
  if (N > (int64_t(1) << 34) || K > (int64_t(1) << 30)) return false;
  g->bits = bits;
  g->N = N;
  g->K = K;
  g->T = (N + kTileRows - 1) / kTileRows;
  g->k_per_chunk = bits == 8 ? 32 : 64;
  g->C = (K + g->k_per_chunk - 1) / g->k_per_chunk;
  g->chunk_bytes = bits == 4 ? 1152 : bits == 5 ? 1408 : bits == 6 ? 1664 : 1088;
  return true;
}

// q5 / q6: the q4 chunk's code blocks hold the low nibble of u = q + 16 (q5)
// or q + 32 (q6); the high bits of lane L sit in a plane after them (q5: 8
// bytes at 1024 + 8L, word h; q6: 16 bytes at 1024 + 16L, word 2h + (j >> 1)),
// at the positions below, then the scales (q4 placement) at 1024 + 256 (q5)
// or 1024 + 512 (q6).  Nibble i of code word j belongs to tensor-core register
// r = i & 3, half-word el = i >> 2.
constexpr int kWideShift5[8] = {-4, -3, -2, -1, 4, 5, 6, 7};  // by 2j + (r >> 1)
constexpr int kWideShift6[4] = {-4, -2, 4, 6};                 // by 2 (j & 1) + (r >> 1)

inline int wide_hi_pos(int bits, int j, int i) {
  const int r = i & 3, el = i >> 2;
  const int target = (r & 1) ? 8 : 4;
  const int sh = bits == 5 ? kWideShift5[2 * j + (r >> 1)] : kWideShift6[2 * (j & 1) + (r >> 1)];
  return 16 * el + sh + target;
}

inline int64_t wide_hi_offset(int bits, int h, int lane, int j) {
  return bits == 5 ? 1024 + 8 * lane + 4 * h : 1024 + 16 * lane + 8 * h + 4 * (j >> 1);
}

inline int64_t wide_scale_base(int bits) { return bits == 5 ? 1024 + 256 : 1024 + 512; }

// Row and column of nibble i of word j in slot (gi, ti) of half h of q4
// chunk (t, c).
inline void q4_coord(int64_t t, int64_t c, int h, int gi, int ti, int j, int i, int64_t* row, int64_t* col) {
  const int G = j >> 1, e = j & 1;
  *row = kTileRows * t + 16 * h + gi + 8 * (i & 1);
  *col = 64 * c + 32 * G + 8 * ti + 4 * e + 2 * ((i >> 1) & 1) + (i >> 2);
}

// Row and column of byte b of word j in slot (gi, ti) of half h of q8 chunk (t, c).
inline void q8_coord(int64_t t, int64_t c, int h, int gi, int ti, int j, int b, int64_t* row, int64_t* col) {
  const int e = j >> 1, f = j & 1;
  *row = kTileRows * t + 16 * h + gi + 8 * (b & 1);
  *col = 32 * c + 8 * ti + 4 * e + 2 * f + (b >> 1);
}

// Row of scale slot (h, up) of entry gi in tile t: 16h + gi + 8up.
inline int64_t scale_row(int64_t t, int h, int gi, int up) { return kTileRows * t + 16 * h + gi + 8 * up; }

inline int canon_q4(const uint8_t* q, int64_t K, int64_t row, int64_t col) {
  const uint8_t byte = q[row * (K / 2) + col / 2];
  const int nib = (col & 1) ? (byte >> 4) : (byte & 0xF);
  return nib >= 8 ? nib - 16 : nib;
}

inline uint32_t load32(const uint8_t* p) {
  uint32_t v;
  std::memcpy(&v, p, 4);
  return v;
}

inline void store32(uint8_t* p, uint32_t v) { std::memcpy(p, &v, 4); }

// q5 / q6 codes (canonical int8 [N][K], q in [-16, 15] or [-32, 31]) into
// the packed chunks (K % 64 == 0; see wide_hi_pos).
void pack_wide(const Geometry& g, const int8_t* q, const uint16_t* scales, uint8_t* dst) {
  const int bits = g.bits, off = bits == 5 ? 16 : 32;
  const int64_t hi_bytes = bits == 5 ? 256 : 512, sbase = wide_scale_base(bits), G = g.K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < g.T; ++t) {
    for (int64_t c = 0; c < g.C; ++c) {
      uint8_t* chunk = dst + (t * g.C + c) * g.chunk_bytes;
      std::memset(chunk + 1024, 0, hi_bytes);
      for (int h = 0; h < 2; ++h)
        for (int gi = 0; gi < 8; ++gi)
          for (int ti = 0; ti < 4; ++ti) {
            const int lane = 4 * gi + ti;
            uint32_t words[4] = {0, 0, 0, 0};
            for (int j = 0; j < 4; ++j)
              for (int i = 0; i < 8; ++i) {
                int64_t row, col;
                q4_coord(t, c, h, gi, ti, j, i, &row, &col);
                const int u = (row < g.N ? q[row * g.K + col] : 0) + off;
                words[j] |= static_cast<uint32_t>(u & 15) << (4 * i);
                uint8_t* hp = chunk + wide_hi_offset(bits, h, lane, j);
                store32(hp, load32(hp) | (static_cast<uint32_t>(u >> 4) << wide_hi_pos(bits, j, i)));
              }
            std::memcpy(chunk + 512 * h + 16 * lane, words, 16);
          }
      for (int gi = 0; gi < 8; ++gi) {
        uint16_t s8[8];
        for (int h = 0; h < 2; ++h)
          for (int up = 0; up < 2; ++up)
            for (int gg = 0; gg < 2; ++gg) {
              const int64_t row = scale_row(t, h, gi, up), grp = 2 * c + gg;
              s8[4 * h + 2 * up + gg] = row < g.N ? scales[row * G + grp] : 0;
            }
        std::memcpy(chunk + sbase + 16 * gi, s8, 16);
      }
    }
  }
}

void unpack_wide(const Geometry& g, const uint8_t* src, int8_t* q, uint16_t* scales) {
  const int bits = g.bits, off = bits == 5 ? 16 : 32;
  const int64_t sbase = wide_scale_base(bits), G = g.K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < g.T; ++t) {
    for (int64_t c = 0; c < g.C; ++c) {
      const uint8_t* chunk = src + (t * g.C + c) * g.chunk_bytes;
      for (int h = 0; h < 2; ++h)
        for (int gi = 0; gi < 8; ++gi)
          for (int ti = 0; ti < 4; ++ti) {
            const int lane = 4 * gi + ti;
            for (int j = 0; j < 4; ++j) {
              const uint32_t w = load32(chunk + 512 * h + 16 * lane + 4 * j);
              const uint32_t hw = load32(chunk + wide_hi_offset(bits, h, lane, j));
              for (int i = 0; i < 8; ++i) {
                int64_t row, col;
                q4_coord(t, c, h, gi, ti, j, i, &row, &col);
                if (row >= g.N) continue;
                const int hi = static_cast<int>((hw >> wide_hi_pos(bits, j, i)) & (bits == 5 ? 1u : 3u));
                const int u = static_cast<int>((w >> (4 * i)) & 15u) + 16 * hi;
                q[row * g.K + col] = static_cast<int8_t>(u - off);
              }
            }
          }
      for (int gi = 0; gi < 8; ++gi)
        for (int h = 0; h < 2; ++h)
          for (int up = 0; up < 2; ++up)
            for (int gg = 0; gg < 2; ++gg) {
              const int64_t row = scale_row(t, h, gi, up), grp = 2 * c + gg;
              if (row < g.N) {
                uint16_t v;
                std::memcpy(&v, chunk + sbase + 16 * gi + 2 * (4 * h + 2 * up + gg), 2);
                scales[row * G + grp] = v;
              }
            }
    }
  }
}

}  // namespace

extern "C" Q4_API size_t q4_packed_bytes(int bits, int64_t N, int64_t K) {
  Geometry g;
  if (!geometry(bits, N, K, &g)) return 0;
  return static_cast<size_t>(g.T * g.C * g.chunk_bytes);
}

extern "C" Q4_API int q4_pack_weights(int bits, const void* canon_q, const uint16_t* scales, int64_t N, int64_t K,
                                      void* out, size_t out_bytes) {
  Geometry g;
  if (bits != 4 && bits != 5 && bits != 6 && bits != 8) {
    q4::set_error("q4_pack_weights: bits must be 4, 5, 6 or 8");
    return Q4_ERR_INVALID_ARG;
  }
  if (!geometry(bits, N, K, &g)) {
    q4::set_error("q4_pack_weights: need N >= 0, K >= 0, K % 32 == 0 (K % 64 == 0 for 5 and 6 bits; "
                  "sizes below 2^34 x 2^30)");
    return Q4_ERR_SHAPE;
  }
  const size_t need = static_cast<size_t>(g.T * g.C * g.chunk_bytes);
  if (need == 0) return Q4_OK;
  if (!canon_q || !scales || !out) {
    q4::set_error("q4_pack_weights: null pointer");
    return Q4_ERR_INVALID_ARG;
  }
  if (out_bytes < need) {
    q4::set_error("q4_pack_weights: out_bytes " + std::to_string(out_bytes) + " < " + std::to_string(need));
    return Q4_ERR_BUFFER_TOO_SMALL;
  }
  if (bits == 5 || bits == 6) {
    const int8_t* q = static_cast<const int8_t*>(canon_q);
    const int lim = bits == 5 ? 16 : 32;
    for (int64_t e = 0; e < N * K; ++e)
      if (q[e] < -lim || q[e] >= lim) {
        q4::set_error("q4_pack_weights: a code outside [" + std::to_string(-lim) + ", " + std::to_string(lim - 1) +
                      "] for " + std::to_string(bits) + " bits");
        return Q4_ERR_INVALID_ARG;
      }
    pack_wide(g, q, scales, static_cast<uint8_t*>(out));
    return Q4_OK;
  }
  const int64_t G = K / 32;
  uint8_t* dst = static_cast<uint8_t*>(out);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < g.T; ++t) {
    for (int64_t c = 0; c < g.C; ++c) {
      uint8_t* chunk = dst + (t * g.C + c) * g.chunk_bytes;
      for (int h = 0; h < 2; ++h) {
        for (int gi = 0; gi < 8; ++gi) {
          for (int ti = 0; ti < 4; ++ti) {
            uint32_t words[4];
            for (int j = 0; j < 4; ++j) {
              uint32_t w = 0;
              if (bits == 4) {
                for (int i = 0; i < 8; ++i) {
                  int64_t row, col;
                  q4_coord(t, c, h, gi, ti, j, i, &row, &col);
                  int q = 0;
                  if (row < N && col < K) q = canon_q4(static_cast<const uint8_t*>(canon_q), K, row, col);
                  w |= static_cast<uint32_t>(q + 8) << (4 * i);
                }
              } else {
                for (int b = 0; b < 4; ++b) {
                  int64_t row, col;
                  q8_coord(t, c, h, gi, ti, j, b, &row, &col);
                  int q = 0;
                  if (row < N && col < K) q = static_cast<const int8_t*>(canon_q)[row * K + col];
                  w |= static_cast<uint32_t>(q + 128) << (8 * b);
                }
              }
              words[j] = w;
            }
            std::memcpy(chunk + 512 * h + 16 * (4 * gi + ti), words, 16);
          }
        }
      }
      // scales: entry gi lists rows 16h + gi + 8up for h, up in {0, 1}
      for (int gi = 0; gi < 8; ++gi) {
        if (bits == 4) {
          uint16_t s8[8];
          for (int h = 0; h < 2; ++h)
            for (int up = 0; up < 2; ++up)
              for (int gg = 0; gg < 2; ++gg) {
                const int64_t row = scale_row(t, h, gi, up), grp = 2 * c + gg;
                s8[4 * h + 2 * up + gg] = (row < N && grp < G) ? scales[row * G + grp] : 0;
              }
          std::memcpy(chunk + 1024 + 16 * gi, s8, 16);
        } else {
          uint16_t s4[4];
          for (int h = 0; h < 2; ++h)
            for (int up = 0; up < 2; ++up) {
              const int64_t row = scale_row(t, h, gi, up);
              s4[2 * h + up] = row < N ? scales[row * G + c] : 0;
            }
          std::memcpy(chunk + 1024 + 8 * gi, s4, 8);
        }
      }
    }
  }
  return Q4_OK;
}

extern "C" Q4_API int q4_unpack_weights(int bits, const void* packed, size_t packed_bytes, int64_t N, int64_t K,
                                        void* canon_q_out, uint16_t* scales_out) {
  Geometry g;
  if (bits != 4 && bits != 5 && bits != 6 && bits != 8) {
    q4::set_error("q4_unpack_weights: bits must be 4, 5, 6 or 8");
    return Q4_ERR_INVALID_ARG;
  }
  if (!geometry(bits, N, K, &g)) {
    q4::set_error("q4_unpack_weights: need N >= 0, K >= 0, K % 32 == 0");
    return Q4_ERR_SHAPE;
  }
  const size_t need = static_cast<size_t>(g.T * g.C * g.chunk_bytes);
  if (need == 0) return Q4_OK;
  if (!packed || !canon_q_out || !scales_out) {
    q4::set_error("q4_unpack_weights: null pointer");
    return Q4_ERR_INVALID_ARG;
  }
  if (packed_bytes < need) {
    q4::set_error("q4_unpack_weights: packed_bytes too small");
    return Q4_ERR_BUFFER_TOO_SMALL;
  }
  if (bits == 5 || bits == 6) {
    unpack_wide(g, static_cast<const uint8_t*>(packed), static_cast<int8_t*>(canon_q_out), scales_out);
    return Q4_OK;
  }
  const int64_t G = K / 32;
  const uint8_t* src = static_cast<const uint8_t*>(packed);
  if (bits == 4) std::memset(canon_q_out, 0, static_cast<size_t>(N * (K / 2)));
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < g.T; ++t) {
    for (int64_t c = 0; c < g.C; ++c) {
      const uint8_t* chunk = src + (t * g.C + c) * g.chunk_bytes;
      for (int h = 0; h < 2; ++h) {
        for (int gi = 0; gi < 8; ++gi) {
          for (int ti = 0; ti < 4; ++ti) {
            uint32_t words[4];
            std::memcpy(words, chunk + 512 * h + 16 * (4 * gi + ti), 16);
            for (int j = 0; j < 4; ++j) {
              if (bits == 4) {
                for (int i = 0; i < 8; ++i) {
                  int64_t row, col;
                  q4_coord(t, c, h, gi, ti, j, i, &row, &col);
                  if (row >= N || col >= K) continue;
                  const int q = static_cast<int>((words[j] >> (4 * i)) & 0xF) - 8;
                  uint8_t* byte = static_cast<uint8_t*>(canon_q_out) + row * (K / 2) + col / 2;
                  const uint8_t nib = static_cast<uint8_t>(q & 0xF);
                  // each (row, col) is visited once and the two nibbles of a
                  // byte belong to the same tile, so this thread owns the byte
                  *byte = (col & 1) ? static_cast<uint8_t>((*byte & 0x0F) | (nib << 4))
                                    : static_cast<uint8_t>((*byte & 0xF0) | nib);
                }
              } else {
                for (int b = 0; b < 4; ++b) {
                  int64_t row, col;
                  q8_coord(t, c, h, gi, ti, j, b, &row, &col);
                  if (row >= N || col >= K) continue;
                  static_cast<int8_t*>(canon_q_out)[row * K + col] =
                      static_cast<int8_t>(static_cast<int>((words[j] >> (8 * b)) & 0xFF) - 128);
                }
              }
            }
          }
        }
      }
      for (int gi = 0; gi < 8; ++gi) {
        if (bits == 4) {
          uint16_t s8[8];
          std::memcpy(s8, chunk + 1024 + 16 * gi, 16);
          for (int h = 0; h < 2; ++h)
            for (int up = 0; up < 2; ++up)
              for (int gg = 0; gg < 2; ++gg) {
                const int64_t row = scale_row(t, h, gi, up), grp = 2 * c + gg;
                if (row < N && grp < G) scales_out[row * G + grp] = s8[4 * h + 2 * up + gg];
              }
        } else {
          uint16_t s4[4];
          std::memcpy(s4, chunk + 1024 + 8 * gi, 8);
          for (int h = 0; h < 2; ++h)
            for (int up = 0; up < 2; ++up) {
              const int64_t row = scale_row(t, h, gi, up);
              if (row < N) scales_out[row * G + c] = s4[2 * h + up];
            }
        }
      }
    }
  }
  return Q4_OK;
}

// ----------------------------------------------------------------------------
// NVFP4 (FP4 E2M1 codes, one FP8 E4M3 scale per 16 values along K, one fp32
// scale per tensor).  The chunk is that of q4 -- 32 rows x 64 columns, 1024
// code bytes then 128 scale bytes -- with the codes of one tensor-core A
// register in one byte (the hardware converts a byte of two E2M1 codes to an
// fp16 pair, low nibble to the low half).  Byte r of word j in slot (gi, ti)
// of half h holds row 16h + gi + 8 (r & 1), columns 32 (j >> 1) + 8 ti +
// 4 (j & 1) + 2 (r >> 1) + {0, 1} of the chunk: the same positions as the q4
// nibbles of register r, so both formats share the activation fragments.  A
// lane then needs the block 4c + 2G + ti / 2 of group G: the 8 scale bytes at
// 1024 + 8 (2 gi + ti / 2) are, at 4h + 2G + up, row 16h + gi + 8up.  The
// tensor scale sits in the 16 bytes after the last chunk.
// ----------------------------------------------------------------------------
namespace {

constexpr int64_t kNvfp4Trailer = 16;

bool nvfp4_geometry(int64_t N, int64_t K, Geometry* g) {
  if (!geometry(4, N, K, g)) return false;
  return K % 64 == 0;
}

inline void nvfp4_coord(int64_t t, int64_t c, int h, int gi, int ti, int j, int r, int64_t* row, int64_t* col) {
  *row = kTileRows * t + 16 * h + gi + 8 * (r & 1);
  *col = 64 * c + 32 * (j >> 1) + 8 * ti + 4 * (j & 1) + 2 * (r >> 1);
}

inline int64_t nvfp4_scale_row(int64_t t, int h, int gi, int up) { return kTileRows * t + 16 * h + gi + 8 * up; }

}  // namespace

extern "C" Q4_API size_t q4_nvfp4_packed_bytes(int64_t N, int64_t K) {
  Geometry g;
  if (!nvfp4_geometry(N, K, &g)) return 0;
  return static_cast<size_t>(g.T * g.C * g.chunk_bytes + kNvfp4Trailer);
}

extern "C" Q4_API int q4_pack_nvfp4(const uint8_t* codes, const uint8_t* scales, float tensor_scale, int64_t N,
                                    int64_t K, void* out, size_t out_bytes) {
  Geometry g;
  if (!nvfp4_geometry(N, K, &g)) {
    q4::set_error("q4_pack_nvfp4: need N >= 0, K >= 0, K % 64 == 0");
    return Q4_ERR_SHAPE;
  }
  const size_t need = static_cast<size_t>(g.T * g.C * g.chunk_bytes + kNvfp4Trailer);
  if (!out || (N * K > 0 && (!codes || !scales))) {
    q4::set_error("q4_pack_nvfp4: null pointer");
    return Q4_ERR_INVALID_ARG;
  }
  if (out_bytes < need) {
    q4::set_error("q4_pack_nvfp4: out_bytes " + std::to_string(out_bytes) + " < " + std::to_string(need));
    return Q4_ERR_BUFFER_TOO_SMALL;
  }
  const int64_t B = K / 16;
  uint8_t* dst = static_cast<uint8_t*>(out);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < g.T; ++t) {
    for (int64_t c = 0; c < g.C; ++c) {
      uint8_t* chunk = dst + (t * g.C + c) * g.chunk_bytes;
      for (int h = 0; h < 2; ++h)
        for (int gi = 0; gi < 8; ++gi)
          for (int ti = 0; ti < 4; ++ti) {
            uint8_t slot[16];
            for (int j = 0; j < 4; ++j)
              for (int r = 0; r < 4; ++r) {
                int64_t row, col;
                nvfp4_coord(t, c, h, gi, ti, j, r, &row, &col);
                // col is even: the two codes are the two nibbles of one canonical byte
                slot[4 * j + r] = row < N ? codes[row * (K / 2) + col / 2] : 0;
              }
            std::memcpy(chunk + 512 * h + 16 * (4 * gi + ti), slot, 16);
          }
      for (int gi = 0; gi < 8; ++gi)
        for (int tb = 0; tb < 2; ++tb) {
          uint8_t s8[8];
          for (int h = 0; h < 2; ++h)
            for (int G = 0; G < 2; ++G)
              for (int up = 0; up < 2; ++up) {
                const int64_t row = nvfp4_scale_row(t, h, gi, up), blk = 4 * c + 2 * G + tb;
                s8[4 * h + 2 * G + up] = row < N ? scales[row * B + blk] : 0;
              }
          std::memcpy(chunk + 1024 + 8 * (2 * gi + tb), s8, 8);
        }
    }
  }
  uint8_t trailer[kNvfp4Trailer] = {};
  std::memcpy(trailer, &tensor_scale, 4);
  std::memcpy(dst + g.T * g.C * g.chunk_bytes, trailer, kNvfp4Trailer);
  return Q4_OK;
}

extern "C" Q4_API int q4_unpack_nvfp4(const void* packed, size_t packed_bytes, int64_t N, int64_t K,
                                      uint8_t* codes_out, uint8_t* scales_out, float* tensor_scale_out) {
  Geometry g;
  if (!nvfp4_geometry(N, K, &g)) {
    q4::set_error("q4_unpack_nvfp4: need N >= 0, K >= 0, K % 64 == 0");
    return Q4_ERR_SHAPE;
  }
  const size_t need = static_cast<size_t>(g.T * g.C * g.chunk_bytes + kNvfp4Trailer);
  if (!packed || !tensor_scale_out || (N * K > 0 && (!codes_out || !scales_out))) {
    q4::set_error("q4_unpack_nvfp4: null pointer");
    return Q4_ERR_INVALID_ARG;
  }
  if (packed_bytes < need) {
    q4::set_error("q4_unpack_nvfp4: packed_bytes too small");
    return Q4_ERR_BUFFER_TOO_SMALL;
  }
  const int64_t B = K / 16;
  const uint8_t* src = static_cast<const uint8_t*>(packed);
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < g.T; ++t) {
    for (int64_t c = 0; c < g.C; ++c) {
      const uint8_t* chunk = src + (t * g.C + c) * g.chunk_bytes;
      for (int h = 0; h < 2; ++h)
        for (int gi = 0; gi < 8; ++gi)
          for (int ti = 0; ti < 4; ++ti)
            for (int j = 0; j < 4; ++j)
              for (int r = 0; r < 4; ++r) {
                int64_t row, col;
                nvfp4_coord(t, c, h, gi, ti, j, r, &row, &col);
                if (row < N) codes_out[row * (K / 2) + col / 2] = chunk[512 * h + 16 * (4 * gi + ti) + 4 * j + r];
              }
      for (int gi = 0; gi < 8; ++gi)
        for (int tb = 0; tb < 2; ++tb)
          for (int h = 0; h < 2; ++h)
            for (int G = 0; G < 2; ++G)
              for (int up = 0; up < 2; ++up) {
                const int64_t row = nvfp4_scale_row(t, h, gi, up), blk = 4 * c + 2 * G + tb;
                if (row < N) scales_out[row * B + blk] = chunk[1024 + 8 * (2 * gi + tb) + 4 * h + 2 * G + up];
              }
    }
  }
  std::memcpy(tensor_scale_out, src + g.T * g.C * g.chunk_bytes, 4);
  return Q4_OK;
}
