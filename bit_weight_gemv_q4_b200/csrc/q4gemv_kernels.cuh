// sm_100a kernels of the group-quantised weight x activation product
// y[m][n] = sum_k s[n][k/32] q[n][k] x[m][k], M <= 4 activation rows.
//
// Design (B200):
//  * The product is bound by HBM: each weight byte is read once and the work
//    is a byte stream, not a dense contraction.  Every warp streams ONE
//    contiguous byte range of the packed tensor: the flat sequence of chunks
//    (32 rows x 64 or 32 columns, in memory order) is cut into equal ranges,
//    one per warp of a grid sized to the SMs ("stream-K"), so all warps finish
//    together whatever N and K are.
//  * Bytes move HBM -> shared memory with 1-D bulk async copies
//    (cp.async.bulk, the non-tensor TMA path) into a per-warp ring of D
//    stages completed on mbarriers, with an L2 evict-first hint (the weights
//    are read once).  Lane 0 of each warp is that warp's producer.
//  * Dequantisation happens in registers.  A 32-bit word of codes decodes to
//    four bf16 pairs with one mask-and-or and one bf16x2 subtraction each:
//    the code u becomes the mantissa of 128 + u, and subtracting 128 + the
//    code offset leaves the integer q exactly (for q8 the byte is split into
//    a 16 u_hi - 128 and a u_lo part that sum to q).  The pairs are already
//    the A fragments of mma.sync m16n8k16 (bf16 in, fp32 accumulate) and the
//    activations are its B fragments (columns >= M are never stored).  Every
//    product of a <= 8-bit integer and a bf16 is exact, so a group's fp32
//    sum errs only relative to sum |q x|; it is scaled by its fp16 scale with
//    one fp32 FMA per output.
//  * Tiles split between warps are finished deterministically: each warp
//    writes its partial sums to the workspace, and the last of the tile's
//    warps to arrive (an integer counter) adds them in fixed warp order,
//    writes y and re-zeroes the counter.  No float atomics: y is bitwise
//    reproducible.
//  * Programmatic dependent launch: a kernel issues its first weight copies,
//    waits for its predecessor (griddepcontrol.wait) before touching x, y or
//    the workspace, then lets its successor launch.
//  * Every wait on an mbarrier is bounded by a %globaltimer limit; on expiry
//    the warp records kStatusTimeout in the workspace, waits (bounded) for its
//    own copies in flight and returns.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

// Single-product kernel: CTAs per SM it is compiled for, and whether it
// lets the next kernel launch (programmatic dependent launch) at its start
// rather than after its own dependency wait.
#ifndef Q4_TUNE_CTAS_PER_SM
#define Q4_TUNE_CTAS_PER_SM 1
#endif
#ifndef Q4_TUNE_EARLY_TRIGGER
#define Q4_TUNE_EARLY_TRIGGER 0
#endif

namespace q4k {

constexpr int kTileRows = 32;        // rows per tile: two m16 tensor-core tiles
constexpr int kHalfBytes = 512;      // integer codes of one 16-row half (32 lanes x 16 B)
constexpr int kCodeBytes = 1024;     // integer codes of a chunk
constexpr unsigned kStatusTimeout = 1u;

template <int BITS>
struct Format;
template <>
struct Format<4> {
  static constexpr int kKPerChunk = 64;    // two groups of 32
  static constexpr int kChunkBytes = 1152; // 1024 code bytes + 32 rows x 2 groups x fp16
};
template <>
struct Format<8> {
  static constexpr int kKPerChunk = 32;    // one group
  static constexpr int kChunkBytes = 1088; // 1024 code bytes + 32 rows x fp16
};

struct GemvParams {
  const uint8_t* packed;     // packed chunks, 16-byte aligned
  const uint16_t* x;         // bf16 bits [M][K]
  float* y;                  // [M][N]
  float* partials;           // split-tile words, [P][M][32] tagged 64-bit (zero between launches)
  unsigned* counters;        // unused by gemv_kernel (the workspace keeps the region)
  unsigned* status;          // status word
  long long N, K;
  long long TC;              // T * C, the number of chunks
  int T, C;                  // tiles, chunks per tile
  int P;                     // warps with work (P <= TC / U)
  int khalf;                 // q4 with K % 64 == 32: the last chunk of a tile holds one group
  int interleave;            // warp p of the split runs as warp p / gridDim.x of CTA p % gridDim.x
  unsigned long long timeout_ns;
};

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Polls, warp-uniformly, until the phase with the given parity completes or
// timeout_ns passes (lane 0's clock decides, so every lane leaves together).
__device__ __noinline__ bool mbar_wait_slow(uint32_t bar, uint32_t parity, unsigned long long timeout_ns) {
  const unsigned long long t0 = global_timer_ns();
  while (true) {
    if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
    const unsigned long long waited = __shfl_sync(0xFFFFFFFFu, global_timer_ns() - t0, 0);
    if (waited > timeout_ns) return false;
  }
}

// Waits for the phase with the given parity to complete, for at most
// timeout_ns.  Returns false when the limit was reached.  Every lane of the
// warp calls it; control flow and result are uniform across the warp.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity, unsigned long long timeout_ns) {
  if (__all_sync(0xFFFFFFFFu, mbar_try_wait(bar, parity))) return true;
  return mbar_wait_slow(bar, parity, timeout_ns);
}

__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t policy;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(policy));
  return policy;
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::
          "r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// Lane 0 (pred) arms `bar` for `bytes` and starts the bulk copy; every lane
// executes this one predicated block, so the warp does not branch.
__device__ __forceinline__ void bulk_copy_g2s_if(bool pred, uint32_t dst, const void* src, uint32_t bytes,
                                                 uint32_t bar, uint64_t policy) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%3], %2;\n\t"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
      "\n\t}" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy), "r"(static_cast<int>(pred))
      : "memory");
}

// Lane 0 (pred) arms `bar` for a stage of weights and its activation slice
// (bytes_w + bytes_x), copies the weights (L2 evict-first: read once) and,
// when with_x, the activations (default policy: many warps read them); a
// stage armed without them gets them from bulk_copy_x_if later.  One
// predicated block, so the warp does not branch.
__device__ __forceinline__ void bulk_copy_g2s_x_if(bool pred, uint32_t dst_w, const void* src_w, uint32_t bytes_w,
                                                   uint32_t dst_x, const void* src_x, uint32_t bytes_x, bool with_x,
                                                   uint32_t bar, uint64_t policy) {
  asm volatile(
      "{\n\t.reg .pred p, px;\n\tsetp.ne.b32 p, %8, 0;\n\t"
      "setp.ne.and.b32 px, %9, 0, p;\n\t"
      "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%6], %7;\n\t"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%6], %10;"
      "\n\t"
      "@px cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%3], [%4], %5, [%6];"
      "\n\t}" ::"r"(dst_w),
      "l"(src_w), "r"(bytes_w), "r"(dst_x), "l"(src_x), "r"(bytes_x), "r"(bar), "r"(bytes_w + bytes_x),
      "r"(static_cast<int>(pred)), "r"(static_cast<int>(with_x)), "l"(policy)
      : "memory");
}

// Lane 0 (pred) copies an activation slice into a stage that is already
// armed for its bytes.
__device__ __forceinline__ void bulk_copy_x_if(bool pred, uint32_t dst, const void* src, uint32_t bytes,
                                               uint32_t bar) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      "\n\t}" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "r"(static_cast<int>(pred))
      : "memory");
}

__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dependents_launch() { asm volatile("griddepcontrol.launch_dependents;"); }

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
  return v;
}

// 16-byte activation load done only by the lanes whose B column is a real
// token (pred); the other lanes keep their register values, which only feed
// output columns >= M that are never stored.
__device__ __forceinline__ void ldg128_pred(uint4& v, const uint16_t* ptr, bool pred) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %5, 0;\n\t"
      "@p ld.global.v4.u32 {%0, %1, %2, %3}, [%4];\n\t}"
      : "+r"(v.x), "+r"(v.y), "+r"(v.z), "+r"(v.w)
      : "l"(ptr), "r"(static_cast<int>(pred))
      : "memory");
}

__device__ __forceinline__ uint32_t lop3_and_or(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(d) : "r"(a), "r"(mask), "r"(bits));  // (a & mask) | bits
  return d;
}

// D += A (16x16, row) * B (16x8, col), fp32 accumulators; A and B both bf16
// (F16 = false) or both fp16 (F16 = true).
template <bool F16 = false>
__device__ __forceinline__ void mma_m16n8k16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// D = A * B (no accumulator input).
template <bool F16 = false>
__device__ __forceinline__ void mma_m16n8k16_first(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  const float z = 0.f;
  if constexpr (F16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%10, %10, %10, %10};"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(z));
  }
}

__device__ __forceinline__ float2 half2_bits_to_float2(uint32_t h2) {
  return __half22float2(*reinterpret_cast<const __half2*>(&h2));
}

// ----------------------------------------------------------------------------
// In-register dequantisation (shared by the product and the debug decoder)
// ----------------------------------------------------------------------------
constexpr uint32_t kNibbleMask = 0x000F000Fu;
constexpr uint32_t kBf16_128 = 0x43004300u;   // bf16 pair (128, 128): mantissa LSB = 1
constexpr uint32_t kBf16_2048 = 0x45004500u;  // (2048, 2048): mantissa LSB = 16
constexpr uint32_t kBf16_136 = 0x43084308u;   // (136, 136) = 128 + the q4 code offset 8
constexpr uint32_t kBf16_2176 = 0x45084508u;  // (2176, 2176) = 2048 + the q8 code offset 128

// a - b on bf16 pairs.  Used only where the result is an exactly
// representable small integer, so the rounding mode never matters.
__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// One q4 word -> A fragment registers a[0..3] holding the codes q exactly as
// bf16.  a[i] takes nibbles i and i + 4 (bits 4i and 16 + 4i).  The mask-and-
// or makes the nibble u = q + 8 the mantissa of 128 + u; subtracting 136
// leaves q, exact in bf16.  (Removing the offset here, not after the
// accumulation, keeps every product q * x and every partial sum free of the
// offset, so the fp32 sums err only relative to sum |q x|: an all-zero row
// gives exactly 0.)
__device__ __forceinline__ void dequant_q4_word(uint32_t w, uint32_t (&a)[4]) {
  a[0] = bf16x2_sub(lop3_and_or(w, kNibbleMask, kBf16_128), kBf16_136);
  a[1] = bf16x2_sub(lop3_and_or(w >> 4, kNibbleMask, kBf16_128), kBf16_136);
  a[2] = bf16x2_sub(lop3_and_or(w >> 8, kNibbleMask, kBf16_128), kBf16_136);
  a[3] = bf16x2_sub(lop3_and_or(w >> 12, kNibbleMask, kBf16_128), kBf16_136);
}

// Two q8 words (one m16n8k16 block) -> A fragments hi, lo with hi + lo = q
// exactly: the byte u = q + 128 = 16 u_hi + u_lo gives hi = 16 u_hi - 128
// (from 2048 + 16 u_hi) and lo = u_lo (from 128 + u_lo), both exact in bf16.
__device__ __forceinline__ void dequant_q8_block(uint32_t w0, uint32_t w1, uint32_t (&hi)[4], uint32_t (&lo)[4]) {
  lo[0] = bf16x2_sub(lop3_and_or(w0, kNibbleMask, kBf16_128), kBf16_128);
  lo[1] = bf16x2_sub(lop3_and_or(w0 >> 8, kNibbleMask, kBf16_128), kBf16_128);
  lo[2] = bf16x2_sub(lop3_and_or(w1, kNibbleMask, kBf16_128), kBf16_128);
  lo[3] = bf16x2_sub(lop3_and_or(w1 >> 8, kNibbleMask, kBf16_128), kBf16_128);
  hi[0] = bf16x2_sub(lop3_and_or(w0 >> 4, kNibbleMask, kBf16_2048), kBf16_2176);
  hi[1] = bf16x2_sub(lop3_and_or(w0 >> 12, kNibbleMask, kBf16_2048), kBf16_2176);
  hi[2] = bf16x2_sub(lop3_and_or(w1 >> 4, kNibbleMask, kBf16_2048), kBf16_2176);
  hi[3] = bf16x2_sub(lop3_and_or(w1 >> 12, kNibbleMask, kBf16_2048), kBf16_2176);
}

// fp16 decode (activations in fp16, see xprep_kernel).  fp16 has 10
// mantissa bits, so a nibble sits in the mantissa of 1024 + v at bits 0-3 or
// 4-7 without a shift, and a q8 byte at bits 0-7.
constexpr uint32_t kNibbleMaskHi = 0x00F000F0u;
constexpr uint32_t kByteMask = 0x00FF00FFu;
constexpr uint32_t kF16_1024 = 0x64006400u;   // fp16 pair (1024, 1024): mantissa LSB = 1
constexpr uint32_t kF16_1032 = 0x64086408u;   // (1032, 1032) = 1024 + the q4 code offset 8
constexpr uint32_t kF16_1152 = 0x64806480u;   // (1152, 1152) = 1024 + the q8 code offset 128
constexpr uint32_t kF16_1_16 = 0x2C002C00u;   // (1/16, 1/16)
constexpr uint32_t kF16_m72 = 0xD480D480u;    // (-72, -72) = -(1024 / 16 + 8)

// a - b and a * b + c on fp16 pairs, used only where the result is an exactly
// representable small integer.
__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t f16x2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// One q4 word -> the same four A fragments as dequant_q4_word, in fp16: the
// nibbles at bits 4-7 of each half become 1024 + 16 u, brought to q by
// (v / 16) - 72; one shift instead of three.
__device__ __forceinline__ void dequant_q4_word_f16(uint32_t w, uint32_t (&a)[4]) {
  const uint32_t t = w >> 8;
  a[0] = f16x2_sub(lop3_and_or(w, kNibbleMask, kF16_1024), kF16_1032);
  a[1] = f16x2_fma(lop3_and_or(w, kNibbleMaskHi, kF16_1024), kF16_1_16, kF16_m72);
  a[2] = f16x2_sub(lop3_and_or(t, kNibbleMask, kF16_1024), kF16_1032);
  a[3] = f16x2_fma(lop3_and_or(t, kNibbleMaskHi, kF16_1024), kF16_1_16, kF16_m72);
}

// Two q8 words -> the four A fragments of one m16n8k16 block holding q
// exactly (a[0], a[1] from w0's bytes (0, 2) and (1, 3); a[2], a[3] from w1).
__device__ __forceinline__ void dequant_q8_block_f16(uint32_t w0, uint32_t w1, uint32_t (&a)[4]) {
  a[0] = f16x2_sub(lop3_and_or(w0, kByteMask, kF16_1024), kF16_1152);
  a[1] = f16x2_sub(lop3_and_or(w0 >> 8, kByteMask, kF16_1024), kF16_1152);
  a[2] = f16x2_sub(lop3_and_or(w1, kByteMask, kF16_1024), kF16_1152);
  a[3] = f16x2_sub(lop3_and_or(w1 >> 8, kByteMask, kF16_1024), kF16_1152);
}

// ----------------------------------------------------------------------------
// One chunk's contribution to this lane's accumulators acc[h][0..3]
// (half h: rows 16h + gi and 16h + gi + 8 of the tile; columns 2ti, 2ti + 1).
// ----------------------------------------------------------------------------
struct ChunkRegs {
  uint4 codes[2];  // this lane's 16 code bytes of each half
  uint4 scales;    // q4: (R0: 2c, 2c+1) (R0+8) (R1) (R1+8);  q8: .x = (R0, R0+8), .y = (R1, R1+8)
};

// acc[0..1] += s d[0..1] and acc[2..3] += s8 d[2..3], each a fused fp32
// multiply-add rounded once.  X2 issues them as two paired fp32 FMAs
// (fma.rn.f32x2, the same two roundings per element): for products whose
// odd columns are stored (M >= 2).  With one token column the odd outputs are
// dead and the compiler drops their FMAs, so the scalar form is the cheaper.
__device__ __forceinline__ void fma_f32x2(float& a0, float& a1, float s, float d0, float d1) {
  asm("{\n\t.reg .b64 pa, ps, pd;\n\t"
      "mov.b64 pa, {%0, %1};\n\tmov.b64 ps, {%2, %2};\n\tmov.b64 pd, {%3, %4};\n\t"
      "fma.rn.f32x2 pa, ps, pd, pa;\n\tmov.b64 {%0, %1}, pa;\n\t}"
      : "+f"(a0), "+f"(a1)
      : "f"(s), "f"(d0), "f"(d1));
}
template <bool X2>
__device__ __forceinline__ void scale_fma(float (&acc)[4], float s, float s8, const float (&d)[4]) {
  if constexpr (X2) {
    fma_f32x2(acc[0], acc[1], s, d[0], d[1]);
    fma_f32x2(acc[2], acc[3], s8, d[2], d[3]);
  } else {
    acc[0] = fmaf(s, d[0], acc[0]);
    acc[1] = fmaf(s, d[1], acc[1]);
    acc[2] = fmaf(s8, d[2], acc[2]);
    acc[3] = fmaf(s8, d[3], acc[3]);
  }
}

// F16: activations and codes in fp16 (xprep_kernel made x fp16-exact),
// else bf16.  X2: see scale_fma.
template <bool F16 = false, bool X2 = false>
__device__ __forceinline__ void q4_chunk_mac(float (&acc)[2][4], const ChunkRegs& r, const uint4& xa,
                                             const uint4& xb) {
  const uint32_t sc[4] = {r.scales.x, r.scales.y, r.scales.z, r.scales.w};
#pragma unroll
  for (int G = 0; G < 2; ++G) {  // the chunk's two groups
    const uint4& xg = G ? xb : xa;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4& w = r.codes[h];
      float d[4];
      uint32_t a[4];
      if constexpr (F16) dequant_q4_word_f16(G ? w.z : w.x, a); else dequant_q4_word(G ? w.z : w.x, a);
      mma_m16n8k16_first<F16>(d, a, xg.x, xg.y);
      if constexpr (F16) dequant_q4_word_f16(G ? w.w : w.y, a); else dequant_q4_word(G ? w.w : w.y, a);
      mma_m16n8k16<F16>(d, a, xg.z, xg.w);
      const float2 s_r = half2_bits_to_float2(sc[2 * h]);       // row 16h + gi: groups 2c, 2c+1
      const float2 s_r8 = half2_bits_to_float2(sc[2 * h + 1]);  // row 16h + gi + 8
      scale_fma<X2>(acc[h], G ? s_r.y : s_r.x, G ? s_r8.y : s_r8.x, d);
    }
  }
}

template <bool F16 = false, bool X2 = false>
__device__ __forceinline__ void q8_chunk_mac(float (&acc)[2][4], const ChunkRegs& r, const uint4& xa) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4& w = r.codes[h];
    float d[4];
    if constexpr (F16) {
      uint32_t a[4];
      dequant_q8_block_f16(w.x, w.y, a);
      mma_m16n8k16_first<true>(d, a, xa.x, xa.y);
      dequant_q8_block_f16(w.z, w.w, a);
      mma_m16n8k16<true>(d, a, xa.z, xa.w);
    } else {
      uint32_t hi[4], lo[4];
      dequant_q8_block(w.x, w.y, hi, lo);
      mma_m16n8k16_first<false>(d, hi, xa.x, xa.y);
      mma_m16n8k16<false>(d, lo, xa.x, xa.y);
      dequant_q8_block(w.z, w.w, hi, lo);
      mma_m16n8k16<false>(d, hi, xa.z, xa.w);
      mma_m16n8k16<false>(d, lo, xa.z, xa.w);
    }
    const float2 s = half2_bits_to_float2(h ? r.scales.y : r.scales.x);  // rows 16h + gi, 16h + gi + 8
    scale_fma<X2>(acc[h], s.x, s.y, d);
  }
}

// The flat sequence of TB blocks (U chunks each) is cut into P ranges,
// range p = [floor(p*TB/P), floor((p+1)*TB/P)); P <= TB, so none is empty.
// owner_of(i) is the range holding block i: the largest p with begin <= i,
// i.e. floor(((i+1)*P - 1) / TB).
// Both floors are computed in double precision, which is exact here: the
// numerators are integers below 2^52 (the host keeps TB*P below 2^52), and a
// non-integer quotient lies at least 1/denominator from the next integer,
// far more than the quotient's rounding error.  (64-bit integer division has
// no hardware instruction and costs a long software sequence.)
__device__ __forceinline__ long long floor_div(long long num, long long den) {
  return static_cast<long long>(floor(static_cast<double>(num) / static_cast<double>(den)));
}
__device__ __forceinline__ int owner_of(long long i, long long TB, int P) {
  return static_cast<int>(floor_div((i + 1) * P - 1, TB));
}
__device__ __forceinline__ long long range_begin(int p, long long TB, int P) {
  return floor_div(static_cast<long long>(p) * TB, P);
}

// ----------------------------------------------------------------------------
// Finishing tiles.  A tile covered entirely by one warp's range is stored
// directly.  A tile split between warps (at most two per warp: the one its
// range starts in and the one it ends in) is finished after the warp's last
// chunk: the warp writes its partial sums to its slot (0: the tile holding
// its first chunk, 1: otherwise), then arrives on the tile's counter; the last
// arrival adds every contributor's partial in warp order (one row per lane,
// independent loads) and writes y.
// ----------------------------------------------------------------------------
// How a product's flat sequence of blocks (U chunks each) is cut among warps.
struct Partition {
  long long TB;        // blocks in the partitioned sequence
  int P;               // warps with work
  float* partials;     // [P][2][M][32]
};

// A tile split between warps: its output rows, its arrival counter, and its
// blocks [blo, bhi) in the partitioned sequence.
struct SplitTile {
  float* y;
  long long N;
  int r;
  unsigned* counter;
  long long blo, bhi;
};

template <int M>
__device__ __forceinline__ void store_tile(float* y, long long N, int r, const float (&v)[2][4], int lane) {
  const int gi = lane >> 2, ti = lane & 3;
  const int m0 = 2 * ti, m1 = 2 * ti + 1;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const long long row0 = static_cast<long long>(r) * kTileRows + 16 * h + gi;
    const long long row1 = row0 + 8;
    if (m0 < M) {
      if (row0 < N) y[m0 * N + row0] = v[h][0];
      if (row1 < N) y[m0 * N + row1] = v[h][2];
    }
    if (m1 < M) {
      if (row0 < N) y[m1 * N + row0] = v[h][1];
      if (row1 < N) y[m1 * N + row1] = v[h][3];
    }
  }
}

template <int M>
__device__ __forceinline__ void write_partial(float* partials, int pw, int slot, const float (&acc)[2][4], int lane) {
  const int gi = lane >> 2, ti = lane & 3;
  const int m0 = 2 * ti, m1 = 2 * ti + 1;
  float* mine = partials + (static_cast<long long>(pw) * 2 + slot) * (M * kTileRows);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row0 = 16 * h + gi, row1 = row0 + 8;
    if (m0 < M) {
      mine[m0 * kTileRows + row0] = acc[h][0];
      mine[m0 * kTileRows + row1] = acc[h][2];
    }
    if (m1 < M) {
      mine[m1 * kTileRows + row0] = acc[h][1];
      mine[m1 * kTileRows + row1] = acc[h][3];
    }
  }
}

__device__ __forceinline__ unsigned tile_contributors(const Partition& pt, const SplitTile& st) {
  return static_cast<unsigned>(owner_of(st.bhi - 1, pt.TB, pt.P) - owner_of(st.blo, pt.TB, pt.P) + 1);
}

// Last arrival on a split tile: sum the partials of its contributing warps in
// warp order (one row per lane) and store the tile; then re-zero its counter.
// The partials' loads go out 32 at a time (contributors x rows) before any is
// added, so a tile split between many warps costs a few round trips to L2, not
// one per contributor; the additions keep warp order.  Out of line: its
// registers do not weigh on the streaming loop.
constexpr int kReduceBatch = 32;

template <int M>
__device__ __noinline__ void reduce_tile(const Partition& pt, const SplitTile& st, int lane) {
  const int p_lo = owner_of(st.blo, pt.TB, pt.P);
  const int p_hi = owner_of(st.bhi - 1, pt.TB, pt.P);
  const long long row = static_cast<long long>(st.r) * kTileRows + lane;
  // Warp p_lo's range begins at or before the tile: the tile is its first
  // (slot 0) only if it begins exactly at blo.  Every later contributor
  // begins inside the tile, so the tile is its first: slot 0.
  const int slot_lo = (range_begin(p_lo, pt.TB, pt.P) == st.blo) ? 0 : 1;
  const float* base = pt.partials + lane;
  float sum[M];
#pragma unroll
  for (int m = 0; m < M; ++m)
    sum[m] = __ldcg(base + (static_cast<long long>(p_lo) * 2 + slot_lo) * (M * kTileRows) + m * kTileRows);
  // word j of the rest: contributor p_lo + 1 + j / M, row m = j % M
  const int rest = (p_hi - p_lo) * M;
  for (int j0 = 0; j0 < rest; j0 += kReduceBatch) {
    float v[kReduceBatch];
#pragma unroll
    for (int k = 0; k < kReduceBatch; ++k) {
      const int j = j0 + k;
      const int q = p_lo + 1 + j / M, m = j % M;
      v[k] = j < rest ? __ldcg(base + (static_cast<long long>(q) * 2) * (M * kTileRows) + m * kTileRows) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kReduceBatch; ++k) {
      const int j = j0 + k;
      if (j < rest) sum[j % M] += v[k];
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (row < st.N) st.y[m * st.N + row] = sum[m];
  if (lane == 0) *st.counter = 0u;
}

// Finishes the (at most two) split tiles of warp pw after its last chunk:
// `first` (partial kept in acc_first, slot 0) is the tile holding the range's
// first block when that tile began in an earlier warp's range; `last`
// (acc_last, slot_last) is the tile holding the range's last block when the
// range ends inside it.  Absent tiles have r < 0.
template <int M>
__device__ __forceinline__ void finish_split_tiles(const Partition& pt, int pw, const SplitTile& first,
                                                   const float (&acc_first)[2][4], const SplitTile& last,
                                                   int slot_last, const float (&acc_last)[2][4], int lane) {
  if (first.r < 0 && last.r < 0) return;
  if (first.r >= 0) write_partial<M>(pt.partials, pw, 0, acc_first, lane);
  if (last.r >= 0) write_partial<M>(pt.partials, pw, slot_last, acc_last, lane);
  __threadfence();
  __syncwarp();
  unsigned a_first = 0, a_last = 0;
  if (lane == 0) {
    if (first.r >= 0) a_first = atomicAdd(first.counter, 1u);
    if (last.r >= 0) a_last = atomicAdd(last.counter, 1u);
  }
  a_first = __shfl_sync(0xFFFFFFFFu, a_first, 0);
  a_last = __shfl_sync(0xFFFFFFFFu, a_last, 0);
  const bool red_first = first.r >= 0 && a_first + 1 == tile_contributors(pt, first);
  const bool red_last = last.r >= 0 && a_last + 1 == tile_contributors(pt, last);
  if (red_first || red_last) __threadfence();
  if (red_first) reduce_tile<M>(pt, first, lane);
  if (red_last) reduce_tile<M>(pt, last, lane);
}

// ----------------------------------------------------------------------------
// The product kernel.  NW warps per CTA, each with a ring of D stages of U
// chunks in shared memory.  Warp ranges are whole blocks of U chunks and U
// divides C, so a stage never straddles two tiles: the tile bookkeeping runs
// once per stage.  With XS the activations are staged once per CTA in shared
// memory (one bulk copy per row, rows padded with 64 zero bytes so the empty
// half of a last q4 chunk reads zeros); otherwise they are read from global
// memory through L1.
// ----------------------------------------------------------------------------
constexpr int kXPadBytes = 64;

// ----------------------------------------------------------------------------
// Split tiles of the single-product kernel.  A warp whose range begins inside
// a tile publishes its part of the tile as tagged 64-bit words (the float's
// bits, tag kPartTag in the high half; one word per token row and tile row):
// a 64-bit store is single-copy atomic, so a reader that sees the tag sees the
// value, and no fence or counter is needed.  The warp holding the tile's
// first block (its owner) polls its contributors' words, adds the parts in
// warp order, stores the tile and writes the words back to zero, so every
// completed launch leaves them zero for the next (which reads none of them
// before griddepcontrol.wait has seen this one complete).  Words: [warp][M][32].
// ----------------------------------------------------------------------------
constexpr unsigned long long kPartTag = 1ull << 32;
constexpr int kPartBatch = 32;  // words a lane keeps in flight while polling

__device__ __forceinline__ void part_store(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long part_load(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// The tile's values by row: lane l gets row l of every token column m < M
// from the mma accumulator layout (half h: rows 16h + gi and 16h + gi + 8,
// columns 2ti and 2ti + 1).
template <int M>
__device__ __forceinline__ void tile_rows_shfl(const float (&acc)[2][4], int lane, float (&out)[M]) {
  const int h = lane >> 4, hi = (lane >> 3) & 1, g = lane & 7;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const int src = g * 4 + (m >> 1);
    const float v00 = __shfl_sync(0xFFFFFFFFu, acc[0][m & 1], src);
    const float v01 = __shfl_sync(0xFFFFFFFFu, acc[0][2 + (m & 1)], src);
    const float v10 = __shfl_sync(0xFFFFFFFFu, acc[1][m & 1], src);
    const float v11 = __shfl_sync(0xFFFFFFFFu, acc[1][2 + (m & 1)], src);
    out[m] = h ? (hi ? v11 : v10) : (hi ? v01 : v00);
  }
}

// A contributor's part of the tile that began before its range.
template <int M>
__device__ __forceinline__ void publish_part(unsigned long long* words, int pw, const float (&acc)[2][4], int lane) {
  float v[M];
  tile_rows_shfl<M>(acc, lane, v);
#pragma unroll
  for (int m = 0; m < M; ++m)
    part_store(words + (static_cast<long long>(pw) * M + m) * kTileRows + lane, kPartTag | __float_as_uint(v[m]));
}

// The owner (warp pw) of tile r: its own part (acc) plus contributors
// pw + 1 .. p_hi, in warp order, into y; false when a wait gave up.
template <int M>
__device__ __noinline__ bool own_tile(unsigned long long* words, float* y, long long N, int r, int pw, int p_hi,
                                      const float (&acc)[2][4], int lane, unsigned long long timeout_ns) {
  float sum[M];
  tile_rows_shfl<M>(acc, lane, sum);
  constexpr int GQ = kPartBatch / M;  // contributors per round trip
  unsigned long long t0 = 0;
  for (int q0 = pw + 1; q0 <= p_hi; q0 += GQ) {
    const int nq = min(GQ, p_hi - q0 + 1);
    unsigned long long* base = words + static_cast<long long>(q0) * M * kTileRows + lane;
    unsigned long long w[kPartBatch];
#pragma unroll
    for (int k = 0; k < kPartBatch; ++k) w[k] = k < nq * M ? part_load(base + k * kTileRows) : kPartTag;
    while (true) {
      bool mine = true;
#pragma unroll
      for (int k = 0; k < kPartBatch; ++k) mine = mine && (w[k] >> 32) == 1u;
      if (__all_sync(0xFFFFFFFFu, mine)) break;
      if (t0 == 0) t0 = global_timer_ns();
      const unsigned long long waited = __shfl_sync(0xFFFFFFFFu, global_timer_ns() - t0, 0);
      if (waited > timeout_ns) return false;
#pragma unroll
      for (int k = 0; k < kPartBatch; ++k)
        if (k < nq * M && (w[k] >> 32) != 1u) w[k] = part_load(base + k * kTileRows);
    }
#pragma unroll
    for (int k = 0; k < kPartBatch; ++k) {
      if (k < nq * M) {
        sum[k % M] += __uint_as_float(static_cast<unsigned>(w[k]));
        part_store(base + k * kTileRows, 0ull);
      }
    }
  }
  const long long row = static_cast<long long>(r) * kTileRows + lane;
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (row < N) y[m * N + row] = sum[m];
  return true;
}

template <int BITS, int NW, int D, int U>
struct GemvConfig {
  static constexpr int kChunkBytes = Format<BITS>::kChunkBytes;
  static constexpr int kStageBytes = U * kChunkBytes;
  static constexpr int kRingBytes = D * kStageBytes;
  static constexpr int kBarOffset = NW * kRingBytes;
  static constexpr int kXBarOffset = kBarOffset + NW * D * 8;
  static constexpr int kXOffset = (kXBarOffset + 8 + 127) / 128 * 128;  // activations (XS)
  static constexpr int kThreads = NW * 32;
};

__host__ __device__ constexpr long long x_row_stride_bytes(long long K) { return 2 * K + kXPadBytes; }

template <int BITS, int M, int NW, int D, int U, bool XS>
__global__ void __launch_bounds__(NW * 32, Q4_TUNE_CTAS_PER_SM) gemv_kernel(const GemvParams p) {
  using Cfg = GemvConfig<BITS, NW, D, U>;
  constexpr int CB = Cfg::kChunkBytes;
  constexpr int KC = Format<BITS>::kKPerChunk;
  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int gi = lane >> 2, ti = lane & 3;
  // warp index in the split: consecutive within a CTA, or, for a product
  // split between fewer warps than the GPU holds, interleaved over one CTA per
  // SM so that every SM streams (p.interleave)
  const int pw = p.interleave ? warp * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x)
                              : static_cast<int>(blockIdx.x) * NW + warp;

  const uint32_t ring = smem_addr(smem + warp * Cfg::kRingBytes);
  const uint32_t bars = smem_addr(smem + Cfg::kBarOffset) + warp * D * 8;
  const uint32_t xbar = smem_addr(smem + Cfg::kXBarOffset);
  const uint32_t xsm = smem_addr(smem + Cfg::kXOffset);
  const uint32_t xstride = static_cast<uint32_t>(x_row_stride_bytes(p.K));

  // this warp's range of chunks: whole blocks of U chunks
  const long long TB = p.TC / U;
  long long b = 0, e = 0;
  if (pw < p.P) {
    b = range_begin(pw, TB, p.P) * U;
    e = range_begin(pw + 1, TB, p.P) * U;
  }
  const int nst = static_cast<int>((e - b) / U);

  if (Q4_TUNE_EARLY_TRIGGER) grid_dependents_launch();
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(bars + 8 * s, 1);
    if (XS && warp == 0) mbar_init(xbar, 1);
    fence_barrier_init();
  }
  if (XS) {
    // zero the pad after each activation row (bytes the bulk copies never write)
    for (int i = threadIdx.x; i < M * (kXPadBytes / 16); i += NW * 32) {
      const int m = i / (kXPadBytes / 16), q = i % (kXPadBytes / 16);
      const uint32_t addr = xsm + m * xstride + static_cast<uint32_t>(2 * p.K) + 16 * q;
      asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(addr), "r"(0) : "memory");
    }
  }
  __syncthreads();

  const uint64_t policy = l2_evict_first_policy();
  const uint8_t* src = p.packed + b * CB;
  if (lane == 0) {
    const int first = nst < D ? nst : D;
    for (int s = 0; s < first; ++s) {
      mbar_arrive_expect_tx(bars + 8 * s, Cfg::kStageBytes);
      bulk_copy_g2s(ring + s * Cfg::kStageBytes, src + static_cast<long long>(s) * Cfg::kStageBytes,
                    Cfg::kStageBytes, bars + 8 * s, policy);
    }
  }
  int issued = nst < D ? nst : D;

  // The weights do not depend on the previous kernel; x, y and the workspace may.
  grid_dependency_wait();
  if (!Q4_TUNE_EARLY_TRIGGER) grid_dependents_launch();

  if (XS && threadIdx.x == 0) {
    mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(M * 2 * p.K));
    for (int m = 0; m < M; ++m) {
      asm volatile(
          "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
              xsm + m * xstride),
          "l"(p.x + static_cast<long long>(m) * p.K), "r"(static_cast<uint32_t>(2 * p.K)), "r"(xbar)
          : "memory");
    }
  }

  int r = static_cast<int>(floor_div(b, p.C));
  int c = static_cast<int>(b - static_cast<long long>(r) * p.C);
  const bool x_lane = gi < M;
  // shared-memory activations: lanes whose column is not a token read row 0
  const uint32_t xs_lane = xsm + (x_lane ? gi : 0) * xstride + 16 * ti;
  const uint16_t* xrow = p.x + static_cast<long long>(x_lane ? gi : 0) * p.K + 8 * ti;
  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  unsigned long long* words = reinterpret_cast<unsigned long long*>(p.partials);
  uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);

  bool ok = true;
  if (XS) ok = mbar_wait_bounded(xbar, 0, p.timeout_ns);
  int slot = 0;
  uint32_t phase = 0;
  int i = 0;
  for (; ok && i < nst; ++i) {
    if (!mbar_wait_bounded(bars + 8 * slot, phase, p.timeout_ns)) {
      ok = false;
      break;
    }
    const uint32_t stage = ring + slot * Cfg::kStageBytes;
    ChunkRegs regs[U];
#pragma unroll
    for (int j = 0; j < U; ++j) {
      regs[j].codes[0] = lds128(stage + j * CB + 16 * lane);
      regs[j].codes[1] = lds128(stage + j * CB + kHalfBytes + 16 * lane);
      if (BITS == 4) {
        regs[j].scales = lds128(stage + j * CB + kCodeBytes + 16 * gi);
      } else {
        const uint2 s2 = lds64(stage + j * CB + kCodeBytes + 8 * gi);
        regs[j].scales = make_uint4(s2.x, s2.y, 0u, 0u);
      }
    }
    // Every lane has read the stage (warp-synchronous order, as an mbarrier
    // release would give a separate consumer); lane 0 refills the slot.
    __syncwarp();
    if (i + D < nst) {
      bulk_copy_g2s_if(lane == 0, stage, src + static_cast<long long>(i + D) * Cfg::kStageBytes, Cfg::kStageBytes,
                       bars + 8 * slot, policy);
      issued = i + D + 1;
    }
#pragma unroll
    for (int j = 0; j < U; ++j) {
      if (XS) {
        const uint32_t xo = xs_lane + 2 * KC * (c + j);
        xa = lds128(xo);
        if (BITS == 4) xb = lds128(xo + 64);
      } else {
        const uint16_t* xs = xrow + static_cast<long long>(c + j) * KC;
        ldg128_pred(xa, xs, x_lane);
        if (BITS == 4) {
          // a K that is an odd multiple of 32 leaves the last chunk half empty
          const bool half_empty = p.khalf && c + j == p.C - 1;
          ldg128_pred(xb, xs + 32, x_lane && !half_empty);
          if (half_empty) xb = make_uint4(0, 0, 0, 0);
        }
      }
      if (BITS == 4)
        q4_chunk_mac<false, (M > 1)>(acc, regs[j], xa, xb);
      else
        q8_chunk_mac<false, (M > 1)>(acc, regs[j], xa);
    }
    c += U;
    if (c == p.C) {
      const long long tile_lo = static_cast<long long>(r) * p.C;
      if (tile_lo < b)  // the first tile began in an earlier warp's range: its owner adds this part
        publish_part<M>(words, pw, acc, lane);
      else
        store_tile<M>(p.y, p.N, r, acc, lane);
      ++r;
      c = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
    }
    if (++slot == D) {
      slot = 0;
      phase ^= 1u;
    }
  }
  if (!ok) {
    if (lane == 0) atomicOr(p.status, kStatusTimeout);
    // wait (bounded) for this warp's own copies still in flight, then leave
    for (int s = i; s < issued; ++s) {
      if (!mbar_wait_bounded(bars + 8 * (s % D), (s / D) & 1, p.timeout_ns)) break;
    }
    if (XS) (void)mbar_wait_bounded(xbar, 0, p.timeout_ns);
    return;
  }
  if (nst == 0 || c == 0) return;
  // the range ends inside tile r: its part, if the tile began in an earlier
  // range; else this warp owns the tile
  if (static_cast<long long>(r) * p.C < b) {
    publish_part<M>(words, pw, acc, lane);
    return;
  }
  const long long bpt = p.C / U;  // blocks per tile
  const int p_hi = owner_of((static_cast<long long>(r) + 1) * bpt - 1, TB, p.P);
  if (!own_tile<M>(words, p.y, p.N, r, pw, p_hi, acc, lane, p.timeout_ns) && lane == 0)
    atomicOr(p.status, kStatusTimeout);
}

// ----------------------------------------------------------------------------
// Debug decoder: one warp per chunk, using the same in-register dequantisation
// as the product kernel; writes int8 q [N][K] and fp16 scales [N][K/32].
// ----------------------------------------------------------------------------
__device__ __forceinline__ int f16_bits_to_int(uint32_t h) {
  return static_cast<int>(__half2float(__ushort_as_half(static_cast<unsigned short>(h & 0xFFFF))));
}

__device__ __forceinline__ int bf16_bits_to_int(uint32_t h) {
  const uint16_t b = static_cast<uint16_t>(h & 0xFFFF);
  return static_cast<int>(__bfloat162float(*reinterpret_cast<const __nv_bfloat16*>(&b)));
}

template <int BITS>
__global__ void unpack_kernel(const uint8_t* packed, long long N, long long K, int T, int C, int8_t* q_out,
                              uint16_t* s_out) {
  constexpr int CB = Format<BITS>::kChunkBytes;
  const int lane = threadIdx.x & 31;
  const long long chunk = static_cast<long long>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (chunk >= static_cast<long long>(T) * C) return;
  const int t = static_cast<int>(chunk / C), c = static_cast<int>(chunk % C);
  const int gi = lane >> 2, ti = lane & 3;
  const uint8_t* base = packed + chunk * CB;
  const long long G = K / 32;
  auto put = [&](long long row, long long col, int q) {
    if (row < N && col < K) q_out[row * K + col] = static_cast<int8_t>(q);
  };
  for (int h = 0; h < 2; ++h) {
    const uint4 codes = *reinterpret_cast<const uint4*>(base + kHalfBytes * h + 16 * lane);
    const uint32_t w[4] = {codes.x, codes.y, codes.z, codes.w};
    const long long R = static_cast<long long>(t) * kTileRows + 16 * h + gi;
    // the bf16 and the fp16 decode must agree; a disagreement writes -128,
    // a value neither format holds
    auto both = [](int qb, int qh) { return qb == qh ? qb : -128; };
    if (BITS == 4) {
      for (int j = 0; j < 4; ++j) {
        uint32_t a[4], af[4];
        dequant_q4_word(w[j], a);
        dequant_q4_word_f16(w[j], af);
        const long long kb = 64LL * c + 32 * (j >> 1) + 8 * ti + 4 * (j & 1);
        // a[0]: row R, k kb, kb+1; a[1]: row R+8; a[2]: row R, kb+2, kb+3; a[3]: row R+8
        for (int reg = 0; reg < 4; ++reg) {
          const long long row = R + 8 * (reg & 1);
          const long long col = kb + 2 * (reg >> 1);
          put(row, col, both(bf16_bits_to_int(a[reg]), f16_bits_to_int(af[reg])));
          put(row, col + 1, both(bf16_bits_to_int(a[reg] >> 16), f16_bits_to_int(af[reg] >> 16)));
        }
      }
    } else {
      for (int blk = 0; blk < 2; ++blk) {
        uint32_t hi[4], lo[4], af[4];
        dequant_q8_block(w[2 * blk], w[2 * blk + 1], hi, lo);
        dequant_q8_block_f16(w[2 * blk], w[2 * blk + 1], af);
        const long long kb = 32LL * c + 8 * ti + 4 * blk;
        for (int reg = 0; reg < 4; ++reg) {
          const long long row = R + 8 * (reg & 1);
          const long long col = kb + 2 * (reg >> 1);
          put(row, col, both(bf16_bits_to_int(hi[reg]) + bf16_bits_to_int(lo[reg]), f16_bits_to_int(af[reg])));
          put(row, col + 1,
              both(bf16_bits_to_int(hi[reg] >> 16) + bf16_bits_to_int(lo[reg] >> 16), f16_bits_to_int(af[reg] >> 16)));
        }
      }
    }
  }
  if (ti == 0) {
    const uint16_t* s = reinterpret_cast<const uint16_t*>(base + kCodeBytes + (BITS == 4 ? 16 : 8) * gi);
    for (int h = 0; h < 2; ++h) {
      for (int up = 0; up < 2; ++up) {
        const long long row = static_cast<long long>(t) * kTileRows + 16 * h + gi + 8 * up;
        if (row >= N) continue;
        if (BITS == 4) {
          for (int g = 0; g < 2; ++g) {
            const long long grp = 2LL * c + g;
            if (grp < G) s_out[row * G + grp] = s[4 * h + 2 * up + g];
          }
        } else {
          s_out[row * G + c] = s[2 * h + up];
        }
      }
    }
  }
}

// ----------------------------------------------------------------------------
// Device repack: canonical q and scales -> packed chunks, one thread per
// 16-byte code slot (the same placement as the host packer).
// ----------------------------------------------------------------------------
template <int BITS>
__global__ void pack_kernel(const uint8_t* q, const uint16_t* s, long long N, long long K, int T, int C,
                            uint8_t* out) {
  constexpr int CB = Format<BITS>::kChunkBytes;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(T) * C * 64) return;
  const long long chunk = idx >> 6;
  const int h = static_cast<int>((idx >> 5) & 1);
  const int slot = static_cast<int>(idx & 31);
  const int gi = slot >> 2, ti = slot & 3;
  const long long t = chunk / C, c = chunk % C;
  const long long R = t * kTileRows + 16 * h + gi;
  uint32_t w[4];
  for (int j = 0; j < 4; ++j) {
    uint32_t word = 0;
    if (BITS == 4) {
      const int G = j >> 1, e = j & 1;
      for (int i = 0; i < 8; ++i) {
        const long long row = R + 8 * (i & 1);
        const long long col = 64 * c + 32 * G + 8 * ti + 4 * e + 2 * ((i >> 1) & 1) + (i >> 2);
        int v = 0;
        if (row < N && col < K) {
          const int byte = q[row * (K / 2) + col / 2];
          const int nib = (col & 1) ? (byte >> 4) : (byte & 0xF);
          v = nib >= 8 ? nib - 16 : nib;
        }
        word |= static_cast<uint32_t>(v + 8) << (4 * i);
      }
    } else {
      const int e = j >> 1, f = j & 1;
      for (int b = 0; b < 4; ++b) {
        const long long row = R + 8 * (b & 1);
        const long long col = 32 * c + 8 * ti + 4 * e + 2 * f + (b >> 1);
        int v = 0;
        if (row < N && col < K) v = static_cast<int8_t>(q[row * K + col]);
        word |= static_cast<uint32_t>(v + 128) << (8 * b);
      }
    }
    w[j] = word;
  }
  uint8_t* dst = out + chunk * CB;
  *reinterpret_cast<uint4*>(dst + kHalfBytes * h + 16 * slot) = make_uint4(w[0], w[1], w[2], w[3]);
  if (ti == 0 && h == 0) {
    const long long G = K / 32;
    uint16_t v[8];
    for (int hh = 0; hh < 2; ++hh) {
      for (int up = 0; up < 2; ++up) {
        const long long row = t * kTileRows + 16 * hh + gi + 8 * up;
        if (BITS == 4) {
          for (int g = 0; g < 2; ++g) {
            const long long grp = 2 * c + g;
            v[4 * hh + 2 * up + g] = (row < N && grp < G) ? s[row * G + grp] : 0;
          }
        } else {
          v[2 * hh + up] = row < N ? s[row * G + c] : 0;
        }
      }
    }
    if (BITS == 4) {
      *reinterpret_cast<uint4*>(dst + kCodeBytes + 16 * gi) =
          make_uint4(v[0] | (static_cast<uint32_t>(v[1]) << 16), v[2] | (static_cast<uint32_t>(v[3]) << 16),
                     v[4] | (static_cast<uint32_t>(v[5]) << 16), v[6] | (static_cast<uint32_t>(v[7]) << 16));
    } else {
      *reinterpret_cast<uint2*>(dst + kCodeBytes + 8 * gi) =
          make_uint2(v[0] | (static_cast<uint32_t>(v[1]) << 16), v[2] | (static_cast<uint32_t>(v[3]) << 16));
    }
  }
}

// ----------------------------------------------------------------------------
// Self-test of the bounded wait: a barrier expecting two arrivals gets one.
// ----------------------------------------------------------------------------
__global__ void wait_selftest_kernel(unsigned long long timeout_ns, int* result) {
  __shared__ __align__(8) unsigned long long bar_storage;
  const uint32_t bar = smem_addr(&bar_storage);
  if (threadIdx.x == 0) {
    mbar_init(bar, 2);
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) mbar_arrive(bar);
  __syncwarp();
  const bool ok = mbar_wait_bounded(bar, 0, timeout_ns);
  if (threadIdx.x == 0) *result = ok ? 0 : 1;
}

}  // namespace q4k
