// The dependent decode chain (products with residual + RMSNorm and SwiGLU
// steps between them) as ONE persistent cooperative kernel, M = 1..4.
//
// The pages describe the decode step as a 64-layer sequence of weight
// streams (ai-coding.wiselychen.com guide, section "Before deploying";
// bs178.com llamAmpere post, "Why it is this fast") whose products depend on
// one another through the layer's normalisation and gated MLP.  Launched one
// kernel per op, every product pays a launch, a ramp-up and a tail.  Here one
// CTA per SM walks the whole op list:
//  * A product is split between all warps stream-K style, as a one-product
//    stream-mode stack splits it (same ranges, same fp16 decode of resident
//    activations, same partial sums added in the same order).
//  * Each warp's bulk-copy ring runs ahead ACROSS ops, and a second cursor
//    prefetches the stages after the ring's into L2: weights never depend on
//    activations, so HBM keeps streaming while the CTAs finish a step.
//  * No fence, atomic or grid barrier sits on the path from one product to
//    the next.  On B200 a memory fence waits for the SM's bulk copies in
//    flight (about 1.7 us with the rings running ahead, 0.3 us without), so
//    every value another warp must see is written as one 64-bit word holding
//    the value and a tag (the run and the op), which is single-copy atomic:
//    a reader polls a word until its tag is the one it expects.
//  * A tile split between warps is finished by its owner, the warp whose
//    range holds the tile's first chunk: the others write their partial sums
//    tagged, the owner polls them and adds them in warp order.
//  * A step is split in two.  Its elementwise part runs where the values
//    become final: the owner of each tile of the product before it adds the
//    tile to the residual stream and writes the tile's sum of squares
//    (RMSNorm), or, for a (gate, up) tile pair, the up tile's owner writes its
//    values tagged and the gate tile's owner writes silu(gate) * up rounded
//    to bf16 (SwiGLU).  Then every CTA finishes the step for itself from the
//    tagged words: the mean square from the tile sums (RMSNorm), the bf16
//    activations, converted to fp16 when exact, into its shared-memory copy of
//    the next product's activations.  A step whose input is not the preceding
//    product's output does its elementwise part split between the CTAs.
//  * The residual stream: every norm writes its result as tagged words of its
//    own, which the step's finish and the next norm of the stream read; the
//    stream's last norm also writes the caller's buffer.  (A plain store is
//    not ordered before a later tagged word, so values other warps read are
//    never plain stores made in the same launch, except after a barrier.)
//  * Workspace reuse that the data flow does not order (the partial
//    buffers) is checked on the host, which puts a grid barrier (an arrival
//    counter) before an op that would otherwise overwrite words a slow warp
//    may still read.
//  * Every wait is bounded: a wait that gives up marks the CTA aborted, the
//    CTA stops at its next op, drains its copies (bounded) and exits; the
//    other CTAs' waits then give up too, and the status word records it.
//
// The sum of squares has one association everywhere (this kernel, the
// captured chain's residual_rmsnorm_kernel): fp32 squares, a butterfly
// (xor-shuffle) sum over each tile of 32 consecutive values, lane l adding the
// sums of tiles l, l + 32, l + 64, ... in order, and a butterfly over the 32
// lanes; so both give bitwise the same activations from the same inputs.
#pragma once

#include <climits>

#include "q4chain_kernel.cuh"
#include "q4stack_kernel.cuh"

namespace q4k {

constexpr int kChainProduct = 0;
constexpr int kChainRmsnorm = 1;
constexpr int kChainSwiglu = 2;
// product epilogues
constexpr int kEpiNone = 0;
constexpr int kEpiResid = 1;   // the RMSNorm after it: residual add, tile sums of squares
constexpr int kEpiSwiglu = 2;  // the SwiGLU after it: silu(gate) * up of each (gate, up) tile pair
// products use this many partial-sum buffers in turn
constexpr int kChainPartialBufs = 4;

struct ChainOpDev {
  int kind;      // kChainProduct / kChainRmsnorm / kChainSwiglu
  int barrier;   // a grid barrier precedes the op (workspace reuse the data flow does not order)
  int stage_x;   // product: copy x from global memory into the CTA's activation buffer first
  int entry;     // product: its StackEntryDev
  int pbuf;      // product: its partial-sum buffer
  int epi;       // product: kEpi*; step: 1 when the product before it runs its elementwise part
  int step;      // product with an epilogue: index of that step's op
  int set;       // RMSNorm: h <- y instead of h <- h + y
  int N;         // steps: output row length
  int kc;        // values per chunk of the activation buffer's layout ([K/kc][M][kc]; 64 q4, 32 q8)
  int tw;        // RMSNorm: first word of its h ([M][N]); SwiGLU: of its output pairs ([M][N/2])
  int uw;        // SwiGLU (fused): first word of the up values ([M][N])
  int pre_next;  // op whose prepared activations this op's start copies into the buffer's tail (-1: none)
  int pre_off;   // staged product: byte offset of that copy in the buffer (-1: staged from x by the CTA)
  int prep;      // staged product with a prepared copy: its index (the launch prepares it first), else -1
  long long prep_at;  // its prepared copy's first value in ChainParams::prep
  int src_op;    // RMSNorm: the stream's previous norm, whose tagged h it adds to (-1: h_src, or set)
  const uint16_t* x;      // product: bf16 [M][K] (read when stage_x)
  const float* y;         // steps: fp32 input (RMSNorm: [M][N] or null; SwiGLU: [M][2N])
  const uint16_t* gamma;  // RMSNorm: bf16 [N] or null
  uint16_t* out;          // steps: bf16 [M][N]
  const float* h_src;     // RMSNorm: the stream as the launch found it (the first norm, unless set)
  float* h_dst;           // RMSNorm: the caller's stream, written by its last norm (else null)
};

struct ChainParams {
  const ChainOpDev* ops;
  int n_ops;
  const StackEntryDev* entries;  // the products, in op order (blk_off 0: each is its own sequence)
  int E;
  unsigned long long* parts;      // kChainPartialBufs x [warps][M][32] tagged partial sums
  long long pbuf_words;           // words per partial buffer
  unsigned long long* words;      // the steps' tagged words
  unsigned* run_ctr;              // [G] runs completed, per CTA
  unsigned long long* bar_count;  // grid-barrier arrivals (only grows, a multiple of G between runs)
  uint16_t* prep;                 // prepared activations of the staged products (chunk-major, fp16 when exact)
  int* prep_info;                 // per prepared copy: fp16 exact, sigma
  const int* prep_ops;            // per prepared copy: its product's op index
  int n_prep;
  int tiles_off;                  // dynamic shared memory: the norms' tile sums of squares
  unsigned* status;
  int G;
  int x_off;       // dynamic shared memory: byte offset of the activation buffer
  int scr_off;     // dynamic shared memory: per-warp scratch [NW][M][32] floats
  int pad;
  unsigned long long timeout_ns;
};

// What stream_segment reads from its parameters.
struct ChainSegParams {
  unsigned long long timeout_ns;
  unsigned long long* parts;  // this product's partial buffer
  uint32_t tag;
};

// ---- tagged words -------------------------------------------------------------
__device__ __forceinline__ unsigned long long tagged(uint32_t tag, uint32_t bits) {
  return (static_cast<unsigned long long>(tag) << 32) | bits;
}
__device__ __forceinline__ void st_word(unsigned long long* p, unsigned long long v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long ld_word(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ bool tag_is(unsigned long long w, uint32_t tag) {
  return static_cast<uint32_t>(w >> 32) == tag;
}

// Loads words p[i * stride] for i < n (n <= NMAX; the others read as valid
// zeros) into v[], polling until each holds `tag`, for at most timeout_ns.
template <int NMAX>
__device__ __forceinline__ bool poll_words(const unsigned long long* p, long long stride, int n, uint32_t tag,
                                           unsigned long long (&v)[NMAX], unsigned long long timeout_ns) {
  unsigned pending = 0;
#pragma unroll
  for (int i = 0; i < NMAX; ++i) {
    v[i] = i < n ? ld_word(p + i * stride) : tagged(tag, 0u);
    if (!tag_is(v[i], tag)) pending |= 1u << i;
  }
  if (!pending) return true;
  const unsigned long long t0 = global_timer_ns();
  while (pending) {
#pragma unroll
    for (int i = 0; i < NMAX; ++i)
      if (pending & (1u << i)) v[i] = ld_word(p + i * stride);
#pragma unroll
    for (int i = 0; i < NMAX; ++i)
      if (tag_is(v[i], tag)) pending &= ~(1u << i);
    if (pending && global_timer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// The 2-D form: words p[m * sm + i * si] for m < NM, i < n (n <= NB), all
// loads issued before the first tag is checked.
template <int NM, int NB>
__device__ __forceinline__ bool poll_words2(const unsigned long long* p, long long sm, long long si, int n,
                                            uint32_t tag, unsigned long long (&v)[NM][NB],
                                            unsigned long long timeout_ns) {
  static_assert(NM * NB <= 64, "one pending bit per word");
  unsigned long long pending = 0;
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int i = 0; i < NB; ++i) v[m][i] = i < n ? ld_word(p + m * sm + i * si) : tagged(tag, 0u);
#pragma unroll
  for (int m = 0; m < NM; ++m)
#pragma unroll
    for (int i = 0; i < NB; ++i)
      if (!tag_is(v[m][i], tag)) pending |= 1ull << (m * NB + i);
  if (!pending) return true;
  const unsigned long long t0 = global_timer_ns();
  while (pending) {
#pragma unroll
    for (int m = 0; m < NM; ++m)
#pragma unroll
      for (int i = 0; i < NB; ++i)
        if (pending & (1ull << (m * NB + i))) {
          v[m][i] = ld_word(p + m * sm + i * si);
          if (tag_is(v[m][i], tag)) pending &= ~(1ull << (m * NB + i));
        }
    if (pending && global_timer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// ---- the fallback grid barrier ---------------------------------------------------
__device__ __forceinline__ unsigned long long ld_acquire_gpu_u64(const unsigned long long* p) {
  unsigned long long v;
  asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}

// All threads call it; thread 0 counts the run's barriers in *s_nbar (the
// run's base of the arrival counter in *s_base).  Returns false when this CTA
// is aborting.
__device__ __forceinline__ bool chain_barrier(const ChainParams& cp, volatile int* s_abort,
                                              unsigned long long* s_nbar, const unsigned long long* s_base) {
  __syncthreads();
  if (threadIdx.x == 0 && !*s_abort) {
    const unsigned long long target = *s_base + (++*s_nbar) * static_cast<unsigned long long>(cp.G);
    __threadfence();  // this CTA's writes before its arrival
    atomicAdd(cp.bar_count, 1ull);
    const unsigned long long t0 = global_timer_ns();
    while (ld_acquire_gpu_u64(cp.bar_count) < target) {
      if (global_timer_ns() - t0 > cp.timeout_ns) {
        *s_abort = 1;
        atomicOr(cp.status, kStatusTimeout);
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  return !*s_abort;
}

// ---- walking a warp's stages of every product -----------------------------
// In product e the warp takes the blocks [range_begin(pw), range_begin(pw + 1))
// of its own stream-K split (SU chunks per block and stage).
template <int SU>
struct ChainCursor {
  int pe = -1;
  int left = 0;  // a warp's stages in one product are far below 2^31
  const uint8_t* src = nullptr;
  uint32_t bytes = 0;

  __device__ __forceinline__ bool next(const StackEntryDev* entries, int E, int pw, const uint8_t** s,
                                       uint32_t* b) {
    while (left == 0) {
      if (pe + 1 >= E) return false;
      ++pe;
      const StackEntryDev& en = entries[pe];
      if (pw >= en.P) continue;
      const long long TB = en.TC / SU;
      const long long first = range_begin(pw, TB, en.P);
      const int CB = en.bits == 8 ? Format<8>::kChunkBytes : Format<4>::kChunkBytes;
      src = en.packed + first * SU * CB;
      left = static_cast<int>(range_begin(pw + 1, TB, en.P) - first);
      bytes = static_cast<uint32_t>(SU * CB);
    }
    *s = src;
    *b = bytes;
    src += bytes;
    --left;
    return true;
  }
};

// The ring's producer: copies the next stage into a slot (lane 0) and, PF
// stages further on, prefetches one more stage into L2.
template <int SU, int PF>
struct ChainProducer {
  const StackEntryDev* entries;
  int E;
  int pw;
  ChainCursor<SU> ring, ahead;

  template <class SP>
  __device__ __forceinline__ bool issue(const SP&, uint32_t dst, uint32_t bar, uint64_t policy, int lane, bool,
                                        const uint16_t**, uint32_t*) {
    const uint8_t* s;
    uint32_t b;
    if (!ring.next(entries, E, pw, &s, &b)) return false;
    bulk_copy_g2s_if(lane == 0, dst, s, b, bar, policy);
    if constexpr (PF > 0) {
      const uint8_t* a;
      uint32_t nb;
      if (ahead.next(entries, E, pw, &a, &nb) && lane == 0) bulk_prefetch_l2(a, nb);
    }
    return true;
  }
};

// ---- small helpers ------------------------------------------------------------
__device__ __forceinline__ float warp_sum_xor(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// 1 / sqrt(mean square + eps) from the sum of squares of a row of N values.
__device__ __forceinline__ float rms_factor(float ss, int N) {
  return 1.f / sqrtf(ss / static_cast<float>(N) + 1e-6f);
}

// silu(g) * u rounded to bf16 (bits).
__device__ __forceinline__ uint16_t swiglu_bf16(float g, float u) {
  const float silu = g / (1.f + expf(-g));
  return __bfloat16_as_ushort(__float2bfloat16_rn(silu * u));
}

// Index of (m, k) in an activation buffer laid out [K/KC][M][KC].
template <int M>
__device__ __forceinline__ int x_index(int m, int k, int KC) {
  if constexpr (M == 1) {
    return k;
  } else {
    const int c = k / KC;
    return (c * M + m) * KC + (k - c * KC);
  }
}

// The fp16-exactness scan (xprep_kernel's rule) of bf16 values.
struct XScan {
  int emax = INT_MIN, lsb = INT_MAX, bad = 0;
  __device__ __forceinline__ void add(uint32_t b16) { xprep_scan(b16, emax, lsb, bad); }
};

// Block-wide decision: the warps' partial scans meet in shared memory (one
// CTA synchronisation) and every thread combines them in the same order.
template <int NW>
__device__ __forceinline__ void chain_x_decision(XScan s, int* s_red, int& ok, int& sigma) {
  for (int o = 16; o > 0; o >>= 1) {
    s.emax = max(s.emax, __shfl_xor_sync(0xFFFFFFFFu, s.emax, o));
    s.lsb = min(s.lsb, __shfl_xor_sync(0xFFFFFFFFu, s.lsb, o));
    s.bad |= __shfl_xor_sync(0xFFFFFFFFu, s.bad, o);
  }
  const int warp = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {
    s_red[warp] = s.emax;
    s_red[NW + warp] = s.lsb;
    s_red[2 * NW + warp] = s.bad;
  }
  __syncthreads();
  int emax = INT_MIN, lsb = INT_MAX, bad = 0;
#pragma unroll
  for (int w = 0; w < NW; ++w) {
    emax = max(emax, s_red[w]);
    lsb = min(lsb, s_red[NW + w]);
    bad |= s_red[2 * NW + w];
  }
  sigma = 0;
  ok = !bad;
  if (emax != INT_MIN) {
    sigma = emax - 15;
    ok = ok && (lsb - sigma >= -24);
  }
}

// bf16 bits -> fp16 bits of x * 2^-sigma (exact by the decision: the value is
// below 2^16 and a multiple of 2^-24).
__device__ __forceinline__ uint32_t bf16_to_f16_scaled(uint32_t b16, int sigma) {
  const float v = __uint_as_float(b16 << 16);
  if (sigma >= -126 && sigma <= 126) return __half_as_ushort(__float2half_rn(v * pow2_float(-sigma)));
  return __half_as_ushort(__double2half(static_cast<double>(v) * ldexp(1.0, -sigma)));
}

// In place: the n bf16 values of the buffer -> fp16 (n % 8 == 0).  Ends with
// the CTA synchronised.
template <int NW>
__device__ __forceinline__ void chain_x_to_f16(uint16_t* xs, int n, int sigma) {
  uint4* x8 = reinterpret_cast<uint4*>(xs);
  for (int i = threadIdx.x; i < n / 8; i += NW * 32) {
    uint4 v = x8[i];
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q)
      w[q] = bf16_to_f16_scaled(w[q] & 0xFFFF, sigma) | (bf16_to_f16_scaled(w[q] >> 16, sigma) << 16);
    x8[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();
}

// Decides fp16 or bf16 for the buffer's n bf16 values and converts them; the
// next product's outputs are multiplied by `scale` (2^sigma, or 1 for bf16).
template <int NW>
__device__ __forceinline__ void chain_x_finish(uint16_t* xs, int n, const XScan& s, int* s_red, bool& f16,
                                               float& scale) {
  int ok, sigma;
  chain_x_decision<NW>(s, s_red, ok, sigma);
  f16 = ok != 0;
  scale = f16 ? pow2_float(sigma) : 1.f;
  if (f16)
    chain_x_to_f16<NW>(xs, n, sigma);
  else
    __syncthreads();
}

// The CTA's slice [lo, hi) of n items: the global writes it owns.
__device__ __forceinline__ void cta_slice(int n, int G, int& lo, int& hi) {
  lo = static_cast<int>(static_cast<long long>(n) * blockIdx.x / G);
  hi = static_cast<int>(static_cast<long long>(n) * (blockIdx.x + 1) / G);
}

// The warp's scratch: a tile's values turned from the mma layout into rows.
template <int M>
__device__ __forceinline__ float* warp_scratch(const ChainParams& cp) {
  extern __shared__ __align__(128) unsigned char smem[];
  return reinterpret_cast<float*>(smem + cp.scr_off) + (threadIdx.x >> 5) * (M * kTileRows);
}

// ---- the steps' elementwise parts ------------------------------------------
// RMSNorm on tile t (lane = row, values v[m] of the input y; has_y false: no
// input, h unchanged): h <- h_prev + y (or y when set), with h_prev the
// previous norm's tagged words (or the stream as the launch found it), into
// the step's tagged h words (and the caller's buffer at the stream's last
// norm).  run_base: this run's tag of op -1.  Returns false if a wait gave up
// (warp-uniform).
template <int M>
__device__ __forceinline__ bool resid_tile(const ChainParams& cp, const ChainOpDev& sop, uint32_t tag,
                                           uint32_t run_base, int t, const float (&v)[M], bool has_y, int lane,
                                           const unsigned long long* hw = nullptr) {
  const int N = sop.N;
  const int row = t * kTileRows + lane;
  float hp[M];
  bool got = true;
  if (!sop.set) {
    if (sop.src_op >= 0) {
      const ChainOpDev& prev = cp.ops[sop.src_op];
      const uint32_t ptag = run_base + static_cast<uint32_t>(sop.src_op) + 1u;
      unsigned long long w[M];
      bool have = hw != nullptr;  // loaded earlier by the caller
#pragma unroll
      for (int m = 0; m < M; ++m) {
        if (have) w[m] = hw[m];
        have = have && (row >= N || tag_is(w[m], ptag));
      }
      if (!have)
        got = poll_words<M>(cp.words + prev.tw + (row < N ? row : 0), N, row < N ? M : 0, ptag, w, cp.timeout_ns);
#pragma unroll
      for (int m = 0; m < M; ++m) hp[m] = __uint_as_float(static_cast<uint32_t>(w[m]));
    } else {
#pragma unroll
      for (int m = 0; m < M; ++m) hp[m] = row < N ? __ldcg(sop.h_src + static_cast<long long>(m) * N + row) : 0.f;
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float hv = 0.f;
    if (row < N) {
      hv = sop.set ? v[m] : (has_y ? hp[m] + v[m] : hp[m]);
      if (sop.h_dst) sop.h_dst[static_cast<long long>(m) * N + row] = hv;
      st_word(cp.words + sop.tw + static_cast<long long>(m) * N + row, tagged(tag, __float_as_uint(hv)));
    }
  }
  return __all_sync(0xFFFFFFFFu, got);
}

// SwiGLU on one pair p of 32-value slices (lane = value, gate g[m], up u[m]):
// the bf16 outputs, plain and as tagged pairs.
template <int M>
__device__ __forceinline__ void swiglu_pair(const ChainParams& cp, const ChainOpDev& sop, uint32_t tag, int p,
                                            const float (&g)[M], const float (&u)[M], int lane) {
  const int F = sop.N;
  const int k = p * kTileRows + lane;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const uint32_t b = k < F ? swiglu_bf16(g[m], u[m]) : 0u;
    if (k < F) sop.out[static_cast<long long>(m) * F + k] = static_cast<uint16_t>(b);
    const uint32_t hi = __shfl_down_sync(0xFFFFFFFFu, b, 1);
    if ((lane & 1) == 0 && k < F)
      st_word(cp.words + sop.tw + (static_cast<long long>(m) * F + k) / 2, tagged(tag, b | (hi << 16)));
  }
}

// The owner of finished tile t of a product with an epilogue (lane = row, the
// tile's final values v[m], already stored in y).  Returns false if a wait
// gave up.
template <int M>
__device__ __forceinline__ bool tile_epilogue(const ChainParams& cp, const ChainOpDev& sop, int epi, uint32_t tag,
                                              uint32_t run_base, int t, const float (&v)[M], int lane,
                                              unsigned long long timeout_ns, const unsigned long long* hw = nullptr) {
  if (epi == kEpiResid) return resid_tile<M>(cp, sop, tag, run_base, t, v, true, lane, hw);
  // kEpiSwiglu: tile t holds gate rows (t < TF) or up rows of pair t mod TF
  const int F = sop.N;
  const int TF = F / kTileRows;
  if (t >= TF) {  // up rows: tagged for the gate tile's owner
    const int p = t - TF;
#pragma unroll
    for (int m = 0; m < M; ++m)
      st_word(cp.words + sop.uw + static_cast<long long>(m) * F + p * kTileRows + lane,
              tagged(tag, __float_as_uint(v[m])));
    return true;
  }
  unsigned long long w[M];
  const bool got = poll_words<M>(cp.words + sop.uw + t * kTileRows + lane, F, M, tag, w, timeout_ns);
  if (!__all_sync(0xFFFFFFFFu, got)) return false;  // warp-uniform before the shuffles below
  float u[M];
#pragma unroll
  for (int m = 0; m < M; ++m) u[m] = __uint_as_float(static_cast<uint32_t>(w[m]));
  swiglu_pair<M>(cp, sop, tag, t, v, u, lane);
  return true;
}

// A tile's values from the mma accumulator layout (as store_tile) to lane =
// row, through the warp's scratch.
template <int M>
__device__ __forceinline__ void tile_rows(const float (&acc)[2][4], float* scr, int lane, float (&v)[M]) {
  const int gi = lane >> 2, ti = lane & 3;
  const int m0 = 2 * ti, m1 = 2 * ti + 1;
  __syncwarp();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row0 = 16 * h + gi, row1 = row0 + 8;
    if (m0 < M) {
      scr[m0 * kTileRows + row0] = acc[h][0];
      scr[m0 * kTileRows + row1] = acc[h][2];
    }
    if (m1 < M) {
      scr[m1 * kTileRows + row0] = acc[h][1];
      scr[m1 * kTileRows + row1] = acc[h][3];
    }
  }
  __syncwarp();
#pragma unroll
  for (int m = 0; m < M; ++m) v[m] = scr[m * kTileRows + lane];
}

// A warp's partial sums of a tile it does not own: tagged, in the mma layout
// (as write_partial), in its slot of the product's partial buffer.
template <int M>
__device__ __forceinline__ void write_partial_tagged(unsigned long long* parts, uint32_t tag, int pw,
                                                     const float (&acc)[2][4], int lane) {
  const int gi = lane >> 2, ti = lane & 3;
  const int m0 = 2 * ti, m1 = 2 * ti + 1;
  unsigned long long* mine = parts + static_cast<long long>(pw) * (M * kTileRows);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int row0 = 16 * h + gi, row1 = row0 + 8;
    if (m0 < M) {
      st_word(mine + m0 * kTileRows + row0, tagged(tag, __float_as_uint(acc[h][0])));
      st_word(mine + m0 * kTileRows + row1, tagged(tag, __float_as_uint(acc[h][2])));
    }
    if (m1 < M) {
      st_word(mine + m1 * kTileRows + row0, tagged(tag, __float_as_uint(acc[h][1])));
      st_word(mine + m1 * kTileRows + row1, tagged(tag, __float_as_uint(acc[h][3])));
    }
  }
}

// stream_segment's hooks for the chain: a tile finished inside the range is
// stored and gets the epilogue of the step after the product; the partial of
// the range's first tile (begun in an earlier warp's range) is written tagged.
struct ChainTileStore {
  const ChainParams* cp;
  const ChainOpDev* sop;
  int epi;
  uint32_t step_tag;  // the step's tag (its words)
  uint32_t run_base;  // this run's tag of op -1
  mutable bool ok;    // false once a wait gave up

  template <int M>
  __device__ __forceinline__ void store(const StackEntryDev* __restrict__ ep, int r, const float (&acc)[2][4],
                                        int lane) const {
    store_tile<M>(ep->y, ep->N, r, acc, lane);
    if (epi != kEpiNone) {
      float v[M];
      tile_rows<M>(acc, warp_scratch<M>(*cp), lane, v);
      if (!tile_epilogue<M>(*cp, *sop, epi, step_tag, run_base, r, v, lane, cp->timeout_ns)) ok = false;
    }
  }
  template <int M, class SP>
  __device__ __forceinline__ void first_partial(const SP& sp, int pw, const float (&acc)[2][4], int lane) const {
    write_partial_tagged<M>(sp.parts, sp.tag, pw, acc, lane);
  }
};

// The end of warp pw's range [b, ...) of one product: the partial of its last
// tile when the tile began before the range (a middle contributor), or, when
// the tile began inside the range (the warp owns it), the owner's sum: its
// own values, then the other contributors' tagged partials in warp order.
// (The first tile's partial was written by the segment.)  Returns false if a
// wait gave up.
template <int M>
__device__ __forceinline__ bool chain_finish_product(const ChainParams& cp, const ChainSegParams& sp,
                                                     const StackEntryDev* ep, long long TB, int SU, long long b,
                                                     int r, int c, float scale, float (&acc)[2][4], int pw, int lane,
                                                     const ChainTileStore& ts) {
  if (c == 0) return true;  // the range ended at a tile boundary: nothing open
  const int bpt = ep->C / SU;
  const long long tg = static_cast<long long>(r) * bpt;  // the tile's first block
  scale_acc(acc, scale);
  if (tg < b) {  // began in an earlier warp's range: that warp owns it
    write_partial_tagged<M>(sp.parts, sp.tag, pw, acc, lane);
    return true;
  }
  // this warp owns the tile; contributors pw + 1 .. p_hi wrote their slots.
  // The residual rows its epilogue adds to are loaded first, so that round
  // trip overlaps the wait for the partials.
  unsigned long long hw[M];
  bool have_h = false;
  if (ts.epi == kEpiResid && !ts.sop->set && ts.sop->src_op >= 0) {
    const int N = ts.sop->N;
    const long long hrow = static_cast<long long>(r) * kTileRows + lane;
    const unsigned long long* hp = cp.words + cp.ops[ts.sop->src_op].tw + (hrow < N ? hrow : 0);
#pragma unroll
    for (int m = 0; m < M; ++m) hw[m] = ld_word(hp + static_cast<long long>(m) * N);
    have_h = true;
  }
  float sum[M];
  tile_rows<M>(acc, warp_scratch<M>(cp), lane, sum);
  const int p_hi = owner_of(tg + bpt - 1, TB, ep->P);
  constexpr int GQ = 16 / M;  // contributors whose words one round trip loads (16 words)
  bool got = true;
  for (int q0 = pw + 1; q0 <= p_hi; q0 += GQ) {
    const int nq = min(GQ, p_hi - q0 + 1);
    // word j * M + m: contributor q0 + j, row m (parts[q][m][lane])
    unsigned long long w[GQ * M];
    unsigned pending = 0;
#pragma unroll
    for (int j = 0; j < GQ; ++j)
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const unsigned long long* p = sp.parts + static_cast<long long>(q0 + j) * (M * kTileRows) + m * kTileRows + lane;
        w[j * M + m] = j < nq ? ld_word(p) : tagged(sp.tag, 0u);
        if (!tag_is(w[j * M + m], sp.tag)) pending |= 1u << (j * M + m);
      }
    if (pending) {
      const unsigned long long t0 = global_timer_ns();
      while (pending) {
#pragma unroll
        for (int j = 0; j < GQ; ++j)
#pragma unroll
          for (int m = 0; m < M; ++m)
            if (pending & (1u << (j * M + m))) {
              w[j * M + m] = ld_word(sp.parts + static_cast<long long>(q0 + j) * (M * kTileRows) + m * kTileRows + lane);
              if (tag_is(w[j * M + m], sp.tag)) pending &= ~(1u << (j * M + m));
            }
        if (pending && global_timer_ns() - t0 > cp.timeout_ns) {
          got = false;
          break;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < GQ; ++j)
#pragma unroll
      for (int m = 0; m < M; ++m)
        if (j < nq) sum[m] += __uint_as_float(static_cast<uint32_t>(w[j * M + m]));
  }
  if (!__all_sync(0xFFFFFFFFu, got)) return false;  // warp-uniform before the epilogue's shuffles
  const long long row = static_cast<long long>(r) * kTileRows + lane;
#pragma unroll
  for (int m = 0; m < M; ++m)
    if (row < ep->N) ep->y[m * ep->N + row] = sum[m];
  if (ts.epi != kEpiNone)
    return tile_epilogue<M>(cp, *ts.sop, ts.epi, ts.step_tag, ts.run_base, r, sum, lane, cp.timeout_ns,
                            have_h ? hw : nullptr);
  return true;
}

// ---- the steps, in every CTA -------------------------------------------------
// RMSNorm: the step's tagged h words, their sum of squares in the fixed
// association (each warp's lanes at one value index are one tile: the tile's
// butterfly sum goes to shared memory, and every warp then adds the tile sums
// lane by lane in order and takes the butterfly, as the norm kernel does),
// then x = bf16(h * r * gamma) into the activation buffer (and the CTA's
// slice of out), then fp16 when exact.  h stays in registers when the row
// fits one batch (B values per thread), else it is read again.  Returns false
// if a wait gave up.
template <int M, int NW>
__device__ __forceinline__ bool chain_norm_finish(const ChainParams& cp, const ChainOpDev& op, uint32_t tag,
                                                  uint16_t* xs, float* s_tiles, int* s_red, bool& f16,
                                                  float& scale) {
  constexpr int T = NW * 32;
  constexpr int B = M == 1 ? 10 : (M == 2 ? 10 : (M == 3 ? 7 : 5));  // values of k per thread and batch
  const int N = op.N;
  const int tiles = (N + kTileRows - 1) / kTileRows;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const bool one = N <= T * B;
  bool ok = true;
  float hv[M][B];
  for (int base = 0; base < N; base += T * B) {
    const int k0 = base + threadIdx.x;
    const int nb = k0 < N ? min(B, (N - k0 + T - 1) / T) : 0;
    unsigned long long w[M][B];
    ok = poll_words2<M, B>(cp.words + op.tw + k0, N, T, nb, tag, w, cp.timeout_ns) && ok;
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int i = 0; i < B; ++i) {
        hv[m][i] = i < nb ? __uint_as_float(static_cast<uint32_t>(w[m][i])) : 0.f;
        // value i of this warp's lanes is tile (base + T i) / 32 + warp
        const int t = (base + i * T) / kTileRows + warp;
        const float sq = warp_sum_xor(__fmul_rn(hv[m][i], hv[m][i]));
        if (lane == 0 && t < tiles) s_tiles[m * tiles + t] = sq;
      }
  }
  __syncthreads();
  float r[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    float ssum = 0.f;
    for (int t = lane; t < tiles; t += 32) ssum += s_tiles[m * tiles + t];
    r[m] = rms_factor(warp_sum_xor(ssum), N);
  }
  int lo, hi;
  cta_slice(N, cp.G, lo, hi);
  XScan s;
  for (int base = 0; base < N; base += T * B) {
    const int k0 = base + threadIdx.x;
    const int nb = k0 < N ? min(B, (N - k0 + T - 1) / T) : 0;
    // gamma first, into registers: the loop below stores to out, which the
    // compiler cannot prove distinct from gamma, so a load inside it would
    // wait out the store before it
    float g[B];
#pragma unroll
    for (int i = 0; i < B; ++i)
      g[i] = (op.gamma && i < nb) ? __uint_as_float(static_cast<uint32_t>(__ldg(op.gamma + k0 + i * T)) << 16) : 1.f;
    if (!one) {  // h again (its words are complete)
#pragma unroll
      for (int m = 0; m < M; ++m)
#pragma unroll
        for (int i = 0; i < B; ++i)
          hv[m][i] = i < nb ? __uint_as_float(static_cast<uint32_t>(
                                  ld_word(cp.words + op.tw + static_cast<long long>(m) * N + k0 + i * T)))
                            : 0.f;
    }
#pragma unroll
    for (int m = 0; m < M; ++m) {
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const int k = k0 + i * T;
        if (i < nb) {
          float o = __fmul_rn(hv[m][i], r[m]);
          if (op.gamma) o = __fmul_rn(o, g[i]);
          const uint16_t bv = __bfloat16_as_ushort(__float2bfloat16_rn(o));
          s.add(bv);
          if (k >= lo && k < hi) op.out[static_cast<long long>(m) * N + k] = bv;
          xs[x_index<M>(m, k, op.kc)] = bv;
        }
      }
    }
  }
  chain_x_finish<NW>(xs, M * N, s, s_red, f16, scale);
  return ok;
}

// SwiGLU: its tagged output pairs into the activation buffer, then fp16 when
// exact.  Returns false if a wait gave up.
template <int M, int NW>
__device__ __forceinline__ bool chain_swiglu_finish(const ChainParams& cp, const ChainOpDev& op, uint32_t tag,
                                                    uint16_t* xs, int* s_red, bool& f16, float& scale) {
  constexpr int T = NW * 32;
  constexpr int B = M == 1 ? 17 : (M == 2 ? 9 : (M == 3 ? 6 : 5));  // words (two values each) per thread and poll
  const int F = op.N;
  const int nw = F / 2;
  XScan s;
  bool ok = true;
  for (int base = 0; base < nw; base += T * B) {
    unsigned long long w[M][B];
    const int i0 = base + threadIdx.x;
    ok = poll_words2<M, B>(cp.words + op.tw + i0, nw, T, i0 < nw ? min(B, (nw - i0 + T - 1) / T) : 0, tag, w,
                           cp.timeout_ns) && ok;
#pragma unroll
    for (int m = 0; m < M; ++m)
#pragma unroll
      for (int j = 0; j < B; ++j) {
        const int i = i0 + j * T;
        if (i < nw) {
          const uint32_t pair = static_cast<uint32_t>(w[m][j]);
          s.add(pair & 0xFFFF);
          s.add(pair >> 16);
          *reinterpret_cast<uint32_t*>(xs + x_index<M>(m, 2 * i, op.kc)) = pair;
        }
      }
  }
  chain_x_finish<NW>(xs, M * F, s, s_red, f16, scale);
  return ok;
}

// A product's activations: bf16 [M][K] (K % 8 == 0, row-major) from global or
// shared memory into the activation buffer laid out for chunks of KC, then
// fp16 when exact.
template <int M, int NW, bool SHARED_SRC>
__device__ __forceinline__ void chain_load_x(const uint16_t* src, int K, int KC, uint16_t* xs, int* s_red, bool& f16,
                                             float& scale) {
  constexpr int T = NW * 32;
  constexpr int V = 4;  // 16-byte groups per thread and batch
  const int k8 = K / 8;
  XScan s;
#pragma unroll
  for (int m = 0; m < M; ++m) {
    const uint4* src8 = reinterpret_cast<const uint4*>(src + static_cast<long long>(m) * K);
    for (int base = 0; base < k8; base += T * V) {
      uint4 v[V];
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int i = base + threadIdx.x + q * T;
        v[q] = i < k8 ? (SHARED_SRC ? src8[i] : __ldcg(src8 + i)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int i = base + threadIdx.x + q * T;
        if (i < k8) {
          const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            s.add(w[e] & 0xFFFF);
            s.add(w[e] >> 16);
          }
          *reinterpret_cast<uint4*>(xs + x_index<M>(m, 8 * i, KC)) = v[q];
        }
      }
    }
  }
  chain_x_finish<NW>(xs, M * K, s, s_red, f16, scale);
}

// The launch's first work: a staged product's activations (an input of the
// launch: no op writes them) converted once, as chain_load_x would, into a
// prepared copy in global memory (chunk-major, fp16 when exact) with its
// decision; a bulk copy brings it into the activation buffer later.  The
// CTA's activation buffer serves as the staging area.
template <int M, int NW>
__device__ __forceinline__ void chain_prepare(const ChainParams& cp, int j, uint16_t* xs, int* s_red) {
  const ChainOpDev& op = cp.ops[cp.prep_ops[j]];
  const int K = static_cast<int>(cp.entries[op.entry].K);
  bool f16;
  float scale;
  chain_load_x<M, NW, false>(op.x, K, op.kc, xs, s_red, f16, scale);  // ends synchronised
  uint4* dst = reinterpret_cast<uint4*>(cp.prep + op.prep_at);
  const uint4* src = reinterpret_cast<const uint4*>(xs);
  for (int i = threadIdx.x; i < M * K / 8; i += NW * 32) dst[i] = src[i];
  if (threadIdx.x == 0) {
    int sigma = 0;
    if (f16) sigma = static_cast<int>((__float_as_uint(scale) >> 23) & 0xFF) - 127;  // scale = 2^sigma, normal
    if (f16 && scale < 1.17549435e-38f) sigma = -149 + 31 - __clz(static_cast<int>(__float_as_uint(scale)));
    cp.prep_info[2 * j] = f16 ? 1 : 0;
    cp.prep_info[2 * j + 1] = sigma;
  }
  __syncthreads();
}

// A step whose input is not the preceding product's output: its elementwise
// part split between the CTAs (one warp per tile or pair).
template <int M, int NW>
__device__ __forceinline__ bool chain_step_slices(const ChainParams& cp, const ChainOpDev& op, uint32_t tag,
                                                  uint32_t run_base, int warp, int lane) {
  bool ok = true;
  const int N = op.N;
  const int tiles = (N + kTileRows - 1) / kTileRows;
  int lo, hi;
  cta_slice(tiles, cp.G, lo, hi);
  for (int t = lo + warp; t < hi; t += NW) {
    const int k = t * kTileRows + lane;
    if (op.kind == kChainRmsnorm) {
      float v[M];
#pragma unroll
      for (int m = 0; m < M; ++m) v[m] = (op.y && k < N) ? __ldcg(op.y + static_cast<long long>(m) * N + k) : 0.f;
      ok = resid_tile<M>(cp, op, tag, run_base, t, v, op.y != nullptr, lane) && ok;
    } else {
      float g[M], u[M];
#pragma unroll
      for (int m = 0; m < M; ++m) {
        g[m] = k < N ? __ldcg(op.y + 2LL * m * N + k) : 0.f;
        u[m] = k < N ? __ldcg(op.y + 2LL * m * N + N + k) : 0.f;
      }
      swiglu_pair<M>(cp, op, tag, t, g, u, lane);
    }
  }
  return ok;
}

// ---- the kernel -------------------------------------------------------------
template <int M, int NW, int D, int SU, int PF>
__global__ void __launch_bounds__(NW * 32, 1) chain_kernel(const ChainParams cp) {
  constexpr int FC = 3;  // q4 / q8 products, activations resident in shared memory
  constexpr int SLOT = StreamSlot<SU, M, FC>::kBytes;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  __shared__ unsigned s_run;
  __shared__ unsigned long long s_base;  // the fallback barrier: this run's base of the arrival counter
  __shared__ unsigned long long s_nbar;  // barriers passed in this run
  __shared__ __align__(8) unsigned long long s_xbar;  // the prefetched activations' copy
  __shared__ int s_red[3 * NW];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pw = blockIdx.x * NW + warp;
  StreamRing rg;
  rg.ring = smem_addr(smem + warp * D * SLOT);
  rg.bars = smem_addr(smem + NW * D * SLOT) + warp * D * 8;
  rg.rx = smem_addr(smem + cp.x_off);
  const uint32_t xbar = smem_addr(&s_xbar);

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_run = cp.run_ctr[blockIdx.x] + 1u;  // every CTA counts the same runs
    // every run adds G arrivals per barrier, so the counter is a multiple of
    // G between runs; other CTAs may already have arrived at this run's first
    // barrier (fewer than G of them), none can have passed it
    const unsigned long long c0 = ld_acquire_gpu_u64(cp.bar_count);
    s_base = c0 - c0 % static_cast<unsigned long long>(cp.G);
    s_nbar = 0;
  }
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(rg.bars + 8 * s, 1);
    if (warp == 0) mbar_init(xbar, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const uint64_t policy = l2_evict_first_policy();

  // the ring's first D stages, then PF stages beyond them into L2
  ChainProducer<SU, PF> pr{cp.entries, cp.E, pw};
  if constexpr (PF > 0) {
    for (int s = 0; s < D + PF; ++s) {
      const uint8_t* a;
      uint32_t nb;
      if (!pr.ahead.next(cp.entries, cp.E, pw, &a, &nb)) break;
      if (s >= D && lane == 0) bulk_prefetch_l2(a, nb);
    }
  }
  for (int s = 0; s < D; ++s) {
    const uint8_t* src;
    uint32_t nb;
    if (!pr.ring.next(cp.entries, cp.E, pw, &src, &nb)) break;
    bulk_copy_g2s_if(lane == 0, rg.ring + s * SLOT, src, nb, rg.bars + 8 * s, policy);
    ++rg.in_flight;
  }

  bool f16 = false;
  float scale = 1.f;
  uint32_t xpar = 0;       // parity of the prefetch barrier's next phase
  bool x_pending = false;  // a prefetch copy is in flight
  bool ok = true;          // this warp's waits all ended in time
  if (cp.n_prep > 0) {
    // the staged products' activations, prepared by the CTAs in turn; one
    // grid barrier makes them visible, and a proxy fence orders them before
    // the bulk copies that read them
    uint16_t* xs = reinterpret_cast<uint16_t*>(smem + cp.x_off);
    for (int j = blockIdx.x; j < cp.n_prep; j += cp.G) chain_prepare<M, NW>(cp, j, xs, s_red);
    chain_barrier(cp, &s_abort, &s_nbar, &s_base);
    if (threadIdx.x == 0) asm volatile("fence.proxy.async.global;" ::: "memory");
  }
  for (int oi = 0; oi < cp.n_ops; ++oi) {
    const ChainOpDev* __restrict__ opp = cp.ops + oi;  // fields are read where used, not held in registers
    const int kind = opp->kind;
    if (!ok && lane == 0) {
      atomicOr(cp.status, kStatusTimeout);
      atomicOr(&s_abort, 1);
    }
    if (opp->barrier) {
      if (!chain_barrier(cp, &s_abort, &s_nbar, &s_base)) break;
    } else if (kind != kChainProduct || (opp->stage_x && opp->pre_off < 0)) {
      __syncthreads();  // the op writes the activation buffer that warps of the op before may still read
      if (s_abort) break;
    } else if (*static_cast<volatile int*>(&s_abort)) {
      break;
    }
    // op i's tag in this run (never 0, the words' initial tag)
    const uint32_t tag = s_run * static_cast<uint32_t>(cp.n_ops) + static_cast<uint32_t>(oi) + 1u;
    // the activations of the next, staged product: one bulk copy into the
    // buffer's tail, which this op does not use
    const int pre_next = opp->pre_next;
    if (pre_next >= 0) {
      if (threadIdx.x == 0) {
        const ChainOpDev* nx = cp.ops + pre_next;
        const uint32_t bytes = static_cast<uint32_t>(M * cp.entries[nx->entry].K * 2);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // earlier generic accesses of the tail
        mbar_arrive_expect_tx(xbar, bytes);
        bulk_copy_x_if(true, rg.rx + static_cast<uint32_t>(nx->pre_off), cp.prep + nx->prep_at, bytes, xbar);
      }
      x_pending = true;
    }
    const uint32_t run_base = s_run * static_cast<uint32_t>(cp.n_ops);
    if (kind != kChainProduct) {
      const ChainOpDev op = *opp;
      uint16_t* xs = reinterpret_cast<uint16_t*>(smem + cp.x_off);
      if (!op.epi) ok = chain_step_slices<M, NW>(cp, op, tag, run_base, warp, lane);
      float* s_tiles = reinterpret_cast<float*>(smem + cp.tiles_off);
      ok = (kind == kChainRmsnorm ? chain_norm_finish<M, NW>(cp, op, tag, xs, s_tiles, s_red, f16, scale)
                                  : chain_swiglu_finish<M, NW>(cp, op, tag, xs, s_red, f16, scale)) && ok;
      ok = __all_sync(0xFFFFFFFFu, ok);
      continue;
    }
    const int entry = opp->entry;
    const StackEntryDev* __restrict__ ep = cp.entries + entry;
    if (opp->stage_x) {
      uint16_t* xs = reinterpret_cast<uint16_t*>(smem + cp.x_off);
      const int K = static_cast<int>(ep->K);
      const int pre_off = opp->pre_off;
      if (pre_off >= 0) {  // prepared, and copied in during the op before: read in place
        ok = mbar_wait_bounded(xbar, xpar, cp.timeout_ns);
        xpar ^= 1u;
        x_pending = false;
        if (!ok) continue;  // the next op stops the CTA
        const int j = opp->prep;
        f16 = cp.prep_info[2 * j] != 0;
        scale = f16 ? pow2_float(cp.prep_info[2 * j + 1]) : 1.f;
      } else {
        chain_load_x<M, NW, false>(opp->x, K, opp->kc, xs, s_red, f16, scale);
      }
    }
    if (pw >= ep->P) continue;
    const long long TB = ep->TC / SU;
    const long long b = range_begin(pw, TB, ep->P);
    const long long n = range_begin(pw + 1, TB, ep->P) - b;
    const ChainSegParams sp{cp.timeout_ns, cp.parts + opp->pbuf * cp.pbuf_words, tag};
    const int epi = opp->epi;
    ChainTileStore ts{&cp, nullptr, epi, 0u, run_base, true};
    if (epi != kEpiNone) {
      const int step = opp->step;
      ts.sop = cp.ops + step;
      ts.step_tag = run_base + static_cast<uint32_t>(step) + 1u;
    }
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int e_first = -1, r_first = -1, r = 0, c = 0;
    bool seg;
    if (ep->bits == 4)
      seg = f16 ? stream_segment<4, M, D, SU, true, FC>(sp, ep, entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                        e_first, r_first, r, c, lane, ts)
                : stream_segment<4, M, D, SU, false, FC>(sp, ep, entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                         e_first, r_first, r, c, lane, ts);
    else
      seg = f16 ? stream_segment<8, M, D, SU, true, FC>(sp, ep, entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                        e_first, r_first, r, c, lane, ts)
                : stream_segment<8, M, D, SU, false, FC>(sp, ep, entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                         e_first, r_first, r, c, lane, ts);
    ok = seg && ts.ok && chain_finish_product<M>(cp, sp, ep, TB, SU, b, r, c, scale, acc, pw, lane, ts);
  }
  if (!ok && lane == 0) {
    atomicOr(cp.status, kStatusTimeout);
    atomicOr(&s_abort, 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) cp.run_ctr[blockIdx.x] = s_run;
  if (s_abort) {
    // wait (bounded) for the activation copy and this warp's weight copies
    // still in flight, then leave
    if (x_pending) mbar_wait_bounded(xbar, xpar, cp.timeout_ns);
    for (int k = 0; k < rg.in_flight; ++k) {
      if (!mbar_wait_bounded(rg.bars + 8 * rg.slot, rg.phase, cp.timeout_ns)) break;
      if (++rg.slot == D) {
        rg.slot = 0;
        rg.phase ^= 1u;
      }
    }
  }
}

}  // namespace q4k
