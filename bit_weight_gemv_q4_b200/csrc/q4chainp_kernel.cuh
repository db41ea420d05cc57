// The dependent decode chain (products with residual + RMSNorm and SwiGLU
// steps between them) as ONE persistent cooperative kernel, M = 1.
//
// The pages describe the decode step as a 64-layer sequence of weight
// streams (ai-coding.wiselychen.com guide, section "Before deploying";
// bs178.com llamAmpere post, "Why it is this fast") whose products depend on
// one another through the layer's normalisation and gated MLP.  Launched one
// kernel per op, every product pays a launch, a ramp-up and a tail.  Here one
// CTA per SM walks the whole op list:
//  * A product is split between all warps stream-K style, exactly as a
//    one-product stream-mode stack splits it (same ranges, same fp16 decode of
//    resident activations, same split-tile fix-up), so each output is bitwise
//    the stream-mode product of the same activations.
//  * Each warp's bulk-copy ring runs ahead ACROSS ops: weights never depend
//    on activations, so while the CTA waits at a barrier or computes a step,
//    the next product's first stages are already landing.
//  * A step reads a product's output only after a grid-wide barrier (every
//    tile and split-tile fix-up of that product written).  Every CTA then
//    computes the whole step itself, into its own shared-memory copy of the
//    next product's activations: no second barrier, and the residual stream h
//    lives in each CTA's shared memory for the whole launch (loaded once at
//    the start, each CTA writing its slice back to global memory as it
//    changes).  The steps follow residual_rmsnorm_kernel and swiglu_kernel
//    operation for operation (the sum of squares in the same association), so
//    their outputs are bitwise those kernels' outputs on the same inputs.
//  * Every wait is bounded: a ring wait that gives up marks the CTA aborted,
//    the CTA stops at its next synchronisation point, drains its copies
//    (bounded) and exits; the other CTAs' barrier waits then give up too, and
//    the status word records the time-out.
#pragma once

#include <climits>

#include "q4chain_kernel.cuh"
#include "q4stack_kernel.cuh"

namespace q4k {

constexpr int kChainProduct = 0;
constexpr int kChainRmsnorm = 1;
constexpr int kChainSwiglu = 2;
// The host admits grids of up to 32 x kChainFlagsPerLane CTAs (one polling
// warp, a few flags per lane per poll; B200 has 148 SMs).
constexpr int kChainFlagsPerLane = 8;

struct ChainOpDev {
  int kind;      // kChainProduct / kChainRmsnorm / kChainSwiglu
  int barrier;   // a grid barrier precedes the op
  int stage_x;   // product: copy x from global memory into the CTA's activation buffer first
  int entry;     // product: its StackEntryDev
  int pbuf;      // product: split-tile partial buffer (0 / 1)
  int set;       // RMSNorm: h <- y instead of h <- h + y
  int N;         // steps: output row length
  int h_off;     // RMSNorm: offset of its residual stream in shared memory (floats)
  const uint16_t* x;      // product: bf16 [K] (read when stage_x)
  const float* y;         // steps: fp32 input (RMSNorm: [N] or null; SwiGLU: [2N])
  const uint16_t* gamma;  // RMSNorm: bf16 [N] or null
  uint16_t* out;          // steps: bf16 [N]
  float* resid;           // RMSNorm: h, fp32 [N]
};

struct ChainResid {
  const float* h;  // its value at launch
  int N;
  int h_off;       // floats
};

struct ChainParams {
  const ChainOpDev* ops;
  int n_ops;
  const StackEntryDev* entries;  // the products, in op order (blk_off 0: each is its own sequence)
  int E;
  const ChainResid* resids;
  int n_resids;
  float* partials;        // [2][warps][2][32]
  long long pbuf_floats;  // floats per partial buffer
  unsigned* counters;     // one per tile of every product
  unsigned* status;
  unsigned* bar_flags;    // [G] per-CTA barrier epochs
  int G;
  int x_off;   // dynamic shared memory: byte offset of the activation buffer
  int h_base;  // byte offset of the residual streams
  unsigned long long timeout_ns;
};

// What stream_segment reads from its parameters.
struct ChainSegParams {
  unsigned long long timeout_ns;
  float* partials;
};

// The warp's stages of every product in op order: in product e, the blocks
// [range_begin(pw), range_begin(pw + 1)) of its own stream-K split.
template <int SU>
struct ChainProducer {
  const StackEntryDev* entries;
  int E;
  int pw;
  int pe = -1;
  long long left = 0;
  const uint8_t* src = nullptr;
  uint32_t bytes = 0;

  template <class SP>
  __device__ __forceinline__ bool issue(const SP&, uint32_t dst, uint32_t bar, uint64_t policy, int lane, bool,
                                        const uint16_t**, uint32_t*) {
    while (left == 0) {
      if (pe + 1 >= E) return false;
      ++pe;
      const StackEntryDev& en = entries[pe];
      if (pw >= en.P) continue;
      const long long TB = en.TC / SU;
      const long long b = range_begin(pw, TB, en.P);
      const int CB = en.bits == 8 ? Format<8>::kChunkBytes : Format<4>::kChunkBytes;
      src = en.packed + b * SU * CB;
      left = range_begin(pw + 1, TB, en.P) - b;
      bytes = static_cast<uint32_t>(SU * CB);
    }
    bulk_copy_g2s_if(lane == 0, dst, src, bytes, bar, policy);
    src += bytes;
    --left;
    return true;
  }
};

// Grid-wide barrier of the G resident CTAs (all threads call it).  CTA b
// publishes `epoch` in its own flag (release store after a fence), and one
// warp polls every flag with acquire loads.  The acquire loads of a poll
// complete one after another, which keeps the polling rate low: the 148
// flags share five cache lines, and polling them with every load in flight
// at once delayed the late CTAs' arrival stores (9 % slower on the 64-layer
// chain).  Bounded by timeout_ns.  Returns false when this CTA is aborting.
__device__ __forceinline__ bool chain_barrier(const ChainParams& cp, unsigned epoch, volatile int* s_abort) {
  __syncthreads();
  if (threadIdx.x < 32 && !*s_abort) {
    const int lane = threadIdx.x;
    if (lane == 0) {
      __threadfence();
      st_release_gpu(cp.bar_flags + blockIdx.x, epoch);
    }
    __syncwarp();
    const unsigned long long t0 = global_timer_ns();
    while (true) {
      bool here = true;
      for (int i = lane; i < cp.G; i += 32) here &= static_cast<int>(ld_acquire_gpu(cp.bar_flags + i) - epoch) >= 0;
      if (__all_sync(0xFFFFFFFFu, here)) break;
      const unsigned long long waited = __shfl_sync(0xFFFFFFFFu, global_timer_ns() - t0, 0);
      if (waited > cp.timeout_ns) {
        if (lane == 0) {
          *s_abort = 1;
          atomicOr(cp.status, kStatusTimeout);
        }
        break;
      }
    }
    __threadfence();
  }
  __syncthreads();
  return !*s_abort;
}

// ---- the activation buffer: bf16 values written by the CTA, then, when
// fp16-exact after a power-of-two scaling, converted in place (the rule of
// xprep_kernel: sigma = emax - 15, exact iff lsb - sigma >= -24, no inf / NaN)

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

// In place: the K bf16 values of the buffer -> fp16 x * 2^-sigma (exact by
// the decision).  K % 8 == 0.  Ends with the CTA synchronised.
template <int NW>
__device__ __forceinline__ void chain_x_to_f16(uint16_t* xs, int K, int sigma) {
  const double down = ldexp(1.0, -sigma);
  uint4* x8 = reinterpret_cast<uint4*>(xs);
  for (int i = threadIdx.x; i < K / 8; i += NW * 32) {
    uint4 v = x8[i];
    uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double lo = static_cast<double>(__uint_as_float(w[q] << 16)) * down;
      const double hi = static_cast<double>(__uint_as_float(w[q] & 0xFFFF0000u)) * down;
      w[q] = static_cast<uint32_t>(__half_as_ushort(__double2half(lo))) |
             (static_cast<uint32_t>(__half_as_ushort(__double2half(hi))) << 16);
    }
    x8[i] = make_uint4(w[0], w[1], w[2], w[3]);
  }
  __syncthreads();
}

// Decides fp16 or bf16 for the buffer and converts it; the product's outputs
// are multiplied by `scale` (2^sigma, or 1 for bf16).
template <int NW>
__device__ __forceinline__ void chain_x_finish(uint16_t* xs, int K, const XScan& s, int* s_red, bool& f16,
                                               float& scale) {
  int ok, sigma;
  chain_x_decision<NW>(s, s_red, ok, sigma);
  f16 = ok != 0;
  scale = f16 ? pow2_float(sigma) : 1.f;
  if (f16)
    chain_x_to_f16<NW>(xs, K, sigma);
  else
    __syncthreads();
}

// The CTA's slice [lo, hi) of a length-N row: the global writes it owns.
__device__ __forceinline__ void cta_slice(int N, int G, int& lo, int& hi) {
  lo = static_cast<int>(static_cast<long long>(N) * blockIdx.x / G);
  hi = static_cast<int>(static_cast<long long>(N) * (blockIdx.x + 1) / G);
}

// Values per thread and batch in the steps: every global load of a batch is
// issued before any of its results is used or any store is made (a store to
// global memory between two loads would keep the compiler from overlapping
// them: each would wait out its own round trip to L2).
constexpr int kChainBatch = 16;

// A product's activations from global memory (bf16 [K], K % 8 == 0).
template <int NW>
__device__ __forceinline__ void chain_stage_x(const uint16_t* x, int K, uint16_t* xs, int* s_red, bool& f16,
                                              float& scale) {
  constexpr int T = NW * 32;
  XScan s;
  const uint4* src = reinterpret_cast<const uint4*>(x);
  uint4* dst = reinterpret_cast<uint4*>(xs);
  const int n8 = K / 8;
  for (int base = 0; base < n8; base += T * kChainBatch / 2) {
    uint4 v[kChainBatch / 2];
#pragma unroll
    for (int q = 0; q < kChainBatch / 2; ++q) {
      const int i = base + threadIdx.x + q * T;
      v[q] = i < n8 ? src[i] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int q = 0; q < kChainBatch / 2; ++q) {
      const int i = base + threadIdx.x + q * T;
      if (i < n8) {
        dst[i] = v[q];
        const uint32_t w[4] = {v[q].x, v[q].y, v[q].z, v[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          s.add(w[e] & 0xFFFF);
          s.add(w[e] >> 16);
        }
      }
    }
  }
  chain_x_finish<NW>(xs, K, s, s_red, f16, scale);
}

// Residual + RMSNorm (M = 1), the arithmetic of residual_rmsnorm_kernel: its
// 1024 threads are emulated by the NW * 32 = 512 threads here, thread t
// taking the values of threads t and t + 512 (k = t + 512 i: i even belongs
// to thread t, i odd to thread t + 512), each of the two sums taken in its
// own increasing order, reduced by the same shuffle tree, and the 32 warp
// sums added in warp order.
template <int NW>
__device__ __forceinline__ void chain_rmsnorm(const ChainOpDev& op, int G, float* hs, uint16_t* xs, float* s_part,
                                              int* s_red, bool& f16, float& scale) {
  constexpr int T = NW * 32;
  static_assert(T * 2 == kNormThreads, "the emulated norm kernel has twice this CTA's threads");
  static_assert(kChainBatch % 2 == 0, "batches hold whole pairs of the emulated threads' values");
  const int t = threadIdx.x;
  const int N = op.N;
  float* h = hs + op.h_off;
  const float* y = op.y;
  float ss[2] = {0.f, 0.f};
  for (int base = 0; base < N; base += T * kChainBatch) {
    float yv[kChainBatch];
#pragma unroll
    for (int i = 0; i < kChainBatch; ++i) {
      const int k = base + t + i * T;
      yv[i] = (y && k < N) ? y[k] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kChainBatch; ++i) {
      const int k = base + t + i * T;
      if (k < N) {
        const float v = op.set ? yv[i] : (y ? h[k] + yv[i] : h[k]);
        h[k] = v;
        ss[i & 1] = fmaf(v, v, ss[i & 1]);
      }
    }
  }
#pragma unroll
  for (int half = 0; half < 2; ++half)
    for (int o = 16; o > 0; o >>= 1) ss[half] += __shfl_xor_sync(0xFFFFFFFFu, ss[half], o);
  if ((t & 31) == 0) {
    s_part[t >> 5] = ss[0];
    s_part[NW + (t >> 5)] = ss[1];
  }
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int w = 0; w < 2 * NW; ++w) tot += s_part[w];
  const float r = 1.f / sqrtf(tot / static_cast<float>(N) + 1e-6f);
  int lo, hi;
  cta_slice(N, G, lo, hi);
  XScan s;
  for (int base = 0; base < N; base += T * kChainBatch) {
    uint32_t g[kChainBatch];
#pragma unroll
    for (int i = 0; i < kChainBatch; ++i) {
      const int k = base + t + i * T;
      g[i] = (op.gamma && k < N) ? op.gamma[k] : 0u;
    }
#pragma unroll
    for (int i = 0; i < kChainBatch; ++i) {
      const int k = base + t + i * T;
      if (k < N) {
        const float v = h[k];
        float o = v * r;
        if (op.gamma) o *= __uint_as_float(g[i] << 16);
        const uint16_t b = __bfloat16_as_ushort(__float2bfloat16_rn(o));
        xs[k] = b;
        s.add(b);
        if (k >= lo && k < hi) {
          op.out[k] = b;
          op.resid[k] = v;
        }
      }
    }
  }
  chain_x_finish<NW>(xs, N, s, s_red, f16, scale);
}

// SwiGLU (M = 1), the arithmetic of swiglu_kernel.
template <int NW>
__device__ __forceinline__ void chain_swiglu(const ChainOpDev& op, int G, uint16_t* xs, int* s_red, bool& f16,
                                             float& scale) {
  constexpr int T = NW * 32;
  const int N = op.N;
  int lo, hi;
  cta_slice(N, G, lo, hi);
  XScan s;
  for (int base = 0; base < N; base += T * kChainBatch) {
    float g[kChainBatch], u[kChainBatch];
#pragma unroll
    for (int i = 0; i < kChainBatch; ++i) {
      const int k = base + threadIdx.x + i * T;
      g[i] = k < N ? op.y[k] : 0.f;
      u[i] = k < N ? op.y[N + k] : 0.f;
    }
#pragma unroll
    for (int i = 0; i < kChainBatch; ++i) {
      const int k = base + threadIdx.x + i * T;
      if (k < N) {
        const float silu = g[i] / (1.f + expf(-g[i]));
        const uint16_t b = __bfloat16_as_ushort(__float2bfloat16_rn(silu * u[i]));
        xs[k] = b;
        s.add(b);
        if (k >= lo && k < hi) op.out[k] = b;
      }
    }
  }
  chain_x_finish<NW>(xs, N, s, s_red, f16, scale);
}

// The split tiles of warp pw's range [b, e) of one product, as at the end of
// stream_kernel (the first one's partial is already in slot 0).
__device__ __forceinline__ void chain_finish_product(const ChainParams& cp, const ChainSegParams& sp,
                                                     const StackEntryDev* ep, long long TB, int SU, long long b,
                                                     int r_first, int r, int c, float scale, float (&acc)[2][4],
                                                     int pw, int lane) {
  const int bpt = ep->C / SU;
  SplitTile first{nullptr, 0, -1, cp.counters, 0, 0}, last{nullptr, 0, -1, cp.counters, 0, 0};
  if (r_first >= 0) {
    const long long tg = static_cast<long long>(r_first) * bpt;
    first = SplitTile{ep->y, ep->N, r_first, cp.counters + ep->tile_off + r_first, tg, tg + bpt};
  }
  if (c != 0) {
    const long long tg = static_cast<long long>(r) * bpt;
    last = SplitTile{ep->y, ep->N, r, cp.counters + ep->tile_off + r, tg, tg + bpt};
    scale_acc(acc, scale);
    write_partial<1>(sp.partials, pw, tg <= b ? 0 : 1, acc, lane);
  }
  if (first.r < 0 && last.r < 0) return;
  __threadfence();
  __syncwarp();
  unsigned a_first = 0, a_last = 0;
  if (lane == 0) {
    if (first.r >= 0) a_first = atomicAdd(first.counter, 1u);
    if (last.r >= 0) a_last = atomicAdd(last.counter, 1u);
  }
  a_first = __shfl_sync(0xFFFFFFFFu, a_first, 0);
  a_last = __shfl_sync(0xFFFFFFFFu, a_last, 0);
  const Partition pt{TB, ep->P, sp.partials};
  const bool red_first = first.r >= 0 && a_first + 1 == tile_contributors(pt, first);
  const bool red_last = last.r >= 0 && a_last + 1 == tile_contributors(pt, last);
  if (red_first || red_last) __threadfence();
  if (red_first) reduce_tile<1>(pt, first, lane);
  if (red_last) reduce_tile<1>(pt, last, lane);
}

template <int NW, int D, int SU>
__global__ void __launch_bounds__(NW * 32, 1) chain_kernel(const ChainParams cp) {
  constexpr int M = 1;
  constexpr int FC = 3;  // q4 / q8 products, activations resident in shared memory
  constexpr int SLOT = StreamSlot<SU, M, FC>::kBytes;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  __shared__ unsigned s_epoch0;
  __shared__ float s_part[2 * NW];
  __shared__ int s_red[3 * NW];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pw = blockIdx.x * NW + warp;
  StreamRing rg;
  rg.ring = smem_addr(smem + warp * D * SLOT);
  rg.bars = smem_addr(smem + NW * D * SLOT) + warp * D * 8;
  rg.rx = smem_addr(smem + cp.x_off);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + cp.x_off);
  float* hs = reinterpret_cast<float*>(smem + cp.h_base);

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_epoch0 = ld_acquire_gpu(cp.bar_flags + blockIdx.x);  // this CTA's last epoch of the previous run
  }
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(rg.bars + 8 * s, 1);
    fence_barrier_init();
  }
  for (int i = 0; i < cp.n_resids; ++i) {
    const ChainResid rs = cp.resids[i];
    for (int base = 0; base < rs.N; base += NW * 32 * kChainBatch) {
      float v[kChainBatch];
#pragma unroll
      for (int q = 0; q < kChainBatch; ++q) {
        const int k = base + threadIdx.x + q * NW * 32;
        v[q] = k < rs.N ? rs.h[k] : 0.f;
      }
#pragma unroll
      for (int q = 0; q < kChainBatch; ++q) {
        const int k = base + threadIdx.x + q * NW * 32;
        if (k < rs.N) hs[rs.h_off + k] = v[q];
      }
    }
  }
  __syncthreads();
  const unsigned epoch0 = s_epoch0;
  const uint64_t policy = l2_evict_first_policy();

  ChainProducer<SU> pr{cp.entries, cp.E, pw};
  for (int s = 0; s < D; ++s) {
    if (!pr.issue(cp, rg.ring + s * SLOT, rg.bars + 8 * s, policy, lane, true, nullptr, nullptr)) break;
    ++rg.in_flight;
  }

  unsigned n_bar = 0;
  bool f16 = false;
  float scale = 1.f;
  for (int oi = 0; oi < cp.n_ops; ++oi) {
    const ChainOpDev op = cp.ops[oi];
    if (op.barrier) {
      if (!chain_barrier(cp, epoch0 + (++n_bar), &s_abort)) break;
    } else {
      __syncthreads();
      if (s_abort) break;
    }
    if (op.kind == kChainRmsnorm) {
      chain_rmsnorm<NW>(op, cp.G, hs, xs, s_part, s_red, f16, scale);
      continue;
    }
    if (op.kind == kChainSwiglu) {
      chain_swiglu<NW>(op, cp.G, xs, s_red, f16, scale);
      continue;
    }
    const StackEntryDev* __restrict__ ep = cp.entries + op.entry;
    if (op.stage_x) chain_stage_x<NW>(op.x, static_cast<int>(ep->K), xs, s_red, f16, scale);
    const long long TB = ep->TC / SU;
    if (pw >= ep->P) continue;
    const long long b = range_begin(pw, TB, ep->P);
    const long long n = range_begin(pw + 1, TB, ep->P) - b;
    const ChainSegParams sp{cp.timeout_ns, cp.partials + op.pbuf * cp.pbuf_floats};
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int e_first = -1, r_first = -1, r = 0, c = 0;
    bool ok;
    if (ep->bits == 4)
      ok = f16 ? stream_segment<4, M, D, SU, true, FC>(sp, ep, op.entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                       e_first, r_first, r, c, lane)
               : stream_segment<4, M, D, SU, false, FC>(sp, ep, op.entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                        e_first, r_first, r, c, lane);
    else
      ok = f16 ? stream_segment<8, M, D, SU, true, FC>(sp, ep, op.entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                       e_first, r_first, r, c, lane)
               : stream_segment<8, M, D, SU, false, FC>(sp, ep, op.entry, b, n, b, rg, pr, policy, scale, acc, pw,
                                                        e_first, r_first, r, c, lane);
    if (!ok) {
      if (lane == 0) {
        atomicOr(cp.status, kStatusTimeout);
        atomicOr(&s_abort, 1);
      }
      continue;  // the next op's synchronisation stops the CTA
    }
    chain_finish_product(cp, sp, ep, TB, SU, b, r_first, r, c, scale, acc, pw, lane);
  }
  __syncthreads();
  if (s_abort) {
    // wait (bounded) for this warp's copies still in flight, then leave
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
