// The layer stack as ONE persistent cooperative kernel.
//
// A decode step is an ordered list of products (the 64 layers' q|k|v, o,
// gate|up, down, then the output head).  Launching one kernel per product
// pays a launch, a prologue and a tail per product; here one CTA per SM runs
// the whole list:
//  * For each product every warp streams its stream-K range exactly as the
//    single-product kernel does (same ranges, same arithmetic, same fix-up),
//    so every output is bitwise equal to the corresponding q4_gemv / q8_gemv.
//  * The warp's bulk-copy ring runs ahead ACROSS products: while a warp
//    finishes product e (and waits at the barrier below), the first stages of
//    its range in product e+1 are already in flight.  Weights never depend on
//    activations, so prefetching them early is always valid.
//  * Between products a grid-wide barrier (generation counter, bounded wait)
//    guarantees that every output of product e, including the split-tile
//    fix-ups, is written before any warp reads product e+1's activations:
//    the same ordering as a stream of one launch per product.
//  * Every wait is bounded.  A warp whose ring wait gives up marks the CTA
//    aborted; the CTA stops at the next barrier, drains its in-flight copies
//    (bounded) and exits; the other CTAs' barrier waits then give up too.
#pragma once

#include <climits>

#include "q4gemv_kernels.cuh"
#include "q4nvfp4_kernel.cuh"
#include "q4wide_kernel.cuh"

namespace q4k {

// Activation preparation for stream mode (xprep_kernel).  An activation
// tensor is used in fp16 when a power of two 2^sigma exists with every
// x * 2^-sigma exactly representable in fp16: then x16 = x * 2^-sigma, and
// outputs computed from x16 are multiplied back by scale = 2^sigma (exact).
// Otherwise (a dynamic range beyond fp16's, inf or NaN) ok = 0 and the
// products of that tensor use the bf16 path on x itself.
struct XInfo {
  int ok;
  int sigma;
  float scale;
  int pad;
};

// xc: the activations chunk-major, [K/KC][M][KC] (KC = k per chunk of the
// product's format), so the slice of a stage of chunks is one contiguous
// copy: fp16 x * 2^-sigma when info->ok, else the bf16 x itself.
struct XPrepJob {
  const uint16_t* x;  // bf16 [M][K]
  uint16_t* xc;       // [K/KC][M][KC]
  XInfo* info;
  long long K;
  int KC;
  int rx_off;         // stream mode: offset of xc's copy in a group's shared memory, or -1 (not that group's)
};

struct StackEntryDev {
  const uint8_t* packed;
  const uint16_t* x;
  float* y;
  const uint16_t* xc;    // stream mode: chunk-major activations (XPrepJob)
  const XInfo* xinfo;    // stream mode
  long long N, K, TC;
  long long blk_off;  // first block of this product in the concatenated sequence (stream mode)
  int T, C, bits, P, khalf;
  int tile_off;       // first counter of this product (stream mode)
  int rx_off;         // stream mode with resident activations: their offset in shared memory
};

struct StackParams {
  const StackEntryDev* entries;
  int E;
  float* partials;      // [P][2][M][32]
  unsigned* counters;   // one per tile of the largest product (re-zeroed as used)
  unsigned* status;
  unsigned* bar_flags;  // ordered mode: [G] per-CTA barrier epochs
  int G;                // CTAs in the grid (all resident: cooperative launch)
  unsigned long long timeout_ns;
  long long TBg;        // stream mode: blocks of all products, concatenated
  int Pg;               // stream mode: warps with work
  const XPrepJob* jobs; // stream mode with resident activations: the prepared activations to stage
  int n_jobs;
  int rx_bytes;         // their bytes in shared memory
};

constexpr int kStackU = 2;                                   // chunks per stage
constexpr int kStackSlotBytes = kStackU * Format<4>::kChunkBytes;  // the larger of the two formats

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// L2 prefetch of a contiguous byte range (no shared memory involved).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Walks one warp's stages of all products in order: (source, bytes) of the
// next stage.  Warp-uniform state.
struct StageCursor {
  int pe = -1;
  int left = 0;
  const uint8_t* src = nullptr;
  uint32_t bytes = 0;

  __device__ __forceinline__ bool next(const StackParams& sp, int pw, const uint8_t** out_src, uint32_t* out_bytes);
};

__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier of the G resident CTAs; all threads of the CTA call it.
// CTA b announces its arrival at barrier `epoch` by storing the epoch
// (release) in its own flag, and passes once every CTA's flag has reached it
// (acquire loads, one warp polling all G flags): no atomic, no contention on
// one address.  Epochs only grow: each run continues from the last epoch its
// CTA stored.  Returns false when this CTA is aborting (its own abort flag,
// or a wait that gave up).
__device__ __forceinline__ bool grid_barrier(const StackParams& sp, unsigned epoch, int* s_abort) {
  __syncthreads();
  if (threadIdx.x < 32 && !*s_abort) {
    const int lane = threadIdx.x;
    if (lane == 0) {
      __threadfence();  // this CTA's outputs before its arrival
      st_release_gpu(sp.bar_flags + blockIdx.x, epoch);
    }
    __syncwarp();
    const unsigned long long t0 = global_timer_ns();
    while (true) {
      bool here = true;
      for (int i = lane; i < sp.G; i += 32) here &= static_cast<int>(ld_acquire_gpu(sp.bar_flags + i) - epoch) >= 0;
      if (__all_sync(0xFFFFFFFFu, here)) break;
      const unsigned long long waited = __shfl_sync(0xFFFFFFFFu, global_timer_ns() - t0, 0);
      if (waited > sp.timeout_ns) {
        if (lane == 0) {
          *s_abort = 1;
          atomicOr(sp.status, kStatusTimeout);
        }
        break;
      }
    }
  }
  __syncthreads();
  return !*s_abort;
}

__device__ __forceinline__ bool StageCursor::next(const StackParams& sp, int pw, const uint8_t** out_src,
                                                  uint32_t* out_bytes) {
  while (left == 0) {
    if (pe + 1 >= sp.E) return false;
    ++pe;
    const StackEntryDev& en = sp.entries[pe];
    if (pw >= en.P) continue;
    const long long TB = en.TC / kStackU;
    const long long b = range_begin(pw, TB, en.P) * kStackU;
    const long long e = range_begin(pw + 1, TB, en.P) * kStackU;
    const int CB = en.bits == 4 ? Format<4>::kChunkBytes : Format<8>::kChunkBytes;
    src = en.packed + b * CB;
    left = static_cast<int>((e - b) / kStackU);
    bytes = static_cast<uint32_t>(kStackU * CB);
  }
  *out_src = src;
  *out_bytes = bytes;
  src += bytes;
  --left;
  return true;
}

// PF: how many stages ahead of the shared-memory ring the weights are
// prefetched into L2, so HBM keeps streaming while warps wait at a barrier.
template <int M, int NW, int D, int PF>
__global__ void __launch_bounds__(NW * 32, 1) stack_kernel(const StackParams sp) {
  constexpr int U = kStackU;
  constexpr int SLOT = kStackSlotBytes;
  extern __shared__ __align__(128) unsigned char smem[];
  __shared__ int s_abort;
  __shared__ unsigned s_epoch0;

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int gi = lane >> 2, ti = lane & 3;
  // interleaved over the CTAs, as in gemv_kernel: a product split between
  // fewer warps than the grid holds spreads them over every SM
  const int pw = warp * static_cast<int>(gridDim.x) + static_cast<int>(blockIdx.x);
  const uint32_t ring = smem_addr(smem + warp * D * SLOT);
  const uint32_t bars = smem_addr(smem + NW * D * SLOT) + warp * D * 8;

  if (threadIdx.x == 0) {
    s_abort = 0;
    s_epoch0 = ld_acquire_gpu(sp.bar_flags + blockIdx.x);  // the last barrier of the previous run
  }
  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(bars + 8 * s, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const unsigned epoch0 = s_epoch0;
  const uint64_t policy = l2_evict_first_policy();

  // ---- producer: the warp's stages of all products, in order; `ahead` runs
  // PF stages in front and only prefetches into L2
  StageCursor ring_cur, ahead;
  int g_issued = 0, g_consumed = 0;  // stages of this warp, all products
  for (int s = 0; s < D + PF; ++s) {
    const uint8_t* a;
    uint32_t nb;
    if (!ahead.next(sp, pw, &a, &nb)) break;
    if (s >= D && lane == 0) bulk_prefetch_l2(a, nb);
  }
  auto produce = [&]() {
    const uint8_t* src;
    uint32_t nbytes;
    if (!ring_cur.next(sp, pw, &src, &nbytes)) return;
    const int slot = g_issued % D;
    bulk_copy_g2s_if(lane == 0, ring + slot * SLOT, src, nbytes, bars + 8 * slot, policy);
    ++g_issued;
    if (PF > 0) {
      const uint8_t* a;
      uint32_t nb;
      if (ahead.next(sp, pw, &a, &nb) && lane == 0) bulk_prefetch_l2(a, nb);
    }
  };
  for (int s = 0; s < D; ++s) produce();

  grid_dependency_wait();
  grid_dependents_launch();

  for (int ei = 0; ei < sp.E; ++ei) {
    const StackEntryDev en = sp.entries[ei];
    const long long TB = en.TC / U;
    long long b = 0, e = 0;
    if (pw < en.P) {
      b = range_begin(pw, TB, en.P) * U;
      e = range_begin(pw + 1, TB, en.P) * U;
    }
    const int nst = static_cast<int>((e - b) / U);
    int r = static_cast<int>(floor_div(b, en.C));
    int c = static_cast<int>(b - static_cast<long long>(r) * en.C);
    const bool x_lane = gi < M;
    const uint16_t* xrow = en.x + static_cast<long long>(x_lane ? gi : 0) * en.K + 8 * ti;
    float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    float acc_first[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
    int r_first = -1;
    uint4 xa = make_uint4(0, 0, 0, 0), xb = make_uint4(0, 0, 0, 0);
    const int KC = en.bits == 4 ? Format<4>::kKPerChunk : Format<8>::kKPerChunk;
    const int CB = en.bits == 4 ? Format<4>::kChunkBytes : Format<8>::kChunkBytes;

    bool ok = true;
    for (int i = 0; i < nst; ++i) {
      const int slot = g_consumed % D;
      const uint32_t phase = static_cast<uint32_t>((g_consumed / D) & 1);
      if (!mbar_wait_bounded(bars + 8 * slot, phase, sp.timeout_ns)) {
        ok = false;
        break;
      }
      const uint32_t stage = ring + slot * SLOT;
      ChunkRegs regs[U];
      if (en.bits == 4) {
#pragma unroll
        for (int j = 0; j < U; ++j) {
          regs[j].codes[0] = lds128(stage + j * Format<4>::kChunkBytes + 16 * lane);
          regs[j].codes[1] = lds128(stage + j * Format<4>::kChunkBytes + kHalfBytes + 16 * lane);
          regs[j].scales = lds128(stage + j * Format<4>::kChunkBytes + kCodeBytes + 16 * gi);
        }
      } else {
#pragma unroll
        for (int j = 0; j < U; ++j) {
          regs[j].codes[0] = lds128(stage + j * Format<8>::kChunkBytes + 16 * lane);
          regs[j].codes[1] = lds128(stage + j * Format<8>::kChunkBytes + kHalfBytes + 16 * lane);
          const uint2 s2 = lds64(stage + j * Format<8>::kChunkBytes + kCodeBytes + 8 * gi);
          regs[j].scales = make_uint4(s2.x, s2.y, 0u, 0u);
        }
      }
      // every lane has read the slot; lane 0 refills it with the next stage
      __syncwarp();
      produce();
      ++g_consumed;
      (void)CB;
#pragma unroll
      for (int j = 0; j < U; ++j) {
        const uint16_t* xs = xrow + static_cast<long long>(c + j) * KC;
        ldg128_pred(xa, xs, x_lane);
        if (en.bits == 4) {
          const bool half_empty = en.khalf && c + j == en.C - 1;
          ldg128_pred(xb, xs + 32, x_lane && !half_empty);
          if (half_empty) xb = make_uint4(0, 0, 0, 0);
          q4_chunk_mac<false, (M > 1)>(acc, regs[j], xa, xb);
        } else {
          q8_chunk_mac<false, (M > 1)>(acc, regs[j], xa);
        }
      }
      c += U;
      if (c == en.C) {
        if (static_cast<long long>(r) * en.C < b) {
          r_first = r;
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int q = 0; q < 4; ++q) acc_first[h][q] = acc[h][q];
        } else {
          store_tile<M>(en.y, en.N, r, acc, lane);
        }
        ++r;
        c = 0;
#pragma unroll
        for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
      }
    }
    if (!ok) {
      if (lane == 0) {
        atomicOr(sp.status, kStatusTimeout);
        atomicOr(&s_abort, 1);
      }
    } else if (nst > 0) {
      int r_last = -1, slot_last = 1;
      if (c != 0) {
        r_last = r;
        slot_last = (static_cast<long long>(r) * en.C <= b) ? 0 : 1;
      }
      const Partition pt{TB, en.P, sp.partials};
      const int bpt = en.C / U;
      const SplitTile first{en.y, en.N, r_first, sp.counters + (r_first < 0 ? 0 : r_first),
                            static_cast<long long>(r_first) * bpt, static_cast<long long>(r_first + 1) * bpt};
      const SplitTile last{en.y, en.N, r_last, sp.counters + (r_last < 0 ? 0 : r_last),
                           static_cast<long long>(r_last) * bpt, static_cast<long long>(r_last + 1) * bpt};
      finish_split_tiles<M>(pt, pw, first, acc_first, last, slot_last, acc, lane);
    }
    // every output of this product is written before the next reads its input
    if (ei + 1 < sp.E) {
      if (!grid_barrier(sp, epoch0 + static_cast<unsigned>(ei) + 1u, &s_abort)) break;
    }
  }
  if (s_abort) {
    // wait (bounded) for this warp's copies still in flight, then leave
    for (int g = g_consumed; g < g_issued; ++g) {
      if (!mbar_wait_bounded(bars + 8 * (g % D), static_cast<uint32_t>((g / D) & 1), sp.timeout_ns)) break;
    }
  }
}

// ----------------------------------------------------------------------------
// xprep_kernel: grid (G, jobs).  Every CTA of a job scans the whole tensor
// (16-byte loads; the tensor is small and L2-resident) for the largest binary
// exponent emax and the lowest set significand bit lsb over the nonzero
// elements, so all G CTAs reach the same decision without a grid-wide sync;
// then CTA g writes its share of the chunk-major copy.  With
// sigma = emax - 15 every element scaled by 2^-sigma is below 2^16 in
// magnitude (fp16 max 65504 > 1.9921875 * 2^15), and it is exact in fp16 when
// its lowest set bit is at least 2^-24 (the fp16 subnormal step):
// lsb - sigma >= -24 for every element.
// ----------------------------------------------------------------------------
constexpr int kXPrepThreads = 1024;

__device__ __forceinline__ float pow2_float(int e) {  // 2^e for e in [-149, 127], built from its bits
  return e >= -126 ? __int_as_float((e + 127) << 23) : __int_as_float(1 << (e + 149));
}

__device__ __forceinline__ void xprep_scan(uint32_t b, int& emax, int& lsb, int& bad) {
  const int e = static_cast<int>((b >> 7) & 0xFF);
  const uint32_t f = b & 0x7F;
  if (e == 0xFF) {  // inf or NaN
    bad = 1;
  } else if (e != 0) {  // normal: (0x80 | f) * 2^(e - 134)
    emax = max(emax, e - 127);
    lsb = min(lsb, e - 134 + __ffs(static_cast<int>(0x80 | f)) - 1);
  } else if (f != 0) {  // subnormal: f * 2^-133
    emax = max(emax, -133 + 31 - __clz(static_cast<int>(f)));
    lsb = min(lsb, -133 + __ffs(static_cast<int>(f)) - 1);
  }
}

// M * K is a multiple of 8 and x is 16-byte aligned (K % 32 == 0 for every product).
__global__ void __launch_bounds__(kXPrepThreads) xprep_kernel(const XPrepJob* jobs, int M) {
  asm volatile("griddepcontrol.launch_dependents;");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ int s_emax[32], s_lsb[32], s_bad[32];
  __shared__ int s_ok, s_sigma;
  const XPrepJob j = jobs[blockIdx.y];
  const long long n8 = static_cast<long long>(M) * j.K / 8;  // 16-byte groups of 8 values
  const uint4* x8 = reinterpret_cast<const uint4*>(j.x);
  int emax = INT_MIN, lsb = INT_MAX, bad = 0;
  for (long long i = threadIdx.x; i < n8; i += blockDim.x) {
    const uint4 v = x8[i];
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      xprep_scan(w[q] & 0xFFFF, emax, lsb, bad);
      xprep_scan(w[q] >> 16, emax, lsb, bad);
    }
  }
  for (int o = 16; o > 0; o >>= 1) {
    emax = max(emax, __shfl_xor_sync(0xFFFFFFFFu, emax, o));
    lsb = min(lsb, __shfl_xor_sync(0xFFFFFFFFu, lsb, o));
    bad |= __shfl_xor_sync(0xFFFFFFFFu, bad, o);
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  if (lane == 0) {
    s_emax[warp] = emax;
    s_lsb[warp] = lsb;
    s_bad[warp] = bad;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < nw; ++w) {
      emax = max(emax, s_emax[w]);
      lsb = min(lsb, s_lsb[w]);
      bad |= s_bad[w];
    }
    int sigma = 0, ok = !bad;
    if (emax != INT_MIN) {
      sigma = emax - 15;
      ok = ok && (lsb - sigma >= -24);
    }
    s_ok = ok;
    s_sigma = sigma;
    if (blockIdx.x == 0) {
      j.info->ok = ok;
      j.info->sigma = sigma;
      j.info->scale = pow2_float(sigma);
    }
  }
  __syncthreads();
  const bool f16 = s_ok != 0;
  const double down = ldexp(1.0, -s_sigma);
  // this CTA's share: 16-byte groups [g0, g1); a group is 8 consecutive k of
  // one row, inside one chunk (KC is a multiple of 8), so it stays 16 contiguous
  // bytes in the chunk-major copy
  const long long per = (n8 + gridDim.x - 1) / gridDim.x;
  const long long g0 = per * blockIdx.x, g1 = min(n8, g0 + per);
  uint4* xc8 = reinterpret_cast<uint4*>(j.xc);
  const long long k8 = j.K / 8, kc8 = j.KC / 8;
  for (long long i = g0 + threadIdx.x; i < g1; i += blockDim.x) {
    uint4 v = x8[i];
    if (f16) {
      uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const double lo = static_cast<double>(__uint_as_float(w[q] << 16)) * down;
        const double hi = static_cast<double>(__uint_as_float(w[q] & 0xFFFF0000u)) * down;
        // exact by the test above
        w[q] = static_cast<uint32_t>(__half_as_ushort(__double2half(lo))) |
               (static_cast<uint32_t>(__half_as_ushort(__double2half(hi))) << 16);
      }
      v = make_uint4(w[0], w[1], w[2], w[3]);
    }
    const long long m = i / k8, k = i - m * k8;  // row, group of 8 within the row
    const long long chunk = k / kc8, kk = k - chunk * kc8;
    xc8[(chunk * M + m) * kc8 + kk] = v;
  }
}

// ----------------------------------------------------------------------------
// Stream mode: the products do not read each other's outputs, so the whole
// list is ONE stream-K problem.  Its blocks (SU chunks each) are concatenated
// product after product, and every warp streams one contiguous range of the
// concatenation, crossing product boundaries (which are tile boundaries)
// without any synchronisation.  Only the tiles holding a range's two ends are
// split between warps, so each warp finishes at most two split tiles, at the
// very end.  No grid barrier; every wait is a bounded ring wait.
// ----------------------------------------------------------------------------

// Product holding concatenated block gb (products are in block order).
__device__ __forceinline__ int entry_of_block(const StackParams& sp, long long gb) {
  int lo = 0, hi = sp.E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (sp.entries[mid].blk_off <= gb)
      lo = mid;
    else
      hi = mid - 1;
  }
  return lo;
}

// The producer side of a warp's ring in stream mode: the next stage (SU
// chunks) to copy in the warp's range, crossing products.  Warp-uniform state.
// A stage is SU chunks of weights followed, in the same slot and on the same
// mbarrier, by the matching activation slice (SU chunks x M rows x KC
// values, one contiguous copy from the chunk-major xc).
// Format classes of a stream-mode list: 0 = q4 / q8, 1 = also NVFP4, 2 = also
// q5 / q6.  A class's kernel carries only its formats' segments, and its slot
// fits the largest chunk among them.
template <int FC>
struct FormatClass {
  // classes 3 and 4 are classes 0 and 1 with resident activations: every CTA
  // copies each prepared activation tensor into shared memory once, and the
  // stages carry weights only
  static constexpr bool kResidentX = FC >= 3;
  static constexpr int kClass = FC >= 3 ? FC - 3 : FC;
  static constexpr int kMaxChunkBytes = kClass == 2 ? Wide<6>::kChunkBytes : Format<4>::kChunkBytes;
};

// Chunk bytes of a stack entry's format.
__device__ __forceinline__ int entry_chunk_bytes(int bits) {
  return bits == 8 ? Format<8>::kChunkBytes
                   : bits == 5 ? Wide<5>::kChunkBytes : bits == 6 ? Wide<6>::kChunkBytes : Format<4>::kChunkBytes;
}

template <int SU, int M, int FC>
struct StreamSlot {
  static constexpr int kWeightBytes = SU * FormatClass<FC>::kMaxChunkBytes;
  static constexpr int kXBytes = FormatClass<FC>::kResidentX ? 0 : SU * M * Format<4>::kKPerChunk * 2;
  static constexpr int kBytes = kWeightBytes + kXBytes;
};

// The producer side of a warp's ring in stream mode: the next stage (SU
// chunks) to copy in the warp's range, crossing products.  Warp-uniform state.
template <int SU, int M, int FC>
struct StreamProducer {
  int e = 0;                 // product of the next stage
  int left_entry = 0;        // stages left in that product
  long long left_total = 0;  // stages left in the range
  const uint8_t* src = nullptr;
  uint32_t bytes = 0;
  const uint16_t* xc = nullptr;  // the product's chunk-major activations
  int cpos = 0;                  // chunk of the tile where the next stage starts
  int C = 0, KC = 0;

  __device__ __forceinline__ void enter(const StackParams& sp, int entry, long long lb) {
    const StackEntryDev& en = sp.entries[entry];
    // NVFP4, q5 and q6 have the q4 geometry; only class 2 lists hold q5 / q6
    const int CB = FormatClass<FC>::kClass == 2 ? entry_chunk_bytes(en.bits)
                                                : (en.bits == 8 ? Format<8>::kChunkBytes : Format<4>::kChunkBytes);
    e = entry;
    bytes = static_cast<uint32_t>(SU * CB);
    src = en.packed + lb * SU * CB;
    const long long in_entry = en.TC / SU - lb;
    left_entry = static_cast<int>(in_entry < left_total ? in_entry : left_total);
    xc = en.xc;
    C = en.C;
    KC = en.bits == 8 ? Format<8>::kKPerChunk : Format<4>::kKPerChunk;
    const int bpt = en.C / SU;
    cpos = static_cast<int>(lb - static_cast<long long>(floor_div(lb, bpt)) * bpt) * SU;
  }
  __device__ __forceinline__ const uint16_t* x_src() const { return xc + static_cast<long long>(cpos) * M * KC; }
  __device__ __forceinline__ uint32_t x_bytes() const { return static_cast<uint32_t>(SU * M * KC * 2); }
  // Copies the next stage into the slot at `dst` (lane 0), completing on
  // `bar`; with_x = false leaves the activation slice for issue_x (before
  // griddepcontrol.wait, when the activations may not be ready yet), but the
  // barrier already expects its bytes.
  __device__ __forceinline__ bool issue(const StackParams& sp, uint32_t dst, uint32_t bar, uint64_t policy,
                                        int lane, bool with_x, const uint16_t** x_later, uint32_t* x_later_bytes) {
    if (left_total == 0) return false;
    if (left_entry == 0) enter(sp, e + 1, 0);
    if constexpr (FormatClass<FC>::kResidentX) {
      // the slots carry weights only; the activations are already resident
      bulk_copy_g2s_if(lane == 0, dst, src, bytes, bar, policy);
    } else {
      const uint32_t xb = x_bytes();
      bulk_copy_g2s_x_if(lane == 0, dst, src, bytes, dst + StreamSlot<SU, M, FC>::kWeightBytes, x_src(), xb, with_x,
                         bar, policy);
      if (!with_x) {
        *x_later = x_src();
        *x_later_bytes = xb;
      }
      cpos += SU;
      if (cpos == C) cpos = 0;
    }
    src += bytes;
    --left_entry;
    --left_total;
    return true;
  }
};

// Multiplies a tile's accumulators by a power of two (exact).
__device__ __forceinline__ void scale_acc(float (&acc)[2][4], float scale) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int q = 0; q < 4; ++q) acc[h][q] *= scale;
}

// The warp's ring: D slots of one stage each, and the stage counters; rx:
// the resident activations (classes 3 and 4).
struct StreamRing {
  uint32_t ring, bars, rx;
  int slot = 0;          // slot of the next stage to consume
  uint32_t phase = 0;
  int in_flight = 0;     // stages issued and not yet consumed
};

// Consumes `nblk` stages (SU chunks each) of one product (format BITS: 4, 8
// or kFmtNvfp4), from
// local block lb0.  Keeps the split-tile bookkeeping of the warp's range
// [gb, ...): the partial of a tile that began before gb goes to partial slot
// 0 when the tile ends (e_first, r_first); a tile still open at the end stays
// in acc with (r, c).  Returns false if a ring wait gave up.
// F16: the activations are used in fp16 (en.x16).  Finished tile sums are
// multiplied by `scale` (2^sigma when F16, times t for NVFP4).
// SP supplies timeout_ns and partials; PR refills the ring (issue), so the
// persistent chain kernel runs the same loop with its own per-product ranges;
// TS stores a tile finished inside the range (the chain adds its step's
// elementwise part there) and the partial of a tile that began in an earlier
// warp's range (the chain writes it with a tag).
struct TileStoreY {
  template <int M>
  __device__ __forceinline__ void store(const StackEntryDev* __restrict__ ep, int r, const float (&acc)[2][4],
                                        int lane) const {
    store_tile<M>(ep->y, ep->N, r, acc, lane);
  }
  template <int M, class SP>
  __device__ __forceinline__ void first_partial(const SP& sp, int pw, const float (&acc)[2][4], int lane) const {
    write_partial<M>(sp.partials, pw, 0, acc, lane);
  }
};

template <int BITS, int M, int D, int SU, bool F16, int FC, class SP = StackParams,
          class PR = StreamProducer<SU, M, FC>, class TS = TileStoreY>
__device__ __forceinline__ bool stream_segment(const SP& sp, const StackEntryDev* __restrict__ ep, int e,
                                               long long lb0,
                                               long long nblk, long long gb, StreamRing& rg,
                                               PR& pr, uint64_t policy, float scale,
                                               float (&acc)[2][4], int pw, int& e_first, int& r_first, int& r,
                                               int& c, int lane, const TS& ts = TS()) {
  constexpr int U = SU;
  constexpr int SLOT = StreamSlot<SU, M, FC>::kBytes;
  constexpr bool NV = BITS == kFmtNvfp4;
  constexpr bool WIDE = BITS == 5 || BITS == 6;
  constexpr int FB = BITS == 8 ? 8 : 4;  // NVFP4, q5 and q6 chunks have the q4 geometry
  constexpr int CB = WIDE ? Wide<WIDE ? BITS : 5>::kChunkBytes : Format<FB>::kChunkBytes;
  constexpr int KC = Format<FB>::kKPerChunk;
  const int gi = lane >> 2, ti = lane & 3;
  const int C = ep->C;  // the entry's other fields are read where they are used, not held in registers
  const int bpt = C / U;
  // this lane's B fragment in the slot's activation slice (or, resident, in
  // the chunk's slice of the tensor's copy): row min(gi, M-1) (columns >= M
  // only feed outputs that are never stored), 8 values at 8 ti
  constexpr bool RX = FormatClass<FC>::kResidentX;
  const uint32_t xrow = ((gi < M ? gi : M - 1) * KC + 8 * ti) * 2;
  const uint32_t xlane = StreamSlot<SU, M, FC>::kWeightBytes + xrow;
  const uint32_t xres = RX ? rg.rx + static_cast<uint32_t>(ep->rx_off) + xrow : 0u;
  r = static_cast<int>(floor_div(lb0, bpt));
  c = static_cast<int>(lb0 - static_cast<long long>(r) * bpt) * U;
  const int n_stages = static_cast<int>(nblk);  // a warp's range is far below 2^31 stages
  for (int i = 0; i < n_stages; ++i) {
    const uint32_t bar = rg.bars + 8 * rg.slot;
    if (!mbar_wait_bounded(bar, rg.phase, sp.timeout_ns)) return false;
    const uint32_t stage = rg.ring + rg.slot * SLOT;
#pragma unroll
    for (int j = 0; j < U; ++j) {
      ChunkRegs cr;
      const uint32_t xaddr = RX ? xres + static_cast<uint32_t>(c + j) * (M * KC * 2) : stage + xlane + j * M * KC * 2;
      const uint4 xa = lds128(xaddr);
      const uint4 xb = FB == 4 ? lds128(xaddr + 64) : make_uint4(0, 0, 0, 0);
      cr.codes[0] = lds128(stage + j * CB + 16 * lane);
      cr.codes[1] = lds128(stage + j * CB + kHalfBytes + 16 * lane);
      uint4 hi = make_uint4(0u, 0u, 0u, 0u);
      if (NV) {
        const uint2 s2 = lds64(stage + j * CB + kCodeBytes + 8 * (2 * gi + (ti >> 1)));
        cr.scales = make_uint4(s2.x, s2.y, 0u, 0u);
      } else if (WIDE) {
        hi = wide_load_hi<WIDE ? BITS : 5>(stage + j * CB, lane);
        cr.scales = lds128(stage + j * CB + Wide<WIDE ? BITS : 5>::kScaleBase + 16 * gi);
      } else if (BITS == 4) {
        cr.scales = lds128(stage + j * CB + kCodeBytes + 16 * gi);
      } else {
        const uint2 s2 = lds64(stage + j * CB + kCodeBytes + 8 * gi);
        cr.scales = make_uint4(s2.x, s2.y, 0u, 0u);
      }
      if (j == U - 1) {
        // every lane has read the slot; lane 0 refills it with the next stage
        __syncwarp();
        if (!pr.issue(sp, stage, bar, policy, lane, true, nullptr, nullptr)) --rg.in_flight;
        if (++rg.slot == D) {
          rg.slot = 0;
          rg.phase ^= 1u;
        }
      }
      if (NV) {
        nvfp4_chunk_mac<F16>(acc, cr.codes, make_uint2(cr.scales.x, cr.scales.y), xa, xb);
      } else if (WIDE) {
        wide_chunk_mac<WIDE ? BITS : 5, F16>(acc, cr.codes, hi, cr.scales, xa, xb);
      } else if (BITS == 4) {  // stream mode has whole q4 chunks only (K % 64 == 0, checked on the host)
        q4_chunk_mac<F16, (M > 1)>(acc, cr, xa, xb);
      } else {
        q8_chunk_mac<F16, (M > 1)>(acc, cr, xa);
      }
    }
    c += U;
    if (c == C) {
      if (F16 || NV) scale_acc(acc, scale);
      const long long tile_g = ep->blk_off + static_cast<long long>(r) * bpt;  // the tile's first block
      if (tile_g < gb) {  // began in an earlier warp's range: its partial goes to slot 0 now
        ts.template first_partial<M>(sp, pw, acc, lane);
        e_first = e;
        r_first = r;
      } else {
        ts.template store<M>(ep, r, acc, lane);
      }
      ++r;
      c = 0;
#pragma unroll
      for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
    }
  }
  return true;
}

// Thread 0 of a CTA: every resident prepared activation tensor of the list
// (rx_off >= 0: M rows of K values, chunk-major) into its place in shared
// memory, completing on xbar (armed for all their bytes, sp.rx_bytes).
// Called after griddepcontrol.wait (the preparation kernel has completed).
template <int M>
__device__ __forceinline__ void stage_resident_x(const StackParams& sp, uint32_t rx, uint32_t xbar) {
  mbar_arrive_expect_tx(xbar, static_cast<uint32_t>(sp.rx_bytes));
  for (int k = 0; k < sp.n_jobs; ++k) {
    const XPrepJob& j = sp.jobs[k];
    if (j.rx_off < 0) continue;
    const uint32_t bytes = static_cast<uint32_t>(M * j.K * 2);
    bulk_copy_x_if(true, rx + static_cast<uint32_t>(j.rx_off), j.xc, bytes, xbar);
  }
}

// SU: chunks per stage and per stream-K block (2 or 4; every product's
// chunks per tile is a multiple of SU, checked on the host).  FC: the list's
// format class (FormatClass): the NVFP4 and q5 / q6 segments are compiled
// only into the instances whose lists hold them, so lists of q4 / q8 products
// run the code without them.
template <int M, int NW, int D, int SU, int FC>
__global__ void __launch_bounds__(NW * 32, 1) stream_kernel(const StackParams sp) {
  constexpr int SLOT = StreamSlot<SU, M, FC>::kBytes;
  constexpr bool RX = FormatClass<FC>::kResidentX;
  extern __shared__ __align__(128) unsigned char smem[];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int pw = blockIdx.x * NW + warp;
  StreamRing rg;
  rg.ring = smem_addr(smem + warp * D * SLOT);
  rg.bars = smem_addr(smem + NW * D * SLOT) + warp * D * 8;
  // resident activations: one barrier after the warps' ones, the copies at the next 128-byte boundary
  const uint32_t xbar = smem_addr(smem + NW * D * SLOT) + NW * D * 8;
  rg.rx = smem_addr(smem) + ((NW * D * SLOT + NW * D * 8 + 8 + 127) / 128) * 128;

  if (lane == 0) {
    for (int s = 0; s < D; ++s) mbar_init(rg.bars + 8 * s, 1);
    if (RX && warp == 0) mbar_init(xbar, 1);
    fence_barrier_init();
  }
  if (RX)
    __syncthreads();  // every warp waits on the activation barrier warp 0 set up
  else
    __syncwarp();
  const uint64_t policy = l2_evict_first_policy();

  long long gb = 0, ge = 0;
  if (pw < sp.Pg) {
    gb = range_begin(pw, sp.TBg, sp.Pg);
    ge = range_begin(pw + 1, sp.TBg, sp.Pg);
  }
  if (ge <= gb) {
    grid_dependency_wait();
    grid_dependents_launch();
    if (RX && warp == 0) {
      // the copies of the resident activations are this warp's: issue them for
      // the CTA's other warps and wait (bounded) before leaving
      if (lane == 0) stage_resident_x<M>(sp, rg.rx, xbar);
      __syncwarp();
      if (!mbar_wait_bounded(xbar, 0, sp.timeout_ns) && lane == 0) atomicOr(sp.status, kStatusTimeout);
    }
    return;
  }
  const int e0 = entry_of_block(sp, gb);
  StreamProducer<SU, M, FC> pr;
  pr.left_total = ge - gb;
  pr.enter(sp, e0, gb - sp.entries[e0].blk_off);
  // the first stages' weights now; their activation slices once the
  // activation preparation (the preceding kernel) has completed
  const uint16_t* x_later[D];
  uint32_t x_later_bytes[D];
  for (int s = 0; s < D; ++s) {
    if (!pr.issue(sp, rg.ring + s * SLOT, rg.bars + 8 * s, policy, lane, false, &x_later[s], &x_later_bytes[s]))
      break;
    ++rg.in_flight;
  }

  grid_dependency_wait();
  grid_dependents_launch();
  if constexpr (RX) {
    if (threadIdx.x == 0) stage_resident_x<M>(sp, rg.rx, xbar);
  } else {
#pragma unroll
    for (int s = 0; s < D; ++s) {
      if (s < rg.in_flight)
        bulk_copy_x_if(lane == 0, rg.ring + s * SLOT + StreamSlot<SU, M, FC>::kWeightBytes, x_later[s],
                       x_later_bytes[s], rg.bars + 8 * s);
    }
  }

  float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
  int e_first = -1, r_first = -1;  // split first tile (its partial is written when it completes)
  int r = 0, c = 0;
  int e = e0;
  long long lb = gb - sp.entries[e0].blk_off;
  long long left = ge - gb;
  const StackEntryDev* __restrict__ ep = sp.entries + e;
  bool ok = true;
  float scale = 1.f;
  if (RX) ok = mbar_wait_bounded(xbar, 0, sp.timeout_ns);  // the resident activations have landed
  while ((!RX || ok) && left > 0) {
    const long long in_entry = ep->TC / SU - lb;
    const long long n = in_entry < left ? in_entry : left;
    const XInfo xi = *ep->xinfo;  // written by xprep_kernel, complete once griddepcontrol.wait returned
    scale = xi.ok ? xi.scale : 1.f;
    if (FormatClass<FC>::kClass >= 1 && ep->bits == kFmtNvfp4) {
      scale *= *reinterpret_cast<const float*>(ep->packed + ep->TC * Format<4>::kChunkBytes);  // t
      ok = xi.ok ? stream_segment<kFmtNvfp4, M, D, SU, true, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc,
                                                                 pw, e_first, r_first, r, c, lane)
                 : stream_segment<kFmtNvfp4, M, D, SU, false, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc,
                                                                  pw, e_first, r_first, r, c, lane);
    } else if (FormatClass<FC>::kClass == 2 && ep->bits == 5) {
      ok = xi.ok ? stream_segment<5, M, D, SU, true, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                         e_first, r_first, r, c, lane)
                 : stream_segment<5, M, D, SU, false, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                          e_first, r_first, r, c, lane);
    } else if (FormatClass<FC>::kClass == 2 && ep->bits == 6) {
      ok = xi.ok ? stream_segment<6, M, D, SU, true, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                         e_first, r_first, r, c, lane)
                 : stream_segment<6, M, D, SU, false, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                          e_first, r_first, r, c, lane);
    } else if (ep->bits == 4) {
      ok = xi.ok ? stream_segment<4, M, D, SU, true, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                         e_first, r_first, r, c, lane)
                 : stream_segment<4, M, D, SU, false, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                          e_first, r_first, r, c, lane);
    } else {
      ok = xi.ok ? stream_segment<8, M, D, SU, true, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                         e_first, r_first, r, c, lane)
                 : stream_segment<8, M, D, SU, false, FC>(sp, ep, e, lb, n, gb, rg, pr, policy, scale, acc, pw,
                                                          e_first, r_first, r, c, lane);
    }
    if (!ok) break;
    left -= n;
    if (left > 0) {
      ep = sp.entries + (++e);
      lb = 0;
    }
  }
  if (!ok) {
    if (lane == 0) atomicOr(sp.status, kStatusTimeout);
    // wait (bounded) for this warp's copies still in flight, then leave
    for (int k = 0; k < rg.in_flight; ++k) {
      if (!mbar_wait_bounded(rg.bars + 8 * rg.slot, rg.phase, sp.timeout_ns)) break;
      if (++rg.slot == D) {
        rg.slot = 0;
        rg.phase ^= 1u;
      }
    }
    return;
  }
  // finish the split tiles: the first one's partial is already in slot 0
  SplitTile first{nullptr, 0, -1, sp.counters, 0, 0}, last{nullptr, 0, -1, sp.counters, 0, 0};
  if (r_first >= 0) {
    const StackEntryDev& ef = sp.entries[e_first];
    const int bpt = ef.C / SU;
    const long long tile_g = ef.blk_off + static_cast<long long>(r_first) * bpt;
    first = SplitTile{ef.y, ef.N, r_first, sp.counters + ef.tile_off + r_first, tile_g, tile_g + bpt};
  }
  if (c != 0) {
    const int bpt = ep->C / SU;
    const long long tile_g = ep->blk_off + static_cast<long long>(r) * bpt;
    last = SplitTile{ep->y, ep->N, r, sp.counters + ep->tile_off + r, tile_g, tile_g + bpt};
    scale_acc(acc, scale);
    write_partial<M>(sp.partials, pw, tile_g <= gb ? 0 : 1, acc, lane);
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
  const Partition pt{sp.TBg, sp.Pg, sp.partials};
  const bool red_first = first.r >= 0 && a_first + 1 == tile_contributors(pt, first);
  const bool red_last = last.r >= 0 && a_last + 1 == tile_contributors(pt, last);
  if (red_first || red_last) __threadfence();
  if (red_first) reduce_tile<M>(pt, first, lane);
  if (red_last) reduce_tile<M>(pt, last, lane);
}

}  // namespace q4k
