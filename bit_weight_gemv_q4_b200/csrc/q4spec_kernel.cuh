// MTP draft / verify on the device: softmax statistics, the keep-or-reject
// test of each drafted token (keep with probability min(1, p/q)), and the
// inverse-CDF draws (the draft token, the correction at the first rejection
// from max(0, p - q), the bonus token), as the bs178.com llamAmpere post
// describes speculative decoding with a vocabulary-mapped draft head ("Why it
// is this fast", part four).
//
// One thread-block cluster of kSpecCtas CTAs per logits row: each CTA takes a
// contiguous slice of the row, and the CTAs exchange their partial maxima,
// sums and totals through distributed shared memory, so every reduction has
// one fixed order (results are bitwise reproducible) and no global atomics or
// zero-filled workspace are needed.  A CTA walks its slice in tiles of
// kSpecTile values; in a tile thread t sums the kSpecRun consecutive values
// at kSpecRun * t sequentially (the warp reads one contiguous kilobyte), and a
// block scan of those sums (in thread order) gives each thread its range
// [lower, upper) of the tile's running total, consecutive threads sharing a
// bound, so the ranges tile the tile's total without gaps.  Tiles add up in
// order.  A draw finds the CTA, then the tile, then the thread whose range
// holds u * total, and that thread walks its run.
#pragma once

#include <cooperative_groups.h>
#include <stdint.h>

namespace q4k {

namespace cg = cooperative_groups;

// Tunables (measured on B200 for a 248,320-token row: runs of 8 beat runs
// of 16 by ~30 %; 16-CTA clusters, above the portable size, saved ~12 % on
// the verify kernel and cost ~25 % on the draft kernel).
#ifndef Q4_TUNE_SPEC_CTAS
#define Q4_TUNE_SPEC_CTAS 8
#endif
#ifndef Q4_TUNE_SPEC_RUN
#define Q4_TUNE_SPEC_RUN 8
#endif
constexpr int kSpecCtas = Q4_TUNE_SPEC_CTAS;  // CTAs per cluster (one cluster per logits row)
constexpr int kSpecThreads = 1024;  // 32 warps per CTA
constexpr int kSpecWarps = kSpecThreads / 32;
constexpr int kSpecUnroll = 8;      // loads in flight per thread in the strided max pass
constexpr int kSpecRun = Q4_TUNE_SPEC_RUN;  // consecutive values a thread sums in a tile
constexpr int kSpecMaxTiles = 64;   // tile totals a CTA keeps for its draw (more: recomputed)
constexpr int kSpecTile = kSpecRun * kSpecThreads;
constexpr unsigned kFull = 0xFFFFFFFFu;

// The slice of a row of n values that CTA `rank` takes.
struct SpecSlice {
  long long lo, hi;
  __device__ SpecSlice(long long n, int rank) {
    const long long per = (n + kSpecCtas - 1) / kSpecCtas;
    lo = rank * per < n ? rank * per : n;
    hi = lo + per < n ? lo + per : n;
  }
};

// This thread's run in the tile starting at tb: the weights (0 past hi) and
// their sequential sum.
template <class W>
__device__ __forceinline__ float run_weights(long long tb, long long hi, const W& weight, float (&w)[kSpecRun]) {
  const long long a = tb + static_cast<long long>(kSpecRun) * threadIdx.x;
#pragma unroll
  for (int k = 0; k < kSpecRun; ++k) w[k] = a + k < hi ? weight(a + k) : 0.f;
  float s = 0.f;
#pragma unroll
  for (int k = 0; k < kSpecRun; ++k) s += w[k];
  return s;
}

// Per-CTA values exchanged through distributed shared memory.
struct SpecXch {
  float max_p, max_q, sum_p, sum_q, sum_r;
  int arg_p;
};

struct SpecShared {
  SpecXch x;
  float red[kSpecWarps];
  int redi[kSpecWarps];
  float woff[kSpecWarps + 1];  // warps' offsets in a block scan, then the block total
  float tiles_p[kSpecMaxTiles];  // tile totals of exp((l - max) / T)
  float tiles_r[kSpecMaxTiles];  // tile totals of the residual weights
  int found;
  long long found_index;
};

__device__ __forceinline__ float block_max(float v, SpecShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  __syncthreads();
  if (lane == 0) sh.red[warp] = v;
  __syncthreads();
  float m = sh.red[lane];  // every warp reduces the 32 warp maxima
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, o));
  return m;
}

// (largest value, its first index) of the block; ties go to the lower index.
__device__ __forceinline__ void block_argmax(float& v, int& i, SpecShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(kFull, v, o);
    const int i2 = __shfl_xor_sync(kFull, i, o);
    if (v2 > v || (v2 == v && i2 < i)) {
      v = v2;
      i = i2;
    }
  }
  __syncthreads();
  if (lane == 0) {
    sh.red[warp] = v;
    sh.redi[warp] = i;
  }
  __syncthreads();
  v = sh.red[lane];  // every warp reduces the 32 warp results
  i = sh.redi[lane];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const float v2 = __shfl_xor_sync(kFull, v, o);
    const int i2 = __shfl_xor_sync(kFull, i, o);
    if (v2 > v || (v2 == v && i2 < i)) {
      v = v2;
      i = i2;
    }
  }
}

// This thread's range [lower, upper) of the block's running total of the
// threads' sums s, in thread order (an inclusive warp scan, warp offsets
// added in warp order).  upper of thread i is bitwise lower of thread i + 1.
// Returns the block total.
struct SpecRange {
  float lower, upper;
};
__device__ __forceinline__ float block_scan(float s, SpecRange& r, SpecShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const float y = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += y;
  }
  const float excl = __shfl_up_sync(kFull, incl, 1);
  __syncthreads();
  if (lane == 31) sh.red[warp] = incl;
  __syncthreads();
  if (warp == 0) {  // the warps' offsets: an inclusive scan of their totals, in warp order
    const float t = sh.red[lane];
    float x = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float y = __shfl_up_sync(kFull, x, o);
      if (lane >= o) x += y;
    }
    const float before = __shfl_up_sync(kFull, x, 1);
    sh.woff[lane] = lane == 0 ? 0.f : before;
    if (lane == 31) sh.woff[kSpecWarps] = x;
  }
  __syncthreads();
  r.lower = lane == 0 ? sh.woff[warp] : sh.woff[warp] + excl;
  r.upper = lane == 31 ? sh.woff[warp + 1] : sh.woff[warp] + incl;
  return sh.woff[kSpecWarps];
}

// In a tile whose thread ranges r hold t (relative to the tile's start): the
// thread whose range holds t (if rounding leaves none, the last non-empty
// thread) walks its run.  Every thread returns the index.
__device__ __forceinline__ long long tile_find(long long tb, const float (&w)[kSpecRun], const SpecRange& r, float t,
                                               SpecShared& sh) {
  const bool nonempty = r.upper > r.lower;
  if (threadIdx.x == 0) sh.found = -1;
  __syncthreads();
  if (nonempty && r.lower <= t && t < r.upper) atomicMax(&sh.found, kSpecThreads + static_cast<int>(threadIdx.x));
  __syncthreads();
  if (sh.found < kSpecThreads && nonempty) atomicMax(&sh.found, static_cast<int>(threadIdx.x));
  __syncthreads();
  const int f = sh.found;
  const int owner = f >= kSpecThreads ? f - kSpecThreads : f;
  if (static_cast<int>(threadIdx.x) == owner) {
    const long long a = tb + static_cast<long long>(kSpecRun) * threadIdx.x;
    long long idx = -1;
    float run = r.lower;
#pragma unroll
    for (int k = 0; k < kSpecRun; ++k) {
      if (w[k] > 0.f && idx < 0) {
        if (run + w[k] > t) idx = a + k;
      }
      run += w[k];
    }
    if (idx < 0)  // rounding gap: the run's last positive weight
      for (int k = kSpecRun - 1; k >= 0 && idx < 0; --k)
        if (w[k] > 0.f) idx = a + k;
    sh.found_index = idx;
  }
  __syncthreads();
  const long long res = sh.found_index;
  __syncthreads();
  return res;
}

// The total of weight over the CTA slice: tiles in order, each tile's total
// from the block scan of its threads' run sums.  The first kSpecMaxTiles tile
// totals are kept in `tiles` (if given) for slice_find.
template <class W>
__device__ float slice_total(const SpecSlice& sl, const W& weight, SpecShared& sh, float* tiles) {
  float total = 0.f;
  int k = 0;
  for (long long tb = sl.lo; tb < sl.hi; tb += kSpecTile, ++k) {
    float w[kSpecRun];
    SpecRange r;
    const float tt = block_scan(run_weights(tb, sl.hi, weight, w), r, sh);
    if (tiles && k < kSpecMaxTiles && threadIdx.x == 0) tiles[k] = tt;
    total += tt;
  }
  return total;
}

// The first index of the CTA slice whose running total (tiles in order, then
// threads, then the run) exceeds t, with the same sums as slice_total; if
// rounding leaves none, the last index with a positive weight.  With the
// tile totals kept by slice_total only the chosen tile is recomputed.  Every
// thread returns it.
template <class W>
__device__ long long slice_find(const SpecSlice& sl, const W& weight, float t, SpecShared& sh, const float* tiles) {
  const long long ntiles = (sl.hi - sl.lo + kSpecTile - 1) / kSpecTile;
  float run = 0.f;
  long long sel = -1, last = -1;
  float t_sel = INFINITY;
  if (tiles && ntiles <= kSpecMaxTiles) {
    for (int k = 0; k < ntiles; ++k) {
      const float tt = tiles[k];
      if (tt > 0.f) last = k;
      if (tt > 0.f && run + tt > t) {
        sel = k;
        t_sel = t - run;
        break;
      }
      run += tt;
    }
  } else {
    for (long long tb = sl.lo; tb < sl.hi; tb += kSpecTile) {
      float w[kSpecRun];
      SpecRange r;
      const float tt = block_scan(run_weights(tb, sl.hi, weight, w), r, sh);
      const long long k = (tb - sl.lo) / kSpecTile;
      if (tt > 0.f) last = k;
      if (tt > 0.f && run + tt > t) return tile_find(tb, w, r, t - run, sh);
      run += tt;
    }
  }
  if (sel < 0) sel = last;  // t beyond the slice (rounding): its last positive weight
  if (sel < 0) return -1;
  const long long tb = sl.lo + sel * kSpecTile;
  float w[kSpecRun];
  SpecRange r;
  block_scan(run_weights(tb, sl.hi, weight, w), r, sh);
  return tile_find(tb, w, r, t_sel, sh);
}

// The draw of one row: the first index whose running total (CTAs in rank
// order, then the CTA's own order) exceeds u * total.  cta_tot[c]: the CTAs'
// totals (the same array in every CTA).  Returns the index in the CTA that
// holds it, -1 in the others.
template <class W>
__device__ long long cluster_draw(const float* cta_tot, const SpecSlice& sl, int rank, float u, const W& weight,
                                  SpecShared& sh, const float* tiles) {
  float total = 0.f;
  for (int c = 0; c < kSpecCtas; ++c) total += cta_tot[c];
  const float t = u * total;
  // the CTA: the first whose running total exceeds t, else the last non-empty one
  float run = 0.f;
  int cta = -1, last = -1;
  for (int c = 0; c < kSpecCtas; ++c) {
    if (cta_tot[c] > 0.f) last = c;
    if (cta < 0 && cta_tot[c] > 0.f && run + cta_tot[c] > t) cta = c;
    if (cta < 0) run += cta_tot[c];
  }
  if (cta < 0) {
    cta = last;
    run = 0.f;
    for (int c = 0; c < last; ++c) run += cta_tot[c];
  }
  if (cta != rank) return -1;
  return slice_find(sl, weight, t - run, sh, tiles);
}

// Reads field F of every CTA's exchange record, in rank order.
template <class F>
__device__ __forceinline__ void gather_xch(cg::cluster_group& cl, SpecShared& sh, float (&out)[kSpecCtas], F field) {
  for (int c = 0; c < kSpecCtas; ++c) out[c] = field(*cl.map_shared_rank(&sh.x, c));
}

struct SpecDraftParams {
  const float* z;       // [n_map]
  long long n_map;
  const int32_t* vmap;  // [n_map]
  float inv_t;          // 1 / T (T > 0); unused when greedy
  int greedy;
  const float* u;       // [1]
  int32_t* row_out;
  int32_t* token_out;
  float* q_out;
};

// (max, first index of the max) of a[v] over this thread's share of the CTA
// slice: strided by the block (coalesced loads, kSpecUnroll in flight); the
// maximum and its first index do not depend on the visiting order.
__device__ __forceinline__ void slice_argmax(const float* a, const SpecSlice& sl, float& m, int& mi) {
  m = -INFINITY;
  mi = 0x7FFFFFFF;
  for (long long base = sl.lo + threadIdx.x; base < sl.hi; base += kSpecThreads * kSpecUnroll) {
    float x[kSpecUnroll];
#pragma unroll
    for (int k = 0; k < kSpecUnroll; ++k) {
      const long long v = base + static_cast<long long>(k) * kSpecThreads;
      x[k] = v < sl.hi ? a[v] : -INFINITY;
    }
#pragma unroll
    for (int k = 0; k < kSpecUnroll; ++k) {
      if (x[k] > m) {  // visited in increasing index: the first maximum stays
        m = x[k];
        mi = static_cast<int>(base + static_cast<long long>(k) * kSpecThreads);
      }
    }
  }
}

// One cluster: the draft token from softmax(z / T) over the mapped rows.
__global__ void __launch_bounds__(kSpecThreads) spec_draft_kernel(const SpecDraftParams P) {
  cg::cluster_group cl = cg::this_cluster();
  __shared__ SpecShared sh;
  const int rank = static_cast<int>(cl.block_rank());
  const SpecSlice sl(P.n_map, rank);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float m;
  int mi;
  slice_argmax(P.z, sl, m, mi);
  block_argmax(m, mi, sh);
  if (threadIdx.x == 0) {
    sh.x.max_q = m;
    sh.x.arg_p = mi;
  }
  cl.sync();
  float gm = -INFINITY;
  int gi = 0x7FFFFFFF;
  for (int c = 0; c < kSpecCtas; ++c) {
    const SpecXch& o = *cl.map_shared_rank(&sh.x, c);
    if (o.max_q > gm || (o.max_q == gm && o.arg_p < gi)) {
      gm = o.max_q;
      gi = o.arg_p;
    }
  }
  if (P.greedy) {
    if (rank == 0 && threadIdx.x == 0) {
      *P.row_out = gi;
      *P.token_out = P.vmap[gi];
      *P.q_out = 1.f;
    }
    cl.sync();
    return;
  }
  const float inv_t = P.inv_t;
  const float* z = P.z;
  auto e = [=](long long v) { return expf((z[v] - gm) * inv_t); };
  const float ctot = slice_total(sl, e, sh, sh.tiles_p);
  if (threadIdx.x == 0) sh.x.sum_q = ctot;
  cl.sync();
  float tots[kSpecCtas];
  gather_xch(cl, sh, tots, [](const SpecXch& o) { return o.sum_q; });
  const long long i = cluster_draw(tots, sl, rank, *P.u, e, sh, sh.tiles_p);
  if (i >= 0 && threadIdx.x == 0) {
    float total = 0.f;
    for (int c = 0; c < kSpecCtas; ++c) total += tots[c];
    *P.row_out = static_cast<int32_t>(i);
    *P.token_out = P.vmap[i];
    *P.q_out = e(i) / total;
  }
  cl.sync();  // no CTA leaves while others may still read its shared memory
  asm volatile("griddepcontrol.launch_dependents;");
}

struct SpecVerifyParams {
  const float* target;     // [n + 1][V]
  long long V;
  const float* drafts;     // [n][n_map]
  long long n_map;
  const int32_t* vmap;     // [n_map]
  const int32_t* inv_map;  // [V]
  const int32_t* rows;     // [n] drafted mapped rows
  int n;
  float inv_t;
  int greedy;
  const float* u;          // [2n + 1]
  int32_t* out;            // [3n + 3]
};

// Cluster j (blockIdx.y) handles position j: the keep test of draft j (j < n)
// and, where it is rejected, the correction draw; position n draws the bonus.
// Writes keep[j] to out[n + 2 + j] and the draw to out[2n + 2 + j] (-1 if the
// draft is kept).
__global__ void __launch_bounds__(kSpecThreads) spec_verify_kernel(const SpecVerifyParams P) {
  cg::cluster_group cl = cg::this_cluster();
  __shared__ SpecShared sh;
  const int rank = static_cast<int>(cl.block_rank());
  const int j = blockIdx.y;
  const bool is_draft = j < P.n;
  const float* l = P.target + static_cast<long long>(j) * P.V;
  const float* z = is_draft ? P.drafts + static_cast<long long>(j) * P.n_map : nullptr;
  const SpecSlice sl(P.V, rank), slq(P.n_map, rank);
  int32_t* keep_out = P.out + P.n + 2;
  int32_t* draw_out = P.out + 2 * P.n + 2;
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // defaults, ordered before every later write by the cluster barriers below
  if (rank == 0 && threadIdx.x == 0) {
    if (is_draft) keep_out[j] = 0;
    draw_out[j] = -1;
  }

  // maxima (and, greedy, the first index of the maximum) of l_j and z_j
  float m;
  int mi;
  slice_argmax(l, sl, m, mi);
  block_argmax(m, mi, sh);
  float mq = -INFINITY;
  if (is_draft && !P.greedy) {
    int unused;
    slice_argmax(z, slq, mq, unused);
    mq = block_max(mq, sh);
  }
  if (threadIdx.x == 0) {
    sh.x.max_p = m;
    sh.x.arg_p = mi;
    sh.x.max_q = mq;
  }
  cl.sync();
  float gm = -INFINITY, gmq = -INFINITY;
  int gi = 0x7FFFFFFF;
  for (int c = 0; c < kSpecCtas; ++c) {
    const SpecXch& o = *cl.map_shared_rank(&sh.x, c);
    if (o.max_p > gm || (o.max_p == gm && o.arg_p < gi)) {
      gm = o.max_p;
      gi = o.arg_p;
    }
    gmq = fmaxf(gmq, o.max_q);
  }
  // the drafted row and token; rows or tokens out of range are never kept
  const int32_t row = is_draft ? P.rows[j] : -1;
  const bool row_ok = row >= 0 && row < P.n_map;
  const int32_t d = row_ok ? P.vmap[row] : -1;
  const bool d_ok = d >= 0 && d < P.V;
  if (P.greedy) {
    if (rank == 0 && threadIdx.x == 0) {
      const bool keep = is_draft && d_ok && d == gi;
      if (is_draft) keep_out[j] = keep ? 1 : 0;
      draw_out[j] = keep ? -1 : gi;
    }
    cl.sync();
    asm volatile("griddepcontrol.launch_dependents;");
    return;
  }

  // totals of exp((l - max) / T) and of exp((z - max) / T)
  const float inv_t = P.inv_t;
  auto ep = [=](long long v) { return expf((l[v] - gm) * inv_t); };
  const float cp = slice_total(sl, ep, sh, sh.tiles_p);
  float cq = 0.f;
  if (is_draft) {
    auto eq = [=](long long v) { return expf((z[v] - gmq) * inv_t); };
    cq = slice_total(slq, eq, sh, nullptr);
  }
  if (threadIdx.x == 0) {
    sh.x.sum_p = cp;
    sh.x.sum_q = cq;
  }
  cl.sync();
  float tot_p[kSpecCtas], tot_q[kSpecCtas];
  gather_xch(cl, sh, tot_p, [](const SpecXch& o) { return o.sum_p; });
  gather_xch(cl, sh, tot_q, [](const SpecXch& o) { return o.sum_q; });
  float sp = 0.f, sq = 0.f;
  for (int c = 0; c < kSpecCtas; ++c) {
    sp += tot_p[c];
    sq += tot_q[c];
  }

  if (!is_draft) {  // the bonus token, from p
    const long long i = cluster_draw(tot_p, sl, rank, P.u[2 * P.n], ep, sh, sh.tiles_p);
    if (i >= 0 && threadIdx.x == 0) draw_out[j] = static_cast<int32_t>(i);
    cl.sync();
    asm volatile("griddepcontrol.launch_dependents;");
    return;
  }
  // keep draft d with probability min(1, p/q): u * q < p
  const float pd = d_ok ? expf((l[d] - gm) * inv_t) / sp : 0.f;
  const float qd = row_ok ? expf((z[row] - gmq) * inv_t) / sq : 0.f;
  const bool keep = P.u[j] * qd < pd;
  if (keep) {
    if (rank == 0 && threadIdx.x == 0) {
      keep_out[j] = 1;
      draw_out[j] = -1;
    }
    cl.sync();
    asm volatile("griddepcontrol.launch_dependents;");
    return;
  }
  // rejected: the correction from max(0, p - q) over the whole vocabulary
  const int32_t* inv = P.inv_map;
  const long long n_map = P.n_map;
  const float inv_sp = 1.f / sp, inv_sq = 1.f / sq;
  auto er = [=](long long v) {
    const int32_t r = inv[v];
    const float qv = (r >= 0 && r < n_map) ? expf((z[r] - gmq) * inv_t) * inv_sq : 0.f;
    return fmaxf(expf((l[v] - gm) * inv_t) * inv_sp - qv, 0.f);
  };
  const float cr = slice_total(sl, er, sh, sh.tiles_r);
  if (threadIdx.x == 0) sh.x.sum_r = cr;
  cl.sync();
  float tot_r[kSpecCtas];
  gather_xch(cl, sh, tot_r, [](const SpecXch& o) { return o.sum_r; });
  float sr = 0.f;
  for (int c = 0; c < kSpecCtas; ++c) sr += tot_r[c];
  long long i;
  if (sr > 0.f)
    i = cluster_draw(tot_r, sl, rank, P.u[P.n + j], er, sh, sh.tiles_r);
  else  // p and q agree to rounding: draw from p
    i = cluster_draw(tot_p, sl, rank, P.u[P.n + j], ep, sh, sh.tiles_p);
  if (i >= 0 && threadIdx.x == 0) draw_out[j] = static_cast<int32_t>(i);
  cl.sync();
  asm volatile("griddepcontrol.launch_dependents;");
}

// out[0] = number of leading kept drafts a; out[1 .. a] the kept tokens;
// out[a + 1] the draw of position a (correction or bonus); out[a + 2 .. n + 1] = -1.
__global__ void spec_accept_kernel(const int32_t* vmap, const int32_t* rows, int n, int32_t* out) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  if (threadIdx.x != 0) return;
  const int32_t* keep = out + n + 2;
  const int32_t* draw = out + 2 * n + 2;
  int a = 0;
  while (a < n && keep[a]) ++a;
  out[0] = a;
  for (int k = 0; k < a; ++k) out[1 + k] = vmap[rows[k]];
  out[1 + a] = draw[a];
  for (int k = a + 1; k <= n; ++k) out[1 + k] = -1;
}

}  // namespace q4k
