// MTP draft / verify on the device: softmax statistics, the keep-or-reject
// test of each drafted token (keep with probability min(1, p/q)), and the
// inverse-CDF draws (the draft token, the correction at the first rejection
// from max(0, p - q), the bonus token), as the bs178.com llamAmpere post
// describes speculative decoding with a vocabulary-mapped draft head ("Why it
// is this fast", part four).
//
// One thread-block cluster of kSpecCtas CTAs per logits row: each CTA takes a
// contiguous slice of the row, and the CTAs exchange their partial maxima,
// sums and running totals through distributed shared memory, so every
// reduction has one fixed order (results are bitwise reproducible) and no
// global atomics or zero-filled workspace are needed.  Within a CTA each warp
// takes a contiguous sub-slice and walks it in steps of 32 values; a step's
// sum is a fixed shuffle tree, the warp's running sum adds the steps in order.
// A draw finds the CTA, then the warp, then the step, then the lane whose
// running sum first exceeds u * total, re-walking only that warp's sub-slice.
#pragma once

#include <cooperative_groups.h>
#include <stdint.h>

namespace q4k {

namespace cg = cooperative_groups;

constexpr int kSpecCtas = 8;        // CTAs per cluster (one cluster per logits row)
constexpr int kSpecThreads = 1024;  // 32 warps per CTA
constexpr int kSpecWarps = kSpecThreads / 32;
constexpr int kSpecUnroll = 8;      // steps of 32 values loaded ahead
constexpr unsigned kFull = 0xFFFFFFFFu;

// The slice of a row of n values that CTA `rank` takes, and warp w's part of
// it (a multiple of 32 values, so the steps of every warp start aligned).
struct SpecSlice {
  long long lo, hi;  // CTA slice
  long long per_warp;
  __device__ SpecSlice(long long n, int rank) {
    const long long per = (n + kSpecCtas - 1) / kSpecCtas;
    lo = rank * per < n ? rank * per : n;
    hi = lo + per < n ? lo + per : n;
    per_warp = ((hi - lo + kSpecWarps - 1) / kSpecWarps + 31) / 32 * 32;
  }
  __device__ long long wlo(int w) const { return lo + w * per_warp < hi ? lo + w * per_warp : hi; }
  __device__ long long whi(int w) const { return lo + (w + 1) * per_warp < hi ? lo + (w + 1) * per_warp : hi; }
};

// Sum of a warp's 32 values by a fixed tree, the same in every lane.
__device__ __forceinline__ float warp_tree_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(kFull, v, o);
  return __shfl_sync(kFull, v, 0);
}

// The running sum of weight(v) over [lo, hi) in steps of 32 (every lane
// returns it).
template <class W>
__device__ __forceinline__ float warp_walk_sum(long long lo, long long hi, const W& weight, int lane) {
  float run = 0.f;
  for (long long base = lo; base < hi; base += 32 * kSpecUnroll) {
    float w[kSpecUnroll];
#pragma unroll
    for (int k = 0; k < kSpecUnroll; ++k) {
      const long long v = base + 32 * k + lane;
      w[k] = v < hi ? weight(v) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kSpecUnroll; ++k) run += warp_tree_sum(w[k]);
  }
  return run;
}

// The first v in [lo, hi) where the warp's running sum (as warp_walk_sum
// forms it) exceeds t; if rounding leaves none, the last v with a positive
// weight; -1 if all weights are zero.
template <class W>
__device__ __forceinline__ long long warp_walk_find(long long lo, long long hi, const W& weight, float t, int lane) {
  float run = 0.f;
  long long last_pos = -1;
  for (long long base = lo; base < hi; base += 32 * kSpecUnroll) {
    float w[kSpecUnroll];
#pragma unroll
    for (int k = 0; k < kSpecUnroll; ++k) {
      const long long v = base + 32 * k + lane;
      w[k] = v < hi ? weight(v) : 0.f;
    }
#pragma unroll
    for (int k = 0; k < kSpecUnroll; ++k) {
      const float step = warp_tree_sum(w[k]);
      const unsigned pos = __ballot_sync(kFull, w[k] > 0.f);
      if (pos) last_pos = base + 32 * k + 31 - __clz(pos);
      if (run + step > t) {
        // inclusive scan of the step's 32 weights, in lane order
        float s = w[k];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const float y = __shfl_up_sync(kFull, s, o);
          if (lane >= o) s += y;
        }
        const unsigned hit = __ballot_sync(kFull, run + s > t && w[k] > 0.f);
        if (hit) return base + 32 * k + __ffs(hit) - 1;
        return last_pos;  // t fell in the step's rounding gap
      }
      run += step;
    }
  }
  return last_pos;
}

// Per-CTA values exchanged through distributed shared memory.
struct SpecXch {
  float max_p, max_q, sum_p, sum_q, sum_r;
  int arg_p;
};

struct SpecShared {
  SpecXch x;
  float warp_p[kSpecWarps];  // warps' running totals of exp((l - max) / T)
  float warp_r[kSpecWarps];  // warps' running totals of the residual weights
  float red[kSpecWarps];
  int redi[kSpecWarps];
};

__device__ __forceinline__ float block_max(float v, SpecShared& sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  __syncthreads();
  if (lane == 0) sh.red[warp] = v;
  __syncthreads();
  float m = sh.red[0];
  for (int w = 1; w < kSpecWarps; ++w) m = fmaxf(m, sh.red[w]);
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
  v = sh.red[0];
  i = sh.redi[0];
  for (int w = 1; w < kSpecWarps; ++w)
    if (sh.red[w] > v || (sh.red[w] == v && sh.redi[w] < i)) {
      v = sh.red[w];
      i = sh.redi[w];
    }
}

// Warp totals of a walk -> the CTA total (warps in order); each warp's total
// is stored in `tot`.
__device__ __forceinline__ float block_walk_total(float warp_total, float* tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) tot[warp] = warp_total;
  __syncthreads();
  float s = 0.f;
  for (int w = 0; w < kSpecWarps; ++w) s += tot[w];
  return s;
}

// The draw of one row: the first index whose running total (CTAs in rank
// order, then warps, then steps, then lanes) exceeds u * total.  cta_tot[c]
// are the CTAs' totals (the same array in every CTA), warp_tot this CTA's
// warps' totals.  Returns the index in the CTA that holds it, -1 elsewhere.
template <class W>
__device__ long long cluster_draw(const float* cta_tot, const float* warp_tot, const SpecSlice& sl, int rank, float u,
                                  const W& weight) {
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
  float t_in = t - run;
  // the warp, likewise
  float wrun = 0.f;
  int wsel = -1, wlast = -1;
  for (int w = 0; w < kSpecWarps; ++w) {
    if (warp_tot[w] > 0.f) wlast = w;
    if (wsel < 0 && warp_tot[w] > 0.f && wrun + warp_tot[w] > t_in) wsel = w;
    if (wsel < 0) wrun += warp_tot[w];
  }
  if (wsel < 0) {
    wsel = wlast;
    wrun = 0.f;
    for (int w = 0; w < wlast; ++w) wrun += warp_tot[w];
  }
  if (wsel < 0) return -1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __shared__ long long s_found;
  if (warp == wsel) {
    const long long v = warp_walk_find(sl.wlo(warp), sl.whi(warp), weight, t_in - wrun, lane);
    if (lane == 0) s_found = v;
  }
  __syncthreads();
  return s_found;
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

// One cluster: the draft token from softmax(z / T) over the mapped rows.
__global__ void __launch_bounds__(kSpecThreads) spec_draft_kernel(const SpecDraftParams P) {
  cg::cluster_group cl = cg::this_cluster();
  __shared__ SpecShared sh;
  const int rank = static_cast<int>(cl.block_rank());
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const SpecSlice sl(P.n_map, rank);
  asm volatile("griddepcontrol.wait;" ::: "memory");
  float m = -INFINITY;
  int mi = 0x7FFFFFFF;
  for (long long v = sl.lo + threadIdx.x; v < sl.hi; v += kSpecThreads) {
    const float x = P.z[v];
    if (x > m) {
      m = x;
      mi = static_cast<int>(v);
    }
  }
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
  const float wsum = warp_walk_sum(sl.wlo(warp), sl.whi(warp), e, lane);
  const float ctot = block_walk_total(wsum, sh.warp_p);
  if (threadIdx.x == 0) sh.x.sum_q = ctot;
  cl.sync();
  float tots[kSpecCtas];
  gather_xch(cl, sh, tots, [](const SpecXch& o) { return o.sum_q; });
  const long long i = cluster_draw(tots, sh.warp_p, sl, rank, *P.u, e);
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
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
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
  float m = -INFINITY;
  int mi = 0x7FFFFFFF;
  for (long long v = sl.lo + threadIdx.x; v < sl.hi; v += kSpecThreads) {
    const float x = l[v];
    if (x > m) {
      m = x;
      mi = static_cast<int>(v);
    }
  }
  block_argmax(m, mi, sh);
  float mq = -INFINITY;
  if (is_draft && !P.greedy) {
    for (long long v = slq.lo + threadIdx.x; v < slq.hi; v += kSpecThreads) mq = fmaxf(mq, z[v]);
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
  const float cp = block_walk_total(warp_walk_sum(sl.wlo(warp), sl.whi(warp), ep, lane), sh.warp_p);
  float cq = 0.f;
  if (is_draft) {
    auto eq = [=](long long v) { return expf((z[v] - gmq) * inv_t); };
    // these sums only normalise q: a plain strided sum, reduced in a fixed order
    float s = 0.f;
    for (long long v = slq.lo + threadIdx.x; v < slq.hi; v += kSpecThreads) s += eq(v);
    cq = block_walk_total(warp_tree_sum(s), sh.red);
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
    const long long i = cluster_draw(tot_p, sh.warp_p, sl, rank, P.u[2 * P.n], ep);
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
  const float cr = block_walk_total(warp_walk_sum(sl.wlo(warp), sl.whi(warp), er, lane), sh.warp_r);
  if (threadIdx.x == 0) sh.x.sum_r = cr;
  cl.sync();
  float tot_r[kSpecCtas];
  gather_xch(cl, sh, tot_r, [](const SpecXch& o) { return o.sum_r; });
  float sr = 0.f;
  for (int c = 0; c < kSpecCtas; ++c) sr += tot_r[c];
  long long i;
  if (sr > 0.f)
    i = cluster_draw(tot_r, sh.warp_r, sl, rank, P.u[P.n + j], er);
  else  // p and q agree to rounding: draw from p
    i = cluster_draw(tot_p, sh.warp_p, sl, rank, P.u[P.n + j], ep);
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
