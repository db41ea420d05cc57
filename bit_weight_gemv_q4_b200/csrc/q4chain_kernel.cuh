// The steps between the products of a dependent decode chain, as kernels:
// each turns a product's fp32 output into the next product's bf16
// activations.  The pages name the layer structure (64 layers, 16 gated
// attention and 48 Gated DeltaNet: ai-coding.wiselychen.com guide, section
// "Before deploying: weights, KV cache, memory bandwidth") but not these
// steps; their plain textbook forms:
//   residual + RMSNorm:  h <- h + y (set: h <- y, the step's first);
//                        x = bf16( h / sqrt(mean_k h_k^2 + eps) * gamma )
//   SwiGLU:              x = bf16( silu(g) * u ),  silu(z) = z / (1 + e^-z),
//                        (g, u) the two halves of the fused gate|up output
// Both run with programmatic dependent launch: they wait (griddepcontrol.wait)
// for the product before them, and the product after them waits for them.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace q4k {

constexpr int kNormThreads = 1024;

// One CTA per activation row m.  The sum of squares has one fixed
// association, shared with the one-launch chain kernel: fp32 squares, a
// butterfly (xor-shuffle) sum over each tile of 32 consecutive values, the
// tile sums t = w, w + 32, w + 64, ... added in order (warp w of the 32 warps
// holds exactly those tiles, since thread t takes k = t + 1024 j), and a
// butterfly over the 32 warps' sums; so the two give bitwise the same
// activations.  Rows of up to kNormThreads * kNormPer values keep each
// thread's values in registers: every load (h, y, gamma) is issued at once
// and h is not read back; longer rows take the same arithmetic in loops.
constexpr int kNormPer = 8;

__device__ __forceinline__ float norm_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

// Every thread: the row's sum of squares from its warp's running tile sum.
__device__ __forceinline__ float norm_block_total(float warp_tiles) {
  __shared__ float s_part[32];
  __shared__ float s_t;
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = warp_tiles;
  __syncthreads();
  if (threadIdx.x < 32) {
    const float t = norm_warp_sum(s_part[threadIdx.x]);
    if (threadIdx.x == 0) s_t = t;
  }
  __syncthreads();
  return s_t;
}

__global__ void __launch_bounds__(kNormThreads) residual_rmsnorm_kernel(float* __restrict__ h,
                                                                       const float* __restrict__ y,
                                                                       const uint16_t* __restrict__ gamma,
                                                                       uint16_t* __restrict__ x, int N, float eps,
                                                                       int set) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const long long row = static_cast<long long>(blockIdx.x) * N;
  if (N <= kNormThreads * kNormPer) {
    float v[kNormPer], g[kNormPer];
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
      const int k = threadIdx.x + j * kNormThreads;
      v[j] = 0.f;
      g[j] = 1.f;
      if (k < N) {
        const float hv = set ? 0.f : h[row + k];
        const float yv = y ? y[row + k] : 0.f;
        v[j] = set ? yv : (y ? hv + yv : hv);
        if (gamma) g[j] = __uint_as_float(static_cast<uint32_t>(gamma[k]) << 16);
      }
    }
    float tiles = 0.f;
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
      const int k = threadIdx.x + j * kNormThreads;
      if (k < N) h[row + k] = v[j];
      if (j * kNormThreads < N) tiles += norm_warp_sum(__fmul_rn(v[j], v[j]));
    }
    const float r = 1.f / sqrtf(norm_block_total(tiles) / static_cast<float>(N) + eps);
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
      const int k = threadIdx.x + j * kNormThreads;
      if (k < N) {
        float o = __fmul_rn(v[j], r);
        if (gamma) o = __fmul_rn(o, g[j]);
        x[row + k] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
      }
    }
    return;
  }
  float tiles = 0.f;
  for (int base = 0; base < N; base += kNormThreads) {
    const int k = base + threadIdx.x;
    float v = 0.f;
    if (k < N) {
      v = set ? y[row + k] : h[row + k];
      if (y && !set) v += y[row + k];
      h[row + k] = v;
    }
    tiles += norm_warp_sum(__fmul_rn(v, v));
  }
  const float r = 1.f / sqrtf(norm_block_total(tiles) / static_cast<float>(N) + eps);
  for (int k = threadIdx.x; k < N; k += blockDim.x) {
    float v = __fmul_rn(h[row + k], r);
    if (gamma) v = __fmul_rn(v, __uint_as_float(static_cast<uint32_t>(gamma[k]) << 16));
    x[row + k] = __bfloat16_as_ushort(__float2bfloat16_rn(v));
  }
}

// Elementwise over M x N; y_gu rows hold 2N values (gate, then up).
__global__ void swiglu_kernel(const float* __restrict__ y_gu, uint16_t* __restrict__ x, int N, int M) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;");
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= static_cast<long long>(M) * N) return;
  const long long m = i / N, k = i - m * N;
  const float g = y_gu[m * 2 * N + k], u = y_gu[m * 2 * N + N + k];
  const float silu = g / (1.f + expf(-g));
  x[i] = __bfloat16_as_ushort(__float2bfloat16_rn(silu * u));
}

}  // namespace q4k
