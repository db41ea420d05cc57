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

// One CTA per activation row m.  The sum of squares is reduced in a fixed
// order (per-thread strided sums, a shuffle tree per warp, warps in order), so
// it is bitwise reproducible.  Rows of up to kNormThreads * kNormPer values
// keep each thread's values in registers: every load (h, y, gamma) is issued
// at once and h is not read back, so the step costs one memory round trip
// instead of one per value; longer rows take the same arithmetic in loops.
constexpr int kNormPer = 8;

__device__ __forceinline__ float norm_block_reduce(float ss) {
  __shared__ float s_part[32];
  __shared__ float s_t;
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xFFFFFFFFu, ss, o);
  if ((threadIdx.x & 31) == 0) s_part[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) t += s_part[w];
    s_t = t;
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
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
      const int k = threadIdx.x + j * kNormThreads;
      if (k < N) {
        h[row + k] = v[j];
        ss = fmaf(v[j], v[j], ss);
      }
    }
    const float r = 1.f / sqrtf(norm_block_reduce(ss) / static_cast<float>(N) + eps);
#pragma unroll
    for (int j = 0; j < kNormPer; ++j) {
      const int k = threadIdx.x + j * kNormThreads;
      if (k < N) {
        float o = v[j] * r;
        if (gamma) o *= g[j];
        x[row + k] = __bfloat16_as_ushort(__float2bfloat16_rn(o));
      }
    }
    return;
  }
  float ss = 0.f;
  for (int k = threadIdx.x; k < N; k += blockDim.x) {
    float v = set ? y[row + k] : h[row + k];
    if (y && !set) v += y[row + k];
    h[row + k] = v;
    ss = fmaf(v, v, ss);
  }
  const float r = 1.f / sqrtf(norm_block_reduce(ss) / static_cast<float>(N) + eps);
  for (int k = threadIdx.x; k < N; k += blockDim.x) {
    float v = h[row + k] * r;
    if (gamma) v *= __uint_as_float(static_cast<uint32_t>(gamma[k]) << 16);
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
