// Seeded synthetic inputs (see synth_core.h for the definition).  Host
// functions fill host arrays with OpenMP; the *_device functions fill device
// arrays with identical bits.  Compiled with -fmad=false and
// -ffp-contract=off.  Nothing here computes the quantised product.
#include <cuda_runtime.h>

#include <cstdint>

#include "synth_core.h"

#define SYNTH_API extern "C" __attribute__((visibility("default")))

namespace {

bool shape_ok(int64_t K, int64_t row0, int64_t nrows) { return K > 0 && K % 32 == 0 && row0 >= 0 && nrows >= 0; }

__global__ void q4_kernel(uint64_t key, int64_t K, int64_t row0, int64_t nrows, uint8_t* out) {
  const int64_t per_row = K / 2;
  const int64_t total = nrows * per_row;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_q4_byte(key, K, row0 + i / per_row, i % per_row);
}

__global__ void q8_kernel(uint64_t key, int64_t K, int64_t row0, int64_t nrows, int8_t* out) {
  const int64_t total = nrows * K;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_q8_value(key, K, row0 + i / K, i % K);
}

__global__ void scales_kernel(uint64_t key, int64_t G, int64_t row0, int64_t nrows, double std, uint16_t* out) {
  const int64_t total = nrows * G;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_scale_value(key, G, row0 + i / G, i % G, std);
}

__global__ void e4m3_scales_kernel(uint64_t key, int64_t B, int64_t row0, int64_t nrows, uint8_t* out) {
  const int64_t total = nrows * B;
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_e4m3_scale(key, B, row0 + i / B, i % B);
}

__global__ void bf16_normals_kernel(uint64_t key, int64_t i0, int64_t count, uint16_t* out) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x)
    out[i] = synth_f64_to_bf16(synth_normal(key, (uint64_t)(i0 + i)));
}

unsigned grid_for(int64_t n) {
  const int64_t blocks = (n + 255) / 256;
  return (unsigned)(blocks < 65536 ? (blocks > 0 ? blocks : 1) : 65536);
}

int launched() { return cudaGetLastError() == cudaSuccess ? 0 : -2; }

}  // namespace

// ---------------------------------------------------------------- host side
SYNTH_API uint64_t synth_key_of(uint64_t seed, uint64_t stream) { return synth_key(seed, stream); }

SYNTH_API int synth_q4(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, uint8_t* out) {
  if (!shape_ok(K, row0, nrows) || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  const int64_t per_row = K / 2;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r)
    for (int64_t j = 0; j < per_row; ++j) out[r * per_row + j] = synth_q4_byte(key, K, row0 + r, j);
  return 0;
}

SYNTH_API int synth_q8(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, int8_t* out) {
  if (!shape_ok(K, row0, nrows) || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r)
    for (int64_t k = 0; k < K; ++k) out[r * K + k] = synth_q8_value(key, K, row0 + r, k);
  return 0;
}

SYNTH_API int synth_scales(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, double std,
                           uint16_t* out) {
  if (!shape_ok(K, row0, nrows) || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  const int64_t G = K / 32;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r)
    for (int64_t g = 0; g < G; ++g) out[r * G + g] = synth_scale_value(key, G, row0 + r, g, std);
  return 0;
}

// NVFP4 block scales (E4M3 bytes) [nrows][K/16]; K a multiple of 16.
SYNTH_API int synth_e4m3_scales(uint64_t seed, uint64_t stream, int64_t K, int64_t row0, int64_t nrows, uint8_t* out) {
  if (K < 0 || K % 16 || row0 < 0 || nrows < 0 || (!out && nrows > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  const int64_t B = K / 16;
#pragma omp parallel for schedule(static)
  for (int64_t r = 0; r < nrows; ++r)
    for (int64_t b = 0; b < B; ++b) out[r * B + b] = synth_e4m3_scale(key, B, row0 + r, b);
  return 0;
}

SYNTH_API int synth_bf16_normals(uint64_t seed, uint64_t stream, int64_t i0, int64_t count, uint16_t* out) {
  if (count < 0 || i0 < 0 || (!out && count > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < count; ++i) out[i] = synth_f64_to_bf16(synth_normal(key, (uint64_t)(i0 + i)));
  return 0;
}

SYNTH_API int synth_normals_f64(uint64_t seed, uint64_t stream, int64_t i0, int64_t count, double* out) {
  if (count < 0 || i0 < 0 || (!out && count > 0)) return -1;
  const uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i) out[i] = synth_normal(key, (uint64_t)(i0 + i));
  return 0;
}

SYNTH_API void synth_f64_to_f16_array(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_f64_to_f16(in[i]);
}

SYNTH_API void synth_f64_to_bf16_array(const double* in, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_f64_to_bf16(in[i]);
}

SYNTH_API void synth_log_array(const double* in, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_log(in[i]);
}

SYNTH_API void synth_cos2pi_array(const double* in, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = synth_cos2pi(in[i]);
}

SYNTH_API void synth_words(uint64_t seed, uint64_t stream, int64_t i0, int64_t count, uint64_t* out) {
  const uint64_t key = synth_key(seed, stream);
  for (int64_t i = 0; i < count; ++i) out[i] = synth_word(key, (uint64_t)(i0 + i));
}

// -------------------------------------------------------------- device side
// Same outputs as the host functions above, written to device memory
// asynchronously on `stream`.  Return 0, -1 on bad arguments, -2 on a CUDA
// launch error.
SYNTH_API int synth_q4_device(uint64_t seed, uint64_t stream_id, int64_t K, int64_t row0, int64_t nrows,
                              uint8_t* out, void* stream) {
  if (!shape_ok(K, row0, nrows) || (!out && nrows > 0)) return -1;
  if (nrows == 0) return 0;
  q4_kernel<<<grid_for(nrows * (K / 2)), 256, 0, (cudaStream_t)stream>>>(synth_key(seed, stream_id), K, row0, nrows,
                                                                           out);
  return launched();
}

SYNTH_API int synth_q8_device(uint64_t seed, uint64_t stream_id, int64_t K, int64_t row0, int64_t nrows,
                              int8_t* out, void* stream) {
  if (!shape_ok(K, row0, nrows) || (!out && nrows > 0)) return -1;
  if (nrows == 0) return 0;
  q8_kernel<<<grid_for(nrows * K), 256, 0, (cudaStream_t)stream>>>(synth_key(seed, stream_id), K, row0, nrows, out);
  return launched();
}

SYNTH_API int synth_scales_device(uint64_t seed, uint64_t stream_id, int64_t K, int64_t row0, int64_t nrows,
                                  double std, uint16_t* out, void* stream) {
  if (!shape_ok(K, row0, nrows) || (!out && nrows > 0)) return -1;
  if (nrows == 0) return 0;
  scales_kernel<<<grid_for(nrows * (K / 32)), 256, 0, (cudaStream_t)stream>>>(synth_key(seed, stream_id), K / 32,
                                                                                 row0, nrows, std, out);
  return launched();
}

SYNTH_API int synth_e4m3_scales_device(uint64_t seed, uint64_t stream_id, int64_t K, int64_t row0, int64_t nrows,
                                       uint8_t* out, void* stream) {
  if (K < 0 || K % 16 || row0 < 0 || nrows < 0 || (!out && nrows > 0)) return -1;
  if (nrows == 0 || K == 0) return 0;
  e4m3_scales_kernel<<<grid_for(nrows * (K / 16)), 256, 0, (cudaStream_t)stream>>>(synth_key(seed, stream_id), K / 16,
                                                                                     row0, nrows, out);
  return launched();
}

SYNTH_API int synth_bf16_normals_device(uint64_t seed, uint64_t stream_id, int64_t i0, int64_t count, uint16_t* out,
                                        void* stream) {
  if (count < 0 || i0 < 0 || (!out && count > 0)) return -1;
  if (count == 0) return 0;
  bf16_normals_kernel<<<grid_for(count), 256, 0, (cudaStream_t)stream>>>(synth_key(seed, stream_id), i0, count, out);
  return launched();
}
