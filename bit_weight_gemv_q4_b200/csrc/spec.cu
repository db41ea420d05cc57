// Host entry points of the MTP draft / verify step and of the row gather that
// builds a vocabulary-mapped draft head (kernels in q4spec_kernel.cuh).
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <string>

#include "q4gemv.h"
#include "q4spec_kernel.cuh"

namespace q4 {
void set_error(const std::string& msg);
}  // namespace q4

namespace {

int sfail(int code, const std::string& msg) {
  q4::set_error(msg);
  return code;
}

bool misaligned4(const void* p) { return reinterpret_cast<uintptr_t>(p) % 4 != 0; }

int check_device(const char* who) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  int major = 0;
  if (err == cudaSuccess) err = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  if (err != cudaSuccess) return sfail(Q4_ERR_CUDA, std::string(who) + ": " + cudaGetErrorString(err));
  if (major < 10) return sfail(Q4_ERR_UNSUPPORTED, std::string(who) + ": needs an sm_100 device");
  return Q4_OK;
}

// Launch with one cluster of kSpecCtas CTAs per row (grid.x == kSpecCtas) and
// programmatic dependent launch (the kernels wait on griddepcontrol before
// reading their inputs).
template <class P>
int launch_cluster(void (*kernel)(P), const P& params, unsigned rows, cudaStream_t stream, const char* who) {
  if (q4k::kSpecCtas > 8) {  // clusters above the portable size must be allowed per kernel
    const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return sfail(Q4_ERR_CUDA, std::string(who) + ": cluster size: " + cudaGetErrorString(e));
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(q4k::kSpecCtas, rows, 1);
  cfg.blockDim = dim3(q4k::kSpecThreads, 1, 1);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = q4k::kSpecCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, kernel, params);
  return err == cudaSuccess ? Q4_OK : sfail(Q4_ERR_CUDA, std::string(who) + ": launch: " + cudaGetErrorString(err));
}

int check_temperature(float t, const char* who) {
  if (!(t >= 0.f) || std::isinf(t)) return sfail(Q4_ERR_INVALID_ARG, std::string(who) + ": temperature must be finite and >= 0");
  return Q4_OK;
}

__global__ void gather_rows_kernel(const uint8_t* src, long long row_bytes, long long n_src, const int32_t* rows,
                                   long long n_rows, uint8_t* dst) {
  const long long r = blockIdx.y + static_cast<long long>(blockIdx.z) * 65535;
  if (r >= n_rows) return;
  const int32_t s = rows[r];
  const bool ok = s >= 0 && s < n_src;
  const uint8_t* from = src + (ok ? s : 0) * row_bytes;
  uint8_t* to = dst + r * row_bytes;
  if ((row_bytes & 15) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
      (reinterpret_cast<uintptr_t>(dst) & 15) == 0) {
    for (long long i = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) * 16; i < row_bytes;
         i += static_cast<long long>(gridDim.x) * blockDim.x * 16)
      *reinterpret_cast<uint4*>(to + i) = ok ? *reinterpret_cast<const uint4*>(from + i) : make_uint4(0, 0, 0, 0);
  } else {
    for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < row_bytes;
         i += static_cast<long long>(gridDim.x) * blockDim.x)
      to[i] = ok ? from[i] : 0;
  }
}

}  // namespace

extern "C" Q4_API int q4_gather_rows_device(const void* src, int64_t row_bytes, int64_t n_src, const int32_t* rows,
                                            int64_t n_rows, void* dst, void* stream) {
  const char* who = "q4_gather_rows_device";
  if (row_bytes < 0 || n_src < 0 || n_rows < 0 || n_src > INT32_MAX || n_rows > (int64_t(65535) * 65535))
    return sfail(Q4_ERR_SHAPE, std::string(who) + ": bad sizes");
  if (row_bytes == 0 || n_rows == 0) return Q4_OK;
  if (!src || !rows || !dst) return sfail(Q4_ERR_INVALID_ARG, std::string(who) + ": null pointer");
  if (misaligned4(rows)) return sfail(Q4_ERR_ALIGN, std::string(who) + ": rows must be 4-byte aligned");
  int rc = check_device(who);
  if (rc) return rc;
  const unsigned bx = static_cast<unsigned>(std::min<int64_t>(64, (row_bytes + 4095) / 4096));
  const dim3 grid(bx, static_cast<unsigned>(std::min<int64_t>(n_rows, 65535)),
                  static_cast<unsigned>((n_rows + 65534) / 65535));
  gather_rows_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(src), row_bytes, n_src, rows, n_rows, static_cast<uint8_t*>(dst));
  const cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? Q4_OK : sfail(Q4_ERR_CUDA, std::string(who) + ": launch: " + cudaGetErrorString(err));
}

extern "C" Q4_API int q4_spec_draft(const float* z, int64_t n_map, const int32_t* vmap, float temperature,
                                    const float* u, int32_t* row_out, int32_t* token_out, float* q_out,
                                    void* stream) {
  const char* who = "q4_spec_draft";
  if (n_map < 1 || n_map > INT32_MAX) return sfail(Q4_ERR_SHAPE, std::string(who) + ": need 1 <= n_map < 2^31");
  int rc = check_temperature(temperature, who);
  if (rc) return rc;
  if (!z || !vmap || !u || !row_out || !token_out || !q_out)
    return sfail(Q4_ERR_INVALID_ARG, std::string(who) + ": null pointer");
  if (misaligned4(z) || misaligned4(vmap) || misaligned4(u) || misaligned4(row_out) || misaligned4(token_out) ||
      misaligned4(q_out))
    return sfail(Q4_ERR_ALIGN, std::string(who) + ": pointers must be 4-byte aligned");
  if ((rc = check_device(who))) return rc;
  q4k::SpecDraftParams p{};
  p.z = z;
  p.n_map = n_map;
  p.vmap = vmap;
  p.greedy = temperature == 0.f ? 1 : 0;
  p.inv_t = temperature == 0.f ? 0.f : 1.f / temperature;
  p.u = u;
  p.row_out = row_out;
  p.token_out = token_out;
  p.q_out = q_out;
  return launch_cluster(q4k::spec_draft_kernel, p, 1, static_cast<cudaStream_t>(stream), who);
}

extern "C" Q4_API int q4_spec_verify(const float* target, int64_t V, const float* drafts, int64_t n_map,
                                     const int32_t* vmap, const int32_t* inv_map, const int32_t* rows, int n_draft,
                                     float temperature, const float* u, int32_t* out, void* stream) {
  const char* who = "q4_spec_verify";
  if (n_draft < 0 || n_draft > Q4_SPEC_MAX_DRAFT)
    return sfail(Q4_ERR_INVALID_ARG, std::string(who) + ": n_draft must be in 0..15");
  if (V < 1 || V > INT32_MAX || (n_draft > 0 && (n_map < 1 || n_map > V)))
    return sfail(Q4_ERR_SHAPE, std::string(who) + ": need 1 <= V < 2^31 and 1 <= n_map <= V");
  int rc = check_temperature(temperature, who);
  if (rc) return rc;
  if (!target || !u || !out || (n_draft > 0 && (!drafts || !vmap || !inv_map || !rows)))
    return sfail(Q4_ERR_INVALID_ARG, std::string(who) + ": null pointer");
  if (misaligned4(target) || misaligned4(u) || misaligned4(out) || misaligned4(drafts) || misaligned4(vmap) ||
      misaligned4(inv_map) || misaligned4(rows))
    return sfail(Q4_ERR_ALIGN, std::string(who) + ": pointers must be 4-byte aligned");
  if ((rc = check_device(who))) return rc;
  q4k::SpecVerifyParams p{};
  p.target = target;
  p.V = V;
  p.drafts = drafts;
  p.n_map = n_draft > 0 ? n_map : 1;
  p.vmap = vmap;
  p.inv_map = inv_map;
  p.rows = rows;
  p.n = n_draft;
  p.greedy = temperature == 0.f ? 1 : 0;
  p.inv_t = temperature == 0.f ? 0.f : 1.f / temperature;
  p.u = u;
  p.out = out;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = launch_cluster(q4k::spec_verify_kernel, p, static_cast<unsigned>(n_draft + 1), st, who))) return rc;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(1, 1, 1);
  cfg.blockDim = dim3(32, 1, 1);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t err = cudaLaunchKernelEx(&cfg, q4k::spec_accept_kernel, vmap, rows, n_draft, out);
  return err == cudaSuccess ? Q4_OK : sfail(Q4_ERR_CUDA, std::string(who) + ": launch: " + cudaGetErrorString(err));
}
