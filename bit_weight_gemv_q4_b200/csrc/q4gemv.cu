// C-ABI of the group-quantised weight x activation product on B200 (sm_100a).
// Host side: argument validation, launch-shape selection, the workspace
// contract, and the CUDA-graph-captured layer stack.  Device code lives in
// q4gemv_kernels.cuh.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include "q4gemv.h"
#include "q4gemv_kernels.cuh"
#include "q4chain_kernel.cuh"
#include "q4stack_kernel.cuh"
#include "q4chainp_kernel.cuh"

namespace q4 {

thread_local std::string g_last_error;

void set_error(const std::string& msg) { g_last_error = msg; }

namespace {

constexpr unsigned long long kDefaultTimeoutNs = 2000000000ULL;
std::atomic<unsigned long long> g_timeout_ns{kDefaultTimeoutNs};

// Launch shape of the product kernel: one persistent CTA of NW warps per SM;
// per warp a ring of kRingChunks chunks cut into D = kRingChunks / U stages of
// U chunks (U = 2 when it divides the chunks per tile, else 1).  Measured on
// B200: bulk-copy streaming holds ~7 TB/s with 16 warps per SM and 32-64
// copies in flight per SM, and falls off sharply beyond that.  The defaults
// can be changed at compile time for tuning sweeps.
#ifndef Q4_TUNE_NW
#define Q4_TUNE_NW 16
#endif
#ifndef Q4_TUNE_CTAS_PER_SM
#define Q4_TUNE_CTAS_PER_SM 1
#endif
#ifndef Q4_TUNE_RING_CHUNKS
#define Q4_TUNE_RING_CHUNKS 4
#endif
// Split-tile width of a single product: each warp takes at least
// Q4_TUNE_MIN_BLOCKS stream-K blocks (fewer warps share each tile, so the
// split-tile fix-up reduces fewer partials) as long as that still leaves
// Q4_TUNE_MIN_WARPS_PER_SM warps per SM; smaller products keep one block per
// warp and their parallelism.
#ifndef Q4_TUNE_MIN_BLOCKS
#define Q4_TUNE_MIN_BLOCKS 4
#endif
#ifndef Q4_TUNE_MIN_WARPS_PER_SM
#define Q4_TUNE_MIN_WARPS_PER_SM 8
#endif
#ifndef Q4_TUNE_MAX_U
#define Q4_TUNE_MAX_U 2
#endif
constexpr int kNW = Q4_TUNE_NW;  // warps per CTA of the single-product kernel
constexpr int kCtasPerSm = Q4_TUNE_CTAS_PER_SM;
constexpr int kRingChunks = Q4_TUNE_RING_CHUNKS;
constexpr int kMaxU = Q4_TUNE_MAX_U;
static_assert(kRingChunks % 2 == 0 && kRingChunks >= 4, "ring must hold two stages of two chunks");
#ifndef Q4_TUNE_STREAM_GROUPS  // 0: M >= 2 stream lists run as one launch
#define Q4_TUNE_STREAM_GROUPS 1
#endif
#ifndef Q4_TUNE_STACK_D
#define Q4_TUNE_STACK_D 2
#endif
#ifndef Q4_TUNE_STACK_PF
#define Q4_TUNE_STACK_PF 0
#endif
#ifndef Q4_TUNE_STACK_NW
#define Q4_TUNE_STACK_NW 16
#endif
#ifndef Q4_TUNE_STREAM_U
#define Q4_TUNE_STREAM_U 4
#endif
constexpr int kStackD = Q4_TUNE_STACK_D;    // stages per warp in the persistent stack kernels
constexpr int kStackPF = Q4_TUNE_STACK_PF;  // further stages prefetched into L2 (ordered mode)
constexpr int kStreamU = Q4_TUNE_STREAM_U;  // chunks per stage in stream mode, when the shapes allow
constexpr int kStackNW = Q4_TUNE_STACK_NW;  // warps per CTA of the persistent kernels (one CTA per SM)
#ifndef Q4_TUNE_CHAIN_PF
#define Q4_TUNE_CHAIN_PF 0
#endif
constexpr int kChainPF = Q4_TUNE_CHAIN_PF;  // one-launch chain: stages prefetched into L2 beyond each ring
// shared memory a CTA may use (B200: 227 KB per CTA)
constexpr int kSmemLimit = 227 * 1024 / kCtasPerSm;  // single-product kernel, per CTA
constexpr int kStackSmemLimit = 227 * 1024;           // persistent kernels: one CTA per SM
constexpr size_t kWsHeader = 256;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t err, const char* what) {
  return fail(Q4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorString(err), cudaGetErrorName(err));
}

struct DeviceInfo {
  int sms = 0;
  bool ok = false;
  std::string why;
};

std::mutex g_dev_mutex;
std::vector<DeviceInfo> g_devices;

// Per-device facts, checked once: an sm_100 device and its SM count.
int device_info(DeviceInfo* out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_dev_mutex);
  if (static_cast<int>(g_devices.size()) <= dev) g_devices.resize(dev + 1);
  DeviceInfo& info = g_devices[dev];
  if (!info.ok && info.why.empty()) {
    int major = 0, minor = 0, sms = 0;
    if ((err = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess ||
        (err = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess ||
        (err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
      return cuda_fail(err, "cudaDeviceGetAttribute");
    if (major != 10 || minor != 0) {
      info.why = "device " + std::to_string(dev) + " is sm_" + std::to_string(major) + std::to_string(minor) +
                 "; this library is built for sm_100a only";
    } else {
      info.sms = sms;
      info.ok = true;
    }
  }
  if (!info.ok) return fail(Q4_ERR_UNSUPPORTED, "%s", info.why.c_str());
  *out = info;
  return Q4_OK;
}

struct Shape {
  int bits;
  long long N, K;
  int T, C;
  long long TC;
};

int make_shape(int bits, int64_t N, int64_t K, Shape* s, const char* who) {
  if (bits != 4 && bits != 8) return fail(Q4_ERR_INVALID_ARG, "%s: bits must be 4 or 8", who);
  if (N < 0 || K < 0 || K % 32 != 0)
    return fail(Q4_ERR_SHAPE, "%s: need N >= 0, K >= 0 and K %% 32 == 0 (N=%lld K=%lld)", who, (long long)N,
                (long long)K);
  if (N > (int64_t(1) << 34) || K > (int64_t(1) << 30))
    return fail(Q4_ERR_SHAPE, "%s: N or K too large", who);
  s->bits = bits;
  s->N = N;
  s->K = K;
  s->T = static_cast<int>((N + q4k::kTileRows - 1) / q4k::kTileRows);
  const int kc = bits == 4 ? 64 : 32;
  s->C = static_cast<int>((K + kc - 1) / kc);
  s->TC = static_cast<long long>(s->T) * s->C;
  // the kernels' range arithmetic needs (chunks x warps) below 2^52
  if (s->TC >= (int64_t(1) << 38)) return fail(Q4_ERR_SHAPE, "%s: tensor too large", who);
  return Q4_OK;
}

// A stack entry's shape: bits 4 or 8, or 5, 6 or Q4_FMT_NVFP4 (the q4 chunk
// geometry, K a multiple of 64).
int entry_shape(int bits, int64_t N, int64_t K, Shape* s, const char* who) {
  if (bits != Q4_FMT_NVFP4 && bits != 5 && bits != 6) return make_shape(bits, N, K, s, who);
  const int rc = make_shape(4, N, K, s, who);
  if (rc) return rc;
  if (K % 64 != 0) return fail(Q4_ERR_SHAPE, "%s: %d-bit formats need K %% 64 == 0 (K=%lld)", who, bits, (long long)K);
  s->bits = bits;
  return Q4_OK;
}

// Formats that run in stream mode only.
bool stream_only(int bits) { return bits == Q4_FMT_NVFP4 || bits == 5 || bits == 6; }

// Chunk bytes of a stack entry's format.
int chunk_bytes_of(int bits) {
  return bits == 8 ? q4k::Format<8>::kChunkBytes
                   : bits == 5 ? q4k::Wide<5>::kChunkBytes : bits == 6 ? q4k::Wide<6>::kChunkBytes
                                                                       : q4k::Format<4>::kChunkBytes;
}

// CTAs per SM a single product's grid fills at most (kCtasPerSm: fits; fewer
// leaves room for the next kernel's CTAs)
#ifndef Q4_TUNE_GRID_PER_SM
#define Q4_TUNE_GRID_PER_SM Q4_TUNE_CTAS_PER_SM
#endif
constexpr int kGridPerSm = Q4_TUNE_GRID_PER_SM;
long long max_warps(const DeviceInfo& dev) { return static_cast<long long>(dev.sms) * kGridPerSm * kNW; }

// Warps that split one product of TB stream-K blocks (the single-product
// kernel and, per product, the ordered persistent kernel, so their outputs
// stay bitwise equal): at most `most`, at least Q4_TUNE_MIN_BLOCKS blocks per
// warp while that leaves Q4_TUNE_MIN_WARPS_PER_SM warps per SM.
long long product_warps(long long TB, long long most, const DeviceInfo& dev) {
  const long long floor_warps = std::min(TB, static_cast<long long>(dev.sms) * Q4_TUNE_MIN_WARPS_PER_SM);
  return std::min(most, std::max(TB / Q4_TUNE_MIN_BLOCKS, floor_warps));
}

// Warps a single product (or a product of an ordered stack, which splits it
// the same way) is split between, in blocks of U chunks.  A product with
// fewer than 4 blocks per warp is bound by its split tiles' fix-up more than
// by streaming: at most kPartBatch / M contributors per tile there, so that
// each tile's owner collects their words in one batch of loads (measured on
// the 1024 x 5120 product at M = 4: 5.1 us instead of 10.3; on the
// 5120 x 17408 one, 9 blocks per warp, the cap cost 19 %).
long long split_warps(const Shape& s, int U, int M, long long most, const DeviceInfo& dev) {
  long long P = product_warps(s.TC / U, most, dev);
  if (s.TC / U < 4 * P)
    P = std::max<long long>(1, std::min(P, static_cast<long long>(s.T) * std::max(1, q4k::kPartBatch / std::max(M, 1))));
  return P;
}

// Workspace layout: [status word | partial sums | tile counters].  The
// partial-sum region has one fixed size per device (M = 4 worst case), so the
// counters sit at the same offset for every shape and M: one zero-filled
// workspace serves any sequence of products, each leaving its counters zero.
// partial sums of split tiles: two slots of up to 4 x 32 floats per warp, for
// the most warps any kernel runs (single-product or persistent)
size_t partials_bytes(const DeviceInfo& dev) {
  const long long warps = std::max(max_warps(dev), static_cast<long long>(dev.sms) * kStackNW);
  return static_cast<size_t>(warps) * 2 * 4 * q4k::kTileRows * sizeof(float);
}

size_t workspace_bytes(const Shape& s, int M, const DeviceInfo& dev) {
  (void)M;
  const size_t counters = (static_cast<size_t>(s.T) * 4 + 255) / 256 * 256;
  return kWsHeader + partials_bytes(dev) + counters;
}

template <int BITS, int M, int U, bool XS>
void* kernel_ptr() {
  return reinterpret_cast<void*>(&q4k::gemv_kernel<BITS, M, kNW, kRingChunks / U, U, XS>);
}

template <int BITS, int U>
int smem_base() {
  using Cfg = q4k::GemvConfig<BITS, kNW, kRingChunks / U, U>;
  return Cfg::kXOffset;
}

int pick_u(int C) { return (kMaxU >= 2 && C % 2 == 0) ? 2 : 1; }

void* select_kernel(int bits, int M, int U, bool xs) {
#define Q4_ROW(B, M_) \
  {{kernel_ptr<B, M_, 1, false>(), kernel_ptr<B, M_, 1, true>()}, {kernel_ptr<B, M_, 2, false>(), kernel_ptr<B, M_, 2, true>()}}
  static void* const table[2][4][2][2] = {
      {Q4_ROW(4, 1), Q4_ROW(4, 2), Q4_ROW(4, 3), Q4_ROW(4, 4)},
      {Q4_ROW(8, 1), Q4_ROW(8, 2), Q4_ROW(8, 3), Q4_ROW(8, 4)},
  };
#undef Q4_ROW
  return table[bits == 4 ? 0 : 1][M - 1][U - 1][xs ? 1 : 0];
}

// Dynamic shared memory of a launch: the rings, the barriers and, with the
// activations staged, M padded rows.
int smem_bytes(int bits, int U, int M, long long K, bool xs) {
  const int base = bits == 4 ? (U == 2 ? smem_base<4, 2>() : smem_base<4, 1>())
                             : (U == 2 ? smem_base<8, 2>() : smem_base<8, 1>());
  return base + (xs ? static_cast<int>(M * q4k::x_row_stride_bytes(K)) : 0);
}

#ifndef Q4_TUNE_STAGE_X
#define Q4_TUNE_STAGE_X 1
#endif
bool stage_x(int bits, int U, int M, long long K) {
  return Q4_TUNE_STAGE_X &&
         static_cast<long long>(smem_bytes(bits, U, M, 0, false)) + M * q4k::x_row_stride_bytes(K) <= kSmemLimit;
}

struct Launch {
  void* fn = nullptr;
  dim3 grid, block;
  int smem = 0;
  q4k::GemvParams params{};
  bool zero_fill = false;  // K == 0: y = 0
  size_t zero_bytes = 0;
  bool noop = false;
};

int prepare(int bits, const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y, void* workspace,
            size_t workspace_bytes_given, const char* who, Launch* L) {
  Shape s;
  int rc = make_shape(bits, N, K, &s, who);
  if (rc) return rc;
  if (M < 0 || M > 4) return fail(Q4_ERR_INVALID_ARG, "%s: M must be in 0..4 (got %d)", who, M);
  if (N == 0 || M == 0) {
    L->noop = true;
    return Q4_OK;
  }
  if (!y) return fail(Q4_ERR_INVALID_ARG, "%s: y is null", who);
  if (reinterpret_cast<uintptr_t>(y) % 4) return fail(Q4_ERR_ALIGN, "%s: y must be 4-byte aligned", who);
  if (K == 0) {
    L->zero_fill = true;
    L->zero_bytes = static_cast<size_t>(M) * static_cast<size_t>(N) * sizeof(float);
    return Q4_OK;
  }
  if (!packed || !x || !workspace) return fail(Q4_ERR_INVALID_ARG, "%s: null device pointer", who);
  if (reinterpret_cast<uintptr_t>(packed) % 16) return fail(Q4_ERR_ALIGN, "%s: packed must be 16-byte aligned", who);
  if (reinterpret_cast<uintptr_t>(x) % 16) return fail(Q4_ERR_ALIGN, "%s: x must be 16-byte aligned", who);
  if (reinterpret_cast<uintptr_t>(workspace) % 16)
    return fail(Q4_ERR_ALIGN, "%s: workspace must be 16-byte aligned", who);
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const size_t need = workspace_bytes(s, M, dev);
  if (workspace_bytes_given < need)
    return fail(Q4_ERR_BUFFER_TOO_SMALL, "%s: workspace %zu bytes < %zu required", who, workspace_bytes_given, need);

  const int U = pick_u(s.C);
  const bool xs = stage_x(bits, U, M, s.K);
  const long long P = split_warps(s, U, M, max_warps(dev), dev);
  // Split between every warp the GPU holds: consecutive warps per CTA (the
  // contributors of a split tile mostly share an SM: measured 10 % faster on
  // the 17,408 x 5120 products).  Between fewer: one CTA per SM with the warps
  // interleaved over them, so every SM streams (measured 8-10 % faster on the
  // 4096- and 5120-row products than filling half the SMs).
  const bool interleave = P < max_warps(dev);
  const int G = interleave ? static_cast<int>(std::min<long long>(P, static_cast<long long>(dev.sms) * kGridPerSm))
                           : static_cast<int>((P + kNW - 1) / kNW);
  unsigned char* ws = static_cast<unsigned char*>(workspace);

  q4k::GemvParams& p = L->params;
  p.packed = static_cast<const uint8_t*>(packed);
  p.x = x;
  p.y = y;
  p.status = reinterpret_cast<unsigned*>(ws);
  p.partials = reinterpret_cast<float*>(ws + kWsHeader);
  p.counters = reinterpret_cast<unsigned*>(ws + kWsHeader + partials_bytes(dev));
  p.N = s.N;
  p.K = s.K;
  p.TC = s.TC;
  p.T = s.T;
  p.C = s.C;
  p.P = static_cast<int>(P);
  p.khalf = (bits == 4 && K % 64 == 32) ? 1 : 0;
  p.interleave = interleave ? 1 : 0;
  p.timeout_ns = g_timeout_ns.load();
  L->fn = select_kernel(bits, M, U, xs);
  L->grid = dim3(G);
  L->block = dim3(kNW * 32);
  L->smem = smem_bytes(bits, U, M, s.K, xs);
  return Q4_OK;
}

int launch(Launch& L, cudaStream_t stream, bool pdl) {
  cudaError_t err;
  if (L.noop) return Q4_OK;
  if (L.zero_fill) {
    err = cudaMemsetAsync(L.params.y, 0, L.zero_bytes, stream);
    return err == cudaSuccess ? Q4_OK : cuda_fail(err, "cudaMemsetAsync(y)");
  }
  static std::once_flag smem_once;
  static cudaError_t smem_err = cudaSuccess;
  std::call_once(smem_once, [] {
    for (int bits : {4, 8})
      for (int M = 1; M <= 4; ++M)
        for (int U : {1, 2})
          for (bool xs : {false, true}) {
            cudaError_t e = cudaFuncSetAttribute(select_kernel(bits, M, U, xs),
                                                 cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemLimit);
            if (e != cudaSuccess) smem_err = e;
          }
  });
  if (smem_err != cudaSuccess) return cuda_fail(smem_err, "cudaFuncSetAttribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = L.grid;
  cfg.blockDim = L.block;
  cfg.dynamicSmemBytes = static_cast<size_t>(L.smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  void* args[] = {&L.params};
  err = cudaLaunchKernelExC(&cfg, L.fn, args);
  if (err != cudaSuccess) return cuda_fail(err, "kernel launch");
  return Q4_OK;
}

int gemv_entry(int bits, const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y,
               void* workspace, size_t workspace_bytes_given, void* stream, const char* who) {
  Launch L;
  // the zero-fill path needs y in params
  int rc = prepare(bits, packed, N, K, x, M, y, workspace, workspace_bytes_given, who, &L);
  if (rc) return rc;
  L.params.y = y;
  return launch(L, static_cast<cudaStream_t>(stream), true);
}

}  // namespace
}  // namespace q4

using namespace q4;

extern "C" Q4_API const char* q4_last_error(void) { return g_last_error.c_str(); }

extern "C" Q4_API size_t q4_gemv_workspace_bytes(int bits, int64_t N, int64_t K, int M) {
  Shape s;
  if (make_shape(bits, N, K, &s, "q4_gemv_workspace_bytes")) return 0;
  if (M < 0 || M > 4) {
    fail(Q4_ERR_INVALID_ARG, "q4_gemv_workspace_bytes: M must be in 0..4");
    return 0;
  }
  DeviceInfo dev;
  if (device_info(&dev)) return 0;
  return workspace_bytes(s, M, dev);
}

extern "C" Q4_API int q4_gemv(const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y,
                              void* workspace, size_t workspace_bytes_given, void* stream) {
  return gemv_entry(4, packed, N, K, x, M, y, workspace, workspace_bytes_given, stream, "q4_gemv");
}

extern "C" Q4_API int q8_gemv(const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y,
                              void* workspace, size_t workspace_bytes_given, void* stream) {
  return gemv_entry(8, packed, N, K, x, M, y, workspace, workspace_bytes_given, stream, "q8_gemv");
}

extern "C" Q4_API int q4_workspace_check(void* workspace, size_t workspace_bytes_given, void* stream) {
  if (!workspace) return fail(Q4_ERR_INVALID_ARG, "q4_workspace_check: workspace is null");
  if (workspace_bytes_given < kWsHeader)
    return fail(Q4_ERR_BUFFER_TOO_SMALL, "q4_workspace_check: workspace smaller than its header");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t err = cudaStreamSynchronize(s);
  if (err != cudaSuccess) return cuda_fail(err, "cudaStreamSynchronize");
  unsigned status = 0;
  err = cudaMemcpy(&status, workspace, sizeof(status), cudaMemcpyDeviceToHost);
  if (err != cudaSuccess) return cuda_fail(err, "cudaMemcpy(status)");
  if (status == 0) return Q4_OK;
  err = cudaMemset(workspace, 0, workspace_bytes_given);
  if (err != cudaSuccess) return cuda_fail(err, "cudaMemset(workspace)");
  return fail(Q4_ERR_TIMEOUT, "a device wait gave up after %llu ns; the affected outputs are undefined",
              static_cast<unsigned long long>(g_timeout_ns.load()));
}

extern "C" Q4_API int q4_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
  return Q4_OK;
}

extern "C" Q4_API int q4_unpack_device(int bits, const void* packed, int64_t N, int64_t K, int8_t* q_out,
                                       uint16_t* scales_out, void* stream) {
  Shape s;
  if (bits == Q4_FMT_NVFP4) return fail(Q4_ERR_INVALID_ARG, "q4_unpack_device: bits must be 4, 5, 6 or 8");
  int rc = entry_shape(bits, N, K, &s, "q4_unpack_device");
  if (rc) return rc;
  if (s.TC == 0) return Q4_OK;
  if (!packed || !q_out || !scales_out) return fail(Q4_ERR_INVALID_ARG, "q4_unpack_device: null pointer");
  if (reinterpret_cast<uintptr_t>(packed) % 16)
    return fail(Q4_ERR_ALIGN, "q4_unpack_device: packed must be 16-byte aligned");
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const int warps = 8;
  const long long blocks = (s.TC + warps - 1) / warps;
  if (blocks > 0x7FFFFFFFLL) return fail(Q4_ERR_SHAPE, "q4_unpack_device: tensor too large");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (bits == 5)
    q4k::unpack_wide_kernel<5><<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(
        static_cast<const uint8_t*>(packed), s.N, s.K, s.T, s.C, q_out, scales_out);
  else if (bits == 6)
    q4k::unpack_wide_kernel<6><<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(
        static_cast<const uint8_t*>(packed), s.N, s.K, s.T, s.C, q_out, scales_out);
  else if (bits == 4)
    q4k::unpack_kernel<4><<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(
        static_cast<const uint8_t*>(packed), s.N, s.K, s.T, s.C, q_out, scales_out);
  else
    q4k::unpack_kernel<8><<<static_cast<unsigned>(blocks), warps * 32, 0, st>>>(
        static_cast<const uint8_t*>(packed), s.N, s.K, s.T, s.C, q_out, scales_out);
  cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? Q4_OK : cuda_fail(err, "unpack kernel launch");
}

extern "C" Q4_API int q4_pack_weights_device(int bits, const void* canon_q, const uint16_t* scales_fp16, int64_t N,
                                             int64_t K, void* out, size_t out_bytes, void* stream) {
  Shape s;
  if (bits == Q4_FMT_NVFP4) return fail(Q4_ERR_INVALID_ARG, "q4_pack_weights_device: bits must be 4, 5, 6 or 8");
  int rc = entry_shape(bits, N, K, &s, "q4_pack_weights_device");
  if (rc) return rc;
  const size_t need = static_cast<size_t>(s.TC) * chunk_bytes_of(bits);
  if (need == 0) return Q4_OK;
  if (!canon_q || !scales_fp16 || !out) return fail(Q4_ERR_INVALID_ARG, "q4_pack_weights_device: null pointer");
  if (reinterpret_cast<uintptr_t>(out) % 16)
    return fail(Q4_ERR_ALIGN, "q4_pack_weights_device: out must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(scales_fp16) % 2)
    return fail(Q4_ERR_ALIGN, "q4_pack_weights_device: scales must be 2-byte aligned");
  if (out_bytes < need)
    return fail(Q4_ERR_BUFFER_TOO_SMALL, "q4_pack_weights_device: out_bytes %zu < %zu", out_bytes, need);
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const long long threads = s.TC * 64;
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return fail(Q4_ERR_SHAPE, "q4_pack_weights_device: tensor too large");
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const uint8_t* q = static_cast<const uint8_t*>(canon_q);
  if (bits == 5)
    q4k::pack_wide_kernel<5><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        reinterpret_cast<const int8_t*>(q), scales_fp16, s.N, s.K, s.T, s.C, static_cast<uint8_t*>(out));
  else if (bits == 6)
    q4k::pack_wide_kernel<6><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        reinterpret_cast<const int8_t*>(q), scales_fp16, s.N, s.K, s.T, s.C, static_cast<uint8_t*>(out));
  else if (bits == 4)
    q4k::pack_kernel<4><<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, scales_fp16, s.N, s.K, s.T, s.C,
                                                                        static_cast<uint8_t*>(out));
  else
    q4k::pack_kernel<8><<<static_cast<unsigned>(blocks), 256, 0, st>>>(q, scales_fp16, s.N, s.K, s.T, s.C,
                                                                        static_cast<uint8_t*>(out));
  cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? Q4_OK : cuda_fail(err, "pack kernel launch");
}

extern "C" Q4_API int q4_pack_nvfp4_device(const uint8_t* codes, const uint8_t* scales, float tensor_scale,
                                           int64_t N, int64_t K, void* out, size_t out_bytes, void* stream) {
  Shape s;
  int rc = entry_shape(Q4_FMT_NVFP4, N, K, &s, "q4_pack_nvfp4_device");
  if (rc) return rc;
  const size_t need = static_cast<size_t>(s.TC) * q4k::Format<4>::kChunkBytes + q4k::kNvfp4TrailerBytes;
  if (!out || (s.TC > 0 && (!codes || !scales))) return fail(Q4_ERR_INVALID_ARG, "q4_pack_nvfp4_device: null pointer");
  if (reinterpret_cast<uintptr_t>(out) % 16)
    return fail(Q4_ERR_ALIGN, "q4_pack_nvfp4_device: out must be 16-byte aligned");
  if (out_bytes < need)
    return fail(Q4_ERR_BUFFER_TOO_SMALL, "q4_pack_nvfp4_device: out_bytes %zu < %zu", out_bytes, need);
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const long long threads = std::max(1LL, s.TC * 64);
  const long long blocks = (threads + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return fail(Q4_ERR_SHAPE, "q4_pack_nvfp4_device: tensor too large");
  q4k::pack_nvfp4_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      codes, scales, tensor_scale, s.N, s.K, s.T, s.C, static_cast<uint8_t*>(out));
  cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? Q4_OK : cuda_fail(err, "NVFP4 pack kernel launch");
}

extern "C" Q4_API int q4_nvfp4_dequant_device(const void* packed, int64_t N, int64_t K, float* w_out, void* stream) {
  Shape s;
  int rc = entry_shape(Q4_FMT_NVFP4, N, K, &s, "q4_nvfp4_dequant_device");
  if (rc) return rc;
  if (s.TC == 0) return Q4_OK;
  if (!packed || !w_out) return fail(Q4_ERR_INVALID_ARG, "q4_nvfp4_dequant_device: null pointer");
  if (reinterpret_cast<uintptr_t>(packed) % 16 || reinterpret_cast<uintptr_t>(w_out) % 4)
    return fail(Q4_ERR_ALIGN, "q4_nvfp4_dequant_device: packed must be 16-byte, w_out 4-byte aligned");
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const long long blocks = (s.TC * 64 + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return fail(Q4_ERR_SHAPE, "q4_nvfp4_dequant_device: tensor too large");
  q4k::dequant_nvfp4_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint8_t*>(packed), s.N, s.K, s.T, s.C, w_out);
  cudaError_t err = cudaGetLastError();
  return err == cudaSuccess ? Q4_OK : cuda_fail(err, "NVFP4 dequant kernel launch");
}

extern "C" Q4_API int q4_selftest_wait_timeout(uint64_t timeout_ns, int* status_out) {
  if (!status_out) return fail(Q4_ERR_INVALID_ARG, "q4_selftest_wait_timeout: status_out is null");
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  int* d_result = nullptr;
  cudaError_t err = cudaMalloc(&d_result, sizeof(int));
  if (err != cudaSuccess) return cuda_fail(err, "cudaMalloc");
  err = cudaMemset(d_result, 0xFF, sizeof(int));
  if (err == cudaSuccess) {
    q4k::wait_selftest_kernel<<<1, 32>>>(static_cast<unsigned long long>(timeout_ns), d_result);
    err = cudaGetLastError();
  }
  if (err == cudaSuccess) err = cudaDeviceSynchronize();
  int h = -1;
  if (err == cudaSuccess) err = cudaMemcpy(&h, d_result, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d_result);
  if (err != cudaSuccess) return cuda_fail(err, "wait self-test");
  *status_out = h;
  return Q4_OK;
}

// ----------------------------------------------------------------------------
// q4 product without a caller-provided workspace.  Some callers cannot
// allocate device memory at the point where they run the product: plug-ins
// that run inside a host application which owns the device memory budget (its
// own pool or allocator, none of it handed to them), and latency-critical
// loops that must not call cudaMalloc, which can synchronise the whole device.
// For them the split-tile scratch lives in this file-scope device array
// instead.  Every GPU that loads the library holds it until the process exits.
// ----------------------------------------------------------------------------
constexpr size_t kNoAllocWorkspaceBytes = size_t(4) << 20;  // 4 MiB per device
static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoAllocWorkspaceBytes];

namespace {
std::mutex g_noalloc_mutex;
std::vector<void*> g_noalloc_ptr;  // device address of the array, per device

// The array's name in host code is only a stand-in: its device address comes
// from cudaGetSymbolAddress, once per device, with that device current.
int noalloc_workspace(void** out) {
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return cuda_fail(err, "q4_gemv_noalloc: cudaGetDevice");
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (static_cast<int>(g_noalloc_ptr.size()) <= dev) g_noalloc_ptr.resize(dev + 1, nullptr);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    err = cudaGetSymbolAddress(&ptr, g_noalloc_workspace);
    if (err != cudaSuccess) return cuda_fail(err, "q4_gemv_noalloc: cudaGetSymbolAddress");
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return Q4_OK;
}
}  // namespace

extern "C" Q4_API int q4_gemv_noalloc(const void* packed, int64_t N, int64_t K, const uint16_t* x, int M, float* y,
                                      void* stream) {
  const char* who = "q4_gemv_noalloc";
  Shape s;
  int rc = make_shape(4, N, K, &s, who);
  if (rc) return rc;
  if (M < 0 || M > 4) return fail(Q4_ERR_INVALID_ARG, "%s: M must be in 0..4 (got %d)", who, M);
  if (N == 0 || M == 0 || K == 0)  // nothing to stage: same as q4_gemv
    return gemv_entry(4, packed, N, K, x, M, y, nullptr, 0, stream, who);
  DeviceInfo dev;
  if ((rc = device_info(&dev))) return rc;
  const size_t need = workspace_bytes(s, M, dev);
  if (need > kNoAllocWorkspaceBytes) {
    // rows whose tile counters fit beside the header and the partial sums
    // (counters take whole 256-byte blocks of 64 tiles, 32 rows each)
    const size_t fixed = kWsHeader + partials_bytes(dev);
    const long long max_rows =
        fixed >= kNoAllocWorkspaceBytes ? 0 : static_cast<long long>((kNoAllocWorkspaceBytes - fixed) / 256 * 64 * 32);
    return fail(Q4_ERR_UNSUPPORTED,
                "%s: this shape needs %zu bytes of scratch, more than the %zu-byte static array "
                "(at most %lld rows on this device); use q4_gemv with a workspace",
                who, need, kNoAllocWorkspaceBytes, max_rows);
  }
  void* ws = nullptr;
  if ((rc = noalloc_workspace(&ws))) return rc;
  Launch L;
  if ((rc = prepare(4, packed, N, K, x, M, y, ws, kNoAllocWorkspaceBytes, who, &L))) return rc;
  L.params.y = y;
  // The array keeps whatever the last call left (a call whose wait gave up
  // leaves words set): clear the status word and the split-tile words this
  // launch's warps use, which must start at zero.
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned char* base = static_cast<unsigned char*>(ws);
  cudaError_t err = cudaMemsetAsync(base, 0, kWsHeader, st);
  if (err == cudaSuccess)
    err = cudaMemsetAsync(base + kWsHeader, 0,
                          static_cast<size_t>(L.params.P) * M * q4k::kTileRows * sizeof(unsigned long long), st);
  if (err != cudaSuccess) return cuda_fail(err, "q4_gemv_noalloc: cudaMemsetAsync");
  return launch(L, st, true);
}

// ----------------------------------------------------------------------------
// Layer stack: the ordered products of one decode step.
// ----------------------------------------------------------------------------
struct q4_stack {
  // graph mode: one kernel per product, captured once
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
  // persistent mode: one cooperative kernel over the whole list
  bool persistent = false;
  q4k::StackEntryDev* entries_dev = nullptr;
  void* fn = nullptr;
  int grid = 0, block = 0, smem = 0;
  q4k::StackParams params{};
  bool cooperative = false;  // ordered mode: its grid barrier needs every CTA resident
  // stream mode: one activation preparation per distinct (x, K), run before
  // the stream kernel on every layer_stack_run
  q4k::XPrepJob* xprep_dev = nullptr;
  int xprep_jobs = 0;
  int xprep_ctas = 1;  // CTAs per job
  int rx_bytes = 0;    // stream mode: resident activations' bytes (0: slices through the rings)
  // stream mode split into groups (M >= 2): one stream_kernel launch per
  // group after the preparation, each with its own entries, stages and
  // resident activations; empty when the list runs as one launch (fn, params)
  struct Group {
    void* fn = nullptr;
    int smem = 0;
    q4k::StackParams params{};
  };
  std::vector<Group> groups;
  // persistent chain (Q4_CHAIN_PERSISTENT): one cooperative chain_kernel launch
  bool chain = false;
  q4k::ChainParams chain_params{};
  q4k::ChainOpDev* chain_ops_dev = nullptr;
  int M = 1;
  void* workspace = nullptr;
  size_t workspace_bytes = 0;
  int launches = 0;
  int device = 0;
};

namespace {

template <int M>
void* stack_kernel_ptr() {
  return reinterpret_cast<void*>(&q4k::stack_kernel<M, kStackNW, kStackD, kStackPF>);
}

template <int M, int SU, int FC>
void* stream_kernel_ptr() {
  return reinterpret_cast<void*>(&q4k::stream_kernel<M, kStackNW, kStackD, SU, FC>);
}

template <int SU, int FC>
struct StreamRow {
  static void* at(int M) {
    static void* const row[4] = {stream_kernel_ptr<1, SU, FC>(), stream_kernel_ptr<2, SU, FC>(),
                                 stream_kernel_ptr<3, SU, FC>(), stream_kernel_ptr<4, SU, FC>()};
    return row[M - 1];
  }
};

// su: chunks per stage of the stream-mode kernel (0 = ordered mode); fc: the
// list's format class (0 q4 / q8, 1 also NVFP4, 2 also q5 / q6).  Class 2 with
// stages of four chunks exists for M = 1 only (its slots fit shared memory
// there; create_persistent picks stages of two otherwise).
void* select_stack_kernel(int M, int su, int fc) {
  static void* const ordered[4] = {stack_kernel_ptr<1>(), stack_kernel_ptr<2>(), stack_kernel_ptr<3>(),
                                   stack_kernel_ptr<4>()};
  if (su == 0) return ordered[M - 1];
  if (fc == 3 && M >= 2) {  // a group of a stream list with its activations resident (M = 2..4)
    static void* const row[3] = {stream_kernel_ptr<2, kStreamU, 3>(), stream_kernel_ptr<3, kStreamU, 3>(),
                                 stream_kernel_ptr<4, kStreamU, 3>()};
    return row[M - 2];
  }
  if (fc >= 3)  // resident activations: M = 1, stages of kStreamU chunks only
    return fc == 3 ? stream_kernel_ptr<1, kStreamU, 3>() : stream_kernel_ptr<1, kStreamU, 4>();
  if (fc == 0) return su == 2 ? StreamRow<2, 0>::at(M) : StreamRow<kStreamU, 0>::at(M);
  if (fc == 1) return su == 2 ? StreamRow<2, 1>::at(M) : StreamRow<kStreamU, 1>::at(M);
  if (su != 2 && M == 1) return stream_kernel_ptr<1, kStreamU, 2>();
  return StreamRow<2, 2>::at(M);
}

// su: stream mode with stages of su chunks (weights + activation slice of M
// rows), or 0 for ordered mode (weights only, stages of kStackU chunks).
// fc 3 / 4 (resident activations): weights-only slots, one more barrier, and
// the activation copies (rx_bytes) from the next 128-byte boundary.
int stack_smem_bytes(int su, int M, int fc, int rx_bytes = 0) {
  constexpr int nw = kStackNW;
  if (su == 0) return nw * kStackD * q4k::kStackU * q4k::Format<4>::kChunkBytes + nw * kStackD * 8;
  const int cb = fc == 2 ? q4k::Wide<6>::kChunkBytes : q4k::Format<4>::kChunkBytes;
  const int xb = fc >= 3 ? 0 : M * q4k::Format<4>::kKPerChunk * 2;
  const int rings = nw * kStackD * su * (cb + xb);
  if (fc >= 3) return (rings + nw * kStackD * 8 + 8 + 127) / 128 * 128 + rx_bytes;
  return rings + nw * kStackD * 8;
}

// A persistent kernel's dynamic shared-memory limit is a property of the
// function, shared by every stack that launches it with its own size: allow
// the most one CTA per SM can take beside the function's static shared memory.
cudaError_t allow_dynamic_smem(void* fn) {
  cudaFuncAttributes a{};
  cudaError_t err = cudaFuncGetAttributes(&a, fn);
  if (err != cudaSuccess) return err;
  return cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kStackSmemLimit - static_cast<int>(a.sharedSizeBytes));
}

void free_stack(q4_stack* st) {
  if (st->exec) cudaGraphExecDestroy(st->exec);
  if (st->graph) cudaGraphDestroy(st->graph);
  if (st->entries_dev) cudaFree(st->entries_dev);
  if (st->xprep_dev) cudaFree(st->xprep_dev);  // also holds the groups' job tables
  if (st->chain_ops_dev) cudaFree(st->chain_ops_dev);
  if (st->workspace) cudaFree(st->workspace);
  delete st;
}

// Persistent mode: every product non-empty, with an even number of chunks per
// tile (stages of two chunks).
bool stack_eligible(const q4_stack_entry* entries, int n) {
  if (n <= 0) return false;
  for (int i = 0; i < n; ++i) {
    Shape s;
    if (entry_shape(entries[i].bits, entries[i].N, entries[i].K, &s, "layer_stack_create")) return false;
    if (s.N == 0 || s.K == 0 || s.C % 2 != 0) return false;
  }
  return true;
}

// su: stream mode with stages of su chunks (every product's C a multiple of
// su), or 0 for ordered mode.
int create_persistent(const q4_stack_entry* entries, int n, int M, int su, const DeviceInfo& dev, q4_stack* st) {
  int fc = 0;
  for (int i = 0; i < n; ++i) {
    if (entries[i].bits == Q4_FMT_NVFP4) fc = std::max(fc, 1);
    if (entries[i].bits == 5 || entries[i].bits == 6) fc = 2;
  }
  // stages of four chunks of the widest formats fit shared memory at M = 1 only
  if (su != 0 && fc == 2 && M > 1) su = 2;
  const bool independent = su != 0;
  const long long blk = independent ? su : q4k::kStackU;  // chunks per stream-K block
  long long max_t = 1, total_blocks = 0, total_tiles = 0;
  std::vector<q4k::StackEntryDev> host(static_cast<size_t>(n));
  const long long warps = static_cast<long long>(dev.sms) * kStackNW;
  for (int i = 0; i < n; ++i) {
    const q4_stack_entry& en = entries[i];
    char who[64];
    snprintf(who, sizeof(who), "layer_stack_create entry %d", i);
    Shape s;
    int rc = entry_shape(en.bits, en.N, en.K, &s, who);
    if (rc) return rc;
    if (!en.packed || !en.x || !en.y) return fail(Q4_ERR_INVALID_ARG, "%s: null device pointer", who);
    if (reinterpret_cast<uintptr_t>(en.packed) % 16 || reinterpret_cast<uintptr_t>(en.x) % 16 ||
        reinterpret_cast<uintptr_t>(en.y) % 4)
      return fail(Q4_ERR_ALIGN, "%s: packed and x must be 16-byte aligned, y 4-byte aligned", who);
    // ordered mode splits each product as a single call does (bitwise the same y)
    const long long P = split_warps(s, q4k::kStackU, M, warps, dev);
    q4k::StackEntryDev& d = host[static_cast<size_t>(i)];
    d.packed = static_cast<const uint8_t*>(en.packed);
    d.x = en.x;
    d.y = en.y;
    d.N = s.N;
    d.K = s.K;
    d.TC = s.TC;
    d.T = s.T;
    d.C = s.C;
    d.bits = en.bits;
    d.P = static_cast<int>(P);
    d.khalf = (en.bits == 4 && s.K % 64 == 32) ? 1 : 0;
    d.blk_off = total_blocks;
    d.tile_off = static_cast<int>(total_tiles);
    total_blocks += s.TC / blk;
    total_tiles += s.T;
    if (s.T > max_t) max_t = s.T;
  }
  if (total_tiles >= (1LL << 31)) return fail(Q4_ERR_SHAPE, "layer_stack_create: too many tiles");
  // ordered mode re-uses one counter per tile of the largest product; stream
  // mode keeps one per tile of every product
  const size_t counters = (static_cast<size_t>(independent ? total_tiles : max_t) * 4 + 255) / 256 * 256;
  int rx_bytes = 0;  // stream mode with resident activations: their bytes in shared memory
  int fc_sel = fc;   // the kernel's class: fc, or 3 + fc (activations resident)
  // stream mode: per distinct (x, K, format) a chunk-major copy of x and its XInfo
  std::vector<q4k::XPrepJob> jobs;
  std::vector<size_t> job_of(static_cast<size_t>(n), 0), x16_off, info_off;
  size_t prep_bytes = 0;
  if (independent) {
    for (int i = 0; i < n; ++i) {
      const int KC = entries[i].bits == 8 ? q4k::Format<8>::kKPerChunk : q4k::Format<4>::kKPerChunk;  // 64: q4-geometry formats
      size_t jdx = jobs.size();
      for (size_t k = 0; k < jobs.size(); ++k)
        if (jobs[k].x == entries[i].x && jobs[k].K == entries[i].K && jobs[k].KC == KC) jdx = k;
      if (jdx == jobs.size()) {
        q4k::XPrepJob j{};
        j.x = entries[i].x;
        j.K = entries[i].K;
        j.KC = KC;
        jobs.push_back(j);
        x16_off.push_back(prep_bytes);
        prep_bytes += (static_cast<size_t>(M) * entries[i].K * 2 + 255) / 256 * 256;
        info_off.push_back(prep_bytes);
        prep_bytes += 256;
      }
      job_of[static_cast<size_t>(i)] = jdx;
    }
  }
  // stream-mode groups (see below)
  struct GroupPlan {
    int su, fc;
    long long rx;
  };
  std::vector<GroupPlan> plan;
  std::vector<std::vector<int>> group_rx;  // per group and job: the job's offset in shared memory, or -1
  std::vector<int> job_group(jobs.size(), -1);
  const bool grouped = independent && Q4_TUNE_STREAM_GROUPS && M >= 2 && su == kStreamU && fc == 0;
  // ordered mode: one barrier flag per CTA
  const size_t flags_bytes = independent ? 0 : (static_cast<size_t>(dev.sms) * 4 + 255) / 256 * 256;
  const size_t flags_base = kWsHeader + partials_bytes(dev) + counters;
  const size_t prep_base = flags_base + flags_bytes;
  st->workspace_bytes = prep_base + prep_bytes;
  cudaError_t err = cudaMalloc(&st->workspace, st->workspace_bytes);
  if (err == cudaSuccess) err = cudaMemset(st->workspace, 0, st->workspace_bytes);
  st->cooperative = !independent;
  st->M = M;
  if (independent && err == cudaSuccess) {
    unsigned char* base = static_cast<unsigned char*>(st->workspace) + prep_base;
    for (size_t k = 0; k < jobs.size(); ++k) {
      jobs[k].xc = reinterpret_cast<uint16_t*>(base + x16_off[k]);
      jobs[k].info = reinterpret_cast<q4k::XInfo*>(base + info_off[k]);
    }
    // resident activations (stages of kStreamU).  M = 1, classes 0 / 1:
    // every CTA keeps each prepared tensor in shared memory when they all
    // fit, and the stages carry weights only.
    for (auto& j : jobs) j.rx_off = -1;
    // M >= 2, q4 / q8 lists with stages of kStreamU: the list runs as groups,
    // one launch each.  The prepared tensors, narrowest first, join the first
    // group whose resident activations they fit beside the weights-only
    // stages; a tensor that fits no group leaves its products to one group
    // whose stages carry the activation slices.  Every CTA of a resident group
    // copies the group's tensors into shared memory once.  (On the decode
    // stream, interleaved on one B200: M = 4 5,302 GB/s at 1,530 MHz against
    // 5,124 at 1,552 as one launch with every slice in the slots; M = 2 and 3
    // +3 % and +2 % against one launch that kept only the 5120-value inputs
    // resident beside slots with room for slices.  A resident 17,408-value
    // group with stages of two chunks streamed no faster than its slices in
    // stages of four and executed 146 instead of ~127 warp instructions per
    // chunk.)
    if (grouped) {
      std::vector<size_t> order(jobs.size());
      for (size_t k = 0; k < jobs.size(); ++k) order[k] = k;
      std::stable_sort(order.begin(), order.end(), [&](size_t a, size_t b) { return jobs[a].K < jobs[b].K; });
      int ring_group = -1;
      auto fits = [&](int gsu, long long rx) {
        return rx < (1LL << 30) && stack_smem_bytes(gsu, M, 3, static_cast<int>(rx)) <= kStackSmemLimit;
      };
      for (size_t k : order) {
        // the copy's bytes, resident only when a whole number of 128-byte
        // blocks (always, with stages of four chunks: K % 128 == 0)
        const long long bytes = static_cast<long long>(M) * jobs[k].K * 2;
        int g = -1;
        for (size_t q = 0; q < plan.size() && g < 0; ++q)
          if (plan[q].fc == 3 && bytes % 128 == 0 && fits(plan[q].su, plan[q].rx + bytes)) g = static_cast<int>(q);
        if (g < 0) {
          const int gsu = bytes % 128 == 0 && fits(kStreamU, bytes) ? kStreamU : 0;
          if (gsu != 0 || ring_group < 0) {
            plan.push_back(GroupPlan{gsu != 0 ? gsu : kStreamU, gsu != 0 ? 3 : 0, 0});
            group_rx.emplace_back(jobs.size(), -1);
            if (gsu == 0) ring_group = static_cast<int>(plan.size()) - 1;
          }
          g = gsu != 0 ? static_cast<int>(plan.size()) - 1 : ring_group;
        }
        if (plan[static_cast<size_t>(g)].fc == 3) {
          group_rx[static_cast<size_t>(g)][k] = static_cast<int>(plan[static_cast<size_t>(g)].rx);
          plan[static_cast<size_t>(g)].rx += bytes;
        }
        job_group[k] = g;
      }
    } else if (M == 1 && su == kStreamU && fc <= 1) {
      int off = 0;
      for (auto& j : jobs) {
        j.rx_off = off;
        off += static_cast<int>((j.K * 2 + 127) / 128 * 128);
      }
      if (stack_smem_bytes(su, M, fc + 3, off) <= kStackSmemLimit) {
        rx_bytes = off;
        fc_sel = fc + 3;
      }
    }
    for (int i = 0; i < n; ++i) {
      const size_t jk = job_of[static_cast<size_t>(i)];
      const q4k::XPrepJob* j = &jobs[jk];
      host[static_cast<size_t>(i)].xc = j->xc;
      host[static_cast<size_t>(i)].xinfo = j->info;
      host[static_cast<size_t>(i)].rx_off =
          grouped ? group_rx[static_cast<size_t>(job_group[jk])][jk] : j->rx_off;
    }
    // the preparation's job table, then per group a copy with that group's
    // shared-memory offsets (the tensors it stages)
    std::vector<q4k::XPrepJob> tables(jobs);
    for (size_t g = 0; g < plan.size(); ++g)
      for (size_t k = 0; k < jobs.size(); ++k) {
        tables.push_back(jobs[k]);
        tables.back().rx_off = group_rx[g][k];
      }
    err = cudaMalloc(&st->xprep_dev, sizeof(q4k::XPrepJob) * tables.size());
    if (err == cudaSuccess)
      err = cudaMemcpy(st->xprep_dev, tables.data(), sizeof(q4k::XPrepJob) * tables.size(), cudaMemcpyHostToDevice);
    st->xprep_jobs = static_cast<int>(jobs.size());
    st->rx_bytes = rx_bytes;
    long long most = 0;
    for (const auto& j : jobs) most = std::max(most, static_cast<long long>(M) * j.K / 8);
    st->xprep_ctas = static_cast<int>(std::max(1LL, (most + q4k::kXPrepThreads - 1) / q4k::kXPrepThreads));
  }
  // groups: the entries ordered by group, each group's blocks (of its own
  // stage size) numbered from 0
  std::vector<size_t> group_first(plan.size() + 1, 0);
  std::vector<long long> group_blocks(plan.size(), 0);
  if (grouped) {
    std::vector<q4k::StackEntryDev> sorted;
    for (size_t g = 0; g < plan.size(); ++g) {
      group_first[g] = sorted.size();
      for (int i = 0; i < n; ++i) {
        if (job_group[job_of[static_cast<size_t>(i)]] != static_cast<int>(g)) continue;
        q4k::StackEntryDev d = host[static_cast<size_t>(i)];
        d.blk_off = group_blocks[g];
        group_blocks[g] += d.TC / plan[g].su;
        sorted.push_back(d);
      }
    }
    group_first[plan.size()] = sorted.size();
    host.swap(sorted);
  }
  if (err == cudaSuccess) err = cudaMalloc(&st->entries_dev, sizeof(q4k::StackEntryDev) * host.size());
  if (err == cudaSuccess)
    err = cudaMemcpy(st->entries_dev, host.data(), sizeof(q4k::StackEntryDev) * host.size(), cudaMemcpyHostToDevice);
  if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: allocation");
  st->fn = select_stack_kernel(M, su, fc_sel);
  st->smem = stack_smem_bytes(su, M, fc_sel, rx_bytes);
  st->block = kStackNW * 32;
  st->grid = dev.sms;
  err = allow_dynamic_smem(st->fn);
  if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: cudaFuncSetAttribute");
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, st->fn, st->block, st->smem);
  if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: occupancy query");
  if (per_sm < 1) return fail(Q4_ERR_UNSUPPORTED, "layer_stack_create: the stack kernel does not fit on an SM");
  unsigned char* ws = static_cast<unsigned char*>(st->workspace);
  q4k::StackParams& p = st->params;
  p.entries = st->entries_dev;
  p.E = n;
  p.status = reinterpret_cast<unsigned*>(ws);
  p.bar_flags = reinterpret_cast<unsigned*>(ws + flags_base);
  p.partials = reinterpret_cast<float*>(ws + kWsHeader);
  p.counters = reinterpret_cast<unsigned*>(ws + kWsHeader + partials_bytes(dev));
  p.G = st->grid;
  p.timeout_ns = g_timeout_ns.load();
  p.TBg = total_blocks;
  p.Pg = static_cast<int>(total_blocks < warps ? total_blocks : warps);
  p.jobs = st->xprep_dev;
  p.n_jobs = st->xprep_jobs;
  p.rx_bytes = rx_bytes;
  st->persistent = true;
  st->launches = independent ? 2 : 1;  // stream mode: xprep_kernel + stream_kernel
  for (size_t g = 0; grouped && g < plan.size(); ++g) {
    q4_stack::Group grp;
    grp.fn = select_stack_kernel(M, plan[g].su, plan[g].fc);
    grp.smem = stack_smem_bytes(plan[g].su, M, plan[g].fc, static_cast<int>(plan[g].rx));
    err = allow_dynamic_smem(grp.fn);
    if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: cudaFuncSetAttribute");
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, grp.fn, st->block, grp.smem);
    if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: occupancy query");
    if (per_sm < 1) return fail(Q4_ERR_UNSUPPORTED, "layer_stack_create: a stream kernel does not fit on an SM");
    grp.params = p;
    grp.params.entries = st->entries_dev + group_first[g];
    grp.params.E = static_cast<int>(group_first[g + 1] - group_first[g]);
    grp.params.TBg = group_blocks[g];
    grp.params.Pg = static_cast<int>(group_blocks[g] < warps ? group_blocks[g] : warps);
    grp.params.jobs = st->xprep_dev + (g + 1) * jobs.size();
    grp.params.rx_bytes = static_cast<int>(plan[g].rx);
    st->groups.push_back(grp);
  }
  if (grouped) st->launches = 1 + static_cast<int>(st->groups.size());
  return Q4_OK;
}

int create_graph(const q4_stack_entry* entries, int n, int M, int flags, const DeviceInfo& dev, q4_stack* st) {
  size_t ws = kWsHeader;
  for (int i = 0; i < n; ++i) {
    Shape s;
    char who[64];
    snprintf(who, sizeof(who), "layer_stack_create entry %d", i);
    int rc = make_shape(entries[i].bits, entries[i].N, entries[i].K, &s, who);
    if (rc) return rc;
    const size_t need = workspace_bytes(s, M, dev);
    if (need > ws) ws = need;
  }
  cudaError_t err = cudaMalloc(&st->workspace, ws);
  if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: cudaMalloc(workspace)");
  st->workspace_bytes = ws;
  err = cudaMemset(st->workspace, 0, ws);
  if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: cudaMemset(workspace)");
  std::vector<Launch> launches(static_cast<size_t>(n));
  for (int i = 0; i < n; ++i) {
    const q4_stack_entry& en = entries[i];
    char who[64];
    snprintf(who, sizeof(who), "layer_stack_create entry %d", i);
    int rc = prepare(en.bits, en.packed, en.N, en.K, en.x, M, en.y, st->workspace, ws, who, &launches[i]);
    if (rc) return rc;
    launches[i].params.y = en.y;
  }
  cudaStream_t cs = nullptr;
  err = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
  if (err == cudaSuccess) err = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (err != cudaSuccess) {
    if (cs) cudaStreamDestroy(cs);
    return cuda_fail(err, "layer_stack_create: begin capture");
  }
  const bool pdl = (flags & Q4_STACK_NO_PDL) == 0;
  int rc = Q4_OK;
  for (auto& L : launches) {
    if (L.noop) continue;
    rc = launch(L, cs, pdl);
    if (rc) break;
    ++st->launches;
  }
  cudaGraph_t graph = nullptr;
  cudaError_t end_err = cudaStreamEndCapture(cs, &graph);
  cudaStreamDestroy(cs);
  if (rc || end_err != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    return rc ? rc : cuda_fail(end_err, "layer_stack_create: end capture");
  }
  st->graph = graph;
  err = cudaGraphInstantiate(&st->exec, graph, 0);
  if (err != cudaSuccess) return cuda_fail(err, "layer_stack_create: cudaGraphInstantiate");
  return Q4_OK;
}

}  // namespace

extern "C" Q4_API int layer_stack_create(const q4_stack_entry* entries, int n_entries, int M, int flags,
                                         q4_stack** out) {
  if (!out) return fail(Q4_ERR_INVALID_ARG, "layer_stack_create: out is null");
  *out = nullptr;
  if (n_entries < 0 || (n_entries > 0 && !entries))
    return fail(Q4_ERR_INVALID_ARG, "layer_stack_create: bad entry list");
  if (M < 1 || M > 4) return fail(Q4_ERR_INVALID_ARG, "layer_stack_create: M must be in 1..4");
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  // NVFP4, q5 and q6 products run in stream mode only
  for (int i = 0; i < n_entries; ++i) {
    if (!stream_only(entries[i].bits)) continue;
    char who[64];
    snprintf(who, sizeof(who), "layer_stack_create entry %d", i);
    Shape s;
    if ((rc = entry_shape(entries[i].bits, entries[i].N, entries[i].K, &s, who))) return rc;
    if ((flags & Q4_STACK_INDEPENDENT) == 0 || (flags & (Q4_STACK_GRAPH | Q4_STACK_NO_PDL)) != 0)
      return fail(Q4_ERR_UNSUPPORTED, "%s: NVFP4, q5 and q6 products need stream mode (Q4_STACK_INDEPENDENT alone)",
                  who);
    if (!stack_eligible(entries, n_entries))
      return fail(Q4_ERR_UNSUPPORTED, "%s: stream mode needs every product non-empty with an even chunk count", who);
  }
  q4_stack* st = new q4_stack();
  cudaGetDevice(&st->device);
  // graph mode unless a persistent mode is asked for (and the list is eligible)
  const bool graph = (flags & (Q4_STACK_GRAPH | Q4_STACK_NO_PDL)) != 0 ||
                     (flags & (Q4_STACK_INDEPENDENT | Q4_STACK_ORDERED)) == 0 || !stack_eligible(entries, n_entries);
  // stream mode also needs whole q4 chunks (K a multiple of 64); else ordered.
  // Its stages hold kStreamU chunks when every product's chunks per tile is a
  // multiple of kStreamU, else 2.
  int su = (flags & Q4_STACK_INDEPENDENT) != 0 ? kStreamU : 0;
  for (int i = 0; su != 0 && i < n_entries; ++i) {
    if (entries[i].bits == 4 && entries[i].K % 64 != 0) {
      su = 0;
    } else {
      const long long kc = entries[i].bits == 8 ? 32 : 64;
      const long long C = (entries[i].K + kc - 1) / kc;
      if (C % su != 0) su = 2;
    }
  }
  for (int i = 0; i < n_entries; ++i)
    if (stream_only(entries[i].bits) && su == 0) {
      free_stack(st);
      return fail(Q4_ERR_UNSUPPORTED, "layer_stack_create: NVFP4, q5 and q6 products need stream mode, and a q4 "
                                      "product with K %% 64 != 0 rules it out");
    }
  rc = graph ? create_graph(entries, n_entries, M, flags, dev, st)
             : create_persistent(entries, n_entries, M, su, dev, st);
  if (rc) {
    free_stack(st);
    return rc;
  }
  *out = st;
  return Q4_OK;
}

namespace {

int launch_pdl(const void* fn, dim3 grid, dim3 block, void** args, cudaStream_t stream, bool pdl, const char* who) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  const cudaError_t err = cudaLaunchKernelExC(&cfg, fn, args);
  return err == cudaSuccess ? Q4_OK : cuda_fail(err, who);
}

bool misaligned(const void* p, uintptr_t a) { return reinterpret_cast<uintptr_t>(p) % a != 0; }

int check_chain_op(const q4_chain_op& op, int i) {
  char who[64];
  snprintf(who, sizeof(who), "layer_chain_create op %d", i);
  if (op.kind == Q4_OP_PRODUCT) {
    Shape s;
    return make_shape(op.bits, op.N, op.K, &s, who);
  }
  if (op.kind != Q4_OP_RESIDUAL_RMSNORM && op.kind != Q4_OP_SWIGLU)
    return fail(Q4_ERR_INVALID_ARG, "%s: unknown kind %d", who, op.kind);
  if (op.N <= 0 || op.N > (int64_t(1) << 30)) return fail(Q4_ERR_SHAPE, "%s: N must be in 1..2^30", who);
  if (!op.out) return fail(Q4_ERR_INVALID_ARG, "%s: out is null", who);
  if (misaligned(op.out, 2)) return fail(Q4_ERR_ALIGN, "%s: out must be 2-byte aligned", who);
  if (op.kind == Q4_OP_RESIDUAL_RMSNORM) {
    if (!op.resid) return fail(Q4_ERR_INVALID_ARG, "%s: resid is null", who);
    if (op.bits == 1 && !op.in) return fail(Q4_ERR_INVALID_ARG, "%s: a setting norm needs in", who);
    if (misaligned(op.resid, 4) || misaligned(op.in, 4) || misaligned(op.packed, 2))
      return fail(Q4_ERR_ALIGN, "%s: resid and in must be 4-byte, gamma 2-byte aligned", who);
  } else {
    if (!op.in) return fail(Q4_ERR_INVALID_ARG, "%s: in is null", who);
    if (misaligned(op.in, 4)) return fail(Q4_ERR_ALIGN, "%s: in must be 4-byte aligned", who);
  }
  return Q4_OK;
}

}  // namespace

extern "C" Q4_API int q4_residual_rmsnorm(float* h, const float* y, const uint16_t* gamma, uint16_t* x, int64_t N,
                                          int M, int set, void* stream) {
  q4_chain_op op{};
  op.kind = Q4_OP_RESIDUAL_RMSNORM;
  op.bits = set ? 1 : 0;
  op.N = N;
  op.packed = gamma;
  op.in = y;
  op.out = x;
  op.resid = h;
  int rc = check_chain_op(op, 0);
  if (rc) return rc;
  if (M < 1 || M > 4) return fail(Q4_ERR_INVALID_ARG, "q4_residual_rmsnorm: M must be in 1..4");
  int Ni = static_cast<int>(N), seti = set ? 1 : 0;
  float eps = 1e-6f;
  void* args[] = {&h, &y, &gamma, &x, &Ni, &eps, &seti};
  return launch_pdl(reinterpret_cast<const void*>(&q4k::residual_rmsnorm_kernel), dim3(M), dim3(q4k::kNormThreads),
                    args, static_cast<cudaStream_t>(stream), true, "q4_residual_rmsnorm: launch");
}

extern "C" Q4_API int q4_swiglu(const float* y_gu, uint16_t* x, int64_t N, int M, void* stream) {
  q4_chain_op op{};
  op.kind = Q4_OP_SWIGLU;
  op.N = N;
  op.in = y_gu;
  op.out = x;
  int rc = check_chain_op(op, 0);
  if (rc) return rc;
  if (M < 1 || M > 4) return fail(Q4_ERR_INVALID_ARG, "q4_swiglu: M must be in 1..4");
  int Ni = static_cast<int>(N), Mi = M;
  void* args[] = {&y_gu, &x, &Ni, &Mi};
  const long long total = static_cast<long long>(M) * N;
  return launch_pdl(reinterpret_cast<const void*>(&q4k::swiglu_kernel), dim3(static_cast<unsigned>((total + 255) / 256)),
                    dim3(256), args, static_cast<cudaStream_t>(stream), true, "q4_swiglu: launch");
}

namespace {

// A byte range an op reads or writes (empty for a null buffer).
struct Span {
  uintptr_t lo = 0, hi = 0;
  bool overlaps(const Span& o) const { return lo < hi && o.lo < o.hi && lo < o.hi && o.lo < hi; }
};

Span span_of(const void* p, long long bytes) {
  Span sp;
  if (p) {
    sp.lo = reinterpret_cast<uintptr_t>(p);
    sp.hi = sp.lo + static_cast<uintptr_t>(bytes);
  }
  return sp;
}

// The persistent chain: one cooperative chain_kernel launch over the whole op
// list (M = 1..4).  Eligible when every product is q4 or q8 with stages of
// chain_su(M) whole chunks, each step's row length is a multiple of 8, no op
// overwrites a buffer an earlier op reads, no two ops write the same bytes
// (except the residual stream, shared by RMSNorm ops), and the largest
// activation tensor fits shared memory beside the rings.
//  * A step directly after the product whose output it reads runs its
//    elementwise part in that product's tile finishers (RMSNorm: the product's
//    N is the norm's; SwiGLU: the product's N is twice the step's, a multiple
//    of 64); other steps split it between the CTAs and add a barrier.
//  * A grid barrier goes before every op that reads bytes another CTA wrote
//    since the last barrier; a product whose activations are those the CTA
//    itself just computed (the preceding step's output) or already holds, in
//    the same chunk layout, reads them from shared memory.  Consecutive
//    products without a barrier alternate between two split-tile partial
//    buffers, so a barrier also goes before a third.
//  * The RMSNorm ops of one residual stream R read and write it in turn
//    through two workspace buffers: the i-th of c reads R (i = 0) or buffer
//    (i - 1) % 2 and writes buffer i % 2, the last one R.
int chain_su(int M) { return M <= 2 ? 4 : 2; }

template <int M, int SU>
void* chain_kernel_ptr() {
  return reinterpret_cast<void*>(&q4k::chain_kernel<M, kStackNW, kStackD, SU, kChainPF>);
}

void* chain_kernel_for(int M) {
  switch (M) {
    case 1: return chain_kernel_ptr<1, 4>();
    case 2: return chain_kernel_ptr<2, 4>();
    case 3: return chain_kernel_ptr<3, 2>();
    default: return chain_kernel_ptr<4, 2>();
  }
}

int create_chain_persistent(const q4_chain_op* ops, int n, int M, const DeviceInfo& dev, q4_stack* st) {
  const char* who = "layer_chain_create (persistent)";
  if (M < 1 || M > 4) return fail(Q4_ERR_INVALID_ARG, "%s: M must be in 1..4", who);
  const int G = dev.sms;
  const int SU = chain_su(M);
  const long long warps = static_cast<long long>(G) * kStackNW;
  struct Access {
    Span r[2], w;
    Span resid;
  };
  std::vector<Access> acc(static_cast<size_t>(n));
  std::vector<q4k::StackEntryDev> entries;
  std::vector<q4k::ChainOpDev> dops(static_cast<size_t>(n));
  std::vector<int> kc_of(static_cast<size_t>(n), 64);  // products: values per chunk
  long long x_max = 0;
  for (int i = 0; i < n; ++i) {
    const q4_chain_op& op = ops[i];
    q4k::ChainOpDev& d = dops[static_cast<size_t>(i)];
    d = q4k::ChainOpDev{};
    d.pre_next = -1;
    d.pre_off = -1;
    d.src_op = -1;
    d.prep = -1;
    Access& a = acc[static_cast<size_t>(i)];
    if (op.kind == Q4_OP_PRODUCT) {
      Shape s;
      make_shape(op.bits, op.N, op.K, &s, who);
      const int KC = op.bits == 4 ? 64 : 32;
      const long long need = static_cast<long long>(SU) * KC;
      if (s.N == 0 || s.K == 0 || s.K % need != 0)
        return fail(Q4_ERR_UNSUPPORTED, "%s: op %d: products need N > 0 and K a multiple of %lld at M = %d", who, i,
                    need, M);
      if (!op.packed || !op.in || !op.out || misaligned(op.packed, 16) || misaligned(op.in, 16) ||
          misaligned(op.out, 4))
        return fail(Q4_ERR_ALIGN, "%s: op %d: packed and in must be 16-byte aligned, out 4-byte", who, i);
      q4k::StackEntryDev e{};
      e.packed = static_cast<const uint8_t*>(op.packed);
      e.x = static_cast<const uint16_t*>(op.in);
      e.y = static_cast<float*>(op.out);
      e.N = s.N;
      e.K = s.K;
      e.TC = s.TC;
      e.T = s.T;
      e.C = s.C;
      e.bits = op.bits;
      const long long TB = s.TC / SU;
      e.P = static_cast<int>(TB < warps ? TB : warps);  // the split of a one-product stream-mode stack
      d.kind = q4k::kChainProduct;
      d.entry = static_cast<int>(entries.size());
      d.x = e.x;
      d.kc = KC;
      kc_of[static_cast<size_t>(i)] = KC;
      entries.push_back(e);
      a.r[0] = span_of(op.in, static_cast<long long>(M) * s.K * 2);
      a.w = span_of(op.out, static_cast<long long>(M) * s.N * 4);
      x_max = std::max(x_max, s.K);
    } else {
      if (op.N % 8 != 0) return fail(Q4_ERR_UNSUPPORTED, "%s: op %d: step rows must be a multiple of 8", who, i);
      if (op.N > (int64_t(1) << 24)) return fail(Q4_ERR_UNSUPPORTED, "%s: op %d: step row too long", who, i);
      if (misaligned(op.out, 16))  // its outputs are read back 16 bytes at a time
        return fail(Q4_ERR_ALIGN, "%s: op %d: a step's out must be 16-byte aligned", who, i);
      d.kc = 8;  // the activation buffer's layout when no product reads this output from it
      d.N = static_cast<int>(op.N);
      d.out = static_cast<uint16_t*>(op.out);
      d.y = static_cast<const float*>(op.in);
      a.w = span_of(op.out, static_cast<long long>(M) * op.N * 2);
      x_max = std::max(x_max, static_cast<long long>(op.N));
      if (op.kind == Q4_OP_SWIGLU) {
        d.kind = q4k::kChainSwiglu;
        a.r[0] = span_of(op.in, static_cast<long long>(M) * op.N * 8);
      } else {
        d.kind = q4k::kChainRmsnorm;
        d.set = op.bits == 1 ? 1 : 0;
        d.gamma = static_cast<const uint16_t*>(op.packed);
        a.r[0] = span_of(op.in, static_cast<long long>(M) * op.N * 4);
        a.r[1] = span_of(op.packed, op.N * 2);
        a.resid = span_of(op.resid, static_cast<long long>(M) * op.N * 4);
      }
    }
  }
  if (entries.empty()) return fail(Q4_ERR_UNSUPPORTED, "%s: no product", who);
  // hazards the kernel does not order
  for (int j = 0; j < n; ++j) {
    const Access& aj = acc[static_cast<size_t>(j)];
    for (int i = 0; i < n; ++i) {
      const Access& ai = acc[static_cast<size_t>(i)];
      if (i <= j && (aj.w.overlaps(ai.r[0]) || aj.w.overlaps(ai.r[1]) || aj.resid.overlaps(ai.r[0]) ||
                     aj.resid.overlaps(ai.r[1])))
        return fail(Q4_ERR_UNSUPPORTED, "%s: op %d writes bytes op %d reads", who, j, i);
      if (aj.r[0].overlaps(ai.resid) || aj.r[1].overlaps(ai.resid))
        return fail(Q4_ERR_UNSUPPORTED, "%s: op %d reads a residual stream", who, j);
      if (i != j && (aj.w.overlaps(ai.w) || aj.w.overlaps(ai.resid) ||
                     (aj.resid.overlaps(ai.resid) && (aj.resid.lo != ai.resid.lo || aj.resid.hi != ai.resid.hi))))
        return fail(Q4_ERR_UNSUPPORTED, "%s: ops %d and %d write the same bytes", who, i, j);
    }
  }
  // the residual streams: norms per stream, in order
  struct Stream {
    float* R;
    long long N;
    std::vector<int> norms;
  };
  std::vector<Stream> streams;
  for (int i = 0; i < n; ++i) {
    if (ops[i].kind != Q4_OP_RESIDUAL_RMSNORM) continue;
    size_t k = 0;
    while (k < streams.size() && streams[k].R != ops[i].resid) ++k;
    if (k == streams.size()) streams.push_back(Stream{ops[i].resid, ops[i].N, {}});
    if (streams[k].N != ops[i].N)
      return fail(Q4_ERR_UNSUPPORTED, "%s: op %d: one residual stream with two lengths", who, i);
    streams[k].norms.push_back(i);
  }
  // fused steps, epilogues, chunk layouts of the activation buffer, tagged words
  long long n_words = 0;
  auto words = [&](long long count) {
    const long long at = n_words;
    n_words += (count + 31) / 32 * 32;
    return at;
  };
  for (int j = 0; j < n; ++j) {
    const q4_chain_op& op = ops[j];
    if (op.kind == Q4_OP_PRODUCT) continue;
    q4k::ChainOpDev& d = dops[static_cast<size_t>(j)];
    if (j + 1 < n && ops[j + 1].kind == Q4_OP_PRODUCT && ops[j + 1].in == op.out && ops[j + 1].K == op.N)
      d.kc = kc_of[static_cast<size_t>(j + 1)];
    const bool after_product = j > 0 && ops[j - 1].kind == Q4_OP_PRODUCT && op.in && ops[j - 1].out == op.in;
    const long long tiles = (op.N + q4k::kTileRows - 1) / q4k::kTileRows;
    if (op.kind == Q4_OP_RESIDUAL_RMSNORM) {
      // its tile sums of squares go to the warps' scratch, one float per tile and row
      if (tiles * M > static_cast<long long>(kStackNW) * M * q4k::kTileRows)
        return fail(Q4_ERR_UNSUPPORTED, "%s: op %d: a norm row of more than %d values", who, j,
                    kStackNW * q4k::kTileRows * q4k::kTileRows);
      d.tw = static_cast<int>(words(M * op.N));
      d.epi = after_product && ops[j - 1].N == op.N ? 1 : 0;
    } else {
      d.tw = static_cast<int>(words(M * op.N / 2));
      d.epi = after_product && ops[j - 1].N == 2 * op.N && op.N % q4k::kTileRows == 0 ? 1 : 0;
      if (d.epi) d.uw = static_cast<int>(words(M * op.N));
    }
    if (d.epi) {
      q4k::ChainOpDev& pd = dops[static_cast<size_t>(j - 1)];
      pd.epi = op.kind == Q4_OP_RESIDUAL_RMSNORM ? q4k::kEpiResid : q4k::kEpiSwiglu;
      pd.step = j;
    }
  }
  if (n_words > (1LL << 31) - 1) return fail(Q4_ERR_UNSUPPORTED, "%s: the steps' words exceed 2^31", who);
  // Products whose activations are not in the CTA's buffer (the op before
  // them neither computed nor read them in the same layout) stage them.  A
  // staged product whose activations no op writes, right after an op that
  // leaves the buffer's tail free, gets a prepared copy: the launch converts
  // it first, and the op before copies it into the tail, where it is read in
  // place.
  {
    const void* t = nullptr;
    long long tn = 0;
    int tk = 0;
    for (int j = 0; j < n; ++j) {
      const q4_chain_op& op = ops[j];
      q4k::ChainOpDev& d = dops[static_cast<size_t>(j)];
      if (op.kind == Q4_OP_PRODUCT) {
        d.stage_x = (op.in == t && op.K == tn && d.kc == tk) ? 0 : 1;
        t = op.in;
        tn = op.K;
      } else {
        t = op.out;
        tn = op.N;
      }
      tk = d.kc;
    }
  }
  const long long X = static_cast<long long>(M) * x_max * 2;  // the activation buffer's bytes
  std::vector<int> prep_ops;
  long long prep_values = 0;
  for (int p = 1; p < n; ++p) {
    q4k::ChainOpDev& d = dops[static_cast<size_t>(p)];
    if (ops[p].kind != Q4_OP_PRODUCT || !d.stage_x || dops[static_cast<size_t>(p - 1)].pre_off >= 0) continue;
    bool written = false;
    for (int i = 0; i < n; ++i)
      if (acc[static_cast<size_t>(i)].w.overlaps(acc[static_cast<size_t>(p)].r[0]) ||
          acc[static_cast<size_t>(i)].resid.overlaps(acc[static_cast<size_t>(p)].r[0]))
        written = true;
    const long long used = static_cast<long long>(M) * (ops[p - 1].kind == Q4_OP_PRODUCT ? ops[p - 1].K : ops[p - 1].N) * 2;
    const long long need = static_cast<long long>(M) * ops[p].K * 2;
    if (written || used + need > X) continue;
    d.pre_off = static_cast<int>(X - need);
    d.prep = static_cast<int>(prep_ops.size());
    d.prep_at = prep_values;
    prep_values += static_cast<long long>(M) * ops[p].K;
    prep_ops.push_back(p);
    dops[static_cast<size_t>(p - 1)].pre_next = p;
    entries[static_cast<size_t>(d.entry)].rx_off = d.pre_off;  // the product reads the copy in place
  }
  // a product after a prepared one reads its activations from the start of
  // the buffer, not from the tail: it stages them itself
  for (int p = 1; p < n; ++p)
    if (ops[p].kind == Q4_OP_PRODUCT && !dops[static_cast<size_t>(p)].stage_x &&
        dops[static_cast<size_t>(p - 1)].prep >= 0)
      dops[static_cast<size_t>(p)].stage_x = 1;
  // Grid barriers (the fallback): a product that stages its activations from
  // global memory itself, or a step not fed by the product before it, reads
  // bytes that other CTAs write with plain stores, so it needs a barrier when
  // it reads bytes written since the last one.  A product reusing a partial
  // buffer needs one unless, since the buffer's last user, a step has waited
  // for every tile of a product to which every warp contributes (so every
  // warp has finished the last user).
  std::vector<Span> since;  // bytes written since the last barrier
  const void* tag = nullptr;
  long long tag_n = 0;
  int tag_kc = 0;
  int n_products = 0;
  std::vector<int> pbuf_user(q4k::kChainPartialBufs, -1);  // product index of each buffer's last user
  int last_completion = -1;                                 // product index of the last awaited full product
  for (int j = 0; j < n; ++j) {
    const q4_chain_op& op = ops[j];
    q4k::ChainOpDev& d = dops[static_cast<size_t>(j)];
    const Access& aj = acc[static_cast<size_t>(j)];
    const bool resident = op.kind == Q4_OP_PRODUCT && op.in == tag && op.K == tag_n && d.kc == tag_kc;
    const bool reads_plain = (op.kind == Q4_OP_PRODUCT && !resident && d.prep < 0) ||
                             (op.kind != Q4_OP_PRODUCT && !d.epi);
    bool need = false;
    if (reads_plain)
      for (const Span& w : since)
        if (aj.r[0].overlaps(w) || aj.r[1].overlaps(w) || aj.resid.overlaps(w)) need = true;
    if (op.kind == Q4_OP_PRODUCT) {
      const int pb = n_products % q4k::kChainPartialBufs;
      if (pbuf_user[static_cast<size_t>(pb)] >= 0 && last_completion <= pbuf_user[static_cast<size_t>(pb)]) need = true;
    }
    if (need) {
      d.barrier = 1;
      since.clear();
      last_completion = n_products - 1;  // every product so far is complete
    }
    if (op.kind == Q4_OP_PRODUCT) {
      d.pbuf = n_products % q4k::kChainPartialBufs;
      pbuf_user[static_cast<size_t>(d.pbuf)] = n_products;
      ++n_products;
      tag = op.in;
      tag_n = op.K;
      tag_kc = d.kc;
      since.push_back(aj.w);
    } else {
      if (d.epi && entries[static_cast<size_t>(dops[static_cast<size_t>(j - 1)].entry)].P == warps)
        last_completion = n_products - 1;
      tag = op.out;
      tag_n = op.N;
      tag_kc = d.kc;
      since.push_back(aj.w);
      since.push_back(aj.resid);
    }
  }
  long long max_tiles = 0;  // of a norm row
  for (int j = 0; j < n; ++j)
    if (ops[j].kind == Q4_OP_RESIDUAL_RMSNORM) max_tiles = std::max<long long>(max_tiles, (ops[j].N + 31) / 32);
  const int rings = kStackNW * kStackD * SU * q4k::Format<4>::kChunkBytes;
  const long long x_off = (rings + kStackNW * kStackD * 8 + 127) / 128 * 128;
  const long long scr_off = x_off + (X + 127) / 128 * 128;
  const long long tiles_off = scr_off + static_cast<long long>(kStackNW) * M * q4k::kTileRows * 4;
  const long long smem = tiles_off + (M * max_tiles * 4 + 127) / 128 * 128;
  if (smem > kStackSmemLimit - 1024)
    return fail(Q4_ERR_UNSUPPORTED, "%s: activations of %lld values x M = %d exceed shared memory", who, x_max, M);
  // workspace: [status | partial buffers | tagged words | per-CTA run counters | barrier counter]
  auto up256 = [](size_t v) { return (v + 255) / 256 * 256; };
  const long long pbuf_words = warps * M * q4k::kTileRows;
  const size_t parts_at = kWsHeader;
  const size_t words_at = parts_at + up256(static_cast<size_t>(q4k::kChainPartialBufs * pbuf_words) * 8);
  const size_t run_at = words_at + up256(static_cast<size_t>(n_words) * 8);
  const size_t bar_at = run_at + up256(static_cast<size_t>(G) * 4);
  const size_t prep_at = bar_at + 256;
  const size_t prep_info_at = prep_at + up256(static_cast<size_t>(prep_values) * 2);
  const size_t prep_ops_at = prep_info_at + up256(prep_ops.size() * 8);
  st->workspace_bytes = prep_ops_at + up256(prep_ops.size() * 4);
  cudaError_t err = cudaMalloc(&st->workspace, st->workspace_bytes);
  if (err == cudaSuccess) err = cudaMemset(st->workspace, 0, st->workspace_bytes);
  if (err != cudaSuccess) return cuda_fail(err, "layer_chain_create: workspace");
  unsigned char* ws = static_cast<unsigned char*>(st->workspace);
  // the norms of a stream: each adds to the previous one's tagged h; the
  // first reads the caller's buffer (unless it sets h), the last writes it
  for (const Stream& sr : streams) {
    const size_t c = sr.norms.size();
    for (size_t i = 0; i < c; ++i) {
      q4k::ChainOpDev& d = dops[static_cast<size_t>(sr.norms[i])];
      d.src_op = i == 0 ? -1 : sr.norms[i - 1];
      d.h_src = i == 0 ? sr.R : nullptr;
      d.h_dst = i + 1 == c ? sr.R : nullptr;
    }
  }
  err = cudaMalloc(&st->entries_dev, sizeof(q4k::StackEntryDev) * entries.size());
  if (err == cudaSuccess)
    err = cudaMemcpy(st->entries_dev, entries.data(), sizeof(q4k::StackEntryDev) * entries.size(),
                     cudaMemcpyHostToDevice);
  if (err == cudaSuccess && !prep_ops.empty())
    err = cudaMemcpy(ws + prep_ops_at, prep_ops.data(), prep_ops.size() * 4, cudaMemcpyHostToDevice);
  if (err == cudaSuccess) err = cudaMalloc(&st->chain_ops_dev, sizeof(q4k::ChainOpDev) * dops.size());
  if (err == cudaSuccess)
    err = cudaMemcpy(st->chain_ops_dev, dops.data(), sizeof(q4k::ChainOpDev) * dops.size(), cudaMemcpyHostToDevice);
  if (err != cudaSuccess) return cuda_fail(err, "layer_chain_create: allocation");
  st->fn = chain_kernel_for(M);
  st->smem = static_cast<int>(smem);
  st->block = kStackNW * 32;
  st->grid = G;
  err = allow_dynamic_smem(st->fn);
  if (err != cudaSuccess) return cuda_fail(err, "layer_chain_create: cudaFuncSetAttribute");
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, st->fn, st->block, st->smem);
  if (err != cudaSuccess) return cuda_fail(err, "layer_chain_create: occupancy query");
  if (per_sm < 1) return fail(Q4_ERR_UNSUPPORTED, "%s: the chain kernel does not fit on an SM", who);
  q4k::ChainParams& p = st->chain_params;
  p.ops = st->chain_ops_dev;
  p.n_ops = n;
  p.entries = st->entries_dev;
  p.E = static_cast<int>(entries.size());
  p.parts = reinterpret_cast<unsigned long long*>(ws + parts_at);
  p.pbuf_words = pbuf_words;
  p.words = reinterpret_cast<unsigned long long*>(ws + words_at);
  p.run_ctr = reinterpret_cast<unsigned*>(ws + run_at);
  p.bar_count = reinterpret_cast<unsigned long long*>(ws + bar_at);
  p.prep = reinterpret_cast<uint16_t*>(ws + prep_at);
  p.prep_info = reinterpret_cast<int*>(ws + prep_info_at);
  p.prep_ops = reinterpret_cast<const int*>(ws + prep_ops_at);
  p.n_prep = static_cast<int>(prep_ops.size());
  p.tiles_off = static_cast<int>(tiles_off);
  p.status = reinterpret_cast<unsigned*>(ws);
  p.G = G;
  p.x_off = static_cast<int>(x_off);
  p.scr_off = static_cast<int>(scr_off);
  p.timeout_ns = g_timeout_ns.load();
  st->chain = true;
  st->M = M;
  st->launches = 1;
  return Q4_OK;
}

}  // namespace

extern "C" Q4_API int layer_chain_create(const q4_chain_op* ops, int n_ops, int M, int flags, q4_stack** out) {
  if (!out) return fail(Q4_ERR_INVALID_ARG, "layer_chain_create: out is null");
  *out = nullptr;
  if (n_ops < 0 || (n_ops > 0 && !ops)) return fail(Q4_ERR_INVALID_ARG, "layer_chain_create: bad op list");
  if (M < 1 || M > 4) return fail(Q4_ERR_INVALID_ARG, "layer_chain_create: M must be in 1..4");
  DeviceInfo dev;
  int rc = device_info(&dev);
  if (rc) return rc;
  size_t ws = kWsHeader;
  for (int i = 0; i < n_ops; ++i) {
    if ((rc = check_chain_op(ops[i], i))) return rc;
    if (ops[i].kind == Q4_OP_PRODUCT) {
      Shape s;
      make_shape(ops[i].bits, ops[i].N, ops[i].K, &s, "layer_chain_create");
      ws = std::max(ws, workspace_bytes(s, M, dev));
    }
  }
  if ((flags & Q4_CHAIN_PERSISTENT) && (flags & (Q4_CHAIN_GRAPH | Q4_STACK_NO_PDL)))
    return fail(Q4_ERR_INVALID_ARG, "layer_chain_create: Q4_CHAIN_PERSISTENT with a graph flag");
  // without a form named: the graph (measured faster on the 64-layer decode
  // chain at M = 1 and 4); the single launch only when asked for
  if (flags & Q4_CHAIN_PERSISTENT) {
    q4_stack* st = new q4_stack();
    cudaGetDevice(&st->device);
    rc = create_chain_persistent(ops, n_ops, M, dev, st);
    if (rc == Q4_OK) {
      *out = st;
      return Q4_OK;
    }
    free_stack(st);
    return rc;
  }
  q4_stack* st = new q4_stack();
  cudaGetDevice(&st->device);
  cudaError_t err = cudaMalloc(&st->workspace, ws);
  if (err == cudaSuccess) err = cudaMemset(st->workspace, 0, ws);
  if (err != cudaSuccess) {
    free_stack(st);
    return cuda_fail(err, "layer_chain_create: workspace");
  }
  st->workspace_bytes = ws;
  std::vector<Launch> products(static_cast<size_t>(n_ops));
  for (int i = 0; i < n_ops; ++i) {
    if (ops[i].kind != Q4_OP_PRODUCT) continue;
    char who[64];
    snprintf(who, sizeof(who), "layer_chain_create op %d", i);
    rc = prepare(ops[i].bits, ops[i].packed, ops[i].N, ops[i].K, static_cast<const uint16_t*>(ops[i].in), M,
                 static_cast<float*>(ops[i].out), st->workspace, ws, who, &products[static_cast<size_t>(i)]);
    if (rc) {
      free_stack(st);
      return rc;
    }
  }
  cudaStream_t cs = nullptr;
  err = cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking);
  if (err == cudaSuccess) err = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal);
  if (err != cudaSuccess) {
    if (cs) cudaStreamDestroy(cs);
    free_stack(st);
    return cuda_fail(err, "layer_chain_create: begin capture");
  }
  const bool pdl = (flags & Q4_STACK_NO_PDL) == 0;
  for (int i = 0; i < n_ops && rc == Q4_OK; ++i) {
    const q4_chain_op& op = ops[i];
    if (op.kind == Q4_OP_PRODUCT) {
      Launch& L = products[static_cast<size_t>(i)];
      if (L.noop) continue;
      rc = launch(L, cs, pdl);
    } else if (op.kind == Q4_OP_RESIDUAL_RMSNORM) {
      float* h = op.resid;
      const float* y = static_cast<const float*>(op.in);
      const uint16_t* gamma = static_cast<const uint16_t*>(op.packed);
      uint16_t* x = static_cast<uint16_t*>(op.out);
      int N = static_cast<int>(op.N);
      float eps = 1e-6f;
      int set = op.bits == 1 ? 1 : 0;
      void* args[] = {&h, &y, &gamma, &x, &N, &eps, &set};
      rc = launch_pdl(reinterpret_cast<const void*>(&q4k::residual_rmsnorm_kernel), dim3(M), dim3(q4k::kNormThreads),
                      args, cs, pdl, "layer_chain_create: rmsnorm launch");
    } else {
      const float* y = static_cast<const float*>(op.in);
      uint16_t* x = static_cast<uint16_t*>(op.out);
      int N = static_cast<int>(op.N), Mi = M;
      void* args[] = {&y, &x, &N, &Mi};
      const long long total = static_cast<long long>(M) * op.N;
      rc = launch_pdl(reinterpret_cast<const void*>(&q4k::swiglu_kernel),
                      dim3(static_cast<unsigned>((total + 255) / 256)), dim3(256), args, cs, pdl,
                      "layer_chain_create: swiglu launch");
    }
    if (rc == Q4_OK) ++st->launches;
  }
  cudaGraph_t graph = nullptr;
  const cudaError_t end_err = cudaStreamEndCapture(cs, &graph);
  cudaStreamDestroy(cs);
  if (rc || end_err != cudaSuccess) {
    if (graph) cudaGraphDestroy(graph);
    free_stack(st);
    return rc ? rc : cuda_fail(end_err, "layer_chain_create: end capture");
  }
  st->graph = graph;
  err = cudaGraphInstantiate(&st->exec, graph, 0);
  if (err != cudaSuccess) {
    free_stack(st);
    return cuda_fail(err, "layer_chain_create: cudaGraphInstantiate");
  }
  *out = st;
  return Q4_OK;
}

extern "C" Q4_API int layer_stack_run(q4_stack* st, void* stream) {
  if (!st) return fail(Q4_ERR_INVALID_ARG, "layer_stack_run: null stack");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (st->chain) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(st->grid);
    cfg.blockDim = dim3(st->block);
    cfg.dynamicSmemBytes = static_cast<size_t>(st->smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;  // its grid barriers need every CTA resident
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    void* args[] = {&st->chain_params};
    cudaError_t err = cudaLaunchKernelExC(&cfg, st->fn, args);
    return err == cudaSuccess ? Q4_OK : cuda_fail(err, "layer_stack_run: chain launch");
  }
  if (st->persistent) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(st->grid);
    cfg.blockDim = dim3(st->block);
    cfg.dynamicSmemBytes = static_cast<size_t>(st->smem);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    if (st->cooperative) {
      attr[0].id = cudaLaunchAttributeCooperative;  // all CTAs resident, or the launch fails
      attr[0].val.cooperative = 1;
    } else {
      // stream mode: the activation preparation, then the stream kernel,
      // which has no grid barrier: a plain launch that starts its weight
      // copies while xprep_kernel runs and waits for it (griddepcontrol.wait)
      // before it reads an activation
      q4k::xprep_kernel<<<dim3(st->xprep_ctas, st->xprep_jobs), q4k::kXPrepThreads, 0, s>>>(st->xprep_dev, st->M);
      cudaError_t perr = cudaGetLastError();
      if (perr != cudaSuccess) return cuda_fail(perr, "layer_stack_run: xprep_kernel launch");
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
    }
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    // groups: one launch each, every one after the one before (programmatic
    // dependent launch: a group starts its weight copies while the one before
    // finishes, and waits for it before it reads an activation or the
    // workspace)
    for (auto& grp : st->groups) {
      cfg.dynamicSmemBytes = static_cast<size_t>(grp.smem);
      void* gargs[] = {&grp.params};
      cudaError_t err = cudaLaunchKernelExC(&cfg, grp.fn, gargs);
      if (err != cudaSuccess) return cuda_fail(err, "layer_stack_run: stream group launch");
    }
    if (!st->groups.empty()) return Q4_OK;
    void* args[] = {&st->params};
    cudaError_t err = cudaLaunchKernelExC(&cfg, st->fn, args);
    return err == cudaSuccess ? Q4_OK : cuda_fail(err, "layer_stack_run: persistent launch");
  }
  if (!st->exec) return Q4_OK;  // nothing to run
  cudaError_t err = cudaGraphLaunch(st->exec, s);
  return err == cudaSuccess ? Q4_OK : cuda_fail(err, "cudaGraphLaunch");
}

extern "C" Q4_API int layer_stack_check(q4_stack* st, void* stream) {
  if (!st) return fail(Q4_ERR_INVALID_ARG, "layer_stack_check: null stack");
  return q4_workspace_check(st->workspace, st->workspace_bytes, stream);
}

extern "C" Q4_API int layer_stack_launches(const q4_stack* st) { return st ? st->launches : 0; }

extern "C" Q4_API void layer_stack_destroy(q4_stack* st) {
  if (!st) return;
  free_stack(st);
}
