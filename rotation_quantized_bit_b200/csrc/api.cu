// api.cu -- the extern "C" boundary of libconvrot_b200.so (declared in
// include/convrot.h).  Validates arguments on the host, carves the caller's
// workspace and enqueues the kernels on the caller's stream.  No allocation,
// no host synchronisation (except convrot_device_error, which is a query).
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/convrot.h"
#include "kernels.cuh"
#include "ptx.cuh"

namespace convrot {

__device__ uint32_t g_device_error = 0;

namespace {

std::atomic<uint64_t> g_counts[kDispatchKinds];

constexpr int kMaxK = 32768;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Cached per device: is it sm_100?  and its SM count.
struct DeviceInfo {
  int ok = -1;  // -1 unknown, 0 no, 1 yes
  int sms = 0;
};
DeviceInfo g_dev[64];

convrot_status_t check_device(int* sms_out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return CONVROT_ERR_DEVICE;
  if (dev >= 64) return CONVROT_ERR_DEVICE;
  DeviceInfo& d = g_dev[dev];
  if (d.ok < 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return CONVROT_ERR_DEVICE;
    d.ok = (major == 10 && minor == 0) ? 1 : 0;
    d.sms = sms;
  }
  if (d.ok != 1) return CONVROT_ERR_DEVICE;
  if (sms_out) *sms_out = d.sms;
  return CONVROT_OK;
}

convrot_status_t check_mk(int M, int K) {
  if (M < 1 || K < 256 || K % 256 != 0 || K > kMaxK) return CONVROT_ERR_SHAPE;
  return CONVROT_OK;
}

convrot_status_t check_mnk(int M, int N, int K) {
  if (check_mk(M, K) != CONVROT_OK || N < 1 || N % 8 != 0) return CONVROT_ERR_SHAPE;
  return CONVROT_OK;
}

convrot_status_t from_cuda(cudaError_t e) { return e == cudaSuccess ? CONVROT_OK : CONVROT_ERR_CUDA; }

convrot_status_t check_device(int* sms_out);

size_t round_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Workspace layout shared by the GEMM and the fused Linear:
//   codes   [M*K] bytes   activation codes as signed bytes (operand layout)
//   s_a     [M] float     per-token scales (fused Linear only)
// each region starting on a 256-byte boundary.
size_t codes_bytes(int M, int K) { return round_up(static_cast<size_t>(M) * static_cast<size_t>(K), 256); }
size_t sa_offset(int M, int K) { return codes_bytes(M, K); }
size_t workspace_bytes_for(int M, int K) {
  return sa_offset(M, K) + round_up(static_cast<size_t>(M) * sizeof(float), 256);
}
// M <= kSmallMaxM takes the small-M kernels: the codes region holds packed
// codes (M*K/2 of its M*K bytes), and the GEMM's scratch (counters and
// partial slabs where it splits K) follows the scales.
bool small_m(int M) { return M <= kSmallMaxM; }
size_t fused_ws_bytes(int M, int N, int K) {
  return workspace_bytes_for(M, K) + (small_m(M) ? small_gemm_scratch_bytes(M, N, K) : 0);
}

convrot_status_t gemm_common(const uint8_t* xq, const float* s_a, const uint8_t* Wq, const float* s_w,
                             const uint16_t* bias, int M, int N, int K, void* out, GemmSink sink, void* ws,
                             size_t ws_bytes, void* stream) {
  if (!xq || !Wq || !out) return CONVROT_ERR_NULL;
  if (sink != GemmSink::kS32 && (!s_a || !s_w)) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(xq) || !aligned16(Wq) || !aligned16(out) || (s_a && !aligned16(s_a)) ||
      (s_w && !aligned16(s_w)) || (bias && !aligned16(bias)))
    return CONVROT_ERR_ALIGN;
  if (!ws || ws_bytes < (small_m(M) ? small_gemm_scratch_bytes(M, N, K) : codes_bytes(M, K)))
    return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  int sms = 0;
  st = check_device(&sms);
  if (st != CONVROT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (small_m(M))  // the small-M GEMM reads the packed codes as they are
    return from_cuda(launch_small_gemm(xq, s_a, Wq, s_w, bias, M, N, K, out, sink, ws, ws_bytes, s));
  int8_t* xs8 = static_cast<int8_t*>(ws);
  if (cudaError_t e = launch_unpack_codes(xq, M, K, xs8, s); e != cudaSuccess) return CONVROT_ERR_CUDA;
  GemmArgs a{xs8, s_a, Wq, s_w, bias, out, M, N, K};
  return from_cuda(launch_w4a4_gemm(a, sink, choose_tiling(M, N, K, sms), s));
}

bool valid_group(int group) { return group == 256 || group == 64 || group == 16; }

convrot_status_t quantize_common(const uint16_t* x, int M, int K, void* ws, size_t ws_bytes, void* stream,
                                 int group = 256) {
  if (!x) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mk(M, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x)) return CONVROT_ERR_ALIGN;
  if (!ws || ws_bytes < workspace_bytes_for(M, K)) return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  st = check_device(nullptr);
  if (st != CONVROT_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (small_m(M))
    return from_cuda(launch_small_rotate_quant(x, M, K, group, base, reinterpret_cast<float*>(base + sa_offset(M, K)),
                                               static_cast<cudaStream_t>(stream)));
  RotateQuantOut o{nullptr, reinterpret_cast<int8_t*>(base), reinterpret_cast<float*>(base + sa_offset(M, K))};
  o.group = group;
  return from_cuda(launch_rotate_quant(x, M, K, o, static_cast<cudaStream_t>(stream)));
}

convrot_status_t gemm_quantized_common(const uint8_t* Wq, const float* s_w, const uint16_t* bias, int M, int N,
                                       int K, void* out, GemmSink sink, void* ws, size_t ws_bytes,
                                       void* stream) {
  if (!Wq || !s_w || !out) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(Wq) || !aligned16(s_w) || !aligned16(out) || (bias && !aligned16(bias))) return CONVROT_ERR_ALIGN;
  if (!ws || ws_bytes < fused_ws_bytes(M, N, K)) return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  int sms = 0;
  st = check_device(&sms);
  if (st != CONVROT_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(ws);
  if (small_m(M))
    return from_cuda(launch_small_gemm(base, reinterpret_cast<const float*>(base + sa_offset(M, K)), Wq, s_w, bias, M,
                                       N, K, out, sink, base + workspace_bytes_for(M, K),
                                       ws_bytes - workspace_bytes_for(M, K), static_cast<cudaStream_t>(stream)));
  GemmArgs a{reinterpret_cast<const int8_t*>(base), reinterpret_cast<const float*>(base + sa_offset(M, K)), Wq, s_w,
             bias, out, M, N, K};
  return from_cuda(launch_w4a4_gemm(a, sink, choose_tiling(M, N, K, sms), static_cast<cudaStream_t>(stream)));
}

convrot_status_t linear_common(const uint16_t* x, const uint8_t* Wq, const float* s_w, const uint16_t* bias, int M,
                               int N, int K, void* out, GemmSink sink, void* ws, size_t ws_bytes, void* stream,
                               int group = 256) {
  if (!x || !Wq || !s_w || !out) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x) || !aligned16(Wq) || !aligned16(s_w) || !aligned16(out) || (bias && !aligned16(bias)))
    return CONVROT_ERR_ALIGN;
  if (!ws || ws_bytes < fused_ws_bytes(M, N, K)) return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  if (!valid_group(group)) return CONVROT_ERR_SHAPE;
  st = quantize_common(x, M, K, ws, ws_bytes, stream, group);
  if (st != CONVROT_OK) return st;
  return gemm_quantized_common(Wq, s_w, bias, M, N, K, out, sink, ws, ws_bytes, stream);
}

// ---- int8 W8A8 formats

bool valid_format(int format) { return format == W8A8_INT8_TENSORWISE || format == W8A8_CONVROT_INT8_ROW; }

// Workspace of the int8 path: codes [M*K], scales [M] (or [1]), 4 bytes of
// reduction scratch; each on a 256-byte boundary.
size_t w8_scales_offset(int M, int K) { return codes_bytes(M, K); }
size_t w8_scratch_offset(int M, int K) { return w8_scales_offset(M, K) + round_up(static_cast<size_t>(M) * 4, 256); }
size_t w8_workspace_bytes(int M, int K) { return w8_scratch_offset(M, K) + 256; }

// Quantize rows of a bf16 [rows, K] matrix into int8 codes and scales.
convrot_status_t quant8_common(const uint16_t* x, int rows, int K, int format, int8_t* codes, float* scales,
                               void* ws, size_t ws_bytes, void* stream, bool weights = false) {
  if (!x || !codes || !scales) return CONVROT_ERR_NULL;
  if (!valid_format(format)) return CONVROT_ERR_SHAPE;
  convrot_status_t st = check_mk(rows, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales)) return CONVROT_ERR_ALIGN;
  st = check_device(nullptr);
  if (st != CONVROT_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (format == W8A8_CONVROT_INT8_ROW) {
    RotateQuantOut o{nullptr, codes, scales};
    o.int8 = true;
    o.early_trigger = !weights;
    return from_cuda(launch_rotate_quant(x, rows, K, o, s));
  }
  if (!ws || ws_bytes < 4) return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  return from_cuda(launch_quant8_tensorwise(x, static_cast<size_t>(rows) * static_cast<size_t>(K), codes, scales,
                                            static_cast<uint32_t*>(ws), s, !weights));
}

convrot_status_t gemm8_common(const int8_t* x8, const float* s_x, const int8_t* Wq8, const float* s_w,
                              const uint16_t* bias, int M, int N, int K, int format, void* out, GemmSink sink,
                              void* stream) {
  if (!x8 || !Wq8 || !out) return CONVROT_ERR_NULL;
  if (sink != GemmSink::kS32 && (!s_x || !s_w)) return CONVROT_ERR_NULL;
  if (!valid_format(format)) return CONVROT_ERR_SHAPE;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x8) || !aligned16(Wq8) || !aligned16(out) || (s_x && !aligned16(s_x)) ||
      (s_w && !aligned16(s_w)) || (bias && !aligned16(bias)))
    return CONVROT_ERR_ALIGN;
  int sms = 0;
  st = check_device(&sms);
  if (st != CONVROT_OK) return st;
  GemmArgs a{x8, s_x, reinterpret_cast<const uint8_t*>(Wq8), s_w, bias, out, M, N, K};
  a.wkind = kWInt8;
  a.sa_stride = format == W8A8_CONVROT_INT8_ROW ? 1 : 0;
  a.sw_stride = format == W8A8_CONVROT_INT8_ROW ? 1 : 0;
  return from_cuda(launch_w4a4_gemm(a, sink, choose_tiling(M, N, K, sms, kWInt8), static_cast<cudaStream_t>(stream)));
}

convrot_status_t linear8_common(const uint16_t* x, const int8_t* Wq8, const float* s_w, const uint16_t* bias, int M,
                                int N, int K, int format, void* out, GemmSink sink, void* ws, size_t ws_bytes,
                                void* stream) {
  if (!x || !Wq8 || !s_w || !out) return CONVROT_ERR_NULL;
  if (!valid_format(format)) return CONVROT_ERR_SHAPE;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!ws || ws_bytes < w8_workspace_bytes(M, K)) return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int8_t* codes = reinterpret_cast<int8_t*>(base);
  float* scales = reinterpret_cast<float*>(base + w8_scales_offset(M, K));
  st = quant8_common(x, M, K, format, codes, scales, base + w8_scratch_offset(M, K), 256, stream);
  if (st != CONVROT_OK) return st;
  return gemm8_common(codes, scales, Wq8, s_w, bias, M, N, K, format, out, sink, stream);
}

// ---- asymmetric W4A8 (codebook weights)

convrot_status_t gemm_cb_common(const int8_t* x8, const float* s_a, const uint8_t* idx, const uint8_t* s_rel,
                                const float* codebook, const float* s_channel, const uint16_t* bias, int M, int N,
                                int K, void* out, GemmSink sink, void* stream) {
  if (!x8 || !idx || !s_rel || !codebook || !out) return CONVROT_ERR_NULL;
  if (sink != GemmSink::kS32 && (!s_a || !s_channel)) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x8) || !aligned16(idx) || !aligned16(s_rel) || !aligned16(codebook) || !aligned16(out) ||
      (s_a && !aligned16(s_a)) || (s_channel && !aligned16(s_channel)) || (bias && !aligned16(bias)))
    return CONVROT_ERR_ALIGN;
  int sms = 0;
  st = check_device(&sms);
  if (st != CONVROT_OK) return st;
  GemmArgs a{x8, s_a, idx, s_channel, bias, out, M, N, K};
  a.wkind = kWCodebook;
  a.s_rel = s_rel;
  a.codebook = codebook;
  return from_cuda(
      launch_w4a4_gemm(a, sink, choose_tiling(M, N, K, sms, kWCodebook), static_cast<cudaStream_t>(stream)));
}

convrot_status_t linear_cb_common(const uint16_t* x, const uint8_t* idx, const uint8_t* s_rel, const float* codebook,
                                  const float* s_channel, const uint16_t* bias, int M, int N, int K, void* out,
                                  GemmSink sink, void* ws, size_t ws_bytes, void* stream) {
  if (!x || !idx || !s_rel || !codebook || !s_channel || !out) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mnk(M, N, K);
  if (st != CONVROT_OK) return st;
  if (!ws || ws_bytes < w8_workspace_bytes(M, K)) return CONVROT_ERR_WORKSPACE;
  if (!aligned16(ws)) return CONVROT_ERR_ALIGN;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int8_t* codes = reinterpret_cast<int8_t*>(base);
  float* scales = reinterpret_cast<float*>(base + w8_scales_offset(M, K));
  st = quant8_common(x, M, K, W8A8_CONVROT_INT8_ROW, codes, scales, base + w8_scratch_offset(M, K), 256, stream);
  if (st != CONVROT_OK) return st;
  return gemm_cb_common(codes, scales, idx, s_rel, codebook, s_channel, bias, M, N, K, out, sink, stream);
}

}  // namespace

void count_dispatch(int which) {
  if (which >= 0 && which < kDispatchKinds) g_counts[which].fetch_add(1, std::memory_order_relaxed);
}

namespace {
thread_local char g_last_error[256] = "";

// One thread waits on an mbarrier that nothing ever arrives at; the bounded
// wait gives up after limit_ns and records the timeout bit.
__global__ void selftest_timeout_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait_for(&bar, 0, limit_ns);
}
}  // namespace

cudaError_t launch_selftest_timeout(unsigned int limit_us, cudaStream_t stream) {
  selftest_timeout_kernel<<<1, 32, 0, stream>>>(static_cast<unsigned long long>(limit_us) * 1000ull);
  return note_cuda(cudaGetLastError(), "selftest_timeout: launch");
}

cudaError_t note_cuda(cudaError_t e, const char* where) {
  if (e != cudaSuccess) snprintf(g_last_error, sizeof(g_last_error), "%s: %s (%s)", where, cudaGetErrorName(e),
                                 cudaGetErrorString(e));
  return e;
}

cudaError_t ensure_dynamic_smem(const void* kernel, int bytes, std::atomic<int>* cache) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (bytes <= cache[dev].load(std::memory_order_acquire)) return cudaSuccess;
  // Slow path, once per kernel and device: serialised, so that the limit a
  // kernel is given only ever grows, whichever host thread gets here first.
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  if (bytes <= cache[dev].load(std::memory_order_relaxed)) return cudaSuccess;
  int optin = 0;
  e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  if (bytes + static_cast<int>(fa.sharedSizeBytes) > optin) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) cache[dev].store(bytes, std::memory_order_release);
  return e;
}

}  // namespace convrot

using namespace convrot;

extern "C" {

const char* convrot_status_string(convrot_status_t status) {
  switch (status) {
    case CONVROT_OK: return "CONVROT_OK";
    case CONVROT_ERR_NULL: return "CONVROT_ERR_NULL: a required pointer is NULL";
    case CONVROT_ERR_SHAPE: return "CONVROT_ERR_SHAPE: need M>=1, N>=1, N%8==0, K%256==0, 256<=K<=32768";
    case CONVROT_ERR_ALIGN: return "CONVROT_ERR_ALIGN: pointers must be 16-byte aligned";
    case CONVROT_ERR_DEVICE: return "CONVROT_ERR_DEVICE: needs an sm_100 (B200) device";
    case CONVROT_ERR_WORKSPACE: return "CONVROT_ERR_WORKSPACE: workspace missing or too small";
    case CONVROT_ERR_CUDA: return "CONVROT_ERR_CUDA: a CUDA call failed";
    case CONVROT_ERR_TIMEOUT: return "CONVROT_ERR_TIMEOUT: a bounded device-side wait expired";
  }
  return "CONVROT_ERR_UNKNOWN";
}

const char* convrot_version(void) { return "convrot-b200 sm_100a"; }

const char* convrot_last_error(void) { return g_last_error; }

convrot_status_t convrot_rotate_quant(const uint16_t* x, int M, int K, uint8_t* xq, float* s_a, void* stream) {
  if (!x || !xq || !s_a) return CONVROT_ERR_NULL;
  convrot_status_t st = check_mk(M, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(s_a)) return CONVROT_ERR_ALIGN;
  st = check_device(nullptr);
  if (st != CONVROT_OK) return st;
  RotateQuantOut o{xq, nullptr, s_a};
  return from_cuda(launch_rotate_quant(x, M, K, o, static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_pack_weight(const uint16_t* W, int N, int K, uint8_t* Wq, float* s_w, void* stream) {
  return convrot_pack_weight_g(W, N, K, 256, Wq, s_w, stream);
}

size_t convrot_gemm_workspace_size(int M, int N, int K) {
  if (check_mnk(M, N, K) != CONVROT_OK) return 0;
  return small_m(M) ? small_gemm_scratch_bytes(M, N, K) : codes_bytes(M, K);
}

size_t convrot_w4a4_workspace_size(int M, int N, int K) {
  if (check_mnk(M, N, K) != CONVROT_OK) return 0;
  return fused_ws_bytes(M, N, K);
}

convrot_status_t w4a4_gemm(const uint8_t* xq, const float* s_a, const uint8_t* Wq, const float* s_w,
                           const uint16_t* bias, int M, int N, int K, uint16_t* y, void* workspace,
                           size_t workspace_bytes, void* stream) {
  return gemm_common(xq, s_a, Wq, s_w, bias, M, N, K, y, GemmSink::kBF16, workspace, workspace_bytes, stream);
}

convrot_status_t w4a4_gemm_s32(const uint8_t* xq, const uint8_t* Wq, int M, int N, int K, int32_t* acc,
                               void* workspace, size_t workspace_bytes, void* stream) {
  return gemm_common(xq, nullptr, Wq, nullptr, nullptr, M, N, K, acc, GemmSink::kS32, workspace, workspace_bytes,
                     stream);
}

convrot_status_t w4a4_gemm_f32(const uint8_t* xq, const float* s_a, const uint8_t* Wq, const float* s_w,
                               const uint16_t* bias, int M, int N, int K, float* y32, void* workspace,
                               size_t workspace_bytes, void* stream) {
  return gemm_common(xq, s_a, Wq, s_w, bias, M, N, K, y32, GemmSink::kF32, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_w4a4_linear(const uint16_t* x, const uint8_t* Wq, const float* s_w, const uint16_t* bias,
                                     int M, int N, int K, uint16_t* y, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  return linear_common(x, Wq, s_w, bias, M, N, K, y, GemmSink::kBF16, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_w4a4_linear_f32(const uint16_t* x, const uint8_t* Wq, const float* s_w,
                                         const uint16_t* bias, int M, int N, int K, float* y32, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  return linear_common(x, Wq, s_w, bias, M, N, K, y32, GemmSink::kF32, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_w4a4_quantize(const uint16_t* x, int M, int K, void* workspace, size_t workspace_bytes,
                                       void* stream) {
  return quantize_common(x, M, K, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_w4a4_gemm_quantized(const uint8_t* Wq, const float* s_w, const uint16_t* bias, int M, int N,
                                             int K, uint16_t* y, void* workspace, size_t workspace_bytes,
                                             void* stream) {
  return gemm_quantized_common(Wq, s_w, bias, M, N, K, y, GemmSink::kBF16, workspace, workspace_bytes, stream);
}

convrot_status_t convrot_selftest_timeout(unsigned int limit_us, void* stream) {
  if (limit_us == 0 || limit_us > 1000000u) return CONVROT_ERR_SHAPE;
  convrot_status_t st = check_device(nullptr);
  if (st != CONVROT_OK) return st;
  return from_cuda(launch_selftest_timeout(limit_us, static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_device_error(void* stream, uint32_t* code) {
  if (!code) return CONVROT_ERR_NULL;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return CONVROT_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(v)) != cudaSuccess) return CONVROT_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_device_error, &zero, sizeof(zero)) != cudaSuccess) return CONVROT_ERR_CUDA;
  *code = v;
  return v ? CONVROT_ERR_TIMEOUT : CONVROT_OK;
}

void convrot_dispatch_counts(uint64_t* counts, int n) {
  if (!counts) return;
  for (int i = 0; i < n && i < kDispatchKinds; ++i) counts[i] = g_counts[i].load(std::memory_order_relaxed);
}

}  // extern "C"

extern "C" {

size_t w8a8_workspace_size(int M, int N, int K, int format) {
  if (!valid_format(format) || check_mnk(M, N, K) != CONVROT_OK) return 0;
  return w8_workspace_bytes(M, K);
}

convrot_status_t w8a8_quantize(const uint16_t* x, int M, int K, int format, int8_t* x8, float* s_x, void* workspace,
                               size_t workspace_bytes, void* stream) {
  uint8_t* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (workspace && check_mk(M, K) == CONVROT_OK && workspace_bytes >= w8_workspace_bytes(M, K)) {
    scratch = static_cast<uint8_t*>(workspace) + w8_scratch_offset(M, K);
    scratch_bytes = 256;
  }
  if (format == W8A8_INT8_TENSORWISE && !scratch && check_mk(M, K) == CONVROT_OK && x && x8 && s_x)
    return CONVROT_ERR_WORKSPACE;
  return quant8_common(x, M, K, format, x8, s_x, scratch, scratch_bytes, stream);
}

convrot_status_t w8a8_pack_weight(const uint16_t* W, int N, int K, int format, int8_t* Wq8, float* s_w,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  // w8a8_quantize on W, except that no successor may start before the
  // weights are complete (the GEMMs stream weights before they wait).
  uint8_t* scratch = nullptr;
  size_t scratch_bytes = 0;
  if (workspace && check_mk(N, K) == CONVROT_OK && workspace_bytes >= w8_workspace_bytes(N, K)) {
    scratch = static_cast<uint8_t*>(workspace) + w8_scratch_offset(N, K);
    scratch_bytes = 256;
  }
  if (format == W8A8_INT8_TENSORWISE && !scratch && check_mk(N, K) == CONVROT_OK && W && Wq8 && s_w)
    return CONVROT_ERR_WORKSPACE;
  return quant8_common(W, N, K, format, Wq8, s_w, scratch, scratch_bytes, stream, /*weights=*/true);
}

convrot_status_t w8a8_gemm(const int8_t* x8, const float* s_x, const int8_t* Wq8, const float* s_w,
                           const uint16_t* bias, int M, int N, int K, int format, uint16_t* y, void* stream) {
  return gemm8_common(x8, s_x, Wq8, s_w, bias, M, N, K, format, y, GemmSink::kBF16, stream);
}

convrot_status_t w8a8_gemm_f32(const int8_t* x8, const float* s_x, const int8_t* Wq8, const float* s_w,
                               const uint16_t* bias, int M, int N, int K, int format, float* y32, void* stream) {
  return gemm8_common(x8, s_x, Wq8, s_w, bias, M, N, K, format, y32, GemmSink::kF32, stream);
}

convrot_status_t w8a8_gemm_s32(const int8_t* x8, const int8_t* Wq8, int M, int N, int K, int32_t* acc,
                               void* stream) {
  return gemm8_common(x8, nullptr, Wq8, nullptr, nullptr, M, N, K, W8A8_CONVROT_INT8_ROW, acc, GemmSink::kS32,
                      stream);
}

convrot_status_t w8a8_linear(const uint16_t* x, const int8_t* Wq8, const float* s_w, const uint16_t* bias, int M,
                             int N, int K, int format, uint16_t* y, void* workspace, size_t workspace_bytes,
                             void* stream) {
  return linear8_common(x, Wq8, s_w, bias, M, N, K, format, y, GemmSink::kBF16, workspace, workspace_bytes, stream);
}

convrot_status_t w8a8_linear_f32(const uint16_t* x, const int8_t* Wq8, const float* s_w, const uint16_t* bias,
                                 int M, int N, int K, int format, float* y32, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  return linear8_common(x, Wq8, s_w, bias, M, N, K, format, y32, GemmSink::kF32, workspace, workspace_bytes,
                        stream);
}

}  // extern "C"

extern "C" {

convrot_status_t convrot_rotate_quant_g(const uint16_t* x, int M, int K, int group, uint8_t* xq, float* s_a,
                                        void* stream) {
  if (!x || !xq || !s_a) return CONVROT_ERR_NULL;
  if (!valid_group(group)) return CONVROT_ERR_SHAPE;
  convrot_status_t st = check_mk(M, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(x) || !aligned16(xq) || !aligned16(s_a)) return CONVROT_ERR_ALIGN;
  st = check_device(nullptr);
  if (st != CONVROT_OK) return st;
  RotateQuantOut o{xq, nullptr, s_a};
  o.group = group;
  return from_cuda(launch_rotate_quant(x, M, K, o, static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_pack_weight_g(const uint16_t* W, int N, int K, int group, uint8_t* Wq, float* s_w,
                                       void* stream) {
  // convrot_rotate_quant_g on W, except that no successor may start before
  // the weights are complete (the GEMMs stream weights before they wait).
  if (!W || !Wq || !s_w) return CONVROT_ERR_NULL;
  if (!valid_group(group)) return CONVROT_ERR_SHAPE;
  convrot_status_t st = check_mk(N, K);
  if (st != CONVROT_OK) return st;
  if (!aligned16(W) || !aligned16(Wq) || !aligned16(s_w)) return CONVROT_ERR_ALIGN;
  st = check_device(nullptr);
  if (st != CONVROT_OK) return st;
  RotateQuantOut o{Wq, nullptr, s_w};
  o.group = group;
  o.early_trigger = false;
  return from_cuda(launch_rotate_quant(W, N, K, o, static_cast<cudaStream_t>(stream)));
}

convrot_status_t convrot_w4a4_quantize_g(const uint16_t* x, int M, int K, int group, void* workspace,
                                         size_t workspace_bytes, void* stream) {
  if (!valid_group(group)) return CONVROT_ERR_SHAPE;
  return quantize_common(x, M, K, workspace, workspace_bytes, stream, group);
}

convrot_status_t convrot_w4a4_linear_g(const uint16_t* x, const uint8_t* Wq, const float* s_w, const uint16_t* bias,
                                       int M, int N, int K, int group, uint16_t* y, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  return linear_common(x, Wq, s_w, bias, M, N, K, y, GemmSink::kBF16, workspace, workspace_bytes, stream, group);
}

convrot_status_t convrot_w4a4_linear_g_f32(const uint16_t* x, const uint8_t* Wq, const float* s_w,
                                           const uint16_t* bias, int M, int N, int K, int group, float* y32,
                                           void* workspace, size_t workspace_bytes, void* stream) {
  return linear_common(x, Wq, s_w, bias, M, N, K, y32, GemmSink::kF32, workspace, workspace_bytes, stream, group);
}

}  // extern "C"

extern "C" {

size_t asym_w4a8_workspace_size(int M, int N, int K) {
  if (check_mnk(M, N, K) != CONVROT_OK) return 0;
  return w8_workspace_bytes(M, K);
}

convrot_status_t asym_w4a8_gemm(const int8_t* x8, const float* s_a, const uint8_t* idx, const uint8_t* s_rel,
                                const float* codebook, const float* s_channel, const uint16_t* bias, int M, int N,
                                int K, uint16_t* y, void* stream) {
  return gemm_cb_common(x8, s_a, idx, s_rel, codebook, s_channel, bias, M, N, K, y, GemmSink::kBF16, stream);
}

convrot_status_t asym_w4a8_gemm_f32(const int8_t* x8, const float* s_a, const uint8_t* idx, const uint8_t* s_rel,
                                    const float* codebook, const float* s_channel, const uint16_t* bias, int M,
                                    int N, int K, float* y32, void* stream) {
  return gemm_cb_common(x8, s_a, idx, s_rel, codebook, s_channel, bias, M, N, K, y32, GemmSink::kF32, stream);
}

convrot_status_t asym_w4a8_gemm_s32(const int8_t* x8, const uint8_t* idx, const uint8_t* s_rel,
                                    const float* codebook, int M, int N, int K, int32_t* acc, void* stream) {
  return gemm_cb_common(x8, nullptr, idx, s_rel, codebook, nullptr, nullptr, M, N, K, acc, GemmSink::kS32, stream);
}

convrot_status_t asym_w4a8_linear(const uint16_t* x, const uint8_t* idx, const uint8_t* s_rel, const float* codebook,
                                  const float* s_channel, const uint16_t* bias, int M, int N, int K, uint16_t* y,
                                  void* workspace, size_t workspace_bytes, void* stream) {
  return linear_cb_common(x, idx, s_rel, codebook, s_channel, bias, M, N, K, y, GemmSink::kBF16, workspace,
                          workspace_bytes, stream);
}

convrot_status_t asym_w4a8_linear_f32(const uint16_t* x, const uint8_t* idx, const uint8_t* s_rel,
                                      const float* codebook, const float* s_channel, const uint16_t* bias, int M,
                                      int N, int K, float* y32, void* workspace, size_t workspace_bytes,
                                      void* stream) {
  return linear_cb_common(x, idx, s_rel, codebook, s_channel, bias, M, N, K, y32, GemmSink::kF32, workspace,
                          workspace_bytes, stream);
}

}  // extern "C"
