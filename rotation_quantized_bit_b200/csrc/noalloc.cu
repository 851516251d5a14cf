// noalloc.cu -- the fused ConvRot W4A4 Linear for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand this library a workspace: code that runs
// inside a host framework which owns every device allocation and forbids
// side allocations, fixed-budget deployments that must not grow their
// footprint after start-up, and plugin or foreign-language callers that have
// no binding to a CUDA allocator.  For them convrot_w4a4_linear_noalloc runs
// the same two kernels as convrot_w4a4_linear, but keeps the activation codes
// and per-token scales in a scratch array that is part of the library image
// itself: a file-scope __device__ array of kNoAllocScratchBytes, which every
// GPU that loads the library holds until the process exits.
//
// Host code may not take the array's name as a device pointer (on the host it
// is only a stand-in symbol), so the array's device address is looked up with
// cudaGetSymbolAddress, with the device current, the first time a device (in
// a given CUDA context) calls in, and kept for later calls.  The lookup is
// repeated when the current context changes (after cudaDeviceReset, or with
// another driver context current on the same device), since the array then
// lives at another address.  A mutex guards the cache, so concurrent first
// calls from several host threads are safe; the kernels of calls that
// overlap on the GPU still share, and race on, the one array.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>
#include <mutex>

#include "../../include/convrot.h"
#include "kernels.cuh"

namespace convrot {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchSlot {
  CUcontext ctx = nullptr;  // the context the address was looked up in
  void* ptr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];
std::mutex g_scratch_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);

CtxGetCurrentFn ctx_get_current() {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<CtxGetCurrentFn>(nullptr);
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  return fn;
}

// The scratch array's device address on the current device (and context), or
// null with *st set.
void* scratch_address(convrot_status_t* st) {
  int dev = 0, major = 0, minor = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess || major != 10 ||
      minor != 0) {
    *st = CONVROT_ERR_DEVICE;  // checked before the library's image is touched on this device
    return nullptr;
  }
  CUcontext ctx = nullptr;
  CtxGetCurrentFn get = ctx_get_current();
  if (get) (void)get(&ctx);
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchSlot& slot = g_scratch[dev];
  if (slot.ptr == nullptr || slot.ctx != ctx) {
    // Set-up, once per device and context, with that device current.
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      note_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "convrot_w4a4_linear_noalloc: cudaGetSymbolAddress");
      *st = CONVROT_ERR_CUDA;
      return nullptr;
    }
    if (get) (void)get(&ctx);  // the runtime's primary context, now that it is surely initialised
    slot.ctx = ctx;
    slot.ptr = p;
  }
  return slot.ptr;
}

}  // namespace
}  // namespace convrot

using namespace convrot;

extern "C" convrot_status_t convrot_w4a4_linear_noalloc(const uint16_t* x, const uint8_t* Wq, const float* s_w,
                                                        const uint16_t* bias, int M, int N, int K, uint16_t* y,
                                                        void* stream) {
  // Same argument rules as convrot_w4a4_linear; the workspace is replaced by
  // the library's static scratch array, so it is checked against that limit.
  if (!x || !Wq || !s_w || !y) return CONVROT_ERR_NULL;
  const size_t need = convrot_w4a4_workspace_size(M, N, K);
  if (need == 0 || N < 1 || N % 8 != 0) return CONVROT_ERR_SHAPE;
  if (need > kNoAllocScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof(msg), "convrot_w4a4_linear_noalloc: the shape needs %zu bytes of scratch, above the %zu-byte limit",
             need, kNoAllocScratchBytes);
    note_cuda(cudaErrorInvalidValue, msg);
    return CONVROT_ERR_WORKSPACE;
  }
  convrot_status_t st = CONVROT_OK;
  void* scratch = scratch_address(&st);
  if (!scratch) return st;
  // Nothing in the scratch needs to start at zero: the first kernel writes
  // every code and scale that the second one reads, and the small-M GEMM
  // clears the counters it uses itself.
  return convrot_w4a4_linear(x, Wq, s_w, bias, M, N, K, y, scratch, kNoAllocScratchBytes, stream);
}
