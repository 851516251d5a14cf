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
// is only a stand-in symbol), so the first call on each device looks its
// device address up with cudaGetSymbolAddress and caches it.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdio>

#include "../../include/convrot.h"
#include "kernels.cuh"

namespace convrot {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;  // 32 MiB per device
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device, looked up on first use.
void* g_scratch_ptr[kMaxDevices] = {nullptr};

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
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return CONVROT_ERR_DEVICE;
  if (g_scratch_ptr[dev] == nullptr) {
    // Set-up, once per device, with that device current.
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      note_cuda(e != cudaSuccess ? e : cudaErrorInvalidSymbol, "convrot_w4a4_linear_noalloc: cudaGetSymbolAddress");
      return CONVROT_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  // Nothing in the scratch needs to start at zero: the first kernel writes
  // every code and scale that the second one reads.
  return convrot_w4a4_linear(x, Wq, s_w, bias, M, N, K, y, g_scratch_ptr[dev], kNoAllocScratchBytes, stream);
}
