// peak.cu -- measurement of the int8 tensor-core rate of this GPU: one CTA
// per SM, one thread issuing back-to-back tcgen05.mma.kind::i8 (128 x N x 32,
// s8 x s8 -> s32) on operands that stay on chip (shared memory, and tensor
// memory for the A-from-tensor-memory form the W4A4 GEMM uses).  Nothing is
// read from or written to global memory except the per-CTA cycle counts, so
// the result is the dense int8 MMA rate the GEMM kernels are measured
// against, and, at small N, the fixed cost of one MMA instruction.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../../include/convrot.h"
#include "kernels.cuh"
#include "ptx.cuh"

namespace convrot {
namespace {

constexpr int kPeakMaxGrid = 256;
__device__ unsigned long long g_peak_cycles[kPeakMaxGrid];

__device__ __forceinline__ void umma_i8_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, 1, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc)
      : "memory");
}

// Shared memory: A tile 128 rows x 128 bytes (16 KB), B tile N rows x 128
// bytes (<= 32 KB), both in the 128-byte-swizzle K-major layout (contents are
// zero; the values do not change the rate).
__global__ void __launch_bounds__(128, 1) mma_i8_rate_kernel(int N, int iters, int a_in_tmem) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar;
  __shared__ uint32_t tbase;
  const int warp = threadIdx.x >> 5;
  for (int i = threadIdx.x; i < (16384 + 32768) / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0, 0, 0, 0);
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    tmem_alloc(&tbase, 512u);
    tmem_relinquish();
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // zeroed smem visible to the tensor core
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tbase;
  if (threadIdx.x == 0) {
    const uint32_t idesc = umma_idesc_i8(128, N, true, true);
    const uint64_t ad = umma_desc_k_sw128(smem_u32(smem));
    const uint64_t bd = umma_desc_k_sw128(smem_u32(smem + 16384));
    const uint32_t a_t = tmem + 256u;  // A in tensor memory: 8 columns per K = 32
    const unsigned long long t0 = clock64();
    if (a_in_tmem) {
      for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) umma_i8_ts(tmem, a_t + 8u * (kk & 3), bd + 2 * (kk & 3), idesc, 1u);
      }
    } else {
      for (int i = 0; i < iters; ++i) {
#pragma unroll
        for (int kk = 0; kk < 16; ++kk) umma_i8_ss(tmem, ad + 2 * (kk & 3), bd + 2 * (kk & 3), idesc);
      }
    }
    umma_commit(&bar);
    const bool ok = mbar_wait(&bar, 0);
    const unsigned long long t1 = clock64();
    if (blockIdx.x < kPeakMaxGrid) g_peak_cycles[blockIdx.x] = ok ? t1 - t0 : 0ull;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512u);
  }
}

}  // namespace
}  // namespace convrot

using namespace convrot;

extern "C" convrot_status_t convrot_measure_mma_i8(int N, int a_in_tmem, int iters, double* tops,
                                                   double* cycles_per_mma) {
  if (!tops || !cycles_per_mma) return CONVROT_ERR_NULL;
  if (N < 16 || N > 256 || N % 16 != 0 || iters < 1 || iters > (1 << 20)) return CONVROT_ERR_SHAPE;
  int dev = 0, sms = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || major != 10)
    return CONVROT_ERR_DEVICE;
  const int grid = sms < kPeakMaxGrid ? sms : kPeakMaxGrid;
  const int smem = 1024 + 16384 + 32768;
  static std::atomic<int> cache[64];
  if (ensure_dynamic_smem(reinterpret_cast<const void*>(mma_i8_rate_kernel), smem, cache) != cudaSuccess)
    return CONVROT_ERR_CUDA;
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return CONVROT_ERR_CUDA;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return CONVROT_ERR_CUDA;
  }
  cudaError_t e = cudaSuccess;
  float ms = 0.0f;
  // One untimed launch (clocks ramp, code loads), then the timed one.
  for (int rep = 0; rep < 2 && e == cudaSuccess; ++rep) {
    cudaEventRecord(e0, 0);
    mma_i8_rate_kernel<<<grid, 128, smem, 0>>>(N, iters, a_in_tmem);
    e = cudaGetLastError();
    cudaEventRecord(e1, 0);
    if (e == cudaSuccess) e = cudaEventSynchronize(e1);
  }
  if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, e0, e1);
  unsigned long long cyc[kPeakMaxGrid] = {0};
  if (e == cudaSuccess) e = cudaMemcpyFromSymbol(cyc, g_peak_cycles, sizeof(unsigned long long) * grid);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (e != cudaSuccess) {
    note_cuda(e, "convrot_measure_mma_i8");
    return CONVROT_ERR_CUDA;
  }
  double mean = 0.0;
  for (int i = 0; i < grid; ++i) mean += static_cast<double>(cyc[i]);
  mean /= grid;
  const double mmas = 16.0 * iters;
  *cycles_per_mma = mean / mmas;
  *tops = 2.0 * 128.0 * N * 32.0 * mmas * grid / (ms * 1e-3) / 1e12;
  return CONVROT_OK;
}
