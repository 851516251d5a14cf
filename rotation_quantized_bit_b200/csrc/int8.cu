// int8.cu -- the int8_tensorwise quantizer (no rotation, one scale for the
// whole tensor).
//
// The pages store their quality-sensitive layers in this stock format next
// to the W4A4 layers ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4
// (+ConvRot, mixed int8 fallback)", intro: the attention value/output
// projections and adaLN modulation Linears are stock int8_tensorwise).  Read
// as: s = amax|x| / 127 over the whole tensor (IEEE division), q =
// clamp(rint(x / s), -127, 127) with the correctly rounded quotient and
// round half to even; s = 0 gives q = 0.  Used for the dynamic activation
// scale and, offline, for the weights.
//
// Two passes over x: a max-reduction of |x| (bf16 bit patterns with the sign
// cleared compare like the magnitudes), then the quantization.  The quotient
// is formed with Markstein's correction exactly as in the rotate/quant
// prologue (see rotate_quant.cu): RN(x / s) from y = RN(1/s) and two FMA
// steps, valid for s >= 2^-100; smaller scales take the IEEE division.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace convrot {
namespace {

constexpr float kMagic8 = 12582912.0f;         // 1.5 * 2^23
constexpr float kMinScale8 = 7.88860905e-31f;  // 2^-100

// Largest |x| of 8 bf16 values in a 16-byte chunk, as bf16 bits.
__device__ __forceinline__ uint32_t chunk_absmax(uint4 v) {
  const uint32_t w[4] = {v.x & 0x7FFF7FFFu, v.y & 0x7FFF7FFFu, v.z & 0x7FFF7FFFu, v.w & 0x7FFF7FFFu};
  uint32_t m = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) m = max(m, max(w[i] & 0xFFFFu, w[i] >> 16));
  return m;
}

__global__ void __launch_bounds__(256) absmax_bf16_kernel(const uint4* __restrict__ x, size_t n16,
                                                          uint32_t* __restrict__ amax_bits) {
  __shared__ uint32_t wmax[8];
  uint32_t m = 0;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x)
    m = max(m, chunk_absmax(__ldg(x + i)));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int i = 1; i < static_cast<int>(blockDim.x >> 5); ++i) m = max(m, wmax[i]);
    atomicMax(amax_bits, m << 16);  // as fp32 bits: the bf16 value widened
  }
}

__global__ void __launch_bounds__(256) quant8_tensor_kernel(const uint4* __restrict__ x, size_t n16,
                                                            const uint32_t* __restrict__ amax_bits,
                                                            uint2* __restrict__ codes, float* __restrict__ scale_out,
                                                            int early_trigger) {
  // Let a dependent GEMM launch now: it streams its weights meanwhile.  Not
  // when this grid writes weights (the GEMMs read weights before they wait
  // for their predecessor).
  if (early_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const float s = __fdiv_rn(__uint_as_float(*amax_bits), 127.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) *scale_out = s;
  const float rcp = s >= kMinScale8 ? __frcp_rn(s) : 0.0f, ns = -s;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const uint4 v = __ldg(x + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float a[2] = {__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)};
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float xv = a[h];
        if (s >= kMinScale8) {
          float q = __fmul_rn(xv, rcp);
          q = __fmaf_rn(__fmaf_rn(ns, q, xv), rcp, q);  // faithful
          q = __fmaf_rn(__fmaf_rn(ns, q, xv), rcp, q);  // RN(x / s)
          c[2 * e + h] = __float_as_uint(__fadd_rn(q, kMagic8)) & 0xFFu;  // rint, two's complement byte
        } else {
          const int qq = s != 0.0f ? __float2int_rn(__fdiv_rn(xv, s)) : 0;
          c[2 * e + h] = static_cast<uint32_t>(min(127, max(-127, qq))) & 0xFFu;
        }
      }
    }
    codes[i] = make_uint2(c[0] | (c[1] << 8) | (c[2] << 16) | (c[3] << 24), c[4] | (c[5] << 8) | (c[6] << 16) | (c[7] << 24));
  }
}

int sm_count() {
  static int n[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (n[dev] == 0) {
    cudaDeviceGetAttribute(&n[dev], cudaDevAttrMultiProcessorCount, dev);
    if (n[dev] <= 0) n[dev] = 148;
  }
  return n[dev];
}

}  // namespace

cudaError_t launch_quant8_tensorwise(const uint16_t* x, size_t n, int8_t* codes, float* scale, uint32_t* scratch,
                                     cudaStream_t stream, bool early_trigger) {
  const size_t n16 = n / 8;  // n is a multiple of 256
  cudaError_t e = cudaMemsetAsync(scratch, 0, sizeof(uint32_t), stream);
  if (e != cudaSuccess) return note_cuda(e, "int8_tensorwise: clear amax");
  size_t want = (n16 + 255) / 256;
  const size_t cap = static_cast<size_t>(sm_count()) * 8;
  const unsigned grid = static_cast<unsigned>(want < 1 ? 1 : (want > cap ? cap : want));
  absmax_bf16_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), n16, scratch);
  e = cudaGetLastError();
  if (e != cudaSuccess) return note_cuda(e, "int8_tensorwise: amax launch");
  quant8_tensor_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(x), n16, scratch,
                                                  reinterpret_cast<uint2*>(codes), scale, early_trigger ? 1 : 0);
  return note_cuda(cudaGetLastError(), "int8_tensorwise: quantize launch");
}

}  // namespace convrot
