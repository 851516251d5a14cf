// rotate_quant.cu -- the ConvRot activation / weight prologue on sm_100a.
//
// Per row of a bf16 matrix [rows, K] (activations per token, or weights per
// output channel):
//   1. widen bf16 -> fp32 (exact),
//   2. rotate every 256-channel group with the regular Hadamard H4^(x4) / 16
//      ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot...)", intro:
//      group-256 regular-Hadamard rotation, activations rotated online),
//   3. s = amax / 7 over the row (dynamic per-token INT4, same paragraph),
//   4. q = clamp(rint(x' / s), -8, 7) and write the codes.
// Bit-exact contract: the butterflies use the fixed stage order (stride 1, 4,
// 16, 64) and association (p=a+b, q=a-b, r=c+d, t=c-d -> p+t, p-t, q+r, r-q)
// with explicitly rounded adds (no contraction), the 1/16 is one multiply,
// the quotient is a correctly rounded IEEE division and rint is round half to
// even -- the same operations in the same order as any plain fp32 evaluation
// of the definition, so the codes and scales are identical bit for bit.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace convrot {

namespace {

constexpr int kThreads = 256;

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// One block rotates and quantizes one row at a time, holding the row in
// shared memory as fp32.
__global__ void __launch_bounds__(kThreads) rotate_quant_kernel(const uint16_t* __restrict__ x, int M, int K,
                                                                RotateQuantOut out) {
  extern __shared__ float row[];  // K floats
  __shared__ float red_f[kThreads / 32];
  const int tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int nchunk = K >> 3;  // 8-element chunks
  const int nbfly = K >> 2;   // radix-4 butterflies per stage

  for (int m = blockIdx.x; m < M; m += gridDim.x) {
    const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(m) * K);
    for (int c = tid; c < nchunk; c += kThreads) {
      uint4 v = __ldg(src + c);
      float* d = row + 8 * c;
      d[0] = bf16_lo(v.x); d[1] = bf16_hi(v.x);
      d[2] = bf16_lo(v.y); d[3] = bf16_hi(v.y);
      d[4] = bf16_lo(v.z); d[5] = bf16_hi(v.z);
      d[6] = bf16_lo(v.w); d[7] = bf16_hi(v.w);
    }
    // Four radix-4 stages; stage s pairs indices that differ only in base-4
    // digit s (stride 4^s).
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      __syncthreads();
      const int st = 1 << (2 * s);
      for (int b = tid; b < nbfly; b += kThreads) {
        const int g = b >> 6, li = b & 63;
        const int low = li & (st - 1);
        const int high = li >> (2 * s);
        const int i = g * 256 + ((high << (2 * s + 2)) | low);
        const float a = row[i], bb = row[i + st], c = row[i + 2 * st], d = row[i + 3 * st];
        const float p = __fadd_rn(a, bb), q = __fsub_rn(a, bb), r = __fadd_rn(c, d), t = __fsub_rn(c, d);
        row[i] = __fadd_rn(p, t);
        row[i + st] = __fsub_rn(p, t);
        row[i + 2 * st] = __fadd_rn(q, r);
        row[i + 3 * st] = __fsub_rn(r, q);
      }
    }
    __syncthreads();
    float amax = 0.0f;
    for (int k = tid; k < K; k += kThreads) {
      const float v = __fmul_rn(row[k], 0.0625f);
      row[k] = v;
      amax = fmaxf(amax, fabsf(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if (lane == 0) red_f[warp] = amax;
    __syncthreads();
    if (tid < 32) {
      float v = tid < kThreads / 32 ? red_f[tid] : 0.0f;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
      if (tid == 0) red_f[0] = v;
    }
    __syncthreads();
    const float scale = __fdiv_rn(red_f[0], 7.0f);
    if (tid == 0) out.scale[m] = scale;

    for (int c = tid; c < nchunk; c += kThreads) {
      int q[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        int v = 0;
        if (scale != 0.0f) {
          v = __float2int_rn(__fdiv_rn(row[8 * c + j], scale));
          v = min(7, max(-8, v));
        }
        q[j] = v;
      }
      if (out.packed) {
        uint32_t w = 0;
#pragma unroll
        for (int j = 0; j < 8; ++j) w |= (static_cast<uint32_t>(q[j]) & 0xFu) << (4 * j);
        reinterpret_cast<uint32_t*>(out.packed + static_cast<size_t>(m) * (K >> 1))[c] = w;
      }
      if (out.s8) {
        uint2 w;
        w.x = (static_cast<uint32_t>(q[0]) & 0xFFu) | ((static_cast<uint32_t>(q[2]) & 0xFFu) << 8) |
              ((static_cast<uint32_t>(q[4]) & 0xFFu) << 16) | ((static_cast<uint32_t>(q[6]) & 0xFFu) << 24);
        w.y = (static_cast<uint32_t>(q[1]) & 0xFFu) | ((static_cast<uint32_t>(q[3]) & 0xFFu) << 8) |
              ((static_cast<uint32_t>(q[5]) & 0xFFu) << 16) | ((static_cast<uint32_t>(q[7]) & 0xFFu) << 24);
        reinterpret_cast<uint2*>(out.s8 + static_cast<size_t>(m) * K)[c] = w;
      }
    }
    __syncthreads();
  }
}

// Packed nibbles -> operand bytes.  A 32-bit word holds codes k..k+7 (even
// index in the low nibble); its low nibbles are codes (0,2,4,6) and its high
// nibbles (1,3,5,7).  u = nibble ^ 8 = q + 8 in [0, 15]; the signed byte is
// (u + 0x78) ^ 0x80 = u - 8 (mod 256), with no carry between bytes.
__global__ void __launch_bounds__(kThreads) unpack_codes_kernel(const uint8_t* __restrict__ packed, int M, int K,
                                                                int8_t* __restrict__ s8) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = kThreads / 32;
  const int nword = K >> 3;
  for (int m = blockIdx.x * warps_per_block + (threadIdx.x >> 5); m < M; m += gridDim.x * warps_per_block) {
    const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + static_cast<size_t>(m) * (K >> 1));
    uint2* dst = reinterpret_cast<uint2*>(s8 + static_cast<size_t>(m) * K);
    for (int i = lane; i < nword; i += 32) {
      const uint32_t w = __ldg(src + i);
      const uint32_t ulo = (w & 0x0F0F0F0Fu) ^ 0x08080808u;
      const uint32_t uhi = ((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u;
      dst[i] = make_uint2((ulo + 0x78787878u) ^ 0x80808080u, (uhi + 0x78787878u) ^ 0x80808080u);
    }
  }
}

int num_sms_cached() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace

cudaError_t launch_rotate_quant(const uint16_t* x, int M, int K, RotateQuantOut out, cudaStream_t stream) {
  const int smem = K * static_cast<int>(sizeof(float));
  static int cache[64] = {0};
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(rotate_quant_kernel), smem, cache);
  if (e != cudaSuccess) return note_cuda(e, "rotate_quant: dynamic shared memory attribute");
  int grid = num_sms_cached() * 4;
  if (grid > M) grid = M;
  rotate_quant_kernel<<<grid, kThreads, smem, stream>>>(x, M, K, out);
  count_dispatch(0);
  return note_cuda(cudaGetLastError(), "rotate_quant: launch");
}

cudaError_t launch_unpack_codes(const uint8_t* packed, int M, int K, int8_t* s8, cudaStream_t stream) {
  const int per_block = kThreads / 32;
  int grid = (M + per_block - 1) / per_block;
  if (grid > num_sms_cached() * 8) grid = num_sms_cached() * 8;
  unpack_codes_kernel<<<grid, kThreads, 0, stream>>>(packed, M, K, s8);
  count_dispatch(1);
  return note_cuda(cudaGetLastError(), "unpack_codes: launch");
}

}  // namespace convrot
