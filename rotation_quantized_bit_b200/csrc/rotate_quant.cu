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
//
// Bit-exact contract.  The butterflies use the fixed stage order (stride 1,
// 4, 16, 64) and association (p=a+b, q=a-b, r=c+d, t=c-d -> p+t, p-t, q+r,
// r-q), every add is a correctly rounded fp32 add (packed f32x2 or scalar, no
// contraction), the 1/16 is one multiply, the scale is an IEEE division, and
// each code equals rint(fl(x' / s)) with ties to even, so codes and scales are
// identical bit for bit to any plain fp32 evaluation of that definition.
//
// Layout.  A lane owns one half (128 channels) of a 256-channel group and
// keeps it in registers as 64 fp32 pairs; pair i holds channels i and i + 64
// of the half, so the radix-4 stages on channel bits (0,1), (2,3), (4,5) are
// packed f32x2 butterflies, and the stage on bits (6,7) combines the two
// members of a pair and the two halves held by the lane pair (lane ^ 1), one
// shuffle per two channels.  Input is staged through shared memory: a warp
// copies its 8 KB tile (16 groups) with coalesced 16-byte cp.async into
// XOR-swizzled slots, so both the copy and each lane's 16 reads of its own
// 256 bytes are free of bank conflicts.  The next row block is prefetched
// while the current one is computed.  Codes leave through the same buffer
// and coalesced 16-byte stores.
//
// Quantization.  The code is rint(q) with q the correctly rounded quotient
// x' / s.  q is formed without a division by Markstein's correction (P.
// Markstein, "Computation of elementary functions on the IBM RISC System/6000
// processor", IBM J. Res. Develop. 34(1), 1990; restated as Markstein's
// theorem in Muller et al., "Handbook of Floating-Point Arithmetic", ch. on
// division with an FMA): with y = RN(1/s), q0 = RN(x' y) is within two ulps of
// x'/s; one step q1 = RN(q0 + RN(x' - s q0) y) makes it faithful, and a second
// step from a faithful q1, whose remainder x' - s q1 is exact, returns
// RN(x'/s) itself.  Both remainders are fused multiply-adds.  The theorem needs
// the remainders and products clear of underflow, which holds for every scale
// s >= 2^-100 wherever the code can be nonzero; rows with a smaller scale (zero
// included) take the IEEE division.  rint is the addition of 1.5 * 2^23, whose
// low byte is then the two's-complement code.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"

namespace convrot {

namespace {

typedef unsigned long long u64;

constexpr int kTileBytes = 8192;          // 16 groups x 256 bf16 per warp
constexpr int kMaxWarps = 8;              // at most 128 groups per row block
constexpr float kMagic = 12582912.0f;     // 1.5 * 2^23: x + kMagic rounds x to an integer, ties to even
constexpr float kMinScale = 7.88860905e-31f;           // 2^-100: below it, codes by division

// ---------------------------------------------------------------- helpers

__device__ __forceinline__ u64 f2(float lo, float hi) {
  u64 d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2_split(u64 v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ u64 f2_add(u64 a, u64 b) {
  u64 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 f2_sub(u64 a, u64 b) {
  u64 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 f2_mul(u64 a, u64 b) {
  u64 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ u64 f2_fma(u64 a, u64 b, u64 c) {
  u64 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// One radix-4 butterfly on packed pairs: (a,b,c,d) -> (p+t, p-t, q+r, r-q).
__device__ __forceinline__ void bfly4(u64& a, u64& b, u64& c, u64& d) {
  const u64 p = f2_add(a, b), q = f2_sub(a, b), r = f2_add(c, d), t = f2_sub(c, d);
  a = f2_add(p, t);
  b = f2_sub(p, t);
  c = f2_add(q, r);
  d = f2_sub(r, q);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(valid ? 16 : 0) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Byte 0 of four words -> one word (the code bytes of four rounded floats).
__device__ __forceinline__ uint32_t gather_b0(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  const uint32_t ab = __byte_perm(a, b, 0x0040);  // [a0, b0, .., ..]
  const uint32_t cd = __byte_perm(c, d, 0x0040);  // [c0, d0, .., ..]
  return __byte_perm(ab, cd, 0x5410);             // [a0, b0, c0, d0]
}

// Eight codes as bytes (natural order, two words) -> packed nibbles, even index low.
__device__ __forceinline__ uint32_t pack_nibbles(uint32_t lo4, uint32_t hi4) {
  const uint32_t a = lo4 & 0x0F0F0F0Fu, b = hi4 & 0x0F0F0F0Fu;
  const uint32_t a2 = a | (a >> 4), b2 = b | (b >> 4);  // bytes 0 and 2 hold two codes each
  return __byte_perm(a2, b2, 0x6420);
}

// Sixteen codes of two chunks (8 + 8, natural order) -> staging.  s8 layout:
// per chunk the operand order (0,2,4,6,1,3,5,7), 16 bytes per chunk pair in
// slot (pair ^ (region & 7)) of the lane's 128-byte region.  Packed layout: 4
// bytes per chunk, 8 bytes per chunk pair, at region * 64 + 8 * pair.
template <bool PACKED>
__device__ __forceinline__ void stage_chunk_pair(uint8_t* stage, int region, int pair, const uint32_t (&c)[16]) {
  if (PACKED) {
    const uint32_t w0 = pack_nibbles(gather_b0(c[0], c[1], c[2], c[3]), gather_b0(c[4], c[5], c[6], c[7]));
    const uint32_t w1 = pack_nibbles(gather_b0(c[8], c[9], c[10], c[11]), gather_b0(c[12], c[13], c[14], c[15]));
    *reinterpret_cast<uint2*>(stage + 64 * region + 8 * pair) = make_uint2(w0, w1);
  } else {
    uint4 o;
    o.x = gather_b0(c[0], c[2], c[4], c[6]);
    o.y = gather_b0(c[1], c[3], c[5], c[7]);
    o.z = gather_b0(c[8], c[10], c[12], c[14]);
    o.w = gather_b0(c[9], c[11], c[13], c[15]);
    *reinterpret_cast<uint4*>(stage + 128 * region + 16 * (pair ^ (region & 7))) = o;
  }
}

struct RQParams {
  const uint16_t* x;
  int M, K;
  int G;        // groups of 256 per row
  int R;        // rows per block
  int nblocks;  // ceil(M / R)
  RotateQuantOut out;
};

// Shared-memory slot of logical 16-byte chunk c = 16 * region + k of the input
// tile: k XOR the region's low three bits.
__device__ __forceinline__ int in_slot(int c) { return (c & ~15) | ((c & 15) ^ ((c >> 4) & 7)); }

template <bool PACKED>
__global__ void __launch_bounds__(kMaxWarps * 32, 1) rotate_quant_kernel(const __grid_constant__ RQParams p) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t row_amax[2][128];
  // Let the dependent GEMM launch now: it streams its weights meanwhile and
  // waits (griddepcontrol.wait) for this grid before reading codes or scales.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* const wbuf0 = smem + (2 * warp) * kTileBytes;
  uint8_t* const wbuf1 = smem + (2 * warp + 1) * kTileBytes;
  const int groups_per_block = p.R * p.G;
  const size_t row_bytes = static_cast<size_t>(p.K) * 2;
  const size_t total_bytes = static_cast<size_t>(p.M) * row_bytes;
  const uint8_t* xb = reinterpret_cast<const uint8_t*>(p.x);

  // Coalesced copy of this warp's tile of row block b into buffer `buf`.
  auto prefetch = [&](int b, int buf) {
    const size_t base = static_cast<size_t>(b) * p.R * row_bytes + static_cast<size_t>(warp) * kTileBytes;
    const size_t block_end = min(static_cast<size_t>(b + 1) * p.R * row_bytes, total_bytes);
    const uint32_t s0 = smem_addr(buf ? wbuf1 : wbuf0);
#pragma unroll
    for (int i = 0; i < kTileBytes / 512; ++i) {
      const int c = 32 * i + lane;
      const size_t g = base + 16 * static_cast<size_t>(c);
      const bool valid = g < block_end;
      cp_async16(s0 + 16 * in_slot(c), valid ? xb + g : xb, valid);
    }
    cp_async_commit();
  };

  for (int i = threadIdx.x; i < 2 * 128; i += blockDim.x) (&row_amax[0][0])[i] = 0u;
  __syncthreads();

  int it = 0;
  if (static_cast<int>(blockIdx.x) < p.nblocks) prefetch(blockIdx.x, 0);
  for (int b = blockIdx.x; b < p.nblocks; b += gridDim.x, ++it) {
    const int buf = it & 1;
    uint8_t* const tile = buf ? wbuf1 : wbuf0;
    uint32_t* const amax_slot = row_amax[it & 1];
    const int nb = b + gridDim.x;
    if (nb < p.nblocks) {
      prefetch(nb, buf ^ 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();

    // This lane's half-group.
    const int f = 16 * warp + (lane >> 1);  // group index within the block
    const int h = lane & 1;                 // which half of the group
    const bool active = f < groups_per_block;
    const int rloc = active ? f / p.G : 0;
    const int row = b * p.R + rloc;
    const bool live = active && row < p.M;

    // ---- 128 bf16 -> 64 fp32 pairs: pair i = (channel i, channel i + 64)
    u64 P[64];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint4 lo = *reinterpret_cast<const uint4*>(tile + 16 * ((lane << 4) | (k ^ (lane & 7))));
      const uint4 hi = *reinterpret_cast<const uint4*>(tile + 16 * ((lane << 4) | ((k + 8) ^ (lane & 7))));
      const uint32_t w0[4] = {lo.x, lo.y, lo.z, lo.w};
      const uint32_t w1[4] = {hi.x, hi.y, hi.z, hi.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        P[8 * k + 2 * e] = f2(__uint_as_float(w0[e] << 16), __uint_as_float(w1[e] << 16));
        P[8 * k + 2 * e + 1] = f2(__uint_as_float(w0[e] & 0xFFFF0000u), __uint_as_float(w1[e] & 0xFFFF0000u));
      }
    }
    __syncwarp();  // the tile buffer becomes the output staging area below

    // ---- rotation: stages on channel bits (0,1), (2,3), (4,5), packed
#pragma unroll
    for (int s = 0; s < 3; ++s) {
      const int st = 1 << (2 * s);
#pragma unroll
      for (int i = 0; i < 64; ++i)
        if (((i >> (2 * s)) & 3) == 0) bfly4(P[i], P[i + st], P[i + 2 * st], P[i + 3 * st]);
    }
    // stage on bits (6,7): bit 6 within the pair, bit 7 across the lane pair.
    // Lane h=0 holds (a, b), lane h=1 holds (c, d); u = own sum, w = own
    // difference; the partner's w completes (p+t, p-t) resp. (q+r, r-q).
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      float a, c;
      f2_split(P[i], a, c);
      const float u = __fadd_rn(a, c), w = __fsub_rn(a, c);
      const float r = __shfl_xor_sync(0xffffffffu, w, 1);
      P[i] = f2(__fadd_rn(u, r), __fsub_rn(u, r));
    }
    // x' = v * 1/16, and the lane's amax
    const u64 sixteenth = f2(0.0625f, 0.0625f);
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      P[i] = f2_mul(P[i], sixteenth);
      float a, c;
      f2_split(P[i], a, c);
      m = max3(m, fabsf(a), fabsf(c));
    }
    if (live) atomicMax(&amax_slot[rloc], __float_as_uint(m));
    __syncthreads();
    const float scale = __fdiv_rn(__uint_as_float(amax_slot[rloc]), 7.0f);
    // The other slot is free now (its last readers finished before this
    // barrier): clear it for the next block.
    if (static_cast<int>(threadIdx.x) < 128) row_amax[(it + 1) & 1][threadIdx.x] = 0u;

    // ---- quantize into the staging area (region `lane` of `tile`)
    if (scale >= kMinScale) {
      const float rcp = __frcp_rn(scale);
      const u64 rr = f2(rcp, rcp), ns = f2(-scale, -scale), mg = f2(kMagic, kMagic);
#pragma unroll
      for (int k = 0; k < 8; k += 2) {
        // pairs 8k .. 8k+15 hold chunks k, k+1 (.x) and k+8, k+9 (.y)
        uint32_t cx[16], cy[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const u64 x = P[8 * k + e];
          u64 q = f2_mul(x, rr);
          q = f2_fma(f2_fma(ns, q, x), rr, q);  // faithful
          q = f2_fma(f2_fma(ns, q, x), rr, q);  // RN(x / s)
          float tx, ty;
          f2_split(f2_add(q, mg), tx, ty);
          cx[e] = __float_as_uint(tx);
          cy[e] = __float_as_uint(ty);
        }
        stage_chunk_pair<PACKED>(tile, lane, k >> 1, cx);
        stage_chunk_pair<PACKED>(tile, lane, (k + 8) >> 1, cy);
      }
    } else {
      // Zero or tiny scale (a whole row takes this branch): IEEE division,
      // in a rolled loop over a local copy to keep the code small.
      float v[128];
#pragma unroll
      for (int i = 0; i < 64; ++i) f2_split(P[i], v[i], v[i + 64]);
#pragma unroll 1
      for (int k = 0; k < 16; ++k) {  // chunk k: channels 8k .. 8k+7 of the half
        uint32_t q[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int qq = scale != 0.0f ? __float2int_rn(__fdiv_rn(v[8 * k + e], scale)) : 0;
          q[e] = static_cast<uint32_t>(min(7, max(-8, qq)));
        }
        if (PACKED) {
          uint32_t w = 0;
#pragma unroll
          for (int e = 0; e < 8; ++e) w |= (q[e] & 0xFu) << (4 * e);
          *reinterpret_cast<uint32_t*>(tile + 64 * lane + 4 * k) = w;
        } else {
          const uint2 o = make_uint2(gather_b0(q[0], q[2], q[4], q[6]), gather_b0(q[1], q[3], q[5], q[7]));
          *reinterpret_cast<uint2*>(tile + 128 * lane + 16 * ((k >> 1) ^ (lane & 7)) + 8 * (k & 1)) = o;
        }
      }
    }
    if (live && h == 0 && f % p.G == 0) p.out.scale[row] = scale;
    __syncwarp();

    // ---- coalesced copy-out of the warp's codes (16 groups x 256 codes)
    {
      constexpr int kOutTile = kTileBytes / (PACKED ? 4 : 2);  // 2 KB packed, 4 KB as bytes
      const size_t code_row = PACKED ? static_cast<size_t>(p.K) / 2 : static_cast<size_t>(p.K);
      const size_t block_end = min(static_cast<size_t>(b + 1) * p.R * code_row, static_cast<size_t>(p.M) * code_row);
      const size_t base = static_cast<size_t>(b) * p.R * code_row + static_cast<size_t>(warp) * kOutTile;
      uint8_t* dst = PACKED ? p.out.packed : reinterpret_cast<uint8_t*>(p.out.s8);
#pragma unroll
      for (int i = 0; i < kOutTile / 512; ++i) {
        const int c = 32 * i + lane;
        uint4 v;
        if (PACKED) {
          v = *reinterpret_cast<const uint4*>(tile + 16 * c);
        } else {
          const int region = c >> 3, k = c & 7;
          v = *reinterpret_cast<const uint4*>(tile + 128 * region + 16 * (k ^ (region & 7)));
        }
        const size_t g = base + 16 * static_cast<size_t>(c);
        if (g < block_end) *reinterpret_cast<uint4*>(dst + g) = v;
      }
    }
    __syncwarp();
  }
}

// Packed nibbles -> operand bytes.  A 32-bit word holds codes k..k+7 (even
// index in the low nibble); its low nibbles are codes (0,2,4,6) and its high
// nibbles (1,3,5,7).  u = nibble ^ 8 = q + 8 in [0, 15]; the signed byte is
// (u + 0x78) ^ 0x80 = u - 8 (mod 256), with no carry between bytes.
__global__ void __launch_bounds__(256) unpack_codes_kernel(const uint8_t* __restrict__ packed, int M, int K,
                                                           int8_t* __restrict__ s8) {
  const int lane = threadIdx.x & 31;
  const int warps_per_block = blockDim.x / 32;
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

cudaError_t launch_rotate_quant(const uint16_t* x, int M, int K, RotateQuantOut out, cudaStream_t stream) {
  RQParams p{};
  p.x = x;
  p.M = M;
  p.K = K;
  p.G = K / 256;
  // Rows per block R: a block holds R*G half-group pairs (at most 128 groups,
  // 8 warps).  Pick the R with the fewest waves of blocks over the SMs and,
  // among those, the fewest warps on the busiest SM.
  const int sms = num_sms_cached();
  const bool packed_out = out.packed != nullptr;
  const void* kfn_sel = packed_out ? reinterpret_cast<const void*>(rotate_quant_kernel<true>)
                                   : reinterpret_cast<const void*>(rotate_quant_kernel<false>);
  static int regs_cache[2][64] = {{0}};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  int& regs = regs_cache[packed_out ? 1 : 0][dev];
  if (regs == 0) {
    cudaFuncAttributes fa;
    regs = (cudaFuncGetAttributes(&fa, kfn_sel) == cudaSuccess && fa.numRegs > 0) ? fa.numRegs : 255;
  }
  const int warp_regs = ((regs * 32 + 255) / 256) * 256;
  int best_R = 1;
  long best_key = -1;
  for (int R = 1; R <= 128 / p.G; ++R) {
    const int nb = (M + R - 1) / R;
    const int w = (R * p.G + 15) / 16;
    int per_sm = 65536 / (warp_regs * w);
    per_sm = min(per_sm, (228 * 1024) / (w * 2 * kTileBytes + 2048));
    per_sm = min(per_sm, 64 / w);
    if (per_sm < 1) continue;
    const long slots = static_cast<long>(sms) * per_sm;
    const long waves = (nb + slots - 1) / slots;
    const long busiest = static_cast<long>((nb + sms - 1) / sms) * w;  // warps on the busiest SM per wave
    const long key = waves * 100000 + (waves > 1 ? 0 : busiest);
    if (best_key < 0 || key < best_key || (key == best_key && R > best_R)) {
      best_key = key;
      best_R = R;
    }
    if (R > M) break;
  }
  const int R = best_R;
  p.R = R;
  p.nblocks = (M + R - 1) / R;
  p.out = out;
  const int warps = (R * p.G + 15) / 16;
  const int smem = warps * 2 * kTileBytes;
  const bool packed = out.packed != nullptr;
  const void* kfn = packed ? reinterpret_cast<const void*>(rotate_quant_kernel<true>)
                           : reinterpret_cast<const void*>(rotate_quant_kernel<false>);
  static int cache_packed[64] = {0}, cache_s8[64] = {0};
  cudaError_t e = ensure_dynamic_smem(kfn, smem, packed ? cache_packed : cache_s8);
  if (e != cudaSuccess) return note_cuda(e, "rotate_quant: dynamic shared memory attribute");
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kfn, warps * 32, smem);
  if (e != cudaSuccess) return note_cuda(e, "rotate_quant: occupancy query");
  if (per_sm < 1) per_sm = 1;
  int grid = sms * per_sm;
  if (grid > p.nblocks) grid = p.nblocks;
  if (packed)
    rotate_quant_kernel<true><<<grid, warps * 32, smem, stream>>>(p);
  else
    rotate_quant_kernel<false><<<grid, warps * 32, smem, stream>>>(p);
  count_dispatch(0);
  return note_cuda(cudaGetLastError(), "rotate_quant: launch");
}

cudaError_t launch_unpack_codes(const uint8_t* packed, int M, int K, int8_t* s8, cudaStream_t stream) {
  const int per_block = 8;
  int grid = (M + per_block - 1) / per_block;
  if (grid > num_sms_cached() * 8) grid = num_sms_cached() * 8;
  unpack_codes_kernel<<<grid, 256, 0, stream>>>(packed, M, K, s8);
  count_dispatch(1);
  return note_cuda(cudaGetLastError(), "unpack_codes: launch");
}

}  // namespace convrot
