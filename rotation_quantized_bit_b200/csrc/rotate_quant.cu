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
// r-q) with correctly rounded fp32 adds (no contraction).  The results equal
// those of the plain fp32 evaluation x' = fl(v / 16), s = fl(amax / 7) and
// code = rint(fl(x' / s)) with ties to even, so codes and scales are
// identical bit for bit to any such evaluation of the definition; the
// Scales and Quantization paragraphs below say how they are reached without
// a division per element.
//
// Layout.  A 256-channel group is one task of 16 lanes (half a warp); each
// lane holds 16 channels of each of two tasks (two groups, from the same row
// or not) as fp32 pairs (task 0, task 1), so that every operation of the path
// is one packed f32x2 instruction for both tasks.  Channel index bits 0-3
// are first the register index and bits 4-7 the lane (lane l holds channels
// 16 l .. 16 l + 15), so the stages on bits (0,1) and (2,3) run in registers.
// A transpose of the pairs through the half-warp's shared-memory tile then
// swaps the roles (lane l holds channels l, 16 + l, ..., 240 + l) and the
// stages on bits (4,5) and (6,7) run in registers as well.  The tile's rows
// are 16 pairs (128 bytes) padded to 144 bytes, so the eight 16-byte stores
// of a lane (a row) and its sixteen 8-byte loads (a column) are free of bank
// conflicts and every address is a per-lane base plus a constant.  A block owns blocks of R whole rows (R * G tasks, G = K
// / 256) in turn, so the per-row amax is a shuffle reduction within each
// task plus one shared-memory atomic max per task.  Each lane then quantizes
// its channels; the code bytes go back to row order through the same tile
// (byte stores at their final positions, one 16-byte load per task) and
// leave with coalesced stores.
//
// Input staging.  The blocks are persistent: one thread keeps a ring of S
// row blocks in flight with 1-D bulk copies (the TMA engine, one contiguous
// copy of R * K bf16 per row block, completion on an mbarrier), so HBM reads
// run ahead of the arithmetic without holding registers.  A stage is
// refilled right after the block barrier that ends its readers' use of it.
//
// Scales.  The butterflies leave v = 2^LOG4G x'; the amax is taken over |v|
// and scaled once per row (RN is monotone, so RN(max|v| 2^-LOG4G) is the
// amax of x' itself).  Every lane forms its two rows' scales
// s = RN(amax / qmax) with two Markstein corrections of RN(amax fl(1/qmax))
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Develop. 34(1), 1990; restated as
// Markstein's theorem in Muller et al., "Handbook of Floating-Point
// Arithmetic", ch. on division with an FMA), which equals the IEEE quotient
// for every amax in [2^-120, 2^120] and qmax 7 or 127 (checked against
// division for each float of that range); other amax values take the IEEE
// division.
//
// Quantization.  The code is c = rint(RN(x'/s)) (ties to even).  Fast path,
// for 2^-100 <= s <= 2^100: k = rint(v y) with y ~ 1/(2^LOG4G s) from the
// approximate reciprocal (one fused multiply-add with 1.5 * 2^23, whose low
// byte is then k in two's complement), and the exact remainder
// d = RN(v - 2^LOG4G s k) from a second one.  If |d| <= 2^LOG4G s (1/2 - m),
// the quotient x'/s lies strictly inside (k - 1/2 + m', k + 1/2 - m') with m'
// above half an ulp of any quotient of magnitude <= qmax (m = 2^-18 for the
// 4-bit codes, 2^-14 for the 8-bit ones), so RN(x'/s) rounds to k as well, and
// c = k; the reciprocal's error only decides how often the check fails.  A
// lane whose check fails anywhere (a quotient within m of a half-integer:
// about one element in 10^5 on random data, every one of an exact tie)
// recomputes its codes by the exact quotient: y = RN(1/s), q0 = RN(x' y)
// within two ulps of x'/s, one correction q1 = RN(q0 + RN(x' - s q0) y) makes
// it faithful, and a second step from a faithful q1, whose remainder is exact,
// returns RN(x'/s) itself (Markstein's theorem again; it needs s >= 2^-100).
// Scales outside [2^-100, 2^100] (zero included) take the IEEE division.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace convrot {

namespace {

constexpr float kMagic = 12582912.0f;           // 1.5 * 2^23: x + kMagic rounds x to an integer, ties to even
constexpr float kMinScale = 0x1p-100f;          // fast and exact-quotient paths: 2^-100 <= s <= 2^100
constexpr float kMaxScale = 0x1p100f;
constexpr int kTileRow = 144;                   // bytes per transpose-tile row: 16 fp32 pairs + 16 of padding
constexpr int kTileBytes = 16 * kTileRow;       // per-half-warp transpose tile
constexpr int kMaxRows = 64;                    // rows per row block (K = 256 -> 64 tasks)
constexpr int kMaxThreads = 1024;

typedef unsigned long long u64;

// Packed fp32 pairs: f2(lo, hi), and correctly rounded f32x2 arithmetic (no
// contraction).
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

// Approximate reciprocal (the hardware's, about one ulp).
__device__ __forceinline__ float rcp_approx(float a) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(a));
  return r;
}

// RN(a / QMAX) for QMAX = 7 or 127: two Markstein corrections of RN(a y),
// y = RN(1 / QMAX), for a in [2^-120, 2^120] (equal to the IEEE quotient for
// every float of that range), the IEEE division elsewhere.
template <int QMAX>
__device__ __forceinline__ float div_by_qmax(float a) {
  constexpr float kQ = static_cast<float>(QMAX);
  constexpr float kY = 1.0f / kQ;
  if (a >= 0x1p-120f && a <= 0x1p120f) {
    float q = __fmul_rn(a, kY);
    q = __fmaf_rn(__fmaf_rn(-kQ, q, a), kY, q);
    q = __fmaf_rn(__fmaf_rn(-kQ, q, a), kY, q);
    return q;
  }
  return __fdiv_rn(a, kQ);
}

// One radix-4 butterfly on pairs: (a,b,c,d) -> (p+t, p-t, q+r, r-q).
__device__ __forceinline__ void bfly4(u64& a, u64& b, u64& c, u64& d) {
  const u64 p = f2_add(a, b), q = f2_sub(a, b), r = f2_add(c, d), t = f2_sub(c, d);
  a = f2_add(p, t);
  b = f2_sub(p, t);
  c = f2_add(q, r);
  d = f2_sub(r, q);
}

// Eight codes as bytes (natural order, two words) -> packed nibbles, even index low.
__device__ __forceinline__ uint32_t pack_nibbles(uint32_t lo4, uint32_t hi4) {
  const uint32_t a = lo4 & 0x0F0F0F0Fu, b = hi4 & 0x0F0F0F0Fu;
  const uint32_t a2 = a | (a >> 4), b2 = b | (b >> 4);  // bytes 0 and 2 hold two codes each
  return __byte_perm(a2, b2, 0x6420);
}

struct RQParams {
  const uint16_t* x;
  int M, K;
  int G;        // groups of 256 per row
  int R;        // rows per row block
  int nblocks;  // ceil(M / R)
  int S;        // stages of the input ring
  RotateQuantOut out;
};

// Output formats of the prologue:
//   kPacked4  4-bit codes, two per byte (convrot_rotate_quant, weight packing)
//   kOperand4 4-bit codes as signed bytes in the W4A4 GEMM's operand order
//   kInt8     8-bit codes (amax / 127, clamp [-127, 127]) in natural order:
//             the ConvRot INT8 row-scaled format
enum : int { kPacked4 = 0, kOperand4 = 1, kInt8 = 2 };

// Byte position of channel c's code within its 16-byte run of the output
// row: natural order, except the W4A4 operand layout, which stores each
// 8-channel chunk in the order (0, 2, 4, 6, 1, 3, 5, 7).
template <int MODE>
__device__ __forceinline__ int code_pos(int c) {
  if (MODE != kOperand4) return c & 15;
  const int e = c & 7;
  return (c & 8) | ((e & 1) ? 4 + (e >> 1) : (e >> 1));
}

// Dynamic shared memory: S input stages of R * K bf16, then one transpose tile
// per half-warp, then S mbarriers.
__host__ __device__ constexpr int rq_stage_bytes(int R, int K) { return R * K * 2; }
__host__ __device__ constexpr int rq_smem_bytes(int R, int K, int S, int threads) {
  return S * rq_stage_bytes(R, K) + (threads / 16) * kTileBytes + 8 * S;
}

// LOG4G: log4 of the rotation group (4: 256, the default; 3: 64; 2: 16 --
// the convrot_groupsize variants).  A group of 4^LOG4G channels takes the
// first LOG4G radix-4 stages and the factor 2^-LOG4G; the per-row scale
// still spans the whole row.
template <int MODE, int LOG4G>
__global__ void __launch_bounds__(kMaxThreads) rotate_quant_kernel(const __grid_constant__ RQParams p) {
  constexpr bool PACKED = MODE == kPacked4;
  constexpr int kQLo = MODE == kInt8 ? -127 : -8, kQHi = MODE == kInt8 ? 127 : 7;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint32_t row_amax[3][kMaxRows];
  // Let the dependent GEMM launch now: it streams its weights meanwhile and
  // waits (griddepcontrol.wait) for this grid before reading codes or scales.
  // Not when this grid writes weights: then its successors start only once it
  // has completed.  This grid itself may have been launched before the
  // preceding kernel finished: wait for it before reading x or writing any
  // output.
  if (p.out.early_trigger) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // Parameters in registers (the inline-asm memory clobbers below would
  // otherwise reload them).
  const int M = p.M, K = p.K, G = p.G, R = p.R, S = p.S;
  const uint16_t* const x = p.x;
  const RotateQuantOut out = p.out;
  const int hw = threadIdx.x >> 4, l = threadIdx.x & 15;
  const int nhw = blockDim.x >> 4;
  const int stage_bytes = rq_stage_bytes(R, K);
  uint8_t* const stages = smem;
  uint8_t* const tile = smem + S * stage_bytes + hw * kTileBytes;
  uint8_t* const tile_w = tile + kTileRow * l;  // this lane's row
  const uint8_t* const tile_r = tile + 8 * l;   // this lane's column
  // Byte tiles of the two tasks inside the pair tile; odd half-warps start 16
  // bytes later so that the two half-warps of a warp hit different banks.
  uint8_t* const btile0 = tile + 16 * (hw & 1);
  uint8_t* const btile1 = btile0 + 256;
  uint8_t* const bw0 = btile0 + code_pos<MODE>(l);
  uint8_t* const bw1 = btile1 + code_pos<MODE>(l);
  uint64_t* const full = reinterpret_cast<uint64_t*>(smem + S * stage_bytes + nhw * kTileBytes);
  const int tasks = R * G;
  const int nb = p.nblocks;
  const int iters = static_cast<int>(blockIdx.x) < nb ? (nb - 1 - static_cast<int>(blockIdx.x)) / gridDim.x + 1 : 0;

  // Thread 0: the bulk copy of this block's row block number `it` into
  // stage `st` (= it mod S).
  auto issue = [&](int it, int st) {
    const int b = static_cast<int>(blockIdx.x) + it * static_cast<int>(gridDim.x);
    const int rows = min(R, M - b * R);
    const uint32_t bytes = static_cast<uint32_t>(rows) * static_cast<uint32_t>(K) * 2u;
    mbar_arrive_expect_tx(&full[st], bytes);
    bulk_load(stages + st * stage_bytes, x + static_cast<size_t>(b) * R * K, bytes, &full[st]);
  };
  if (threadIdx.x == 0) {
    for (int st = 0; st < S; ++st) mbar_init(&full[st], 1);
    fence_mbarrier_init();
    for (int it = 0; it < S && it < iters; ++it) issue(it, it);
  }
  for (int i = threadIdx.x; i < 3 * kMaxRows; i += blockDim.x) (&row_amax[0][0])[i] = 0u;
  __syncthreads();

  // The lane's two tasks: hw and hw + nhw (a task past the end computes on
  // row 0, group 0 of the stage and is never stored).
  const int task0 = hw, task1 = hw + nhw;
  const bool have0 = task0 < tasks, have1 = task1 < tasks;
  const int rloc0 = have0 ? task0 / G : 0, rloc1 = have1 ? task1 / G : 0;
  const int g0 = have0 ? task0 - rloc0 * G : 0, g1 = have1 ? task1 - rloc1 * G : 0;
  const int in0 = (rloc0 * K + g0 * 256 + l * 16) * 2, in1 = (rloc1 * K + g1 * 256 + l * 16) * 2;
  const size_t code_row = PACKED ? static_cast<size_t>(K / 2) : static_cast<size_t>(K);
  const size_t out0 = static_cast<size_t>(rloc0) * code_row + (PACKED ? g0 * 128 + l * 8 : g0 * 256 + l * 16);
  const size_t out1 = static_cast<size_t>(rloc1) * code_row + (PACKED ? g1 * 128 + l * 8 : g1 * 256 + l * 16);
  uint8_t* const codes = PACKED ? out.packed : reinterpret_cast<uint8_t*>(out.s8);

  // Loop counters kept incrementally (no division by runtime values): the
  // stage st = it mod S with its phase parity ph, the amax slot = it mod 3,
  // and the first row of the row block.
  int it = 0, st = 0, ph = 0, slot = 0;
  int row0 = static_cast<int>(blockIdx.x) * R;
  const int row_step = static_cast<int>(gridDim.x) * R;
  for (; it < iters; ++it) {
    const bool ok = mbar_wait(&full[st], ph);
    const uint8_t* stage = stages + st * stage_bytes;
    const bool live0 = ok && have0 && row0 + rloc0 < M;
    const bool live1 = ok && have1 && row0 + rloc1 < M;

    // ---- lane l: channels 16 l .. 16 l + 15 of both tasks, as pairs
    u64 P[16];
    {
      const uint4 a0 = *reinterpret_cast<const uint4*>(stage + in0);
      const uint4 a1 = *reinterpret_cast<const uint4*>(stage + in0 + 16);
      const uint4 b0 = *reinterpret_cast<const uint4*>(stage + in1);
      const uint4 b1 = *reinterpret_cast<const uint4*>(stage + in1 + 16);
      const uint32_t wa[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const uint32_t wb[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        P[2 * e] = f2(__uint_as_float(wa[e] << 16), __uint_as_float(wb[e] << 16));
        P[2 * e + 1] = f2(__uint_as_float(wa[e] & 0xFFFF0000u), __uint_as_float(wb[e] & 0xFFFF0000u));
      }
    }
    // stage on channel bits (0,1): stride 1
#pragma unroll
    for (int i = 0; i < 16; i += 4) bfly4(P[i], P[i + 1], P[i + 2], P[i + 3]);
    // stage on bits (2,3): stride 4
#pragma unroll
    for (int i = 0; i < 4; ++i) bfly4(P[i], P[i + 4], P[i + 8], P[i + 12]);
    // transpose: row l of the tile <- channels 16 l + i
#pragma unroll
    for (int c = 0; c < 8; ++c) *reinterpret_cast<ulonglong2*>(tile_w + 16 * c) = make_ulonglong2(P[2 * c], P[2 * c + 1]);
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 16; ++i) P[i] = *reinterpret_cast<const u64*>(tile_r + kTileRow * i);
    __syncwarp();
    // now P[i] = channel 16 i + l.  stage on bits (4,5): stride 16
    if (LOG4G >= 3) {
#pragma unroll
      for (int i = 0; i < 16; i += 4) bfly4(P[i], P[i + 1], P[i + 2], P[i + 3]);
    }
    // stage on bits (6,7): stride 64
    if (LOG4G >= 4) {
#pragma unroll
      for (int i = 0; i < 4; ++i) bfly4(P[i], P[i + 4], P[i + 8], P[i + 12]);
    }
    // the two tasks' max |v| (v = 2^LOG4G x'; the scaling waits for the row's amax)
    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
      float x0, x1, y0, y1;
      f2_split(P[i], x0, x1);
      f2_split(P[i + 1], y0, y1);
      m0 = max3(m0, fabsf(x0), fabsf(y0));
      m1 = max3(m1, fabsf(x1), fabsf(y1));
    }
    // ---- per-row amax: within each task (16 lanes), then across the row's tasks
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) {
      m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, o));
      m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, o));
    }
    if (l == 0 && live0) atomicMax(&row_amax[slot][rloc0], __float_as_uint(m0));
    if (l == 0 && live1) atomicMax(&row_amax[slot][rloc1], __float_as_uint(m1));
    // Every read of this iteration's stage and every amax contribution is
    // done after this barrier; a failed wait anywhere ends the loop for all.
    if (!__syncthreads_and(ok)) break;
    if (threadIdx.x == 0 && it + S < iters) {
      fence_proxy_async_smem();
      issue(it + S, st);
    }
    // Slot (it + 2) % 3 was last read in iteration it - 1 and is next written
    // in iteration it + 2, after one more barrier.
    if (threadIdx.x < kMaxRows) row_amax[slot == 0 ? 2 : slot - 1][threadIdx.x] = 0u;

    // ---- quantize: every lane forms its two rows' scales from their amax
    constexpr float kInvG = LOG4G == 4 ? 0.0625f : (LOG4G == 3 ? 0.125f : 0.25f);  // 2^-LOG4G
    constexpr float kG = 1.0f / kInvG;
    constexpr float kThr = kG * (0.5f - (MODE == kInt8 ? 0x1p-14f : 0x1p-18f));      // 2^LOG4G (1/2 - m)
    const float scale0 = div_by_qmax<kQHi>(__uint_as_float(row_amax[slot][rloc0]) * kInvG);
    const float scale1 = div_by_qmax<kQHi>(__uint_as_float(row_amax[slot][rloc1]) * kInvG);
    const bool in_range = scale0 >= kMinScale && scale0 <= kMaxScale && scale1 >= kMinScale && scale1 <= kMaxScale;
    // The code bytes of channel 16 i + l go to their row-order positions in
    // the byte tiles as they are formed (a lane that falls back to the exact
    // quotient writes its bytes again).
    bool done = false;
    if (in_range) {
      // k = rint(v y) and the remainder v - 2^LOG4G s k; kept where no
      // remainder reaches 2^LOG4G s (1/2 - m)
      const u64 y = f2(rcp_approx(scale0) * kInvG, rcp_approx(scale1) * kInvG);
      const u64 nd = f2(-(scale0 * kG), -(scale1 * kG));
      const u64 mg = f2(kMagic, kMagic);
      float e0 = 0.0f, e1 = 0.0f;
#pragma unroll
      for (int i = 0; i < 16; i += 2) {
        const u64 ca = f2_fma(P[i], y, mg), cb = f2_fma(P[i + 1], y, mg);
        const u64 da = f2_fma(nd, f2_sub(ca, mg), P[i]), db = f2_fma(nd, f2_sub(cb, mg), P[i + 1]);
        float t0, t1, u0, u1;
        f2_split(ca, t0, t1);
        f2_split(cb, u0, u1);
        bw0[16 * i] = static_cast<uint8_t>(__float_as_uint(t0));
        bw1[16 * i] = static_cast<uint8_t>(__float_as_uint(t1));
        bw0[16 * i + 16] = static_cast<uint8_t>(__float_as_uint(u0));
        bw1[16 * i + 16] = static_cast<uint8_t>(__float_as_uint(u1));
        f2_split(da, t0, t1);
        f2_split(db, u0, u1);
        e0 = max3(e0, fabsf(t0), fabsf(u0));
        e1 = max3(e1, fabsf(t1), fabsf(u1));
      }
      done = e0 <= scale0 * kThr && e1 <= scale1 * kThr;
    }
    if (!done) {
      const u64 inv2 = f2(kInvG, kInvG);
      if (in_range) {
        // A quotient next to a half-integer: the exact quotient RN(x'/s).
        const u64 rr = f2(__frcp_rn(scale0), __frcp_rn(scale1)), ns = f2(-scale0, -scale1);
        const u64 mg = f2(kMagic, kMagic);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const u64 xv = f2_mul(P[i], inv2);
          u64 q = f2_mul(xv, rr);
          q = f2_fma(f2_fma(ns, q, xv), rr, q);  // faithful
          q = f2_fma(f2_fma(ns, q, xv), rr, q);  // RN(x / s)
          float t0, t1;
          f2_split(f2_add(q, mg), t0, t1);       // low byte = rint(q)
          bw0[16 * i] = static_cast<uint8_t>(__float_as_uint(t0));
          bw1[16 * i] = static_cast<uint8_t>(__float_as_uint(t1));
        }
      } else {
        // A zero, tiny or huge scale (a whole row takes this branch): IEEE division.
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float x0, x1;
          f2_split(f2_mul(P[i], inv2), x0, x1);
          const int q0 = scale0 != 0.0f ? __float2int_rn(__fdiv_rn(x0, scale0)) : 0;
          const int q1 = scale1 != 0.0f ? __float2int_rn(__fdiv_rn(x1, scale1)) : 0;
          bw0[16 * i] = static_cast<uint8_t>(min(kQHi, max(kQLo, q0)));
          bw1[16 * i] = static_cast<uint8_t>(min(kQHi, max(kQLo, q1)));
        }
      }
    }
    // ---- back to row order: read the byte tiles, store
    __syncwarp();
    const uint4 o0 = *reinterpret_cast<const uint4*>(btile0 + 16 * l);  // channels 16 l .. 16 l + 15
    const uint4 o1 = *reinterpret_cast<const uint4*>(btile1 + 16 * l);
    __syncwarp();
    const size_t obase = static_cast<size_t>(row0) * code_row;
    if (live0) {
      if (PACKED)
        *reinterpret_cast<uint2*>(codes + obase + out0) = make_uint2(pack_nibbles(o0.x, o0.y), pack_nibbles(o0.z, o0.w));
      else
        *reinterpret_cast<uint4*>(codes + obase + out0) = o0;
      if (g0 == 0 && l == 0) out.scale[row0 + rloc0] = scale0;
    }
    if (live1) {
      if (PACKED)
        *reinterpret_cast<uint2*>(codes + obase + out1) = make_uint2(pack_nibbles(o1.x, o1.y), pack_nibbles(o1.z, o1.w));
      else
        *reinterpret_cast<uint4*>(codes + obase + out1) = o1;
      if (g1 == 0 && l == 0) out.scale[row0 + rloc1] = scale1;
    }
    if (++st == S) {
      st = 0;
      ph ^= 1;
    }
    slot = slot == 2 ? 0 : slot + 1;
    row0 += row_step;
  }
  if (it < iters && threadIdx.x == 0) {
    // A wait gave up: let the copies still in flight land before the block
    // exits (their stages are it .. min(it + S, iters) - 1).
    for (int k = it; k < it + S && k < iters; ++k) (void)mbar_drain(&full[k % S], (k / S) & 1, 100000000ull);
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

template <int MODE, int LOG4G>
cudaError_t launch_rq(const RQParams& p, int threads, cudaStream_t stream) {
  static std::atomic<int> cache[64];
  const int smem = rq_smem_bytes(p.R, p.K, p.S, threads);
  const void* kfn = reinterpret_cast<const void*>(rotate_quant_kernel<MODE, LOG4G>);
  cudaError_t e = ensure_dynamic_smem(kfn, smem, cache);
  if (e != cudaSuccess) return note_cuda(e, "rotate_quant: dynamic shared memory attribute");
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, rotate_quant_kernel<MODE, LOG4G>, threads, smem);
  if (e != cudaSuccess) return note_cuda(e, "rotate_quant: occupancy query");
  if (per_sm < 1) per_sm = 1;
  int grid = num_sms_cached() * per_sm;
  if (grid > p.nblocks) grid = p.nblocks;
  // Programmatic stream serialization: the kernel may launch while the
  // preceding one finishes (it waits for it with griddepcontrol.wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note_cuda(cudaLaunchKernelEx(&cfg, rotate_quant_kernel<MODE, LOG4G>, p), "rotate_quant: launch");
}

}  // namespace

cudaError_t launch_rotate_quant(const uint16_t* x, int M, int K, RotateQuantOut out, cudaStream_t stream) {
  RQParams p{};
  p.x = x;
  p.M = M;
  p.K = K;
  p.G = K / 256;
  p.out = out;
  const int sms = num_sms_cached();
  // One task (16 lanes) per group, two tasks per half-warp.  Rows per row
  // block R: up to 32 tasks, and no more rows than leave about two row blocks
  // per SM, so that small M spreads its rows over the SMs.
  int R = 1;
  if (p.G <= 32) {
    const int by_tasks = 32 / p.G;
    const int by_spread = (M + 2 * sms - 1) / (2 * sms);
    R = by_tasks < by_spread ? by_tasks : by_spread;
    if (R < 1) R = 1;
    if (R > kMaxRows) R = kMaxRows;
  }
  p.R = R;
  p.nblocks = (M + R - 1) / R;
  const int hws = (R * p.G + 1) / 2;
  const int threads = ((hws * 16 + 31) / 32) * 32;
  if (threads > kMaxThreads) return note_cuda(cudaErrorInvalidValue, "rotate_quant: block shape");
  // Blocks per SM by threads and registers (up to 64 per thread); then the
  // input ring: about 128 KB of row blocks in flight per SM, at least 2
  // stages where they fit next to the transpose tiles (fewer blocks per SM
  // otherwise), never more stages than a block has row blocks.
  int per_sm = 65536 / (threads * 64);
  if (per_sm > 2048 / threads) per_sm = 2048 / threads;
  if (per_sm > 8) per_sm = 8;
  if (per_sm < 1) per_sm = 1;
  const int stage = rq_stage_bytes(R, K);
  const int fixed = rq_smem_bytes(R, K, 0, threads) + 64;
  int s_fit = 0;
  for (;;) {
    s_fit = (220 * 1024 / per_sm - fixed) / stage;
    if (s_fit >= 2 || per_sm == 1) break;
    --per_sm;
  }
  int S = (128 * 1024 + per_sm * stage - 1) / (per_sm * stage);
  if (S < 2) S = 2;
  if (S > 8) S = 8;
  if (S > s_fit) S = s_fit;
  const int most_iters = (p.nblocks + sms * per_sm - 1) / (sms * per_sm);
  if (S > most_iters) S = most_iters;
  if (S < 1) S = 1;
  p.S = S;
  cudaError_t e;
  if (out.group != 256 && out.group != 64 && out.group != 16) return note_cuda(cudaErrorInvalidValue, "rotate_quant: group");
  if (out.int8) {
    if (out.group != 256) return note_cuda(cudaErrorInvalidValue, "rotate_quant: int8 group");
    e = launch_rq<kInt8, 4>(p, threads, stream);
  } else if (out.packed != nullptr) {
    e = out.group == 256 ? launch_rq<kPacked4, 4>(p, threads, stream)
        : out.group == 64 ? launch_rq<kPacked4, 3>(p, threads, stream)
                          : launch_rq<kPacked4, 2>(p, threads, stream);
  } else {
    e = out.group == 256 ? launch_rq<kOperand4, 4>(p, threads, stream)
        : out.group == 64 ? launch_rq<kOperand4, 3>(p, threads, stream)
                          : launch_rq<kOperand4, 2>(p, threads, stream);
  }
  count_dispatch(0);
  return e;
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
