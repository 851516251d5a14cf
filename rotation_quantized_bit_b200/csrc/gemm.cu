// gemm.cu -- W4A4 integer GEMM with the rank-one epilogue on sm_100a
// tensor cores (tcgen05.mma kind::i8, accumulators in tensor memory).
//
// What it computes ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4
// (+ConvRot...)", speed table: a rank-one s4 MMA kernel):
//   acc[m, n] = sum_k q_a[m, k] * q_w[n, k]            (exact int32)
//   y[m, n]   = acc * s_a[m] * s_w[n] + bias[n]        (fp32, then bf16 RNE)
//
// Mapping to the B200 tensor core.  sm_100a has no 4-bit integer MMA kind,
// so the 4-bit codes are widened to bytes for kind::i8.  The weight tile
// is the MMA "A" operand and lives in tensor memory (swap-AB: MMA M = 128
// output channels, MMA N = BT tokens):
//   * a TMA producer warp streams packed weight tiles (128 rows x 64 bytes =
//     128 K values) and activation byte tiles (BT rows x 128 bytes, 128-byte
//     swizzle) into a ring of shared-memory stages;
//   * four unpack warps turn each packed weight row into 32 tensor-memory
//     columns with three integer ops per 8 codes: the low nibbles of a
//     32-bit word are codes (0,2,4,6), the high nibbles (1,3,5,7); moving a
//     two's-complement nibble into the high half of a byte gives the signed
//     byte 16 * q_w, so (w << 4) & 0xF0F0F0F0 and w & 0xF0F0F0F0 are the
//     two halves, already sign-correct;
//   * one thread issues tcgen05.mma kind::i8 (A = s8 weights from tensor
//     memory, B = s8 activations from shared memory, K = 32 per
//     instruction).  The activation bytes are stored in the matching per-8
//     chunk order, so the contraction pairs the right codes;
//   * the accumulator is exactly 16 * acc (|16 acc| <= 1024 K < 2^31), and
//     the epilogue shifts it right by 4.
// The W8A8 formats (int8 weights [N, K]) use the same kernel with WK = kWInt8:
// the weight tile goes by TMA straight into shared memory as the MMA's A
// operand (no unpack, no tensor-memory A slots), the accumulator is the
// integer product itself, and per-tensor scales are read with stride 0.
// The asymmetric W4A8 format (WK = kWCodebook; "Nicolaslas/Rebels_w4a8s",
// "What's inside a file") stores 4-bit indices into a 16-level codebook, an
// e4m3 scale per 16 weights along K and a scale per output channel.  Its
// weights take the 4-bit path, but the unpack warps decode each index to
// the int8 weight clamp(rint(level * s_rel), -127, 127) through a per-CTA
// table (16 levels for each of the 256 scale bytes), in natural K order to
// match int8 activation codes; the accumulator is the plain integer sum.
// Work is cut into units of one 256-wide K block of one output tile; see
// the kernel below for the two schedules (whole tiles, and K split over a
// thread-block cluster when there are few tiles) and the exact reduction of
// split tiles in shared memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace convrot {

namespace {

constexpr int kRows = 128;       // output channels per tile (MMA M)
constexpr int kKB = 256;         // K values per unit (pipeline step)
constexpr int kWTileBytes = kRows * kKB / 2;  // 16 KB packed weights per unit
constexpr int kXBox = 128;       // K bytes per activation TMA box (the 128-byte swizzle span)
constexpr int kMaxStages = 16;   // depth limit of the shared-memory TMA ring
constexpr int kDoneRing = 32;    // MMA completion barriers, one per unit mod 32 (>= stages, >= A slots)
constexpr int kMaxASlots = 8;    // tensor-memory A slots (64 columns each)
constexpr int kSRelTileBytes = kRows * kKB / 16;  // 2 KB of e4m3 group scales per unit (codebook weights)
constexpr int kLutBytes = 256 * 16;               // decoded levels per scale byte (codebook weights)

// One packed weight row of a unit (128 bytes = 256 codes) -> 64 tensor-memory
// columns of signed bytes.  The tile landed with the 128-byte TMA swizzle:
// 16-byte chunk c of row r sits at chunk c ^ (r & 7).
__device__ __forceinline__ void unpack_row_to_tmem(const uint8_t* wstage, int row, uint32_t taddr) {
  const int sw = row & 7;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t cols[32];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 v = *reinterpret_cast<const uint4*>(wstage + row * 128 + (((4 * h + c) ^ sw) << 4));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        cols[8 * c + 2 * j] = (w[j] << 4) & 0xF0F0F0F0u;
        cols[8 * c + 2 * j + 1] = w[j] & 0xF0F0F0F0u;
      }
    }
    tmem_st_32x32b_x32(taddr + 32u * h, cols);
  }
}

// Byte permute with the sign-replicate mode: byte i of the result is byte
// (c >> 4i) & 7 of {b, a} (a = bytes 0..3), or, when bit 3 of that selector
// nibble is set, that byte's top bit copied into all 8 bits.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Four 4-bit indices (the low 16 bits of s, index i in bits 4i..4i+3) -> the
// four int8 levels lut[index] of the 16-byte row (t0..t3).  Indices 0..7 come
// from {t1, t0}, 8..15 from {t3, t2}; the per-byte choice is the index's bit
// 3, turned into a 0x00 / 0xFF byte mask by the sign-replicate mode (the top
// bit of byte 0 of s << 4 is bit 3 of index 0, of byte 0 of s bit 3 of
// index 1, and so on: selectors 8, C, 9, D).
__device__ __forceinline__ uint32_t decode4(uint32_t s, const uint4& t) {
  const uint32_t sel = s & 0x7777u;
  const uint32_t lo = prmt(t.x, t.y, sel);
  const uint32_t hi = prmt(t.z, t.w, sel);
  const uint32_t mask = prmt(s << 4, s, 0xD9C8u);
  return (hi & mask) | (lo & ~mask);
}

// One weight row of a unit in codebook form (128 bytes = 256 indices, the
// 128-byte TMA swizzle as above; srow: the row's 16 e4m3 scale bytes, one
// per 16 indices) -> 64 tensor-memory columns of int8 weights in natural K
// order (column c holds k = 4c .. 4c + 3).  lut[b * 16 + i] is the int8
// weight of index i under scale byte b.
__device__ __forceinline__ void decode_row_to_tmem(const uint8_t* wstage, const uint8_t* srow, const uint8_t* lut,
                                                   int row, uint32_t taddr) {
  const int sw = row & 7;
  const uint4 sv = *reinterpret_cast<const uint4*>(srow);
  const uint32_t sb[4] = {sv.x, sv.y, sv.z, sv.w};
#pragma unroll
  for (int qt = 0; qt < 4; ++qt) {  // quarter row: 64 indices -> 16 columns
    uint32_t cols[16];
#pragma unroll
    for (int c2 = 0; c2 < 2; ++c2) {
      const int cc = 2 * qt + c2;  // 16-byte chunk: indices k = 32 cc .. 32 cc + 31
      const uint4 v = *reinterpret_cast<const uint4*>(wstage + row * 128 + ((cc ^ sw) << 4));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int gg = 0; gg < 2; ++gg) {
        const int g = 2 * cc + gg;  // group of 16 indices within the unit
        const uint32_t b = (sb[g >> 2] >> (8 * (g & 3))) & 0xFFu;
        const uint4 t = *reinterpret_cast<const uint4*>(lut + 16 * b);
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * gg + jj;  // word j of the chunk: indices k = 32 cc + 8j .. + 7
          cols[8 * c2 + 2 * j] = decode4(w[j], t);
          cols[8 * c2 + 2 * j + 1] = decode4(w[j] >> 16, t);
        }
      }
    }
    tmem_st_32x32b_x16(taddr + 16u * qt, cols);
  }
}

// e4m3 ("fn": bias 7, no infinities, S.1111.111 = NaN) byte -> fp32, exactly.
__device__ __forceinline__ float e4m3_to_float(uint32_t b) {
  const uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float mag = e == 0 ? __fmul_rn(static_cast<float>(m), 0.001953125f)  // m * 2^-9
                     : __uint_as_float(((e + 120u) << 23) | (m << 20));
  if (e == 15u && m == 7u) mag = __uint_as_float(0x7FC00000u);
  return (b & 0x80u) ? -mag : mag;
}

// The decoded weight of one level under one scale: rint(level * s) clamped
// to [-127, 127], NaN -> 0.
__device__ __forceinline__ int32_t decode_level(float level, float s) {
  float p = __fmul_rn(level, s);
  if (p != p) return 0;
  p = fminf(fmaxf(p, -127.0f), 127.0f);
  return __float2int_rn(p);
}

// int32 -> fp32 without the conversion unit: for |i| < 2^22 the float with
// bits 0x4B400000 + i is exactly 1.5 * 2^23 + i, and subtracting 1.5 * 2^23
// leaves exactly i (the value a correctly rounded conversion gives, since i
// is representable).  |acc| <= 64 K <= 2^21 here.
__device__ __forceinline__ float int_to_float_exact(int32_t i) {
  return __fsub_rn(__int_as_float(0x4B400000 + i), 12582912.0f);
}

// fp32 -> bf16 bits, round to nearest even, with integer operations (finite
// values and infinities; the epilogue produces no NaN from finite inputs).
__device__ __forceinline__ uint16_t bf16_bits_rne(float y) {
  const uint32_t u = __float_as_uint(y);
  return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// One output element from the MMA sum (16 * acc): scales and bias already
// loaded by the caller.
// The accumulator as a float: the W4A4 sum (|acc| <= 2^21) by the exact
// bit trick, the 8-bit sums (up to 127^2 K) by a correctly rounded
// conversion.  PLAIN: the MMA sum is the accumulator itself (8-bit weights
// or decoded codebook weights), not 16 * acc.
template <bool PLAIN>
__device__ __forceinline__ float acc_to_float(int32_t acc) {
  return PLAIN ? __int2float_rn(acc) : int_to_float_exact(acc);
}

template <int SINK, bool PLAIN, class P>
__device__ __forceinline__ void store_output(const P& p, int m, int n, int32_t dsum, float sa, float sw,
                                             float bv) {
  const int32_t acc = PLAIN ? dsum : dsum >> 4;  // 4-bit weights entered the MMA as 16 * q_w
  const size_t idx = static_cast<size_t>(m) * p.N + n;
  if (SINK == static_cast<int>(GemmSink::kS32)) {
    static_cast<int32_t*>(p.out)[idx] = acc;
    return;
  }
  float y = __fmul_rn(__fmul_rn(acc_to_float<PLAIN>(acc), sa), sw);
  if (p.bias) y = __fadd_rn(y, bv);
  if (SINK == static_cast<int>(GemmSink::kF32)) {
    static_cast<float*>(p.out)[idx] = y;
  } else {
    static_cast<uint16_t*>(p.out)[idx] = bf16_bits_rne(y);
  }
}

// Outputs of one 32-token chunk of one output channel n: tokens m .. m +
// count - 1 (count <= 32), accumulators v (16 * acc), token scales sa[0..31]
// (16-byte aligned in shared memory).
template <int SINK, bool PLAIN, class P>
__device__ __forceinline__ void store_chunk(const P& p, int m, int n, const uint32_t (&v)[32], const float* sa,
                                            float sw, float bv, int count) {
  const size_t ld = static_cast<size_t>(p.N);
  const size_t base = static_cast<size_t>(m) * ld + static_cast<size_t>(n);
  if (SINK == static_cast<int>(GemmSink::kS32)) {
    int32_t* o = static_cast<int32_t*>(p.out) + base;
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j < count) o[j * ld] = PLAIN ? static_cast<int32_t>(v[j]) : static_cast<int32_t>(v[j]) >> 4;
    return;
  }
  const float4* sa4 = reinterpret_cast<const float4*>(sa);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 s4 = sa4[q];
    const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = 4 * q + r;
      if (j < count) {
        const int32_t acc = PLAIN ? static_cast<int32_t>(v[j]) : static_cast<int32_t>(v[j]) >> 4;
        float y = __fmul_rn(__fmul_rn(acc_to_float<PLAIN>(acc), sv[r]), sw);
        if (p.bias) y = __fadd_rn(y, bv);
        if (SINK == static_cast<int>(GemmSink::kF32))
          static_cast<float*>(p.out)[base + j * ld] = y;
        else
          static_cast<uint16_t*>(p.out)[base + j * ld] = bf16_bits_rne(y);
      }
    }
  }
}

// ---------------------------------------------------------------- the kernel
//
// A unit is one 256-wide K block of one output tile (BT tokens x 128 output
// channels).  Two schedules:
//   * whole tiles (splits == 1): one CTA per SM walks the tiles c, c + grid,
//     c + 2 grid ... (neighbouring CTAs share activation and weight tiles in
//     L2), each tile's units summed in one tensor-memory accumulator;
//   * split-K (splits == S > 1, few tiles): the S CTAs of a thread-block
//     cluster take even shares of one tile's K blocks.  Each pushes its int32
//     partial tile, in 4-token groups, into the shared memory of the CTA that
//     owns the group (group g -> CTA g % S); after one cluster barrier every
//     CTA adds the S partials of its own groups and stores them.  Integer
//     addition is exact, so the result does not depend on the split.
//   warp 0      TMA producer (ring of `nstages` shared-memory stages)
//   warp 1      TMEM allocation (all 512 columns) and the MMA-issuing thread
//   warps 2..5  weight unpack into 64-column A slots of tensor memory
//   warps 6..13 epilogue, draining one of two accumulators while the MMA
//               fills the other (two warps per tensor-memory lane quadrant,
//               each taking every other 32-column chunk)
// A stage's weight tile lands on wfull[s]; ready[s] completes when its
// activation tile has landed and all four unpack warps have written the
// unit's weights to tensor memory, so the MMA thread waits on ready alone.
// Weight tiles do not depend on the preceding prologue kernel: the first
// stages are requested, and their weights unpacked, before the grid waits
// for that kernel.  The MMA thread issues the units of a tile two at a time
// (16 MMAs between waits: at small token counts an MMA takes ~45 cycles and
// each wait, commit or branch between MMA groups costs about as much), then
// commits once per unit, to done[unit % 32]; that completion frees both the
// unit's shared-memory stage (for the TMA producer) and its A slot (for the
// unpack warps).
constexpr int kPThreads = 448;
constexpr int kEpiThreads = 256;  // warps 6..13

struct PParams {
  const float* s_a;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int M, N, K;
  int BT, m_tiles, num_tiles, nstages, kbn;
  int n_tiles;
  int n_fast;       // tile order: 1 = output-channel tile fastest (activation rows shared by neighbours)
  int acc_stride;   // tensor-memory columns per accumulator (BT rounded up to 32)
  int a_slots;      // A slots of 64 columns after the two accumulators
  int splits;       // 1: whole tiles; S > 1: the cluster of S CTAs splits one tile's K
  int pair;         // the MMA thread issues two units per group
  int sa_stride;    // 0: one activation scale for every row
  int sw_stride;    // 0: one weight scale for every output channel
  const float* codebook;  // [16] levels (codebook weights)
  int lut_off;      // shared-memory offset of the decode table from the header (codebook weights)
};

struct PHeader {
  uint64_t wfull[kMaxStages];   // the stage's weight tile landed
  uint64_t ready[kMaxStages];   // the stage's activation tile landed and its weights are in tensor memory
  uint64_t done[kDoneRing];     // unit i's MMAs have completed (its stage and A slot are free)
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
};

// Token tile and channel tile of a tile index.  The whole-tile schedule walks
// tiles in index order, the CTAs of one round taking consecutive indices.
// With the token tile fastest (n_fast == 0) a round covers every token tile
// for a few channel tiles: the weights of the round are shared from L2 and
// the activations are streamed once per round.  With the channel tile fastest
// (n_fast == 1) a round covers every channel tile for a few token tiles: its
// activation rows are shared from L2 and all the weights stay in L2 from
// round to round, so activations larger than L2 are read from DRAM once
// instead of once per round.
__device__ __forceinline__ int tile_mi(const PParams& p, int tile) {
  const int d = p.n_fast ? p.n_tiles : p.m_tiles, q = tile / d, r = tile - q * d;
  return p.n_fast ? q : r;
}
__device__ __forceinline__ int tile_ni(const PParams& p, int tile) {
  const int d = p.n_fast ? p.n_tiles : p.m_tiles, q = tile / d, r = tile - q * d;
  return p.n_fast ? r : q;
}

// This CTA's first unit (tile, K block) and number of units.
__device__ __forceinline__ void unit_range(const PParams& p, int& tile, int& kb, int& count) {
  if (p.splits > 1) {
    const int j = static_cast<int>(blockIdx.x) % p.splits;  // rank in the cluster
    tile = static_cast<int>(blockIdx.x) / p.splits;
    kb = (j * p.kbn) / p.splits;
    count = ((j + 1) * p.kbn) / p.splits - kb;
  } else {
    tile = static_cast<int>(blockIdx.x);
    kb = 0;
    count = (p.num_tiles - tile + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x) * p.kbn;
  }
}
// The unit after (tile, kb) in this CTA's list.
__device__ __forceinline__ void unit_next(const PParams& p, int& tile, int& kb) {
  if (++kb == p.kbn) {
    kb = 0;
    tile += static_cast<int>(gridDim.x);
  }
}

template <int SINK, int WK>
__global__ void __launch_bounds__(kPThreads, 1)
    w4a4_tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_s, const __grid_constant__ PParams p) {
  constexpr bool W8 = WK == kWInt8;       // int8 weights: shared-memory A operand, no unpack
  constexpr bool CB = WK == kWCodebook;   // codebook indices + group scales, decoded by the unpack warps
  constexpr bool PLAIN = WK != kW4;       // the MMA sum is the accumulator itself
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // The next kernel on the stream (launched with programmatic stream
  // serialization: another GEMM, or a prologue) may start now and prepare
  // what does not depend on this grid; it waits for this grid's completion
  // (griddepcontrol.wait) before touching anything this grid reads or writes.
  pdl_launch_dependents();
  const int BT = p.BT;
  const int ns = p.nstages;
  // Weight bytes of a unit: int8 [128 x 256]; packed [128 x 128] (+ the
  // [128 x 16] e4m3 group scales for codebook weights).
  constexpr int kWBytes = W8 ? 2 * kWTileBytes : (CB ? kWTileBytes + kSRelTileBytes : kWTileBytes);
  const int stage_bytes = kWBytes + BT * kKB;
  const int nas = p.a_slots;
  const uint32_t a_col0 = 2u * static_cast<uint32_t>(p.acc_stride);
  PHeader* hdr = reinterpret_cast<PHeader*>(smem + ns * stage_bytes);
  float* sa_buf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(hdr) + 1024);  // [2][192]
  int32_t* red = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(hdr) + 2560);  // split-K partials
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kbn = p.kbn;
  int tile0, kb0, total;
  unit_range(p, tile0, kb0, total);
  // First weight row and first token row of a tile.
  auto w_row = [&](int tile) { return tile_ni(p, tile) * kRows; };
  auto x_row = [&](int tile) { return tile_mi(p, tile) * BT; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&hdr->wfull[s], 1);
      // W4: the producer (with the activation bytes) + one arrive per unpack
      // warp; W8: the producer twice (weight bytes, activation bytes).
      mbar_init(&hdr->ready[s], W8 ? 2 : 5);
    }
    for (int r = 0; r < kDoneRing; ++r) mbar_init(&hdr->done[r], 1);  // one MMA commit
    for (int b = 0; b < 2; ++b) {
      mbar_init(&hdr->acc_full[b], 1);
      mbar_init(&hdr->acc_empty[b], kEpiThreads / 32);  // one arrive per epilogue warp
    }
    fence_mbarrier_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
    if (CB) prefetch_tmap(&tm_s);
  }
  if (warp == 1) {
    tmem_alloc(&hdr->tmem_base, 512u);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = hdr->tmem_base;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    // A stage's weight tile completes on wfull[s]; its activation tile on
    // ready[s] (the producer's arrival, together with the unpack warps').
    if (lane == 0) {
      const uint32_t xbytes = static_cast<uint32_t>(BT * kKB);
      // The producer walks its units with a cursor that carries the tile's
      // first weight and token rows; they change (two integer divisions)
      // only when the cursor moves to the next tile, and the move is made
      // before the producer waits for the stage it refills, so the waits
      // are followed by the copies at once.
      struct Cursor {
        int tile, kb, wr, xr;
      };
      auto at = [&](int tile, int kb) { return Cursor{tile, kb, w_row(tile), x_row(tile)}; };
      auto next = [&](Cursor& c) {
        if (++c.kb == p.kbn) c = at(c.tile + static_cast<int>(gridDim.x), 0);
      };
      auto load_w = [&](int s, const Cursor& c) {
        if (W8) {
          mbar_arrive_expect_tx(&hdr->ready[s], static_cast<uint32_t>(kWBytes));
          tma_load_2d(smem + s * stage_bytes, &tm_w, &hdr->ready[s], c.kb * kKB, c.wr);
          tma_load_2d(smem + s * stage_bytes + kWTileBytes, &tm_w, &hdr->ready[s], c.kb * kKB + kXBox, c.wr);
        } else {
          mbar_arrive_expect_tx(&hdr->wfull[s], static_cast<uint32_t>(kWBytes));
          tma_load_2d(smem + s * stage_bytes, &tm_w, &hdr->wfull[s], c.kb * (kKB / 2), c.wr);
          if (CB) tma_load_2d(smem + s * stage_bytes + kWTileBytes, &tm_s, &hdr->wfull[s], c.kb * (kKB / 16), c.wr);
        }
      };
      auto load_x = [&](int s, const Cursor& c) {
        uint8_t* xs = smem + s * stage_bytes + kWBytes;
        mbar_arrive_expect_tx(&hdr->ready[s], xbytes);
        tma_load_2d(xs, &tm_x, &hdr->ready[s], c.kb * kKB, c.xr);
        tma_load_2d(xs + BT * kXBox, &tm_x, &hdr->ready[s], c.kb * kKB + kXBox, c.xr);
      };
      // Weight tiles of the first stages do not depend on the preceding
      // prologue kernel: request them before waiting for it.
      const int prime = total < ns ? total : ns;
      Cursor c = at(tile0, kb0);
      for (int i = 0; i < prime; ++i, next(c)) load_w(i, c);
      pdl_wait();
      c = at(tile0, kb0);
      for (int i = 0; i < prime; ++i, next(c)) load_x(i, c);
      int it = prime, s = prime % ns;  // stage of unit `it`
      bool w_only = false;              // unit `it` has its weight copy issued but not its activations
      for (; it < total; ++it, next(c)) {
        const int w = it - ns;  // the unit that last used stage s
        // The stage's weight region is free once unit w's weights are in
        // tensor memory (its ready phase: the unpack warps arrive after their
        // reads), an MMA's duration before the stage's activations are; int8
        // weights are the MMA's own operand and wait for its completion.
        if (!W8) {
          if (!mbar_wait(&hdr->ready[s], (w / ns) & 1)) break;
          load_w(s, c);
          w_only = true;
        }
        if (!mbar_wait(&hdr->done[w % kDoneRing], (w / kDoneRing) & 1)) break;
        w_only = false;
        if (W8) load_w(s, c);
        load_x(s, c);
        if (++s == ns) s = 0;
      }
      // Drain: every issued load has landed before the block may exit.  In
      // the normal case the last stages' barriers have completed; after a
      // failed wait (anywhere in the grid) the weight tiles are awaited with a
      // time limit that ignores the error word (that of unit `it` too, when
      // the loop stopped between its two copies), and the activation tiles,
      // whose barrier also needs the unpack warps, are given a fixed 100 us.
      bool clean = true;
      for (int i = (it > ns ? it - ns : 0); i < it; ++i) {
        if (clean)
          clean = (W8 || mbar_wait(&hdr->wfull[i % ns], (i / ns) & 1)) && mbar_wait(&hdr->ready[i % ns], (i / ns) & 1);
        if (!clean && !W8) (void)mbar_drain(&hdr->wfull[i % ns], (i / ns) & 1, 100000000ull);
      }
      if (w_only) (void)mbar_drain(&hdr->wfull[it % ns], (it / ns) & 1, 100000000ull);
      if (!clean || it < total) {
        const unsigned long long t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    // The whole warp runs the loop, so that the operand descriptors are
    // warp-uniform values; lane 0 issues the MMAs and commits.  ready[s]
    // says both operands of the stage's unit are in place.
    {
      const bool leader = lane == 0;
      const uint32_t idesc = umma_idesc_i8(kRows, BT, /*a_signed=*/true, /*b_signed=*/true);
      const uint32_t x1 = static_cast<uint32_t>(BT * kXBox);  // second activation box of a stage
      const uint32_t smem0 = smem_u32(smem) + static_cast<uint32_t>(kWBytes);
      int kb = kb0, seg = 0, s = 0, a = 0, sph = 0;
      bool ok = true;
      // The 8 MMAs of the unit in stage s / A slot a (acc0: accumulate into
      // the existing sum for the first of them).
      auto issue_unit = [&](uint32_t d_tmem, uint32_t acc0) {
        const uint32_t xs = smem0 + static_cast<uint32_t>(s * stage_bytes);
        const uint64_t bd0 = umma_desc_k_sw128(xs), bd1 = umma_desc_k_sw128(xs + x1);
        if (W8) {
          const uint32_t ws = xs - static_cast<uint32_t>(kWBytes);
          const uint64_t ad0 = umma_desc_k_sw128(ws), ad1 = umma_desc_k_sw128(ws + kWTileBytes);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < kKB / 32; ++kk)
              umma_i8_ss(d_tmem, (kk < 4 ? ad0 : ad1) + 2 * (kk & 3), (kk < 4 ? bd0 : bd1) + 2 * (kk & 3), idesc,
                         kk == 0 ? acc0 : 1u);
          }
        } else {
          const uint32_t at = tmem + a_col0 + 64u * static_cast<uint32_t>(a);
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < kKB / 32; ++kk)
              umma_i8_ts(d_tmem, at + 8 * kk, (kk < 4 ? bd0 : bd1) + 2 * (kk & 3), idesc, kk == 0 ? acc0 : 1u);
          }
        }
      };
      auto advance = [&]() {
        if (++s == ns) {
          s = 0;
          sph ^= 1;
        }
        if (++a == nas) a = 0;
      };
      for (int i = 0; i < total && ok;) {
        const int len = min(total - i, kbn - kb);  // units of this segment
        const int b = seg & 1;
        if (seg >= 2 && !__all_sync(0xffffffffu, mbar_wait(&hdr->acc_empty[b], ((seg / 2) - 1) & 1))) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * p.acc_stride);
        int j = 0;
        // Two units per group when the MMAs are short (small token tiles,
        // enough stages and A slots to prepare two units ahead).
        if (p.pair) {
          for (; j + 1 < len; j += 2, i += 2) {
            const int s1 = s + 1 == ns ? 0 : s + 1;
            const int ph1 = s + 1 == ns ? sph ^ 1 : sph;
            ok = __all_sync(0xffffffffu, mbar_wait(&hdr->ready[s], sph) & mbar_wait(&hdr->ready[s1], ph1));
            if (!ok) break;
            tc_fence_after();
            issue_unit(d_tmem, j > 0 ? 1u : 0u);
            advance();
            issue_unit(d_tmem, 1u);
            advance();
            if (leader) {
              umma_commit(&hdr->done[i & (kDoneRing - 1)]);
              umma_commit(&hdr->done[(i + 1) & (kDoneRing - 1)]);
            }
            __syncwarp();
          }
        }
        for (; ok && j < len; ++j, ++i) {
          ok = __all_sync(0xffffffffu, mbar_wait(&hdr->ready[s], sph));
          if (!ok) break;
          tc_fence_after();
          issue_unit(d_tmem, j > 0 ? 1u : 0u);
          advance();
          if (leader) umma_commit(&hdr->done[i & (kDoneRing - 1)]);
          __syncwarp();
        }
        if (!ok) break;
        if (leader) umma_commit(&hdr->acc_full[b]);  // the segment's accumulator is complete
        __syncwarp();
        ++seg;
        kb = 0;
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------ weight unpack (4-bit weights only)
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    uint8_t* lut = reinterpret_cast<uint8_t*>(hdr) + p.lut_off;
    if (CB) {
      // The decode table: for each e4m3 scale byte b (two per thread), the 16
      // int8 weights of the codebook levels under that scale.
      const int ut = threadIdx.x - 64;  // 0 .. 127
      for (int r = 0; r < 2; ++r) {
        const uint32_t b = static_cast<uint32_t>(ut + 128 * r);
        const float sc = e4m3_to_float(b);
        for (int w = 0; w < 4; ++w) {
          uint32_t q = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            q |= (static_cast<uint32_t>(decode_level(__ldg(p.codebook + 4 * w + i), sc)) & 0xFFu) << (8 * i);
          *reinterpret_cast<uint32_t*>(lut + 16 * b + 4 * w) = q;
        }
      }
      named_barrier(2, 128);  // the four unpack warps
    }
    for (int it = 0, s = 0, ph = 0, a = 0; !W8 && it < total; ++it) {
      bool w = mbar_wait(&hdr->wfull[s], ph & 1);
      if (w && it >= nas) {
        const int u = it - nas;  // the unit that last used A slot a
        w = mbar_wait(&hdr->done[u % kDoneRing], (u / kDoneRing) & 1);
      }
      if (!__all_sync(0xffffffffu, w)) break;  // tcgen05.st below is warp-collective
      tc_fence_after();
      const uint32_t taddr = tmem + lane_base + a_col0 + 64u * static_cast<uint32_t>(a);
      if (CB)
        decode_row_to_tmem(smem + s * stage_bytes, smem + s * stage_bytes + kWTileBytes + 16 * row, lut, row, taddr);
      else
        unpack_row_to_tmem(smem + s * stage_bytes, row, taddr);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hdr->ready[s]);
      if (++s == ns) {
        s = 0;
        ++ph;
      }
      if (++a == nas) a = 0;
    }
  } else {
    // ------------------------------------------------ epilogue
    const int quad = warp & 3;             // tensor-memory lane quadrant (warp id mod 4)
    const int half = (warp - 6) >> 2;      // which chunks of the accumulator this warp drains
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int et = threadIdx.x - 192;  // 0 .. kEpiThreads - 1
    pdl_wait();  // s_a comes from the preceding kernel
    int seg = 0, tile = tile0, kb = kb0;
    for (int i = 0; i < total; ++i, unit_next(p, tile, kb)) {
      if (!(i == total - 1 || kb == kbn - 1)) continue;
      // Segment `seg` (this CTA's units of `tile`) ends at unit i.
      const int b = seg & 1;
      const int m0 = x_row(tile), n0 = w_row(tile);
      const int n = n0 + row;
      // The segment's scales and bias are fetched before its accumulator is
      // waited for, so their latency hides behind the MMAs.
      float* sa = sa_buf + 192 * b;
      float sw = 0.0f, bv = 0.0f;
      if (p.splits == 1) {
        if (SINK != static_cast<int>(GemmSink::kS32))
          for (int c = et; c < BT; c += kEpiThreads)
            sa[c] = (m0 + c < p.M) ? __ldg(p.s_a + (m0 + c) * p.sa_stride) : 0.0f;
        sw = (SINK != static_cast<int>(GemmSink::kS32) && n < p.N) ? __ldg(p.s_w + n * p.sw_stride) : 0.0f;
        bv = (p.bias && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
        named_barrier(1, kEpiThreads);  // s_a staged; all warps are done with segment seg - 2
      }
      // On a failed wait the warp skips the segment's data but keeps taking
      // part in the named and cluster barriers, so no peer is left waiting.
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&hdr->acc_full[b], (seg / 2) & 1));
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(b * p.acc_stride);
      if (p.splits == 1) {
        // 32-column chunks (the accumulator stride is BT rounded up to 32, so
        // the last chunk's extra columns exist and are simply not stored).
        for (int c = 32 * half; ok && c < BT; c += 64) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(acc + static_cast<uint32_t>(c), v);
          tmem_wait_ld();
          const int count = min(min(32, BT - c), p.M - (m0 + c));
          if (n < p.N && count > 0) store_chunk<SINK, PLAIN>(p, m0 + c, n, v, sa + c, sw, bv, count);
        }
      } else {
        // Push the partial tile to its owners: 4-token group g belongs to CTA
        // g % S of the cluster, which keeps it in red[source rank][g / S][row]
        // (16 bytes).  The stores become visible at the cluster barrier.
        const int S = p.splits;
        const int ngl = (BT / 4 + S - 1) / S;
        const uint32_t me = cluster_ctarank();
        const uint32_t red_base = smem_u32(red);
        for (int c = 16 * half; c < BT; c += 32) {
          uint32_t v[16];
          if (ok) {
            tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c), v);
            tmem_wait_ld();
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int g = c / 4 + q;
            const int4 w = ok ? make_int4(static_cast<int32_t>(v[4 * q]), static_cast<int32_t>(v[4 * q + 1]),
                                          static_cast<int32_t>(v[4 * q + 2]), static_cast<int32_t>(v[4 * q + 3]))
                              : make_int4(0, 0, 0, 0);
            const uint32_t slot = ((me * ngl + static_cast<uint32_t>(g / S)) * kRows + row) * 16u;
            st_shared_cluster_v4(map_shared_rank(red_base + slot, static_cast<uint32_t>(g % S)), w);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hdr->acc_empty[b]);
      ++seg;
    }
  }

  if (p.splits > 1) {
    // Scales and bias of this CTA's rows and channels, fetched before the
    // cluster barrier (tokens into sa_buf, made visible by the barrier).
    float sw_red = 0.0f, bv_red = 0.0f;
    if (warp >= 6) {
      const int n = tile_ni(p, tile0) * kRows + (warp & 3) * 32 + lane;
      const int m0 = tile_mi(p, tile0) * BT;
      if (SINK != static_cast<int>(GemmSink::kS32)) {
        for (int c = threadIdx.x - 192; c < BT; c += kEpiThreads)
          sa_buf[c] = (m0 + c < p.M) ? __ldg(p.s_a + (m0 + c) * p.sa_stride) : 0.0f;
        sw_red = n < p.N ? __ldg(p.s_w + n * p.sw_stride) : 0.0f;
      }
      bv_red = (p.bias && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
    }
    __syncwarp();    // the cluster barrier below is .aligned: reconverge first
    cluster_sync();  // every partial has reached its owner's shared memory
    if (warp >= 6) {
      // Sum, from this CTA's own shared memory, the S partials of the groups
      // it owns and store them.  No CTA touches another's shared memory after
      // the barrier, so none has to wait before exiting.
      const int S = p.splits;
      const int ngl = (BT / 4 + S - 1) / S;
      const int half = (warp - 6) >> 2;
      const int row = (warp & 3) * 32 + lane;
      const int n = tile_ni(p, tile0) * kRows + row;
      const int m0 = tile_mi(p, tile0) * BT;
      const int rank = static_cast<int>(cluster_ctarank());
      const float sw = sw_red, bv = bv_red;
      const int4* red4 = reinterpret_cast<const int4*>(red);
      for (int gl = half; gl < ngl; gl += 2) {
        const int g = gl * S + rank;
        if (g >= BT / 4 || m0 + 4 * g >= p.M || n >= p.N) continue;
        int4 sum = make_int4(0, 0, 0, 0);
        for (int j = 0; j < S; ++j) {
          const int4 v = red4[(j * ngl + gl) * kRows + row];
          sum.x += v.x;
          sum.y += v.y;
          sum.z += v.z;
          sum.w += v.w;
        }
        const int32_t sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = m0 + 4 * g + q;
          if (m < p.M) {
            const float sa = SINK != static_cast<int>(GemmSink::kS32) ? sa_buf[m - m0] : 0.0f;
            store_output<SINK, PLAIN>(p, m, n, sv[q], sa, sw, bv);
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512u);
  }
}

// ---------------------------------------------------------------- host side

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

// 2-D uint8 tensor [rows, cols] (row stride = cols bytes), box [box_rows, box_cols].
bool make_map_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows,
                 uint32_t box_cols, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int SINK, int WK>
cudaError_t launch_sink(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& ts, const PParams& prm,
                        const GemmTiling& t, cudaStream_t stream) {
  static std::atomic<int> cache[64];  // static storage: zero-initialised
  const void* kfn = reinterpret_cast<const void*>(w4a4_tc_gemm_kernel<SINK, WK>);
  cudaError_t e = ensure_dynamic_smem(kfn, t.smem_bytes, cache);
  if (e != cudaSuccess) return note_cuda(e, "w4a4_gemm: dynamic shared memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(t.grid, 1, 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(t.smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int nattr = 0;
  attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[nattr].val.programmaticStreamSerializationAllowed = 1;
  ++nattr;
  if (t.splits > 1) {
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = static_cast<unsigned>(t.splits);
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr].val.clusterDim.z = 1;
    ++nattr;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  return note_cuda(cudaLaunchKernelEx(&cfg, w4a4_tc_gemm_kernel<SINK, WK>, tw, tx, ts, prm), "w4a4_gemm: launch");
}

// Clusters of S CTAs (one CTA per SM) that can be resident at once on the
// current device; a conservative estimate when it cannot be queried.
int max_active_clusters(int S, int num_sms) {
  static std::atomic<int> cache[64][9];  // clusters per device and size (0: not yet queried)
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64 || S < 1 || S > 8) return num_sms / (2 * S);
  if (cache[dev][S].load() > 0) return cache[dev][S].load();
  static std::atomic<int> smem_cache[64];
  const int smem = 200 * 1024;
  const void* kfn = reinterpret_cast<const void*>(w4a4_tc_gemm_kernel<0, kW4>);
  int n = 0;
  if (ensure_dynamic_smem(kfn, smem, smem_cache) == cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(S * 64), 1, 1);
    cfg.blockDim = dim3(kPThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(S);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, w4a4_tc_gemm_kernel<0, kW4>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();  // a failed query is not an error of the caller
  if (n <= 0) n = num_sms / (2 * S);
  cache[dev][S].store(n);
  return n;
}

// Estimated cycles of the whole-tile schedule for a token tile of BT: rounds
// of tiles per SM x units x the slower of the MMA (4 * BT cycles per 256-K
// unit at 8192 int8 MACs/clk) and the unit's operand delivery into shared
// memory plus the unit's fixed costs, fitted to measured runs of this kernel
// as about 700 + 3.2 * BT cycles (the BT-dependent part is the BT x 256
// activation bytes); with int8 weights the weight tile is twice as large.
long persistent_cost(int M, int N, int K, int BT, int num_sms, int wk) {
  const bool w8 = wk == kWInt8;
  const long tiles = static_cast<long>((M + BT - 1) / BT) * ((N + kRows - 1) / kRows);
  const long rounds = (tiles + num_sms - 1) / num_sms;
  const long mma = 4L * BT;
  const long data = (w8 ? 1030L : 700L) + (32L * BT) / 10;
  return rounds * (K / kKB) * (mma > data ? mma : data);
}

}  // namespace

namespace {

// Bytes of the split-K receive buffer: S partials of ceil(BT / 4 / S) 4-token
// groups x 128 rows x 16 bytes.
int red_bytes(int BT, int S) { return S > 1 ? S * ((BT / 4 + S - 1) / S) * kRows * 16 : 0; }

// Weight bytes of one unit's stage for a weight kind.
int weight_stage_bytes(int wk) {
  return wk == kWInt8 ? 2 * kWTileBytes : (wk == kWCodebook ? kWTileBytes + kSRelTileBytes : kWTileBytes);
}

// Stages of BT-token units that fit the shared memory of one CTA next to the
// header (1 KB), the s_a staging (1.5 KB), the split-K buffer and (codebook
// weights) the 4 KB decode table, and the dynamic shared memory for them
// (padded so that one CTA, which owns all of tensor memory, occupies an SM).
void set_stages(GemmTiling& t, int wk) {
  const int stage = weight_stage_bytes(wk) + t.BT * kKB;
  const int rb = red_bytes(t.BT, t.splits);
  const int lut = wk == kWCodebook ? kLutBytes : 0;
  int ns = (220 * 1024 - 4096 - rb - lut) / stage;
  if (ns > kMaxStages) ns = kMaxStages;
  t.nstages = ns;
  t.smem_bytes = 1024 + ns * stage + 2560 + rb + lut;
  if (t.smem_bytes < 120 * 1024) t.smem_bytes = 120 * 1024;
  // Tensor memory: two accumulators of BT (rounded up to 32) columns, then
  // 64-column A slots in the rest of the 512.
  t.acc_stride = (t.BT + 31) / 32 * 32;
  t.a_slots = (512 - 2 * t.acc_stride) / 64;
  if (t.a_slots > kMaxASlots) t.a_slots = kMaxASlots;
}

}  // namespace

GemmTiling choose_tiling(int M, int N, int K, int num_sms, int wk) {
  GemmTiling t{};
  const int kbn = K / kKB;
  const int G = num_sms < kMaxGemmGrid ? num_sms : kMaxGemmGrid;
  t.n_tiles = (N + kRows - 1) / kRows;
  t.splits = 1;
  // Large M: whole tiles, with the token tile BT (multiple of 16, <= 192) of
  // the lowest estimated cost, when it yields at least half as many tiles as
  // SMs.
  if (M > 128) {
    int best_bt = 0;
    long best = -1;
    for (int bt = 192; bt >= 64; bt -= 16) {
      const long tiles = static_cast<long>((M + bt - 1) / bt) * t.n_tiles;
      if (2 * tiles < G) continue;
      const long c = persistent_cost(M, N, K, bt, G, wk);
      if (best < 0 || c < best) {
        best = c;
        best_bt = bt;
      }
    }
    if (best_bt > 0) {
      t.BT = best_bt;
      t.m_tiles = (M + best_bt - 1) / best_bt;
      const int tiles = t.m_tiles * t.n_tiles;
      t.grid = tiles < G ? tiles : G;
      // Channel tiles fastest when the activation operand (M*K bytes) is too
      // large to stay in L2 from round to round (above 48 MB; the L2 is 126
      // MB) and all the weights fit comfortably (at most 48 MB): a round then
      // shares its activation rows and the weights stay resident, and the
      // activations are read from DRAM once instead of once per round
      // (measured on 8704 x 12288 x 3072: 865 -> 126 MB of DRAM reads per
      // launch).  Smaller activation operands stay in L2 either way, and the
      // token-tile-fastest order measured a few percent faster on them.
      const double act_bytes = static_cast<double>(M) * K;
      const double w_bytes = static_cast<double>(N) * K / (wk == kWInt8 ? 1.0 : 2.0);
      const double l2_share = 48.0 * (1 << 20);
      t.n_fast = (act_bytes > l2_share && w_bytes <= l2_share) ? 1 : 0;
      set_stages(t, wk);
      return t;
    }
  }
  // Small M (or few tiles): tiles of BT = M rounded up to 16 (at most 128)
  // tokens, K split over a cluster of S CTAs when that is estimated faster:
  // per wave of CTAs, its start-up (kWaveSec: first loads in flight) plus its
  // units per CTA x kUnitSec, and kSplitSec for the exchange of partial tiles
  // when S > 1 (constants measured on B200).
  int bt = M <= 128 ? ((M + 15) / 16) * 16 : 128;
  if (bt < 16) bt = 16;
  t.BT = bt;
  t.m_tiles = (M + bt - 1) / bt;
  const int tiles = t.m_tiles * t.n_tiles;
  constexpr double kUnitSec = 0.5e-6, kSplitSec = 1.0e-6, kWaveSec = 3.0e-6;
  double best = 0;
  for (int S = 1; S <= 8; S *= 2) {
    if (S > kbn) break;
    const int conc = S == 1 ? G : max_active_clusters(S, num_sms);  // tiles in flight at once
    if (conc < 1) continue;
    const int waves = (tiles + conc - 1) / conc;
    const double c = waves * (kWaveSec + ((kbn + S - 1) / S) * kUnitSec) + (S > 1 ? kSplitSec : 0.0);
    if (S == 1 || c < best * 0.999) {
      best = c;
      t.splits = S;
    }
  }
  t.grid = t.splits > 1 ? tiles * t.splits : (tiles < G ? tiles : G);
  set_stages(t, wk);
  return t;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& a, GemmSink sink, const GemmTiling& t, cudaStream_t stream) {
  CUtensorMap tw, tx, ts;
  const bool w8 = a.wkind == kWInt8;
  if (a.wkind < kW4 || a.wkind > kWCodebook || (a.wkind == kWCodebook && (!a.s_rel || !a.codebook)))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: weight kind");
  if (!make_map_u8(&tw, a.Wq, static_cast<uint64_t>(a.N), static_cast<uint64_t>(w8 ? a.K : a.K / 2), kRows,
                   w8 ? kXBox : kKB / 2, CU_TENSOR_MAP_SWIZZLE_128B))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: weight tensor map");
  // Group scales [N, K/16]: one 16-byte row piece per output channel and unit.
  ts = tw;
  if (a.wkind == kWCodebook &&
      !make_map_u8(&ts, a.s_rel, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K / 16), kRows, kKB / 16,
                   CU_TENSOR_MAP_SWIZZLE_NONE))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: group-scale tensor map");
  if (!make_map_u8(&tx, a.xs8, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K),
                   static_cast<uint32_t>(t.BT), kXBox, CU_TENSOR_MAP_SWIZZLE_128B))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: activation tensor map");
  if (t.grid < 1 || (t.splits == 1 && t.grid > kMaxGemmGrid) || t.splits < 1 || t.splits > 8 ||
      t.splits > a.K / kKB || t.a_slots < 2 || t.nstages < 1 || t.nstages > kMaxStages)
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: tiling");
  PParams pp{};
  pp.s_a = a.s_a;
  pp.s_w = a.s_w;
  pp.bias = a.bias;
  pp.out = a.out;
  pp.M = a.M;
  pp.N = a.N;
  pp.K = a.K;
  pp.BT = t.BT;
  pp.m_tiles = t.m_tiles;
  pp.n_tiles = t.n_tiles;
  pp.num_tiles = t.m_tiles * t.n_tiles;
  pp.n_fast = t.n_fast;
  pp.nstages = t.nstages;
  pp.kbn = a.K / kKB;
  pp.acc_stride = t.acc_stride;
  pp.a_slots = t.a_slots;
  pp.splits = t.splits;
  pp.pair = (t.BT <= 128 && (w8 || t.a_slots >= 4) && t.nstages >= 4) ? 1 : 0;
  pp.sa_stride = a.sa_stride;
  pp.sw_stride = a.sw_stride;
  pp.codebook = a.codebook;
  pp.lut_off = 2560 + red_bytes(t.BT, t.splits);
  if (a.wkind == kWCodebook && t.smem_bytes < 1024 + t.nstages * (weight_stage_bytes(kWCodebook) + t.BT * kKB) +
                                                   pp.lut_off + kLutBytes)
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: tiling");
  cudaError_t e;
  if (w8) {
    switch (sink) {
      case GemmSink::kBF16: e = launch_sink<0, kWInt8>(tw, tx, ts, pp, t, stream); break;
      case GemmSink::kF32: e = launch_sink<1, kWInt8>(tw, tx, ts, pp, t, stream); break;
      default: e = launch_sink<2, kWInt8>(tw, tx, ts, pp, t, stream); break;
    }
  } else if (a.wkind == kWCodebook) {
    switch (sink) {
      case GemmSink::kBF16: e = launch_sink<0, kWCodebook>(tw, tx, ts, pp, t, stream); break;
      case GemmSink::kF32: e = launch_sink<1, kWCodebook>(tw, tx, ts, pp, t, stream); break;
      default: e = launch_sink<2, kWCodebook>(tw, tx, ts, pp, t, stream); break;
    }
  } else {
    switch (sink) {
      case GemmSink::kBF16: e = launch_sink<0, kW4>(tw, tx, ts, pp, t, stream); break;
      case GemmSink::kF32: e = launch_sink<1, kW4>(tw, tx, ts, pp, t, stream); break;
      default: e = launch_sink<2, kW4>(tw, tx, ts, pp, t, stream); break;
    }
  }
  count_dispatch(t.splits > 1 ? 3 : 2);
  return e;
}

}  // namespace convrot
