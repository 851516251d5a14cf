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
// Work is cut into units of one 128-wide K block of one output tile; see
// the kernel below for the two schedules (whole tiles for large M, stream-K
// for small M) and the exact cross-CTA reduction of split tiles.
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

// One output element from the MMA sum (16 * acc): scales and bias already
// loaded by the caller.
template <int SINK, class P>
__device__ __forceinline__ void store_output(const P& p, int m, int n, int32_t dsum, float sa, float sw,
                                             float bv) {
  const int32_t acc = dsum >> 4;  // the weights entered the MMA as 16 * q_w
  const size_t idx = static_cast<size_t>(m) * p.N + n;
  if (SINK == static_cast<int>(GemmSink::kS32)) {
    static_cast<int32_t*>(p.out)[idx] = acc;
    return;
  }
  float y = __fmul_rn(__fmul_rn(__int2float_rn(acc), sa), sw);
  if (p.bias) y = __fadd_rn(y, bv);
  if (SINK == static_cast<int>(GemmSink::kF32)) {
    static_cast<float*>(p.out)[idx] = y;
  } else {
    static_cast<uint16_t*>(p.out)[idx] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
  }
}

// ---------------------------------------------------------------- the kernel
//
// One CTA per SM walks its list of units; a unit is one 128-wide K block of
// one output tile (BT tokens x 128 output channels).  Two schedules:
//   * tiles (large M): CTA c takes the whole tiles c, c + grid, c + 2 grid ...
//     (neighbouring CTAs share activation and weight tiles in L2);
//   * stream-K (small M, fewer tiles than SMs): the units of all tiles, in
//     tile-major order, are cut into `grid` contiguous ranges of equal size,
//     so every SM streams the same share of the weights.
// Consecutive units of one tile form a segment, summed in one tensor-memory
// accumulator.  A segment that covers all K blocks of its tile is stored
// directly.  Otherwise (stream-K only; at most the first and the last
// segment of a CTA) its int32 partial tile goes to the CTA's slot in global
// memory and the CTA bumps the tile's arrival counter; the CTA that arrives
// last adds the other contributors' slots to its own accumulator, stores the
// tile and resets the counter to zero for the next launch.  Integer addition
// is exact, so no output bit depends on the order of arrival.
//   warp 0      TMA producer (ring of `nstages` shared-memory stages)
//   warp 1      TMEM allocation (all 512 columns) and the MMA-issuing thread
//   warps 2..5  weight unpack into 64-column A slots of tensor memory
//   warps 6..9  epilogue, draining one of two accumulators while the MMA
//               fills the other
// The MMA thread commits once per unit, to done[unit % 32]; that one
// completion frees both the unit's shared-memory stage (for the TMA producer)
// and its A slot (for the unpack warps).  A unit of 256 K values is 8 MMAs,
// so the waits and the commit of the issuing thread are spread over 8.
constexpr int kPThreads = 320;

struct PParams {
  const float* s_a;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int M, N, K;
  int BT, m_tiles, num_tiles, nstages, kbn;
  int acc_stride;   // tensor-memory columns per accumulator (BT rounded up to 32)
  int a_slots;      // A slots of 64 columns after the two accumulators
  int stream_k;     // 0: whole tiles round-robin, 1: stream-K ranges
  int units;        // num_tiles * kbn
  uint32_t* ctr;    // [num_tiles] arrival counters (stream-K), zero between launches
  int32_t* slots;   // [2 * grid][BT][128] partial tiles (stream-K)
};

struct PHeader {
  uint64_t full[kMaxStages];
  uint64_t done[kDoneRing];     // unit i's MMAs have completed (its stage and A slot are free)
  uint64_t a_full[kMaxASlots];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
  uint32_t last_flag;
};

// First unit of CTA c under stream-K (c in [0, grid]; strictly increasing
// because grid <= units).
__device__ __forceinline__ int sk_begin(const PParams& p, int c) {
  return static_cast<int>((static_cast<long long>(c) * p.units) / static_cast<int>(gridDim.x));
}

// The CTA whose stream-K range holds unit u.
__device__ __forceinline__ int sk_owner(const PParams& p, int u) {
  const int G = static_cast<int>(gridDim.x);
  int c = static_cast<int>((static_cast<long long>(u) * G) / p.units);
  while (c + 1 < G && sk_begin(p, c + 1) <= u) ++c;
  while (c > 0 && sk_begin(p, c) > u) --c;
  return c;
}

// Number of units of this CTA.
__device__ __forceinline__ int unit_count(const PParams& p) {
  if (p.stream_k) return sk_begin(p, blockIdx.x + 1) - sk_begin(p, blockIdx.x);
  const int my_tiles =
      (p.num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
  return my_tiles * p.kbn;
}

// Tile and K block of this CTA's first unit, and the step to the next unit.
__device__ __forceinline__ void unit_first(const PParams& p, int u0, int& tile, int& kb) {
  if (p.stream_k) {
    tile = u0 / p.kbn;
    kb = u0 - tile * p.kbn;
  } else {
    tile = static_cast<int>(blockIdx.x);
    kb = 0;
  }
}
__device__ __forceinline__ void unit_next(const PParams& p, int& tile, int& kb) {
  if (++kb == p.kbn) {
    kb = 0;
    tile += p.stream_k ? 1 : static_cast<int>(gridDim.x);
  }
}

// Partial-tile slot layout: 16-token chunks, each [128 rows][16 tokens], so
// a thread (one row) moves 64 contiguous bytes per chunk.
__device__ __forceinline__ int32_t* slot_chunk(int32_t* slot, int c, int row) {
  return slot + (c >> 4) * (kRows * 16) + row * 16;
}

template <int SINK>
__global__ void __launch_bounds__(kPThreads, 1)
    w4a4_tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ PParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int BT = p.BT;
  const int ns = p.nstages;
  const int stage_bytes = kWTileBytes + BT * kKB;
  const int nas = p.a_slots;
  const uint32_t a_col0 = 2u * static_cast<uint32_t>(p.acc_stride);
  PHeader* hdr = reinterpret_cast<PHeader*>(smem + ns * stage_bytes);
  float* sa_buf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(hdr) + 1024);  // [2][192]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kbn = p.kbn;
  const int u0 = p.stream_k ? sk_begin(p, blockIdx.x) : 0;
  const int total = unit_count(p);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) mbar_init(&hdr->full[s], 1);
    for (int r = 0; r < kDoneRing; ++r) mbar_init(&hdr->done[r], 1);  // one MMA commit
    for (int a = 0; a < nas; ++a) mbar_init(&hdr->a_full[a], 4);      // one arrive per unpack warp
    for (int b = 0; b < 2; ++b) {
      mbar_init(&hdr->acc_full[b], 1);
      mbar_init(&hdr->acc_empty[b], 4);  // one arrive per epilogue warp
    }
    fence_mbarrier_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
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
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(stage_bytes);
      // Weight tiles of the first stages do not depend on the preceding
      // prologue kernel: request them before waiting for it.
      const int prime = total < ns ? total : ns;
      int tile, kb;
      unit_first(p, u0, tile, kb);
      for (int i = 0; i < prime; ++i, unit_next(p, tile, kb)) {
        mbar_arrive_expect_tx(&hdr->full[i], bytes);
        tma_load_2d(smem + i * stage_bytes, &tm_w, &hdr->full[i], kb * (kKB / 2), (tile / p.m_tiles) * kRows);
      }
      pdl_wait();
      unit_first(p, u0, tile, kb);
      for (int i = 0; i < prime; ++i, unit_next(p, tile, kb)) {
        uint8_t* xs = smem + i * stage_bytes + kWTileBytes;
        tma_load_2d(xs, &tm_x, &hdr->full[i], kb * kKB, (tile % p.m_tiles) * BT);
        tma_load_2d(xs + BT * kXBox, &tm_x, &hdr->full[i], kb * kKB + kXBox, (tile % p.m_tiles) * BT);
      }
      int it = prime, s = prime % ns;  // stage of unit `it`
      for (; it < total; ++it, unit_next(p, tile, kb)) {
        const int w = it - ns;  // the unit that last used stage s
        if (!mbar_wait(&hdr->done[w % kDoneRing], (w / kDoneRing) & 1)) break;
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&hdr->full[s], bytes);
        tma_load_2d(st, &tm_w, &hdr->full[s], kb * (kKB / 2), (tile / p.m_tiles) * kRows);
        tma_load_2d(st + kWTileBytes, &tm_x, &hdr->full[s], kb * kKB, (tile % p.m_tiles) * BT);
        tma_load_2d(st + kWTileBytes + BT * kXBox, &tm_x, &hdr->full[s], kb * kKB + kXBox, (tile % p.m_tiles) * BT);
        if (++s == ns) s = 0;
      }
      // Drain: every issued load has landed before the block may exit.
      for (int i = (it > ns ? it - ns : 0); i < it; ++i) mbar_wait(&hdr->full[i % ns], (i / ns) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(kRows, BT, /*a_signed=*/true, /*b_signed=*/true);
      int seg = 0, tile, kb, s = 0, ph = 0, a = 0, aph = 0;
      bool first = true;
      uint32_t d_tmem = tmem;
      unit_first(p, u0, tile, kb);
      for (int i = 0; i < total; ++i, unit_next(p, tile, kb)) {
        if (i == 0 || kb == 0) {  // a segment starts: take accumulator seg & 1
          const int b = seg & 1;
          if (seg >= 2 && !mbar_wait(&hdr->acc_empty[b], ((seg / 2) - 1) & 1)) break;
          tc_fence_after();
          d_tmem = tmem + static_cast<uint32_t>(b * p.acc_stride);
          first = true;
        }
        if (!mbar_wait(&hdr->full[s], ph & 1) || !mbar_wait(&hdr->a_full[a], aph & 1)) break;
        tc_fence_after();
        const uint64_t bdesc0 = umma_desc_k_sw128(smem_u32(smem + s * stage_bytes + kWTileBytes));
        const uint64_t bdesc1 = umma_desc_k_sw128(smem_u32(smem + s * stage_bytes + kWTileBytes + BT * kXBox));
        const uint32_t a_tmem = tmem + a_col0 + 64u * static_cast<uint32_t>(a);
#pragma unroll
        for (int kk = 0; kk < kKB / 32; ++kk)
          umma_i8_ts(d_tmem, a_tmem + 8 * kk, (kk < 4 ? bdesc0 : bdesc1) + 2 * (kk & 3), idesc,
                     (first && kk == 0) ? 0u : 1u);
        first = false;
        umma_commit(&hdr->done[i % kDoneRing]);
        if (++a == nas) {
          a = 0;
          ++aph;
        }
        if (i == total - 1 || kb == kbn - 1) {  // the segment ends
          umma_commit(&hdr->acc_full[seg & 1]);
          ++seg;
        }
        if (++s == ns) {
          s = 0;
          ++ph;
        }
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------ weight unpack
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    for (int it = 0, s = 0, ph = 0, a = 0; it < total; ++it) {
      bool w = mbar_wait(&hdr->full[s], ph & 1);
      if (w && it >= nas) {
        const int u = it - nas;  // the unit that last used A slot a
        w = mbar_wait(&hdr->done[u % kDoneRing], (u / kDoneRing) & 1);
      }
      if (!__all_sync(0xffffffffu, w)) break;  // tcgen05.st below is warp-collective
      tc_fence_after();
      unpack_row_to_tmem(smem + s * stage_bytes, row, tmem + lane_base + a_col0 + 64u * static_cast<uint32_t>(a));
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hdr->a_full[a]);
      if (++s == ns) {
        s = 0;
        ++ph;
      }
      if (++a == nas) a = 0;
    }
  } else {
    // ------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int et = threadIdx.x - 192;  // 0..127
    pdl_wait();  // s_a and the zeroed counters come from the preceding kernel
    int seg = 0, seg_kb0 = 0, tile, kb;
    unit_first(p, u0, tile, kb);
    for (int i = 0; i < total; ++i, unit_next(p, tile, kb)) {
      if (i == 0 || kb == 0) seg_kb0 = kb;
      if (!(i == total - 1 || kb == kbn - 1)) continue;
      // Segment `seg` (K blocks seg_kb0 .. kb of `tile`) ends at unit i.
      const int b = seg & 1;
      const bool whole = seg_kb0 == 0 && kb == kbn - 1;
      const int m0 = (tile % p.m_tiles) * BT, n0 = (tile / p.m_tiles) * kRows;
      float* sa = sa_buf + 192 * b;
      if (SINK != static_cast<int>(GemmSink::kS32))
        for (int c = et; c < BT; c += 128) sa[c] = (m0 + c < p.M) ? __ldg(p.s_a + m0 + c) : 0.0f;
      named_barrier(1, 128);  // s_a staged; all warps are done with segment seg - 2
      const int n = n0 + row;
      const float sw = (SINK != static_cast<int>(GemmSink::kS32) && n < p.N) ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (p.bias && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
      // On a failed wait the warp skips the segment's data but keeps taking
      // part in the named barriers and the counter protocol, so no peer (in
      // this CTA or another) is left waiting and the counters stay balanced.
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&hdr->acc_full[b], (seg / 2) & 1));
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(b * p.acc_stride);
      if (whole) {
        for (int c = 0; ok && c < BT; c += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c), v);
          tmem_wait_ld();
          if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + c + j;
              if (m < p.M) store_output<SINK>(p, m, n, static_cast<int32_t>(v[j]), sa[c + j], sw, bv);
            }
          }
        }
      } else {
        // Partial tile: publish it, then count the arrival.
        int32_t* mine = p.slots + static_cast<size_t>(2 * blockIdx.x + (seg == 0 ? 0 : 1)) * BT * kRows;
        for (int c = 0; ok && c < BT; c += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(c), v);
          tmem_wait_ld();
          int4* dst = reinterpret_cast<int4*>(slot_chunk(mine, c, row));
#pragma unroll
          for (int r = 0; r < 4; ++r)
            dst[r] = make_int4(static_cast<int32_t>(v[4 * r]), static_cast<int32_t>(v[4 * r + 1]),
                               static_cast<int32_t>(v[4 * r + 2]), static_cast<int32_t>(v[4 * r + 3]));
        }
        __threadfence();        // this thread's slot stores precede the arrival below
        named_barrier(1, 128);  // ... for all 128 threads
        const int c_first = sk_owner(p, tile * kbn), c_last = sk_owner(p, tile * kbn + kbn - 1);
        if (et == 0)
          hdr->last_flag = atomicAdd(p.ctr + tile, 1u) == static_cast<uint32_t>(c_last - c_first) ? 1u : 0u;
        named_barrier(1, 128);
        if (hdr->last_flag) {
          __threadfence();  // every other contributor's slot is visible now
          // 32 tokens at a time: the own accumulator from tensor memory plus
          // the other contributors' slots.
          for (int h = 0; ok && h < BT; h += 32) {
            int32_t sum[32];
#pragma unroll
            for (int q = 0; q < 2; ++q) {
              if (h + 16 * q < BT) {  // uniform across the warp (tcgen05.ld is collective)
                uint32_t v[16];
                tmem_ld_32x32b_x16(acc + static_cast<uint32_t>(h + 16 * q), v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 16; ++j) sum[16 * q + j] = static_cast<int32_t>(v[j]);
              }
            }
            // Two contributors per round: 16 independent 16-byte loads in flight.
            for (int cc = c_first;;) {
              int sl[2] = {-1, -1};
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (cc == static_cast<int>(blockIdx.x)) ++cc;
                // Tile `tile` is CTA cc's first segment when cc's range
                // starts inside it, else its last.
                if (cc <= c_last) sl[e] = 2 * cc + (sk_begin(p, cc) >= tile * kbn ? 0 : 1), ++cc;
              }
              if (sl[0] < 0) break;
              int4 v[2][8];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (sl[e] < 0) continue;
                int32_t* other = p.slots + static_cast<size_t>(sl[e]) * BT * kRows;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                  if (h + 16 * q < BT) {
                    const int4* src = reinterpret_cast<const int4*>(slot_chunk(other, h + 16 * q, row));
#pragma unroll
                    for (int r = 0; r < 4; ++r) v[e][4 * q + r] = __ldcg(src + r);
                  }
                }
              }
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                if (sl[e] < 0) continue;
#pragma unroll
                for (int q = 0; q < 2; ++q) {
                  if (h + 16 * q < BT) {
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                      sum[16 * q + 4 * r] += v[e][4 * q + r].x;
                      sum[16 * q + 4 * r + 1] += v[e][4 * q + r].y;
                      sum[16 * q + 4 * r + 2] += v[e][4 * q + r].z;
                      sum[16 * q + 4 * r + 3] += v[e][4 * q + r].w;
                    }
                  }
                }
              }
            }
            if (n < p.N) {
#pragma unroll
              for (int j = 0; j < 32; ++j) {
                const int m = m0 + h + j;
                if (h + j < BT && m < p.M) store_output<SINK>(p, m, n, sum[j], sa[h + j], sw, bv);
              }
            }
          }
          if (et == 0) p.ctr[tile] = 0u;  // ready for the next launch
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hdr->acc_empty[b]);
      ++seg;
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

template <int SINK>
cudaError_t launch_sink(const CUtensorMap& tw, const CUtensorMap& tx, const PParams& prm, const GemmTiling& t,
                        cudaStream_t stream) {
  static int cache[64] = {0};
  const void* kfn = reinterpret_cast<const void*>(w4a4_tc_gemm_kernel<SINK>);
  cudaError_t e = ensure_dynamic_smem(kfn, t.smem_bytes, cache);
  if (e != cudaSuccess) return note_cuda(e, "w4a4_gemm: dynamic shared memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(t.grid, 1, 1);
  cfg.blockDim = dim3(kPThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(t.smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note_cuda(cudaLaunchKernelEx(&cfg, w4a4_tc_gemm_kernel<SINK>, tw, tx, prm), "w4a4_gemm: launch");
}

// Estimated cycles of the whole-tile schedule for a token tile of BT: rounds
// of tiles per SM x units x the slower of the MMA (4 * BT cycles per 256-K
// unit at 8192 int8 MACs/clk) and a per-unit floor of 640 cycles that every
// unit costs whatever BT is (issuing its 8 MMAs and commit, and the 16 KB
// weight tile fetched and unpacked into tensor memory).
long persistent_cost(int M, int N, int K, int BT, int num_sms) {
  const long tiles = static_cast<long>((M + BT - 1) / BT) * ((N + kRows - 1) / kRows);
  const long rounds = (tiles + num_sms - 1) / num_sms;
  const long per_unit = 4L * BT > 640 ? 4L * BT : 640;
  return rounds * (K / kKB) * per_unit;
}

}  // namespace

namespace {

// Stages of BT-token units that fit the shared memory of one CTA, and the
// dynamic shared memory for them (padded so that one CTA, which owns all of
// tensor memory, occupies an SM).
void set_stages(GemmTiling& t) {
  const int stage = kWTileBytes + t.BT * kKB;
  int ns = (220 * 1024 - 4096) / stage;
  if (ns > kMaxStages) ns = kMaxStages;
  t.nstages = ns;
  t.smem_bytes = 1024 + ns * stage + 1024 + 2 * 192 * 4;
  if (t.smem_bytes < 120 * 1024) t.smem_bytes = 120 * 1024;
  // Tensor memory: two accumulators of BT (rounded up to 32) columns, then
  // 64-column A slots in the rest of the 512.
  t.acc_stride = (t.BT + 31) / 32 * 32;
  t.a_slots = (512 - 2 * t.acc_stride) / 64;
  if (t.a_slots > kMaxASlots) t.a_slots = kMaxASlots;
}

}  // namespace

// Stream-K grid: the number of CTAs g (at most one per SM) with the lowest
// modelled time.  The weights stream at the lower of the HBM rate and what g
// SMs pull (kSmBps each); a split tile then costs its last CTA one round of
// L2 loads (kRoundSec) per 32 tokens for every two other contributors.
int streamk_grid(int units, int kbn, int BT, int max_grid) {
  constexpr double kHbmBps = 6.0e12, kSmBps = 150e9, kRoundSec = 0.4e-6;
  const double unit_w = kWTileBytes, unit_all = kWTileBytes + static_cast<double>(BT) * kKB;
  double best = 0;
  int best_g = 1;
  const int gmax = units < max_grid ? units : max_grid;
  for (int g = 1; g <= gmax; ++g) {
    const int most = (units + g - 1) / g, least = units / g;
    int parts = 1;  // contributors of the most split tile
    if (!(units % g == 0 && least % kbn == 0)) {
      parts = (kbn + least - 1) / least + 1;
      if (units % g == 0 && kbn % least == 0) parts = kbn / least;
    }
    const double t_stream = std::max(units * unit_w / kHbmBps, most * unit_all / kSmBps);
    const double t_red = ((parts - 1 + 1) / 2) * ((BT + 31) / 32) * kRoundSec;
    const double t = t_stream + t_red;
    if (g == 1 || t < best * 0.999) {
      best = t;
      best_g = g;
    }
  }
  return best_g;
}

size_t streamk_scratch_bytes(const GemmTiling& t) {
  if (!t.stream_k) return 0;
  return static_cast<size_t>(2 * kMaxGemmGrid) * static_cast<size_t>(t.BT) * kRows * sizeof(int32_t);
}

GemmTiling choose_tiling(int M, int N, int K, int num_sms) {
  GemmTiling t{};
  const int kbn = K / kKB;
  const int G = num_sms < kMaxGemmGrid ? num_sms : kMaxGemmGrid;
  t.n_tiles = (N + kRows - 1) / kRows;
  // Large M: whole tiles, with the token tile BT (multiple of 16, <= 192) of
  // the lowest estimated cost, when it yields at least half as many tiles as
  // SMs.
  if (M > 128) {
    int best_bt = 0;
    long best = -1;
    for (int bt = 192; bt >= 64; bt -= 16) {
      const long tiles = static_cast<long>((M + bt - 1) / bt) * t.n_tiles;
      if (2 * tiles < G) continue;
      const long c = persistent_cost(M, N, K, bt, G);
      if (best < 0 || c < best) {
        best = c;
        best_bt = bt;
      }
    }
    if (best_bt > 0) {
      t.stream_k = false;
      t.BT = best_bt;
      t.m_tiles = (M + best_bt - 1) / best_bt;
      t.units = t.m_tiles * t.n_tiles * kbn;
      const int tiles = t.m_tiles * t.n_tiles;
      t.grid = tiles < G ? tiles : G;
      set_stages(t);
      return t;
    }
  }
  // Small M (or few tiles): stream-K over tiles of BT = M rounded up to 16
  // (at most 128) tokens.
  int bt = M <= 128 ? ((M + 15) / 16) * 16 : 128;
  if (bt < 16) bt = 16;
  t.BT = bt;
  t.m_tiles = (M + bt - 1) / bt;
  const int tiles = t.m_tiles * t.n_tiles;
  t.units = tiles * kbn;
  if (tiles > kMaxSplitTiles) {
    // More tiles than counters (N > 128 * 1024): whole tiles balance anyway.
    t.stream_k = false;
    t.grid = tiles < G ? tiles : G;
  } else {
    t.stream_k = true;
    t.grid = streamk_grid(t.units, kbn, bt, G);
  }
  set_stages(t);
  return t;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& a, GemmSink sink, const GemmTiling& t, cudaStream_t stream) {
  CUtensorMap tw, tx;
  if (!make_map_u8(&tw, a.Wq, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K / 2), kRows, kKB / 2,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: weight tensor map");
  if (!make_map_u8(&tx, a.xs8, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), static_cast<uint32_t>(t.BT),
                   kXBox, CU_TENSOR_MAP_SWIZZLE_128B))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: activation tensor map");
  if (t.grid < 1 || t.grid > kMaxGemmGrid || (t.stream_k && (!a.ctr || !a.slots)) || t.a_slots < 2 ||
      t.nstages < 1 || t.nstages > kMaxStages)
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
  pp.num_tiles = t.m_tiles * t.n_tiles;
  pp.nstages = t.nstages;
  pp.kbn = a.K / kKB;
  pp.acc_stride = t.acc_stride;
  pp.a_slots = t.a_slots;
  pp.stream_k = t.stream_k ? 1 : 0;
  pp.units = t.units;
  pp.ctr = a.ctr;
  pp.slots = a.slots;
  cudaError_t e;
  switch (sink) {
    case GemmSink::kBF16: e = launch_sink<0>(tw, tx, pp, t, stream); break;
    case GemmSink::kF32: e = launch_sink<1>(tw, tx, pp, t, stream); break;
    default: e = launch_sink<2>(tw, tx, pp, t, stream); break;
  }
  count_dispatch(t.stream_k ? 3 : 2);
  return e;
}

}  // namespace convrot
