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
// Split-K (for small M) runs the K-slices of one output tile as a thread
// block cluster and adds the int32 partial tiles through distributed shared
// memory; the sum is exact and independent of order.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace convrot {

namespace {

constexpr int kThreads = 192;    // warp 0 TMA, warp 1 MMA, warps 2..5 unpack + epilogue
constexpr int kRows = 128;       // output channels per tile (MMA M)
constexpr int kKB = 128;         // K values per pipeline step
constexpr int kWTileBytes = kRows * kKB / 2;  // 8 KB packed weights per step
constexpr int kASlots = 2;       // tensor-memory A buffers (32 columns each)

struct Params {
  const float* s_a;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int M, N, K;
  int BT, splits, kb_total, kb_per_split, nstages, tmem_cols;
};

struct SharedHeader {
  uint64_t full[16];
  uint64_t empty[16];
  uint64_t a_full[kASlots];
  uint64_t a_empty[kASlots];
  uint64_t acc_full;
  uint32_t tmem_base;
};

__device__ __forceinline__ void unpack_row_to_tmem(const uint8_t* wstage, int row, uint32_t taddr) {
  // The weight tile landed with the 64-byte TMA swizzle: 16-byte chunk c of
  // row r sits at chunk c ^ ((r >> 1) & 3).
  uint32_t cols[32];
  const int sw = (row >> 1) & 3;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const uint4 v = *reinterpret_cast<const uint4*>(wstage + row * 64 + ((c ^ sw) << 4));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      cols[8 * c + 2 * j] = (w[j] << 4) & 0xF0F0F0F0u;
      cols[8 * c + 2 * j + 1] = w[j] & 0xF0F0F0F0u;
    }
  }
  tmem_st_32x32b_x32(taddr, cols);
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

template <int SINK>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_tc_gemm_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled stage tiles.
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int BT = p.BT;
  const int stage_bytes = kWTileBytes + BT * kKB;
  SharedHeader* hdr = reinterpret_cast<SharedHeader*>(smem + p.nstages * stage_bytes);
  float* sa_tile = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(hdr) + 1024);   // s_a of the BT tokens
  int32_t* red = reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(hdr) + 2048);  // split-K partials

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kRows;
  const int m0 = blockIdx.y * BT;
  // K blocks of this split: an even share [j*KB/S, (j+1)*KB/S), never empty
  // because S <= KB.
  const int split = blockIdx.z;
  const int kb0 = (split * p.kb_total) / p.splits;
  const int nkb = ((split + 1) * p.kb_total) / p.splits - kb0;
  const int ns = p.nstages;
  const uint32_t a_col0 = static_cast<uint32_t>(p.tmem_cols - 32 * kASlots);

  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&hdr->full[s], 1);
      mbar_init(&hdr->empty[s], 1 + 4);  // MMA commit + one arrive per unpack warp
    }
    for (int a = 0; a < kASlots; ++a) {
      mbar_init(&hdr->a_full[a], 4);
      mbar_init(&hdr->a_empty[a], 1);
    }
    mbar_init(&hdr->acc_full, 1);
    fence_mbarrier_init();
    prefetch_tmap(&tm_w);
    prefetch_tmap(&tm_x);
  }
  if (warp == 1) {
    tmem_alloc(&hdr->tmem_base, static_cast<uint32_t>(p.tmem_cols));
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
      // The weights do not depend on the preceding prologue kernel: the first
      // stages' weight tiles are requested before waiting for it.
      const int prime = nkb < ns ? nkb : ns;
      for (int i = 0; i < prime; ++i) {
        mbar_arrive_expect_tx(&hdr->full[i], bytes);
        tma_load_2d(smem + i * stage_bytes, &tm_w, &hdr->full[i], (kb0 + i) * (kKB / 2), n0);
      }
      pdl_wait();
      for (int i = 0; i < prime; ++i)
        tma_load_2d(smem + i * stage_bytes + kWTileBytes, &tm_x, &hdr->full[i], (kb0 + i) * kKB, m0);
      int issued = prime;
      for (int i = prime; i < nkb; ++i) {
        const int s = i % ns;
        if (i >= ns && !mbar_wait(&hdr->empty[s], ((i / ns) - 1) & 1)) break;
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&hdr->full[s], bytes);
        tma_load_2d(st, &tm_w, &hdr->full[s], (kb0 + i) * (kKB / 2), n0);
        tma_load_2d(st + kWTileBytes, &tm_x, &hdr->full[s], (kb0 + i) * kKB, m0);
        ++issued;
      }
      // Drain: every issued load has landed before the block may exit.
      for (int i = (issued > ns ? issued - ns : 0); i < issued; ++i)
        mbar_wait(&hdr->full[i % ns], (i / ns) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(kRows, BT, /*a_signed=*/true, /*b_signed=*/true);
      bool ok = true;
      for (int i = 0; i < nkb && ok; ++i) {
        const int s = i % ns, a = i % kASlots;
        ok = mbar_wait(&hdr->full[s], (i / ns) & 1) && mbar_wait(&hdr->a_full[a], (i / kASlots) & 1);
        if (!ok) break;
        tc_fence_after();
        const uint64_t bdesc = umma_desc_k_sw128(smem_u32(smem + s * stage_bytes + kWTileBytes));
#pragma unroll
        for (int kk = 0; kk < kKB / 32; ++kk) {
          umma_i8_ts(tmem, tmem + a_col0 + 32 * a + 8 * kk, bdesc + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&hdr->empty[s]);
        umma_commit(&hdr->a_empty[a]);
      }
      umma_commit(&hdr->acc_full);
      mbar_wait(&hdr->acc_full, 0);  // all MMAs retired before teardown
    }
  } else {
    // ------------------------------------------------ unpack, then epilogue
    const int quad = warp & 3;  // tensor-memory lane quadrant of this warp
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int et = threadIdx.x - 64;  // 0..127 over the four unpack/epilogue warps
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % ns, a = i % kASlots;
      ok = mbar_wait(&hdr->full[s], (i / ns) & 1);
      if (ok && i >= kASlots) ok = mbar_wait(&hdr->a_empty[a], ((i / kASlots) - 1) & 1);
      ok = __all_sync(0xffffffffu, ok);  // tcgen05.st below is warp-collective
      if (!ok) break;
      unpack_row_to_tmem(smem + s * stage_bytes, row, tmem + lane_base + a_col0 + 32 * a);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&hdr->empty[s]);
        mbar_arrive(&hdr->a_full[a]);
      }
    }
    pdl_wait();  // s_a comes from the preceding prologue kernel
    if (SINK != static_cast<int>(GemmSink::kS32)) {
      for (int c = et; c < BT; c += 128) sa_tile[c] = (m0 + c < p.M) ? __ldg(p.s_a + m0 + c) : 0.0f;
    }
    if (ok) ok = mbar_wait(&hdr->acc_full, 0);
    ok = __all_sync(0xffffffffu, ok);  // tcgen05.ld below is warp-collective
    tc_fence_after();
    named_barrier(1, 128);  // sa_tile written by all four epilogue warps

    const int n = n0 + row;
    if (p.splits == 1) {
      if (ok && nkb > 0) {
        const float sw = (SINK != static_cast<int>(GemmSink::kS32) && n < p.N) ? __ldg(p.s_w + n) : 0.0f;
        const float bv = (p.bias && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
        for (int c = 0; c < BT; c += 16) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(tmem + lane_base + static_cast<uint32_t>(c), v);
          tmem_wait_ld();
          if (n < p.N) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int m = m0 + c + j;
              if (m < p.M) store_output<SINK>(p, m, n, static_cast<int32_t>(v[j]), sa_tile[c + j], sw, bv);
            }
          }
        }
      }
    } else {
      // Push the partial tile to its owners.  4-token group g belongs to CTA
      // g % S of the cluster, which keeps the partials of its groups in slots
      // [source rank][g / S][row] (16 bytes each); the stores are
      // fire-and-forget and become visible at the cluster barrier.
      const int S = p.splits;
      const int ngl = (BT / 4 + S - 1) / S;
      const uint32_t me = cluster_ctarank();
      const uint32_t red_base = smem_u32(red);
      for (int c = 0; c < BT; c += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem + lane_base + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
        const bool keep = ok && nkb > 0;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int g = c / 4 + q;
          const int4 w = keep ? make_int4(static_cast<int32_t>(v[4 * q]), static_cast<int32_t>(v[4 * q + 1]),
                                          static_cast<int32_t>(v[4 * q + 2]), static_cast<int32_t>(v[4 * q + 3]))
                              : make_int4(0, 0, 0, 0);
          const uint32_t slot = ((static_cast<uint32_t>(me) * ngl + static_cast<uint32_t>(g / S)) * kRows + row) * 16u;
          st_shared_cluster_v4(map_shared_rank(red_base + slot, static_cast<uint32_t>(g % S)), w);
        }
      }
    }
  }

  if (p.splits > 1) {
    __syncwarp();    // the cluster barrier below is .aligned: reconverge first
    cluster_sync();  // every partial has reached its owner's shared memory
    if (warp >= 2) {
      // This CTA sums, from its own shared memory, the S partials of the
      // groups it owns and writes their outputs.  No CTA touches another's
      // shared memory after the barrier, so none has to wait before exiting.
      const int S = p.splits;
      const int ngl = (BT / 4 + S - 1) / S;
      const int quad = warp & 3;
      const int row = quad * 32 + lane;
      const int n = n0 + row;
      const int rank = static_cast<int>(cluster_ctarank());
      const float sw = (SINK != static_cast<int>(GemmSink::kS32) && n < p.N) ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (p.bias && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
      const int4* red4 = reinterpret_cast<const int4*>(red);
      for (int gl = 0; gl < ngl; ++gl) {
        const int g = gl * S + rank;
        if (g >= BT / 4 || m0 + 4 * g >= p.M || n >= p.N) continue;
        int4 sum = make_int4(0, 0, 0, 0);
        for (int j = 0; j < S; ++j) {
          const int4 v = red4[(j * ngl + gl) * kRows + row];
          sum.x += v.x; sum.y += v.y; sum.z += v.z; sum.w += v.w;
        }
        const int32_t sv[4] = {sum.x, sum.y, sum.z, sum.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int m = m0 + 4 * g + q;
          if (m < p.M) store_output<SINK>(p, m, n, sv[q], sa_tile[4 * g + q], sw, bv);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}


// ---------------------------------------------------------------- persistent kernel (large M)
//
// One CTA per SM walks the output tiles (tile t -> m tile t % m_tiles, n tile
// t / m_tiles) with a k-block stream that does not drain between tiles:
//   warp 0      TMA producer (ring of `nstages` shared-memory stages)
//   warp 1      TMEM allocation (all 512 columns) and the MMA-issuing thread
//   warps 2..5  weight unpack into four 32-column A slots of tensor memory
//   warps 6..9  epilogue, draining one of two 192-column accumulators while
//               the MMA fills the other
constexpr int kPThreads = 320;
constexpr int kPASlots = 4;
constexpr uint32_t kPAccStride = 192;  // column offset of accumulator 1
constexpr uint32_t kPAColBase = 384;   // first A-slot column

struct PParams {
  const float* s_a;
  const float* s_w;
  const uint16_t* bias;
  void* out;
  int M, N, K;
  int BT, m_tiles, num_tiles, nstages;
};

struct PHeader {
  uint64_t full[8];
  uint64_t empty[8];
  uint64_t a_full[kPASlots];
  uint64_t a_empty[kPASlots];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint32_t tmem_base;
};

template <int SINK>
__global__ void __launch_bounds__(kPThreads, 1)
    w4a4_tc_gemm_persistent_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                                   const __grid_constant__ PParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int BT = p.BT;
  const int ns = p.nstages;
  const int stage_bytes = kWTileBytes + BT * kKB;
  PHeader* hdr = reinterpret_cast<PHeader*>(smem + ns * stage_bytes);
  float* sa_buf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(hdr) + 1024);  // [2][192]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kbn = p.K / kKB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ns; ++s) {
      mbar_init(&hdr->full[s], 1);
      mbar_init(&hdr->empty[s], 1 + 4);  // MMA commit + one arrive per unpack warp
    }
    for (int a = 0; a < kPASlots; ++a) {
      mbar_init(&hdr->a_full[a], 4);
      mbar_init(&hdr->a_empty[a], 1);
    }
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
      const int my_tiles = (p.num_tiles - static_cast<int>(blockIdx.x) + static_cast<int>(gridDim.x) - 1) /
                           static_cast<int>(gridDim.x);
      const int total = my_tiles * kbn;
      auto coords = [&](int i, int& m0, int& n0, int& kb) {
        const int tile = static_cast<int>(blockIdx.x) + (i / kbn) * static_cast<int>(gridDim.x);
        m0 = (tile % p.m_tiles) * BT;
        n0 = (tile / p.m_tiles) * kRows;
        kb = i % kbn;
      };
      // Weight tiles of the first stages do not depend on the preceding
      // prologue kernel: request them before waiting for it.
      const int prime = total < ns ? total : ns;
      for (int i = 0; i < prime; ++i) {
        int m0, n0, kb;
        coords(i, m0, n0, kb);
        mbar_arrive_expect_tx(&hdr->full[i], bytes);
        tma_load_2d(smem + i * stage_bytes, &tm_w, &hdr->full[i], kb * (kKB / 2), n0);
      }
      pdl_wait();
      for (int i = 0; i < prime; ++i) {
        int m0, n0, kb;
        coords(i, m0, n0, kb);
        tma_load_2d(smem + i * stage_bytes + kWTileBytes, &tm_x, &hdr->full[i], kb * kKB, m0);
      }
      int it = prime;
      for (; it < total; ++it) {
        const int s = it % ns;
        if (!mbar_wait(&hdr->empty[s], ((it / ns) - 1) & 1)) break;
        int m0, n0, kb;
        coords(it, m0, n0, kb);
        uint8_t* st = smem + s * stage_bytes;
        mbar_arrive_expect_tx(&hdr->full[s], bytes);
        tma_load_2d(st, &tm_w, &hdr->full[s], kb * (kKB / 2), n0);
        tma_load_2d(st + kWTileBytes, &tm_x, &hdr->full[s], kb * kKB, m0);
      }
      // Drain: every issued load has landed before the block may exit.
      for (int i = (it > ns ? it - ns : 0); i < it; ++i) mbar_wait(&hdr->full[i % ns], (i / ns) & 1);
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(kRows, BT, /*a_signed=*/true, /*b_signed=*/true);
      int it = 0, tc = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x, ++tc) {
        const int b = tc & 1;
        if (tc >= 2 && !mbar_wait(&hdr->acc_empty[b], ((tc / 2) - 1) & 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(b) * kPAccStride;
        for (int kb = 0; kb < kbn; ++kb, ++it) {
          const int s = it % ns, a = it % kPASlots;
          if (!mbar_wait(&hdr->full[s], (it / ns) & 1) || !mbar_wait(&hdr->a_full[a], (it / kPASlots) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = umma_desc_k_sw128(smem_u32(smem + s * stage_bytes + kWTileBytes));
#pragma unroll
          for (int kk = 0; kk < kKB / 32; ++kk)
            umma_i8_ts(d_tmem, tmem + kPAColBase + 32 * a + 8 * kk, bdesc + 2 * kk, idesc,
                       (kb > 0 || kk > 0) ? 1u : 0u);
          umma_commit(&hdr->empty[s]);
          umma_commit(&hdr->a_empty[a]);
        }
        umma_commit(&hdr->acc_full[b]);
      }
    }
  } else if (warp < 6) {
    // ------------------------------------------------ weight unpack
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < p.num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < kbn; ++kb, ++it) {
        const int s = it % ns, a = it % kPASlots;
        bool w = mbar_wait(&hdr->full[s], (it / ns) & 1);
        if (w && it >= kPASlots) w = mbar_wait(&hdr->a_empty[a], ((it / kPASlots) - 1) & 1);
        ok = __all_sync(0xffffffffu, w);  // tcgen05.st below is warp-collective
        if (!ok) break;
        unpack_row_to_tmem(smem + s * stage_bytes, row, tmem + lane_base + kPAColBase + 32 * a);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&hdr->empty[s]);
          mbar_arrive(&hdr->a_full[a]);
        }
      }
    }
  } else {
    // ------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int row = quad * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quad * 32) << 16;
    const int et = threadIdx.x - 192;  // 0..127
    pdl_wait();  // s_a comes from the preceding prologue kernel
    int tc = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x, ++tc) {
      const int b = tc & 1;
      const int m0 = (tile % p.m_tiles) * BT, n0 = (tile / p.m_tiles) * kRows;
      float* sa = sa_buf + 192 * b;
      if (SINK != static_cast<int>(GemmSink::kS32))
        for (int c = et; c < BT; c += 128) sa[c] = (m0 + c < p.M) ? __ldg(p.s_a + m0 + c) : 0.0f;
      named_barrier(1, 128);  // s_a of this tile staged; all warps are done with tile tc - 2
      const int n = n0 + row;
      const float sw = (SINK != static_cast<int>(GemmSink::kS32) && n < p.N) ? __ldg(p.s_w + n) : 0.0f;
      const float bv = (p.bias && n < p.N) ? __uint_as_float(static_cast<uint32_t>(__ldg(p.bias + n)) << 16) : 0.0f;
      // On a failed wait the warp skips the tile's work but keeps taking part
      // in the named barrier above, so no peer waits on it forever.
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&hdr->acc_full[b], (tc / 2) & 1));
      tc_fence_after();
      const uint32_t acc = tmem + lane_base + static_cast<uint32_t>(b) * kPAccStride;
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
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&hdr->acc_empty[b]);
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

int shared_bytes_for(int BT, int nstages, int splits) {
  int bytes = 1024 /*alignment slack*/ + nstages * (kWTileBytes + BT * kKB) + 2048 /*header + s_a tile*/;
  if (splits > 1) bytes += splits * ((BT / 4 + splits - 1) / splits) * kRows * 16;
  return bytes;
}

template <int SINK>
cudaError_t launch_sink(const CUtensorMap& tw, const CUtensorMap& tx, const Params& prm, const GemmTiling& t,
                        cudaStream_t stream) {
  static int cache[64] = {0};
  cudaError_t e = ensure_dynamic_smem(reinterpret_cast<const void*>(w4a4_tc_gemm_kernel<SINK>), t.smem_bytes, cache);
  if (e != cudaSuccess) return note_cuda(e, "w4a4_gemm: dynamic shared memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(t.n_tiles, t.m_tiles, t.splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(t.smem_bytes);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  int nattr = 0;
  attr[nattr].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[nattr].val.programmaticStreamSerializationAllowed = 1;
  ++nattr;
  if (t.splits > 1) {
    attr[nattr].id = cudaLaunchAttributeClusterDimension;
    attr[nattr].val.clusterDim.x = 1;
    attr[nattr].val.clusterDim.y = 1;
    attr[nattr].val.clusterDim.z = static_cast<unsigned>(t.splits);
    ++nattr;
  }
  cfg.attrs = attr;
  cfg.numAttrs = nattr;
  return note_cuda(cudaLaunchKernelEx(&cfg, w4a4_tc_gemm_kernel<SINK>, tw, tx, prm), "w4a4_gemm: launch");
}

template <int SINK>
cudaError_t launch_persistent(const CUtensorMap& tw, const CUtensorMap& tx, const PParams& prm, const GemmTiling& t,
                              cudaStream_t stream) {
  static int cache[64] = {0};
  const void* kfn = reinterpret_cast<const void*>(w4a4_tc_gemm_persistent_kernel<SINK>);
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
  return note_cuda(cudaLaunchKernelEx(&cfg, w4a4_tc_gemm_persistent_kernel<SINK>, tw, tx, prm),
                   "w4a4_gemm: persistent launch");
}

// Estimated cycles of the persistent kernel for a token tile of BT: rounds
// of tiles per SM x k blocks x the slower of the MMA (2 * BT cycles per k
// block at 8192 int8 MACs/clk) and a per-k-block floor of 256 cycles for the
// fixed work every k block carries whatever BT is (the 8 KB weight tile
// fetched from L2 and unpacked into tensor memory).
long persistent_cost(int M, int N, int K, int BT, int num_sms) {
  const long tiles = static_cast<long>((M + BT - 1) / BT) * ((N + kRows - 1) / kRows);
  const long rounds = (tiles + num_sms - 1) / num_sms;
  const long per_kb = 2L * BT > 256 ? 2L * BT : 256;
  return rounds * (K / kKB) * per_kb;
}

}  // namespace

GemmTiling choose_tiling(int M, int N, int K, int num_sms) {
  GemmTiling t{};
  // Large M: the persistent kernel, with the token tile BT (multiple of 16,
  // <= 192) of the lowest estimated cost, when it yields at least half as
  // many tiles as SMs.
  {
    int best_bt = 0;
    long best = -1;
    for (int bt = 192; bt >= 64; bt -= 16) {
      const long tiles = static_cast<long>((M + bt - 1) / bt) * ((N + kRows - 1) / kRows);
      if (2 * tiles < num_sms) continue;
      const long c = persistent_cost(M, N, K, bt, num_sms);
      if (best < 0 || c < best) {
        best = c;
        best_bt = bt;
      }
    }
    if (best_bt > 0 && M > 128) {
      t.persistent = true;
      t.BT = best_bt;
      t.m_tiles = (M + best_bt - 1) / best_bt;
      t.n_tiles = (N + kRows - 1) / kRows;
      t.splits = 1;
      t.kb_per_split = K / kKB;
      const int stage = kWTileBytes + best_bt * kKB;
      int ns = (220 * 1024 - 4096) / stage;
      if (ns > 8) ns = 8;
      t.nstages = ns;
      t.tmem_cols = 512;
      t.smem_bytes = 1024 + ns * stage + 1024 + 2 * 192 * 4;
      if (t.smem_bytes < 120 * 1024) t.smem_bytes = 120 * 1024;  // one CTA per SM (it owns all of TMEM)
      const long tiles = static_cast<long>(t.m_tiles) * t.n_tiles;
      t.grid = static_cast<int>(tiles < num_sms ? tiles : num_sms);
      return t;
    }
  }
  // Small M: one CTA per (tile, K slice), slices of a tile form a cluster.
  const int kb_total = K / kKB;
  // Tokens per tile: one tile when M fits, else the fewest tiles of <= 192.
  const int max_bt = 192;
  int m_tiles = (M + max_bt - 1) / max_bt;
  int bt = (M + m_tiles - 1) / m_tiles;
  bt = ((bt + 15) / 16) * 16;
  if (bt < 16) bt = 16;
  t.BT = bt;
  t.m_tiles = (M + bt - 1) / bt;
  t.n_tiles = (N + kRows - 1) / kRows;
  // Split K across a cluster until the grid covers two CTAs per SM.
  const int tiles = t.m_tiles * t.n_tiles;
  int splits = 1;
  while (splits < 8 && tiles * splits * 2 <= 2 * num_sms && splits * 2 <= kb_total) splits *= 2;
  const int kbps = (kb_total + splits - 1) / splits;  // the largest share
  t.splits = splits;
  t.kb_per_split = kbps;
  // Pipeline depth: as many stages as fit two CTAs per SM (~110 KB each).
  const int stage = kWTileBytes + bt * kKB;
  int ns = (110 * 1024 - 3072 - (splits > 1 ? splits * ((bt / 4 + splits - 1) / splits) * kRows * 16 : 0)) / stage;
  if (ns > 8) ns = 8;
  if (ns > kbps) ns = kbps < 2 ? 2 : kbps;
  if (ns < 2) ns = 2;
  t.nstages = ns;
  int cols = 32;
  while (cols < bt + 32 * kASlots) cols *= 2;
  t.tmem_cols = cols;
  t.smem_bytes = shared_bytes_for(bt, ns, splits);
  // Never let more CTAs share an SM than its 512 tensor-memory columns can
  // hold: a CTA blocked in tcgen05.alloc while its cluster peers wait for it
  // could deadlock.  Shared memory per CTA is padded so that at most
  // 512 / cols CTAs fit in the SM's 228 KB.
  const int max_ctas = 512 / cols;
  const int min_smem = (228 * 1024) / (max_ctas + 1) + 1;
  if (t.smem_bytes < min_smem) t.smem_bytes = min_smem;
  t.persistent = false;
  t.grid = t.n_tiles * t.m_tiles * t.splits;
  return t;
}

cudaError_t launch_w4a4_gemm(const GemmArgs& a, GemmSink sink, const GemmTiling& t, cudaStream_t stream) {
  CUtensorMap tw, tx;
  if (!make_map_u8(&tw, a.Wq, static_cast<uint64_t>(a.N), static_cast<uint64_t>(a.K / 2), kRows, kKB / 2,
                   CU_TENSOR_MAP_SWIZZLE_64B))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: weight tensor map");
  if (!make_map_u8(&tx, a.xs8, static_cast<uint64_t>(a.M), static_cast<uint64_t>(a.K), static_cast<uint32_t>(t.BT),
                   kKB, CU_TENSOR_MAP_SWIZZLE_128B))
    return note_cuda(cudaErrorInvalidValue, "w4a4_gemm: activation tensor map");
  if (t.persistent) {
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
    cudaError_t e;
    switch (sink) {
      case GemmSink::kBF16: e = launch_persistent<0>(tw, tx, pp, t, stream); break;
      case GemmSink::kF32: e = launch_persistent<1>(tw, tx, pp, t, stream); break;
      default: e = launch_persistent<2>(tw, tx, pp, t, stream); break;
    }
    count_dispatch(2);
    return e;
  }
  Params prm{};
  prm.s_a = a.s_a;
  prm.s_w = a.s_w;
  prm.bias = a.bias;
  prm.out = a.out;
  prm.M = a.M;
  prm.N = a.N;
  prm.K = a.K;
  prm.BT = t.BT;
  prm.splits = t.splits;
  prm.kb_total = a.K / kKB;
  prm.kb_per_split = t.kb_per_split;
  prm.nstages = t.nstages;
  prm.tmem_cols = t.tmem_cols;
  cudaError_t e;
  switch (sink) {
    case GemmSink::kBF16: e = launch_sink<0>(tw, tx, prm, t, stream); break;
    case GemmSink::kF32: e = launch_sink<1>(tw, tx, prm, t, stream); break;
    default: e = launch_sink<2>(tw, tx, prm, t, stream); break;
  }
  count_dispatch(t.splits > 1 ? 3 : 2);
  return e;
}

}  // namespace convrot
