// small_m.cu -- the ConvRot W4A4 Linear for a few tokens (M <= 16), where
// streaming the packed weights out of HBM is the whole cost.
//
// What it computes is the same Linear as rotate_quant.cu + gemm.cu
// ("Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot...)": group-256
// rotation, dynamic per-token INT4, integer GEMM, rank-one epilogue), bit for
// bit.  The 76-token text-encoder passes of "Qwen3-VL-4B-W4A8-ConvRot"
// (encode table) and decode-like calls are this regime: at M <= 16 a Linear
// does at most 32 integer MACs per weight byte, far below the B200's ridge
// point, so the kernels are built to keep HBM busy rather than the tensor
// pipe, and to put as few latencies as possible between launch and result.
//
// Two kernels, chained with programmatic dependent launch:
//
// rq_rows_kernel  one CTA per token row: every warp first loads its 256-
//   channel chunks (lane l holds channels 8l .. 8l+7 of a chunk, one 16-byte
//   load), then rotates them in registers and warp shuffles; the row's amax is
//   reduced through shared memory, and the codes are written packed, two to a
//   byte (the public convrot_rotate_quant layout).
//
// w4a4_gemv_kernel (K6)  one CTA (four warps) per slab of 16 output channels
//   (and, only where K is very long or N small, per part of K).  The slab's
//   packed weights are contiguous rows; one bulk copy (cp.async.bulk) per row
//   of the CTA's K range brings them into shared memory at launch, before
//   the grid waits for the prologue, so the whole matrix is requested from
//   HBM at once and no tensor-map descriptor has to be fetched first.  Rows
//   are padded to 64 bytes modulo 128 so that the 16-byte fragment loads are
//   free of bank conflicts.  Warp w multiplies the rows of its share of the
//   K range with mma.sync m16n8k32 s8: the weights are the A
//   operand (MMA rows = channels), the tokens the columns.  Both operands
//   arrive as packed nibbles and are widened in registers: for a 32-bit word
//   w of codes k .. k+7 (even code in the low nibble), (w << 4) & 0xF0F0F0F0
//   holds 16 q for codes (0, 2, 4, 6) and w & 0xF0F0F0F0 holds 16 q for codes
//   (1, 3, 5, 7), both exact signed bytes.  The MMA's k order is then a
//   permutation of the codes' that is the same for both operands, so the dot
//   product is unchanged, and the accumulator is exactly 256 acc (|256 acc|
//   <= 2^14 K <= 2^29).  The four warps' sums meet in shared memory.  Where
//   K is split over several CTAs, each stores its int32 partial slab, counts
//   itself in with an atomic, and the last to arrive adds the partials and
//   applies the epilogue: integer sums are exact, so the result does not
//   depend on the split, and no CTA ever waits for another one.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>

#include "kernels.cuh"
#include "ptx.cuh"

namespace convrot {

namespace {

constexpr int kSlabRows = 16;          // output channels per CTA (the MMA's 16 rows)
constexpr int kBlockK = 128;           // K values per block: 64 packed bytes, 4 MMA k-steps
constexpr int kBlockBytes = kBlockK / 2;
constexpr int kLongKBlocks = 40;       // K blocks per part above which a CTA runs 8 warps instead of 4
constexpr int kMaxPartBlocks = 96;     // K blocks per CTA: a 16 x 6 KB slab (+ padding) in shared memory
constexpr int kMaxParts = 64;          // K parts per slab
constexpr int kTargetCtas = 148;       // at least one CTA per SM where the slabs allow it

// How one launch cuts the work (host and scratch sizing agree on it).
struct GemvPlan {
  int tiles;   // slabs of 16 channels: ceil(N / 16)
  int parts;   // K parts per slab (1: no cross-CTA sum)
  int nb;      // K blocks of 128
};

GemvPlan gemv_plan(int N, int K) {
  GemvPlan g{};
  g.tiles = (N + kSlabRows - 1) / kSlabRows;
  g.nb = K / kBlockK;
  int parts = (g.nb + kMaxPartBlocks - 1) / kMaxPartBlocks;            // slab fits in shared memory
  const int spread = (kTargetCtas + g.tiles - 1) / g.tiles;            // enough CTAs for every SM
  if (spread > parts) parts = spread;
  const int most = g.nb / 4 > 0 ? g.nb / 4 : 1;                        // at least 4 blocks per part
  if (parts > most) parts = most;
  if (parts > kMaxParts) parts = kMaxParts;
  if (parts < 1) parts = 1;
  g.parts = parts;
  return g;
}

struct GemvParams {
  const uint8_t* Wq;      // [N, K/2] packed weights
  const uint8_t* xq;      // [M, K/2] packed activation codes
  const float* s_a;       // [M]
  const float* s_w;       // [N]
  const uint16_t* bias;   // [N] or null
  void* out;              // [M, N]
  int32_t* part;          // [tiles][parts][MT][16] partial slabs (parts > 1)
  uint32_t* ctr;          // [tiles] arrival counters, zero on entry (parts > 1)
  int M, N, K;
  int nb, parts, row_stride;  // row_stride: shared-memory bytes per slab row
};

__device__ __forceinline__ uint4 lds128(const uint8_t* p) { return *reinterpret_cast<const uint4*>(p); }

// d (16x8, s32) += a (16x32, s8, row) * b (32x8, s8, col).
__device__ __forceinline__ void mma_s8(int32_t (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                       uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t even16(uint32_t w) { return (w << 4) & 0xF0F0F0F0u; }  // 16 q, codes 0,2,4,6
__device__ __forceinline__ uint32_t odd16(uint32_t w) { return w & 0xF0F0F0F0u; }          // 16 q, codes 1,3,5,7

__device__ __forceinline__ uint16_t to_bf16_rne(float y) {
  const uint32_t u = __float_as_uint(y);
  return static_cast<uint16_t>((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
}

// One output element from the MMA sum d = 256 acc (scales and bias already
// loaded).
template <int SINK>
__device__ __forceinline__ void put(const GemvParams& p, int m, int n, int32_t d, float sa, float sw, float bv) {
  const int32_t acc = d >> 8;
  const size_t idx = static_cast<size_t>(m) * static_cast<size_t>(p.N) + static_cast<size_t>(n);
  if (SINK == static_cast<int>(GemmSink::kS32)) {
    static_cast<int32_t*>(p.out)[idx] = acc;
    return;
  }
  // The oracle's order: ((float)acc * s_a) * s_w + bias, each rounded once.
  float y = __fmul_rn(__fmul_rn(__int2float_rn(acc), sa), sw);
  if (p.bias) y = __fadd_rn(y, bv);
  if (SINK == static_cast<int>(GemmSink::kF32))
    static_cast<float*>(p.out)[idx] = y;
  else
    static_cast<uint16_t*>(p.out)[idx] = to_bf16_rne(y);
}

// NT n-tiles of 8 tokens (MT = 8 NT); W warps, each taking 1/W of the K range.
template <int SINK, int NT, int W>
__global__ void __launch_bounds__(32 * W, W == 4 ? 6 : 2) w4a4_gemv_kernel(const __grid_constant__ GemvParams p) {
  constexpr int MT = 8 * NT;
  constexpr int D = NT == 1 ? 8 : 4;  // blocks of activation words in flight per warp, in registers
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* slab = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ __align__(8) uint64_t bar;
  __shared__ __align__(16) float s_sw[kSlabRows];        // the slab's weight scales
  __shared__ __align__(16) uint16_t s_bias[kSlabRows];   // and bias
  __shared__ __align__(16) int32_t red[W][MT][kSlabRows];
  __shared__ uint32_t s_last;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = static_cast<int>(blockIdx.x) / p.parts, part = static_cast<int>(blockIdx.x) % p.parts;
  const int n0 = tile * kSlabRows;
  const int rows = p.N - n0 < kSlabRows ? p.N - n0 : kSlabRows;  // 8 or 16 (N % 8 == 0)
  const int b0 = (part * p.nb) / p.parts, b1 = ((part + 1) * p.nb) / p.parts;
  const int wb0 = b0 + (warp * (b1 - b0)) / W, wb1 = b0 + ((warp + 1) * (b1 - b0)) / W;
  const size_t wrow = static_cast<size_t>(p.K) / 2;  // bytes per weight / activation row

  // ---- weights: thread r < rows copies row r's share of the CTA's K range
  // (one bulk copy per row: few, large copies keep the copy engine's per-copy
  // cost out of the way); threads 16 and 17 copy the slab's weight scales and
  // bias, which the epilogue reads from shared memory.  None of them depends
  // on the preceding kernel: all are requested before waiting for it, and no
  // register waits on them before the weights have landed.
  const bool scaled = SINK != static_cast<int>(GemmSink::kS32);
  const uint32_t rbytes = static_cast<uint32_t>((b1 - b0) * kBlockBytes);
  const uint32_t swbytes = scaled ? static_cast<uint32_t>(rows) * 4u : 0u;
  const uint32_t bbytes = p.bias ? static_cast<uint32_t>(rows) * 2u : 0u;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    mbar_arrive_expect_tx(&bar, rbytes * static_cast<uint32_t>(rows) + swbytes + bbytes);
  }
  __syncwarp();
  if (static_cast<int>(threadIdx.x) < rows)
    bulk_load(slab + threadIdx.x * p.row_stride,
              p.Wq + static_cast<size_t>(n0 + threadIdx.x) * wrow + static_cast<size_t>(b0) * kBlockBytes, rbytes,
              &bar);
  if (threadIdx.x == 16 && swbytes) bulk_load(s_sw, p.s_w + n0, swbytes, &bar);
  if (threadIdx.x == 17 && bbytes) bulk_load(s_bias, p.bias + n0, bbytes, &bar);
  __syncthreads();  // the barrier is initialised before any thread waits on it
  // The next kernel on the stream may launch now; it waits for this grid
  // before it touches anything this grid reads or writes.
  pdl_launch_dependents();
  const uint32_t wbytes = static_cast<uint32_t>((wb1 - wb0) * kBlockBytes);
  // Thread i stores channel n0 + i % 16 in the epilogue.
  constexpr int kOut = MT * kSlabRows;
  constexpr int kPerThread = (kOut + 32 * W - 1) / (32 * W);  // 1 or 2
  const int r = threadIdx.x & 15;
  const bool mine_out = static_cast<int>(threadIdx.x) < kOut;  // (kOut is a multiple of 32 W or smaller)
  const bool chan = r < rows && mine_out;
  pdl_wait();  // activations, scales, partial slabs and counters belong to the preceding kernels until now

  // ---- this warp's K range: 4 MMA k-steps per block, two accumulator sets
  // (alternate blocks) so that two MMA chains are in flight (D is even).
  const int g = lane >> 2, t = lane & 3;
  float sa[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int m = (static_cast<int>(threadIdx.x) + 32 * W * k) >> 4;
    sa[k] = (scaled && chan && m < p.M) ? p.s_a[m] : 0.0f;
  }
  int32_t acc[2][NT][4];
#pragma unroll
  for (int a = 0; a < 2; ++a)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[a][j][0] = acc[a][j][1] = acc[a][j][2] = acc[a][j][3] = 0;
  // The activation words come from L2 (every CTA reads the same codes), D
  // blocks of them in flight in registers; they are requested before the
  // wait for this warp's weights.  Long K ranges (8 warps) also ask L1 for
  // the warp's whole range first.
  const uint8_t* xr[NT];
  bool xlive[NT];
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    xlive[j] = 8 * j + g < p.M;
    xr[j] = p.xq + static_cast<size_t>(xlive[j] ? 8 * j + g : 0) * wrow + 16 * t;
  }
  if (W == 8 && t == 0) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
      if (xlive[j])
        for (int b = wb0 + D; b < wb1; ++b)
          asm volatile("prefetch.global.L1 [%0];" ::"l"(xr[j] + static_cast<size_t>(b) * kBlockBytes));
  }
  uint4 xbuf[D][NT];
  auto load_x = [&](int b, uint4 (&dst)[NT]) {
#pragma unroll
    for (int j = 0; j < NT; ++j)
      dst[j] = (b < wb1 && xlive[j]) ? *reinterpret_cast<const uint4*>(xr[j] + static_cast<size_t>(b) * kBlockBytes)
                                     : make_uint4(0, 0, 0, 0);
  };
#pragma unroll
  for (int d = 0; d < D; ++d) load_x(wb0 + d, xbuf[d]);
  const bool landed = mbar_wait(&bar, 0);
  // After a wait that gave up, the copies still in flight must land (bounded)
  // before the block may exit.
  if (!landed) (void)mbar_drain(&bar, 0, 100000000ull);
  const float sw = (scaled && chan && landed) ? s_sw[r] : 0.0f;
  const float bv = (bbytes && chan && landed) ? __uint_as_float(static_cast<uint32_t>(s_bias[r]) << 16) : 0.0f;
  if (landed && wbytes > 0) {
    const uint8_t* wr0 = slab + g * p.row_stride + 16 * t - b0 * kBlockBytes;
    const uint8_t* wr1 = wr0 + 8 * p.row_stride;
    for (int bb = wb0; bb < wb1; bb += D) {
#pragma unroll
      for (int d = 0; d < D; ++d) {
        const int b = bb + d;
        if (b < wb1) {
          uint4 xa[NT];
#pragma unroll
          for (int j = 0; j < NT; ++j) xa[j] = xbuf[d][j];
          load_x(b + D, xbuf[d]);
          const uint4 wa = lds128(wr0 + b * kBlockBytes);
          const uint4 wb = lds128(wr1 + b * kBlockBytes);
          const uint32_t va[4] = {wa.x, wa.y, wa.z, wa.w}, vb[4] = {wb.x, wb.y, wb.z, wb.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // k step q of the block: thread t holds codes 32t + 8q .. +7 of
            // both operands (word q of its 16 bytes).
            const uint32_t a0 = even16(va[q]), a1 = even16(vb[q]), a2 = odd16(va[q]), a3 = odd16(vb[q]);
#pragma unroll
            for (int j = 0; j < NT; ++j) {
              const uint32_t xw = q == 0 ? xa[j].x : q == 1 ? xa[j].y : q == 2 ? xa[j].z : xa[j].w;
              mma_s8(acc[d & 1][j], a0, a1, a2, a3, even16(xw), odd16(xw));
            }
          }
        }
      }
    }
  }
  // ---- the four warps' sums: D[row][token] for rows g, g + 8 and tokens
  // 8j + 2t, 8j + 2t + 1.
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      red[warp][8 * j + 2 * t + e][g] = acc[0][j][e] + acc[1][j][e];
      red[warp][8 * j + 2 * t + e][g + 8] = acc[0][j][2 + e] + acc[1][j][2 + e];
    }
  __syncthreads();
  // Output i = threadIdx.x + 32 W k: row r = i % 16 (consecutive channels ->
  // coalesced stores), token m = i / 16.
  int32_t sum[kPerThread];
#pragma unroll
  for (int k = 0; k < kPerThread; ++k) {
    const int i = static_cast<int>(threadIdx.x) + 32 * W * k;
    sum[k] = 0;
    if (i < kOut)
#pragma unroll
      for (int w = 0; w < W; ++w) sum[k] += red[w][i >> 4][r];
  }
  if (p.parts > 1) {
    // Publish this part's partial slab, count in; the last part sums them all.
    int32_t* mine = p.part + (static_cast<size_t>(tile) * p.parts + part) * MT * kSlabRows;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = static_cast<int>(threadIdx.x) + 32 * W * k;
      if (i < kOut) mine[i] = sum[k];
    }
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const uint32_t before = atomicAdd(&p.ctr[tile], 1u);
      const bool last = before == static_cast<uint32_t>(p.parts - 1);
      if (last) {
        p.ctr[tile] = 0u;  // every part has arrived: ready for the next call
        __threadfence();
      }
      s_last = last ? 1u : 0u;
    }
    __syncthreads();
    if (!s_last) return;
    const int32_t* all = p.part + static_cast<size_t>(tile) * p.parts * MT * kSlabRows;
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int idx = static_cast<int>(threadIdx.x) + 32 * W * k;
      if (idx >= kOut) continue;
      int32_t s = 0;
      // Eight loads in flight at a time.
      for (int q0 = 0; q0 < p.parts; q0 += 8) {
        int32_t v[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          v[u] = (q0 + u < p.parts && q0 + u != part) ? __ldcg(all + static_cast<size_t>(q0 + u) * MT * kSlabRows + idx)
                                                      : 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) s += v[u];
      }
      sum[k] += s;
    }
  }
  const int n = n0 + r;
  if (r < rows && landed && mine_out) {
#pragma unroll
    for (int k = 0; k < kPerThread; ++k) {
      const int i = static_cast<int>(threadIdx.x) + 32 * W * k;
      if (i < kOut && (i >> 4) < p.M) put<SINK>(p, i >> 4, n, sum[k], sa[k], sw, bv);
    }
  }
}

// ---------------------------------------------------------------- prologue

// Rotation of one 256-channel chunk held by a warp, lane l holding channels
// 8l .. 8l + 7 in v (the first LOG4G radix-4 stages, then 2^-LOG4G).  The
// channel index j = 64 d3 + 16 d2 + 4 d1 + d0; stage s combines the four
// channels that differ in digit d_s.  A butterfly (a, b, c, d) -> (p + t,
// p - t, q + r, r - q) with p = a + b, q = a - b, r = c + d, t = c - d gives
// the channel with digit value k the value (v_k + v_k^1) + (v_k^2 - v_k^3):
// for k = 1, 2, 3 this is p + (-t), r + q and r + (-q), the same correctly
// rounded results as p - t, q + r and r - q, since a sum does not depend on
// the order of its operands and negation is exact.  Digit d0 is register
// bits 0-1; d1 is register bit 2 and lane bit 0; d2 and d3 are lane bits 1-2
// and 3-4.
template <int LOG4G>
__device__ __forceinline__ void rotate_chunk(float (&v)[8]) {
  float t[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) t[e] = __fadd_rn(__fadd_rn(v[e], v[e ^ 1]), __fsub_rn(v[e ^ 2], v[e ^ 3]));
  float o[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) o[e] = __shfl_xor_sync(0xffffffffu, t[e], 1);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __fadd_rn(__fadd_rn(t[e], t[e ^ 4]), __fsub_rn(o[e], o[e ^ 4]));
  if (LOG4G >= 3) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float b = __shfl_xor_sync(0xffffffffu, v[e], 2);
      const float c = __shfl_xor_sync(0xffffffffu, v[e], 4);
      const float d = __shfl_xor_sync(0xffffffffu, v[e], 6);
      t[e] = __fadd_rn(__fadd_rn(v[e], b), __fsub_rn(c, d));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = t[e];
  }
  if (LOG4G >= 4) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float b = __shfl_xor_sync(0xffffffffu, v[e], 8);
      const float c = __shfl_xor_sync(0xffffffffu, v[e], 16);
      const float d = __shfl_xor_sync(0xffffffffu, v[e], 24);
      t[e] = __fadd_rn(__fadd_rn(v[e], b), __fsub_rn(c, d));
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] = t[e];
  }
  constexpr float kScale = LOG4G == 4 ? 0.0625f : (LOG4G == 3 ? 0.125f : 0.25f);
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = __fmul_rn(v[e], kScale);
}

// One CTA per row; warp w takes the 256-channel chunks w, w + warps, ...
// (at most CPW of them, kept in registers).  All of a warp's loads are issued
// before the first rotation, so the row costs one memory round trip.
template <int LOG4G, int CPW>
__global__ void __launch_bounds__(1024) rq_rows_kernel(const uint16_t* __restrict__ x, int K,
                                                       uint8_t* __restrict__ xq, float* __restrict__ s_a) {
  __shared__ float warp_max[32];
  // The GEMM that follows may launch now and start its weight stream; this
  // grid itself waits for the preceding kernel before reading x or writing.
  pdl_launch_dependents();
  pdl_wait();
  const int row = static_cast<int>(blockIdx.x);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const int chunks = K >> 8;
  const uint16_t* xr = x + static_cast<size_t>(row) * K;
  uint4 raw[CPW];
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    const int ch = warp + c * nw;
    raw[c] = ch < chunks ? __ldg(reinterpret_cast<const uint4*>(xr + ch * 256 + 8 * lane)) : make_uint4(0, 0, 0, 0);
  }
  float v[CPW][8];
  float amax = 0.0f;
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    const uint32_t wv[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[c][2 * i] = __uint_as_float(wv[i] << 16);
      v[c][2 * i + 1] = __uint_as_float(wv[i] & 0xFFFF0000u);
    }
    if (warp + c * nw < chunks) {  // warp-uniform: every lane takes part in the shuffles
      rotate_chunk<LOG4G>(v[c]);
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(v[c][e]));
    }
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (lane == 0) warp_max[warp] = amax;
  __syncthreads();
  amax = 0.0f;
  for (int w = 0; w < nw; ++w) amax = fmaxf(amax, warp_max[w]);
  const float s = __fdiv_rn(amax, 7.0f);
  // The code is rint of the correctly rounded quotient v / s.  For s >=
  // 2^-100 the quotient is formed by Markstein's correction (P. Markstein,
  // IBM J. Res. Develop. 34(1), 1990): with y = RN(1/s), q0 = RN(v y), and two
  // steps q <- RN(q + RN(v - s q) y), each remainder a fused multiply-add,
  // the second step starts from a faithful quotient, whose remainder is
  // exact, and returns RN(v / s).  Smaller scales (zero included) take the
  // IEEE division.  rint: adding 1.5 * 2^23 rounds to an integer, ties to
  // even, and leaves the two's-complement code in the low bits.
  const bool fast = s >= 7.88860905e-31f;  // 2^-100
  const float y = fast ? __frcp_rn(s) : 0.0f;
  uint8_t* qr = xq + static_cast<size_t>(row) * (K >> 1);
#pragma unroll
  for (int c = 0; c < CPW; ++c) {
    const int ch = warp + c * nw;
    if (ch >= chunks) continue;
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float x = v[c][e];
      int q;
      if (fast) {
        float qq = __fmul_rn(x, y);
        qq = __fmaf_rn(__fmaf_rn(-s, qq, x), y, qq);  // faithful
        qq = __fmaf_rn(__fmaf_rn(-s, qq, x), y, qq);  // RN(x / s)
        q = static_cast<int>(__float_as_uint(__fadd_rn(qq, 12582912.0f)) & 0xFFu);
        q = (q ^ 0x80) - 0x80;  // |x / s| <= 7 up to rounding: the low byte is the code
      } else {
        q = s != 0.0f ? __float2int_rn(__fdiv_rn(x, s)) : 0;
      }
      q = q < -8 ? -8 : (q > 7 ? 7 : q);
      word |= (static_cast<uint32_t>(q) & 0xFu) << (4 * e);
    }
    *reinterpret_cast<uint32_t*>(qr + ch * 128 + 4 * lane) = word;
  }
  if (threadIdx.x == 0) s_a[row] = s;
}

template <int LOG4G, int CPW>
cudaError_t launch_rows_cpw(const uint16_t* x, int M, int K, int warps, uint8_t* xq, float* s_a,
                            cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(M), 1, 1);
  cfg.blockDim = dim3(static_cast<unsigned>(32 * warps), 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note_cuda(cudaLaunchKernelEx(&cfg, rq_rows_kernel<LOG4G, CPW>, x, K, xq, s_a), "small prologue: launch");
}

// One warp per chunk up to 32 warps; then 2 or 4 chunks per warp (K <= 32768
// is 128 chunks at most).
template <int LOG4G>
cudaError_t launch_rows(const uint16_t* x, int M, int K, uint8_t* xq, float* s_a, cudaStream_t stream) {
  const int chunks = K >> 8;
  const int warps = chunks < 32 ? chunks : 32;
  const int cpw = (chunks + warps - 1) / warps;
  if (cpw <= 1) return launch_rows_cpw<LOG4G, 1>(x, M, K, warps, xq, s_a, stream);
  if (cpw <= 2) return launch_rows_cpw<LOG4G, 2>(x, M, K, warps, xq, s_a, stream);
  if (cpw <= 4) return launch_rows_cpw<LOG4G, 4>(x, M, K, warps, xq, s_a, stream);
  return note_cuda(cudaErrorInvalidValue, "small prologue: shape");
}

template <int SINK, int NT, int W>
cudaError_t launch_gemv_sink(const GemvParams& prm, int grid, int smem, cudaStream_t stream) {
  static std::atomic<int> cache[64];
  const void* kfn = reinterpret_cast<const void*>(w4a4_gemv_kernel<SINK, NT, W>);
  cudaError_t e = ensure_dynamic_smem(kfn, smem, cache);
  if (e != cudaSuccess) return note_cuda(e, "small GEMM: dynamic shared memory attribute");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid), 1, 1);
  cfg.blockDim = dim3(32 * W, 1, 1);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return note_cuda(cudaLaunchKernelEx(&cfg, w4a4_gemv_kernel<SINK, NT, W>, prm), "small GEMM: launch");
}

template <int NT, int W>
cudaError_t launch_gemv_nt(const GemvParams& prm, int grid, int smem, GemmSink sink, cudaStream_t stream) {
  switch (sink) {
    case GemmSink::kBF16: return launch_gemv_sink<0, NT, W>(prm, grid, smem, stream);
    case GemmSink::kF32: return launch_gemv_sink<1, NT, W>(prm, grid, smem, stream);
    default: return launch_gemv_sink<2, NT, W>(prm, grid, smem, stream);
  }
}

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

}  // namespace

size_t small_gemm_scratch_bytes(int M, int N, int K) {
  const GemvPlan g = gemv_plan(N, K);
  const size_t mt = M <= 8 ? 8 : 16;
  size_t bytes = 256;
  if (g.parts > 1)
    bytes = round256(static_cast<size_t>(g.tiles) * 4) +
            round256(static_cast<size_t>(g.tiles) * g.parts * mt * kSlabRows * sizeof(int32_t));
  return bytes;
}

cudaError_t launch_small_rotate_quant(const uint16_t* x, int M, int K, int group, uint8_t* xq, float* s_a,
                                      cudaStream_t stream) {
  if (M < 1 || M > kSmallMaxM) return note_cuda(cudaErrorInvalidValue, "small prologue: M");
  cudaError_t e;
  switch (group) {
    case 256: e = launch_rows<4>(x, M, K, xq, s_a, stream); break;
    case 64: e = launch_rows<3>(x, M, K, xq, s_a, stream); break;
    case 16: e = launch_rows<2>(x, M, K, xq, s_a, stream); break;
    default: return note_cuda(cudaErrorInvalidValue, "small prologue: group");
  }
  count_dispatch(4);
  return e;
}

cudaError_t launch_small_gemm(const uint8_t* xq, const float* s_a, const uint8_t* Wq, const float* s_w,
                              const uint16_t* bias, int M, int N, int K, void* out, GemmSink sink, void* scratch,
                              size_t scratch_bytes, cudaStream_t stream) {
  if (M < 1 || M > kSmallMaxM) return note_cuda(cudaErrorInvalidValue, "small GEMM: M");
  const GemvPlan g = gemv_plan(N, K);
  if (scratch_bytes < small_gemm_scratch_bytes(M, N, K)) return note_cuda(cudaErrorInvalidValue, "small GEMM: scratch");
  const long long grid = static_cast<long long>(g.tiles) * g.parts;
  if (grid > (1ll << 31) - 1) return note_cuda(cudaErrorInvalidValue, "small GEMM: shape");
  GemvParams prm{};
  prm.Wq = Wq;
  prm.xq = xq;
  prm.s_a = s_a;
  prm.s_w = s_w;
  prm.bias = bias;
  prm.out = out;
  prm.M = M;
  prm.N = N;
  prm.K = K;
  prm.nb = g.nb;
  prm.parts = g.parts;
  const int part_blocks = (g.nb + g.parts - 1) / g.parts;
  // 64 bytes modulo 128 per row: rows r and r + 1 of a fragment load hit
  // different halves of the banks.
  prm.row_stride = (part_blocks * kBlockBytes + 127) / 128 * 128 + 64;
  if (g.parts > 1) {
    prm.ctr = static_cast<uint32_t*>(scratch);
    prm.part = reinterpret_cast<int32_t*>(static_cast<uint8_t*>(scratch) + round256(static_cast<size_t>(g.tiles) * 4));
    cudaError_t e = cudaMemsetAsync(scratch, 0, static_cast<size_t>(g.tiles) * 4, stream);
    if (e != cudaSuccess) return note_cuda(e, "small GEMM: clear counters");
  }
  const int smem = kSlabRows * prm.row_stride + 128;
  const bool wide = part_blocks > kLongKBlocks;  // long K ranges: 8 warps, fewer blocks per warp
  cudaError_t e;
  if (M <= 8)
    e = wide ? launch_gemv_nt<1, 8>(prm, static_cast<int>(grid), smem, sink, stream)
             : launch_gemv_nt<1, 4>(prm, static_cast<int>(grid), smem, sink, stream);
  else
    e = wide ? launch_gemv_nt<2, 8>(prm, static_cast<int>(grid), smem, sink, stream)
             : launch_gemv_nt<2, 4>(prm, static_cast<int>(grid), smem, sink, stream);
  count_dispatch(5);
  return e;
}

}  // namespace convrot
