// kernels.cuh -- internal launch interface between the C ABI (api.cu) and the
// CUDA kernels (rotate_quant.cu, gemm.cu).  Not installed, not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

namespace convrot {

// Rows are processed by the prologue in 8-element chunks; the activation
// operand of the tensor-core GEMM stores each chunk's codes in the order
// (0, 2, 4, 6, 1, 3, 5, 7), the order in which a packed 32-bit word of weight
// nibbles splits into its low and high nibbles.

// Output sinks of the rotate/quant prologue (packed or s8 may be null).
struct RotateQuantOut {
  uint8_t* packed;  // [M, K/2] two codes per byte, or null
  int8_t* s8;       // [M, K] codes as signed bytes in chunk order (0,2,4,6,1,3,5,7), or null
  float* scale;     // [M]
  bool int8 = false;  // s8 holds 8-bit codes (amax / 127) in natural order instead
  int group = 256;    // rotation group: 256, 64 or 16 (int8: 256 only)
  // Let the next kernel launch while this one runs (programmatic dependent
  // launch).  Off for weight preparation: the GEMMs read weights before they
  // wait for their predecessor, so the kernel that writes weights must not
  // let any successor start before it has completed.
  bool early_trigger = true;
};

// The int8_tensorwise quantizer: one scale s = amax|x| / 127 for the whole
// [rows, K] tensor, codes clamp(rint(x / s), -127, 127), no rotation.
// scratch: 4 bytes of device memory (the amax while it is reduced).
cudaError_t launch_quant8_tensorwise(const uint16_t* x, size_t n, int8_t* codes, float* scale, uint32_t* scratch,
                                     cudaStream_t stream, bool early_trigger = true);

cudaError_t launch_rotate_quant(const uint16_t* x, int M, int K, RotateQuantOut out, cudaStream_t stream);

// Packed codes [M, K/2] -> signed-byte operand layout [M, K].
cudaError_t launch_unpack_codes(const uint8_t* packed, int M, int K, int8_t* s8, cudaStream_t stream);

enum class GemmSink : int { kBF16 = 0, kF32 = 1, kS32 = 2 };

constexpr int kMaxGemmGrid = 160;  // whole-tile CTAs (one per SM)

struct GemmTiling {
  int splits;       // 1: whole tiles round-robin; S in {2,4,8}: a cluster of S CTAs splits each tile's K
  int grid;         // CTAs launched
  int BT;           // tokens per tile (MMA N), multiple of 16 in [16, 192]
  int m_tiles;      // ceil(M / BT)
  int n_tiles;      // ceil(N / 128)
  int nstages;      // depth of the shared-memory TMA ring
  int smem_bytes;   // dynamic shared memory per CTA
  int acc_stride;   // tensor-memory columns per accumulator
  int a_slots;      // 64-column tensor-memory slots for unpacked weights
  int n_fast;       // whole-tile order: channel tile fastest (1) or token tile fastest (0)
};

// Weight kinds of the tensor-core GEMM.
constexpr int kW4 = 0;         // packed two's-complement 4-bit codes [N, K/2]
constexpr int kWInt8 = 1;      // int8 codes [N, K] (the W8A8 formats)
constexpr int kWCodebook = 2;  // packed 4-bit codebook indices [N, K/2], e4m3 group scales [N, K/16], codebook [16]

GemmTiling choose_tiling(int M, int N, int K, int num_sms, int wkind = kW4);

struct GemmArgs {
  const int8_t* xs8;      // [M, K] activation codes (operand layout; natural order for 8-bit codes)
  const float* s_a;       // [M], or [1] with sa_stride 0 (ignored by the s32 sink)
  const uint8_t* Wq;      // [N, K/2] packed weight codes or indices, or [N, K] int8 codes
  const float* s_w;       // [N], or [1] with sw_stride 0
  const uint16_t* bias;   // [N] or null
  void* out;              // [M, N] bf16 / f32 / s32
  int M, N, K;
  int wkind = kW4;        // kW4, kWInt8 or kWCodebook
  const uint8_t* s_rel = nullptr;   // [N, K/16] e4m3 group scales (kWCodebook)
  const float* codebook = nullptr;  // [16] levels (kWCodebook)
  int sa_stride = 1;      // 0: one activation scale for every row
  int sw_stride = 1;      // 0: one weight scale for every output channel
};

// Builds the tensor maps and launches the tensor-core GEMM.
cudaError_t launch_w4a4_gemm(const GemmArgs& a, GemmSink sink, const GemmTiling& t, cudaStream_t stream);

// The small-M path (small_m.cu): M <= kSmallMaxM tokens.  A one-CTA-per-row
// prologue writes packed codes (the convrot_rotate_quant layout) and scales;
// the GEMM reads the packed codes as they are, streams each 16-channel slab
// of packed weights with bulk copies and widens both operands in registers
// for mma.sync s8.  Where it splits K over several CTAs it sums the partial
// slabs through `scratch` (arrival counters, then partial slabs), whose size
// small_gemm_scratch_bytes gives; it clears the counters itself.
constexpr int kSmallMaxM = 16;
size_t small_gemm_scratch_bytes(int M, int N, int K);
cudaError_t launch_small_rotate_quant(const uint16_t* x, int M, int K, int group, uint8_t* xq, float* s_a,
                                      cudaStream_t stream);
cudaError_t launch_small_gemm(const uint8_t* xq, const float* s_a, const uint8_t* Wq, const float* s_w,
                              const uint16_t* bias, int M, int N, int K, void* out, GemmSink sink, void* scratch,
                              size_t scratch_bytes, cudaStream_t stream);

// Host-side dispatch counters (see convrot_dispatch_counts): 0 rotate_quant,
// 1 unpack_codes, 2 tensor-core GEMM, 3 split-K cluster GEMM, 4 small-M
// prologue, 5 small-M GEMM.
constexpr int kDispatchKinds = 6;
void count_dispatch(int which);

// Remember the last failing CUDA call (see convrot_last_error).
cudaError_t note_cuda(cudaError_t e, const char* where);

// Raise a kernel's dynamic shared-memory limit to `bytes` on the current
// device if needed (checked against the opt-in maximum minus static usage).
// `cache` is per kernel: one entry per device (the limit already set).  Safe
// to call from several host threads.
cudaError_t ensure_dynamic_smem(const void* kernel, int bytes, std::atomic<int>* cache);

}  // namespace convrot
