/*
 * convrot.h -- C ABI of the B200 (sm_100a) ConvRot W4A4 quantized Linear.
 *
 * The method (sources by page title and section):
 *   "Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
 *   fallback)", intro paragraph: the weights are rotated by the ConvRot
 *   transform (a regular Hadamard over groups of 256) and stored as signed
 *   INT4, two codes to a byte; the activations get the same rotation at run
 *   time and are quantized to INT4 on the fly; no calibration data is used.
 *   Same card, speed table: one kernel does the rotation and an s4 MMA whose
 *   integer product is rescaled by s_a[m] * s_w[n] (rank one).
 *   "rockerBOO/qwen3-4b-nvfp4-convrot", file table: the Hadamard rotation is
 *   applied per group of 256 channels.
 *   "Nicolaslas/Rebels_w4a8s", "What I do differently": the ConvRot group is
 *   exactly 256, so K must be divisible by 256.
 *
 * Definitions used by every entry point:
 *   R        block-diagonal rotation along K: each group of 256 channels is
 *            multiplied by H/16, H = H4 (x) H4 (x) H4 (x) H4 with
 *            H4 = [[1,1,1,-1],[1,1,-1,1],[1,-1,1,1],[-1,1,1,1]], evaluated
 *            in fp32 as 4 radix-4 butterfly stages (stride 1, 4, 16, 64; each
 *            butterfly (a,b,c,d) -> (p+t, p-t, q+r, r-q) with p=a+b, q=a-b,
 *            r=c+d, t=c-d, no FMA contraction), then one multiply by 1/16.
 *   scale    s[r] = amax_k |R(v)[r,k]| / 7 (one fp32 IEEE division), per row.
 *   code     q = clamp(rint(R(v)/s), -8, 7), a true IEEE fp32 division and
 *            round half to even; s == 0 gives q == 0.
 *   packing  byte i of a row = (q[2i] & 0xF) | ((q[2i+1] & 0xF) << 4).
 *   linear   acc[m,n] = sum_k q_a[m,k] q_w[n,k] (exact int32), then
 *            y[m,n] = acc * s_a[m] * s_w[n] + bias[n], rounded to bf16 (RNE).
 *
 * Conventions for every call:
 *   - All pointers are DEVICE pointers, owned by the caller; the library never
 *     allocates per call.  Pointers must be 16-byte aligned.
 *   - Matrices are row-major and dense (row stride == number of columns).
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream); every
 *     call only enqueues work on it and returns.  Argument errors are reported
 *     synchronously, before anything is enqueued.  Launch failures return
 *     CONVROT_ERR_CUDA.  A device-side wait that gave up (see
 *     convrot_device_error) is reported asynchronously.
 *   - Shapes: M >= 1, N >= 1 (N % 8 == 0 for the linear/GEMM outputs),
 *     K >= 256 with K % 256 == 0, K <= 32768.
 *   - The GPU must be sm_100 (B200); anything else gives CONVROT_ERR_DEVICE.
 */
#ifndef CONVROT_H_
#define CONVROT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  CONVROT_OK = 0,
  CONVROT_ERR_NULL = 1,      /* a required pointer is NULL */
  CONVROT_ERR_SHAPE = 2,     /* M < 1, N < 1, N % 8, K % 256, K > 32768 */
  CONVROT_ERR_ALIGN = 3,     /* a pointer is not 16-byte aligned */
  CONVROT_ERR_DEVICE = 4,    /* no CUDA device, or the current device is not sm_100 */
  CONVROT_ERR_WORKSPACE = 5, /* workspace NULL or smaller than the *_workspace_size */
  CONVROT_ERR_CUDA = 6,      /* a CUDA runtime/driver call failed */
  CONVROT_ERR_TIMEOUT = 7    /* a bounded device-side wait expired (async) */
} convrot_status_t;

/* Human-readable name of a status code (static storage, never NULL). */
const char *convrot_status_string(convrot_status_t status);

/* Offline weight preparation ("weights ... with ConvRot rotation", packed
 * signed INT4, per-output-channel scales; Qwen-Image-Edit-2511 W4A4 card,
 * intro).  Rotates each row n of W along K, quantizes it with its own scale
 * s_w[n] and packs it.
 *   W    [N, K] bf16 bits      (input)
 *   Wq   [N, K/2] uint8        (output, packed codes)
 *   s_w  [N] float             (output)
 * Bit-identical to convrot_rotate_quant applied to W. */
convrot_status_t convrot_pack_weight(const uint16_t *W, int N, int K, uint8_t *Wq, float *s_w,
                                     void *stream);

/* Online activation prologue (rotation + dynamic per-token INT4, same card,
 * intro).
 *   x    [M, K] bf16 bits      (input)
 *   xq   [M, K/2] uint8        (output, packed codes)
 *   s_a  [M] float             (output, per-token scale) */
convrot_status_t convrot_rotate_quant(const uint16_t *x, int M, int K, uint8_t *xq, float *s_a,
                                      void *stream);

/* Bytes of workspace w4a4_gemm* needs for (M, N, K) (0 for an invalid
 * shape).  M > 16: the activation codes widened to bytes, M * K rounded up
 * to 256.  M <= 16 (the small-M kernel, which reads the packed codes as they
 * are): 1 KB of arrival counters and the partial tiles of output tiles whose
 * K range is split between CTAs, 2 * 160 * 128 * (M <= 8 ? 8 : 16) int32. */
size_t convrot_gemm_workspace_size(int M, int N, int K);

/* Integer GEMM with the rank-one epilogue (the card's rank-one s4 MMA, same card,
 * speed table) on codes that are already quantized.
 *   xq   [M, K/2] uint8, s_a [M] float     (from convrot_rotate_quant)
 *   Wq   [N, K/2] uint8, s_w [N] float     (from convrot_pack_weight)
 *   bias [N] bf16 bits, or NULL for none
 *   y    [M, N] bf16 bits                  (output)
 *   workspace: device memory of at least convrot_gemm_workspace_size bytes
 *   (scratch, contents undefined afterwards).
 * Every code nibble is accepted, including -8. */
convrot_status_t w4a4_gemm(const uint8_t *xq, const float *s_a, const uint8_t *Wq,
                           const float *s_w, const uint16_t *bias, int M, int N, int K,
                           uint16_t *y, void *workspace, size_t workspace_bytes, void *stream);

/* Same kernels, different sink: the exact int32 accumulator acc[M, N]
 * (scales and bias are not applied; s_a / s_w / bias are ignored and may be
 * NULL).  For parity checks. */
convrot_status_t w4a4_gemm_s32(const uint8_t *xq, const uint8_t *Wq, int M, int N, int K,
                               int32_t *acc, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Same kernels, fp32 sink y32[M, N] = acc * s_a[m] * s_w[n] + bias[n] before
 * the bf16 rounding.  For parity checks. */
convrot_status_t w4a4_gemm_f32(const uint8_t *xq, const float *s_a, const uint8_t *Wq,
                               const float *s_w, const uint16_t *bias, int M, int N, int K,
                               float *y32, void *workspace, size_t workspace_bytes,
                               void *stream);

/* Bytes of workspace convrot_w4a4_linear* needs for (M, N, K) (0 for an
 * invalid shape): M * K bytes of activation codes and the M per-token
 * scales, each part rounded up to 256 bytes; for M <= 16 followed by the
 * small-M GEMM's counters and partial tiles (see convrot_gemm_workspace_size). */
size_t convrot_w4a4_workspace_size(int M, int N, int K);

/* The fused ConvRot W4A4 Linear: y = W4A4(x) with x rotated and quantized
 * online (same card, intro and speed table).
 *   x    [M, K] bf16 bits  (input activations)
 *   Wq   [N, K/2] uint8, s_w [N] float (from convrot_pack_weight)
 *   bias [N] bf16 bits or NULL
 *   y    [M, N] bf16 bits  (output)
 *   workspace: >= convrot_w4a4_workspace_size bytes of device scratch (holds
 *   the activation codes and scales between the two kernels).
 * Kernels.  M > 16: the rotate/quant prologue, then the tcgen05 tensor-core
 * GEMM (kind::i8, accumulators in tensor memory).  M <= 16: a prologue with
 * one CTA per token, then the bandwidth-bound small-M GEMM, which streams the
 * packed weights with TMA into a ring of shared-memory stages and multiplies
 * with mma.sync s8 (both operands widened from nibbles in registers).  Both
 * give the same bits.
 * Ordering.  Every GEMM here is launched with programmatic dependent launch:
 * it starts streaming Wq while the preceding kernel on the stream finishes,
 * and waits for that kernel before it reads anything else.  Wq must therefore
 * be complete before the preceding kernel starts; convrot_pack_weight and any
 * kernel that does not trigger its dependents early (griddepcontrol) meet
 * this, as does a synchronisation. */
convrot_status_t convrot_w4a4_linear(const uint16_t *x, const uint8_t *Wq, const float *s_w,
                                     const uint16_t *bias, int M, int N, int K, uint16_t *y,
                                     void *workspace, size_t workspace_bytes, void *stream);

/* The fused Linear with an fp32 sink (before the bf16 rounding).  For parity
 * checks. */
convrot_status_t convrot_w4a4_linear_f32(const uint16_t *x, const uint8_t *Wq, const float *s_w,
                                         const uint16_t *bias, int M, int N, int K, float *y32,
                                         void *workspace, size_t workspace_bytes, void *stream);

/* The fused Linear without a caller-supplied workspace, for callers that
 * cannot allocate device memory: code running inside a host framework that
 * owns all device allocations and forbids side allocations, fixed-budget
 * deployments that must not grow their footprint after start-up, and plugin
 * or foreign-language callers with no binding to a CUDA allocator.  The pages
 * have no counterpart of this call; it is a deployment convenience.
 *   Same arguments and results as convrot_w4a4_linear, minus the workspace.
 *   Scratch: a static 32 MiB device array inside the library (held by every
 *   GPU that loads the library until the process exits).  Shapes whose
 *   convrot_w4a4_workspace_size exceeds 32 MiB return CONVROT_ERR_WORKSPACE
 *   (convrot_last_error says by how much).  Allocates nothing: no cudaMalloc,
 *   no cudaFree.
 *   The first call on each device looks up the array's device address
 *   (cudaGetSymbolAddress) with that device current; make that first call
 *   before any stream capture.  The address is kept per device and looked up
 *   again when the device's current CUDA context changes (for example after
 *   cudaDeviceReset); the lookup is guarded, so several host threads may make
 *   their first calls at once.  A device other than sm_100 gives
 *   CONVROT_ERR_DEVICE before any lookup.
 *   Every call shares the one array and it keeps the last call's contents, so
 *   calls that overlap on the GPU (e.g. on two streams at once) race. */
convrot_status_t convrot_w4a4_linear_noalloc(const uint16_t *x, const uint8_t *Wq,
                                             const float *s_w, const uint16_t *bias, int M,
                                             int N, int K, uint16_t *y, void *stream);

/* The two launches that make up convrot_w4a4_linear, for callers that want
 * to time or schedule them separately; convrot_w4a4_linear is exactly
 * convrot_w4a4_quantize followed by convrot_w4a4_gemm_quantized on the same
 * workspace and stream.
 *   convrot_w4a4_quantize: x [M, K] bf16 -> the workspace (activation codes
 *     in the GEMM's operand layout, packed for M <= 16, + per-token scales).
 *     workspace_bytes >= convrot_w4a4_workspace_size(M, N, K) for every N it
 *     will be used with.
 *   convrot_w4a4_gemm_quantized: workspace (from convrot_w4a4_quantize with
 *     the same M, K) x Wq -> y [M, N] bf16.  It does not change the codes or
 *     scales, so one quantization may serve several GEMMs (e.g. projections
 *     that share their input), one after another on one stream: for M <= 16
 *     the GEMM keeps its counters and partial tiles in the workspace's
 *     scratch part (and leaves the counters at zero). */
convrot_status_t convrot_w4a4_quantize(const uint16_t *x, int M, int K, void *workspace,
                                       size_t workspace_bytes, void *stream);
convrot_status_t convrot_w4a4_gemm_quantized(const uint8_t *Wq, const float *s_w,
                                             const uint16_t *bias, int M, int N, int K,
                                             uint16_t *y, void *workspace,
                                             size_t workspace_bytes, void *stream);

/* ---- rotation group-size variants ---------------------------------------------
 * "JoaoZaokk/Z-Image-Turbo-W4A4-ConvRot", "Where Z-Image sits": the
 * convrot_groupsize ablation runs groups of 256, 64 and 16 (an outlier is
 * shared out over the N channels of its rotation group).  These entry points are the ones
 * above with the group as a parameter: each group of `group` (256, 64 or 16)
 * channels is multiplied by H4 Kronecker'd log4(group) times, evaluated as
 * the first log4(group) butterfly stages of R (strides 1, 4, 16), then by
 * 2^-log4(group); the per-token scale, the codes, the packing and the GEMM are
 * unchanged.  group == 256 is exactly the default path.  Other groups give
 * CONVROT_ERR_SHAPE; K % 256 == 0 as everywhere. */
convrot_status_t convrot_rotate_quant_g(const uint16_t *x, int M, int K, int group, uint8_t *xq,
                                        float *s_a, void *stream);
convrot_status_t convrot_pack_weight_g(const uint16_t *W, int N, int K, int group, uint8_t *Wq,
                                       float *s_w, void *stream);
convrot_status_t convrot_w4a4_quantize_g(const uint16_t *x, int M, int K, int group, void *workspace,
                                         size_t workspace_bytes, void *stream);
convrot_status_t convrot_w4a4_linear_g(const uint16_t *x, const uint8_t *Wq, const float *s_w,
                                       const uint16_t *bias, int M, int N, int K, int group,
                                       uint16_t *y, void *workspace, size_t workspace_bytes,
                                       void *stream);
convrot_status_t convrot_w4a4_linear_g_f32(const uint16_t *x, const uint8_t *Wq, const float *s_w,
                                           const uint16_t *bias, int M, int N, int K, int group,
                                           float *y32, void *workspace, size_t workspace_bytes,
                                           void *stream);

/* ---- int8 W8A8 formats -------------------------------------------------------
 * The pages store their quality-sensitive layers in int8 next to the W4A4
 * ones, and both run on the same integer tensor-core path:
 *   W8A8_INT8_TENSORWISE  stock "int8_tensorwise" ("Qwen-Image-Edit-2511 --
 *     INT4 tensorwise W4A4 (+ConvRot, mixed int8 fallback)", intro: the
 *     attention value/output projections and adaLN Linears): no rotation, one
 *     scale for the whole weight tensor and one dynamic scale for the whole
 *     activation tensor.
 *   W8A8_CONVROT_INT8_ROW  "ConvRot INT8 (row-scaled)" ("rockerBOO/qwen3-4b-
 *     nvfp4-convrot", file table: the attention projections): the group-256
 *     rotation R above, one scale per weight row and one dynamic scale per
 *     activation row (token).
 * Codes: s = amax / 127 (one fp32 IEEE division), q = clamp(rint(v / s),
 * -127, 127) with a true division and round half to even, s == 0 -> q = 0;
 * int8 [rows, K] row-major, natural order.  Linear: acc = sum_k q_x q_w
 * (exact int32), y = acc * s_x[m] * s_w[n] + bias[n] -> bf16 (a per-tensor
 * scale is used for every m / n).  Same shape rules as above (K % 256 == 0,
 * N % 8 == 0, 16-byte-aligned pointers). */
typedef enum { W8A8_INT8_TENSORWISE = 0, W8A8_CONVROT_INT8_ROW = 1 } w8a8_format_t;

/* Bytes of workspace w8a8_quantize / w8a8_pack_weight / w8a8_linear* need
 * for (M, N, K) in `format` (0 for an invalid shape or format): the int8
 * activation codes (M * K), the activation scales and 4 bytes of reduction
 * scratch, each part rounded up to 256 bytes. */
size_t w8a8_workspace_size(int M, int N, int K, int format);

/* Quantize x [M, K] bf16 to int8 codes x8 [M, K] and scales s_x ([1] for
 * int8_tensorwise, [M] for ConvRot INT8 row-scaled).  workspace: at least
 * w8a8_workspace_size(M, 8, K, format) bytes of device scratch (only its
 * reduction scratch is used). */
convrot_status_t w8a8_quantize(const uint16_t *x, int M, int K, int format, int8_t *x8, float *s_x,
                               void *workspace, size_t workspace_bytes, void *stream);

/* Offline weight preparation: the same quantizer on W [N, K] bf16 -> Wq8
 * [N, K] int8 and s_w ([1] tensorwise, [N] row-scaled). */
convrot_status_t w8a8_pack_weight(const uint16_t *W, int N, int K, int format, int8_t *Wq8, float *s_w,
                                  void *workspace, size_t workspace_bytes, void *stream);

/* Integer GEMM with the rank-one epilogue on int8 codes: y [M, N] bf16 from
 * x8 [M, K], s_x, Wq8 [N, K], s_w (per `format`), bias [N] or NULL. */
convrot_status_t w8a8_gemm(const int8_t *x8, const float *s_x, const int8_t *Wq8, const float *s_w,
                           const uint16_t *bias, int M, int N, int K, int format, uint16_t *y,
                           void *stream);

/* Same kernel, fp32 sink y32 [M, N] before the bf16 rounding (parity). */
convrot_status_t w8a8_gemm_f32(const int8_t *x8, const float *s_x, const int8_t *Wq8, const float *s_w,
                               const uint16_t *bias, int M, int N, int K, int format, float *y32,
                               void *stream);

/* Same kernel, the exact int32 accumulator acc [M, N] (parity). */
convrot_status_t w8a8_gemm_s32(const int8_t *x8, const int8_t *Wq8, int M, int N, int K, int32_t *acc,
                               void *stream);

/* The fused int8 Linear: x [M, K] bf16 quantized online (per `format`), times
 * Wq8 / s_w from w8a8_pack_weight, plus bias -> y [M, N] bf16.  workspace:
 * >= w8a8_workspace_size(M, N, K, format) bytes. */
convrot_status_t w8a8_linear(const uint16_t *x, const int8_t *Wq8, const float *s_w, const uint16_t *bias,
                             int M, int N, int K, int format, uint16_t *y, void *workspace,
                             size_t workspace_bytes, void *stream);

/* The fused int8 Linear with an fp32 sink (parity). */
convrot_status_t w8a8_linear_f32(const uint16_t *x, const int8_t *Wq8, const float *s_w,
                                 const uint16_t *bias, int M, int N, int K, int format, float *y32,
                                 void *workspace, size_t workspace_bytes, void *stream);

/* ---- asymmetric W4A8 ("asym_w4a8_int8") ------------------------------------
 *
 * The W4A8 layout of "Nicolaslas/Rebels_w4a8s" ("What's inside a file") and
 * "JoaoZaokk/Qwen3-VL-4B-W4A8-ConvRot" (file table: asym_w4a8_int8, group
 * 16, convrot_groupsize 256): per Linear W [N, K], in the ConvRot-rotated
 * basis (group 256),
 *   idx       [N, K/2]  uint8   4-bit codebook indices 0..15, two per byte,
 *                               low nibble = even k
 *   s_rel     [N, K/16] uint8   e4m3 ("fn": bias 7, no infinities) scale of
 *                               each group of 16 consecutive k
 *   s_channel [N]       float   per-output-channel scale
 *   codebook  [16]      float   the tensor's levels
 * The int8 weight the tensor cores multiply is
 *   w8[n, k] = clamp(rint(codebook[idx[n, k]] * s_rel[n, k / 16]), -127, 127)
 * (one fp32 multiply, round half to even, a NaN product -> 0); activations
 * are the ConvRot INT8 row-scaled codes (w8a8_quantize with
 * W8A8_CONVROT_INT8_ROW: rotation, s_a = amax / 127 per token); then
 *   y[m, n] = bf16(((float)acc * s_a[m]) * s_channel[n] + bias[n]),
 *   acc = sum_k x8[m, k] * w8[n, k] (exact int32).
 * The decode rule is a reading: the pages give the storage and say that the
 * arithmetic is int8.  Shapes as for W4A4 (K % 256 == 0, N % 8 == 0, M >= 1);
 * every pointer 16-byte aligned device memory owned by the caller.  The
 * weight tensors (converted offline) are inputs; no call here converts bf16
 * weights to this format. */

/* Bytes of workspace asym_w4a8_linear* need for M tokens (the int8 codes and
 * scales of the activations). */
size_t asym_w4a8_workspace_size(int M, int N, int K);

/* x8 [M, K] int8 and s_a [M] from w8a8_quantize(W8A8_CONVROT_INT8_ROW), the
 * weight tensors above, bias [N] or NULL -> y [M, N] bf16.  The decode runs
 * inside the GEMM (no int8 weight copy is written). */
convrot_status_t asym_w4a8_gemm(const int8_t *x8, const float *s_a, const uint8_t *idx, const uint8_t *s_rel,
                                const float *codebook, const float *s_channel, const uint16_t *bias, int M, int N,
                                int K, uint16_t *y, void *stream);

/* Same kernel, fp32 sink y32 [M, N] before the bf16 rounding (parity). */
convrot_status_t asym_w4a8_gemm_f32(const int8_t *x8, const float *s_a, const uint8_t *idx,
                                    const uint8_t *s_rel, const float *codebook, const float *s_channel,
                                    const uint16_t *bias, int M, int N, int K, float *y32, void *stream);

/* Same kernel, the exact int32 accumulator acc [M, N] (parity). */
convrot_status_t asym_w4a8_gemm_s32(const int8_t *x8, const uint8_t *idx, const uint8_t *s_rel,
                                    const float *codebook, int M, int N, int K, int32_t *acc, void *stream);

/* The fused asymmetric W4A8 Linear: x [M, K] bf16 rotated and quantized
 * online, then the GEMM above -> y [M, N] bf16.  workspace: >=
 * asym_w4a8_workspace_size(M, N, K) bytes. */
convrot_status_t asym_w4a8_linear(const uint16_t *x, const uint8_t *idx, const uint8_t *s_rel,
                                  const float *codebook, const float *s_channel, const uint16_t *bias, int M,
                                  int N, int K, uint16_t *y, void *workspace, size_t workspace_bytes,
                                  void *stream);

/* The fused asymmetric W4A8 Linear with an fp32 sink (parity). */
convrot_status_t asym_w4a8_linear_f32(const uint16_t *x, const uint8_t *idx, const uint8_t *s_rel,
                                      const float *codebook, const float *s_channel, const uint16_t *bias,
                                      int M, int N, int K, float *y32, void *workspace, size_t workspace_bytes,
                                      void *stream);

/* Device-side error word of the current device: bit 0 = a bounded wait
 * inside a kernel expired (the kernel skipped its remaining work and
 * returned; its outputs are invalid).  Synchronizes `stream`, copies the word
 * to *code and clears it.  Returns CONVROT_ERR_TIMEOUT when the word was
 * non-zero, CONVROT_OK otherwise. */
convrot_status_t convrot_device_error(void *stream, uint32_t *code);

/* Exercises the failure path of the bounded device-side waits (the failure
 * detection described above): launches a one-thread kernel that waits on a
 * barrier nothing ever arrives at, for at most limit_us microseconds
 * (1..1000000).  Afterwards convrot_device_error reports CONVROT_ERR_TIMEOUT
 * (and clears the word).  While the word is set, every later bounded wait
 * gives up at once, so call convrot_device_error before further work.  Touches
 * no caller memory; the context stays usable. */
convrot_status_t convrot_selftest_timeout(unsigned int limit_us, void *stream);

/* Host-side count of how many times each kernel path was enqueued by this
 * process: counts[0] = rotate/quant prologue, [1] = packed-code unpack pass,
 * [2] = tensor-core GEMM over whole output tiles, [3] = the same GEMM with
 * each tile's K split over a thread-block cluster (few tiles; the partial
 * tiles are summed exactly in shared memory), [4] = the small-M prologue
 * (one CTA per token), [5] = the small-M GEMM (M <= 16).  `n` is the array
 * length; at most 6 are written. */
void convrot_dispatch_counts(uint64_t *counts, int n);

/* Description of the last CUDA call of this library that failed on the
 * calling thread (which call, error name and text); "" if none.  Valid until
 * the next failing call on the same thread. */
const char *convrot_last_error(void);

/* Measurement of the dense int8 tensor-core rate of the current device (the
 * denominator of the GEMM's roofline fraction; the pages quote no B200
 * figure).  Launches one CTA per SM; one thread per CTA issues 16 * iters
 * back-to-back tcgen05.mma.kind::i8 of shape 128 x N x 32 (s8 x s8 -> s32)
 * whose operands stay on chip: B in shared memory, A in shared memory
 * (a_in_tmem == 0) or in tensor memory (a_in_tmem != 0, the form the W4A4
 * GEMM issues).  No global memory is touched except a per-CTA cycle count.
 *   N       16 .. 256, a multiple of 16
 *   iters   1 .. 2^20
 *   tops    (output) 2 * 128 * N * 32 * MMAs / wall time (CUDA events), 1e12/s
 *   cycles_per_mma (output) mean SM cycles per MMA of one CTA
 * Runs on the legacy default stream and synchronizes it (a host-blocking
 * diagnostic, not for use inside stream capture). */
convrot_status_t convrot_measure_mma_i8(int N, int a_in_tmem, int iters, double *tops,
                                        double *cycles_per_mma);

/* Library build identifier (static string). */
const char *convrot_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CONVROT_H_ */
