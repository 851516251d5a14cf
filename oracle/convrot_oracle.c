/*
 * convrot_oracle.c -- plain, slow, single-threaded CPU oracle for the ConvRot
 * W4A4 quantized Linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this file's library.  The CUDA
 * library never links, includes or calls it, and it shares no code, header,
 * table or constant generator with the CUDA path.
 *
 * What it computes (sources, by page title and section):
 *  - "Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
 *    fallback)" (HF card, intro paragraph): the weights go through the
 *    ConvRot rotation (a regular Hadamard over groups of 256) and are stored
 *    as signed INT4, two codes to a byte; the activations get the same
 *    rotation at run time and are quantized to INT4 on the fly; no
 *    calibration data.  Speed table: the integer product of an s4 MMA is
 *    rescaled by s_a[m] * s_w[n] (rank one).
 *  - "rockerBOO/qwen3-4b-nvfp4-convrot" (file table): group-wise Hadamard
 *    rotation, group size 256.
 *  - "Nicolaslas/Rebels_w4a8s" ("What I do differently"): the ConvRot group is
 *    exactly 256, so K must be a multiple of 256.
 *  - "JoaoZaokk/Z-Image-Turbo-W4A4-ConvRot" ("Where Z-Image sits"): group
 *    sizes 256, 64 and 16 exist (the rotation of order 4^s for s = 4, 3, 2).
 *
 * Readings the pages leave open, fixed here (each is listed in the design
 * notes):
 *  - The regular Hadamard of order 4 is H4 = [[1,1,1,-1],[1,1,-1,1],
 *    [1,-1,1,1],[-1,1,1,1]]; order 256 is H4 (x) H4 (x) H4 (x) H4, scaled by
 *    1/16 so that it is orthonormal.
 *  - It is evaluated as 4 radix-4 butterfly stages, stride 1 first, then 4,
 *    16, 64.  One butterfly on (a, b, c, d) forms p=a+b, q=a-b, r=c+d,
 *    t=c-d and writes (p+t, p-t, q+r, r-q).  Every add is one IEEE fp32
 *    round-to-nearest add with no contraction (compile with
 *    -ffp-contract=off).  The 1/16 is applied last, as one fp32 multiply.
 *  - Per-token scale: s_a[m] = amax_k |x'[m,k]| / 7 (one IEEE fp32 divide),
 *    over the whole row (all groups).  amax == 0 gives s_a = 0 and all codes 0.
 *  - Code: q = clamp(rint(x' / s_a), -8, 7), rint = round half to even, the
 *    quotient is a true IEEE fp32 division.
 *  - Packing: byte i of a row = (q[2i] & 0xF) | ((q[2i+1] & 0xF) << 4).
 *  - GEMM: acc[m,n] = sum_k q_a[m,k] * q_w[n,k] in int64.
 *  - Epilogue: y32 = ((float)acc * s_a[m]) * s_w[n] + (float)bias[n], each op
 *    one fp32 RN op; y = bf16 round-to-nearest-even of y32.
 *
 * The int8 formats the pages use next to W4A4 (a W8A8 path: int8 weights,
 * int8 activations, int32 accumulation, the same rank-one rescale):
 *  - "Qwen-Image-Edit-2511 -- INT4 tensorwise W4A4 (+ConvRot, mixed int8
 *    fallback)", intro: the card keeps the layers that are sensitive to
 *    quantization (among them the attention value and output projections)
 *    in the stock "int8_tensorwise" format -- read as one scale for the
 *    whole weight tensor and one dynamic scale for the whole activation
 *    tensor, no rotation.
 *  - "rockerBOO/qwen3-4b-nvfp4-convrot", file table and notes: "ConvRot INT8
 *    (row-scaled)" -- the group-256 rotation, then int8 with one scale per
 *    weight row; read here with one dynamic scale per activation row (token).
 *  Readings for both: s = amax / 127 (IEEE fp32 divide), q = clamp(rint(v /
 *  s), -127, 127) with a true division and round half to even, s = 0 gives
 *  q = 0; the epilogue is the same rank-one rescale (a per-tensor scale is a
 *  constant vector).
 *
 * The asymmetric W4A8 format ("asym_w4a8_int8": 4-bit codebook indices, an
 * fp8 scale per 16 weights, a per-channel scale, a 16-level codebook per
 * tensor) is at the end of the file, with its own sources and readings, and
 * the offline converter that fits the codebook (Lloyd's algorithm).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_ERR_SHAPE 1
#define ORACLE_ERR_OVERFLOW 2
#define ORACLE_ERR_NOMEM 3

/* ---- bf16 <-> fp32 (plain definitions) -------------------------------- */

/* bf16 is the top 16 bits of an IEEE binary32, so widening is a shift. */
static float bf16_bits_to_f32(uint16_t h) {
  uint32_t u = ((uint32_t)h) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round-to-nearest-even of binary32 to its top 16 bits; NaN stays NaN. */
static uint16_t f32_to_bf16_bits_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

uint16_t oracle_f32_to_bf16(float f) { return f32_to_bf16_bits_rne(f); }
float oracle_bf16_to_f32(uint16_t h) { return bf16_bits_to_f32(h); }

/* ---- rotation ----------------------------------------------------------- */

/* log4 of a supported group size (16, 64, 256), or -1. */
static int group_log4(int group) {
  switch (group) {
    case 16: return 2;
    case 64: return 3;
    case 256: return 4;
    default: return -1;
  }
}

/* One group of G = 4^S values, in place: S radix-4 stages (stride 1, 4, 16,
 * ...), then one multiply by 1/sqrt(G) = 2^-S. */
static void rotate_group(float *v, int S) {
  int G = 1 << (2 * S);
  for (int s = 0; s < S; ++s) {
    int st = 1 << (2 * s);
    for (int i = 0; i < G; ++i) {
      if (((i / st) & 3) != 0) continue; /* digit s of i must be 0 */
      float a = v[i], b = v[i + st], c = v[i + 2 * st], d = v[i + 3 * st];
      float p = a + b;
      float q = a - b;
      float r = c + d;
      float t = c - d;
      v[i] = p + t;
      v[i + st] = p - t;
      v[i + 2 * st] = q + r;
      v[i + 3 * st] = r - q;
    }
  }
  float scale = ldexpf(1.0f, -S);
  for (int i = 0; i < G; ++i) v[i] = v[i] * scale;
}

/* In-place block-diagonal rotation of an fp32 [M, K] matrix, group by group
 * along K.  Returns ORACLE_ERR_SHAPE when K is not a multiple of the group. */
int oracle_rotate_rows_f32(float *data, int M, int K, int group) {
  int S = group_log4(group);
  if (S < 0 || M < 0 || K < 0 || K % group != 0) return ORACLE_ERR_SHAPE;
  for (int m = 0; m < M; ++m)
    for (int g = 0; g < K / group; ++g) rotate_group(data + (size_t)m * K + (size_t)g * group, S);
  return ORACLE_OK;
}

/* ---- packing -------------------------------------------------------------- */

/* Two signed 4-bit codes per byte, the even index in the low nibble. */
void oracle_pack_codes(const int8_t *q, int64_t n, uint8_t *out) {
  for (int64_t i = 0; i < n / 2; ++i)
    out[i] = (uint8_t)(((uint8_t)q[2 * i] & 0x0Fu) | (((uint8_t)q[2 * i + 1] & 0x0Fu) << 4));
}

/* Inverse of oracle_pack_codes: two's-complement sign extension of nibbles. */
void oracle_unpack_codes(const uint8_t *in, int64_t n, int8_t *q) {
  for (int64_t i = 0; i < n / 2; ++i) {
    int lo = in[i] & 0x0F, hi = (in[i] >> 4) & 0x0F;
    q[2 * i] = (int8_t)(lo >= 8 ? lo - 16 : lo);
    q[2 * i + 1] = (int8_t)(hi >= 8 ? hi - 16 : hi);
  }
}

/* ---- rotate + per-row quantize ------------------------------------------- */

/* x: bf16 bits [M, K]; outputs: codes [M, K] (optional), packed [M, K/2]
 * (optional), scales [M], rotated fp32 [M, K] (optional). */
int oracle_rotate_quant_ex(const uint16_t *x, int M, int K, int group, int8_t *codes,
                           uint8_t *packed, float *scale, float *rotated) {
  int S = group_log4(group);
  if (S < 0 || M < 0 || K <= 0 || K % group != 0) return ORACLE_ERR_SHAPE;
  float *row = (float *)malloc(sizeof(float) * (size_t)K);
  int8_t *q = (int8_t *)malloc((size_t)K);
  if (!row || !q) {
    free(row);
    free(q);
    return ORACLE_ERR_NOMEM;
  }
  for (int m = 0; m < M; ++m) {
    const uint16_t *xr = x + (size_t)m * K;
    for (int k = 0; k < K; ++k) row[k] = bf16_bits_to_f32(xr[k]); /* S1 widen */
    for (int g = 0; g < K / group; ++g) rotate_group(row + (size_t)g * group, S); /* S2 */
    float amax = 0.0f; /* S3 per-token amax over the whole row */
    for (int k = 0; k < K; ++k) {
      float a = fabsf(row[k]);
      if (a > amax) amax = a;
    }
    float s = amax / 7.0f;
    for (int k = 0; k < K; ++k) { /* S4 quantize */
      int c = 0;
      if (s != 0.0f) {
        float r = rintf(row[k] / s);
        if (r < -8.0f) r = -8.0f;
        if (r > 7.0f) r = 7.0f;
        c = (int)r;
      }
      q[k] = (int8_t)c;
    }
    scale[m] = s;
    if (codes) memcpy(codes + (size_t)m * K, q, (size_t)K);
    if (packed) oracle_pack_codes(q, K, packed + (size_t)m * (K / 2));
    if (rotated) memcpy(rotated + (size_t)m * K, row, sizeof(float) * (size_t)K);
  }
  free(row);
  free(q);
  return ORACLE_OK;
}

/* The activation prologue: bf16 x[M, K] -> packed codes [M, K/2] + s_a[M]. */
int oracle_rotate_quant(const uint16_t *x, int M, int K, uint8_t *xq, float *s_a) {
  return oracle_rotate_quant_ex(x, M, K, 256, NULL, xq, s_a, NULL);
}

/* Offline weight preparation: the same math on each output channel (row of
 * W[N, K]), which gives per-output-channel scales. */
int oracle_pack_weight(const uint16_t *W, int N, int K, uint8_t *Wq, float *s_w) {
  return oracle_rotate_quant_ex(W, N, K, 256, NULL, Wq, s_w, NULL);
}

/* ---- integer GEMM --------------------------------------------------------- */

/* acc[m, n] = sum_k q_a[m, k] * q_w[n, k] over packed operands, in int64.
 * Rows [m0, m1) only, so a caller can time or check a subset of rows. */
int oracle_gemm_s64_rows(const uint8_t *xq, const uint8_t *Wq, int M, int N, int K, int m0,
                         int m1, int64_t *acc) {
  if (M < 0 || N < 0 || K <= 0 || K % 2 != 0 || m0 < 0 || m1 > M || m0 > m1)
    return ORACLE_ERR_SHAPE;
  int8_t *a = (int8_t *)malloc((size_t)K);
  int8_t *w = (int8_t *)malloc((size_t)K * (size_t)(N > 0 ? N : 1));
  if (!a || !w) {
    free(a);
    free(w);
    return ORACLE_ERR_NOMEM;
  }
  for (int n = 0; n < N; ++n) oracle_unpack_codes(Wq + (size_t)n * (K / 2), K, w + (size_t)n * K);
  for (int m = m0; m < m1; ++m) {
    oracle_unpack_codes(xq + (size_t)m * (K / 2), K, a);
    for (int n = 0; n < N; ++n) {
      const int8_t *wr = w + (size_t)n * K;
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)wr[k];
      acc[(size_t)(m - m0) * N + n] = s;
    }
  }
  free(a);
  free(w);
  return ORACLE_OK;
}

int oracle_gemm_s64(const uint8_t *xq, const uint8_t *Wq, int M, int N, int K, int64_t *acc) {
  return oracle_gemm_s64_rows(xq, Wq, M, N, K, 0, M, acc);
}

/* ---- rank-one epilogue ---------------------------------------------------- */

/* y32 = ((float)acc * s_a[m]) * s_w[n] (+ bias[n]); y16 = bf16 RNE of y32.
 * acc must fit int32 (|acc| <= 64 K), otherwise ORACLE_ERR_OVERFLOW.  Any of
 * y32 / y16 / bias may be NULL. */
int oracle_epilogue(const int64_t *acc, const float *s_a, const float *s_w, const uint16_t *bias,
                    int M, int N, float *y32, uint16_t *y16) {
  for (int m = 0; m < M; ++m)
    for (int n = 0; n < N; ++n) {
      int64_t a = acc[(size_t)m * N + n];
      if (a > INT32_MAX || a < INT32_MIN) return ORACLE_ERR_OVERFLOW;
      float v = (float)a * s_a[m];
      v = v * s_w[n];
      if (bias) v = v + bf16_bits_to_f32(bias[n]);
      if (y32) y32[(size_t)m * N + n] = v;
      if (y16) y16[(size_t)m * N + n] = f32_to_bf16_bits_rne(v);
    }
  return ORACLE_OK;
}

/* ---- the whole Linear ----------------------------------------------------- */

/* y = epilogue(gemm(rotate_quant(x), Wq)); rows [m0, m1) of y only (the rest
 * of the prologue still runs on every row it needs: only rows m0..m1-1). */
int oracle_linear_rows(const uint16_t *x, const uint8_t *Wq, const float *s_w, const uint16_t *bias,
                       int M, int N, int K, int m0, int m1, float *y32, uint16_t *y16) {
  if (M < 0 || N <= 0 || K <= 0 || K % 256 != 0 || m0 < 0 || m1 > M || m0 > m1)
    return ORACLE_ERR_SHAPE;
  int rows = m1 - m0;
  uint8_t *xq = (uint8_t *)malloc((size_t)(rows > 0 ? rows : 1) * (size_t)(K / 2));
  float *s_a = (float *)malloc(sizeof(float) * (size_t)(rows > 0 ? rows : 1));
  int64_t *acc = (int64_t *)malloc(sizeof(int64_t) * (size_t)(rows > 0 ? rows : 1) * (size_t)N);
  int rc = ORACLE_ERR_NOMEM;
  if (xq && s_a && acc) {
    rc = oracle_rotate_quant(x + (size_t)m0 * K, rows, K, xq, s_a);
    if (rc == ORACLE_OK) rc = oracle_gemm_s64(xq, Wq, rows, N, K, acc);
    if (rc == ORACLE_OK) rc = oracle_epilogue(acc, s_a, s_w, bias, rows, N, y32, y16);
  }
  free(xq);
  free(s_a);
  free(acc);
  return rc;
}

int oracle_linear(const uint16_t *x, const uint8_t *Wq, const float *s_w, const uint16_t *bias,
                  int M, int N, int K, float *y32, uint16_t *y16) {
  return oracle_linear_rows(x, Wq, s_w, bias, M, N, K, 0, M, y32, y16);
}

/* ---- int8 formats (int8_tensorwise; ConvRot INT8 row-scaled) -------------- */

/* bf16 x[M, K] -> int8 codes [M, K] and scales.  group = 0: no rotation,
 * group = 256 (or 64, 16): the ConvRot rotation of each group first.
 * per_row = 0: one scale for the whole tensor (scale[0]); per_row = 1: one
 * scale per row (scale[M]).  s = amax / 127, q = clamp(rint(v / s), -127, 127). */
int oracle_quant8(const uint16_t *x, int M, int K, int group, int per_row, int8_t *codes, float *scale) {
  int S = group == 0 ? 0 : group_log4(group);
  if (S < 0 || M < 0 || K <= 0 || (group != 0 && K % group != 0)) return ORACLE_ERR_SHAPE;
  float *v = (float *)malloc(sizeof(float) * (size_t)(M > 0 ? M : 1) * (size_t)K);
  if (!v) return ORACLE_ERR_NOMEM;
  for (size_t i = 0; i < (size_t)M * (size_t)K; ++i) v[i] = bf16_bits_to_f32(x[i]); /* widen */
  if (group != 0)
    for (int m = 0; m < M; ++m)
      for (int g = 0; g < K / group; ++g) rotate_group(v + (size_t)m * K + (size_t)g * group, S);
  float tensor_amax = 0.0f;
  if (!per_row)
    for (size_t i = 0; i < (size_t)M * (size_t)K; ++i) {
      float a = fabsf(v[i]);
      if (a > tensor_amax) tensor_amax = a;
    }
  for (int m = 0; m < M; ++m) {
    const float *row = v + (size_t)m * K;
    float amax = tensor_amax;
    if (per_row) {
      amax = 0.0f;
      for (int k = 0; k < K; ++k) {
        float a = fabsf(row[k]);
        if (a > amax) amax = a;
      }
    }
    float s = amax / 127.0f;
    for (int k = 0; k < K; ++k) {
      int c = 0;
      if (s != 0.0f) {
        float qv = rintf(row[k] / s);
        if (qv < -127.0f) qv = -127.0f;
        if (qv > 127.0f) qv = 127.0f;
        c = (int)qv;
      }
      codes[(size_t)m * K + k] = (int8_t)c;
    }
    if (per_row) scale[m] = s;
    else if (m == 0) scale[0] = s;
  }
  if (!per_row && M == 0) scale[0] = 0.0f;
  free(v);
  return ORACLE_OK;
}

/* acc[m, n] = sum_k x8[m, k] * w8[n, k] in int64, rows [m0, m1). */
int oracle_gemm8_s64_rows(const int8_t *x8, const int8_t *w8, int M, int N, int K, int m0, int m1,
                          int64_t *acc) {
  if (M < 0 || N < 0 || K <= 0 || m0 < 0 || m1 > M || m0 > m1) return ORACLE_ERR_SHAPE;
  for (int m = m0; m < m1; ++m)
    for (int n = 0; n < N; ++n) {
      const int8_t *a = x8 + (size_t)m * K, *w = w8 + (size_t)n * K;
      int64_t s = 0;
      for (int k = 0; k < K; ++k) s += (int64_t)a[k] * (int64_t)w[k];
      acc[(size_t)(m - m0) * N + n] = s;
    }
  return ORACLE_OK;
}

/* The int8 Linear: x quantized with (group, per_row) as above, times the int8
 * weights w8[N, K] with their scales s_w (N of them when per_row, else one),
 * then the rank-one epilogue; rows [m0, m1) of y.  With one scale per tensor
 * the activation scale depends on every row of x, so all M rows are
 * quantized. */
int oracle_linear8_rows(const uint16_t *x, const int8_t *w8, const float *s_w, const uint16_t *bias, int M,
                        int N, int K, int group, int per_row, int m0, int m1, float *y32, uint16_t *y16) {
  if (M < 0 || N <= 0 || K <= 0 || m0 < 0 || m1 > M || m0 > m1) return ORACLE_ERR_SHAPE;
  int rows = m1 - m0;
  int qrows = per_row ? rows : M;
  const uint16_t *xq_src = per_row ? x + (size_t)m0 * K : x;
  int8_t *x8 = (int8_t *)malloc((size_t)(qrows > 0 ? qrows : 1) * (size_t)K);
  float *sx = (float *)malloc(sizeof(float) * (size_t)(qrows > 0 ? qrows : 1));
  float *sa = (float *)malloc(sizeof(float) * (size_t)(rows > 0 ? rows : 1));
  float *sw = (float *)malloc(sizeof(float) * (size_t)N);
  int64_t *acc = (int64_t *)malloc(sizeof(int64_t) * (size_t)(rows > 0 ? rows : 1) * (size_t)N);
  int rc = ORACLE_ERR_NOMEM;
  if (x8 && sx && sa && sw && acc) {
    rc = oracle_quant8(xq_src, qrows, K, group, per_row, x8, sx);
    if (rc == ORACLE_OK) {
      for (int r = 0; r < rows; ++r) sa[r] = per_row ? sx[r] : sx[0];
      for (int n = 0; n < N; ++n) sw[n] = per_row ? s_w[n] : s_w[0];
      int off = per_row ? 0 : m0;
      rc = oracle_gemm8_s64_rows(x8, w8, qrows, N, K, off, off + rows, acc);
    }
    if (rc == ORACLE_OK) rc = oracle_epilogue(acc, sa, sw, bias, rows, N, y32, y16);
  }
  free(x8);
  free(sx);
  free(sa);
  free(sw);
  free(acc);
  return rc;
}

/* ---- asymmetric W4A8 ("asym_w4a8_int8") ------------------------------------
 *
 * Sources: "Nicolaslas/Rebels_w4a8s" ("What's inside a file": int4 codes two
 * per byte, an fp8 scale s_rel per group of 16, one scale per output channel,
 * a 16-level Lloyd-Max codebook fit to the tensor, under a group-256 ConvRot
 * rotation; the math runs on int8 tensor cores) and
 * "JoaoZaokk/Qwen3-VL-4B-W4A8-ConvRot" (file table: asym_w4a8_int8, group 16,
 * convrot_groupsize 256).  Readings (the pages give storage, not arithmetic):
 *  - fp8 is e4m3 "fn": bias 7, 3 mantissa bits, no infinities, S.1111.111 is
 *    NaN, largest finite 448.
 *  - The 4-bit codes are unsigned codebook indices 0..15, low nibble = even k.
 *  - s_rel[n, g] scales codebook levels onto the int8 grid of the row, so the
 *    int8 weight the MMA sees is w8 = clamp(rint(codebook[i] * s_rel), -127,
 *    127): one fp32 multiply, round half to even, NaN -> 0.  The row's real
 *    weights (rotated basis) are s_channel[n] * w8.
 *  - Activations: the ConvRot INT8 row-scaled quantizer above (group 256,
 *    s_a = amax / 127 per token); the epilogue is the rank-one rescale with
 *    s_w = s_channel. */

/* e4m3fn byte -> fp32, exactly: normal (1 + m/8) 2^(e-7), subnormal m 2^-9. */
float oracle_e4m3_to_f32(uint8_t b) {
  int e = (b >> 3) & 15, m = b & 7;
  if (e == 15 && m == 7) return NAN;
  double v = e == 0 ? ldexp((double)m, -9) : ldexp(8.0 + (double)m, e - 10);
  return (float)((b & 0x80) ? -v : v);
}

/* fp32 -> e4m3fn by exhaustive search: the nearest finite code, a tie going
 * to the even code (even mantissa); |f| >= 448 saturates to +-448 (reading);
 * NaN -> 0x7F. */
uint8_t oracle_f32_to_e4m3(float f) {
  if (isnan(f)) return 0x7F;
  uint8_t sign = signbit(f) ? 0x80 : 0x00;
  double a = fabs((double)f);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  int best = 0;
  double bd = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs((double)oracle_e4m3_to_f32((uint8_t)c) - a);
    if (d < bd || (d == bd && (c & 1) == 0)) {
      bd = d;
      best = c;
    }
  }
  return (uint8_t)(sign | best);
}

/* One decoded weight: codebook level `level` under the group scale byte. */
static int8_t asym_decode_one(float level, uint8_t s_rel) {
  float p = level * oracle_e4m3_to_f32(s_rel);
  if (isnan(p)) return 0;
  if (p > 127.0f) return 127;
  if (p < -127.0f) return -127;
  return (int8_t)rintf(p);
}

/* idx[N, K/2] (two indices per byte), s_rel[N, K/16], codebook[16] ->
 * int8 weights w8[N, K]. */
int oracle_asym_decode(const uint8_t *idx, const uint8_t *s_rel, const float *codebook, int N, int K,
                       int8_t *w8) {
  if (N < 0 || K <= 0 || K % 16 != 0) return ORACLE_ERR_SHAPE;
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      uint8_t byte = idx[(size_t)n * (K / 2) + k / 2];
      int i = (k % 2 == 0) ? (byte & 0xF) : (byte >> 4);
      w8[(size_t)n * K + k] = asym_decode_one(codebook[i], s_rel[(size_t)n * (K / 16) + k / 16]);
    }
  return ORACLE_OK;
}

/* The asymmetric W4A8 Linear, rows [m0, m1) of y: decode the weights, then
 * the ConvRot INT8 row-scaled Linear with s_w = s_channel. */
int oracle_asym_linear_rows(const uint16_t *x, const uint8_t *idx, const uint8_t *s_rel, const float *codebook,
                            const float *s_channel, const uint16_t *bias, int M, int N, int K, int m0, int m1,
                            float *y32, uint16_t *y16) {
  if (M < 0 || N <= 0 || K <= 0 || K % 256 != 0) return ORACLE_ERR_SHAPE;
  int8_t *w8 = (int8_t *)malloc((size_t)N * (size_t)K);
  if (!w8) return ORACLE_ERR_NOMEM;
  int rc = oracle_asym_decode(idx, s_rel, codebook, N, K, w8);
  if (rc == ORACLE_OK) rc = oracle_linear8_rows(x, w8, s_channel, bias, M, N, K, 256, 1, m0, m1, y32, y16);
  free(w8);
  return rc;
}

/* Index of the level nearest to u (the lower index on a tie). */
static int nearest_level(const double *c, double u) {
  int best = 0;
  double bd = fabs(u - c[0]);
  for (int j = 1; j < 16; ++j) {
    double d = fabs(u - c[j]);
    if (d < bd) {
      bd = d;
      best = j;
    }
  }
  return best;
}

/* Lloyd's algorithm for the 16-level scalar quantizer of the values u[0..n):
 * levels start at the centres of 16 equal cells of [-1, 1]; each iteration
 * assigns every value to its nearest level, then moves every level to the
 * mean of its values (a level without values stays).  It stops when no
 * assignment changed or after `iters` iterations.  Levels in double. */
int oracle_lloyd_max16(const float *u, int64_t n, int iters, double *levels) {
  if (n < 0 || iters < 0) return ORACLE_ERR_SHAPE;
  for (int j = 0; j < 16; ++j) levels[j] = -1.0 + (2.0 * j + 1.0) / 16.0;
  int *cell = (int *)malloc(sizeof(int) * (size_t)(n > 0 ? n : 1));
  if (!cell) return ORACLE_ERR_NOMEM;
  for (int64_t i = 0; i < n; ++i) cell[i] = -1;
  for (int it = 0; it < iters; ++it) {
    int changed = 0;
    for (int64_t i = 0; i < n; ++i) {
      int j = nearest_level(levels, (double)u[i]);
      if (j != cell[i]) changed = 1;
      cell[i] = j;
    }
    if (!changed) break;
    double sum[16] = {0};
    int64_t cnt[16] = {0};
    for (int64_t i = 0; i < n; ++i) {
      sum[cell[i]] += (double)u[i];
      cnt[cell[i]] += 1;
    }
    for (int j = 0; j < 16; ++j)
      if (cnt[j] > 0) levels[j] = sum[j] / (double)cnt[j];
  }
  free(cell);
  return ORACLE_OK;
}

/* Offline conversion of bf16 weights W[N, K] to the asymmetric W4A8 format
 * (test infrastructure: the pages' converter is not part of the hot path).
 *   1. rotate each row's 256-groups (the ConvRot rotation above);
 *   2. s_channel[n] = amax_k |w'[n,k]| / 127;
 *   3. s_rel[n, g] = e4m3(amax over the 16 values of group g / s_channel[n])
 *      (0 when s_channel is 0);
 *   4. u = w' / (s_channel * s_rel), 0 where that product is 0;
 *   5. codebook = Lloyd-Max levels of all u of the tensor (`iters` at most),
 *      rounded to fp32;
 *   6. idx = the nearest fp32 level to each u (the lower index on a tie). */
int oracle_asym_convert(const uint16_t *W, int N, int K, int iters, uint8_t *idx, uint8_t *s_rel, float *s_channel,
                        float *codebook) {
  if (N <= 0 || K <= 0 || K % 256 != 0) return ORACLE_ERR_SHAPE;
  size_t NK = (size_t)N * (size_t)K;
  float *v = (float *)malloc(sizeof(float) * NK);
  float *u = (float *)malloc(sizeof(float) * NK);
  if (!v || !u) {
    free(v);
    free(u);
    return ORACLE_ERR_NOMEM;
  }
  for (size_t i = 0; i < NK; ++i) v[i] = bf16_bits_to_f32(W[i]);
  for (int n = 0; n < N; ++n)
    for (int g = 0; g < K / 256; ++g) rotate_group(v + (size_t)n * K + (size_t)g * 256, 4);
  for (int n = 0; n < N; ++n) {
    const float *row = v + (size_t)n * K;
    float amax = 0.0f;
    for (int k = 0; k < K; ++k)
      if (fabsf(row[k]) > amax) amax = fabsf(row[k]);
    float sc = amax / 127.0f;
    s_channel[n] = sc;
    for (int g = 0; g < K / 16; ++g) {
      float ga = 0.0f;
      for (int k = 16 * g; k < 16 * g + 16; ++k)
        if (fabsf(row[k]) > ga) ga = fabsf(row[k]);
      uint8_t sb = sc == 0.0f ? 0 : oracle_f32_to_e4m3(ga / sc);
      s_rel[(size_t)n * (K / 16) + g] = sb;
      float d = sc * oracle_e4m3_to_f32(sb);
      for (int k = 16 * g; k < 16 * g + 16; ++k) u[(size_t)n * K + k] = d == 0.0f ? 0.0f : row[k] / d;
    }
  }
  double lv[16];
  int rc = oracle_lloyd_max16(u, (int64_t)NK, iters, lv);
  if (rc == ORACLE_OK) {
    double c32[16];
    for (int j = 0; j < 16; ++j) {
      codebook[j] = (float)lv[j];
      c32[j] = (double)codebook[j];
    }
    memset(idx, 0, NK / 2);
    for (size_t i = 0; i < NK; ++i) {
      int j = nearest_level(c32, (double)u[i]);
      idx[i / 2] |= (uint8_t)((i % 2 == 0) ? j : (j << 4));
    }
  }
  free(v);
  free(u);
  return rc;
}
