/* Host check of two arithmetic rules the CUDA prologue relies on (rotate_quant.cu),
 * restated here in plain C with the same fp32 operations (fmaf is a single rounding).
 *
 *   div   s = RN(a / q) for q = 7 or 127 by two Markstein corrections of RN(a * RN(1/q)),
 *         for a in [2^-120, 2^120]: compared with IEEE division on every float of a
 *         stride through that range (argument 1: the stride; 1 = every float).
 *   quant the checked reciprocal quantizer: k = rint(v y) with y an approximate
 *         1/(2^L s), d = RN(v - 2^L s k); whenever |d| <= 2^L s (1/2 - m) the code k must
 *         equal rint(RN(RN(v 2^-L) / s)) (ties to even), for L in {2, 3, 4}, qmax 7 (m =
 *         2^-18) and 127 (m = 2^-14), quotients within [-qmax, qmax], y off by up to two
 *         ulps, and inputs at, next to and near half-integers (argument 2: the cases).
 *
 * Prints "div <checked> <bad>" and "quant <cases> <fast> <bad>"; exits 1 on any bad case.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

static float f_of(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t u_of(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static uint64_t rnd(void) {  /* xorshift64 */
  rng_state ^= rng_state << 13;
  rng_state ^= rng_state >> 7;
  rng_state ^= rng_state << 17;
  return rng_state;
}
static double urand(void) { return (double)(rnd() >> 11) * (1.0 / 9007199254740992.0); }

static float div_markstein(float a, float q) {
  const float y = 1.0f / q;
  float r = a * y;
  r = fmaf(fmaf(-q, r, a), y, r);
  r = fmaf(fmaf(-q, r, a), y, r);
  return r;
}

int main(int argc, char** argv) {
  const uint32_t stride = argc > 1 ? (uint32_t)strtoul(argv[1], NULL, 10) : 97u;
  const long cases = argc > 2 ? strtol(argv[2], NULL, 10) : 5000000L;
  const float qs[2] = {7.0f, 127.0f};
  uint64_t checked = 0, bad_div = 0;
  for (int j = 0; j < 2; ++j) {
    const uint32_t lo = u_of(ldexpf(1.0f, -120)), hi = u_of(ldexpf(1.0f, 120));
    for (uint32_t u = lo; u < hi; u += stride) {
      const float a = f_of(u);
      if (u_of(div_markstein(a, qs[j])) != u_of(a / qs[j])) ++bad_div;
      ++checked;
    }
    /* every float of the first and last binade */
    for (uint32_t u = lo; u < lo + (1u << 23); ++u, ++checked)
      if (u_of(div_markstein(f_of(u), qs[j])) != u_of(f_of(u) / qs[j])) ++bad_div;
    for (uint32_t u = hi - (1u << 23); u < hi; ++u, ++checked)
      if (u_of(div_markstein(f_of(u), qs[j])) != u_of(f_of(u) / qs[j])) ++bad_div;
  }
  printf("div %llu %llu\n", (unsigned long long)checked, (unsigned long long)bad_div);

  const float magic = 12582912.0f; /* 1.5 * 2^23 */
  uint64_t n = 0, fast = 0, bad_q = 0;
  for (long it = 0; it < cases; ++it) {
    const int L = 2 + (int)(rnd() % 3);
    const float qmax = qs[rnd() % 2];
    const float g = ldexpf(1.0f, L), inv = ldexpf(1.0f, -L);
    float s = ldexpf((float)(1.0 + urand()), (int)(rnd() % 201) - 100);
    const double k0 = (double)((int)(rnd() % (uint64_t)(2 * (int)qmax)) - (int)qmax);
    float v;
    switch (rnd() % 5) {
      case 0: v = (float)((k0 + 0.5) * g * s); break;                                  /* a tie */
      case 1: v = f_of(u_of((float)((k0 + 0.5) * g * s)) + (int)(rnd() % 9) - 4); break; /* ulps from it */
      case 2: v = (float)((urand() * 2.0 - 1.0) * qmax * g * s); break;                  /* anywhere */
      case 3: v = (float)((k0 + 0.5 + (urand() - 0.5) * 1e-5) * g * s); break;           /* near it */
      default: {                                                                         /* the amax itself */
        const float am = (float)(urand() + 0.5) * ldexpf(1.0f, (int)(rnd() % 160) - 80);
        s = am / qmax;
        v = am * g * ((rnd() & 1) ? 1.0f : -1.0f);
      }
    }
    if (!isfinite(v) || !(s >= ldexpf(1.0f, -100) && s <= ldexpf(1.0f, 100))) continue;
    const float m = qmax == 7.0f ? ldexpf(1.0f, -18) : ldexpf(1.0f, -14);
    const float r = f_of(u_of(1.0f / s) + (int)(rnd() % 5) - 2); /* an approximate reciprocal */
    const float y = r * inv, nd = -(s * g), thr = s * (g * (0.5f - m));
    const float c = fmaf(v, y, magic);
    const float k = c - magic;
    const float d = fmaf(nd, k, v);
    ++n;
    if (fabsf(d) <= thr) {
      ++fast;
      const float want = rintf((v * inv) / s);
      if (k != want) ++bad_q;
    }
  }
  printf("quant %llu %llu %llu\n", (unsigned long long)n, (unsigned long long)fast, (unsigned long long)bad_q);
  return (bad_div || bad_q) ? 1 : 0;
}
