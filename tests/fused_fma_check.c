/* Checks, on the host's FMA unit, the identity behind the GEMM's product
 * pass: for one output and one accumulation group, adding every product with
 * one round-toward-zero fused multiply-add into the double
 *     acc = (2^52 + 2^51 + S0) * 2^(e_max - F)
 * -- with B scaled by (1 + 2^-40), zeros as +-2^-500 -- leaves in acc's low
 * mantissa bits S0 plus the model's truncated products, minus one per
 * negative product.  The reference is exact integer truncation of each
 * product's magnitude onto the grid 2^(e_max - F) ("Hawkeye: Reproducing
 * GPU-Level Non-Determinism (MLSys 2026)", Obs. 3 and the recovered pipeline's
 * GroupSum).
 *
 * Planted mistakes (compile-time): -DNO_GROWTH (B not scaled), -DNO_COUNT (no
 * negative-product count), -DROUND_NEAREST (round to nearest).  Each must
 * produce mismatches.  Prints "<mismatches> <cases>". */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <string.h>
#pragma STDC FENV_ACCESS ON

static uint64_t state = 0x9E3779B97F4A7C15ull;
static uint64_t next(void) {
  state ^= state << 13;
  state ^= state >> 7;
  state ^= state << 17;
  return state;
}

typedef struct { int p, emin, emax; } format;                 /* fraction bits, normal exponent range */
static const format FORMATS[3] = {{10, -14, 15}, {7, -126, 127}, {3, -6, 8}};  /* FP16, BF16, E4M3 */
typedef struct { int neg; uint32_t m; int e; } element;       /* value (-1)^neg m 2^(e - p) */

static element draw(format f, int zero_pct, int sub_pct, int spread) {
  element x;
  x.neg = (int)(next() & 1);
  const int r = (int)(next() % 100);
  if (r < zero_pct) { x.m = 0; x.e = f.emin; return x; }
  if (r < zero_pct + sub_pct) { x.m = 1 + (uint32_t)(next() % ((1u << f.p) - 1)); x.e = f.emin; return x; }
  x.m = (1u << f.p) | (uint32_t)(next() & ((1u << f.p) - 1));
  int lo = f.emin, hi = f.emax;
  if (spread) {
    const int c = lo + (int)(next() % (uint64_t)(hi - lo + 1));
    lo = c - spread > f.emin ? c - spread : f.emin;
    hi = c + spread < f.emax ? c + spread : f.emax;
  }
  x.e = lo + (int)(next() % (uint64_t)(hi - lo + 1));
  return x;
}

static double as_double(element x, format f) {
  if (x.m == 0) return x.neg ? -0x1p-500 : 0x1p-500;
  const double v = ldexp((double)x.m, x.e - f.p);
  return x.neg ? -v : v;
}

int main(void) {
  const int widths[3] = {23, 24, 25};
  long bad = 0, cases = 0;
  for (int fi = 0; fi < 3; fi++)
    for (int wi = 0; wi < 3; wi++)
      for (int t = 0; t < 40000; t++) {
        const format f = FORMATS[fi];
        const int F = widths[wi], n = (t & 1) ? 16 : 8;
        const int zero_pct = (int)(next() % 40), sub_pct = (int)(next() % 30), spread = (int)(next() % 8);
        element a[16], b[16];
        for (int k = 0; k < n; k++) {
          a[k] = draw(f, zero_pct, sub_pct, spread);
          b[k] = draw(f, zero_pct, sub_pct, spread);
        }
        /* group maximum over nonzero products, floored at -133; a carried
           term may raise it */
        int emax = -100000;
        for (int k = 0; k < n; k++)
          if (a[k].m && b[k].m && a[k].e + b[k].e > emax) emax = a[k].e + b[k].e;
        if (emax < -133) emax = -133;
        if (next() % 4 == 0) emax += (int)(next() % 40);
        const int64_t s0 = (int64_t)(next() % (1u << 26)) - (1 << 25);

        int64_t want = s0;
        for (int k = 0; k < n; k++) {
          const uint64_t mm = (uint64_t)a[k].m * b[k].m; /* |ab| = mm 2^(ea + eb - 2p) */
          const int shift = (emax - F) - (a[k].e + b[k].e - 2 * f.p);
          const uint64_t T = shift <= 0 ? mm << -shift : shift >= 64 ? 0 : mm >> shift;
          want += (a[k].neg ^ b[k].neg) ? -(int64_t)T : (int64_t)T;
        }

#ifdef ROUND_NEAREST
        fesetround(FE_TONEAREST);
#else
        fesetround(FE_TOWARDZERO);
#endif
        volatile double acc = ldexp(6755399441055744.0 + (double)(s0 & 0xFFFFFFFFll), emax - F);
        int negatives = 0;
        for (int k = 0; k < n; k++) {
          volatile double av = as_double(a[k], f), bv = as_double(b[k], f);
#ifndef NO_GROWTH
          bv = bv * (1.0 + 0x1p-40); /* exact */
#endif
          acc = fma(av, bv, acc);
          negatives += a[k].neg ^ b[k].neg;
        }
        fesetround(FE_TONEAREST);
#ifdef NO_COUNT
        negatives = 0;
#endif
        const double final = acc;
        uint64_t bits;
        memcpy(&bits, &final, sizeof bits);
        const int32_t got = (int32_t)((uint32_t)bits + (uint32_t)negatives);
        cases++;
        if ((int64_t)got != want) bad++;
      }
  printf("%ld %ld\n", bad, cases);
  return 0;
}
