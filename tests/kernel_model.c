/*
 * Host restatement of the GEMM and tile kernels' arithmetic (the "exact
 * double" path), used to check the kernels' design against the oracle on the
 * CPU.  It is NOT the oracle: it models the CUDA code's own steps -- packed
 * 16-bit exponent codes, the grid base built from a packed code, one
 * round-toward-zero fused multiply-add per term, the sign-pair count, the
 * subtraction that recovers the exact group value, the 24-bit truncation by
 * masking, and the scaled ("checked") state with its rare paths -- so that a
 * mistake in that design shows up as a difference from the oracle before any
 * GPU time is spent.  It shares no code with the oracle or the library.
 *
 * The model being emulated ("Hawkeye: Reproducing GPU-Level Non-Determinism
 * (MLSys 2026)" notes: Obs. 1-3, the recovered Ampere FP16 pipeline with its
 * Hopper and BF16 paragraphs, Algorithm 10): per 16-deep K chunk, groups
 * {C, P1..8}, {S1, P9..16} (Ampere) or {C, P1..16} (Hopper, B200); each term
 * aligned to the group's largest exponent (floored at -133) on the grid
 * 2^(e_max - F) by truncation of its magnitude; exact signed sum; Ampere
 * hand-over truncated to 24 bits; toward-zero fp32 write-back with overflow to
 * infinity and gradual, truncated underflow.
 *
 * Needs an FMA instruction (-mfma) and a compiler that honours the dynamic
 * rounding mode (-frounding-math).  -DMISTAKE_* plants one mistake in the
 * design (no negative-term count, no growth factor, no 24-bit truncation, no
 * -133 floor, no exponent override for a subnormal carry, round-to-nearest
 * write-back, an untruncated carry for Hopper and B200 as well as Ampere); the
 * tests require each to be caught.
 */
#include <fenv.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#pragma STDC FENV_ACCESS ON

enum { KM_AMPERE = 0, KM_HOPPER = 1, KM_B200 = 2 };
enum { KM_FP16 = 0, KM_BF16 = 1, KM_E4M3 = 2 };

typedef struct { int P, BIAS, EBITS, NBITS, IEEE; } kfmt;
static const kfmt KFMT[3] = {{10, 15, 5, 16, 1}, {7, 127, 8, 16, 1}, {3, 7, 4, 8, 0}};
static const int KF[3] = {23, 24, 25};
static const uint32_t KNAN[3] = {0x7FC00000u, 0x7FC00000u, 0x7FFFFFFFu};

/* exponent codes: ncode(e) = (1024 - e) * 16, an operand carries (512 - e) * 16 */
#define QZ 14336   /* zero operand (multiple of 16) */
#define QINF 14337 /* infinite operand */
#define QNAN 14338 /* NaN operand */
#ifdef MISTAKE_NO_FLOOR
#define FLOOR_CODE 32767
#else
#define FLOOR_CODE 18512 /* ncode(-133): the floor on e_max */
#endif
#define SUBN_CODE 18400  /* ncode(-126): exponent of an fp32 subnormal carry */
#define S_WB 896         /* scale of a checked fp32 state: 2^(1024-128) */
#define S_HO 512         /* scale of a checked Ampere hand-over */

static uint64_t dbits(double x) { uint64_t u; memcpy(&u, &x, 8); return u; }
static double bitsd(uint64_t u) { double x; memcpy(&x, &u, 8); return x; }
static uint32_t hiw(double x) { return (uint32_t)(dbits(x) >> 32); }
static double mkd(uint32_t hi, uint32_t lo) { return bitsd(((uint64_t)hi << 32) | lo); }
static double mask24(double x) {
#if defined(MISTAKE_NO_MASK)
  return x;
#elif defined(MISTAKE_NEAREST_WRITEBACK)
  return (double)(float)x;
#else
  return bitsd(dbits(x) & 0xFFFFFFFFE0000000ull);
#endif
}

static uint32_t vadd2(uint32_t a, uint32_t b) {
  return ((a + b) & 0xFFFFu) | (((a >> 16) + (b >> 16)) << 16);
}
static uint32_t vmin2(uint32_t a, uint32_t b) {
  int16_t a0 = (int16_t)(a & 0xFFFF), a1 = (int16_t)(a >> 16), b0 = (int16_t)(b & 0xFFFF), b1 = (int16_t)(b >> 16);
  return (uint32_t)(uint16_t)(a0 < b0 ? a0 : b0) | ((uint32_t)(uint16_t)(a1 < b1 ? a1 : b1) << 16);
}
static uint32_t pair16(int lo, int hi) { return ((uint32_t)lo & 0xFFFFu) | ((uint32_t)hi << 16); }

/* decoded operand: exact value (Inf/NaN/zero as a signed zero), code, sign
 * pair.  Sign words: element k = 8h + 2j + b of a row of A (column of B) owns
 * bit NB(k) = 2j + h + 16b and bit NB(k) + 8.  A row sets NB(k) + 8 for a
 * positive nonzero finite a[k] and NB(k) for a negative one; a B column sets
 * NB(k) for a positive b[k] and NB(k) + 8 for a negative one -- so that the
 * AND of the two words has one bit per negative product of nonzero finite
 * operands.  k < 8 uses the even bits, k >= 8 the odd ones. */
static int NB(int k) { return (k & 6) + (k >> 3) + 16 * (k & 1); }
typedef struct { double v; int q; int pos, neg; int neg_sign; } kdec;

static kdec kdecode(int fmt, uint32_t x) {
  const kfmt f = KFMT[fmt];
  const uint32_t top = (1u << f.EBITS) - 1u, field = (x >> f.P) & top, frac = x & ((1u << f.P) - 1u);
  const int s = (int)((x >> (f.NBITS - 1)) & 1u);
  kdec d;
  d.neg_sign = s;
  d.pos = d.neg = 0;
  d.v = s ? -0.0 : 0.0;
  if (f.IEEE && field == top) { d.q = frac ? QNAN : QINF; return d; }
  if (!f.IEEE && (x & 0x7Fu) == 0x7Fu) { d.q = QNAN; return d; }
  const uint32_t m = frac | (field ? (1u << f.P) : 0u);
  const int e = (int)(field ? field : 1u) - f.BIAS;
  if (m == 0) { d.q = QZ; return d; }
  d.v = ldexp((double)m, e - f.P) * (s ? -1.0 : 1.0);
  d.q = (512 - e) * 16;
  d.pos = !s;
  d.neg = s;
  return d;
}

/* per-output running state of the kernels */
typedef struct {
  double d;    /* value (checked: times 2^896); zeros as +0 */
  int negzero; /* the state is -0 */
} kstate;

typedef struct {
  int model, fmt, F, checked;
  const kdec *a; /* 16 decoded A elements of this chunk (row m) */
  const kdec *b0, *b1; /* 16 decoded B elements for the two columns */
} kctx;

static uint32_t sign_word_a(const kdec *a) {
  uint32_t w = 0;
  for (int k = 0; k < 16; k++) w |= ((uint32_t)a[k].pos << (NB(k) + 8)) | ((uint32_t)a[k].neg << NB(k));
  return w;
}
static uint32_t sign_word_b(const kdec *b) {
  uint32_t w = 0;
  for (int k = 0; k < 16; k++) w |= ((uint32_t)b[k].pos << NB(k)) | ((uint32_t)b[k].neg << (NB(k) + 8));
  return w;
}

/* One accumulation group for an adjacent pair of outputs (the packed lanes).
 * carry[2]: the carried values (scaled by 2^s_in in the checked form; s_in =
 * 0 unchecked); subn[q] forces lane q's carried code to ncode(-126) (an fp32
 * subnormal carry); returns the exact group values v[2] (not scaled). */
static void group_pair(const kctx *c, int k0, int kn, const double carry[2], int s_in, const int subn[2],
                       double v[2]) {
  /* carried terms' codes from the top 16 bits of their doubles */
  const uint32_t x = (hiw(carry[0]) >> 16) | (hiw(carry[1]) & 0xFFFF0000u);
  uint32_t nm;
  if (!c->checked) {
    if (c->fmt == KM_BF16) abort(); /* BF16 always runs checked */
    nm = ~x & 0x7FF07FF0u;
  } else {
    uint32_t cc = vadd2(~x & 0x3FF03FF0u, pair16(s_in * 16, s_in * 16));
#ifndef MISTAKE_SUBNORMAL_CODE
    if (subn[0]) cc = (cc & 0xFFFF0000u) | SUBN_CODE;
    if (subn[1]) cc = (cc & 0xFFFFu) | ((uint32_t)SUBN_CODE << 16);
#endif
    nm = vmin2(cc, pair16(FLOOR_CODE, FLOOR_CODE));
  }
  for (int k = k0; k < k0 + kn; k++)
    nm = vmin2(vadd2(pair16(c->a[k].q, c->a[k].q), pair16(c->b0[k].q, c->b1[k].q)), nm);
  const uint32_t KHI = ((uint32_t)(2099 - c->F) << 20) | 0x80000u;
  const uint32_t hi[2] = {KHI + nm * 0xFFFF0000u, KHI - nm};
  uint32_t gm = 0;
  for (int k = k0; k < k0 + kn; k++) gm |= 0x101u << NB(k);
  const uint32_t sa = sign_word_a(c->a), sb[2] = {sign_word_b(c->b0), sign_word_b(c->b1)};
#ifdef MISTAKE_NO_SKEW
  const double growth = 1.0;
#else
  const double growth = 1.0 + 0x1p-40;
#endif
  const double skew = ldexp(growth, -s_in);
  for (int q = 0; q < 2; q++) {
    const kdec *b = q ? c->b1 : c->b0;
#ifdef MISTAKE_NO_COUNT
    const uint32_t cnt = 0;
#else
    const uint32_t cnt = (uint32_t)__builtin_popcount(sa & sb[q] & gm) + (hiw(carry[q]) >> 31);
#endif
    fesetround(FE_TOWARDZERO);
    volatile double acc = mkd(hi[q], cnt);
    acc = fma(carry[q], skew, acc);
    for (int k = k0; k < k0 + kn; k++) acc = fma(c->a[k].v, b[k].v * growth, acc);
    fesetround(FE_TONEAREST);
    v[q] = acc - mkd(hi[q], 0);
  }
}

/* special-value outcome of one output: 0 none, 1 NaN, 2 +Inf, 3 -Inf */
static int special_code(const kctx *c, int q, const kstate *in) {
  const kdec *b = q ? c->b1 : c->b0;
  int nan = 0, ip = 0, in_ = 0;
  if (c->checked) {
    if (isnan(in->d)) nan = 1;
    else if (isinf(in->d)) { if (in->d < 0) in_ = 1; else ip = 1; }
  }
  for (int k = 0; k < 16; k++) {
    const int aq = c->a[k].q, bq = b[k].q;
    if (aq == QNAN || bq == QNAN) nan = 1;
    else if (aq == QINF || bq == QINF) {
      if (aq == QZ || bq == QZ) nan = 1;
      else if (c->a[k].neg_sign != b[k].neg_sign) in_ = 1;
      else ip = 1;
    }
  }
  return (nan || (ip && in_)) ? 1 : ip ? 2 : in_ ? 3 : 0;
}

static int all_products_negative_zero(const kctx *c, int q) {
  const kdec *b = q ? c->b1 : c->b0;
  for (int k = 0; k < 16; k++) {
    const int z = c->a[k].q == QZ || b[k].q == QZ;
    if (!z || c->a[k].neg_sign == b[k].neg_sign) return 0;
  }
  return 1;
}

/* checked states below 2^-126: truncate onto the subnormal grid (returns 1
 * if the state is an fp32 subnormal, whose carried exponent is -126) */
static int fix_subnormal(kstate *s) {
  if (s->d == 0.0 || isinf(s->d) || isnan(s->d)) return 0;
  const double x = ldexp(s->d, -S_WB);
  if (fabs(x) >= 0x1p-126) return 0;
  const double q = floor(fabs(x) * 0x1p149);
  if (q == 0.0) {
    s->negzero = x < 0;
    s->d = 0.0;
    return 0;
  }
  s->d = ldexp(q, -149 + S_WB) * (x < 0 ? -1.0 : 1.0);
  return 1;
}

/* one 16-deep chunk for an output pair, in place */
static void chunk_pair(kctx *c, kstate st[2]) {
  int subn[2] = {0, 0};
  if (c->checked)
    for (int q = 0; q < 2; q++) subn[q] = fix_subnormal(&st[q]);
  double carry[2] = {st[0].d, st[1].d}, v[2];
  const kstate in[2] = {st[0], st[1]};
  const int two = c->model == KM_AMPERE;
  const int none[2] = {0, 0};
  /* stage 1 (or the only stage) */
  group_pair(c, 0, two ? 8 : 16, carry, c->checked ? S_WB : 0, subn, v);
  if (two) {
    /* hand-over: the stage-1 value truncated to 24 bits, exponent unbounded
       (checked: carried times 2^512).  The unchecked form carries the exact
       stage value: the next grid, 2^(e_max - 23) with e_max at least the
       value's own exponent, is never finer than its 24-bit unit, and
       truncations to nested power-of-two grids compose. */
    double h[2];
    for (int q = 0; q < 2; q++) h[q] = c->checked ? ldexp(mask24(v[q]), S_HO) : v[q];
    group_pair(c, 8, 8, h, c->checked ? S_HO : 0, none, v);
  }
  /* toward-zero write-back; the unchecked Ampere form again carries the
     exact value (the next chunk's first grid is 2^(e_max - 23) too), while
     Hopper's and B200's finer grids need the truncated one */
#ifdef MISTAKE_HOPPER_UNTRUNCATED
  const int exact_carry = !c->checked;
#else
  const int exact_carry = !c->checked && c->model == KM_AMPERE;
#endif
  for (int q = 0; q < 2; q++) {
    const double wb = mask24(v[q]);
    st[q].d = c->checked ? wb * 0x1p896 /* round to nearest: overflow -> Inf */
                         : exact_carry ? v[q] : wb;
    if (st[q].negzero) {
      if (v[q] == 0.0) st[q].negzero = all_products_negative_zero(c, q);
      else st[q].negzero = 0;
    }
  }
  /* special values */
  int any = 0, code[2];
  for (int q = 0; q < 2; q++) {
    code[q] = special_code(c, q, &in[q]);
    any |= code[q] != 0;
  }
  if (any && !c->checked) {
    /* switch to the checked form (truncating an exact Ampere carry) */
    for (int q = 0; q < 2; q++) st[q].d = mask24(st[q].d) * 0x1p896;
    c->checked = 1;
  }
  for (int q = 0; q < 2; q++) {
    if (!code[q]) continue;
    st[q].negzero = 0;
    st[q].d = code[q] == 1 ? NAN : code[q] == 2 ? INFINITY : -INFINITY;
  }
}

static uint32_t f32bits(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }
static float bitsf(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }

static uint32_t final_bits(const kctx *c, kstate *s) {
  if (c->checked) fix_subnormal(s);
  if (isnan(s->d)) return KNAN[c->model];
  if (isinf(s->d)) return s->d < 0 ? 0xFF800000u : 0x7F800000u;
  if (s->d == 0.0) return s->negzero ? 0x80000000u : 0u;
  const double x = c->checked ? ldexp(s->d, -S_WB) : s->d;
  return f32bits((float)mask24(x)); /* exact once truncated to 24 bits */
}

static uint32_t elem(const void *p, int fmt, size_t i) {
  return fmt == KM_E4M3 ? ((const uint8_t *)p)[i] : ((const uint16_t *)p)[i];
}

/* initial state from an fp32 C value; returns whether the unchecked form
 * may take it (FP16 / E4M3 only: +-0 or 2^-126 <= |c| < 2^100) */
static int init_state(uint32_t cb, int fmt, int checked, kstate *s) {
  const uint32_t field = (cb >> 23) & 0xFFu;
  s->negzero = cb == 0x80000000u;
  const float cf = bitsf(cb);
  if ((cb & 0x7FFFFFFFu) == 0) s->d = 0.0;
  else if (field == 0xFFu) s->d = isnan(cf) ? NAN : (double)cf;
  else s->d = checked ? ldexp((double)cf, S_WB) : (double)cf;
  const int ok = fmt != KM_BF16 && ((cb & 0x7FFFFFFFu) == 0 || (field >= 1 && field < 227));
  return ok;
}

/* D = C + A.B over 16-wide K chunks for an M x N GEMM (N even); C may be
 * NULL.  force_checked selects the checked form for every output. */
int km_gemm(int model, int fmt, int M, int N, int K, const void *A, const void *B, const uint32_t *C, uint32_t *D,
            int force_checked) {
  if ((N & 1) || (K & 15)) return -1;
  if ((model == KM_AMPERE || model == KM_B200) && fmt == KM_E4M3) return -1;
  kdec a[16], b0[16], b1[16];
  for (int m = 0; m < M; m++)
    for (int n = 0; n < N; n += 2) {
      kctx c = {model, fmt, KF[model], 0, a, b0, b1};
      kstate st[2];
      int ok = 1;
      for (int q = 0; q < 2; q++) {
        const uint32_t cb = C ? C[(size_t)m * N + n + q] : 0u;
        ok &= init_state(cb, fmt, 0, &st[q]);
      }
      if (!ok || force_checked) {
        c.checked = 1;
        for (int q = 0; q < 2; q++) init_state(C ? C[(size_t)m * N + n + q] : 0u, fmt, 1, &st[q]);
      }
      for (int j = 0; j < K; j += 16) {
        for (int k = 0; k < 16; k++) {
          a[k] = kdecode(fmt, elem(A, fmt, (size_t)m * K + j + k));
          b0[k] = kdecode(fmt, elem(B, fmt, (size_t)(j + k) * N + n));
          b1[k] = kdecode(fmt, elem(B, fmt, (size_t)(j + k) * N + n + 1));
        }
        chunk_pair(&c, st);
      }
      for (int q = 0; q < 2; q++) D[(size_t)m * N + n + q] = final_bits(&c, &st[q]);
    }
  fesetround(FE_TONEAREST);
  return 0;
}
