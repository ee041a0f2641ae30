/*
 * libmmaemu probe API -- the characterise half of characterise-then-simulate.
 *
 * Runs the target tests of "Hawkeye: Reproducing GPU-Level Non-Determinism
 * (MLSys 2026)" (reading notes: "Target Tests" table -- summation dependency
 * and order, internal precision, rounding mode, normalisation stage,
 * subnormal behaviour; Algorithm 4, the computationally neutral subgroup
 * test) against ANY 16x16x16 tile MMA given as a callback: this library's
 * emulation (mmaemu_mma_emulated), B200's own tensor cores
 * (mmaemu_mma_native), or a caller's function.  The pages name running the
 * same target tests on Blackwell as future work; mmaemu_mma_native makes
 * that a library call.
 *
 * Probe construction: every probe instance uses one diagonal element of a
 * tile -- A row i, B column i, C[i][i], read back from D[i][i] -- so one
 * tile carries 16 independent instances; off-diagonal outputs are ignored
 * (a callback may leave them unwritten).  Probes compare outputs bit for
 * bit, mostly as differential pairs (the same instance with and without the
 * probed bit), so they do not depend on how the MMA rounds its final
 * result, except the write-back probe which measures exactly that.
 *
 * All buffers passed to callbacks are HOST memory owned by the probe call.
 * Probes are synchronous.  Return value: MMAEMU_OK or a negative code from
 * mmaemu.h, or MMAEMU_ECALLBACK when the callback returned nonzero.
 */
#ifndef MMAEMU_PROBE_H
#define MMAEMU_PROBE_H

#include <stddef.h>
#include <stdint.h>

#include "mmaemu.h"

#ifdef __cplusplus
extern "C" {
#endif

/* A tile MMA: for t < ntiles, D[t] = C[t] + A[t] . B[t] on 16x16x16 tiles,
 * layouts as mmaemu_tiles (A (m,k) and B (k,n) row-major in fmt; C and D
 * fp32 bit patterns, (m,n) row-major).  Host pointers.  Return 0 on
 * success, nonzero to abort the probe.                                      */
typedef int (*mmaemu_mma_fn)(void *ctx, int fmt, const void *A, const void *B, const uint32_t *C,
                             uint32_t *D, size_t ntiles);

/* Built-in callbacks.  Both copy the tiles to the current CUDA device, run
 * there on the stream selected with mmaemu_set_stream, and copy D back.
 *  mmaemu_mma_emulated: ctx points to an int holding MMAEMU_AMPERE or
 *                       MMAEMU_HOPPER; runs mmaemu_tiles.
 *  mmaemu_mma_native:   ctx unused; runs mmaemu_native_tiles (B200's
 *                       tensor cores).                                       */
int mmaemu_mma_emulated(void *ctx, int fmt, const void *A, const void *B, const uint32_t *C, uint32_t *D,
                        size_t ntiles);
int mmaemu_mma_native(void *ctx, int fmt, const void *A, const void *B, const uint32_t *C, uint32_t *D,
                      size_t ntiles);

/* B200's own MMA on a tile batch (device pointers, asynchronous, layouts as
 * mmaemu_tiles): mma.sync m16n8k16 with fp32 accumulation for FP16 and
 * BF16, m16n8k32 with k >= 16 zero for E4M3.  Not an emulation: it is what
 * the probes characterise.  Errors as mmaemu_tiles.                         */
int mmaemu_native_tiles(int fmt, const void *A, const void *B, const float *C, float *D, size_t ntiles);

/* Internal precision ("Internal Precision Detection"): C = 2^E0 plus
 * sixteen products of 2^(E0 - j) for j = 16 .. 27.  The products are kept
 * exactly -- D is the exact sum -- when j <= F, the number of fraction bits
 * kept below the group's largest exponent (internal significand width
 * F + 1); beyond it they are dropped or rounded to whole units, whatever
 * the rounding.  *fraction_bits = the largest j kept exactly, 15 if none
 * is, 27 if all are (a lower bound).                                        */
int mmaemu_probe_precision(int fmt, mmaemu_mma_fn mma, void *ctx, int *fraction_bits);

/* Rounding modes reported by the next two probes. */
enum {
  MMAEMU_ROUND_TOWARD_ZERO = 0,
  MMAEMU_ROUND_NEAREST = 1,   /* to nearest (ties not resolved by the probe) */
  MMAEMU_ROUND_DOWN = 2,      /* toward -Inf (floor of the signed value)     */
  MMAEMU_ROUND_UP = 3,        /* toward +Inf                                 */
  MMAEMU_ROUND_NEAREST_EVEN = 4,
  MMAEMU_ROUND_OTHER = 5,
  MMAEMU_ROUND_NEAREST_AWAY = 6  /* to nearest, ties away from zero           */
};

/* Alignment rounding ("Rounding Mode Detection"): C = 2^E0 plus sixteen
 * products of +-0.75 units of the grid 2^(E0 - F), where F comes from
 * mmaemu_probe_precision.  Truncation drops both signs; rounding to nearest
 * keeps one unit of each; floor/ceil keep one sign.  *mode is one of
 * TOWARD_ZERO, NEAREST, DOWN, UP.                                           */
int mmaemu_probe_alignment_rounding(int fmt, mmaemu_mma_fn mma, void *ctx, int fraction_bits, int *mode);

/* Write-back rounding (the final cast to fp32): exact sums +-(3.5 - 2^-23)
 * and +-(3.5 - 3 2^-23), each a tie between two fp32 values, the even one
 * above and below in magnitude respectively (C = 2 - 2^-23 or 2 - 3 2^-23,
 * one product 1.5 as the last term, P[16], so that only the final cast sees
 * the tie).  *mode is TOWARD_ZERO, NEAREST_EVEN, NEAREST_AWAY,
 * DOWN, UP or OTHER.  Needs F >= 23 so that the sums are held exactly.     */
int mmaemu_probe_writeback_rounding(int fmt, mmaemu_mma_fn mma, void *ctx, int *mode);

/* Normalisation stage ("Normalization Stage Detection"): products 1.5 x 1.5
 * and 1.5 x -1.5 cancel; C carries a bit 2^-F below the products' exponent
 * 0.  If products are accumulated unnormalised (exponent 0) C comes back
 * exactly; if 2.25 is first normalised to exponent 1 the bit is half a unit
 * of the grid and is dropped or rounded away.  *delayed = 1 (delayed
 * normalisation) or 0 (normalised first).  Needs 23 <= F <= 27.            */
int mmaemu_probe_normalization(int fmt, mmaemu_mma_fn mma, void *ctx, int fraction_bits, int *delayed);

/* Subnormal products ("Subnormal Behavior Detection"): the smallest
 * subnormal times 1.0, plus a C term of a quarter unit of the grid the
 * product sets if it keeps the format's minimum exponent.  *renormalized =
 * 1 when the sum comes back exactly (the product was renormalised to its
 * true exponent, which makes the grid fine enough), 0 otherwise.
 * MMAEMU_EUNSUPPORTED for BF16, whose subnormal products lie below fp32's
 * range, and where F + 2 - p > 23 (the sum would not be an fp32 value).   */
int mmaemu_probe_subnormal(int fmt, mmaemu_mma_fn mma, void *ctx, int fraction_bits, int *renormalized);

/* Computationally neutral subgroups ("Summation Dependency & Order",
 * Algorithm 4).  Terms: bit 0 = C, bit i = P[i] = A[m][i-1] B[i-1][n].  For
 * each subset S (a bit mask over the 17 terms, 2 <= |S| <= 16), two
 * instances are run: S's terms engineered to cancel exactly (+X on its first
 * term, -X on its last, the rest zero) and S's terms all zero, with
 * distinct small terms outside S whose low bits a large group maximum would
 * truncate.  neutral[s] = 1 when the two are bitwise equal.  Passing all
 * 2^17 masks is the exhaustive search (16384 tiles).  EINVAL for a mask
 * outside the size range.                                                  */
int mmaemu_probe_neutral(int fmt, mmaemu_mma_fn mma, void *ctx, const uint32_t *subsets, size_t nsubsets,
                         uint8_t *neutral);

/* Exponent threshold (the BF16 paragraph of the recovered pipeline: "max
 * exponent threshold -133").  For a candidate floor L, one instance sums
 * (2^k - 2) units of 2^(L - F) (k = F - L - 149, so 2^k units make
 * 2^-149) and fifteen products of 0.875 units: with the group maximum
 * floored at L or above, the small products truncate away and the result is
 * +0; with a lower floor (or none) they carry the sum to 2^-149.  L runs
 * over F - 158 .. F - 150 (-133 is always inside).  *e_floor = the largest L
 * that gives +0; MMAEMU_NO_FLOOR if none does (no floor at or above
 * F - 158); F - 150 if all do (a lower bound).  BF16 only (other formats'
 * products cannot reach the threshold): MMAEMU_EUNSUPPORTED otherwise.     */
#define MMAEMU_NO_FLOOR (-100000)
int mmaemu_probe_floor(int fmt, mmaemu_mma_fn mma, void *ctx, int fraction_bits, int *e_floor);

/* A model as data: what the target tests measure, and what the emulation
 * needs ("Hawkeye: Reproducing GPU-Level Non-Determinism (MLSys 2026)"
 * reading notes -- Obs. 2 and 3 for the fields; the BF16 paragraph for the
 * threshold).                                                              */
#define MMAEMU_FLOOR_ANY 100000 /* in an identify query: the floor was not measured */
typedef struct mmaemu_model_desc {
  int fraction_bits;          /* F: bits kept below the group's largest exponent  */
  int stages;                 /* accumulation stages (C joins the first)          */
  int stage_products[4];      /* products per stage, in k order; they sum to 16   */
  int e_floor;                /* floor on each group's max exponent, NO_FLOOR,   */
                              /* or (in a query) FLOOR_ANY                        */
  int alignment_rounding;     /* MMAEMU_ROUND_*                                   */
  int writeback_rounding;     /* MMAEMU_ROUND_*                                   */
  int delayed_normalization;  /* 1: products accumulate unnormalised              */
  int subnormal_renormalized; /* 1: subnormal products are renormalised           */
  uint32_t nan_bits;          /* fp32 NaN result pattern; 0 in a query: any       */
} mmaemu_model_desc;

/* The parameters of a built-in model (MMAEMU_AMPERE, _HOPPER, _B200;
 * MMAEMU_LOVELACE is Ampere).  Errors: MMAEMU_EINVAL.                     */
int mmaemu_model_describe(int model, mmaemu_model_desc *out);

/* The built-in model with exactly these parameters (nan_bits 0 matches any
 * NaN pattern, e_floor FLOOR_ANY any floor; stage_products beyond `stages`
 * are ignored) -- e.g. the
 * result of the target tests on some MMA.  MMAEMU_EUNSUPPORTED when no
 * built-in model matches: the library can describe that MMA but not
 * emulate it.  Errors: MMAEMU_EINVAL.                                      */
int mmaemu_model_identify(const mmaemu_model_desc *desc, int *model);

#ifdef __cplusplus
}
#endif

#endif /* MMAEMU_PROBE_H */
