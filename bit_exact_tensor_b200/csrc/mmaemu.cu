// libmmaemu: bit-exact emulation of Ampere / Hopper Tensor Core MMA arithmetic
// on B200 CUDA cores (sm_100a), behind the C ABI declared in include/mmaemu.h.
//
// Kernels
//   gemm_kernel   -- D = C + A.B over 16-wide K chunks (ascending, each chunk's
//                    fp32 result feeding the next), fused per-tile xorsum;
//                    operand panels decoded once per call (decode_a_kernel,
//                    decode_b_kernel) and staged by bulk asynchronous copies.
//   tiles_kernel  -- independent 16x16x16 tiles, two per warp (4 x 4 outputs a lane).
//   xorsum_kernel -- XOR of a buffer of 32-bit words.
// The arithmetic model and its exact-double formulation are described in
// mmaemu_core.cuh.  Tensor cores are deliberately not used: B200's own MMA
// arithmetic is not the arithmetic being emulated.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "mmaemu.h"
#include "mmaemu_core.cuh"
#include "host_slabs.h"

namespace mmaemu {

// ---------------------------------------------------------------------------
// device status word: bit 0 -- a bounded wait gave up; bit 1 -- a bounds
// check of the checking build failed (mmaemu_device_status reads it)
// ---------------------------------------------------------------------------
__device__ uint32_t g_status;
constexpr uint32_t STATUS_TIMEOUT = 1u, STATUS_BOUNDS = 2u;

#ifdef MMAEMU_BOUNDS_CHECK
// checking build: an index outside its buffer is recorded and the access
// that would use it is skipped
#define MMAEMU_CHECK(ok, cond)                      \
  do {                                              \
    if (!(cond)) {                                  \
      (ok) = false;                                 \
      atomicOr(&::mmaemu::g_status, STATUS_BOUNDS); \
    }                                               \
  } while (0)
#else
#define MMAEMU_CHECK(ok, cond) \
  do {                         \
  } while (0)
#endif

// Per-output bit masks of a thread's R x CC block (bit r*CC+c): 32 bits for
// up to 32 outputs, 64 beyond.
template <int N> struct OutMaskT { using type = uint32_t; };
template <> struct OutMaskT<64> { using type = unsigned long long; };
template <int N> using OutMask = typename OutMaskT<N>::type;

// ---------------------------------------------------------------------------
// decoded operand panels in shared memory, [k][row] for A and [k][col] for B
// ---------------------------------------------------------------------------
// One 16-deep K chunk: the operands as exact doubles (B times 1 + 2^-40),
// their exponent codes, per row of A and column of B the sign word, and a
// word that is nonzero when the chunk holds an Inf or NaN operand.  Sign
// words: element k = 8h + 2j + b owns bit sign_bit(k) = 2j + h + 16b and bit
// sign_bit(k) + 8 (k < 8 the even bits, k >= 8 the odd ones -- the positions
// the packed decode produces directly).  A sets sign_bit(k) for a negative
// nonzero finite a[k] and sign_bit(k) + 8 for a positive one; B the other way
// round, so the AND of a row's and a column's words has one bit per negative
// product of nonzero finite operands.  Zero, Inf and NaN operands set none.
template <int BM, int BN>
struct __align__(16) Panel {
  double aV[16][BM];
  uint32_t aQ2[16][BM];  // (q, q): an A code paired with two B codes
  uint32_t aS[BM];
  uint32_t aF[4];
  double bV[16][BN];     // column pairs swizzled in 64-column panels (bslot)
  int16_t bQ[16][BN];
  uint32_t bS[BN];
  uint32_t bF[4];
  // Slot of column n in a row of bV.  A GEMM thread reads its 8 consecutive
  // columns as 4 pairs, and the 8 threads of a quarter warp read the 8
  // column groups, 64 bytes apart: groups g and g + 2, g + 4, g + 6 would
  // share banks.  Storing pair q of group g at pair q ^ ((g >> 1) & 3) gives
  // every group of a quarter warp a bank range of its own.  The tile
  // kernel's 16-column panels keep natural order (its 4-column groups are
  // conflict-free).
  static __host__ __device__ constexpr int bslot(int n) {
    return BN == 64 ? ((n & ~7) | ((((n >> 1) & 3) ^ ((n >> 4) & 3)) << 1) | (n & 1)) : n;
  }
};

__host__ __device__ constexpr int sign_bit(int k) { return (k & 6) + (k >> 3) + 16 * (k & 1); }

template <class PanelT>
__device__ __forceinline__ int32_t code_a(const PanelT &P, int k, int m) { return lo16(P.aQ2[k][m]); }
template <class PanelT>
__device__ __forceinline__ int32_t code_b(const PanelT &P, int k, int n) { return P.bQ[k][n]; }
template <class PanelT>
__device__ __forceinline__ bool neg_a(const PanelT &P, int k, int m) { return __double2hiint(P.aV[k][m]) < 0; }
template <class PanelT>
__device__ __forceinline__ bool neg_b(const PanelT &P, int k, int n) {
  return __double2hiint(P.bV[k][PanelT::bslot(n)]) < 0;
}

// Unroll of the GEMM's product loops, measured per model and format:
// Ampere FP16 2, BF16 4; the one-stage models 8 for FP16 and E4M3, 4 for
// BF16 (Ampere's exponent pass is unrolled fully, see mma_chunk).
#ifndef MMAEMU_KUNROLL
template <int MODEL, int FMT>
constexpr int kUnroll = MODEL == MODEL_AMPERE ? (FMT == FMT_FP16 ? 2 : 4) : (FMT == FMT_BF16 ? 4 : 8);
#else
template <int MODEL, int FMT>
constexpr int kUnroll = MMAEMU_KUNROLL;
#endif

template <int R, typename T>
__device__ __forceinline__ void lds_vec(const T *p, T (&v)[R]) {
  static_assert(sizeof(T) == 4, "32-bit elements");
  if constexpr (R == 8) {
    const uint4 a = reinterpret_cast<const uint4 *>(p)[0], b = reinterpret_cast<const uint4 *>(p)[1];
    v[0] = (T)a.x; v[1] = (T)a.y; v[2] = (T)a.z; v[3] = (T)a.w;
    v[4] = (T)b.x; v[5] = (T)b.y; v[6] = (T)b.z; v[7] = (T)b.w;
  } else if constexpr (R == 4) {
    const uint4 a = reinterpret_cast<const uint4 *>(p)[0];
    v[0] = (T)a.x; v[1] = (T)a.y; v[2] = (T)a.z; v[3] = (T)a.w;
  } else if constexpr (R == 2) {
    const uint2 a = reinterpret_cast<const uint2 *>(p)[0];
    v[0] = (T)a.x; v[1] = (T)a.y;
  } else {
#pragma unroll
    for (int i = 0; i < R; i++) v[i] = p[i];
  }
}
template <int R>
__device__ __forceinline__ void lds_dvec(const double *p, double (&v)[R]) {
  static_assert(R % 2 == 0, "pairs of doubles");
#pragma unroll
  for (int i = 0; i < R / 2; i++) {
    const double2 t = reinterpret_cast<const double2 *>(p)[i];
    v[2 * i] = t.x;
    v[2 * i + 1] = t.y;
  }
}

__device__ __forceinline__ double fma_rz(double a, double b, double c) {
  double d;
  asm("fma.rz.f64 %0, %1, %2, %3;" : "=d"(d) : "d"(a), "d"(b), "d"(c));
  return d;
}
__device__ __forceinline__ double fma_rn(double a, double b, double c) {
  double d;
  asm("fma.rn.f64 %0, %1, %2, %3;" : "=d"(d) : "d"(a), "d"(b), "d"(c));
  return d;
}
// truncation to 24 significant bits (toward zero) of a normal double, zero,
// Inf or NaN with an all-ones high word
__device__ __forceinline__ double mask24(double v) {
  return __hiloint2double(__double2hiint(v), __double2loint(v) & (int)0xE0000000u);
}
// 2^k as a double (normal k)
__host__ __device__ constexpr double pow2d(int k) {
  double r = 1.0;
  for (; k > 0; k--) r *= 2.0;
  for (; k < 0; k++) r *= 0.5;
  return r;
}

// High word of a group's base 1.5 * 2^52 * u, u = 2^(e_max - F), from the
// packed code pair nm (lane 0 for the even output, lane 1 for the odd one):
// e_max = 1024 - nm / 16 gives the exponent field 2099 - F - nm / 16.  For
// the odd output the low lane's code is subtracted from the low mantissa
// bits as well (it is below 2^15, so it never borrows from the exponent):
// that base is a little below 1.5 * 2^52 u, still a multiple of u in the
// same binade, and the same value is used to add and to subtract it.
template <int F, int ODD>
__device__ __forceinline__ uint32_t base_hi(uint32_t nm) {
  constexpr uint32_t KHI = ((uint32_t)(2099 - F) << 20) | 0x80000u;
  return ODD ? KHI - nm : KHI + nm * 0xFFFF0000u;
}

// Carried terms' codes, two outputs per word, from the top 16 bits of their
// doubles: unchecked (value as is) ncode(e) = (2047 - field) * 16 directly;
// checked (value times 2^s, field >= 1024 for every nonzero value) the low
// ten exponent bits give ncode(e) - 16 s, and the offset is added later.
template <bool CHK, int R, int CC>
__device__ __forceinline__ void carry_codes(const double (&X)[R][CC], uint32_t (&c2)[R][CC / 2]) {
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) {
      const uint32_t x = __byte_perm((uint32_t)__double2hiint(X[r][2 * p]), (uint32_t)__double2hiint(X[r][2 * p + 1]),
                                     0x7632);
      c2[r][p] = ~x & (CHK ? 0x3FF03FF0u : 0x7FF07FF0u);
    }
}

// Group codes: from the carried terms' codes (carry_codes; checked codes get
// their offset to ncode and the -133 floor, which changes nothing but BF16)
// down to the minimum over the group's products, qa + qb for k in [K0, K0 +
// KN), two outputs per packed add-and-min: nm becomes ncode(e_max).
template <int FMT, bool CHK, int KN, int UNR, int R, int C2, class PanelT>
__device__ __forceinline__ void group_codes(const PanelT &P, int rl, int cl, int K0, uint32_t (&nm)[R][C2],
                                            int SIN) {
  constexpr int CC = 2 * C2;
  if constexpr (CHK) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int p = 0; p < C2; p++)
        nm[r][p] = vmin2(vadd2(nm[r][p], (uint32_t)(16 * SIN) * 0x10001u), pair16(FLOOR_CODE, FLOOR_CODE));
  } else {
    static_assert(!kNeedsFloor<FMT>, "BF16 runs checked");
  }
#pragma unroll UNR
  for (int i = 0; i < KN; i++) {
    const int k = K0 + i;
    uint32_t an2[R], bn2[C2];
    lds_vec<R>(&P.aQ2[k][rl], an2);
    lds_vec<C2>(reinterpret_cast<const uint32_t *>(&P.bQ[k][cl]), bn2);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int p = 0; p < C2; p++) nm[r][p] = vmin2(vadd2(an2[r], bn2[p]), nm[r][p]);
  }
  (void)CC;
}

// Accumulators of one group: base plus the count of negative terms, then the
// carried value (X on entry) added like a product, times the same 1 + 2^-40.
template <int F, int R, int CC, int C2, class PanelT>
__device__ __forceinline__ void group_start(const PanelT &P, int rl, int cl, double (&X)[R][CC],
                                            const uint32_t (&nm)[R][C2], double SKEW, uint32_t GM) {
  uint32_t sa[R], sb[CC];
  lds_vec<R>(&P.aS[rl], sa);
  lds_vec<CC>(&P.bS[cl], sb);
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t hi = (c & 1) ? base_hi<F, 1>(nm[r][c / 2]) : base_hi<F, 0>(nm[r][c / 2]);
      const uint32_t cnt = __popc(sa[r] & sb[c] & GM) + ((uint32_t)__double2hiint(X[r][c]) >> 31);
      X[r][c] = fma_rz(X[r][c], SKEW, __hiloint2double((int)hi, (int)cnt));
    }
}

// One round-toward-zero fused multiply-add per product of k in [K0, K0+KN).
template <int KN, int UNR, int R, int CC, class PanelT>
__device__ __forceinline__ void group_products(const PanelT &P, int rl, int cl, int K0, double (&X)[R][CC]) {
  static_assert(CC == 8 || CC == 4, "column groups of 8 or 4");
  const int sw = (cl >> 4) & 3;  // the column group's pair swizzle (Panel::bslot)
#pragma unroll UNR
  for (int i = 0; i < KN; i++) {
    const int k = K0 + i;
    double a[R], b[CC];
    lds_dvec<R>(&P.aV[k][rl], a);
    if constexpr (CC == 8) {
#pragma unroll
      for (int q = 0; q < 4; q++) {
        const double2 t = *reinterpret_cast<const double2 *>(&P.bV[k][cl + 2 * (q ^ sw)]);
        b[2 * q] = t.x;
        b[2 * q + 1] = t.y;
      }
    } else {
      lds_dvec<CC>(&P.bV[k][cl], b);
    }
#pragma unroll
    for (int c = 0; c < CC; c++)
#pragma unroll
      for (int r = 0; r < R; r++) X[r][c] = fma_rz(a[r], b[c], X[r][c]);
  }
}

// exact group value: accumulator minus its base
template <int F, int R, int CC>
__device__ __forceinline__ double group_value(const double (&X)[R][CC], const uint32_t (&nm)[R][CC / 2], int r,
                                              int c) {
  uint32_t hi;
  constexpr uint32_t KHI = ((uint32_t)(2099 - F) << 20) | 0x80000u;
  if (c & 1) asm volatile("sub.u32 %0, %1, %2;" : "=r"(hi) : "r"(KHI), "r"(nm[r][c / 2]));
  else asm volatile("mad.lo.u32 %0, %1, %2, %3;" : "=r"(hi) : "r"(nm[r][c / 2]), "r"(0xFFFF0000u), "r"(KHI));
  return X[r][c] - __hiloint2double((int)hi, 0);
}

// Checked states below 2^-126 in magnitude: truncate onto the fp32 subnormal
// grid 2^-149 (a value that truncates to zero keeps the sign of the sum), and
// give the carried term the exponent -126 of an fp32 subnormal.  c2 holds the
// carried codes of carry_codes<true>: normal scaled fp32 values give 16..4064,
// zero 16368, Inf and NaN 0, fp32 subnormals lie strictly between.
template <int R, int CC>
__device__ __forceinline__ void subnormal_states(double (&X)[R][CC], uint32_t (&c2)[R][CC / 2],
                                                 OutMask<R * CC> &dneg0) {
  uint32_t t = 0xFFFFFFFFu;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) t = vminu2(t, vadd2(c2[r][p], pair16(-4065, -4065)));
  if ((t & 0xFFFFu) >= 12303u && (t >> 16) >= 12303u) return;
  // rare: unrolled, so that the states stay in registers
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t code = (c & 1) ? (c2[r][c / 2] >> 16) : (c2[r][c / 2] & 0xFFFFu);
      if (code <= 4064u || code >= 16368u) continue;
      const OutMask<R * CC> bit = OutMask<R * CC>(1) << (r * CC + c);
      const double x = X[r][c];
      constexpr double TO_Q = pow2d(-(S_WB - 149)), FROM_Q = pow2d(S_WB - 149);
    const double q = trunc(fabs(x) * TO_Q);  // |value| 2^149
      if (q == 0.0) {
        X[r][c] = 0.0;
        dneg0 = x < 0.0 ? (dneg0 | bit) : (dneg0 & ~bit);
      } else {
        X[r][c] = copysign(q * FROM_Q, x);
        const uint32_t sub = (uint32_t)(SUBN_CODE - 16 * S_WB);
        c2[r][c / 2] = (c & 1) ? ((c2[r][c / 2] & 0xFFFFu) | (sub << 16)) : ((c2[r][c / 2] & 0xFFFF0000u) | sub);
      }
    }
}

// Special-value outcome of each output of an R x CC block whose chunk holds
// Inf or NaN somewhere in its A or B panel: 2 bits per output (0 none, 1 NaN,
// 2 +Inf, 3 -Inf).  Any NaN, or Inf x 0, gives NaN; infinities of both signs
// (including an infinite incoming value) give NaN, of one sign that Inf.
// c_nan / c_infp / c_infn flag outputs whose incoming value is NaN / +Inf /
// -Inf.  Kept out of line: it is rare.
template <int R, int CC, class PanelT>
__device__ __forceinline__ uint64_t special_codes(const PanelT *P, int rl, int cl, uint32_t c_nan, uint32_t c_infp,
                                               uint32_t c_infn) {
  uint64_t codes = 0;
#pragma unroll 1
  for (int o = 0; o < R * CC; o++) {
    const int r = o / CC, c = o % CC;
    bool nan = (c_nan >> o) & 1u, ip = (c_infp >> o) & 1u, in = (c_infn >> o) & 1u;
#pragma unroll 1
    for (int k = 0; k < 16; k++) {
      const int32_t aq = code_a(*P, k, rl + r), bq = code_b(*P, k, cl + c);
      if (aq == QNAN || bq == QNAN) {
        nan = true;
      } else if (aq == QINF || bq == QINF) {
        if (aq == QZ || bq == QZ) nan = true;
        else if (neg_a(*P, k, rl + r) != neg_b(*P, k, cl + c)) in = true;
        else ip = true;
      }
    }
    const uint64_t code = (nan || (ip && in)) ? 1u : ip ? 2u : in ? 3u : 0u;
    codes |= code << (2 * o);
  }
  return codes;
}

// zero-sign rule for a zero sum: -0 only when the incoming value is -0 and
// all 16 products are zeros of negative sign
template <class PanelT>
__device__ __forceinline__ bool all_products_negative_zero(const PanelT *P, int m, int n) {
#pragma unroll 1
  for (int k = 0; k < 16; k++) {
    const bool zero = code_a(*P, k, m) == QZ || code_b(*P, k, n) == QZ;
    if (!zero || neg_a(*P, k, m) == neg_b(*P, k, n)) return false;
  }
  return true;
}

// Ampere hand-over: the stage-1 value truncated to 24 bits, exponent
// unbounded (checked: times 2^512, formed in one exact fused multiply-add); a
// zero stage adds nothing.  The unchecked form hands over the exact value:
// stage 2's grid 2^(e_max - 23), with e_max at least the value's own
// exponent, is never finer than its 24-bit unit, and truncations to nested
// power-of-two grids compose, so stage 2 adds the same.
template <bool CHK, int F, int R, int CC>
__device__ __forceinline__ void hand_over(double (&X)[R][CC], const uint32_t (&nm)[R][CC / 2]) {
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      if constexpr (CHK) {
        constexpr double UP_HO = pow2d(S_HO);
        const uint32_t hi = (c & 1) ? base_hi<F, 1>(nm[r][c / 2]) : base_hi<F, 0>(nm[r][c / 2]);
        X[r][c] = mask24(fma_rn(X[r][c], UP_HO, -__hiloint2double((int)(hi + ((uint32_t)S_HO << 20)), 0)));
      } else {
        X[r][c] = group_value<F>(X, nm, r, c);
      }
    }
}

// Toward-zero write-back (checked: times 2^896, rounded to nearest, so that
// values from 2^128 up become infinite).  The unchecked Ampere form carries
// the exact value for the reason given at the hand-over (the next chunk's
// first group has F = 23 as well); its truncation to fp32 happens once, in
// states_to_fp32 or scale_states.  Hopper's and B200's groups have finer
// grids than the fp32 unit, so their carried value must be truncated here.
template <bool CHK, int F, int R, int CC>
__device__ __forceinline__ void write_back(double (&X)[R][CC], const uint32_t (&nm)[R][CC / 2]) {
  constexpr bool kExactCarry = !CHK && F == 23;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      constexpr double UP_WB = pow2d(S_WB);
      const double g = group_value<F>(X, nm, r, c);
      const double v = kExactCarry ? g : mask24(g);
      X[r][c] = CHK ? __dmul_rn(v, UP_WB) : v;
    }
}

// Kinds of the incoming values (bit r*CC+c per output), needed only when a
// chunk's A or B holds Inf or NaN.
template <int R, int CC>
__device__ __forceinline__ void incoming_kinds(const double (&X)[R][CC], OutMask<R * CC> &c_nan,
                                               OutMask<R * CC> &c_infp, OutMask<R * CC> &c_infn) {
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const OutMask<R * CC> bit = OutMask<R * CC>(1) << (r * CC + c);
      if (isnan(X[r][c])) c_nan |= bit;
      else if (isinf(X[r][c])) (X[r][c] < 0.0 ? c_infn : c_infp) |= bit;
    }
}

// End of a chunk, after the write-back: the zero-sign rule and the outputs
// that Inf / NaN operands decide.
template <bool CHK, int R, int CC, class PanelT>
__device__ __forceinline__ void chunk_finish(const PanelT &P, int rl, int cl, double (&X)[R][CC],
                                             OutMask<R * CC> &dneg0, bool panel_special, OutMask<R * CC> c_nan,
                                             OutMask<R * CC> c_infp, OutMask<R * CC> c_infn, bool &to_checked) {
  using Mask = OutMask<R * CC>;
  // signed zeros: only an output whose incoming value was -0 can give -0,
  // and only when its sum is zero and all its 16 products are zeros of
  // negative sign
  if (dneg0) {
    Mask zero = 0;  // outputs whose sum is zero (a zero state is +0 here)
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) zero |= (Mask)(__double2hiint(X[r][c]) == 0) << (r * CC + c);
    dneg0 &= zero;
    if (dneg0) {  // rare: a -0 input met a zero sum
#pragma unroll
      for (int r = 0; r < R; r++)
#pragma unroll
        for (int c = 0; c < CC; c++) {
          const Mask bit = Mask(1) << (r * CC + c);
          if ((dneg0 & bit) && !all_products_negative_zero(&P, rl + r, cl + c)) dneg0 &= ~bit;
        }
    }
  }
  // Inf / NaN operands (special_codes covers 32 outputs per call)
  if (panel_special) {
    constexpr int RH = R * CC > 32 ? 32 / CC : R;
#pragma unroll
    for (int h = 0; h < R / RH; h++) {
      const int sh = h * RH * CC;
      const uint64_t spec = special_codes<RH, CC>(&P, rl + h * RH, cl, (uint32_t)(c_nan >> sh),
                                                  (uint32_t)(c_infp >> sh), (uint32_t)(c_infn >> sh));
#pragma unroll
      for (int r = 0; r < RH; r++)
#pragma unroll
        for (int c = 0; c < CC; c++) {
          const uint32_t code = (uint32_t)(spec >> (2 * (r * CC + c))) & 3u;
          if (code == 0u) continue;
          X[h * RH + r][c] = code == 1u ? __longlong_as_double(0x7FF8000000000000ll)
                                        : code == 2u ? __longlong_as_double(0x7FF0000000000000ll)
                                                     : __longlong_as_double((long long)0xFFF0000000000000ull);
          dneg0 &= ~(Mask(1) << (sh + r * CC + c));
          if (!CHK) to_checked = true;
        }
    }
  }
}

// One 16-deep K chunk for an R x CC block of outputs, updating the states X
// in place.  CHK selects the checked form (values times 2^896; overflow,
// underflow, Inf and NaN handled); the unchecked form serves FP16 / E4M3
// states that cannot leave the normal fp32 range (see init_states).
//   dneg0      -- bit r*CC+c set when that output's state is -0 (stored +0)
//   to_checked -- set by the unchecked form when an Inf/NaN operand made a
//                 result infinite or NaN: the caller scales the states and
//                 continues checked
// Ampere's two stages run as a loop over one copy of the group code, so
// that the compiler cannot interleave them (which costs registers).
template <int MODEL, int FMT, bool CHK, int UNR, int R, int CC, class PanelT>
__device__ __forceinline__ void mma_chunk(const PanelT &P, int rl, int cl, double (&X)[R][CC],
                                          OutMask<R * CC> &dneg0, bool panel_special, bool &to_checked) {
  constexpr int F = ModelT<MODEL>::F;
  constexpr int KN = ModelT<MODEL>::STAGE1;  // group size
  constexpr int NST = MODEL == MODEL_AMPERE ? 2 : 1;
  // the exponent pass holds few registers: Ampere's 8-deep groups unroll it
  // fully (measured: 5.7% off the FP16 GEMM; Hopper's 16-deep ones are
  // slower fully unrolled and keep UNR)
  constexpr int CUNR = MODEL == MODEL_AMPERE ? KN : UNR;
  static_assert((R * CC <= 32 || R * CC == 64) && CC % 2 == 0, "per-output masks hold 32 or 64 outputs");
  constexpr double SKEW_PLAIN = 1.0 + pow2d(-40), SKEW_WB = SKEW_PLAIN * pow2d(-S_WB),
                   SKEW_HO = SKEW_PLAIN * pow2d(-S_HO);

  OutMask<R * CC> c_nan = 0, c_infp = 0, c_infn = 0;
  if (CHK && panel_special) incoming_kinds(X, c_nan, c_infp, c_infn);
  uint32_t nm[R][CC / 2];
  carry_codes<CHK>(X, nm);
  if constexpr (CHK) subnormal_states(X, nm, dneg0);
#pragma unroll 1
  for (int st = 0; st < NST; st++) {
    const int sin = !CHK ? 0 : st ? S_HO : S_WB;
    const double skew = !CHK ? SKEW_PLAIN : st ? SKEW_HO : SKEW_WB;
    const uint32_t gm = NST == 1 ? 0xFFFFFFFFu : st ? 0xAAAAAAAAu : 0x55555555u;  // the group's sign bits
    const int k0 = KN * st;
    group_codes<FMT, CHK, KN, CUNR>(P, rl, cl, k0, nm, sin);
    group_start<F>(P, rl, cl, X, nm, skew, gm);
    if constexpr (NST == 1 || FMT == FMT_FP16) {
      // the last product outside the loop, so that the scheduler can run
      // the write-back's (or hand-over's) integer work beside its FP64
      // multiply-adds (measured: faster for the one-stage models and Ampere
      // FP16, slower for Ampere BF16)
      group_products<KN - 1, UNR>(P, rl, cl, k0, X);
      group_products<1, 1>(P, rl, cl, k0 + KN - 1, X);
    } else {
      group_products<KN, UNR>(P, rl, cl, k0, X);
    }
    if (st + 1 < NST) {
      hand_over<CHK, F>(X, nm);
      carry_codes<CHK>(X, nm);
    }
  }
  write_back<CHK, F>(X, nm);
  chunk_finish<CHK>(P, rl, cl, X, dneg0, panel_special, c_nan, c_infp, c_infn, to_checked);
}

// ---------------------------------------------------------------------------
// states from C and back to fp32
// ---------------------------------------------------------------------------
// The unchecked form takes FP16 / E4M3 blocks whose C values are all +-0 or
// of magnitude in [2^-126, 2^100): a group with a nonzero product then has
// e_max >= -28 and a nonzero sum of at least 2^-53, and without one the sum
// is the carried value itself, so every result stays normal (or zero), and
// over any K < 2^31 the values stay below 2^101 (FP16 products are below
// 2^32, E4M3 products below 2^18; truncation never rounds up).
// (the range test, for a block: the largest |c| bit pattern below 2^100's,
// the smallest nonzero one at least 2^-126's; zeros wrap to the top in
// |c| - 1 and drop out of the minimum)
constexpr uint32_t UNCHECKED_MAX_BITS = 0x71800000u, UNCHECKED_MIN_BITS = 0x00800000u;

// track_neg0 = false: the caller knows that no output can end as -0 from
// a -0 incoming value (every product of the chunk is nonzero), so the -0
// mask starts empty.
template <int FMT, int R, int CC>
__device__ __forceinline__ bool init_states(const uint32_t (&cb)[R][CC], double (&X)[R][CC],
                                            OutMask<R * CC> &dneg0, bool track_neg0 = true) {
  uint32_t amax = 0, amin1 = 0xFFFFFFFFu;
  dneg0 = 0;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t v = cb[r][c], a = v & 0x7FFFFFFFu;
      amax = max(amax, a);
      amin1 = min(amin1, a - 1u);
      if (track_neg0) dneg0 |= (OutMask<R * CC>)(v == 0x80000000u) << (r * CC + c);
      // exact; -0 becomes +0 (its sign lives in dneg0); Inf and NaN stay so
      X[r][c] = (double)(__uint_as_float(v) + 0.0f);
    }
  const bool ok = FMT != FMT_BF16 && amax < UNCHECKED_MAX_BITS && amin1 >= UNCHECKED_MIN_BITS - 1u;
  if (!ok) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        constexpr double UP_WB = pow2d(S_WB);
        X[r][c] = __dmul_rn(X[r][c], UP_WB);  // Inf and NaN stay so
      }
  }
  return !ok;  // checked
}

template <int MODEL, int R, int CC>
__device__ __forceinline__ void states_to_fp32(double (&X)[R][CC], bool chk, OutMask<R * CC> dneg0,
                                               uint32_t (&D)[R][CC]) {
  if (!chk) {
    // unchecked states are +0 (a set dneg0 bit marks -0) or lie in the
    // normal fp32 range, where the conversion toward zero is the 24-bit
    // truncation (exact for a state that is truncated already)
    if (dneg0 == 0u) {
#pragma unroll
      for (int r = 0; r < R; r++)
#pragma unroll
        for (int c = 0; c < CC; c++) D[r][c] = __float_as_uint(__double2float_rz(X[r][c]));
      return;
    }
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++)
        D[r][c] = __float_as_uint(__double2float_rz(X[r][c])) | ((uint32_t)((dneg0 >> (r * CC + c)) & 1u) << 31);
    return;
  }
  uint32_t c2[R][CC / 2];
  carry_codes<true>(X, c2);
  subnormal_states(X, c2, dneg0);
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const double x = X[r][c];
      uint32_t bits;
      if (x == 0.0) bits = ((dneg0 >> (r * CC + c)) & 1u) ? 0x80000000u : 0u;
      else if (isnan(x)) bits = ModelT<MODEL>::NAN_BITS;
      else {
        constexpr double DOWN_WB = pow2d(-S_WB);
        bits = __float_as_uint(__double2float_rn(x * DOWN_WB));  // exact (Inf stays Inf)
      }
      D[r][c] = bits;
    }
}

// Unchecked states to the checked form: truncated to fp32 (an unchecked
// Ampere state may carry more bits; Inf and NaN pass unchanged) and scaled.
template <int R, int CC>
__device__ __forceinline__ void scale_states(double (&X)[R][CC]) {
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      constexpr double UP_WB = pow2d(S_WB);
      X[r][c] = __dmul_rn(mask24(X[r][c]), UP_WB);
    }
}

// raw fp32 bits of an R x CC block (row stride ldc), or +0 if !have_c
template <int R, int CC>
__device__ __forceinline__ void load_bits(const float *C, size_t ldc, bool have_c, uint32_t (&V)[R][CC]) {
#pragma unroll
  for (int r = 0; r < R; r++) {
    if (have_c) {
#pragma unroll
      for (int q = 0; q < CC / 4; q++) {
        const uint4 v = reinterpret_cast<const uint4 *>(C + r * ldc)[q];
        V[r][4 * q] = v.x; V[r][4 * q + 1] = v.y; V[r][4 * q + 2] = v.z; V[r][4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < CC; c++) V[r][c] = 0u;
    }
  }
}

// ---------------------------------------------------------------------------
// raw operand loading
// ---------------------------------------------------------------------------
template <int FMT>
struct Raw8 {  // 8 consecutive raw elements
  uint32_t w[FMT == FMT_E4M3 ? 2 : 4];
  __device__ __forceinline__ uint32_t get(int i) const {
    if constexpr (FMT == FMT_E4M3) return (w[i >> 2] >> (8 * (i & 3))) & 0xFFu;
    else return (w[i >> 1] >> (16 * (i & 1))) & 0xFFFFu;
  }
};

template <int FMT>
__device__ __forceinline__ Raw8<FMT> load_row8(const void *base, size_t elem_off, bool valid) {
  Raw8<FMT> r;
  if constexpr (FMT == FMT_E4M3) {
    uint2 v = valid ? *reinterpret_cast<const uint2 *>(static_cast<const uint8_t *>(base) + elem_off)
                    : make_uint2(0, 0);
    r.w[0] = v.x; r.w[1] = v.y;
  } else {
    uint4 v = valid ? *reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(base) + elem_off)
                    : make_uint4(0, 0, 0, 0);
    r.w[0] = v.x; r.w[1] = v.y; r.w[2] = v.z; r.w[3] = v.w;
  }
  return r;
}

// 8 elements of one column, stride ld elements apart
template <int FMT>
__device__ __forceinline__ Raw8<FMT> load_col8(const void *base, size_t elem_off, size_t ld, bool valid) {
  Raw8<FMT> r;
#pragma unroll
  for (int i = 0; i < (FMT == FMT_E4M3 ? 2 : 4); i++) r.w[i] = 0;
  if (valid) {
#pragma unroll
    for (int i = 0; i < 8; i++) {
      uint32_t x;
      if constexpr (FMT == FMT_E4M3) {
        x = static_cast<const uint8_t *>(base)[elem_off + i * ld];
        r.w[i >> 2] |= x << (8 * (i & 3));
      } else {
        x = static_cast<const uint16_t *>(base)[elem_off + i * ld];
        r.w[i >> 1] |= x << (16 * (i & 1));
      }
    }
  }
  return r;
}

// Decode 8 k-consecutive elements (k = 8h .. 8h+7) of A row m, or of B
// column n, into a panel; returns the sign-word bits of those 8 elements and
// whether one of them is Inf or NaN.
template <int FMT, class PanelT>
__device__ __forceinline__ uint32_t store_a8(PanelT &P, int m, int h, const Raw8<FMT> &raw, uint32_t &special) {
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const DecElem d = decode_elem<FMT>(raw.get(i));
    const int k = 8 * h + i;
    P.aV[k][m] = d.v;
    P.aQ2[k][m] = d.q | (d.q << 16);
    bits |= (d.neg << sign_bit(k)) | (d.pos << (sign_bit(k) + 8));
    special |= d.special;
  }
  return bits;
}
template <int FMT, class PanelT>
__device__ __forceinline__ uint32_t store_b8(PanelT &P, int n, int h, const Raw8<FMT> &raw, uint32_t &special) {
  uint32_t bits = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const DecElem d = decode_elem<FMT>(raw.get(i));
    const int k = 8 * h + i;
    constexpr double GROW = 1.0 + pow2d(-40);
    P.bV[k][PanelT::bslot(n)] = d.v * GROW;  // exact
    P.bQ[k][n] = (int16_t)d.q;
    bits |= (d.pos << sign_bit(k)) | (d.neg << (sign_bit(k) + 8));
    special |= d.special;
  }
  return bits;
}

// Fast decode of 8 k-consecutive elements (k = 8h .. 8h+7) of A row idx or
// B column idx into a tile panel, right for elements that hold no Inf or NaN
// (the caller tests fmax afterwards and decodes such tiles again).  Values come from exact hardware conversions (fp16
// and, through its fp32 bit pattern, bf16 to fp64; e4m3 first to an exact
// f16 pair), subnormals included.  The exponent codes and sign bits come
// from packed operations on element pairs of the 16-bit form: for e4m3 that
// form is fp16, whose exponent field is clamped below at 9 (e = -6, the e4m3
// subnormal exponent) instead of 1.
// two e4m3 (low byte first) to an fp16 pair, exactly
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t b16) {
  uint32_t r;
  asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(r) : "r"(b16));
  return r;
}
// an fp16 pair to two doubles, exactly
__device__ __forceinline__ void f16x2_to_f64(uint32_t w, double &lo, double &hi) {
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f64.f16 %0, l;\n\tcvt.f64.f16 %1, h;\n\t}"
      : "=d"(lo), "=d"(hi)
      : "r"(w));
}

// fmax: the running packed maximum of the 16-bit form's exponent fields,
// for the caller's Inf/NaN test after the fact (a field of all ones).
template <int FMT, bool ISB, class PanelT>
__device__ __forceinline__ uint32_t fast_store8(PanelT &P, int idx, int h, const Raw8<FMT> &raw, uint32_t &fmax) {
  // the 16-bit form: bf16 as stored, fp16 as stored, e4m3 converted to fp16
  constexpr bool BF = FMT == FMT_BF16;
  constexpr int P16 = BF ? 7 : 10, BIAS16 = BF ? 127 : 15;
  constexpr uint32_t EM2 = (BF ? 0xFFu : 0x1Fu) * 0x10001u;
  constexpr uint32_t FMIN = FMT == FMT_E4M3 ? 9u : 1u;  // smallest exponent field (subnormal exponent)
  // op_code(e) = K2 - 16 max(field, FMIN) for a nonzero element, QZ for a
  // zero one (field 0, so max(field, FMIN) = FMIN): with z = 1 for nonzero,
  // code = (K2 + QZ_ADD) - 16 max(field, FMIN) - z QZ_ADD, lane by lane
  // (every lane stays in [0, 2^16), so nothing borrows across lanes)
  constexpr uint32_t K2 = (uint32_t)(512 + BIAS16) * 16u;
  constexpr uint32_t QZ_ADD = (uint32_t)QZ - K2 + 16u * FMIN;
  constexpr uint32_t KQ = (K2 + QZ_ADD) * 0x10001u;
  static_assert(K2 + QZ_ADD < 65536u && K2 > 16u * 255u, "codes stay inside their 16-bit lanes");
  constexpr double GROW = 1.0 + pow2d(-40);
  uint32_t w16[4];
  if constexpr (FMT == FMT_E4M3) {
#pragma unroll
    for (int j = 0; j < 4; j++) w16[j] = e4m3x2_to_f16x2((raw.w[j >> 1] >> (16 * (j & 1))) & 0xFFFFu);
  } else {
#pragma unroll
    for (int j = 0; j < 4; j++) w16[j] = raw.w[j];
  }
  uint32_t sg = 0, nzw = 0;  // element 2j+b's sign / nonzero bit at bit 2j + 16b, before the offset h
#pragma unroll
  for (int j = 0; j < 4; j++) {
    const uint32_t w = w16[j];
    const int k = 8 * h + 2 * j;
    double v0, v1;
    if constexpr (BF) {
      v0 = (double)__uint_as_float(w << 16);
      v1 = (double)__uint_as_float(w & 0xFFFF0000u);
    } else {
      f16x2_to_f64(w, v0, v1);
    }
    if constexpr (ISB) {
      v0 *= GROW;  // exact
      v1 *= GROW;
    }
    const uint32_t z = vminu2(w & 0x7FFF7FFFu, 0x00010001u);  // 1 per nonzero element
    const uint32_t f = vmaxu2_16((w >> P16) & EM2, FMIN * 0x10001u);
    fmax = vmaxu2_16(fmax, f);
    const uint32_t q2 = KQ - 16u * f - QZ_ADD * z;
    if constexpr (ISB) {
      P.bV[k][PanelT::bslot(idx)] = v0;
      P.bV[k + 1][PanelT::bslot(idx)] = v1;
      P.bQ[k][idx] = (int16_t)(q2 & 0xFFFFu);
      P.bQ[k + 1][idx] = (int16_t)(q2 >> 16);
    } else {
      P.aV[k][idx] = v0;
      P.aV[k + 1][idx] = v1;
      P.aQ2[k][idx] = __byte_perm(q2, 0, 0x1010);
      P.aQ2[k + 1][idx] = __byte_perm(q2, 0, 0x3232);
    }
    sg |= (w >> (15 - 2 * j)) & (0x00010001u << (2 * j));
    nzw |= z << (2 * j);
  }
  const uint32_t neg = sg & nzw, pos = ~sg & nzw;
  return ISB ? (pos << h) | (neg << (h + 8)) : (neg << h) | (pos << (h + 8));
}

// ---------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------
// A block computes 64 x 64 outputs with 64 threads, one warp per 32 x 64
// and an 8 x 8 block of outputs per thread (about 250 registers); 4 blocks
// per SM.  Against 128 threads with 4 x 8 outputs each (128 registers, 16
// warps per SM) this halves the shared loads per product and doubles each
// thread's independent accumulators (measured: FP16 Ampere 4096^3
// 10.44 -> 9.85 ms).
#ifndef MMAEMU_GMINB
#define MMAEMU_GMINB 4
#endif
constexpr int GBM = 64, GBN = 64, GTHREADS = 64, GR = 8, GCC = 8;
using GPanel = Panel<GBM, GBN>;

// Everything a GEMM launch needs.  Element (m, k) of op(A) sits at
// A[m * lda + k] (ta == 0) or A[k * lda + m] (ta == 1); element (k, n) of
// op(B) at B[k * ldb + n] (tb == 0) or B[n * ldb + k] (tb == 1); C, D and
// Dref are row-major with their own leading dimensions.  Batch b (blockIdx.z)
// adds b times the batch stride to every pointer.  D, Dref, fp and mism may
// each be null; C null means +0.  The *_n fields are the extents (elements,
// or bytes for the workspace) the checking build bounds every index by.
struct GemmParams {
  const void *A, *B;
  const float *C;
  float *D;
  const float *Dref;        // claimed result to compare with (verify mode)
  uint32_t *fp;             // per-16x16-tile xorsum of the computed D
  unsigned long long *mism; // [0] mismatch count, [1] smallest mismatching index
  int M, N, K, ta, tb;
  long long lda, ldb, ldc, ldd, ldr;
  long long sA, sB, sC, sD, sR, sF;
  // decoded operand panels (workspace written by the decode pass): for each
  // batch entry, 64-row block of A or 64-column block of B, and K chunk, a
  // blob laid out exactly like that part of a shared-memory panel
  unsigned char *dA, *dB;
  int batch;
  size_t a_n, b_n, c_n, d_n, r_n, fp_n, dA_n, dB_n;
};

// Decoded panel blobs: the A part (aV .. aF) and the B part (bV .. bF) of a
// GPanel, stored contiguously in that order.
constexpr size_t ABLOB = offsetof(GPanel, bV), BBLOB = sizeof(GPanel) - offsetof(GPanel, bV);
static_assert(ABLOB == 16 * GBM * 8 + 16 * GBM * 4 + GBM * 4 + 16 && BBLOB == 16 * GBN * 8 + 16 * GBN * 2 + GBN * 4 + 16 &&
                  ABLOB % 16 == 0 && BBLOB % 16 == 0,
              "panel layout");

// Decode pass, A side: one block of 128 threads per blob (64 rows x 16 k):
// thread t decodes k = 8h .. 8h+7 of row m = rb * 64 + (t & 63), h = t >> 6.
template <int FMT>
__global__ void __launch_bounds__(128) decode_a_kernel(const GemmParams p) {
  constexpr int ESIZE = FMT == FMT_E4M3 ? 1 : 2;
  __shared__ uint32_t sgn[GBM];
  const int rb = blockIdx.x, j = blockIdx.y, nrb = gridDim.x, nch = gridDim.y;
  const size_t bz = blockIdx.z;
  const int t = threadIdx.x, ml = t & 63, h = t >> 6;
  const int m = rb * GBM + ml;
  if (t < GBM) sgn[t] = 0;
  __syncthreads();
  bool ok = true;
  const bool valid = m < p.M;
  const size_t k = 16 * (size_t)j + 8 * h, lda = (size_t)p.lda;
  const size_t off = bz * (size_t)p.sA + (!p.ta ? (size_t)m * lda + k : k * lda + m);
  MMAEMU_CHECK(ok, !valid || (!p.ta ? off + 8 : off + 7 * lda + 1) <= p.a_n);
  const Raw8<FMT> raw = !p.ta ? load_row8<FMT>(p.A, off, valid && ok) : load_col8<FMT>(p.A, off, lda, valid && ok);
  const size_t blob_i = (bz * nrb + rb) * (size_t)nch + j;
  MMAEMU_CHECK(ok, (blob_i + 1) * ABLOB <= p.dA_n);
  GPanel &P = *reinterpret_cast<GPanel *>(p.dA + blob_i * ABLOB);  // only the A part is written
  uint32_t special = 0;
  uint32_t bits = 0;
  if (ok) bits = store_a8<FMT>(P, ml, h, raw, special);
  atomicOr(&sgn[ml], bits);
  const int any = __syncthreads_or((int)special);
  if (ok && t < GBM) P.aS[t] = sgn[t];
  if (ok && t == 0) {
    P.aF[0] = (uint32_t)any;
    P.aF[1] = P.aF[2] = P.aF[3] = 0;
  }
  (void)ESIZE;
}

// Decode pass, B side: one block of 128 threads per blob (16 k x 64 columns):
// thread t decodes k = 8h .. 8h+7 of column n = cb * 64 + (t & 63).
template <int FMT>
__global__ void __launch_bounds__(128) decode_b_kernel(const GemmParams p) {
  __shared__ uint32_t sgn[GBN];
  const int cb = blockIdx.x, j = blockIdx.y, ncb = gridDim.x, nch = gridDim.y;
  const size_t bz = blockIdx.z;
  const int t = threadIdx.x, nl = t & 63, h = t >> 6;
  const int n = cb * GBN + nl;
  if (t < GBN) sgn[t] = 0;
  __syncthreads();
  bool ok = true;
  const bool valid = n < p.N;
  const size_t k = 16 * (size_t)j + 8 * h, ldb = (size_t)p.ldb;
  const size_t off = bz * (size_t)p.sB + (!p.tb ? k * ldb + n : (size_t)n * ldb + k);
  MMAEMU_CHECK(ok, !valid || (!p.tb ? off + 7 * ldb + 1 : off + 8) <= p.b_n);
  const Raw8<FMT> raw = !p.tb ? load_col8<FMT>(p.B, off, ldb, valid && ok) : load_row8<FMT>(p.B, off, valid && ok);
  const size_t blob_i = (bz * ncb + cb) * (size_t)nch + j;
  MMAEMU_CHECK(ok, (blob_i + 1) * BBLOB <= p.dB_n);
  // the B part of a panel starts ABLOB bytes into it
  GPanel &P = *reinterpret_cast<GPanel *>(p.dB + blob_i * BBLOB - ABLOB);
  uint32_t special = 0;
  uint32_t bits = 0;
  if (ok) bits = store_b8<FMT>(P, nl, h, raw, special);
  atomicOr(&sgn[nl], bits);
  const int any = __syncthreads_or((int)special);
  if (ok && t < GBN) P.bS[t] = sgn[t];
  if (ok && t == 0) {
    P.bF[0] = (uint32_t)any;
    P.bF[1] = P.bF[2] = P.bF[3] = 0;
  }
}

// ---- bulk asynchronous copies completed on an mbarrier --------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_init_fence() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// one bulk copy of this GPU's global memory into this block's shared memory
// (no multicast), with an L2 cache policy (createpolicy) for the source lines
__device__ __forceinline__ void bulk_g2s_hint(void *dst, const void *src, uint32_t bytes, uint64_t *bar,
                                              uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for a phase with a bound: false when the bound ran out (the caller
// records a timeout and winds the block down).
#ifndef MMAEMU_WAIT_LIMIT
#define MMAEMU_WAIT_LIMIT (1u << 22)
#endif
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity) {
  for (uint32_t i = 0; i < MMAEMU_WAIT_LIMIT; i++)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Blocks are visited in groups of GROUP_ROWS row blocks, column block by
// column block, so that the blocks resident at one time share A and B
// panels and the decoded operands are reused from L2.
constexpr int GROUP_ROWS = 16;

template <int MODEL, int FMT>
__global__ void __launch_bounds__(GTHREADS, MMAEMU_GMINB) gemm_kernel(const GemmParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GPanel *panels = reinterpret_cast<GPanel *>(smem_raw);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem_raw + 2 * sizeof(GPanel));
  const int M = p.M, N = p.N, K = p.K;
  const size_t bz = blockIdx.z;

  // grouped block order (row block rb, column block cb)
  const int nrb = gridDim.y, ncb = gridDim.x;
  const int lin = blockIdx.y * ncb + blockIdx.x, per_group = GROUP_ROWS * ncb;
  const int g = lin / per_group, rem = lin - g * per_group, first = g * GROUP_ROWS;
  const int rows = min(GROUP_ROWS, nrb - first);
  const int rb = first + rem % rows, cb = rem / rows;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row0 = rb * GBM, col0 = cb * GBN;
  // warp tiles of 32 x 64 outputs, lanes 4 x 8, 8 x 8 outputs each
  const int rl = warp * 32 + (lane >> 3) * GR;
  const int cl = (lane & 7) * GCC;
  const bool out_valid = (row0 + rl < M) && (col0 + cl < N);
  bool ok = true;

  // Per chunk, thread 0 copies the block's decoded A and B blobs into one of
  // two panel buffers with two bulk copies completed on that buffer's
  // mbarrier; the copy of chunk j + 1 overlaps the arithmetic of chunk j.
  const int nchunks = K / 16;
  const size_t blob_a0 = (bz * nrb + rb) * (size_t)nchunks, blob_b0 = (bz * ncb + cb) * (size_t)nchunks;
  MMAEMU_CHECK(ok, (blob_a0 + nchunks) * ABLOB <= p.dA_n && (blob_b0 + nchunks) * BBLOB <= p.dB_n);
  auto issue_chunk = [&](int j) {
    GPanel &P = panels[j & 1];
    mbar_expect_tx(&bars[j & 1], (uint32_t)(ABLOB + BBLOB));
    // L2 policy: a block row's A blobs serve every column block of its
    // group, a column's B blobs only the group's blocks in that column,
    // which run at the same time (measured: DRAM traffic -11%, time equal)
    bulk_g2s_hint(&P, p.dA + (blob_a0 + j) * ABLOB, (uint32_t)ABLOB, &bars[j & 1], policy_evict_last());
    bulk_g2s_hint(reinterpret_cast<unsigned char *>(&P) + ABLOB, p.dB + (blob_b0 + j) * BBLOB, (uint32_t)BBLOB,
                  &bars[j & 1], policy_evict_first());
  };
  auto parity = [](int j) { return (uint32_t)(j >> 1) & 1u; };
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    mbar_init_fence();
  }
  __syncthreads();
  if (tid == 0 && ok) issue_chunk(0);

  // states: exact doubles (see mmaemu_core.cuh), from C
  double X[GR][GCC];
  OutMask<GR * GCC> dneg0;
  bool chk;
  {
    uint32_t cb_[GR][GCC];
    const size_t c_off = bz * (size_t)p.sC + (size_t)(row0 + rl) * p.ldc + col0 + cl;
    const bool have_c = p.C != nullptr && out_valid;
    MMAEMU_CHECK(ok, !have_c || c_off + (GR - 1) * (size_t)p.ldc + GCC <= p.c_n);
    load_bits<GR, GCC>(p.C + (have_c ? c_off : 0), (size_t)p.ldc, have_c && ok, cb_);
    chk = init_states<FMT>(cb_, X, dneg0);
  }

  bool timed_out = false;
  int abandoned_at = -1;
#pragma unroll 1
  for (int j = 0; j < nchunks; j++) {
    if (tid == 0 && ok && j + 1 < nchunks) issue_chunk(j + 1);
    const GPanel &P = panels[j & 1];
    if (!mbar_wait_bounded(&bars[j & 1], parity(j))) timed_out = true;
    const bool panel_special = (P.aF[0] | P.bF[0]) != 0;
    if constexpr (FMT == FMT_BF16) {
      bool unused = false;
      mma_chunk<MODEL, FMT, true, kUnroll<MODEL, FMT>>(P, rl, cl, X, dneg0, panel_special, unused);
    } else {
      if (chk) {
        bool unused = false;
        mma_chunk<MODEL, FMT, true, kUnroll<MODEL, FMT>>(P, rl, cl, X, dneg0, panel_special, unused);
      } else {
        bool to_checked = false;
        mma_chunk<MODEL, FMT, false, kUnroll<MODEL, FMT>>(P, rl, cl, X, dneg0, panel_special, to_checked);
        if (to_checked) {
          scale_states(X);
          chk = true;
        }
      }
    }
    // every thread is done with this buffer before it is refilled (and every
    // thread learns whether a wait ran out anywhere in the block)
    if (__syncthreads_or(timed_out)) {
      abandoned_at = j;
      break;
    }
  }
  if (abandoned_at >= 0) {
    // a bounded wait ran out: record it and leave the outputs unwritten,
    // after waiting (bounded) for the copies this block may still have in
    // flight (chunks up to abandoned_at + 1 were requested)
    if (tid == 0) {
      atomicOr(&g_status, STATUS_TIMEOUT);
      for (int j = abandoned_at; j <= abandoned_at + 1 && j < nchunks; j++)
        (void)mbar_wait_bounded(&bars[j & 1], parity(j));
    }
    return;
  }

  // epilogue: store D, compare with the claimed D, per-16x16-tile xorsum
  uint32_t D[GR][GCC];
  states_to_fp32<MODEL>(X, chk, dneg0, D);
  if (p.D != nullptr && out_valid) {
    const size_t d_off = bz * (size_t)p.sD + (size_t)(row0 + rl) * p.ldd + col0 + cl;
    MMAEMU_CHECK(ok, d_off + (GR - 1) * (size_t)p.ldd + GCC <= p.d_n);
    if (ok) {
      float *Db = p.D + d_off;
#pragma unroll
      for (int i = 0; i < GR; i++) {
        uint4 *dst = reinterpret_cast<uint4 *>(Db + (size_t)i * p.ldd);
        dst[0] = make_uint4(D[i][0], D[i][1], D[i][2], D[i][3]);
        dst[1] = make_uint4(D[i][4], D[i][5], D[i][6], D[i][7]);
      }
    }
  }
  if (p.Dref != nullptr) {
    // bitwise comparison; the smallest mismatching position of the block is
    // found as the smallest in-block offset (row-major order is preserved)
    uint32_t count = 0, firstm = 0xFFFFFFFFu;
    if (out_valid) {
      const size_t r_off = bz * (size_t)p.sR + (size_t)(row0 + rl) * p.ldr + col0 + cl;
      MMAEMU_CHECK(ok, r_off + (GR - 1) * (size_t)p.ldr + GCC <= p.r_n);
      if (ok) {
        const float *Rb = p.Dref + r_off;
#pragma unroll
        for (int i = 0; i < GR; i++) {
          const uint4 *src = reinterpret_cast<const uint4 *>(Rb + (size_t)i * p.ldr);
          const uint4 v0 = src[0], v1 = src[1];
          const uint32_t got[GCC] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int c = GCC - 1; c >= 0; c--)
            if (got[c] != D[i][c]) {
              count++;
              firstm = min(firstm, (uint32_t)((rl + i) * GBN + cl + c));
            }
        }
      }
    }
    count = __reduce_add_sync(0xFFFFFFFFu, count);
    firstm = __reduce_min_sync(0xFFFFFFFFu, firstm);
    if (lane == 0 && count != 0) {
      const unsigned long long idx = (unsigned long long)bz * M * N +
                                     (unsigned long long)(row0 + firstm / GBN) * N + col0 + firstm % GBN;
      atomicAdd(&p.mism[0], (unsigned long long)count);
      atomicMin(&p.mism[1], idx);
    }
  }
  if (p.fp != nullptr) {
    uint32_t x = 0;
#pragma unroll
    for (int i = 0; i < GR; i++)
#pragma unroll
      for (int j = 0; j < GCC; j++) x ^= D[i][j];
    // the 4 lanes sharing a 16x16 tile differ in lane bits 0 and 3
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 1);
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 8);
    if (out_valid && (rl & 15) == 0 && (cl & 15) == 0) {
      const int tr = (row0 + rl) >> 4, tc = (col0 + cl) >> 4;
      const size_t f_off = bz * (size_t)p.sF + (size_t)tr * (N >> 4) + tc;
      MMAEMU_CHECK(ok, f_off < p.fp_n);
      if (ok) p.fp[f_off] = x;
    }
  }
}

// ---------------------------------------------------------------------------
// independent tiles, two per warp: one per half-warp, each lane 4 x 4
// outputs of its tile and the decode of one A row and one B column.  Against
// one tile per warp with 2 x 4 outputs per lane (3 blocks per SM at 80
// registers), this halves the shared loads per product and doubles each
// lane's independent accumulators: 100k Ampere-FP16 tiles 0.143 -> 0.126 ms.
// ---------------------------------------------------------------------------
using TPanel = Panel<16, 16>;
constexpr int T4WARPS = 8;
// resident blocks per SM and k-loop unroll of the tile kernel (measured)
#ifndef MMAEMU_T4MINB
#define MMAEMU_T4MINB 2
#endif
#ifndef MMAEMU_TUNROLL
#define MMAEMU_TUNROLL 4
#endif
template <int MODEL, int FMT>
__global__ void __launch_bounds__(T4WARPS * 32, MMAEMU_T4MINB)
    tiles_kernel(const void *__restrict__ A, const void *__restrict__ B, const float *__restrict__ C,
                   float *__restrict__ Dout, size_t ntiles) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int half = lane >> 4, l16 = lane & 15;
  TPanel &P = reinterpret_cast<TPanel *>(smem_raw)[2 * warp + half];
  const int rl = (l16 >> 2) * 4, cl = (l16 & 3) * 4;
  const size_t stride = (size_t)gridDim.x * T4WARPS * 2;
  size_t w0 = ((size_t)blockIdx.x * T4WARPS + warp) * 2;  // this warp's first tile (warp-uniform)
  if (w0 >= ntiles) return;
  size_t t = w0 + half;
  bool act = t < ntiles;  // the second half may have no tile at the end

  auto load_a = [&](size_t u, int h, bool v) { return load_row8<FMT>(A, u * 256 + l16 * 16 + 8 * h, v); };
  auto load_b = [&](size_t u, int h, bool v) { return load_col8<FMT>(B, u * 256 + (8 * h) * 16 + l16, 16, v); };
  auto load_c = [&](size_t u, bool v, uint32_t(&cv)[4][4]) {
    const bool have = C != nullptr && v;
    load_bits<4, 4>(C + (have ? u * 256 + rl * 16 + cl : 0), 16, have, cv);
  };
  Raw8<FMT> ra0 = load_a(t, 0, act), ra1 = load_a(t, 1, act), rb0 = load_b(t, 0, act), rb1 = load_b(t, 1, act);
  uint32_t cnext[4][4];
  load_c(t, act, cnext);
  double X[4][4];
  OutMask<16> dneg0;
  for (;;) {
    __syncwarp();  // the previous tiles' reads of the panels are done
    uint32_t sp = 0, aw, bw;
    // fast decode first; a tile pair whose operands hold Inf or NaN (an
    // exponent field of all ones in the 16-bit form) is decoded again
    // element by element, over the fast decode's panel entries
    {
      constexpr uint32_t EMAX = (FMT == FMT_BF16 ? 0xFFu : 0x1Fu) * 0x10001u;
      uint32_t fmax = 0;
      aw = fast_store8<FMT, false>(P, l16, 0, ra0, fmax) | fast_store8<FMT, false>(P, l16, 1, ra1, fmax);
      bw = fast_store8<FMT, true>(P, l16, 0, rb0, fmax) | fast_store8<FMT, true>(P, l16, 1, rb1, fmax);
      const bool special_here = (fmax & 0xFFFFu) == (EMAX & 0xFFFFu) || (fmax >> 16) == (EMAX >> 16);
      if (__any_sync(0xFFFFFFFFu, special_here)) {
        __syncwarp();
        aw = store_a8<FMT>(P, l16, 0, ra0, sp) | store_a8<FMT>(P, l16, 1, ra1, sp);
        bw = store_b8<FMT>(P, l16, 0, rb0, sp) | store_b8<FMT>(P, l16, 1, rb1, sp);
      }
    }
    P.aS[l16] = aw;
    P.bS[l16] = bw;
    // either tile's Inf/NaN sends both through the per-output special path,
    // which finds no special output in a tile without them
    const bool panel_special = __any_sync(0xFFFFFFFFu, sp != 0);
    // -0 can only come out of an output whose 16 products are all zero; when
    // every operand of both tiles is nonzero and finite (each sign word has
    // a bit for every k) no output can, and the -0 mask is not kept
    const bool all_nonzero = __all_sync(0xFFFFFFFFu, ((aw | (aw >> 8)) & 0x00FF00FFu) == 0x00FF00FFu &&
                                                         ((bw | (bw >> 8)) & 0x00FF00FFu) == 0x00FF00FFu);
    bool chk = init_states<FMT>(cnext, X, dneg0, !all_nonzero);
    __syncwarp();
    const size_t w_next = w0 + stride, next = t + stride;
    const bool act_next = next < ntiles;
    if (w_next < ntiles) {
      ra0 = load_a(next, 0, act_next);
      ra1 = load_a(next, 1, act_next);
      rb0 = load_b(next, 0, act_next);
      rb1 = load_b(next, 1, act_next);
      load_c(next, act_next, cnext);
    }
    if constexpr (FMT == FMT_BF16) {
      bool unused = false;
      mma_chunk<MODEL, FMT, true, MMAEMU_TUNROLL>(P, rl, cl, X, dneg0, panel_special, unused);
    } else {
      if (chk) {
        bool unused = false;
        mma_chunk<MODEL, FMT, true, MMAEMU_TUNROLL>(P, rl, cl, X, dneg0, panel_special, unused);
      } else {
        bool to_checked = false;
        mma_chunk<MODEL, FMT, false, MMAEMU_TUNROLL>(P, rl, cl, X, dneg0, panel_special, to_checked);
        if (to_checked) {
          scale_states(X);
          chk = true;
        }
      }
    }
    uint32_t D[4][4];
    states_to_fp32<MODEL>(X, chk, dneg0, D);
    if (act) {
#pragma unroll
      for (int i = 0; i < 4; i++)
        *reinterpret_cast<uint4 *>(Dout + t * 256 + (rl + i) * 16 + cl) = make_uint4(D[i][0], D[i][1], D[i][2], D[i][3]);
    }
    w0 = w_next;
    t = next;
    act = act_next;
    if (w0 >= ntiles) break;
  }
}

// ---------------------------------------------------------------------------
// xorsum
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) xorsum_kernel(const uint4 *__restrict__ v, size_t nvec,
                                                     const uint32_t *__restrict__ tail, int ntail,
                                                     uint32_t *__restrict__ out) {
  __shared__ uint32_t part[8];
  uint32_t x = 0;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += (size_t)gridDim.x * blockDim.x) {
    const uint4 q = v[i];
    x ^= q.x ^ q.y ^ q.z ^ q.w;
  }
  if (blockIdx.x == 0 && (int)threadIdx.x < ntail) x ^= tail[threadIdx.x];
  x = __reduce_xor_sync(0xFFFFFFFFu, x);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t y = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); w++) y ^= part[w];
    atomicXor(out, y);
  }
}

// A kernel whose only job is a bounded wait that nothing completes: thread 0
// arms an mbarrier for bytes that never arrive and waits on it with a bound of
// `spins` tries, then records a timeout exactly as the GEMM does.  Used to
// check that a wait that runs out leaves the device usable and is reported.
__global__ void __launch_bounds__(32) wait_timeout_kernel(uint32_t spins, uint32_t *out) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_init_fence();
    mbar_expect_tx(&bar, 16);  // arrives, but 16 transaction bytes stay pending
    uint32_t i = 0;
    bool done = false;
    for (; i < spins && !done; i++) done = mbar_try_wait(&bar, 0);
    if (!done) atomicOr(&g_status, STATUS_TIMEOUT);
    *out = done ? 1u : 0u;
  }
}

// ---------------------------------------------------------------------------
// B200's own tensor-core MMA on the same tile batches (a probe target, not
// part of the emulation): one warp per 16x16x16 tile, two mma.sync
// m16n8k16 (FP16/BF16) or m16n8k32 with k >= 16 zero (E4M3) per tile, fp32
// accumulate.  Fragment layouts are those of the PTX mma.sync description.
// ---------------------------------------------------------------------------
template <int FMT>
__global__ void __launch_bounds__(256) native_tiles_kernel(const void *__restrict__ A, const void *__restrict__ B,
                                                         const float *__restrict__ C, float *__restrict__ D,
                                                         size_t ntiles) {
  const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
  for (size_t t = (size_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < ntiles;
       t += (size_t)gridDim.x * (blockDim.x >> 5)) {
    uint32_t a[4], b[2][2];
    if constexpr (FMT == FMT_E4M3) {
      const uint8_t *At = static_cast<const uint8_t *>(A) + t * 256;
      const uint8_t *Bt = static_cast<const uint8_t *>(B) + t * 256;
      auto row4 = [&](int m) { return *reinterpret_cast<const uint32_t *>(At + m * 16 + 4 * tig); };
      a[0] = row4(gid);
      a[1] = row4(gid + 8);
      a[2] = a[3] = 0u;  // k = 16 .. 31
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int n = 8 * h + gid;
        uint32_t v = 0;
#pragma unroll
        for (int i = 0; i < 4; i++) v |= (uint32_t)Bt[(4 * tig + i) * 16 + n] << (8 * i);
        b[h][0] = v;
        b[h][1] = 0u;
      }
    } else {
      const uint16_t *At = static_cast<const uint16_t *>(A) + t * 256;
      const uint16_t *Bt = static_cast<const uint16_t *>(B) + t * 256;
      auto pair = [&](const uint16_t *p, int stride) { return (uint32_t)p[0] | ((uint32_t)p[stride] << 16); };
      a[0] = pair(At + gid * 16 + 2 * tig, 1);
      a[1] = pair(At + (gid + 8) * 16 + 2 * tig, 1);
      a[2] = pair(At + gid * 16 + 2 * tig + 8, 1);
      a[3] = pair(At + (gid + 8) * 16 + 2 * tig + 8, 1);
#pragma unroll
      for (int h = 0; h < 2; h++) {
        const int n = 8 * h + gid;
        b[h][0] = pair(Bt + (2 * tig) * 16 + n, 16);
        b[h][1] = pair(Bt + (2 * tig + 8) * 16 + n, 16);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; h++) {
      const int col = 8 * h + 2 * tig;
      float c[4] = {0.f, 0.f, 0.f, 0.f}, d[4];
      if (C != nullptr) {
        const float *Ct = C + t * 256;
        c[0] = Ct[gid * 16 + col];
        c[1] = Ct[gid * 16 + col + 1];
        c[2] = Ct[(gid + 8) * 16 + col];
        c[3] = Ct[(gid + 8) * 16 + col + 1];
      }
      if constexpr (FMT == FMT_FP16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[h][0]), "r"(b[h][1]), "f"(c[0]), "f"(c[1]),
              "f"(c[2]), "f"(c[3]));
      } else if constexpr (FMT == FMT_BF16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[h][0]), "r"(b[h][1]), "f"(c[0]), "f"(c[1]),
              "f"(c[2]), "f"(c[3]));
      } else {
        asm volatile(
            "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%10,%11,%12,%13};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[h][0]), "r"(b[h][1]), "f"(c[0]), "f"(c[1]),
              "f"(c[2]), "f"(c[3]));
      }
      float *Dt = D + t * 256;
      Dt[gid * 16 + col] = d[0];
      Dt[gid * 16 + col + 1] = d[1];
      Dt[(gid + 8) * 16 + col] = d[2];
      Dt[(gid + 8) * 16 + col + 1] = d[3];
    }
  }
}

}  // namespace mmaemu

// ===========================================================================
// host side: validation, dispatch, C ABI
// ===========================================================================
namespace {

thread_local cudaStream_t t_stream = nullptr;

constexpr int kMaxDevices = 64;
std::atomic<int> g_dev_ok[kMaxDevices];  // 0 unknown, 1 sm_100, 2 other
std::atomic<int> g_sm_count[kMaxDevices];

int check_device(int *sms = nullptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  int st = g_dev_ok[dev].load(std::memory_order_relaxed);
  if (st == 0) {
    int major = 0, minor = 0, count = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return MMAEMU_ECUDA;
    st = (major == 10 && minor == 0) ? 1 : 2;
    g_sm_count[dev].store(count, std::memory_order_relaxed);
    g_dev_ok[dev].store(st, std::memory_order_relaxed);
  }
  if (sms) *sms = g_sm_count[dev].load(std::memory_order_relaxed);
  return st == 1 ? MMAEMU_OK : MMAEMU_EUNSUPPORTED;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Library-private stream-ordered memory pool per device for the GEMM's
// decoded-operand workspace.  By default its release threshold is 0: memory
// freed by a GEMM goes back to the device at the next synchronisation, so
// nothing stays allocated between calls.  mmaemu_set_workspace_cache(1)
// raises the threshold so that repeated GEMMs reuse the memory instead.
std::mutex g_pool_mutex;
cudaMemPool_t g_pool[kMaxDevices] = {};
bool g_cache[kMaxDevices] = {};

cudaMemPool_t workspace_pool() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  if (!g_pool[dev]) {
    cudaMemPoolProps props = {};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool = nullptr;
    if (cudaMemPoolCreate(&pool, &props) != cudaSuccess) return nullptr;
    uint64_t threshold = g_cache[dev] ? UINT64_MAX : 0;
    if (cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &threshold) != cudaSuccess) {
      cudaMemPoolDestroy(pool);
      return nullptr;
    }
    g_pool[dev] = pool;
  }
  return g_pool[dev];
}

bool valid_pair(int model, int fmt) {
  if (model != MMAEMU_AMPERE && model != MMAEMU_HOPPER && model != MMAEMU_B200) return false;
  if (fmt != MMAEMU_FP16 && fmt != MMAEMU_BF16 && fmt != MMAEMU_E4M3) return false;
  return !((model == MMAEMU_AMPERE || model == MMAEMU_B200) && fmt == MMAEMU_E4M3);
}

#define MMAEMU_DISPATCH(model, fmt, CALL)                                               \
  do {                                                                                  \
    if (model == MMAEMU_AMPERE && fmt == MMAEMU_FP16) return CALL(0, 0);                \
    if (model == MMAEMU_AMPERE && fmt == MMAEMU_BF16) return CALL(0, 1);                \
    if (model == MMAEMU_HOPPER && fmt == MMAEMU_FP16) return CALL(1, 0);                \
    if (model == MMAEMU_HOPPER && fmt == MMAEMU_BF16) return CALL(1, 1);                \
    if (model == MMAEMU_HOPPER && fmt == MMAEMU_E4M3) return CALL(1, 2);                \
    if (model == MMAEMU_B200 && fmt == MMAEMU_FP16) return CALL(2, 0);                  \
    if (model == MMAEMU_B200 && fmt == MMAEMU_BF16) return CALL(2, 1);                  \
    return MMAEMU_EINVAL;                                                               \
  } while (0)

// Workspace sizes of one GEMM (all batch entries): decoded A and B blobs.
struct GemmSizes {
  int nrb, ncb, nch;
  size_t a_bytes, b_bytes;
};
GemmSizes gemm_sizes(int M, int N, int K, int batch) {
  GemmSizes z;
  z.nrb = (M + mmaemu::GBM - 1) / mmaemu::GBM;
  z.ncb = (N + mmaemu::GBN - 1) / mmaemu::GBN;
  z.nch = K / 16;
  z.a_bytes = (size_t)batch * z.nrb * z.nch * mmaemu::ABLOB;
  z.b_bytes = (size_t)batch * z.ncb * z.nch * mmaemu::BBLOB;
  return z;
}
size_t up256(size_t x) { return (x + 255) & ~(size_t)255; }

// Extents (one past the largest element index) of every buffer a GEMM
// touches, for the checking build's bounds checks.
void set_extents(mmaemu::GemmParams &p, int batch) {
  const size_t bm1 = (size_t)(batch - 1);
  const size_t a_rows = p.ta ? (size_t)p.K : (size_t)p.M, a_row = p.ta ? (size_t)p.M : (size_t)p.K;
  const size_t b_rows = p.tb ? (size_t)p.N : (size_t)p.K, b_row = p.tb ? (size_t)p.K : (size_t)p.N;
  p.a_n = bm1 * (size_t)p.sA + (a_rows - 1) * (size_t)p.lda + a_row;
  p.b_n = bm1 * (size_t)p.sB + (b_rows - 1) * (size_t)p.ldb + b_row;
  p.c_n = p.C ? bm1 * (size_t)p.sC + (size_t)(p.M - 1) * p.ldc + p.N : 0;
  p.d_n = p.D ? bm1 * (size_t)p.sD + (size_t)(p.M - 1) * p.ldd + p.N : 0;
  p.r_n = p.Dref ? bm1 * (size_t)p.sR + (size_t)(p.M - 1) * p.ldr + p.N : 0;
  p.fp_n = p.fp ? bm1 * (size_t)p.sF + (size_t)(p.M / 16) * (p.N / 16) : 0;
}

// Decode pass for B (p.dB set) on `stream`.
template <int MODEL, int FMT>
int launch_decode_b(const mmaemu::GemmParams &p, int batch, cudaStream_t stream) {
  const GemmSizes z = gemm_sizes(p.M, p.N, p.K, batch);
  mmaemu::decode_b_kernel<FMT><<<dim3(z.ncb, z.nch, batch), 128, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
}

constexpr size_t kGemmSmem = 2 * sizeof(mmaemu::GPanel) + 16;  // two panel buffers and their mbarriers

// Decode pass for A and the MMA kernel (B already decoded) on `stream`.
template <int MODEL, int FMT>
int launch_decode_a_gemm(const mmaemu::GemmParams &p, int batch, cudaStream_t stream) {
  const GemmSizes z = gemm_sizes(p.M, p.N, p.K, batch);
  auto kern = mmaemu::gemm_kernel<MODEL, FMT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kGemmSmem) != cudaSuccess)
    return MMAEMU_ECUDA;
  mmaemu::decode_a_kernel<FMT><<<dim3(z.nrb, z.nch, batch), 128, 0, stream>>>(p);
  kern<<<dim3(z.ncb, z.nrb, batch), mmaemu::GTHREADS, kGemmSmem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
}

template <int MODEL, int FMT>
int launch_gemm(const mmaemu::GemmParams &p_in, int batch) {
  mmaemu::GemmParams p = p_in;
  const GemmSizes z = gemm_sizes(p.M, p.N, p.K, batch);
  // workspace: decoded blobs, stream-ordered, released after the GEMM
  unsigned char *ws = nullptr;
  cudaMemPool_t pool = workspace_pool();
  const size_t total = up256(z.a_bytes) + up256(z.b_bytes);
  if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws), total, pool, t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  p.dA = ws;
  p.dB = ws + up256(z.a_bytes);
  p.dA_n = z.a_bytes;
  p.dB_n = z.b_bytes;
  p.batch = batch;
  set_extents(p, batch);
  int rc = launch_decode_b<MODEL, FMT>(p, batch, t_stream);
  if (rc == MMAEMU_OK) rc = launch_decode_a_gemm<MODEL, FMT>(p, batch, t_stream);
  if (cudaFreeAsync(ws, t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  return rc;
}

mmaemu::GemmParams row_major_params(int M, int N, int K, const void *A, const void *B, const float *C, float *D,
                                    uint32_t *fp) {
  mmaemu::GemmParams p{};
  p.A = A; p.B = B; p.C = C; p.D = D; p.fp = fp;
  p.M = M; p.N = N; p.K = K;
  p.lda = K; p.ldb = N; p.ldc = N; p.ldd = N; p.ldr = N;
  return p;
}

// Library-owned streams per device for mmaemu_gemm_host: copies in, copies
// out, and a second compute stream.
cudaStream_t g_copy_in[kMaxDevices] = {}, g_copy_out[kMaxDevices] = {}, g_compute2[kMaxDevices] = {};

int host_streams(cudaStream_t &in, cudaStream_t &out, cudaStream_t &compute2) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MMAEMU_ECUDA;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  for (cudaStream_t *st : {&g_copy_in[dev], &g_copy_out[dev], &g_compute2[dev]})
    if (!*st && cudaStreamCreateWithFlags(st, cudaStreamNonBlocking) != cudaSuccess) return MMAEMU_ECUDA;
  in = g_copy_in[dev];
  out = g_copy_out[dev];
  compute2 = g_compute2[dev];
  return MMAEMU_OK;
}

// mmaemu_gemm from host memory: B is copied and decoded once; A and C go in
// row slabs (host_slabs.h) on a copy stream while earlier slabs compute,
// alternately on the caller's stream and a second compute stream (so that
// one slab's last partial wave of blocks overlaps the next slab), and each
// slab's D (and fingerprints) returns on another copy stream as soon as
// that slab is done.
template <int MODEL, int FMT>
int launch_gemm_host(int M, int N, int K, const void *A_h, const void *B_h, const float *C_h, float *D_h,
                     uint32_t *fp_h, int sms) {
  constexpr size_t ES = FMT == mmaemu::FMT_E4M3 ? 1 : 2;
  cudaStream_t s_in, s_out, c2;
  int rc = host_streams(s_in, s_out, c2);
  if (rc != MMAEMU_OK) return rc;
  const cudaStream_t cs[2] = {t_stream, c2};
  int r0s[mmaemu_host::kHostMaxSlabs + 1];
  const int nslab = mmaemu_host::host_slabs(M, N, mmaemu::GBM, mmaemu::GBN, (long long)sms * MMAEMU_GMINB, r0s);
  int max_rows = 0;
  for (int sl = 0; sl < nslab; sl++)
    if (r0s[sl + 1] - r0s[sl] > max_rows) max_rows = r0s[sl + 1] - r0s[sl];
  const GemmSizes zs = gemm_sizes(max_rows, N, K, 1), zb = gemm_sizes(M, N, K, 1);
  const size_t a_bytes = (size_t)M * K * ES, b_bytes = (size_t)K * N * ES, cd_bytes = (size_t)M * N * 4;
  const size_t fp_bytes = fp_h ? (size_t)(M / 16) * (N / 16) * 4 : 0;
  // device buffers, each 256-byte aligned inside one pool allocation; two
  // A-blob workspaces, one per compute stream
  const size_t o_b = up256(a_bytes), o_c = o_b + up256(b_bytes), o_d = o_c + (C_h ? up256(cd_bytes) : 0);
  const size_t o_fp = o_d + (D_h ? up256(cd_bytes) : 0), o_wa = o_fp + up256(fp_bytes);
  const size_t o_wb = o_wa + 2 * up256(zs.a_bytes);
  const size_t total = o_wb + up256(zb.b_bytes);
  unsigned char *buf = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void **>(&buf), total, pool, t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  unsigned char *dA = buf, *dB = buf + o_b;
  float *dC = C_h ? reinterpret_cast<float *>(buf + o_c) : nullptr;
  float *dD = D_h ? reinterpret_cast<float *>(buf + o_d) : nullptr;  // fingerprint-only: no D at all
  uint32_t *dfp = fp_h ? reinterpret_cast<uint32_t *>(buf + o_fp) : nullptr;

  const int nev = 2 + 2 * nslab + 3;
  cudaEvent_t ev[2 + 2 * mmaemu_host::kHostMaxSlabs + 3];
  int made = 0;
  for (; made < nev; made++)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) {
      rc = MMAEMU_ECUDA;
      break;
    }
  cudaEvent_t &e_alloc = ev[0], &e_b = ev[1], &e_out = ev[nev - 1], &e_bdec = ev[nev - 2], &e_c2 = ev[nev - 3];
  auto e_in = [&](int sl) -> cudaEvent_t & { return ev[2 + sl]; };
  auto e_done = [&](int sl) -> cudaEvent_t & { return ev[2 + nslab + sl]; };
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess) rc = MMAEMU_ECUDA;
    return rc == MMAEMU_OK;
  };
  if (rc == MMAEMU_OK && ok(cudaEventRecord(e_alloc, t_stream)) && ok(cudaStreamWaitEvent(s_in, e_alloc, 0)) &&
      ok(cudaStreamWaitEvent(s_out, e_alloc, 0)) && ok(cudaStreamWaitEvent(c2, e_alloc, 0)) &&
      ok(cudaMemcpyAsync(dB, B_h, b_bytes, cudaMemcpyHostToDevice, s_in)))
    ok(cudaEventRecord(e_b, s_in));
  for (int sl = 0; sl < nslab && rc == MMAEMU_OK; sl++) {
    const size_t r0 = r0s[sl], rows = r0s[sl + 1] - r0s[sl];
    if (!ok(cudaMemcpyAsync(dA + r0 * K * ES, static_cast<const unsigned char *>(A_h) + r0 * K * ES, rows * K * ES,
                            cudaMemcpyHostToDevice, s_in)))
      break;
    if (C_h && !ok(cudaMemcpyAsync(dC + r0 * N, C_h + r0 * N, rows * N * 4, cudaMemcpyHostToDevice, s_in))) break;
    ok(cudaEventRecord(e_in(sl), s_in));
  }
  mmaemu::GemmParams p = row_major_params(M, N, K, dA, dB, dC, dD, dfp);
  p.dB = buf + o_wb;
  p.dB_n = zb.b_bytes;
  p.batch = 1;
  set_extents(p, 1);
  if (rc == MMAEMU_OK && ok(cudaStreamWaitEvent(t_stream, e_b, 0))) rc = launch_decode_b<MODEL, FMT>(p, 1, t_stream);
  if (rc == MMAEMU_OK && ok(cudaEventRecord(e_bdec, t_stream))) ok(cudaStreamWaitEvent(c2, e_bdec, 0));
  for (int sl = 0; sl < nslab && rc == MMAEMU_OK; sl++) {
    const size_t r0 = r0s[sl];
    const int rows = r0s[sl + 1] - r0s[sl];
    const cudaStream_t st = cs[sl & 1];
    mmaemu::GemmParams q = p;
    q.M = rows;
    q.A = dA + r0 * K * ES;
    q.C = dC ? dC + r0 * N : nullptr;
    q.D = dD ? dD + r0 * N : nullptr;
    q.fp = dfp ? dfp + (r0 / 16) * (N / 16) : nullptr;
    q.dA = buf + o_wa + (sl & 1) * up256(zs.a_bytes);
    q.dA_n = zs.a_bytes;
    set_extents(q, 1);
    if (!ok(cudaStreamWaitEvent(st, e_in(sl), 0))) break;
    rc = launch_decode_a_gemm<MODEL, FMT>(q, 1, st);
    if (rc != MMAEMU_OK || !ok(cudaEventRecord(e_done(sl), st)) || !ok(cudaStreamWaitEvent(s_out, e_done(sl), 0)))
      break;
    if (D_h && !ok(cudaMemcpyAsync(D_h + r0 * N, dD + r0 * N, (size_t)rows * N * 4, cudaMemcpyDeviceToHost, s_out)))
      break;
    if (fp_h && !ok(cudaMemcpyAsync(fp_h + (r0 / 16) * (N / 16), dfp + (r0 / 16) * (N / 16),
                                    (size_t)(rows / 16) * (N / 16) * 4, cudaMemcpyDeviceToHost, s_out)))
      break;
  }
  // the buffers go back to the pool once every copy has finished
  if (made == nev) {
    ok(cudaEventRecord(e_out, s_out));
    ok(cudaEventRecord(e_in(nslab - 1), s_in));
    ok(cudaEventRecord(e_c2, c2));
    ok(cudaStreamWaitEvent(t_stream, e_out, 0));
    ok(cudaStreamWaitEvent(t_stream, e_in(nslab - 1), 0));
    ok(cudaStreamWaitEvent(t_stream, e_c2, 0));
  } else {
    cudaStreamSynchronize(s_in);
    cudaStreamSynchronize(s_out);
    cudaStreamSynchronize(c2);
  }
  if (cudaFreeAsync(buf, t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (cudaStreamSynchronize(t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  for (int i = 0; i < made; i++) cudaEventDestroy(ev[i]);
  return rc;
}

// Shape, layout and alignment rules shared by the GEMM entry points.
int validate_gemm(const mmaemu::GemmParams &p, long long batch) {
  if (p.M <= 0 || p.N <= 0 || p.K <= 0 || (p.M & 15) || (p.N & 15) || (p.K & 15)) return MMAEMU_EINVAL;
  if (batch < 1 || batch > 65535) return MMAEMU_EINVAL;
  if ((long long)p.M / mmaemu::GBM >= 65535) return MMAEMU_EINVAL;  // grid y (row blocks)
  if ((long long)p.K / 8 > 65535) return MMAEMU_EINVAL;             // decode-pass grid y (chunks), with margin
  if (!p.A || !p.B) return MMAEMU_EINVAL;
  if (!p.D && !p.fp && !p.Dref) return MMAEMU_EINVAL;  // nothing to produce
  if (p.Dref && !p.mism) return MMAEMU_EINVAL;
  if ((p.ta != 0 && p.ta != 1) || (p.tb != 0 && p.tb != 1)) return MMAEMU_EINVAL;
  // leading dimensions cover a row of the stored matrix; vector-loaded rows
  // (A not transposed, B transposed, C, D, Dref) start on 16-byte boundaries
  const long long a_row = p.ta ? p.M : p.K, b_row = p.tb ? p.K : p.N;
  if (p.lda < a_row || p.ldb < b_row) return MMAEMU_EINVAL;
  constexpr long long vec = 8;  // elements per operand vector load (16 B of fp16/bf16, 8 B of e4m3)
  if (!aligned16(p.A) || !aligned16(p.B)) return MMAEMU_EINVAL;
  if (!p.ta && (p.lda % vec || p.sA % vec)) return MMAEMU_EINVAL;
  if (p.tb && (p.ldb % vec || p.sB % vec)) return MMAEMU_EINVAL;
  if (p.sA < 0 || p.sB < 0 || p.sC < 0 || p.sD < 0 || p.sR < 0 || p.sF < 0) return MMAEMU_EINVAL;
  struct F32 { const void *ptr; long long ld, stride; };
  const F32 mats[3] = {{p.C, p.ldc, p.sC}, {p.D, p.ldd, p.sD}, {p.Dref, p.ldr, p.sR}};
  for (const F32 &m : mats) {
    if (!m.ptr) continue;
    if (!aligned16(m.ptr) || m.ld < p.N || m.ld % 4 || m.stride % 4) return MMAEMU_EINVAL;
  }
  if (p.fp && ((uintptr_t)p.fp & 3u)) return MMAEMU_EINVAL;
  if (batch > 1 && p.fp && p.sF < (long long)(p.M / 16) * (p.N / 16)) return MMAEMU_EINVAL;
  return MMAEMU_OK;
}

int run_gemm(int model, int fmt, mmaemu::GemmParams &p, long long batch) {
  if (!valid_pair(model, fmt)) return MMAEMU_EINVAL;
  int rc = validate_gemm(p, batch);
  if (rc != MMAEMU_OK) return rc;
  rc = check_device();
  if (rc != MMAEMU_OK) return rc;
  if (p.Dref) {
    // count 0, smallest index all-ones ("none")
    if (cudaMemsetAsync(p.mism, 0, sizeof(unsigned long long), t_stream) != cudaSuccess ||
        cudaMemsetAsync(p.mism + 1, 0xFF, sizeof(unsigned long long), t_stream) != cudaSuccess)
      return MMAEMU_ECUDA;
  }
#define CALL_GEMM(M_, F_) launch_gemm<M_, F_>(p, (int)batch)
  MMAEMU_DISPATCH(model, fmt, CALL_GEMM);
#undef CALL_GEMM
}

template <int MODEL, int FMT>
int launch_tiles(const void *A, const void *B, const float *C, float *D, size_t ntiles, int sms) {
  const size_t smem = 2 * mmaemu::T4WARPS * sizeof(mmaemu::TPanel);
  auto kern = mmaemu::tiles_kernel<MODEL, FMT>;
  constexpr int TPB = 2 * mmaemu::T4WARPS;  // tiles per block and pass
  constexpr int THREADS = mmaemu::T4WARPS * 32;
  // the shared-memory attribute and the resident blocks per SM, once per
  // device (a batch of tiles is short, so the per-call host time shows)
  static std::atomic<int> s_per_sm[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MMAEMU_ECUDA;
  int per_sm = s_per_sm[dev].load(std::memory_order_acquire);
  if (per_sm == 0) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MMAEMU_ECUDA;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, THREADS, smem) != cudaSuccess)
      return MMAEMU_ECUDA;
    if (per_sm < 1) per_sm = 1;
    s_per_sm[dev].store(per_sm, std::memory_order_release);
  }
  const size_t want = (ntiles + TPB - 1) / TPB;
  const size_t cap = (size_t)sms * per_sm;
  const unsigned blocks = (unsigned)(want < cap ? want : cap);
  kern<<<blocks, THREADS, smem, t_stream>>>(A, B, C, D, ntiles);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
}

// mmaemu_tiles from host memory: the tiles go in chunks.  A chunk's A, B
// and C are copied in on a library copy stream, its tiles run on the
// selected stream once they have arrived, and its D goes back on a second
// copy stream, so that the copies in both directions overlap each other and
// the arithmetic.
constexpr int kTileHostMaxChunks = 8;
constexpr size_t kTileHostMinChunk = 4096;  // tiles per chunk, at least (a chunk of fewer is one launch)
template <int MODEL, int FMT>
int launch_tiles_host(const void *A_h, const void *B_h, const float *C_h, float *D_h, size_t ntiles, int sms) {
  constexpr size_t ES = FMT == mmaemu::FMT_E4M3 ? 1 : 2;
  cudaStream_t s_in, s_out, c2;
  int rc = host_streams(s_in, s_out, c2);
  if (rc != MMAEMU_OK) return rc;
  size_t nch = ntiles / kTileHostMinChunk;
  nch = nch < 1 ? 1 : nch > (size_t)kTileHostMaxChunks ? (size_t)kTileHostMaxChunks : nch;
  const size_t per = (ntiles + nch - 1) / nch;
  nch = (ntiles + per - 1) / per;
  const size_t ab_bytes = ntiles * 256 * ES, cd_bytes = ntiles * 256 * 4;
  const size_t o_b = up256(ab_bytes), o_c = o_b + up256(ab_bytes), o_d = o_c + (C_h ? up256(cd_bytes) : 0);
  const size_t total = o_d + up256(cd_bytes);
  unsigned char *buf = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void **>(&buf), total, pool, t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  unsigned char *dA = buf, *dB = buf + o_b;
  float *dC = C_h ? reinterpret_cast<float *>(buf + o_c) : nullptr;
  float *dD = reinterpret_cast<float *>(buf + o_d);

  const int nev = 2 + 2 * (int)nch;
  cudaEvent_t ev[2 + 2 * kTileHostMaxChunks];
  int made = 0;
  for (; made < nev; made++)
    if (cudaEventCreateWithFlags(&ev[made], cudaEventDisableTiming) != cudaSuccess) {
      rc = MMAEMU_ECUDA;
      break;
    }
  cudaEvent_t &e_alloc = ev[0], &e_out = ev[nev - 1];
  auto e_in = [&](size_t ch) -> cudaEvent_t & { return ev[1 + ch]; };
  auto e_done = [&](size_t ch) -> cudaEvent_t & { return ev[1 + nch + ch]; };
  auto ok = [&](cudaError_t e) {
    if (e != cudaSuccess) rc = MMAEMU_ECUDA;
    return rc == MMAEMU_OK;
  };
  if (rc == MMAEMU_OK && ok(cudaEventRecord(e_alloc, t_stream)) && ok(cudaStreamWaitEvent(s_in, e_alloc, 0)))
    ok(cudaStreamWaitEvent(s_out, e_alloc, 0));
  for (size_t ch = 0; ch < nch && rc == MMAEMU_OK; ch++) {
    const size_t t0 = ch * per, n = t0 + per < ntiles ? per : ntiles - t0;
    const size_t ab0 = t0 * 256 * ES, abn = n * 256 * ES;
    if (!ok(cudaMemcpyAsync(dA + ab0, static_cast<const unsigned char *>(A_h) + ab0, abn, cudaMemcpyHostToDevice,
                            s_in)) ||
        !ok(cudaMemcpyAsync(dB + ab0, static_cast<const unsigned char *>(B_h) + ab0, abn, cudaMemcpyHostToDevice,
                            s_in)))
      break;
    if (C_h && !ok(cudaMemcpyAsync(dC + t0 * 256, C_h + t0 * 256, n * 256 * 4, cudaMemcpyHostToDevice, s_in)))
      break;
    ok(cudaEventRecord(e_in(ch), s_in));
  }
  for (size_t ch = 0; ch < nch && rc == MMAEMU_OK; ch++) {
    const size_t t0 = ch * per, n = t0 + per < ntiles ? per : ntiles - t0;
    if (!ok(cudaStreamWaitEvent(t_stream, e_in(ch), 0))) break;
    rc = launch_tiles<MODEL, FMT>(dA + t0 * 256 * ES, dB + t0 * 256 * ES, dC ? dC + t0 * 256 : nullptr,
                                  dD + t0 * 256, n, sms);
    if (rc != MMAEMU_OK || !ok(cudaEventRecord(e_done(ch), t_stream)) ||
        !ok(cudaStreamWaitEvent(s_out, e_done(ch), 0)))
      break;
    if (!ok(cudaMemcpyAsync(D_h + t0 * 256, dD + t0 * 256, n * 256 * 4, cudaMemcpyDeviceToHost, s_out))) break;
  }
  // the buffers go back to the pool once every copy has finished
  if (made == nev) {
    ok(cudaEventRecord(e_out, s_out));
    ok(cudaStreamWaitEvent(t_stream, e_out, 0));
    ok(cudaEventRecord(e_in(nch - 1), s_in));
    ok(cudaStreamWaitEvent(t_stream, e_in(nch - 1), 0));
  } else {
    cudaStreamSynchronize(s_in);
    cudaStreamSynchronize(s_out);
  }
  if (cudaFreeAsync(buf, t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (cudaStreamSynchronize(t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  for (int i = 0; i < made; i++) cudaEventDestroy(ev[i]);
  return rc;
}

}  // namespace

extern "C" {

int mmaemu_set_stream(void *cuda_stream) {
  t_stream = static_cast<cudaStream_t>(cuda_stream);
  return MMAEMU_OK;
}

int mmaemu_tiles(int model, int fmt, const void *A, const void *B, const float *C, float *D, size_t ntiles) {
  if (!valid_pair(model, fmt)) return MMAEMU_EINVAL;
  if (ntiles == 0) return MMAEMU_OK;
  if (!A || !B || !D) return MMAEMU_EINVAL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || (C && !aligned16(C))) return MMAEMU_EINVAL;
  if (ntiles > ((size_t)1 << 40)) return MMAEMU_EINVAL;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc != MMAEMU_OK) return rc;
#define CALL_TILES(M_, F_) launch_tiles<M_, F_>(A, B, C, D, ntiles, sms)
  MMAEMU_DISPATCH(model, fmt, CALL_TILES);
#undef CALL_TILES
}

int mmaemu_tiles_host(int model, int fmt, const void *A, const void *B, const float *C, float *D, size_t ntiles) {
  if (!valid_pair(model, fmt)) return MMAEMU_EINVAL;
  if (ntiles == 0) return MMAEMU_OK;
  if (!A || !B || !D) return MMAEMU_EINVAL;
  if (ntiles > ((size_t)1 << 40)) return MMAEMU_EINVAL;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc != MMAEMU_OK) return rc;
#define CALL_TILES_HOST(M_, F_) launch_tiles_host<M_, F_>(A, B, C, D, ntiles, sms)
  MMAEMU_DISPATCH(model, fmt, CALL_TILES_HOST);
#undef CALL_TILES_HOST
}

int mmaemu_native_tiles(int fmt, const void *A, const void *B, const float *C, float *D, size_t ntiles) {
  if (fmt != MMAEMU_FP16 && fmt != MMAEMU_BF16 && fmt != MMAEMU_E4M3) return MMAEMU_EINVAL;
  if (ntiles == 0) return MMAEMU_OK;
  if (!A || !B || !D) return MMAEMU_EINVAL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || (C && !aligned16(C))) return MMAEMU_EINVAL;
  if (ntiles > ((size_t)1 << 40)) return MMAEMU_EINVAL;
  int sms = 0;
  const int rc = check_device(&sms);
  if (rc != MMAEMU_OK) return rc;
  const size_t want = (ntiles + 7) / 8, cap = (size_t)sms * 8;
  const unsigned blocks = (unsigned)(want < cap ? want : cap);
  if (fmt == MMAEMU_FP16)
    mmaemu::native_tiles_kernel<mmaemu::FMT_FP16><<<blocks, 256, 0, t_stream>>>(A, B, C, D, ntiles);
  else if (fmt == MMAEMU_BF16)
    mmaemu::native_tiles_kernel<mmaemu::FMT_BF16><<<blocks, 256, 0, t_stream>>>(A, B, C, D, ntiles);
  else
    mmaemu::native_tiles_kernel<mmaemu::FMT_E4M3><<<blocks, 256, 0, t_stream>>>(A, B, C, D, ntiles);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
}

int mmaemu_gemm(int model, int fmt, int M, int N, int K, const void *A, const void *B, const float *C, float *D,
                uint32_t *fingerprint_out) {
  mmaemu::GemmParams p = row_major_params(M, N, K, A, B, C, D, fingerprint_out);
  if (!D && !fingerprint_out) return MMAEMU_EINVAL;
  return run_gemm(model, fmt, p, 1);
}

int mmaemu_gemm_verify(int model, int fmt, int M, int N, int K, const void *A, const void *B, const float *C,
                       const float *D_claimed, uint32_t *fingerprint_out, unsigned long long *mismatch_out) {
  if (!D_claimed || !mismatch_out) return MMAEMU_EINVAL;
  mmaemu::GemmParams p = row_major_params(M, N, K, A, B, C, nullptr, fingerprint_out);
  p.Dref = D_claimed;
  p.mism = mismatch_out;
  return run_gemm(model, fmt, p, 1);
}

int mmaemu_gemm_strided_batched(int model, int fmt, int trans_a, int trans_b, int M, int N, int K, int batch,
                                const void *A, long long lda, long long stride_a, const void *B, long long ldb,
                                long long stride_b, const float *C, long long ldc, long long stride_c, float *D,
                                long long ldd, long long stride_d, uint32_t *fingerprint_out,
                                long long stride_fp) {
  mmaemu::GemmParams p{};
  p.A = A; p.B = B; p.C = C; p.D = D; p.fp = fingerprint_out;
  p.M = M; p.N = N; p.K = K; p.ta = trans_a; p.tb = trans_b;
  p.lda = lda; p.ldb = ldb; p.ldc = C ? ldc : N; p.ldd = D ? ldd : N; p.ldr = N;
  p.sA = stride_a; p.sB = stride_b; p.sC = C ? stride_c : 0; p.sD = D ? stride_d : 0;
  p.sF = fingerprint_out ? stride_fp : 0;
  if (!D && !fingerprint_out) return MMAEMU_EINVAL;
  return run_gemm(model, fmt, p, batch);
}

int mmaemu_gemm_host(int model, int fmt, int M, int N, int K, const void *A, const void *B, const float *C,
                     float *D, uint32_t *fingerprint_out) {
  if (!valid_pair(model, fmt)) return MMAEMU_EINVAL;
  if (!D && !fingerprint_out) return MMAEMU_EINVAL;
  mmaemu::GemmParams p = row_major_params(M, N, K, A, B, C, D, fingerprint_out);
  int rc = validate_gemm(p, 1);
  if (rc != MMAEMU_OK) return rc;
  int sms = 0;
  rc = check_device(&sms);
  if (rc != MMAEMU_OK) return rc;
#define CALL_HOST(M_, F_) launch_gemm_host<M_, F_>(M, N, K, A, B, C, D, fingerprint_out, sms)
  MMAEMU_DISPATCH(model, fmt, CALL_HOST);
#undef CALL_HOST
}

int mmaemu_xorsum(const void *D, size_t n, uint32_t *out_host) {
  if (!out_host || (n && !D) || (n && !aligned16(D))) return MMAEMU_EINVAL;
  int sms = 0;
  int rc = check_device(&sms);
  if (rc != MMAEMU_OK) return rc;
  *out_host = 0;
  if (n == 0) return MMAEMU_OK;
  uint32_t *scratch = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void **>(&scratch), sizeof(uint32_t), t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  rc = MMAEMU_OK;
  const size_t nvec = n / 4;
  const int ntail = (int)(n % 4);
  const size_t want = (nvec + 255) / 256;
  const size_t cap = (size_t)sms * 8;
  const unsigned blocks = (unsigned)(want == 0 ? 1 : (want < cap ? want : cap));
  uint32_t result = 0;
  if (cudaMemsetAsync(scratch, 0, sizeof(uint32_t), t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (rc == MMAEMU_OK) {
    mmaemu::xorsum_kernel<<<blocks, 256, 0, t_stream>>>(static_cast<const uint4 *>(D), nvec,
                                                        static_cast<const uint32_t *>(D) + 4 * nvec, ntail, scratch);
    if (cudaGetLastError() != cudaSuccess) rc = MMAEMU_ECUDA;
  }
  if (rc == MMAEMU_OK &&
      cudaMemcpyAsync(&result, scratch, sizeof(uint32_t), cudaMemcpyDeviceToHost, t_stream) != cudaSuccess)
    rc = MMAEMU_ECUDA;
  if (cudaFreeAsync(scratch, t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (cudaStreamSynchronize(t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (rc == MMAEMU_OK) *out_host = result;
  return rc;
}

int mmaemu_set_workspace_cache(int enable) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  g_cache[dev] = enable != 0;
  if (g_pool[dev]) {
    uint64_t threshold = enable ? UINT64_MAX : 0;
    if (cudaMemPoolSetAttribute(g_pool[dev], cudaMemPoolAttrReleaseThreshold, &threshold) != cudaSuccess)
      return MMAEMU_ECUDA;
    if (!enable && cudaMemPoolTrimTo(g_pool[dev], 0) != cudaSuccess) return MMAEMU_ECUDA;
  }
  return MMAEMU_OK;
}

int mmaemu_workspace_reserved(size_t *bytes) {
  if (!bytes) return MMAEMU_EINVAL;
  *bytes = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  if (!g_pool[dev]) return MMAEMU_OK;
  uint64_t v = 0;
  if (cudaMemPoolGetAttribute(g_pool[dev], cudaMemPoolAttrReservedMemCurrent, &v) != cudaSuccess) return MMAEMU_ECUDA;
  *bytes = (size_t)v;
  return MMAEMU_OK;
}

int mmaemu_trim_workspace(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  if (g_pool[dev] && cudaMemPoolTrimTo(g_pool[dev], 0) != cudaSuccess) return MMAEMU_ECUDA;
  return MMAEMU_OK;
}

int mmaemu_device_status(int clear, uint32_t *bits_out) {
  int rc = check_device();
  if (rc != MMAEMU_OK) return rc;
  if (cudaStreamSynchronize(t_stream) != cudaSuccess) return MMAEMU_ECUDA;
  uint32_t bits = 0;
  if (cudaMemcpyFromSymbol(&bits, mmaemu::g_status, sizeof bits) != cudaSuccess) return MMAEMU_ECUDA;
  if (clear && bits) {
    const uint32_t zero = 0;
    if (cudaMemcpyToSymbol(mmaemu::g_status, &zero, sizeof zero) != cudaSuccess) return MMAEMU_ECUDA;
  }
  if (bits_out) *bits_out = bits;
  if (bits & mmaemu::STATUS_BOUNDS) return MMAEMU_EBOUNDS;
  if (bits & mmaemu::STATUS_TIMEOUT) return MMAEMU_ETIMEOUT;
  return MMAEMU_OK;
}

int mmaemu_selftest_wait_timeout(unsigned spins, int *completed_out) {
  int rc = check_device();
  if (rc != MMAEMU_OK) return rc;
  uint32_t *flag = nullptr;
  if (cudaMallocAsync(reinterpret_cast<void **>(&flag), sizeof(uint32_t), t_stream) != cudaSuccess) return MMAEMU_ECUDA;
  mmaemu::wait_timeout_kernel<<<1, 32, 0, t_stream>>>(spins, flag);
  rc = cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
  uint32_t done = 0;
  if (rc == MMAEMU_OK &&
      cudaMemcpyAsync(&done, flag, sizeof done, cudaMemcpyDeviceToHost, t_stream) != cudaSuccess)
    rc = MMAEMU_ECUDA;
  if (cudaFreeAsync(flag, t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (cudaStreamSynchronize(t_stream) != cudaSuccess) rc = MMAEMU_ECUDA;
  if (rc == MMAEMU_OK && completed_out) *completed_out = (int)done;
  return rc;
}

int mmaemu_bounds_checking(void) {
#ifdef MMAEMU_BOUNDS_CHECK
  return 1;
#else
  return 0;
#endif
}

const char *mmaemu_strerror(int code) {
  switch (code) {
    case MMAEMU_OK: return "ok";
    case MMAEMU_EINVAL: return "invalid argument (enum, model/format pair, pointer, alignment or size)";
    case MMAEMU_ECUDA: return "CUDA runtime error";
    case MMAEMU_ETIMEOUT: return "a bounded device wait gave up";
    case MMAEMU_EUNSUPPORTED: return "unsupported: the current CUDA device is not an sm_100 (B200-class) GPU, "
                                     "or the probe cannot be built for this format";
    case MMAEMU_ECALLBACK: return "the MMA callback of a probe reported an error";
    case MMAEMU_EBOUNDS: return "a bounds check of the checking build failed (an index left its buffer)";
    default: return "unknown error code";
  }
}

}  // extern "C"

// ===========================================================================
// xorsum that allocates nothing
//
// For callers that cannot allocate device memory at the moment they need a
// fingerprint -- for instance a verification step that runs after the device
// has run out of memory, or inside a process whose device memory is entirely
// reserved by another allocator -- mmaemu_xorsum_noalloc does the same
// reduction with a fixed scratch array that lives in the library image
// instead of a per-call allocation.  Each block of xorsum_partials_kernel
// folds a fixed span of the input into one word of the array;
// xorsum_finish_kernel folds those words into the result slot, which is then
// copied to the host.
// ===========================================================================
namespace mmaemu {

constexpr unsigned kNoAllocThreads = 256;
constexpr size_t kNoAllocVecPerThread = 8;  // uint4 loads per thread
constexpr size_t kNoAllocVecPerBlock = kNoAllocThreads * kNoAllocVecPerThread;
constexpr size_t kNoAllocWordsPerBlock = 4 * kNoAllocVecPerBlock;  // 8192 words
constexpr size_t kNoAllocPartials = MMAEMU_XORSUM_NOALLOC_MAX_WORDS / kNoAllocWordsPerBlock;  // 16384
static_assert(kNoAllocPartials * kNoAllocWordsPerBlock == MMAEMU_XORSUM_NOALLOC_MAX_WORDS, "exact fit");

// One word per block, then the result slot.  Every word a call reads has been
// written earlier in the same call, so nothing needs clearing between calls.
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocPartials + 1];

__global__ void __launch_bounds__(kNoAllocThreads) xorsum_partials_kernel(const uint4 *__restrict__ v, size_t nvec,
                                                                          const uint32_t *__restrict__ tail,
                                                                          int ntail, uint32_t *__restrict__ partials) {
  __shared__ uint32_t part[kNoAllocThreads / 32];
  uint32_t x = 0;
  const size_t base = (size_t)blockIdx.x * kNoAllocVecPerBlock;
#pragma unroll
  for (size_t i = 0; i < kNoAllocVecPerThread; i++) {
    const size_t idx = base + i * kNoAllocThreads + threadIdx.x;
    if (idx < nvec) {
      const uint4 q = v[idx];
      x ^= q.x ^ q.y ^ q.z ^ q.w;
    }
  }
  if (blockIdx.x == 0 && (int)threadIdx.x < ntail) x ^= tail[threadIdx.x];
  x = __reduce_xor_sync(0xFFFFFFFFu, x);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t y = 0;
    for (unsigned w = 0; w < kNoAllocThreads / 32; w++) y ^= part[w];
    partials[blockIdx.x] = y;
  }
}

__global__ void __launch_bounds__(kNoAllocThreads) xorsum_finish_kernel(const uint32_t *__restrict__ partials,
                                                                        unsigned nparts, uint32_t *__restrict__ result) {
  __shared__ uint32_t part[kNoAllocThreads / 32];
  uint32_t x = 0;
  for (unsigned i = threadIdx.x; i < nparts; i += kNoAllocThreads) x ^= partials[i];
  x = __reduce_xor_sync(0xFFFFFFFFu, x);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = x;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t y = 0;
    for (unsigned w = 0; w < kNoAllocThreads / 32; w++) y ^= part[w];
    *result = y;
  }
}

}  // namespace mmaemu

namespace {

// Device address of the scratch array, looked up once per device (with that
// device current).  In host code the array's name only stands for the device
// symbol; it is not an address a kernel may be given.  The same first call
// also loads both kernels onto the device (CUDA loads modules lazily, and
// loading takes device memory), so that later calls need none.
std::atomic<uint32_t *> g_noalloc_scratch_ptr[kMaxDevices];

int noalloc_scratch(uint32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  uint32_t *p = g_noalloc_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    cudaFuncAttributes fa;
    if (cudaFuncGetAttributes(&fa, mmaemu::xorsum_partials_kernel) != cudaSuccess ||
        cudaFuncGetAttributes(&fa, mmaemu::xorsum_finish_kernel) != cudaSuccess)
      return MMAEMU_ECUDA;
    if (cudaGetSymbolAddress(reinterpret_cast<void **>(&p), mmaemu::g_noalloc_scratch) != cudaSuccess ||
        p == nullptr)
      return MMAEMU_ECUDA;
    g_noalloc_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return MMAEMU_OK;
}

}  // namespace

extern "C" int mmaemu_xorsum_noalloc(const void *D, size_t n, uint32_t *out_host) {
  if (!out_host || (n && !D) || (n && !aligned16(D))) return MMAEMU_EINVAL;
  if (n > MMAEMU_XORSUM_NOALLOC_MAX_WORDS) return MMAEMU_EINVAL;
  int rc = check_device();
  if (rc != MMAEMU_OK) return rc;
  uint32_t *scratch = nullptr;
  rc = noalloc_scratch(&scratch);
  if (rc != MMAEMU_OK) return rc;
  *out_host = 0;
  if (n == 0) return MMAEMU_OK;
  const size_t nvec = n / 4;
  const int ntail = (int)(n % 4);
  size_t nblocks = (nvec + mmaemu::kNoAllocVecPerBlock - 1) / mmaemu::kNoAllocVecPerBlock;
  if (nblocks == 0) nblocks = 1;  // only the tail words
  uint32_t *result_slot = scratch + mmaemu::kNoAllocPartials;
  mmaemu::xorsum_partials_kernel<<<(unsigned)nblocks, mmaemu::kNoAllocThreads, 0, t_stream>>>(
      static_cast<const uint4 *>(D), nvec, static_cast<const uint32_t *>(D) + 4 * nvec, ntail, scratch);
  if (cudaGetLastError() != cudaSuccess) return MMAEMU_ECUDA;
  mmaemu::xorsum_finish_kernel<<<1, mmaemu::kNoAllocThreads, 0, t_stream>>>(scratch, (unsigned)nblocks, result_slot);
  if (cudaGetLastError() != cudaSuccess) return MMAEMU_ECUDA;
  uint32_t result = 0;
  if (cudaMemcpyAsync(&result, result_slot, sizeof(uint32_t), cudaMemcpyDeviceToHost, t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  if (cudaStreamSynchronize(t_stream) != cudaSuccess) return MMAEMU_ECUDA;
  *out_host = result;
  return MMAEMU_OK;
}
