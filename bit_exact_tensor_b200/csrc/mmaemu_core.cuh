// Device-side arithmetic of the emulated Tensor Core MMA (sm_100a CUDA cores).
//
// Model: "Hawkeye: Reproducing GPU-Level Non-Determinism (MLSys 2026)" reading
// notes -- Obs. 1 (exact products inside the dot-product path), Obs. 2 (Ampere
// two-stage {C,P[1..8]} then {S1,P[9..16]}; Hopper one 17-term stage), Obs. 3
// (24/25-bit internal significand, truncating alignment, delayed normalisation,
// subnormal products not renormalised, toward-zero write-back), the recovered
// Ampere FP16 pipeline (Algorithms 12-14, Figure 1: "m_raw << 3", GroupSum
// with "m_i >> delta_e" truncation) with its Hopper and BF16 paragraphs (BF16
// extended range, max-exponent threshold -133), and Algorithm 10 (final cast
// to FP32 overflows to infinity).
//
// Integer formulation used by the kernels (one output element, one group):
//   every term is (n, X): n = -e (negated exponent; zero operands get ZSENT so
//   they never win the max), and a magnitude A at F fraction bits below 2^e.
//   e_max = max e  <=>  nmin = min n.
//   A product's magnitude is A = (ma << (F - 2p)) * mb, computed by one IMAD
//   from operands pre-scaled at decode time.
//   Truncating alignment is a logical right shift of the magnitude by
//   delta = n_k - nmin (clamped at 32 by the PTX shift, giving 0).
//   The sign is applied as ones' complement, T ^ sgn (sgn = 0 or all ones),
//   and the group sum adds the number of negative terms back:
//       sum_k (-1)^s_k T_k  =  sum_k (T_k ^ sgn_k)  +  #{k : s_k = 1}.
//   Because ~x shifted arithmetically equals ~(x shifted logically), a term
//   already held in ones' complement form (the stage-1 result, or C) is
//   aligned with an arithmetic shift.
#pragma once
#include <stdint.h>

namespace mmaemu {

enum : int { MODEL_AMPERE = 0, MODEL_HOPPER = 1 };
enum : int { FMT_FP16 = 0, FMT_BF16 = 1, FMT_E4M3 = 2 };

// Negated exponent given to zero operands: larger than any real n sum, so a
// zero term never sets the group's max exponent; sums of two stay far below
// 2^15, which keeps packed 16-bit arithmetic exact.
constexpr int ZSENT = 0x2000;
// Markers for Inf / NaN operands (only read by the special-value path).
constexpr int NINF = 0x3000;
constexpr int NNAN = 0x3001;
// Floor on the group max exponent, as a bound on nmin: e_max >= -133.
constexpr int NFLOOR = 133;

template <int FMT> struct FmtT;
template <> struct FmtT<FMT_FP16> {
  static constexpr int P = 10, BIAS = 15, EBITS = 5, NBITS = 16;
  static constexpr bool IEEE = true;
};
template <> struct FmtT<FMT_BF16> {
  static constexpr int P = 7, BIAS = 127, EBITS = 8, NBITS = 16;
  static constexpr bool IEEE = true;
};
template <> struct FmtT<FMT_E4M3> {
  static constexpr int P = 3, BIAS = 7, EBITS = 4, NBITS = 8;
  static constexpr bool IEEE = false;
};

template <int MODEL> struct ModelT;
template <> struct ModelT<MODEL_AMPERE> {
  static constexpr int F = 23;  // 24-bit internal significand
  static constexpr int STAGES = 2;
};
template <> struct ModelT<MODEL_HOPPER> {
  static constexpr int F = 24;  // 25-bit internal significand
  static constexpr int STAGES = 1;
};

// The floor can only bind for BF16: fp16/e4m3 terms and fp32 C values are all
// multiples of 2^-149, so coarsening a grid to 2^-156 (or 2^-157) drops
// nothing and the result is the same with or without it.
template <int FMT> constexpr bool kNeedsFloor = (FMT == FMT_BF16);

// ---------------------------------------------------------------------------
// small integer helpers with defined behaviour for any shift amount
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t shr_u32(uint32_t x, uint32_t n) {
  uint32_t r;
  asm("shr.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));  // n >= 32 gives 0
  return r;
}
__device__ __forceinline__ int32_t shr_s32(int32_t x, uint32_t n) {
  int32_t r;
  asm("shr.s32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));  // n >= 32 gives sign fill
  return r;
}
__device__ __forceinline__ uint32_t shl_u32(uint32_t x, uint32_t n) {
  uint32_t r;
  asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(n));  // n >= 32 gives 0
  return r;
}

// ---------------------------------------------------------------------------
// operand decode
// ---------------------------------------------------------------------------
struct Dec {
  uint32_t m;  // significand with implicit bit (none for subnormals)
  int32_t n;   // -e, ZSENT for zero, NINF / NNAN for specials
  uint32_t s;  // 0 or 0xFFFFFFFF
  uint32_t special;  // 1 for Inf or NaN
};

// e = max(field, 1) - bias, m = frac + (field != 0) 2^p: subnormals keep the
// minimum exponent and no implicit bit (they enter the products unchanged).
template <int FMT>
__device__ __forceinline__ Dec decode(uint32_t x) {
  using T = FmtT<FMT>;
  constexpr uint32_t EMASK = (1u << T::EBITS) - 1u, FMASK = (1u << T::P) - 1u;
  const uint32_t field = (x >> T::P) & EMASK;
  const uint32_t frac = x & FMASK;
  Dec d;
  d.s = ((x >> (T::NBITS - 1)) & 1u) ? 0xFFFFFFFFu : 0u;
  d.m = frac | (field ? (1u << T::P) : 0u);
  const int e = (int)(field ? field : 1u) - T::BIAS;
  d.n = d.m ? -e : ZSENT;
  if (T::IEEE) {
    d.special = field == EMASK;
    if (d.special) {
      d.n = frac ? NNAN : NINF;
      d.m = 0;
    }
  } else {
    d.special = (x & 0x7Fu) == 0x7Fu;
    if (d.special) {
      d.n = NNAN;
      d.m = 0;
    }
  }
  return d;
}

// fp32 accumulator input as a term: n = -e (ZSENT for zero), X = magnitude
// at F fraction bits in ones' complement form for a negative value.
template <int F>
__device__ __forceinline__ void c_term(uint32_t c, int32_t &n, int32_t &X) {
  const uint32_t field = (c >> 23) & 0xFFu;
  const uint32_t m = (c & 0x7FFFFFu) | (field ? 0x800000u : 0u);
  n = m ? (127 - (int)(field ? field : 1u)) : ZSENT;
  X = (int32_t)((m << (F - 23)) ^ (uint32_t)((int32_t)c >> 31));
}

// ---------------------------------------------------------------------------
// toward-zero cast of (S, nmin) to fp32 -- common (normal) case only.
// Returns the bits and sets rare = 1 when S == 0 or the exponent is out of
// the normal range; those are finished by cast_rare.
// ---------------------------------------------------------------------------
template <int F>
__device__ __forceinline__ uint32_t cast_normal(int32_t S, int32_t nmin, uint32_t &rare) {
  const uint32_t mag = (uint32_t)(S < 0 ? -S : S);
  const uint32_t z = __clz(mag);
  const int E = -nmin - F + 31 - (int)z;  // exponent of the leading bit
  const uint32_t sig = shl_u32(mag, z) >> 8;  // 24 bits, bit 23 set (mag != 0)
  rare = (S == 0) | ((uint32_t)(E + 126) > 253u);
  return ((uint32_t)S & 0x80000000u) + ((uint32_t)(E + 126) << 23) + sig;
}

// Out-of-range exponents: overflow -> +-Inf; below 2^-126 -> truncated onto
// the subnormal grid 2^-149 (a result that truncates away is a zero with the
// sign of S).  S == 0 is handled by the caller's zero-sign rule.
template <int F>
__device__ __forceinline__ uint32_t cast_out_of_range(int32_t S, int32_t nmin) {
  const uint32_t sign = (uint32_t)S & 0x80000000u;
  const uint32_t mag = (uint32_t)(S < 0 ? -S : S);
  const int E = -nmin - F + 31 - (int)__clz(mag);
  if (E > 127) return sign | 0x7F800000u;
  const int sh = -nmin - F + 149;  // value = mag * 2^(e_max - F); grid 2^-149
  const uint32_t q = sh >= 0 ? shl_u32(mag, (uint32_t)sh) : shr_u32(mag, (uint32_t)(-sh));
  return sign | q;
}

}  // namespace mmaemu
