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
// Exact-double formulation of one output element and one accumulation group
// (see group_step in mmaemu.cu):
//  * every operand carries an exponent code q = (512 - e) * 16 in 16 bits, so
//    that a product's code qa + qb is ncode(ea + eb) = (1024 - e) * 16; the
//    carried term's code is read straight from the top 16 bits of its double;
//    e_max over the group is the minimum code, found two outputs at a time
//    with packed 16-bit add-and-min;
//  * the group is summed in a double acc whose value is (1.5 * 2^52 + L) u on
//    the grid u = 2^(e_max - F): every double in [2^52 u, 2^53 u) is a
//    multiple of u, so a round-toward-zero fused multiply-add of a term adds
//    exactly floor(term / u) -- the truncated magnitude for a positive term,
//    minus one more than it for a negative one (B is stored times 1 + 2^-40,
//    so no product sits on the grid).  L starts as the number of negative
//    terms, which makes every term's contribution its sign-magnitude
//    truncation;
//  * the exact group value is acc minus the base 1.5 * 2^52 u, one
//    subtraction; truncating it to 24 significant bits is a mask of the low
//    29 mantissa bits: the Ampere hand-over and the fp32 write-back (the
//    unchecked Ampere form carries the exact value instead and truncates
//    once at the end, which gives the same result: the next group's grid is
//    never finer than the carried value's 24-bit unit).
#pragma once
#include <stdint.h>

namespace mmaemu {

enum : int { MODEL_AMPERE = 0, MODEL_HOPPER = 1, MODEL_B200 = 2 };
enum : int { FMT_FP16 = 0, FMT_BF16 = 1, FMT_E4M3 = 2 };

// ---------------------------------------------------------------------------
// exponent codes
// ---------------------------------------------------------------------------
// ncode(e) = (1024 - e) * 16; an operand carries (512 - e) * 16, so the code
// of a product is the sum of its operands' codes.  Every code of a nonzero
// finite term lies in [12320, 20416] (BF16 product exponents -252..254).
__host__ __device__ constexpr int op_code(int e) { return (512 - e) * 16; }
__host__ __device__ constexpr int ncode(int e) { return (1024 - e) * 16; }
// Zero, infinite and NaN operands: large enough that a product with one never
// sets the group maximum (QZ + the smallest operand code > the floor code),
// small enough that two of them still fit a signed 16-bit lane.
constexpr int QZ = 14336, QINF = QZ + 1, QNAN = QZ + 2;
// The -133 threshold on the group's max exponent (BF16 paragraph), and the
// exponent an fp32 subnormal carried value takes part in the maximum with.
constexpr int FLOOR_CODE = ncode(-133);  // 18512
constexpr int SUBN_CODE = ncode(-126);   // 18400
// A checked state (see group_step) holds its fp32 value times 2^S_WB, so that
// values from 2^128 up overflow to infinity in the scaling multiply; the
// checked Ampere hand-over is carried times 2^S_HO.
constexpr int S_WB = 896, S_HO = 512;

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
  static constexpr int STAGE1 = 8;  // {C, P[1..8]}, then {S1, P[9..16]}
  static constexpr uint32_t NAN_BITS = 0x7FC00000u;
};
template <> struct ModelT<MODEL_HOPPER> {
  static constexpr int F = 24;  // 25-bit internal significand
  static constexpr int STAGE1 = 16;  // one 17-term stage
  static constexpr uint32_t NAN_BITS = 0x7FC00000u;
};
// B200's own FP16/BF16 tensor-core MMA, as measured with the target tests:
// one 17-term stage like Hopper, 26-bit internal significand, NaN written as
// 0x7FFFFFFF.
template <> struct ModelT<MODEL_B200> {
  static constexpr int F = 25;
  static constexpr int STAGE1 = 16;
  static constexpr uint32_t NAN_BITS = 0x7FFFFFFFu;
};

// The -133 floor can only bind for BF16: fp16/e4m3 terms and fp32 C values
// are all multiples of 2^-149 and every group with a nonzero term has e_max >=
// -126, so the floor changes nothing for them; a group with no nonzero term
// sums to zero on any grid.
template <int FMT> constexpr bool kNeedsFloor = (FMT == FMT_BF16);

// ---------------------------------------------------------------------------
// bit helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t vadd2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("add.s16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t vmin2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.s16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t vminu2(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("min.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__device__ __forceinline__ uint32_t vmaxu2_16(uint32_t a, uint32_t b) {
  uint32_t r;
  asm("max.u16x2 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(b));
  return r;
}
__host__ __device__ constexpr uint32_t pair16(int lo, int hi) {
  return ((uint32_t)lo & 0xFFFFu) | ((uint32_t)hi << 16);
}
__device__ __forceinline__ int32_t lo16(uint32_t p) { return (int32_t)(int16_t)(p & 0xFFFFu); }
__device__ __forceinline__ int32_t hi16(uint32_t p) { return (int32_t)p >> 16; }

// ---------------------------------------------------------------------------
// operand decode (one element)
// ---------------------------------------------------------------------------
// e = max(field, 1) - bias, m = frac + (field != 0) 2^p: subnormals keep the
// minimum exponent and no implicit bit (they enter the products unchanged).
// The value is exact as a double; zero, Inf and NaN operands become a zero of
// their sign (the special-value path reads their codes).  pos / neg: the
// operand is nonzero and finite with that sign.
struct DecElem {
  double v;
  uint32_t q;  // op_code(e), or QZ / QINF / QNAN
  uint32_t pos, neg, special;
};

template <int FMT>
__device__ __forceinline__ DecElem decode_elem(uint32_t x) {
  using T = FmtT<FMT>;
  constexpr uint32_t EMASK = (1u << T::EBITS) - 1u, FMASK = (1u << T::P) - 1u;
  const uint32_t field = (x >> T::P) & EMASK, frac = x & FMASK;
  const uint32_t s = (x >> (T::NBITS - 1)) & 1u;
  const uint32_t m = frac | (field ? (1u << T::P) : 0u);
  const int e = (int)(field ? field : 1u) - T::BIAS;
  const bool special = T::IEEE ? field == EMASK : (x & 0x7Fu) == 0x7Fu;
  const bool nan = T::IEEE ? (special && frac != 0) : special;
  DecElem d;
  d.special = special;
  const bool nz = m != 0 && !special;
  d.q = special ? (nan ? QNAN : QINF) : m ? (uint32_t)op_code(e) : (uint32_t)QZ;
  // 2^(e - p) is a normal double for every format
  const double mag = nz ? (double)m * __hiloint2double((1023 + e - T::P) << 20, 0) : 0.0;
  d.v = s ? -mag : mag;
  d.pos = nz && !s;
  d.neg = nz && s;
  return d;
}

}  // namespace mmaemu
