// libmmaemu: bit-exact emulation of Ampere / Hopper Tensor Core MMA arithmetic
// on B200 CUDA cores (sm_100a), behind the C ABI declared in include/mmaemu.h.
//
// Kernels
//   gemm_kernel   -- D = C + A.B over 16-wide K chunks (ascending, each chunk's
//                    fp32 result feeding the next), fused per-tile xorsum.
//   tiles_kernel  -- independent 16x16x16 tiles, one warp per tile.
//   xorsum_kernel -- XOR of a buffer of 32-bit words.
// The arithmetic itself is in mmaemu_core.cuh; see the model citations there.
// Tensor cores are deliberately not used: B200's own MMA arithmetic is not the
// arithmetic being emulated.  Everything is exact: both kernels keep the
// exponent-max pass, the carried terms and the write-back in integer (or
// exact float) steps, and do each product's truncating alignment and signed
// accumulation in one fused FP64 multiply-add with round-toward-zero, on an
// integer held in a double's mantissa (see group_products).
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "mmaemu.h"
#include "mmaemu_core.cuh"

namespace mmaemu {

// ---------------------------------------------------------------------------
// decoded operand panels in shared memory, [k][row] for A and [k][col] for B
// ---------------------------------------------------------------------------
// Operand panels of one 16-deep K chunk: the operands as exact doubles for
// the fused truncate-and-add step of group_products below, the packed
// negated exponents of the max pass, and the chunk's sign bits per row of A
// and per column of B.
template <int BM, int BN>
struct __align__(16) Panel {
  double aV[16][BM];     // A value; zero, Inf and NaN as +-2^-500
  uint32_t aN2[16][BM];  // (-ea, -ea) packed (ZSENT / NINF / NNAN markers)
  uint16_t aS[BM];       // bit k: sign of A[m][k]
  double bV[16][BN];     // B value times (1 + 2^-40); zero, Inf and NaN as +-2^-500
  int16_t bN2[16][BN];   // -eb (markers as for A)
  uint16_t bS[BN];       // bit k: sign of B[k][n]
};

// Slot of column n (0..BN-1) in a row of bV in the GEMM's panels (the tile
// kernel's panels keep natural order).  A GEMM thread reads its 8
// consecutive columns as 4 pairs, and the 4 threads of a quarter warp read
// 4 column groups 64 bytes apart, which would put groups 0 and 2 (and 1 and
// 3) on the same banks; storing pair q of group g at pair q ^ (g & 2) gives
// each a bank range of its own.
__host__ __device__ constexpr int bv_slot(int n) {
  return (n & ~7) | ((((n >> 1) & 3) ^ ((n >> 3) & 2)) << 1) | (n & 1);
}

// Per-element reads used off the main path (zero-sign rule, Inf/NaN).
template <int BM, int BN>
__device__ __forceinline__ int32_t n_a(const Panel<BM, BN> &P, int k, int m) { return lo16(P.aN2[k][m]); }
template <int BM, int BN>
__device__ __forceinline__ int32_t n_b(const Panel<BM, BN> &P, int k, int n) { return P.bN2[k][n]; }
template <int BM, int BN>
__device__ __forceinline__ bool neg_a(const Panel<BM, BN> &P, int k, int m) { return (P.aS[m] >> k) & 1u; }
template <int BM, int BN>
__device__ __forceinline__ bool neg_b(const Panel<BM, BN> &P, int k, int n) { return (P.bS[n] >> k) & 1u; }

// Unroll of the k loops per model and format (measured on the GEMM: 4 for
// Ampere FP16, 1 for the B200 model, whose 64-bit carry keeps more registers
// live, else 2).
#ifndef MMAEMU_KUNROLL
template <int MODEL, int FMT>
constexpr int kUnroll = MODEL == MODEL_AMPERE && FMT == FMT_FP16 ? 4 : MODEL == MODEL_B200 ? 1 : 2;
#else
template <int MODEL, int FMT>
constexpr int kUnroll = MMAEMU_KUNROLL;
#endif

template <int R, typename T>
__device__ __forceinline__ void lds_vec(const T *p, T (&v)[R]) {
  static_assert(sizeof(T) == 4, "32-bit elements");
  if constexpr (R == 8) {
    const uint4 a = reinterpret_cast<const uint4 *>(p)[0];
    const uint4 b = reinterpret_cast<const uint4 *>(p)[1];
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

// Pass 1 of a group over k in [K0, K0 + KN): nmin (= -e_max) of every output,
// starting from the carried terms' negated exponents Np (packed pairs).
template <int FMT, int K0, int KN, int R, int CC, int UNR, class PanelT>
__device__ __forceinline__ void group_max(const PanelT &P, int rl, int cl, const uint32_t (&Np)[R][CC / 2],
                                          int32_t (&nmin)[R][CC]) {
  uint32_t nm2[R][CC / 2];
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) nm2[r][p] = Np[r][p];
#pragma unroll UNR
  for (int k = K0; k < K0 + KN; k++) {
    uint32_t an2[R], bn2[CC / 2];
    lds_vec<R>(&P.aN2[k][rl], an2);
    lds_vec<CC / 2>(reinterpret_cast<const uint32_t *>(&P.bN2[k][cl]), bn2);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int p = 0; p < CC / 2; p++) nm2[r][p] = vmin2(nm2[r][p], vadd2(an2[r], bn2[p]));
  }
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) {
      uint32_t v = nm2[r][p];
      if constexpr (kNeedsFloor<FMT>) v = vmin2(v, (uint32_t)NFLOOR | ((uint32_t)NFLOOR << 16));
      nmin[r][2 * p] = lo16(v);
      nmin[r][2 * p + 1] = hi16(v);
    }
}

__device__ __forceinline__ double fma_rz(double a, double b, double c) {
  double d;
  asm("fma.rz.f64 %0, %1, %2, %3;" : "=d"(d) : "d"(a), "d"(b), "d"(c));
  return d;
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

// Pass 2 of a group: add every product's aligned (truncated) magnitude, with
// its sign, to S (which holds the carried term's contribution), with one
// fused multiply-add per product.
// Per output, acc holds (2^52 + 2^51 + L) u on the group's grid u =
// 2^(e_max - F), with L = S mod 2^32 in its low mantissa bits; every double
// in [2^52 u, 2^53 u) is a multiple of u, so fma.rz(a, b', acc) -- one
// rounding, toward zero, of a positive result -- adds floor(a b' / u):
//  * a positive product adds T = floor(|ab| / u), its truncated magnitude,
//    because b' = b (1 + 2^-40) moves it by less than the distance to the
//    next multiple of u (|ab| 2^-40 < 2^(ea+eb+2-40), while |ab| and the grid
//    points are multiples of 2^(ea+eb-2p) and u >= 2^(ea+eb-F), F < 38);
//  * a negative product adds -ceil(|ab'| / u) = -T - 1 for the same reason
//    (|ab'| is never a multiple of u), and a zero stand-in adds 0 or -1 the
//    same way (T = 0);
// so the exact sum is L plus the number of negative products, which is the
// popcount of the XOR of the row's and the column's sign bits over the
// group.  L stays far inside the 51-bit field, and the low 32 bits of acc
// give the sum modulo 2^32 (the sums here fit in int32).
// The exponent field is 1075 - F - nmin, formed modulo 2^32: the marker
// values of nmin (ZSENT, NINF and sums with them) are multiples of 2^12
// plus a real n, so they wrap to a valid grid; such a group has no nonzero
// term (or is overwritten as Inf/NaN), and every product of a zero stand-in
// (below 2^-371) truncates to zero on it.
template <int F, int K0, int KN, int R, int CC, int UNR, int BM, int BN>
__device__ __forceinline__ void group_products(const Panel<BM, BN> &P, int rl, int cl,
                                               const int32_t (&nmin)[R][CC], int32_t (&S)[R][CC]) {
  double acc[R][CC];
  constexpr uint32_t HI0 = ((uint32_t)(1075 - F) << 20) | 0x80000u;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++)
      acc[r][c] = __hiloint2double((int)(HI0 - ((uint32_t)nmin[r][c] << 20)), S[r][c]);
  // 8-column groups (GEMM) are stored with their pairs swizzled (bv_slot);
  // 4-column groups (tile kernel) in natural order, which is conflict-free
  static_assert(CC == 8 || CC == 4, "column groups of 8 or 4");
  const int sw = (cl >> 3) & 2;
#pragma unroll UNR
  for (int k = K0; k < K0 + KN; k++) {
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
      for (int r = 0; r < R; r++) acc[r][c] = fma_rz(a[r], b[c], acc[r][c]);
  }
  constexpr uint32_t GM = ((1u << KN) - 1u) << K0;
  uint32_t sa[R], sb[CC];
#pragma unroll
  for (int r = 0; r < R; r++) sa[r] = P.aS[rl + r];
#pragma unroll
  for (int c = 0; c < CC; c++) sb[c] = P.bS[cl + c];
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++)
      S[r][c] = (int32_t)((uint32_t)__double2loint(acc[r][c]) + __popc((sa[r] ^ sb[c]) & GM));
}

// One accumulation group with a carried term in the state form (Np, X):
// returns S (exact signed sum of the aligned terms) and nmin (= -e_max).
template <int FMT, int F, int K0, int KN, int R, int CC, int UNR, class PanelT>
__device__ __forceinline__ void group_sum(const PanelT &P, int rl, int cl, const uint32_t (&Np)[R][CC / 2],
                                          const int32_t (&X)[R][CC], int32_t (&nmin)[R][CC], int32_t (&S)[R][CC]) {
  group_max<FMT, K0, KN, R, CC, UNR>(P, rl, cl, Np, nmin);
  constexpr int CSH = 30 - F;  // the state's significand sits at bits 30..7
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const int32_t nc = (c & 1) ? hi16(Np[r][c / 2]) : lo16(Np[r][c / 2]);
      // ones' complement -> exact: ~(M >> d) + 1 = -(M >> d)
      S[r][c] = shr_s32(X[r][c], (uint32_t)(nc - nmin[r][c] + CSH)) + (int32_t)((uint32_t)X[r][c] >> 31);
    }
  group_products<F, K0, KN, R, CC, UNR>(P, rl, cl, nmin, S);
}

// normalise a sum to the state form: X with its leading bit at bit 30 (in
// ones' complement when negative) and n = -(exponent of the leading bit).
// S == 0 gives X == 0 (its n is meaningless and is fixed by the caller).
__device__ __forceinline__ uint32_t msb_pos(uint32_t x) {  // -1 (all ones) for x == 0
  uint32_t p;
  asm("bfind.u32 %0, %1;" : "=r"(p) : "r"(x));
  return p;
}
template <int F>
__device__ __forceinline__ void to_state(int32_t s, int32_t nmin, int32_t &n, int32_t &X, uint32_t mask) {
  const uint32_t mag = (uint32_t)(s < 0 ? -s : s);
  const int32_t p = (int32_t)msb_pos(mag);
  const uint32_t M = shl_u32(mag, (uint32_t)(30 - p));
  n = nmin + F - p;  // the leading bit is worth 2^(e_max - F + p)
  X = (int32_t)((M & mask) ^ (uint32_t)(s >> 31));
}
// the same for a sum that may need 33 bits (F = 25)
template <int F>
__device__ __forceinline__ void to_state64(int64_t s, int32_t nmin, int32_t &n, int32_t &X, uint32_t mask) {
  const uint64_t mag = (uint64_t)(s < 0 ? -s : s);
  const int32_t p = 63 - __clzll((long long)mag);  // -1 for 0
  const uint32_t M = p > 30 ? (uint32_t)(mag >> (p - 30)) : shl_u32((uint32_t)mag, (uint32_t)(30 - p));
  n = nmin + F - p;
  X = (int32_t)((M & mask) ^ (uint32_t)(s < 0 ? 0xFFFFFFFFu : 0u));
}

// Zero tests of panel operands (the zero-sign rule needs them).
template <class PanelT>
__device__ __forceinline__ bool zero_a(const PanelT &P, int k, int m) { return n_a(P, k, m) == ZSENT; }
template <class PanelT>
__device__ __forceinline__ bool zero_b(const PanelT &P, int k, int n) { return n_b(P, k, n) == ZSENT; }

// Special-value outcome of each output of an R x CC block whose chunk holds
// Inf or NaN somewhere in its A or B panel: 2 bits per output (0 none, 1 NaN,
// 2 +Inf, 3 -Inf).  c_nan / c_infp / c_infn flag outputs whose incoming value
// is NaN / +Inf / -Inf.  Kept out of line: it is rare and would otherwise
// crowd the registers of the main path.
template <int R, int CC, class PanelT>
__device__ __noinline__ uint64_t special_codes(const PanelT *P, int rl, int cl, uint32_t c_nan, uint32_t c_infp,
                                               uint32_t c_infn);
template <int R, int CC, class PanelT>
__device__ __forceinline__ uint64_t special_codes(const PanelT &P, int rl, int cl, uint32_t c_nan, uint32_t c_infp,
                                                  uint32_t c_infn) {
  return special_codes<R, CC>(&P, rl, cl, c_nan, c_infp, c_infn);
}
template <int R, int CC, class PanelT>
__device__ __noinline__ uint64_t special_codes(const PanelT *P, int rl, int cl, uint32_t c_nan, uint32_t c_infp,
                                               uint32_t c_infn) {
  uint64_t codes = 0;
#pragma unroll 1
  for (int o = 0; o < R * CC; o++) {
    const int r = o / CC, c = o % CC;
    bool nan = (c_nan >> o) & 1u, ip = (c_infp >> o) & 1u, in = (c_infn >> o) & 1u;
#pragma unroll 1
    for (int k = 0; k < 16; k++) {
      const int32_t an = n_a(*P, k, rl + r), bn = n_b(*P, k, cl + c);
      if (an == NNAN || bn == NNAN) {
        nan = true;
      } else if (an == NINF || bn == NINF) {
        if (an == ZSENT || bn == ZSENT) nan = true;
        else if (neg_a(*P, k, rl + r) != neg_b(*P, k, cl + c)) in = true;
        else ip = true;
      }
    }
    const uint64_t code = (nan || (ip && in)) ? 1u : ip ? 2u : in ? 3u : 0u;
    codes |= code << (2 * o);
  }
  return codes;
}

// One 16-deep K chunk for an R x CC block of outputs at panel row rl, col cl,
// updating the accumulator state (Np, X, dneg0) in place.
//   Np    -- n of adjacent output pairs, packed
//   X     -- significands (see mmaemu_core.cuh)
//   dneg0 -- bit r*CC+c set when that output's state is -0
template <int MODEL, int FMT, int R, int CC, class PanelT>
__device__ __forceinline__ void mma_chunk(const PanelT &P, int rl, int cl, uint32_t (&Np)[R][CC / 2],
                                          int32_t (&X)[R][CC], uint32_t &dneg0, bool panel_special) {
  constexpr int F = ModelT<MODEL>::F;
  constexpr int UNR = kUnroll<MODEL, FMT>;
  static_assert(R * CC <= 32 && CC % 2 == 0, "per-output masks hold 32 outputs");
  // with 24 or more fraction bits the grid would see state bits below the
  // fp32 value's 24: keep bits 0..6 clear
  constexpr uint32_t XMASK = F >= 24 ? 0x7FFFFF80u : 0x7FFFFFFFu;

  // kinds of the incoming values, needed only when A/B hold Inf or NaN
  uint32_t c_nan = 0, c_infp = 0, c_infn = 0;
  if (panel_special) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const int32_t n = (c & 1) ? hi16(Np[r][c / 2]) : lo16(Np[r][c / 2]);
        const uint32_t bit = 1u << (r * CC + c);
        if (n == STATE_NAN) c_nan |= bit;
        if (n == STATE_INF) {
          if (X[r][c] < 0) c_infn |= bit;
          else c_infp |= bit;
        }
      }
  }

  int32_t S[R][CC], nmin[R][CC];
  if constexpr (MODEL == MODEL_AMPERE) {
    // stage 1: {C, P[1..8]}
    group_sum<FMT, F, 0, 8, R, CC, UNR>(P, rl, cl, Np, X, nmin, S);
    // hand-over: the stage-1 sum as a 24-bit term (the state form keeps extra
    // low bits, but stage 2 shifts it right by at least 7, which truncates
    // them exactly like the normalisation would); a zero sum adds no term
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int p = 0; p < CC / 2; p++) {
        int32_t n0, n1;
        to_state<F>(S[r][2 * p], nmin[r][2 * p], n0, X[r][2 * p], 0x7FFFFFFFu);
        to_state<F>(S[r][2 * p + 1], nmin[r][2 * p + 1], n1, X[r][2 * p + 1], 0x7FFFFFFFu);
        Np[r][p] = pack16(S[r][2 * p] ? n0 : ZSENT, S[r][2 * p + 1] ? n1 : ZSENT);
      }
    // stage 2: {S1, P[9..16]}
    group_sum<FMT, F, 8, 8, R, CC, UNR>(P, rl, cl, Np, X, nmin, S);
  } else if constexpr (kWideSum<MODEL>) {
    // one stage {C, P[1..16]}: the products here, C in the write-back
    group_max<FMT, 0, 16, R, CC, UNR>(P, rl, cl, Np, nmin);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) S[r][c] = 0;
    group_products<F, 0, 16, R, CC, UNR>(P, rl, cl, nmin, S);
  } else {
    // one stage: {C, P[1..16]}
    group_sum<FMT, F, 0, 16, R, CC, UNR>(P, rl, cl, Np, X, nmin, S);
  }

  // toward-zero write-back into the state (the fp32 value is its top 24 bits)
  bool any_rare = false;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) {
      int32_t n0, n1;
      if constexpr (kWideSum<MODEL>) {
        // add the carried state (ones' complement alignment, as group_sum)
        // to the products in 64 bits
        int32_t nn[2];
#pragma unroll
        for (int q = 0; q < 2; q++) {
          const int c = 2 * p + q;
          const int32_t nc = q ? hi16(Np[r][p]) : lo16(Np[r][p]);
          const int32_t carry = shr_s32(X[r][c], (uint32_t)(nc - nmin[r][c] + 30 - F)) +
                                (int32_t)((uint32_t)X[r][c] >> 31);
          to_state64<F>((int64_t)S[r][c] + carry, nmin[r][c], nn[q], X[r][c], XMASK);
        }
        n0 = nn[0];
        n1 = nn[1];
      } else {
        to_state<F>(S[r][2 * p], nmin[r][2 * p], n0, X[r][2 * p], XMASK);
        to_state<F>(S[r][2 * p + 1], nmin[r][2 * p + 1], n1, X[r][2 * p + 1], XMASK);
      }
      Np[r][p] = pack16(n0, n1);
      // zero (X == 0 exactly when S == 0), or the exponent outside [-126, 127]
      any_rare = any_rare || X[r][2 * p] == 0 || (uint32_t)(n0 + 127) > 253u || X[r][2 * p + 1] == 0 ||
                 (uint32_t)(n1 + 127) > 253u;
    }
  uint32_t rare = 0;
  if (any_rare) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const int32_t n0 = (c & 1) ? hi16(Np[r][c / 2]) : lo16(Np[r][c / 2]);
        if (X[r][c] == 0 || (uint32_t)(n0 + 127) > 253u) rare |= 1u << (r * CC + c);
      }
  }
  dneg0 &= rare;  // every ordinary result is nonzero

  if (rare) {
    // Only the new state is used here: S == 0 left X == 0, and for S != 0
    // X ^ sgn = (|S| << clz) >> 1 with n = -(exponent of the leading bit).
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const uint32_t bit = 1u << (r * CC + c);
        if (!(rare & bit)) continue;
        const int32_t x0 = X[r][c];
        const int32_t n0 = (c & 1) ? hi16(Np[r][c / 2]) : lo16(Np[r][c / 2]);
        const uint32_t sg = (uint32_t)(x0 >> 31);
        int32_t n;
        int32_t x;
        bool negz = false;
        if (x0 == 0) {
          // zero-sign rule: -0 only when C and all 16 products are -0
          bool neg = (dneg0 & bit) != 0;
          for (int k = 0; k < 16 && neg; k++) {
            const bool zero = zero_a(P, k, rl + r) || zero_b(P, k, cl + c);
            neg = zero && neg_a(P, k, rl + r) != neg_b(P, k, cl + c);
          }
          n = ZSENT;
          x = neg ? -1 : 0;
          negz = neg;
        } else if (n0 <= STATE_NAN + 50) {  // a NaN carried in
          n = STATE_NAN;
          x = 0x40000000;
        } else if (n0 < -127) {  // exponent above 127: overflow to infinity
          n = STATE_INF;
          x = (int32_t)(0x40000000u ^ sg);
        } else {
          // below 2^-126: truncate onto the subnormal grid 2^-149, i.e.
          // q = floor(|S| 2^(e_max - F + 149)) = ((X ^ sgn) >> (n - 119))
          const uint32_t q = shr_u32((uint32_t)x0 ^ sg, (uint32_t)(n0 - 119));
          if (q == 0) {
            n = ZSENT;
            x = (int32_t)sg;
            negz = sg != 0;
          } else {
            n = 126;
            x = (int32_t)((q << 7) ^ sg);
          }
        }
        X[r][c] = x;
        Np[r][c / 2] = (c & 1) ? pack16(lo16(Np[r][c / 2]), n) : pack16(n, hi16(Np[r][c / 2]));
        dneg0 = negz ? (dneg0 | bit) : (dneg0 & ~bit);
      }
  }

  // special values: NaN anywhere or Inf x 0 -> NaN; Inf of one sign -> that
  // Inf; both signs -> NaN
  if (panel_special) {
    const uint64_t codes = special_codes<R, CC>(P, rl, cl, c_nan, c_infp, c_infn);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const uint32_t code = (uint32_t)(codes >> (2 * (r * CC + c))) & 3u;
        if (code == 0u) continue;
        const int32_t n = code == 1u ? STATE_NAN : STATE_INF;
        X[r][c] = code == 3u ? (int32_t)0xBFFFFFFFu : 0x40000000;
        Np[r][c / 2] = (c & 1) ? pack16(lo16(Np[r][c / 2]), n) : pack16(n, hi16(Np[r][c / 2]));
        dneg0 &= ~(1u << (r * CC + c));
      }
  }
}

// ---------------------------------------------------------------------------
// Float-assisted chunk (FP16 and E4M3 inputs).  The accumulator state is the
// fp32 value D itself (plus n = -e(D) in packed pairs), and the steps around
// the integer group sums run on the conversion and FMA units:
//  * a carried fp32 value c contributes trunc(c 2^(F - e_max)): one exact
//    multiply by a power of two and one toward-zero conversion to int;
//  * cvt.rz.f32.s32(S) is S truncated to 24 significant bits with its sign
//    and exponent -- the Ampere stage hand-over (W = 24) and the fp32
//    write-back, which is that float times 2^(e_max - F).
//
// Range.  A thread takes this path only if every C value it starts from is
// +-0 or of magnitude in [2^-60, 2^63).  FP16 products are below 2^32 and
// E4M3 products below 2^18, so over any K < 2^31 a running value stays below
// 2^64 (truncation never rounds up).  A group with a nonzero product has
// e_max >= -28, so a nonzero sum is at least one unit of the grid
// 2^(e_max - F) >= 2^-52; without one, the sum is the carried value itself.
// Hence every D is +-0 or normal with n = -e(D) in [-63, 60]: the write-back
// can neither overflow nor underflow, and every power of two formed below
// is a normal float.  Inf/NaN operands hand the thread to the integer path.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float i2f_rz(int32_t s) {
  float f;
  asm("cvt.rz.f32.s32 %0, %1;" : "=f"(f) : "r"(s));
  return f;
}
__device__ __forceinline__ int32_t f2i_rz(float f) {
  int32_t r;
  asm("cvt.rzi.s32.f32 %0, %1;" : "=r"(r) : "f"(f));
  return r;
}
// biased exponent field of a float (0 for zero)
__device__ __forceinline__ int32_t exp_field(float f) { return (int32_t)((__float_as_uint(f) << 1) >> 24); }
// 2^k as a float for k in [-126, 127] (one IMAD)
__device__ __forceinline__ float pow2f(int32_t k) { return __uint_as_float((uint32_t)k * 0x800000u + 0x3F800000u); }

// the path's range of accumulator magnitudes: [2^-FAST_NMAX, 2^FAST_EMAX)
constexpr int FAST_NMAX = 60, FAST_EMAX = 63;
// BF16 products and sums reach exponents far outside the float range
template <int FMT> constexpr bool kFloatAssisted = FMT != FMT_BF16;
// Ampere stage hand-over: S1 is carried as g1 = S1_24 2^(-HX - e_max1) and
// scaled by 2^(HX + e_max2) in stage 2.  With HX = 42 both factors stay
// normal for e_max in [-60, 63], and when S1 == 0 (its n then reads
// e_max1 + 150 instead of a zero marker) the stage-2 factor, if that n
// becomes stage 2's maximum, is a finite float: the zero carry stays zero.
constexpr int HX = 42;

template <int MODEL, int FMT, int R, int CC, class PanelT>
__device__ __forceinline__ void mma_chunk_fast(const PanelT &P, int rl, int cl, uint32_t (&Np)[R][CC / 2],
                                               uint32_t (&V)[R][CC], uint32_t &dneg0, bool panel_special,
                                               bool &to_integer) {
  constexpr int F = ModelT<MODEL>::F;
  static_assert(FMT != FMT_BF16, "BF16 exponents leave the float range");
  int32_t S[R][CC], nmin[R][CC];
  constexpr int KN1 = MODEL == MODEL_AMPERE ? 8 : 16;
  constexpr bool WIDE = kWideSum<MODEL>;
  constexpr int UNR = kUnroll<MODEL, FMT>;
  // first (or only) group: carried D plus products (the carried term is
  // added in the write-back when the sum may need 33 bits)
  group_max<FMT, 0, KN1, R, CC, UNR>(P, rl, cl, Np, nmin);
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++)
      S[r][c] = WIDE ? 0 : f2i_rz(__uint_as_float(V[r][c]) * pow2f(F + nmin[r][c]));
  group_products<F, 0, KN1, R, CC, UNR>(P, rl, cl, nmin, S);
  if constexpr (MODEL == MODEL_AMPERE) {
    // hand-over: the stage-1 sum truncated to 24 bits; a zero sum needs no
    // marker (see HX): its n exceeds every nonzero product's n (<= 28)
    float g1[R][CC];
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int p = 0; p < CC / 2; p++) {
        int32_t n1[2];
#pragma unroll
        for (int q = 0; q < 2; q++) {
          const int c = 2 * p + q;
          const float f1 = i2f_rz(S[r][c]);
          n1[q] = nmin[r][c] + (F + 127) - exp_field(f1);
          g1[r][c] = f1 * pow2f(-HX - nmin[r][c]);
        }
        Np[r][p] = pack16(n1[0], n1[1]);
      }
    group_max<FMT, 8, 8, R, CC, UNR>(P, rl, cl, Np, nmin);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) S[r][c] = f2i_rz(g1[r][c] * pow2f(nmin[r][c] + HX));
    group_products<F, 8, 8, R, CC, UNR>(P, rl, cl, nmin, S);
  }

  // write-back: D = cvt.rz(S) 2^(e_max - F), exact (D is normal)
  bool any_zero = false;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) {
      int32_t nn[2];
#pragma unroll
      for (int q = 0; q < 2; q++) {
        const int c = 2 * p + q;
        float f2;
        if constexpr (WIDE) {
          const int64_t s64 = (int64_t)S[r][c] + f2i_rz(__uint_as_float(V[r][c]) * pow2f(F + nmin[r][c]));
          asm("cvt.rz.f32.s64 %0, %1;" : "=f"(f2) : "l"(s64));
          S[r][c] = s64 != 0;  // only the zero test below reads S
        } else {
          f2 = i2f_rz(S[r][c]);
        }
        nn[q] = nmin[r][c] + (F + 127) - exp_field(f2);
        V[r][c] = __float_as_uint(f2 * pow2f(-F - nmin[r][c]));
        any_zero = any_zero || S[r][c] == 0;
      }
      Np[r][p] = pack16(nn[0], nn[1]);
    }
  uint32_t zero = 0;
  if (any_zero) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        if (S[r][c] != 0) continue;
        const uint32_t bit = 1u << (r * CC + c);
        zero |= bit;
        // zero-sign rule: -0 only when C and all 16 products are -0
        bool neg = (dneg0 & bit) != 0;
        for (int k = 0; k < 16 && neg; k++) {
          const bool z = zero_a(P, k, rl + r) || zero_b(P, k, cl + c);
          neg = z && neg_a(P, k, rl + r) != neg_b(P, k, cl + c);
        }
        V[r][c] = neg ? 0x80000000u : 0u;
        Np[r][c / 2] = (c & 1) ? pack16(lo16(Np[r][c / 2]), ZSENT) : pack16(ZSENT, hi16(Np[r][c / 2]));
        dneg0 = neg ? (dneg0 | bit) : (dneg0 & ~bit);
      }
  }
  dneg0 &= zero;

  // Inf/NaN operands (the incoming values are finite on this path)
  if (panel_special) {
    const uint64_t codes = special_codes<R, CC>(P, rl, cl, 0u, 0u, 0u);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const uint32_t code = (uint32_t)(codes >> (2 * (r * CC + c))) & 3u;
        if (code == 0u) continue;
        V[r][c] = code == 1u ? ModelT<MODEL>::NAN_BITS : code == 2u ? 0x7F800000u : 0xFF800000u;
        dneg0 &= ~(1u << (r * CC + c));
        to_integer = true;  // the caller rebuilds the integer state from V
      }
  }
}

// switch a thread's state from fp32 values (float-assisted path) to (n, X)
template <int R, int CC>
__device__ __forceinline__ void values_to_state(uint32_t (&Np)[R][CC / 2], uint32_t (&V)[R][CC]) {
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int p = 0; p < CC / 2; p++) {
      int32_t n0, n1, x0, x1;
      bool z;
      state_from_fp32(V[r][2 * p], n0, x0, z);
      state_from_fp32(V[r][2 * p + 1], n1, x1, z);
      V[r][2 * p] = (uint32_t)x0;
      V[r][2 * p + 1] = (uint32_t)x1;
      Np[r][p] = pack16(n0, n1);
    }
}

// Packed n and -0 mask of an R x CC block of fp32 values V (raw bits); returns
// whether all of them suit the float-assisted path (zero, or of magnitude in
// [2^-FAST_NMAX, 2^FAST_EMAX)).
template <int R, int CC>
__device__ __forceinline__ bool classify_values(const uint32_t (&V)[R][CC], uint32_t (&Np)[R][CC / 2],
                                                uint32_t &dneg0) {
  dneg0 = 0;
  bool ok = true;
#pragma unroll
  for (int r = 0; r < R; r++) {
    int32_t n[CC];
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t field = (V[r][c] >> 23) & 0xFFu;
      const bool zero = (V[r][c] << 1) == 0u;
      if (zero && V[r][c]) dneg0 |= 1u << (r * CC + c);
      n[c] = zero ? ZSENT : 127 - (int32_t)field;
      ok = ok && (zero || (field >= 127u - FAST_NMAX && field < 127u + FAST_EMAX));
    }
#pragma unroll
    for (int p = 0; p < CC / 2; p++) Np[r][p] = pack16(n[2 * p], n[2 * p + 1]);
  }
  return ok;
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

// fp32 C values of an R x CC block as raw bits with their packed n (the
// same as load_bits + classify_values, row by row: this order schedules
// better in the GEMM's prologue)
template <int R, int CC>
__device__ __forceinline__ bool load_values(const float *C, size_t ldc, bool have_c, uint32_t (&Np)[R][CC / 2],
                                            uint32_t (&V)[R][CC], uint32_t &dneg0) {
  dneg0 = 0;
  bool ok = true;
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
    int32_t n[CC];
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t field = (V[r][c] >> 23) & 0xFFu;
      const bool zero = (V[r][c] << 1) == 0u;
      if (zero && V[r][c]) dneg0 |= 1u << (r * CC + c);
      n[c] = zero ? ZSENT : 127 - (int32_t)field;
      ok = ok && (zero || (field >= 127u - FAST_NMAX && field < 127u + FAST_EMAX));
    }
#pragma unroll
    for (int p = 0; p < CC / 2; p++) Np[r][p] = pack16(n[2 * p], n[2 * p + 1]);
  }
  return ok;
}

// state of an R x CC block from fp32 C values (row stride ldc), or +0
template <int R, int CC>
__device__ __forceinline__ void load_state(const float *C, size_t ldc, bool have_c, uint32_t (&Np)[R][CC / 2],
                                           int32_t (&X)[R][CC], uint32_t &dneg0) {
  dneg0 = 0;
#pragma unroll
  for (int r = 0; r < R; r++) {
    uint32_t cv[CC];
    if (have_c) {
#pragma unroll
      for (int q = 0; q < CC / 4; q++) {
        const uint4 v = reinterpret_cast<const uint4 *>(C + r * ldc)[q];
        cv[4 * q] = v.x; cv[4 * q + 1] = v.y; cv[4 * q + 2] = v.z; cv[4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int c = 0; c < CC; c++) cv[c] = 0u;
    }
    int32_t n[CC];
#pragma unroll
    for (int c = 0; c < CC; c++) {
      bool nz;
      state_from_fp32(cv[c], n[c], X[r][c], nz);
      if (nz) dneg0 |= 1u << (r * CC + c);
    }
#pragma unroll
    for (int p = 0; p < CC / 2; p++) Np[r][p] = pack16(n[2 * p], n[2 * p + 1]);
  }
}

template <int R, int CC>
__device__ __forceinline__ void state_to_fp32(const uint32_t (&Np)[R][CC / 2], const int32_t (&X)[R][CC],
                                              uint32_t (&D)[R][CC], uint32_t nan_bits) {
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++)
      D[r][c] = fp32_from_state((c & 1) ? hi16(Np[r][c / 2]) : lo16(Np[r][c / 2]), X[r][c], nan_bits);
}

// ---------------------------------------------------------------------------
// raw operand loading and decoding into a panel
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

// Exact value of a decoded element as a double, m 2^(e - p) with its sign;
// zero, Inf and NaN become +-2^-500 (the special-value path reads their
// markers instead).
template <int FMT>
__device__ __forceinline__ double dec_value(const Dec &d) {
  constexpr int P = FmtT<FMT>::P;
  const double scale = __hiloint2double((1023 - d.n - P) << 20, 0);  // 2^(e - p), normal for every format
  const double v = d.m ? (double)d.m * scale : 0x1p-500;
  return d.s ? -v : v;
}

// Decode 8 k-consecutive elements of A row m (k = 8h .. 8h+7) into a tile
// kernel's panel (4-column groups, natural order), or of B column n.
template <int MODEL, int FMT, int BM, int BN>
__device__ __forceinline__ uint32_t store_a8(Panel<BM, BN> &P, int m, int h, const Raw8<FMT> &raw) {
  uint32_t special = 0, signs = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const Dec d = decode<FMT>(raw.get(i));
    P.aV[8 * h + i][m] = dec_value<FMT>(d);
    P.aN2[8 * h + i][m] = pack16(d.n, d.n);
    signs |= (d.s & 1u) << i;
    special |= d.special;
  }
  reinterpret_cast<uint8_t *>(&P.aS[m])[h] = (uint8_t)signs;
  return special;
}

template <int FMT, int BM, int BN>
__device__ __forceinline__ uint32_t store_b8(Panel<BM, BN> &P, int n, int h, const Raw8<FMT> &raw) {
  uint32_t special = 0, signs = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const Dec d = decode<FMT>(raw.get(i));
    P.bV[8 * h + i][n] = dec_value<FMT>(d) * (1.0 + 0x1p-40);  // exact
    P.bN2[8 * h + i][n] = (int16_t)d.n;
    signs |= (d.s & 1u) << i;
    special |= d.special;
  }
  reinterpret_cast<uint8_t *>(&P.bS[n])[h] = (uint8_t)signs;
  return special;
}

// ---------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------
// Tuning knobs (compile-time): resident blocks per SM and the unroll of the k loops.
// A block computes GBM x GBN outputs with one warp per 32 x 32 and a 4 x 8
// block of outputs per thread.  Measured: 64 x 64 blocks of 128 threads, 4
// per SM, are 3-5% faster than 64 x 128 blocks of 256 threads, 2 per SM (the
// same registers and warps per SM, but half as many warps wait at each
// block's per-chunk barrier).
#ifndef MMAEMU_GBN
#define MMAEMU_GBN 64
#endif
#ifndef MMAEMU_GMINB
#define MMAEMU_GMINB (256 / MMAEMU_GBN)
#endif
constexpr int GBM = 64, GBN = MMAEMU_GBN, GWN = GBN / 32, GTHREADS = 32 * 2 * GWN, GR = 4, GCC = 8;
using GPanel = Panel<GBM, GBN>;

// Everything a GEMM launch needs.  Element (m, k) of op(A) sits at
// A[m * lda + k] (ta == 0) or A[k * lda + m] (ta == 1); element (k, n) of
// op(B) at B[k * ldb + n] (tb == 0) or B[n * ldb + k] (tb == 1); C, D and
// Dref are row-major with their own leading dimensions.  Batch b (blockIdx.z)
// adds b times the batch stride to every pointer.  D, Dref, fp and mism may
// each be null; C null means +0.
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
  // batch entry, 64-row block of A or 128-column block of B, and K chunk, a
  // blob laid out exactly like that part of a shared-memory panel; and one
  // special-value flag word per blob
  unsigned char *dA, *dB;
  uint32_t *flags_a, *flags_b;
  int batch;
};

// Decoded panel blobs: the A part (aV, aN2, aS) and the B part (bV, bN2,
// bS) of a GPanel, stored contiguously in that order.
constexpr size_t ABLOB = offsetof(GPanel, bV), BBLOB = sizeof(GPanel) - offsetof(GPanel, bV);
constexpr size_t OFF_AN2 = offsetof(GPanel, aN2), OFF_AS = offsetof(GPanel, aS);
constexpr size_t OFF_BN2 = offsetof(GPanel, bN2) - ABLOB, OFF_BS = offsetof(GPanel, bS) - ABLOB;
static_assert(ABLOB == 16 * GBM * 8 + 16 * GBM * 4 + GBM * 2 && BBLOB == 16 * GBN * 8 + 16 * GBN * 2 + GBN * 2 &&
                  ABLOB % 16 == 0 && BBLOB % 16 == 0,
              "panel layout");

// Decode pass, A side: one thread per 8 k-consecutive elements (row m,
// chunk j, half h) into the blob of (batch entry, m / 64, j).
template <int MODEL, int FMT>
__global__ void __launch_bounds__(256) decode_a_kernel(const GemmParams p) {
  constexpr int ESIZE = FMT == FMT_E4M3 ? 1 : 2;
  const int nrb = (p.M + GBM - 1) / GBM, nch = p.K / 16;
  const int m = blockIdx.x * blockDim.x + threadIdx.x;
  if (m >= nrb * GBM) return;
  const int j = blockIdx.y >> 1, h = blockIdx.y & 1;
  const size_t bz = blockIdx.z;
  const void *A = static_cast<const unsigned char *>(p.A) + bz * (size_t)p.sA * ESIZE;
  const bool valid = m < p.M;
  const size_t k = 16 * (size_t)j + 8 * h, lda = (size_t)p.lda;
  const Raw8<FMT> raw = !p.ta ? load_row8<FMT>(A, (size_t)m * lda + k, valid) : load_col8<FMT>(A, k * lda + m, lda, valid);
  const int rb = m / GBM, ml = m % GBM;
  unsigned char *blob = p.dA + ((bz * nrb + rb) * nch + j) * ABLOB;
  uint32_t special = 0, signs = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const Dec d = decode<FMT>(raw.get(i));
    const size_t kk = (size_t)(8 * h + i);
    *reinterpret_cast<double *>(blob + (kk * GBM + ml) * 8) = dec_value<FMT>(d);
    *reinterpret_cast<uint32_t *>(blob + OFF_AN2 + (kk * GBM + ml) * 4) = pack16(d.n, d.n);
    signs |= (d.s & 1u) << i;
    special |= d.special;
  }
  blob[OFF_AS + 2 * ml + h] = (unsigned char)signs;
  if (special) atomicOr(&p.flags_a[(bz * nrb + rb) * nch + j], 1u);
}

// Decode pass, B side: one thread per 8 k-consecutive elements of column n.
template <int MODEL, int FMT>
__global__ void __launch_bounds__(256) decode_b_kernel(const GemmParams p) {
  constexpr int ESIZE = FMT == FMT_E4M3 ? 1 : 2;
  const int ncb = (p.N + GBN - 1) / GBN, nch = p.K / 16;
  const int n = blockIdx.x * blockDim.x + threadIdx.x;
  if (n >= ncb * GBN) return;
  const int j = blockIdx.y >> 1, h = blockIdx.y & 1;
  const size_t bz = blockIdx.z;
  const void *B = static_cast<const unsigned char *>(p.B) + bz * (size_t)p.sB * ESIZE;
  const bool valid = n < p.N;
  const size_t k = 16 * (size_t)j + 8 * h, ldb = (size_t)p.ldb;
  const Raw8<FMT> raw = !p.tb ? load_col8<FMT>(B, k * ldb + n, ldb, valid) : load_row8<FMT>(B, (size_t)n * ldb + k, valid);
  const int cb = n / GBN, nl = n % GBN;
  unsigned char *blob = p.dB + ((bz * ncb + cb) * nch + j) * BBLOB;
  uint32_t special = 0, signs = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const Dec d = decode<FMT>(raw.get(i));
    const size_t kk = (size_t)(8 * h + i);
    *reinterpret_cast<double *>(blob + (kk * GBN + bv_slot(nl)) * 8) = dec_value<FMT>(d) * (1.0 + 0x1p-40);  // exact
    *reinterpret_cast<int16_t *>(blob + OFF_BN2 + (kk * GBN + nl) * 2) = (int16_t)d.n;
    signs |= (d.s & 1u) << i;
    special |= d.special;
  }
  blob[OFF_BS + 2 * nl + h] = (unsigned char)signs;
  if (special) atomicOr(&p.flags_b[(bz * ncb + cb) * nch + j], 1u);
}

// 16-byte asynchronous global -> shared copy
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Blocks are visited in groups of GROUP_ROWS row blocks, column block by
// column block, so that the blocks resident at one time share A and B
// panels and the decoded operands are reused from L2.
constexpr int GROUP_ROWS = 16;

template <int MODEL, int FMT>
__global__ void __launch_bounds__(GTHREADS, MMAEMU_GMINB) gemm_kernel(const GemmParams p) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GPanel *panels = reinterpret_cast<GPanel *>(smem_raw);
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
  // this thread's 4 x 8 outputs
  const int rl = (warp / GWN) * 32 + (lane >> 2) * GR;
  const int cl = (warp % GWN) * 32 + (lane & 3) * GCC;
  const bool out_valid = (row0 + rl < M) && (col0 + cl < N);

  // Per chunk, the block copies its decoded A and B blobs (12,416 + 10,368
  // bytes for 64 x 64 blocks) into the panel with 16-byte asynchronous copies.
  const int nchunks = K / 16;
  const unsigned char *blob_a = p.dA + (bz * nrb + rb) * (size_t)nchunks * ABLOB;
  const unsigned char *blob_b = p.dB + (bz * ncb + cb) * (size_t)nchunks * BBLOB;
  const uint32_t *flag_a = p.flags_a + (bz * nrb + rb) * (size_t)nchunks;
  const uint32_t *flag_b = p.flags_b + (bz * ncb + cb) * (size_t)nchunks;
  auto issue_chunk = [&](int j, GPanel &P) {
    const uint4 *sa = reinterpret_cast<const uint4 *>(blob_a + (size_t)j * ABLOB);
    const uint4 *sb = reinterpret_cast<const uint4 *>(blob_b + (size_t)j * BBLOB);
    uint4 *da = reinterpret_cast<uint4 *>(&P);
    uint4 *db = reinterpret_cast<uint4 *>(reinterpret_cast<unsigned char *>(&P) + ABLOB);
#pragma unroll
    for (int i = 0; i < (int)((ABLOB / 16 + GTHREADS - 1) / GTHREADS); i++)
      if (tid + i * GTHREADS < (int)(ABLOB / 16)) cp_async16(da + tid + i * GTHREADS, sa + tid + i * GTHREADS);
#pragma unroll
    for (int i = 0; i < (int)((BBLOB / 16 + GTHREADS - 1) / GTHREADS); i++)
      if (tid + i * GTHREADS < (int)(BBLOB / 16)) cp_async16(db + tid + i * GTHREADS, sb + tid + i * GTHREADS);
    cp_async_commit();
  };
  static_assert(ABLOB % 16 == 0 && BBLOB % 16 == 0, "16-byte copies");

  // accumulator: fp32 bits V on the float-assisted path (FP16 / E4M3 while
  // the values stay in its range), else the integer state (n, X) in V's place
  uint32_t Np[GR][GCC / 2];
  uint32_t V[GR][GCC];
  int32_t(&X)[GR][GCC] = reinterpret_cast<int32_t(&)[GR][GCC]>(V);
  uint32_t dneg0;
  const float *Cb = p.C ? p.C + bz * (size_t)p.sC + (size_t)(row0 + rl) * p.ldc + col0 + cl : nullptr;
  bool fast = load_values<GR, GCC>(Cb, (size_t)p.ldc, Cb != nullptr && out_valid, Np, V, dneg0);
  if (!kFloatAssisted<FMT>) fast = false;
  if (!fast) values_to_state<GR, GCC>(Np, V);

  issue_chunk(0, panels[0]);
  cp_async_wait_all();
  __syncthreads();
  bool panel_special = (flag_a[0] | flag_b[0]) != 0;
  for (int j = 0; j < nchunks; j++) {
    bool next_special = false;
    if (j + 1 < nchunks) {
      issue_chunk(j + 1, panels[(j + 1) & 1]);
      next_special = (flag_a[j + 1] | flag_b[j + 1]) != 0;
    }
    if constexpr (kFloatAssisted<FMT>) {
      if (fast) {
        bool to_integer = false;
        mma_chunk_fast<MODEL, FMT, GR, GCC>(panels[j & 1], rl, cl, Np, V, dneg0, panel_special, to_integer);
        if (to_integer) {
          values_to_state<GR, GCC>(Np, V);
          fast = false;
        }
      } else {
        mma_chunk<MODEL, FMT, GR, GCC>(panels[j & 1], rl, cl, Np, X, dneg0, panel_special);
      }
    } else {
      mma_chunk<MODEL, FMT, GR, GCC>(panels[j & 1], rl, cl, Np, X, dneg0, panel_special);
    }
    if (j + 1 < nchunks) {
      cp_async_wait_all();
      __syncthreads();
      panel_special = next_special;
    }
  }

  // epilogue: store D, compare with the claimed D, per-16x16-tile xorsum
  uint32_t D[GR][GCC];
  if (fast) {
#pragma unroll
    for (int r = 0; r < GR; r++)
#pragma unroll
      for (int c = 0; c < GCC; c++) D[r][c] = V[r][c];
  } else {
    state_to_fp32<GR, GCC>(Np, X, D, ModelT<MODEL>::NAN_BITS);
  }
  if (p.D != nullptr && out_valid) {
    float *Db = p.D + bz * (size_t)p.sD + (size_t)(row0 + rl) * p.ldd + col0 + cl;
#pragma unroll
    for (int i = 0; i < GR; i++) {
      uint4 *dst = reinterpret_cast<uint4 *>(Db + (size_t)i * p.ldd);
      dst[0] = make_uint4(D[i][0], D[i][1], D[i][2], D[i][3]);
      dst[1] = make_uint4(D[i][4], D[i][5], D[i][6], D[i][7]);
    }
  }
  if (p.Dref != nullptr) {
    // bitwise comparison; the smallest mismatching position of the block is
    // found as the smallest in-block offset (row-major order is preserved)
    uint32_t count = 0, first = 0xFFFFFFFFu;
    if (out_valid) {
      const float *Rb = p.Dref + bz * (size_t)p.sR + (size_t)(row0 + rl) * p.ldr + col0 + cl;
#pragma unroll
      for (int i = 0; i < GR; i++) {
        const uint4 *src = reinterpret_cast<const uint4 *>(Rb + (size_t)i * p.ldr);
        const uint4 v0 = src[0], v1 = src[1];
        const uint32_t got[GCC] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int c = GCC - 1; c >= 0; c--)
          if (got[c] != D[i][c]) {
            count++;
            first = min(first, (uint32_t)((rl + i) * GBN + cl + c));
          }
      }
    }
    count = __reduce_add_sync(0xFFFFFFFFu, count);
    first = __reduce_min_sync(0xFFFFFFFFu, first);
    if (lane == 0 && count != 0) {
      const unsigned long long idx = (unsigned long long)bz * M * N +
                                     (unsigned long long)(row0 + first / GBN) * N + col0 + first % GBN;
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
    // the 8 lanes sharing a 16x16 tile differ in lane bits 0, 2, 3
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 1);
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 4);
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 8);
    if (out_valid && (lane & 0xD) == 0) {
      const int tr = (row0 + rl) >> 4, tc = (col0 + cl) >> 4;
      p.fp[bz * (size_t)p.sF + (size_t)tr * (N >> 4) + tc] = x;
    }
  }
}

// ---------------------------------------------------------------------------
// independent tiles: one warp per 16x16x16 tile, each lane 2 x 4 outputs
// ---------------------------------------------------------------------------
constexpr int TWARPS = 8, TR = 2, TCC = 4;
using TPanel = Panel<16, 16>;

template <int MODEL, int FMT>
__global__ void __launch_bounds__(TWARPS * 32, 3) tiles_kernel(const void *__restrict__ A, const void *__restrict__ B,
                                                            const float *__restrict__ C, float *__restrict__ Dout,
                                                            size_t ntiles) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  TPanel &P = reinterpret_cast<TPanel *>(smem_raw)[warp];
  const int rl = (lane >> 2) * TR, cl = (lane & 3) * TCC;
  const int lm = lane & 15, lh = lane >> 4;
  const size_t stride = (size_t)gridDim.x * TWARPS;
  size_t t = (size_t)blockIdx.x * TWARPS + warp;
  if (t >= ntiles) return;  // warp-uniform

  // raw operands and C of the next tile are loaded while this one computes
  auto load_a = [&](size_t u) { return load_row8<FMT>(A, u * 256 + lm * 16 + 8 * lh, true); };
  auto load_b = [&](size_t u) { return load_col8<FMT>(B, u * 256 + (8 * lh) * 16 + lm, 16, true); };
  auto load_c = [&](size_t u, uint32_t(&cv)[TR][TCC]) {
    load_bits<TR, TCC>(C + u * 256 + rl * 16 + cl, 16, C != nullptr, cv);
  };
  Raw8<FMT> ra = load_a(t), rb = load_b(t);
  uint32_t cnext[TR][TCC];
  load_c(t, cnext);
  uint32_t Np[TR][TCC / 2];
  uint32_t V[TR][TCC];
  int32_t(&X)[TR][TCC] = reinterpret_cast<int32_t(&)[TR][TCC]>(V);
  uint32_t dneg0;
  for (;;) {
#pragma unroll
    for (int i = 0; i < TR; i++)
#pragma unroll
      for (int c = 0; c < TCC; c++) V[i][c] = cnext[i][c];
    bool fast = classify_values<TR, TCC>(V, Np, dneg0);
    if (!kFloatAssisted<FMT>) fast = false;
    if (!fast) values_to_state<TR, TCC>(Np, V);
    __syncwarp();  // the previous tile's reads of P are done
    uint32_t sp = store_a8<MODEL, FMT>(P, lm, lh, ra);
    sp |= store_b8<FMT>(P, lm, lh, rb);
    const bool panel_special = __any_sync(0xFFFFFFFFu, sp != 0);
    __syncwarp();
    const size_t next = t + stride;
    if (next < ntiles) {
      ra = load_a(next);
      rb = load_b(next);
      load_c(next, cnext);
    }
    uint32_t D[TR][TCC];
    if constexpr (kFloatAssisted<FMT>) {
      bool to_integer = false;
      if (fast) {
        mma_chunk_fast<MODEL, FMT, TR, TCC>(P, rl, cl, Np, V, dneg0, panel_special, to_integer);
        if (to_integer) values_to_state<TR, TCC>(Np, V);
      } else {
        mma_chunk<MODEL, FMT, TR, TCC>(P, rl, cl, Np, X, dneg0, panel_special);
      }
      if (fast && !to_integer) {
#pragma unroll
        for (int i = 0; i < TR; i++)
#pragma unroll
          for (int c = 0; c < TCC; c++) D[i][c] = V[i][c];
      } else {
        state_to_fp32<TR, TCC>(Np, X, D, ModelT<MODEL>::NAN_BITS);
      }
    } else {
      mma_chunk<MODEL, FMT, TR, TCC>(P, rl, cl, Np, X, dneg0, panel_special);
      state_to_fp32<TR, TCC>(Np, X, D, ModelT<MODEL>::NAN_BITS);
    }
#pragma unroll
    for (int i = 0; i < TR; i++)
      *reinterpret_cast<uint4 *>(Dout + t * 256 + (rl + i) * 16 + cl) = make_uint4(D[i][0], D[i][1], D[i][2], D[i][3]);
    t = next;
    if (t >= ntiles) break;
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
// decoded-operand workspace.  Freed workspace stays in the pool (release
// threshold: unlimited) so that repeated GEMMs reuse it without new
// device allocations; mmaemu_trim_workspace returns it.
std::mutex g_pool_mutex;
cudaMemPool_t g_pool[kMaxDevices] = {};

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
    uint64_t threshold = UINT64_MAX;
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

// Workspace sizes of one GEMM (all batch entries): decoded A and B blobs
// and their flag words.
struct GemmSizes {
  int nrb, ncb, nch;
  size_t a_bytes, b_bytes, fa_bytes, fb_bytes;
};
GemmSizes gemm_sizes(int M, int N, int K, int batch) {
  GemmSizes z;
  z.nrb = (M + mmaemu::GBM - 1) / mmaemu::GBM;
  z.ncb = (N + mmaemu::GBN - 1) / mmaemu::GBN;
  z.nch = K / 16;
  z.a_bytes = (size_t)batch * z.nrb * z.nch * mmaemu::ABLOB;
  z.b_bytes = (size_t)batch * z.ncb * z.nch * mmaemu::BBLOB;
  z.fa_bytes = (size_t)batch * z.nrb * z.nch * sizeof(uint32_t);
  z.fb_bytes = (size_t)batch * z.ncb * z.nch * sizeof(uint32_t);
  return z;
}

// Decode pass for B (p.dB, p.flags_b set) on `stream`.
template <int MODEL, int FMT>
int launch_decode_b(const mmaemu::GemmParams &p, int batch, cudaStream_t stream) {
  const GemmSizes z = gemm_sizes(p.M, p.N, p.K, batch);
  if (cudaMemsetAsync(p.flags_b, 0, z.fb_bytes, stream) != cudaSuccess) return MMAEMU_ECUDA;
  const dim3 gb((z.ncb * mmaemu::GBN + 255) / 256, 2 * z.nch, batch);
  mmaemu::decode_b_kernel<MODEL, FMT><<<gb, 256, 0, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
}

// Decode pass for A and the MMA kernel (B already decoded) on `stream`.
template <int MODEL, int FMT>
int launch_decode_a_gemm(const mmaemu::GemmParams &p, int batch, cudaStream_t stream) {
  const GemmSizes z = gemm_sizes(p.M, p.N, p.K, batch);
  const size_t smem = 2 * sizeof(mmaemu::GPanel);
  auto kern = mmaemu::gemm_kernel<MODEL, FMT>;
  if (cudaMemsetAsync(p.flags_a, 0, z.fa_bytes, stream) != cudaSuccess ||
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MMAEMU_ECUDA;
  const dim3 ga((z.nrb * mmaemu::GBM + 255) / 256, 2 * z.nch, batch);
  mmaemu::decode_a_kernel<MODEL, FMT><<<ga, 256, 0, stream>>>(p);
  kern<<<dim3(z.ncb, z.nrb, batch), mmaemu::GTHREADS, smem, stream>>>(p);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
}

template <int MODEL, int FMT>
int launch_gemm(const mmaemu::GemmParams &p_in, int batch) {
  mmaemu::GemmParams p = p_in;
  const GemmSizes z = gemm_sizes(p.M, p.N, p.K, batch);
  // workspace: decoded blobs and their flags, stream-ordered, released
  // after the GEMM
  unsigned char *ws = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void **>(&ws),
                                       z.a_bytes + z.b_bytes + z.fa_bytes + z.fb_bytes, pool, t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  p.dA = ws;
  p.dB = ws + z.a_bytes;
  p.flags_a = reinterpret_cast<uint32_t *>(ws + z.a_bytes + z.b_bytes);
  p.flags_b = reinterpret_cast<uint32_t *>(ws + z.a_bytes + z.b_bytes + z.fa_bytes);
  p.batch = batch;
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
// row slabs (a multiple of 64 rows) on a copy stream while earlier slabs
// compute, alternately on the caller's stream and a second compute stream
// (so that one slab's last partial wave of blocks overlaps the next slab),
// and each slab's D (and fingerprints) returns on another copy stream as
// soon as that slab is done.
template <int MODEL, int FMT>
int launch_gemm_host(int M, int N, int K, const void *A_h, const void *B_h, const float *C_h, float *D_h,
                     uint32_t *fp_h) {
  constexpr size_t ES = FMT == mmaemu::FMT_E4M3 ? 1 : 2;
  cudaStream_t s_in, s_out, c2;
  int rc = host_streams(s_in, s_out, c2);
  if (rc != MMAEMU_OK) return rc;
  const cudaStream_t cs[2] = {t_stream, c2};
  const int rows_per = ((M + 7) / 8 + mmaemu::GBM - 1) / mmaemu::GBM * mmaemu::GBM;
  const int nslab = (M + rows_per - 1) / rows_per;
  const GemmSizes zs = gemm_sizes(rows_per, N, K, 1), zb = gemm_sizes(M, N, K, 1);
  const size_t a_bytes = (size_t)M * K * ES, b_bytes = (size_t)K * N * ES, cd_bytes = (size_t)M * N * 4;
  const size_t fp_bytes = fp_h ? (size_t)(M / 16) * (N / 16) * 4 : 0;
  // device buffers, each 256-byte aligned inside one pool allocation
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t o_b = up(a_bytes), o_c = o_b + up(b_bytes), o_d = o_c + (C_h ? up(cd_bytes) : 0);
  // two A-blob workspaces and flag arrays, one per compute stream
  const size_t o_fp = o_d + up(cd_bytes), o_wa = o_fp + up(fp_bytes), o_wb = o_wa + 2 * up(zs.a_bytes);
  const size_t o_fa = o_wb + up(zb.b_bytes), o_fb = o_fa + 2 * up(zs.fa_bytes), total = o_fb + up(zb.fb_bytes);
  unsigned char *buf = nullptr;
  cudaMemPool_t pool = workspace_pool();
  if (!pool || cudaMallocFromPoolAsync(reinterpret_cast<void **>(&buf), total, pool, t_stream) != cudaSuccess)
    return MMAEMU_ECUDA;
  unsigned char *dA = buf, *dB = buf + o_b;
  float *dC = C_h ? reinterpret_cast<float *>(buf + o_c) : nullptr;
  float *dD = reinterpret_cast<float *>(buf + o_d);
  uint32_t *dfp = fp_h ? reinterpret_cast<uint32_t *>(buf + o_fp) : nullptr;

  const int nev = 2 + 2 * nslab + 3;
  cudaEvent_t ev[2 + 2 * 8 + 3];
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
    const size_t r0 = (size_t)sl * rows_per, rows = (size_t)(sl + 1 < nslab ? rows_per : M - (int)r0);
    if (!ok(cudaMemcpyAsync(dA + r0 * K * ES, static_cast<const unsigned char *>(A_h) + r0 * K * ES, rows * K * ES,
                            cudaMemcpyHostToDevice, s_in)))
      break;
    if (C_h && !ok(cudaMemcpyAsync(dC + r0 * N, C_h + r0 * N, rows * N * 4, cudaMemcpyHostToDevice, s_in))) break;
    ok(cudaEventRecord(e_in(sl), s_in));
  }
  mmaemu::GemmParams p = row_major_params(M, N, K, dA, dB, dC, dD, dfp);
  p.dB = buf + o_wb;
  p.flags_b = reinterpret_cast<uint32_t *>(buf + o_fb);
  p.batch = 1;
  if (rc == MMAEMU_OK && ok(cudaStreamWaitEvent(t_stream, e_b, 0))) rc = launch_decode_b<MODEL, FMT>(p, 1, t_stream);
  if (rc == MMAEMU_OK && ok(cudaEventRecord(e_bdec, t_stream))) ok(cudaStreamWaitEvent(c2, e_bdec, 0));
  for (int sl = 0; sl < nslab && rc == MMAEMU_OK; sl++) {
    const size_t r0 = (size_t)sl * rows_per;
    const int rows = sl + 1 < nslab ? rows_per : M - (int)r0;
    const cudaStream_t st = cs[sl & 1];
    mmaemu::GemmParams q = p;
    q.M = rows;
    q.A = dA + r0 * K * ES;
    q.C = dC ? dC + r0 * N : nullptr;
    q.D = dD + r0 * N;
    q.fp = dfp ? dfp + (r0 / 16) * (N / 16) : nullptr;
    q.dA = buf + o_wa + (sl & 1) * up(zs.a_bytes);
    q.flags_a = reinterpret_cast<uint32_t *>(buf + o_fa + (sl & 1) * up(zs.fa_bytes));
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
  if ((long long)p.M / mmaemu::GBM >= 65535) return MMAEMU_EINVAL;
  if ((long long)p.K / 16 * 2 > 65535) return MMAEMU_EINVAL;  // decode-pass grid
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
  const size_t smem = mmaemu::TWARPS * sizeof(mmaemu::TPanel);
  auto kern = mmaemu::tiles_kernel<MODEL, FMT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MMAEMU_ECUDA;
  int per_sm = 1;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, mmaemu::TWARPS * 32, smem) != cudaSuccess)
    return MMAEMU_ECUDA;
  if (per_sm < 1) per_sm = 1;
  const size_t want = (ntiles + mmaemu::TWARPS - 1) / mmaemu::TWARPS;
  const size_t cap = (size_t)sms * per_sm;
  const unsigned blocks = (unsigned)(want < cap ? want : cap);
  kern<<<blocks, mmaemu::TWARPS * 32, smem, t_stream>>>(A, B, C, D, ntiles);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
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
  rc = check_device();
  if (rc != MMAEMU_OK) return rc;
#define CALL_HOST(M_, F_) launch_gemm_host<M_, F_>(M, N, K, A, B, C, D, fingerprint_out)
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

int mmaemu_trim_workspace(void) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pool_mutex);
  if (g_pool[dev] && cudaMemPoolTrimTo(g_pool[dev], 0) != cudaSuccess) return MMAEMU_ECUDA;
  return MMAEMU_OK;
}

const char *mmaemu_strerror(int code) {
  switch (code) {
    case MMAEMU_OK: return "ok";
    case MMAEMU_EINVAL: return "invalid argument (enum, model/format pair, pointer, alignment or size)";
    case MMAEMU_ECUDA: return "CUDA runtime error";
    case MMAEMU_ETIMEOUT: return "bounded device wait expired";
    case MMAEMU_EUNSUPPORTED: return "unsupported: the current CUDA device is not an sm_100 (B200-class) GPU, "
                                     "or the probe cannot be built for this format";
    case MMAEMU_ECALLBACK: return "the MMA callback of a probe reported an error";
    default: return "unknown error code";
  }
}

}  // extern "C"

// ===========================================================================
// xorsum that allocates nothing
//
// For callers that cannot allocate device memory at the moment they need a
// fingerprint -- for instance a verification step that runs after the device has run out
// of memory, or inside a process whose device memory is entirely reserved by
// another allocator -- mmaemu_xorsum_noalloc does the same reduction with a
// fixed scratch array that lives in the library image instead of a per-call
// allocation.  Each block of xorsum_partials_kernel folds a fixed span of the
// input into one word of the array; xorsum_finish_kernel folds those words
// into the result slot, which is then copied to the host.
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
// symbol; it is not an address a kernel may be given.
std::atomic<uint32_t *> g_noalloc_scratch_ptr[kMaxDevices];

int noalloc_scratch(uint32_t **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MMAEMU_ECUDA;
  if (dev < 0 || dev >= kMaxDevices) return MMAEMU_EUNSUPPORTED;
  uint32_t *p = g_noalloc_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
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
