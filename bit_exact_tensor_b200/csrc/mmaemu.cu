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
// arithmetic being emulated, so everything is exact integer work.
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

#include "mmaemu.h"
#include "mmaemu_core.cuh"

namespace mmaemu {

// ---------------------------------------------------------------------------
// decoded operand panels in shared memory, [k][row] for A and [k][col] for B
// ---------------------------------------------------------------------------
template <int BM, int BN>
struct __align__(16) Panel {
  uint32_t aM[16][BM];  // ma << (F - 2p): one IMAD with mb gives the term magnitude
  int32_t aN[16][BM];   // -ea (ZSENT / NINF / NNAN markers)
  uint32_t aS[16][BM];  // sign masks
  uint32_t bM[16][BN];
  int32_t bN[16][BN];
  uint32_t bS[16][BN];
  uint16_t sa16[BM];  // bit k = sign of a[m][k]
  uint16_t sb16[BN];  // bit k = sign of b[k][n]
};

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

// One accumulation group over k in [K0, K0 + KN): returns S (signed sum of
// the aligned terms, carry term included) and nmin (= -e_max) per output.
// The carry term is (nc, Xc) with Xc in ones' complement form.
template <int FMT, int F, int K0, int KN, int R, int CC, int BM, int BN>
__device__ __forceinline__ void group_sum(const Panel<BM, BN> &P, int rl, int cl,
                                          const int32_t (&nc)[R][CC], const int32_t (&Xc)[R][CC],
                                          int32_t (&nmin)[R][CC], int32_t (&S)[R][CC]) {
  // pass 1: the group's max exponent (min of the negated exponents)
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) nmin[r][c] = nc[r][c];
#pragma unroll 1
  for (int k = K0; k < K0 + KN; k++) {
    int32_t an[R], bn[CC];
    lds_vec<R>(&P.aN[k][rl], an);
    lds_vec<CC>(&P.bN[k][cl], bn);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) nmin[r][c] = min(nmin[r][c], an[r] + bn[c]);
  }
  if constexpr (kNeedsFloor<FMT>) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) nmin[r][c] = min(nmin[r][c], NFLOOR);
  }
  // pass 2: align (truncate) and add; the carry first
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++)
      S[r][c] = shr_s32(Xc[r][c], (uint32_t)(nc[r][c] - nmin[r][c])) + (int32_t)((uint32_t)Xc[r][c] >> 31);
#pragma unroll 1
  for (int k = K0; k < K0 + KN; k++) {
    uint32_t am[R], as[R], bm[CC], bs[CC];
    int32_t an[R], bn[CC];
    lds_vec<R>(&P.aM[k][rl], am);
    lds_vec<R>(&P.aN[k][rl], an);
    lds_vec<R>(&P.aS[k][rl], as);
    lds_vec<CC>(&P.bM[k][cl], bm);
    lds_vec<CC>(&P.bN[k][cl], bn);
    lds_vec<CC>(&P.bS[k][cl], bs);
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const uint32_t T = shr_u32(am[r] * bm[c], (uint32_t)(an[r] + bn[c] - nmin[r][c]));
        S[r][c] += (int32_t)(T ^ as[r] ^ bs[c]);
      }
  }
  // ones' complement correction: + number of negative products in the group
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t neg = ((uint32_t)P.sa16[rl + r] ^ (uint32_t)P.sb16[cl + c]) >> K0;
      S[r][c] += __popc(neg & ((1u << KN) - 1u));
    }
}

// One 16-deep K chunk for an R x CC block of outputs at panel row rl, col cl.
// D holds the fp32 accumulator input on entry and the result on exit.
template <int MODEL, int FMT, int R, int CC, int BM, int BN>
__device__ __forceinline__ void mma_chunk(const Panel<BM, BN> &P, int rl, int cl, uint32_t (&D)[R][CC],
                                          bool panel_special) {
  constexpr int F = ModelT<MODEL>::F;
  static_assert(R * CC <= 32, "per-output bit masks hold 32 outputs");
  uint32_t c_negzero = 0, c_nan = 0, c_infp = 0, c_infn = 0;
  int32_t nc[R][CC], Xc[R][CC], nmin[R][CC], S[R][CC];
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      const uint32_t x = D[r][c], bit = 1u << (r * CC + c);
      c_negzero |= (x == 0x80000000u) ? bit : 0u;
      const bool sp = ((x >> 23) & 0xFFu) == 0xFFu;
      c_nan |= (sp && (x & 0x7FFFFFu)) ? bit : 0u;
      c_infp |= (x == 0x7F800000u) ? bit : 0u;
      c_infn |= (x == 0xFF800000u) ? bit : 0u;
      c_term<F>(x, nc[r][c], Xc[r][c]);
    }

  if constexpr (MODEL == MODEL_AMPERE) {
    // stage 1: {C, P[1..8]}
    group_sum<FMT, F, 0, 8, R, CC>(P, rl, cl, nc, Xc, nmin, S);
    // hand-over: the stage-1 sum normalised to 24 bits (truncated), exponent
    // unbounded (BF16 extended range); a zero sum contributes no term
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const int32_t s = S[r][c];
        const uint32_t mag = (uint32_t)(s < 0 ? -s : s);
        const uint32_t z = __clz(mag);
        const uint32_t M = shl_u32(mag, z) >> 8;
        nc[r][c] = s ? nmin[r][c] - 8 + (int32_t)z : ZSENT;
        Xc[r][c] = (int32_t)(M ^ (uint32_t)(s >> 31));
      }
    // stage 2: {S1, P[9..16]}
    group_sum<FMT, F, 8, 8, R, CC>(P, rl, cl, nc, Xc, nmin, S);
  } else {
    // one stage: {C, P[1..16]}
    group_sum<FMT, F, 0, 16, R, CC>(P, rl, cl, nc, Xc, nmin, S);
  }

  // toward-zero write-back
  uint32_t rare = 0;
#pragma unroll
  for (int r = 0; r < R; r++)
#pragma unroll
    for (int c = 0; c < CC; c++) {
      uint32_t rr;
      D[r][c] = cast_normal<F>(S[r][c], nmin[r][c], rr);
      rare |= rr << (r * CC + c);
    }
  if (rare) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const uint32_t bit = 1u << (r * CC + c);
        if (!(rare & bit)) continue;
        if (S[r][c] != 0) {
          D[r][c] = cast_out_of_range<F>(S[r][c], nmin[r][c]);
        } else {
          // zero-sign rule: -0 only when C and all 16 products are -0
          bool neg = (c_negzero & bit) != 0;
          for (int k = 0; k < 16 && neg; k++) {
            const bool zero = P.aN[k][rl + r] == ZSENT || P.bN[k][cl + c] == ZSENT;
            neg = zero && ((P.aS[k][rl + r] ^ P.bS[k][cl + c]) != 0u);
          }
          D[r][c] = neg ? 0x80000000u : 0u;
        }
      }
  }

  // special values: NaN anywhere or Inf x 0 -> NaN; Inf of one sign -> that
  // Inf; both signs -> NaN
  if (panel_special || (c_nan | c_infp | c_infn)) {
#pragma unroll
    for (int r = 0; r < R; r++)
#pragma unroll
      for (int c = 0; c < CC; c++) {
        const uint32_t bit = 1u << (r * CC + c);
        bool nan = (c_nan & bit) != 0, ip = (c_infp & bit) != 0, in = (c_infn & bit) != 0;
        if (panel_special) {
          for (int k = 0; k < 16; k++) {
            const int32_t an = P.aN[k][rl + r], bn = P.bN[k][cl + c];
            if (an == NNAN || bn == NNAN) {
              nan = true;
            } else if (an == NINF || bn == NINF) {
              if (an == ZSENT || bn == ZSENT) nan = true;
              else if (P.aS[k][rl + r] ^ P.bS[k][cl + c]) in = true;
              else ip = true;
            }
          }
        }
        if (nan || (ip && in)) D[r][c] = 0x7FC00000u;
        else if (ip) D[r][c] = 0x7F800000u;
        else if (in) D[r][c] = 0xFF800000u;
      }
  }
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

// Decode 8 k-consecutive elements of A row m (k = 8h .. 8h+7) into the panel.
template <int MODEL, int FMT, int BM, int BN>
__device__ __forceinline__ uint32_t store_a8(Panel<BM, BN> &P, int m, int h, const Raw8<FMT> &raw) {
  constexpr int SH = ModelT<MODEL>::F - 2 * FmtT<FMT>::P;
  uint32_t signs = 0, special = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const Dec d = decode<FMT>(raw.get(i));
    P.aM[8 * h + i][m] = d.m << SH;
    P.aN[8 * h + i][m] = d.n;
    P.aS[8 * h + i][m] = d.s;
    signs |= (d.s & 1u) << i;
    special |= d.special;
  }
  reinterpret_cast<uint8_t *>(P.sa16)[2 * m + h] = (uint8_t)signs;
  return special;
}

template <int FMT, int BM, int BN>
__device__ __forceinline__ uint32_t store_b8(Panel<BM, BN> &P, int n, int h, const Raw8<FMT> &raw) {
  uint32_t signs = 0, special = 0;
#pragma unroll
  for (int i = 0; i < 8; i++) {
    const Dec d = decode<FMT>(raw.get(i));
    P.bM[8 * h + i][n] = d.m;
    P.bN[8 * h + i][n] = d.n;
    P.bS[8 * h + i][n] = d.s;
    signs |= (d.s & 1u) << i;
    special |= d.special;
  }
  reinterpret_cast<uint8_t *>(P.sb16)[2 * n + h] = (uint8_t)signs;
  return special;
}

// ---------------------------------------------------------------------------
// GEMM
// ---------------------------------------------------------------------------
constexpr int GBM = 64, GBN = 128, GTHREADS = 256;
using GPanel = Panel<GBM, GBN>;

template <int MODEL, int FMT>
__global__ void __launch_bounds__(GTHREADS) gemm_kernel(const void *__restrict__ A, const void *__restrict__ B,
                                                        const float *__restrict__ C, float *__restrict__ Dout,
                                                        uint32_t *__restrict__ fp, int M, int N, int K) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  GPanel *panels = reinterpret_cast<GPanel *>(smem_raw);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row0 = blockIdx.y * GBM, col0 = blockIdx.x * GBN;
  // this thread's 4 x 8 outputs
  const int rl = (warp >> 2) * 32 + (lane >> 2) * 4;
  const int cl = (warp & 3) * 32 + (lane & 3) * 8;
  const bool out_valid = (row0 + rl < M) && (col0 + cl < N);

  // loader roles: A row am / half ah (threads < 128); B column bn / half bh
  const int am = tid & (GBM - 1), ah = (tid >> 6) & 1;
  const bool a_loader = tid < 2 * GBM;
  const bool a_valid = a_loader && (row0 + am < M);
  const int bn = tid & (GBN - 1), bh = tid >> 7;
  const bool b_valid = col0 + bn < N;

  const int nchunks = K / 16;
  Raw8<FMT> ra, rb;
  auto load_chunk = [&](int j) {
    const int k0 = 16 * j;
    ra = load_row8<FMT>(A, (size_t)(row0 + am) * K + k0 + 8 * ah, a_valid);
    rb = load_col8<FMT>(B, (size_t)(k0 + 8 * bh) * N + col0 + bn, (size_t)N, b_valid);
  };
  auto store_chunk = [&](GPanel &P) -> uint32_t {
    uint32_t sp = 0;
    if (a_loader) sp |= store_a8<MODEL, FMT>(P, am, ah, ra);
    sp |= store_b8<FMT>(P, bn, bh, rb);
    return sp;
  };

  // accumulator input
  uint32_t D[4][8];
#pragma unroll
  for (int i = 0; i < 4; i++) {
    if (C != nullptr && out_valid) {
      const uint4 *src = reinterpret_cast<const uint4 *>(C + (size_t)(row0 + rl + i) * N + col0 + cl);
      const uint4 a = src[0], b = src[1];
      D[i][0] = a.x; D[i][1] = a.y; D[i][2] = a.z; D[i][3] = a.w;
      D[i][4] = b.x; D[i][5] = b.y; D[i][6] = b.z; D[i][7] = b.w;
    } else {
#pragma unroll
      for (int j = 0; j < 8; j++) D[i][j] = 0u;
    }
  }

  load_chunk(0);
  bool panel_special = __syncthreads_or(store_chunk(panels[0])) != 0;
  for (int j = 0; j < nchunks; j++) {
    if (j + 1 < nchunks) load_chunk(j + 1);
    mma_chunk<MODEL, FMT, 4, 8>(panels[j & 1], rl, cl, D, panel_special);
    if (j + 1 < nchunks) panel_special = __syncthreads_or(store_chunk(panels[(j + 1) & 1])) != 0;
  }

  // epilogue: store D and the per-16x16-tile xorsum
  if (out_valid) {
#pragma unroll
    for (int i = 0; i < 4; i++) {
      uint4 *dst = reinterpret_cast<uint4 *>(Dout + (size_t)(row0 + rl + i) * N + col0 + cl);
      dst[0] = make_uint4(D[i][0], D[i][1], D[i][2], D[i][3]);
      dst[1] = make_uint4(D[i][4], D[i][5], D[i][6], D[i][7]);
    }
  }
  if (fp != nullptr) {
    uint32_t x = 0;
#pragma unroll
    for (int i = 0; i < 4; i++)
#pragma unroll
      for (int j = 0; j < 8; j++) x ^= D[i][j];
    // the 8 lanes sharing a 16x16 tile differ in lane bits 0, 2, 3
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 1);
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 4);
    x ^= __shfl_xor_sync(0xFFFFFFFFu, x, 8);
    if (out_valid && (lane & 0xD) == 0) {
      const int tr = (row0 + rl) >> 4, tc = (col0 + cl) >> 4;
      fp[(size_t)tr * (N >> 4) + tc] = x;
    }
  }
}

// ---------------------------------------------------------------------------
// independent tiles: one warp per 16x16x16 tile, each lane 2 x 4 outputs
// ---------------------------------------------------------------------------
constexpr int TWARPS = 8;
using TPanel = Panel<16, 16>;

template <int MODEL, int FMT>
__global__ void __launch_bounds__(TWARPS * 32) tiles_kernel(const void *__restrict__ A, const void *__restrict__ B,
                                                            const float *__restrict__ C, float *__restrict__ Dout,
                                                            size_t ntiles) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  TPanel &P = reinterpret_cast<TPanel *>(smem_raw)[warp];
  const int rl = (lane >> 2) * 2, cl = (lane & 3) * 4;
  const int lm = lane & 15, lh = lane >> 4;
  for (size_t t = (size_t)blockIdx.x * TWARPS + warp; t < ntiles; t += (size_t)gridDim.x * TWARPS) {
    const Raw8<FMT> ra = load_row8<FMT>(A, t * 256 + lm * 16 + 8 * lh, true);
    const Raw8<FMT> rb = load_col8<FMT>(B, t * 256 + (8 * lh) * 16 + lm, 16, true);
    uint32_t D[2][4];
#pragma unroll
    for (int i = 0; i < 2; i++) {
      if (C != nullptr) {
        const uint4 v = *reinterpret_cast<const uint4 *>(C + t * 256 + (rl + i) * 16 + cl);
        D[i][0] = v.x; D[i][1] = v.y; D[i][2] = v.z; D[i][3] = v.w;
      } else {
        D[i][0] = D[i][1] = D[i][2] = D[i][3] = 0u;
      }
    }
    __syncwarp();  // the previous tile's reads of P are done
    uint32_t sp = store_a8<MODEL, FMT>(P, lm, lh, ra);
    sp |= store_b8<FMT>(P, lm, lh, rb);
    const bool panel_special = __any_sync(0xFFFFFFFFu, sp != 0);
    __syncwarp();
    mma_chunk<MODEL, FMT, 2, 4>(P, rl, cl, D, panel_special);
#pragma unroll
    for (int i = 0; i < 2; i++)
      *reinterpret_cast<uint4 *>(Dout + t * 256 + (rl + i) * 16 + cl) = make_uint4(D[i][0], D[i][1], D[i][2], D[i][3]);
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

bool valid_pair(int model, int fmt) {
  if (model != MMAEMU_AMPERE && model != MMAEMU_HOPPER) return false;
  if (fmt != MMAEMU_FP16 && fmt != MMAEMU_BF16 && fmt != MMAEMU_E4M3) return false;
  return !(model == MMAEMU_AMPERE && fmt == MMAEMU_E4M3);
}

template <int MODEL, int FMT>
int launch_gemm(int M, int N, int K, const void *A, const void *B, const float *C, float *D, uint32_t *fp) {
  const size_t smem = 2 * sizeof(mmaemu::GPanel);
  auto kern = mmaemu::gemm_kernel<MODEL, FMT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MMAEMU_ECUDA;
  dim3 grid((N + mmaemu::GBN - 1) / mmaemu::GBN, (M + mmaemu::GBM - 1) / mmaemu::GBM);
  kern<<<grid, mmaemu::GTHREADS, smem, t_stream>>>(A, B, C, D, fp, M, N, K);
  return cudaGetLastError() == cudaSuccess ? MMAEMU_OK : MMAEMU_ECUDA;
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

#define MMAEMU_DISPATCH(model, fmt, CALL)                                               \
  do {                                                                                  \
    if (model == MMAEMU_AMPERE && fmt == MMAEMU_FP16) return CALL(0, 0);                \
    if (model == MMAEMU_AMPERE && fmt == MMAEMU_BF16) return CALL(0, 1);                \
    if (model == MMAEMU_HOPPER && fmt == MMAEMU_FP16) return CALL(1, 0);                \
    if (model == MMAEMU_HOPPER && fmt == MMAEMU_BF16) return CALL(1, 1);                \
    if (model == MMAEMU_HOPPER && fmt == MMAEMU_E4M3) return CALL(1, 2);                \
    return MMAEMU_EINVAL;                                                               \
  } while (0)

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

int mmaemu_gemm(int model, int fmt, int M, int N, int K, const void *A, const void *B, const float *C, float *D,
                uint32_t *fingerprint_out) {
  if (!valid_pair(model, fmt)) return MMAEMU_EINVAL;
  if (M <= 0 || N <= 0 || K <= 0 || (M & 15) || (N & 15) || (K & 15)) return MMAEMU_EINVAL;
  if ((int64_t)M * K >= ((int64_t)1 << 31) || (int64_t)K * N >= ((int64_t)1 << 31) ||
      (int64_t)M * N >= ((int64_t)1 << 31))
    return MMAEMU_EINVAL;
  if (!A || !B || !D) return MMAEMU_EINVAL;
  if (!aligned16(A) || !aligned16(B) || !aligned16(D) || (C && !aligned16(C)) ||
      (fingerprint_out && !aligned16(fingerprint_out)))
    return MMAEMU_EINVAL;
  const int rc = check_device();
  if (rc != MMAEMU_OK) return rc;
#define CALL_GEMM(M_, F_) launch_gemm<M_, F_>(M, N, K, A, B, C, D, fingerprint_out)
  MMAEMU_DISPATCH(model, fmt, CALL_GEMM);
#undef CALL_GEMM
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

const char *mmaemu_strerror(int code) {
  switch (code) {
    case MMAEMU_OK: return "ok";
    case MMAEMU_EINVAL: return "invalid argument (enum, model/format pair, pointer, alignment or size)";
    case MMAEMU_ECUDA: return "CUDA runtime error";
    case MMAEMU_ETIMEOUT: return "bounded device wait expired";
    case MMAEMU_EUNSUPPORTED: return "the current CUDA device is not an sm_100 (B200-class) GPU";
    default: return "unknown error code";
  }
}

}  // extern "C"

// ===========================================================================
// xorsum that allocates nothing
//
// For callers that cannot allocate device memory at the moment they need a
// fingerprint -- for instance a checker that runs after the device has run out
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
