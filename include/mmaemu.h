/*
 * libmmaemu -- bit-exact emulation of other GPUs' Tensor Core MMA arithmetic
 * on B200 (sm_100a) CUDA cores.  C ABI, no C++ or framework types.
 *
 * The arithmetic follows the characterise-then-simulate models recovered in
 * "Hawkeye: Reproducing GPU-Level Non-Determinism (MLSys 2026)" (reading
 * notes): Key observations Obs. 1-4, the target-test table, the recovered
 * Ampere FP16 pipeline (Algorithms 12-14, Figure 1) with its Hopper and BF16
 * paragraphs, and Algorithm 10 (BF16 extended range).  The per-tile
 * fingerprint is the xorsum of "How AEGIS Turns Training Redundancy into
 * Evidence" (AEGIS chapter 6, "Redundancy already exists in the training
 * computation").
 *
 * Common rules for every call below:
 *  - All data pointers are DEVICE pointers owned by the caller; the library
 *    never frees, keeps or writes outside them.  Inputs are never modified.
 *  - Matrices are dense and row-major (mmaemu_gemm_strided_batched also
 *    takes transposed and strided layouts).  fp16 and bf16 elements are 2
 *    bytes, e4m3 elements 1 byte (OCP FP8 E4M3: no infinities, S.1111.111 is
 *    NaN), C and D are IEEE fp32.  Every pointer must be 16-byte aligned,
 *    except where a call states otherwise.
 *  - Work is enqueued on the stream set with mmaemu_set_stream for the
 *    calling host thread (default: the legacy default stream) and is
 *    asynchronous unless stated otherwise.  Errors of the kernels themselves
 *    surface at the caller's next synchronisation, or at mmaemu_xorsum.
 *  - Results are fully deterministic: the same inputs give the same bits on
 *    every run, whatever the stream or launch history.
 *  - Return value: MMAEMU_OK (0) or a negative MMAEMU_E* code;
 *    mmaemu_strerror gives a message.
 */
#ifndef MMAEMU_H
#define MMAEMU_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Arithmetic models (Obs. 2 and Obs. 3).
 *  MMAEMU_AMPERE:   24-bit internal significand; two accumulation stages,
 *                   {C, P[1..8]} then {stage-1 result, P[9..16]}.
 *  MMAEMU_LOVELACE: the same model (the pages report Lovelace as identical
 *                   to Ampere; another passage contradicts it).
 *  MMAEMU_HOPPER:   25-bit internal significand; one 17-term stage
 *                   {C, P[1..16]}.
 *  MMAEMU_B200:     not on the pages: B200's own FP16/BF16 tensor-core MMA
 *                   (mma.sync, fp32 accumulate) as measured with the pages'
 *                   target tests (mmaemu_probe.h) -- 26-bit internal
 *                   significand, one 17-term stage, the -133 threshold,
 *                   NaN written as 0x7FFFFFFF.  FP16 and BF16 only.       */
enum { MMAEMU_AMPERE = 0, MMAEMU_HOPPER = 1, MMAEMU_B200 = 2, MMAEMU_LOVELACE = MMAEMU_AMPERE };

/* Input formats.  E4M3 exists only with MMAEMU_HOPPER (FP8 is characterised
 * on Hopper only; Ampere has no FP8 MMA; B200's FP8 MMA follows other rules
 * that the target tests do not resolve).                                    */
enum { MMAEMU_FP16 = 0, MMAEMU_BF16 = 1, MMAEMU_E4M3 = 2 };

/* Return codes. */
#define MMAEMU_OK 0
#define MMAEMU_EINVAL (-1)       /* bad enum or pair, NULL or misaligned pointer, bad size */
#define MMAEMU_ECUDA (-2)        /* a CUDA runtime call or launch failed                    */
#define MMAEMU_ETIMEOUT (-3)     /* a bounded device wait gave up (mmaemu_device_status)   */
#define MMAEMU_EUNSUPPORTED (-4) /* the current device is not an sm_100 GPU                 */
#define MMAEMU_ECALLBACK (-5)    /* a probe's MMA callback failed (mmaemu_probe.h)           */
#define MMAEMU_EBOUNDS (-6)      /* checking build: an index left its buffer (mmaemu_device_status) */

/* Select the CUDA stream (a cudaStream_t passed as void*) that the calling
 * host thread's later calls enqueue on; NULL selects the legacy default
 * stream.  The setting is per host thread.  Never fails: returns MMAEMU_OK. */
int mmaemu_set_stream(void *cuda_stream);

/* Independent tile MMAs: for t < ntiles, D[t] = C[t] + A[t] . B[t] on
 * 16x16x16 tiles, every element following the model's arithmetic (exact
 * unnormalised products, truncating alignment to the group's largest
 * exponent, the model's accumulation stages, toward-zero write-back with
 * overflow to +-Inf) -- Obs. 1-3; recovered pipeline.
 *   A: [ntiles][16][16] in fmt, element (m, k) of tile t at A[t*256 + m*16 + k]
 *   B: [ntiles][16][16] in fmt, element (k, n) at B[t*256 + k*16 + n]
 *   C: [ntiles][16][16] fp32 (m, n), or NULL for +0 everywhere
 *   D: [ntiles][16][16] fp32 (m, n); D may equal C (in place); no other overlap
 * ntiles == 0 is a no-op.  Errors: MMAEMU_EINVAL, MMAEMU_ECUDA,
 * MMAEMU_EUNSUPPORTED; on error nothing is enqueued.                        */
int mmaemu_tiles(int model, int fmt, const void *A, const void *B, const float *C, float *D,
                 size_t ntiles);

/* GEMM implementation note (all GEMM calls): each call first decodes A and
 * B once into panel form, then the MMA kernel copies those panels instead of
 * decoding per output block.  The decoded operands live in a stream-ordered
 * workspace of
 *   batch * K/16 * (ceil(M/64) * 12560 + ceil(N/64) * 10512) bytes
 * (about 379 MB for M = N = K = 4096) taken from a memory pool owned by the
 * library.  By default the pool hands freed workspace back to the device at
 * the next synchronisation of the stream, event or device, so the library
 * holds no device memory between calls; mmaemu_set_workspace_cache(1) makes
 * it keep the memory for the next call instead.  A failed workspace
 * allocation returns MMAEMU_ECUDA before anything is enqueued.            */

/* Large MatMul composed of 16x16x16 tiles (Obs. 4): D = C + A . B where K is
 * walked in 16-wide chunks in ascending order and the fp32 result of each
 * chunk is the C of the next, so every output element is
 *   d_0 = C[m][n];  d_{j+1} = MMA16(A[m][16j..16j+15], B[16j..16j+15][n], d_j).
 *   A: [M][K] in fmt; B: [K][N] in fmt; C, D: [M][N] fp32; C may be NULL (+0)
 *   and may equal D (in place); no other overlap.
 *   M, N, K: positive multiples of 16; M / 64 below 65535; K / 8 at most 65535.
 *   fingerprint_out: NULL, or [(M/16)*(N/16)] uint32 written with the
 *   xorsum (XOR of the 256 fp32 bit patterns) of each 16x16 tile of D, tiles
 *   in row-major tile-grid order -- the AEGIS xorsum fingerprint, fused into
 *   the epilogue.
 *   D may be NULL when fingerprint_out is not: the fingerprints are computed
 *   and nothing of D is written (fingerprint-only mode).
 * Errors: MMAEMU_EINVAL (also for D and fingerprint_out both NULL),
 * MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED; on error nothing is enqueued.          */
int mmaemu_gemm(int model, int fmt, int M, int N, int K, const void *A, const void *B,
                const float *C, float *D, uint32_t *fingerprint_out);

/* Verify mode of mmaemu_gemm: recomputes D = C + A . B exactly as
 * mmaemu_gemm does and compares it, bit for bit, with a claimed result
 * instead of storing it -- the auditor's side of the workflow in the Hawkeye
 * notes ("relation to the verifiable-ML workflow": the simulator as oracle,
 * compared with the MatMul outputs a provider publishes), where any
 * difference means the claimed computation was not the modelled one.
 *   D_claimed: [M][N] fp32, row-major, 16-byte aligned; only read.  Every bit
 *   counts: a NaN with another payload, or -0 for +0, is a mismatch.
 *   mismatch_out: device array of 2 unsigned 64-bit words, overwritten (it
 *   needs no initialisation): [0] = number of mismatching elements, [1] =
 *   smallest row-major index m*N + n among them, or 2^64 - 1 if none.
 *   fingerprint_out: NULL, or the fingerprints of the RECOMPUTED D, as in
 *   mmaemu_gemm.
 * Other arguments and rules as mmaemu_gemm.  Asynchronous: read mismatch_out
 * after the stream has reached this call.  Errors: MMAEMU_EINVAL (also NULL
 * D_claimed or mismatch_out), MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED.           */
int mmaemu_gemm_verify(int model, int fmt, int M, int N, int K, const void *A, const void *B,
                       const float *C, const float *D_claimed, uint32_t *fingerprint_out,
                       unsigned long long *mismatch_out);

/* mmaemu_gemm over other storage layouts and batches of independent
 * problems, each with the same K-chained arithmetic -- for MatMuls as they
 * appear in model layers (the Hawkeye notes' "design trade-offs": real
 * training shapes, batches and layouts have to be mapped onto the 16x16
 * MMA tiles).  For batch entry b (0 <= b < batch), with every stride and
 * leading dimension counted in ELEMENTS:
 *   op(A)[m][k] = A[b*stride_a + m*lda + k]   if trans_a == 0  (lda >= K)
 *               = A[b*stride_a + k*lda + m]   if trans_a == 1  (lda >= M)
 *   op(B)[k][n] = B[b*stride_b + k*ldb + n]   if trans_b == 0  (ldb >= N)
 *               = B[b*stride_b + n*ldb + k]   if trans_b == 1  (ldb >= K)
 *   C[b*stride_c + m*ldc + n] (C may be NULL: +0), D[b*stride_d + m*ldd + n]
 *   fingerprint_out[b*stride_fp + (m/16)*(N/16) + n/16] (may be NULL;
 *   stride_fp >= (M/16)*(N/16) when batch > 1)
 * D may be NULL when fingerprint_out is not (fingerprint-only).  Strides may
 * be 0 for inputs shared by every batch entry (e.g. one B for all); the D
 * and fingerprint regions of different entries must not overlap.
 * Layout rules (MMAEMU_EINVAL otherwise): A and B 16-byte aligned; when A is
 * not transposed lda and stride_a are multiples of 8, and likewise ldb and
 * stride_b when B is transposed (those rows are read as 8-element vectors);
 * C and D 16-byte aligned with ldc, ldd >= N and ldc, ldd, stride_c,
 * stride_d multiples of 4; fingerprint_out 4-byte aligned; strides >= 0;
 * 1 <= batch <= 65535; trans_a, trans_b in {0, 1}; M, N, K as mmaemu_gemm.
 * Errors: MMAEMU_EINVAL, MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED.                 */
int mmaemu_gemm_strided_batched(int model, int fmt, int trans_a, int trans_b, int M, int N, int K,
                                int batch, const void *A, long long lda, long long stride_a,
                                const void *B, long long ldb, long long stride_b, const float *C,
                                long long ldc, long long stride_c, float *D, long long ldd,
                                long long stride_d, uint32_t *fingerprint_out, long long stride_fp);

/* mmaemu_gemm from and to HOST memory, synchronous: A, B, C (C may be NULL)
 * and the results D and fingerprint_out (either may be NULL, not both) are
 * host pointers; layouts and rules as mmaemu_gemm.  The call copies B and
 * decodes it once, then streams A and C to the device in row slabs on a
 * library-owned copy stream while earlier slabs compute, alternately on the
 * selected stream and a library-owned second compute stream, and copies
 * each slab's D and fingerprints back on another copy stream as soon as
 * that slab is done -- the transfers overlap the arithmetic.  The first
 * slab is one wave of GEMM blocks (so a GEMM with fewer blocks than the
 * GPU holds at once runs as one slab), the last is short, at most six.  Page-locked host memory lets the copies run asynchronously;
 * other host memory works too, with the copies no longer overlapped.
 * Device memory comes from the library's workspace pool (see the GEMM
 * implementation note).  Returns after D and the fingerprints are in host
 * memory.  Errors: as mmaemu_gemm; MMAEMU_ECUDA also for a failed copy.  */
int mmaemu_gemm_host(int model, int fmt, int M, int N, int K, const void *A, const void *B,
                     const float *C, float *D, uint32_t *fingerprint_out);

/* mmaemu_tiles from and to HOST memory, synchronous: A, B, C (C may be NULL)
 * and D are host pointers with the layouts of mmaemu_tiles (no alignment
 * rule; D may equal C).  The tiles go in chunks of at least 4096 (at most 8
 * chunks): a chunk's A, B and C are copied to the device on a library-owned
 * copy stream, its tiles run on the selected stream once they have arrived,
 * and its D is copied back on a second copy stream, so that the copies in
 * both directions overlap each other and the arithmetic.  Page-locked host
 * memory lets the copies run asynchronously.  Device memory comes from the
 * library's workspace pool.  Returns after D is in host memory.
 * ntiles == 0 is a no-op.  Errors: as mmaemu_tiles; MMAEMU_ECUDA also for a
 * failed copy.                                                              */
int mmaemu_tiles_host(int model, int fmt, const void *A, const void *B, const float *C, float *D,
                      size_t ntiles);

/* xorsum of n 32-bit words at device pointer D (the AEGIS fingerprint of a
 * whole tensor), written to *out_host.  SYNCHRONOUS: returns after the
 * result is on the host (it waits for the selected stream).  n == 0 gives 0.
 * Uses a few bytes of stream-ordered scratch that it releases before
 * returning.  Errors: MMAEMU_EINVAL (NULL pointer, misaligned D),
 * MMAEMU_ECUDA (also reports an earlier asynchronous kernel fault),
 * MMAEMU_EUNSUPPORTED.                                                      */
int mmaemu_xorsum(const void *D, size_t n, uint32_t *out_host);

/* mmaemu_xorsum for callers that cannot allocate device memory when they
 * need the fingerprint -- e.g. a verification step that must still run after the device
 * has run out of memory, or a process whose device memory is wholly reserved
 * by another allocator.  It has no counterpart on the pages; it computes the
 * same value as mmaemu_xorsum.
 *   Scratch: a fixed array inside the library (64 KiB + 4 bytes per GPU,
 *   held by every GPU that loads the library until the process exits); no
 *   cudaMalloc, cudaFree or other allocating call is made.
 *   Limit: n <= MMAEMU_XORSUM_NOALLOC_MAX_WORDS (2^27 words = 512 MiB);
 *   larger n returns MMAEMU_EINVAL before any device work.
 *   The first call on each device looks up the array's device address (with
 *   that device current) and loads this call's two kernels onto the device;
 *   both need device memory once (CUDA loads code lazily).  So make that
 *   first call while memory is still available -- at start-up, as a
 *   warm-up -- and before any stream capture; later calls need none.
 *   All calls share the one array: calls whose work overlaps on the GPU (from
 *   different streams or host threads) race and may return wrong values, so
 *   serialise them.  Nothing in the array needs clearing between calls.
 *   SYNCHRONOUS like mmaemu_xorsum.  Errors: MMAEMU_EINVAL, MMAEMU_ECUDA,
 *   MMAEMU_EUNSUPPORTED.                                                    */
#define MMAEMU_XORSUM_NOALLOC_MAX_WORDS ((size_t)1 << 27)
int mmaemu_xorsum_noalloc(const void *D, size_t n, uint32_t *out_host);

/* Keep (enable != 0) or stop keeping (enable == 0) the GEMM workspace on
 * the current device between calls (see the GEMM implementation note); off
 * by default.  Turning it off also hands back what is held.  It only trades
 * device memory for the cost of a stream-ordered allocation per call.
 * Errors: MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED.                               */
int mmaemu_set_workspace_cache(int enable);

/* Bytes of device memory the workspace pool of the current device holds at
 * this moment (0 before the first GEMM on it).  *bytes must not be NULL.
 * Errors: MMAEMU_EINVAL, MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED.                */
int mmaemu_workspace_reserved(size_t *bytes);

/* Return the current device's unused GEMM workspace (see above) to the
 * device.  Workspace still in use by enqueued GEMMs is kept.  Errors:
 * MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED.                                       */
int mmaemu_trim_workspace(void);

/* The device status word of the current device: bits the kernels set since
 * it was last cleared.  Bit 0: a bounded wait gave up (a GEMM block whose
 * panel copy did not arrive within its bound stops, records this and
 * leaves its outputs unwritten).  Bit 1: in the bounds-checking build
 * (mmaemu_bounds_checking() == 1) an index fell outside its buffer and the
 * access was skipped.  SYNCHRONOUS: waits for the selected stream first.
 * clear != 0 resets the word.  bits_out may be NULL.  Returns MMAEMU_EBOUNDS
 * if bit 1 is set, else MMAEMU_ETIMEOUT if bit 0 is set, else MMAEMU_OK;
 * MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED on failure.                            */
int mmaemu_device_status(int clear, uint32_t *bits_out);

/* Exercises the bounded-wait path: launches one block whose wait can never
 * complete (nothing arrives) with a bound of `spins` tries, which then
 * records a timeout in the device status word exactly as a GEMM block
 * would.  *completed_out (may be NULL) receives whether the wait completed
 * (it does not).  SYNCHRONOUS.  Errors: MMAEMU_ECUDA, MMAEMU_EUNSUPPORTED. */
int mmaemu_selftest_wait_timeout(unsigned spins, int *completed_out);

/* 1 for the bounds-checking build of the library, 0 otherwise. */
int mmaemu_bounds_checking(void);

/* Static message for a return code. */
const char *mmaemu_strerror(int code);

#ifdef __cplusplus
}
#endif

#endif /* MMAEMU_H */
