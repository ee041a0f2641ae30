// Issue-rate probes for the instruction classes the emulation kernels use,
// so that their rooflines rest on measured per-SM rates rather than on unit
// counts.  Each thread runs NCHAIN independent dependency chains of one
// instruction; every block reads the SM cycle counter around its loop, and
// the rate is (threads x iterations x NCHAIN) / cycles per SM, i.e. lanes
// (thread-instructions) per SM per clock, independent of the clock speed.
//
// C ABI (libmmaemu_peaks.so):
//   int mmaemu_peak_rate(int op, int iters, double *lanes_per_sm_clk,
//                        double *seconds);
//     op: one of the PEAK_* codes below; iters: loop iterations per thread
//     (each runs NCHAIN instructions, or NCHAIN pairs for the paired codes,
//     whose rate counts pairs); one block of 1024 threads per SM.
//     Synchronous; returns 0, or -2 on a CUDA error, -1 on a bad op.
#include <cuda_runtime.h>
#include <stdint.h>

namespace {

enum : int {
  PEAK_DFMA = 0,    // fma.rz.f64
  PEAK_DADD = 1,    // add.rn.f64
  PEAK_ADDMIN2 = 2, // add.s16x2 then min.s16x2 (fused by ptxas into one packed add-and-min)
  PEAK_LOP3 = 3,    // lop3.b32
  PEAK_IMAD = 4,    // mad.lo.u32
  PEAK_IADD = 5,    // add.u32
  PEAK_POPC = 6,    // popc.b32 (with an xor to keep the chain moving: 2 instructions)
  PEAK_PRMT = 7,    // prmt.b32
  PEAK_IMNMX = 8,   // min.s32
  PEAK_FFMA = 9,    // fma.rn.f32
  // pairs of instructions on independent chains: whether two pipes overlap
  PEAK_DFMA_LOP3 = 10,
  PEAK_DFMA_IMAD = 11,
  PEAK_DFMA_FFMA = 12,
  PEAK_DFMA_ADDMIN2 = 13,
  PEAK_LOP3_IMAD = 14,
  PEAK_LOP3_FFMA = 15,
  PEAK_COUNT = 16
};
constexpr int NCHAIN = 8, THREADS = 1024;

template <int OP>
__device__ __forceinline__ void step(uint32_t (&u)[NCHAIN], double (&d)[NCHAIN], float (&f)[NCHAIN], uint32_t k) {
#pragma unroll
  for (int i = 0; i < NCHAIN; i++) {
    if constexpr (OP == PEAK_DFMA) {
      asm volatile("fma.rz.f64 %0, %0, %1, %2;" : "+d"(d[i]) : "d"(1.0000001), "d"(0.5));
    } else if constexpr (OP == PEAK_DADD) {
      asm volatile("add.rn.f64 %0, %0, %1;" : "+d"(d[i]) : "d"(0.25));
    } else if constexpr (OP == PEAK_ADDMIN2) {
      uint32_t t;
      asm volatile("add.s16x2 %1, %0, %2;\n\tmin.s16x2 %0, %1, %3;" : "+r"(u[i]), "=r"(t) : "r"(k), "r"(0x70007000u));
    } else if constexpr (OP == PEAK_LOP3) {
      asm volatile("lop3.b32 %0, %0, %1, %2, 0x96;" : "+r"(u[i]) : "r"(k), "r"(0x5A5A5A5Au));
    } else if constexpr (OP == PEAK_IMAD) {
      asm volatile("mad.lo.u32 %0, %0, %1, %2;" : "+r"(u[i]) : "r"(k | 1u), "r"(0x9E3779B9u));
    } else if constexpr (OP == PEAK_IADD) {
      asm volatile("add.u32 %0, %0, %1;" : "+r"(u[i]) : "r"(k));
    } else if constexpr (OP == PEAK_POPC) {
      asm volatile("{\n\t.reg .b32 t;\n\txor.b32 t, %0, %1;\n\tpopc.b32 %0, t;\n\t}" : "+r"(u[i]) : "r"(k));
    } else if constexpr (OP == PEAK_PRMT) {
      asm volatile("prmt.b32 %0, %0, %1, 0x2107;" : "+r"(u[i]) : "r"(k));
    } else if constexpr (OP == PEAK_IMNMX) {
      asm volatile("min.s32 %0, %0, %1;" : "+r"(u[i]) : "r"(k));
    } else {
      asm volatile("fma.rn.f32 %0, %0, %1, %2;" : "+f"(f[i]) : "f"(1.0000001f), "f"(0.5f));
    }
  }
}

// Chains of two kinds of instruction (OP2 < 0: one kind) in separate
// registers; with two kinds each iteration runs NCHAIN of each and the rate
// counts pairs: the slower kind's rate when the two pipes work at the same
// time, the harmonic combination when they take turns.
template <int OP1, int OP2>
__global__ void __launch_bounds__(THREADS, 1) rate_kernel(int iters, unsigned long long *cycles, uint32_t *sink) {
  uint32_t u[NCHAIN], u2[NCHAIN];
  double d[NCHAIN], d2[NCHAIN];
  float f[NCHAIN], f2[NCHAIN];
  const uint32_t k = threadIdx.x * 2654435761u + blockIdx.x;
#pragma unroll
  for (int i = 0; i < NCHAIN; i++) {
    u[i] = k ^ (0x1234567u * (i + 1));
    u2[i] = u[i] ^ 0x5A5A5A5Au;
    d[i] = 1.0 + i;
    d2[i] = 2.0 + i;
    f[i] = 1.0f + i;
    f2[i] = 2.0f + i;
  }
  __syncthreads();
  const unsigned long long t0 = clock64();
#pragma unroll 1
  for (int it = 0; it < iters; it++) {
    step<OP1>(u, d, f, k + (uint32_t)it);
    if constexpr (OP2 >= 0) step<OP2>(u2, d2, f2, k + (uint32_t)it);
  }
  __syncthreads();
  const unsigned long long t1 = clock64();
  uint32_t x = 0;
#pragma unroll
  for (int i = 0; i < NCHAIN; i++)
    x ^= u[i] ^ u2[i] ^ (uint32_t)__double2loint(d[i]) ^ (uint32_t)__double2loint(d2[i]) ^ __float_as_uint(f[i]) ^
         __float_as_uint(f2[i]);
  if (x == 0x12345678u) sink[threadIdx.x] = x;  // keeps the chains alive
  if (threadIdx.x == 0) cycles[blockIdx.x] = t1 - t0;
}

template <int OP1, int OP2 = -1>
int run(int iters, int sms, unsigned long long *cyc, uint32_t *sink, float *ms) {
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess || cudaEventCreate(&e1) != cudaSuccess) return -2;
  rate_kernel<OP1, OP2><<<sms, THREADS>>>(8, cyc, sink);  // warm-up
  cudaEventRecord(e0);
  rate_kernel<OP1, OP2><<<sms, THREADS>>>(iters, cyc, sink);
  cudaEventRecord(e1);
  const int rc = (cudaGetLastError() == cudaSuccess && cudaEventSynchronize(e1) == cudaSuccess) ? 0 : -2;
  if (rc == 0) cudaEventElapsedTime(ms, e0, e1);
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  return rc;
}

}  // namespace

extern "C" int mmaemu_peak_rate(int op, int iters, double *lanes_per_sm_clk, double *seconds) {
  if (op < 0 || op >= PEAK_COUNT || iters < 1 || !lanes_per_sm_clk) return -1;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return -2;
  unsigned long long *cyc = nullptr;
  uint32_t *sink = nullptr;
  if (cudaMalloc(&cyc, sizeof(unsigned long long) * sms) != cudaSuccess) return -2;
  if (cudaMalloc(&sink, sizeof(uint32_t) * THREADS) != cudaSuccess) {
    cudaFree(cyc);
    return -2;
  }
  float ms = 0.f;
  int rc;
  switch (op) {
    case PEAK_DFMA: rc = run<PEAK_DFMA>(iters, sms, cyc, sink, &ms); break;
    case PEAK_DADD: rc = run<PEAK_DADD>(iters, sms, cyc, sink, &ms); break;
    case PEAK_ADDMIN2: rc = run<PEAK_ADDMIN2>(iters, sms, cyc, sink, &ms); break;
    case PEAK_LOP3: rc = run<PEAK_LOP3>(iters, sms, cyc, sink, &ms); break;
    case PEAK_IMAD: rc = run<PEAK_IMAD>(iters, sms, cyc, sink, &ms); break;
    case PEAK_IADD: rc = run<PEAK_IADD>(iters, sms, cyc, sink, &ms); break;
    case PEAK_POPC: rc = run<PEAK_POPC>(iters, sms, cyc, sink, &ms); break;
    case PEAK_PRMT: rc = run<PEAK_PRMT>(iters, sms, cyc, sink, &ms); break;
    case PEAK_IMNMX: rc = run<PEAK_IMNMX>(iters, sms, cyc, sink, &ms); break;
    case PEAK_FFMA: rc = run<PEAK_FFMA>(iters, sms, cyc, sink, &ms); break;
    case PEAK_DFMA_LOP3: rc = run<PEAK_DFMA, PEAK_LOP3>(iters, sms, cyc, sink, &ms); break;
    case PEAK_DFMA_IMAD: rc = run<PEAK_DFMA, PEAK_IMAD>(iters, sms, cyc, sink, &ms); break;
    case PEAK_DFMA_FFMA: rc = run<PEAK_DFMA, PEAK_FFMA>(iters, sms, cyc, sink, &ms); break;
    case PEAK_DFMA_ADDMIN2: rc = run<PEAK_DFMA, PEAK_ADDMIN2>(iters, sms, cyc, sink, &ms); break;
    case PEAK_LOP3_IMAD: rc = run<PEAK_LOP3, PEAK_IMAD>(iters, sms, cyc, sink, &ms); break;
    default: rc = run<PEAK_LOP3, PEAK_FFMA>(iters, sms, cyc, sink, &ms); break;
  }
  if (rc == 0) {
    unsigned long long host[1024];
    const int n = sms < 1024 ? sms : 1024;
    if (cudaMemcpy(host, cyc, sizeof(unsigned long long) * n, cudaMemcpyDeviceToHost) != cudaSuccess) {
      rc = -2;
    } else {
      double sum = 0;
      for (int i = 0; i < n; i++) sum += (double)host[i];
      const double mean_cycles = sum / n;
      *lanes_per_sm_clk = (double)THREADS * iters * NCHAIN / mean_cycles;
      if (seconds) *seconds = ms / 1e3;
    }
  }
  cudaFree(cyc);
  cudaFree(sink);
  return rc;
}
