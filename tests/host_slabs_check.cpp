// Properties of mmaemu_gemm_host's row slabs (host_slabs.h) over many GEMM
// shapes and GPU sizes.  Prints "<violations> <cases>" and, for the shapes
// given as M N SMS triples on the command line, the boundaries.
#include <cstdio>
#include <cstdlib>

#include "host_slabs.h"

using mmaemu_host::host_slabs;
using mmaemu_host::kHostMaxSlabs;
using mmaemu_host::kHostMidSlabs;
using mmaemu_host::kHostTailDiv;

constexpr int TR = 64, TC = 64, PER_SM = 4;  // the GEMM's tiles and tiles resident per SM

static long check(int M, int N, int sms) {
  int r0[kHostMaxSlabs + 2];
  const long long wave = (long long)sms * PER_SM;
  const int n = host_slabs(M, N, TR, TC, wave, r0);
  const int nb = (M + TR - 1) / TR, cb = (N + TC - 1) / TC;
  long bad = 0;
  if (n < 1 || n > kHostMaxSlabs || r0[0] != 0 || r0[n] != M) return 1;
  for (int i = 0; i < n; i++) {
    if (r0[i + 1] <= r0[i]) bad++;
    if (i + 1 < n && r0[i + 1] % TR) bad++;
  }
  // the first slab: one wave of tiles, the fewest row blocks that hold it
  const int head = (r0[1] + TR - 1) / TR;
  if (r0[1] != M && (long long)head * cb < wave) bad++;
  if (head > 1 && (long long)(head - 1) * cb >= wave) bad++;
  if (n == 1) return bad + ((long long)nb * cb > wave && nb > head);
  // the last slab: nb / kHostTailDiv row blocks (at least one)
  const int tail_blocks = (r0[n] - r0[n - 1] + TR - 1) / TR;
  const int want_tail = nb / kHostTailDiv > 1 ? nb / kHostTailDiv : 1;
  if (tail_blocks != want_tail && n > 2) bad++;
  // the middle slabs differ by at most one row block, and there are at most kHostMidSlabs
  if (n - 2 > kHostMidSlabs) bad++;
  int lo = 1 << 30, hi = 0;
  for (int i = 1; i + 1 < n; i++) {
    const int blocks = (r0[i + 1] - r0[i]) / TR;
    lo = blocks < lo ? blocks : lo;
    hi = blocks > hi ? blocks : hi;
  }
  if (n > 2 && hi - lo > 1) bad++;
  return bad;
}

int main(int argc, char **argv) {
  long bad = 0, cases = 0;
  const int sms_list[] = {1, 2, 8, 132, 148, 160};
  for (int sms : sms_list)
    for (int N = 16; N <= 9000; N += 112)
      for (int M = 16; M <= 20000; M += 16) {
        bad += check(M, N, sms);
        cases++;
      }
  printf("%ld %ld\n", bad, cases);
  for (int a = 1; a + 2 < argc; a += 3) {
    int r0[kHostMaxSlabs + 2];
    const int M = atoi(argv[a]), N = atoi(argv[a + 1]), sms = atoi(argv[a + 2]);
    const int n = host_slabs(M, N, TR, TC, (long long)sms * PER_SM, r0);
    for (int i = 0; i <= n; i++) printf("%d%c", r0[i], i == n ? '\n' : ' ');
  }
  return 0;
}
