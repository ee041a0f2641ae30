// Row slabs of mmaemu_gemm_host (host code, no CUDA): which rows of A, C and
// D travel and compute together while the GEMM runs from host memory.
#pragma once

namespace mmaemu_host {

constexpr int kHostMaxSlabs = 8;  // slabs of one call, at most
constexpr int kHostMidSlabs = 4;  // equal slabs between the first and the last
constexpr int kHostTailDiv = 16;  // the last slab: 1/16 of the row blocks (at least one)

// Row boundaries r0[0] = 0 < r0[1] < ... < r0[n] = M of the slabs of an M x N
// GEMM whose output tiles are tile_rows x tile_cols and of which wave_tiles
// run at once on the GPU; returns n (1 <= n <= kHostMaxSlabs).  Every
// boundary but the last is a multiple of tile_rows.
//   - The first slab holds one full wave of tiles, the fewest rows that keep
//     every SM busy while the next slab is copied: nothing computes until B
//     and that slab have arrived.
//   - The last slab is short, since its D is the one copy left once
//     computing ends.
//   - The rows between go in up to kHostMidSlabs slabs that differ by at
//     most one row block.
// A GEMM of one wave or less is one slab.  (Measured on the 4096^3 FP16
// GEMM from pinned memory: 10.86 ms, against 11.0 ms for six equal slabs,
// 11.49 ms for eight and 11.3 ms for a first slab of 128 rows, which leaves
// the GPU idle while the second slab is copied.)
inline int host_slabs(int M, int N, int tile_rows, int tile_cols, long long wave_tiles, int *r0) {
  const int nb = (M + tile_rows - 1) / tile_rows;  // row blocks
  const int cb = (N + tile_cols - 1) / tile_cols;  // column blocks
  long long head_ll = (wave_tiles + cb - 1) / cb;
  if (head_ll < 1) head_ll = 1;
  if (head_ll > nb) head_ll = nb;
  const int head = (int)head_ll;
  int n = 0, b = 0;
  r0[0] = 0;
  auto cut = [&](int blocks) {
    b += blocks;
    r0[++n] = (long long)b * tile_rows < M ? b * tile_rows : M;
  };
  cut(head);
  const int rest = nb - head;
  int tail = nb / kHostTailDiv > 1 ? nb / kHostTailDiv : 1;
  if (tail > rest) tail = rest;
  const int mid = rest - tail, nm = mid < kHostMidSlabs ? mid : kHostMidSlabs;
  for (int i = 0; i < nm; i++) cut(mid / nm + (i < mid % nm));
  if (tail > 0) cut(tail);
  return n;
}

}  // namespace mmaemu_host
