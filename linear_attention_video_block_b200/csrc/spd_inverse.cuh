// In-place inverse of an SPD matrix I + A with every eigenvalue >= 1 (the
// frame solve of Video Delta Attention: project page "Video Delta Attention:
// A Frame-Wise Solution"; "Faster Than It Plays", "Two branches instead of
// one", S = (S_bar + B)(I + A)^-1), by Gauss-Jordan elimination without
// pivoting: every pivot of such a matrix is >= 1.
//
// Step k is written as a rank-1 update: with row k and column k zeroed,
//   a <- a - c r^T,  c = column k (c_k = -1),  r = row k / p (r_k = 1/p),
// which yields the Gauss-Jordan result in every entry. The d x d matrix is
// held by a 16 x 16 grid of threads (tid = 16 tr + tc, 256 threads), thread
// (tr, tc) keeping the interleaved block of rows tr + 16x and columns tc + 16y
// in registers; the pivot row and column go through double-buffered shared
// memory, one block barrier per step. All 256 threads of the block call it.
#pragma once

template <int D>
__device__ __forceinline__ void spd_inverse_blocks(float (&a)[D / 16][D / 16], int tr, int tc,
                                                   float (*rowk)[D], float (*colk)[D]) {
  constexpr int RA = D / 16;
  // pivot k = 16 kb + kr; kb is a compile-time index into the register block
#pragma unroll
  for (int kb = 0; kb < RA; ++kb) {
#pragma unroll 1
    for (int kr = 0; kr < 16; ++kr) {
      const int k = 16 * kb + kr;
      const int buf = k & 1;
      // owners publish row k and column k, then zero them in their registers
      if (tr == kr) {
#pragma unroll
        for (int y = 0; y < RA; ++y) {
          rowk[buf][tc + 16 * y] = a[kb][y];
          a[kb][y] = 0.f;
        }
      }
      if (tc == kr) {
#pragma unroll
        for (int x = 0; x < RA; ++x) {
          colk[buf][tr + 16 * x] = (x == kb && tr == kr) ? -1.f : a[x][kb];
          a[x][kb] = 0.f;
        }
      }
      __syncthreads();
      const float rp = 1.f / rowk[buf][k];
      float r[RA], c[RA];
#pragma unroll
      for (int y = 0; y < RA; ++y) {
        const int j = tc + 16 * y;
        r[y] = (j == k) ? rp : rowk[buf][j] * rp;
      }
#pragma unroll
      for (int x = 0; x < RA; ++x) c[x] = colk[buf][tr + 16 * x];
#pragma unroll
      for (int x = 0; x < RA; ++x)
#pragma unroll
        for (int y = 0; y < RA; ++y) a[x][y] = fmaf(-c[x], r[y], a[x][y]);
    }
  }
}
