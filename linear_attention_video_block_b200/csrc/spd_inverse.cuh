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

// Packed fp32 pairs for the rank-2 updates below (sm_100 f32x2 arithmetic:
// one instruction for two fused multiply-adds).
__device__ __forceinline__ unsigned long long spd_pack(float lo, float hi) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void spd_unpack(unsigned long long p, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(p));
}
__device__ __forceinline__ unsigned long long spd_fma2(unsigned long long a, unsigned long long b,
                                                       unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}

// The same inverse two pivots per block barrier (block Gauss-Jordan with 2 x 2
// pivot blocks P, which for I + A are SPD with eigenvalues >= 1, so det P >= 1):
// with rows and columns k0, k0 + 1 zeroed, a <- a - C R~ where R~ = P^-1 R
// (R~ = P^-1 in the pivot columns) and C the two pivot columns (-I in the
// pivot rows). The thread's block is held as column pairs and the rank-2
// update runs as packed f32x2 fused multiply-adds. Needs D / 16 even (d = 64,
// 128). Buffers: rowk and colk are [2 (double buffer)][2 (pivot)][D].
template <int D>
__device__ __forceinline__ void spd_inverse_blocks2x(float (&a)[D / 16][D / 16], int tr, int tc,
                                                     float (*rowk)[2][D], float (*colk)[2][D]) {
  constexpr int RA = D / 16, RP = RA / 2;
  static_assert(RA % 2 == 0, "column pairs");
  unsigned long long a2[RA][RP];
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int u = 0; u < RP; ++u) a2[x][u] = spd_pack(a[x][2 * u], a[x][2 * u + 1]);
#pragma unroll
  for (int kb = 0; kb < RA; ++kb) {
#pragma unroll 1
    for (int kr0 = 0; kr0 < 16; kr0 += 2) {
      const int k0 = 16 * kb + kr0;
      const int buf = (kr0 >> 1) & 1;
      const int qr = tr - kr0, qc = tc - kr0;
      if (qr == 0 || qr == 1) {
#pragma unroll
        for (int u = 0; u < RP; ++u) {
          float lo, hi;
          spd_unpack(a2[kb][u], lo, hi);
          rowk[buf][qr][tc + 16 * (2 * u)] = lo;
          rowk[buf][qr][tc + 16 * (2 * u + 1)] = hi;
          a2[kb][u] = 0ull;
        }
      }
      if (qc == 0 || qc == 1) {
#pragma unroll
        for (int x = 0; x < RA; ++x) {
          float lo, hi;
          spd_unpack(a2[x][kb >> 1], lo, hi);
          const bool pivot_row = x == kb && (qr == 0 || qr == 1);
          colk[buf][qc][tr + 16 * x] = pivot_row ? (qr == qc ? -1.f : 0.f) : ((kb & 1) ? hi : lo);
          a2[x][kb >> 1] = (kb & 1) ? spd_pack(lo, 0.f) : spd_pack(0.f, hi);
        }
      }
      __syncthreads();
      const float p00 = rowk[buf][0][k0], p01 = rowk[buf][0][k0 + 1];
      const float p10 = rowk[buf][1][k0], p11 = rowk[buf][1][k0 + 1];
      const float idet = 1.f / (p00 * p11 - p01 * p10);
      const float i00 = p11 * idet, i01 = -p01 * idet, i10 = -p10 * idet, i11 = p00 * idet;
      float r0[RA], r1[RA];
#pragma unroll
      for (int y = 0; y < RA; ++y) {
        const int j = tc + 16 * y;
        if (j == k0) {
          r0[y] = i00;
          r1[y] = i10;
        } else if (j == k0 + 1) {
          r0[y] = i01;
          r1[y] = i11;
        } else {
          const float x0 = rowk[buf][0][j], x1 = rowk[buf][1][j];
          r0[y] = fmaf(i00, x0, i01 * x1);
          r1[y] = fmaf(i10, x0, i11 * x1);
        }
      }
      unsigned long long r0p[RP], r1p[RP];
#pragma unroll
      for (int u = 0; u < RP; ++u) {
        r0p[u] = spd_pack(r0[2 * u], r0[2 * u + 1]);
        r1p[u] = spd_pack(r1[2 * u], r1[2 * u + 1]);
      }
#pragma unroll
      for (int x = 0; x < RA; ++x) {
        const float c0 = -colk[buf][0][tr + 16 * x], c1 = -colk[buf][1][tr + 16 * x];
        const unsigned long long c0p = spd_pack(c0, c0), c1p = spd_pack(c1, c1);
#pragma unroll
        for (int u = 0; u < RP; ++u) a2[x][u] = spd_fma2(c1p, r1p[u], spd_fma2(c0p, r0p[u], a2[x][u]));
      }
    }
  }
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int u = 0; u < RP; ++u) spd_unpack(a2[x][u], a[x][2 * u], a[x][2 * u + 1]);
}
