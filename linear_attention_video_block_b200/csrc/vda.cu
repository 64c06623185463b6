// Video Delta Attention states (project page "Video Delta Attention: A
// Frame-Wise Solution"; "Faster Than It Plays", closed form
// S_t = (S_bar + B)(I + A)^-1).
//
// Three frame-parallel / lane-parallel phases:
//   gram     A_f = K_f^T Diag(beta_f) K_f and B_f = V_f^T Diag(beta_f) K_f for
//            every scanned frame and for the text (slot 0), fp32 (bf16 inputs:
//            tensor-core kernel in gram_tc.cu; fp32 inputs: CUDA-core kernel here).
//   inverse  M_f = (I + A_f)^-1 in place of A_f (register-blocked Gauss-Jordan;
//            I + A_f is SPD with every pivot >= 1, so no pivoting is needed).
//   scan     S <- (S + B_f) M_f, forward over 1..fwd_max and reverse over
//            F-2..rev_min, from S0 = 1/2 B_T M_T. Rows of S evolve independently
//            (the update multiplies on the right), so each CTA owns 16 rows of
//            one (b, h, direction) state and the chain needs no cross-CTA sync.
//            States read by each chunk are stored into [B, H, 2, J, d, d].
#include "vdn_internal.cuh"

namespace vdn {
namespace {

constexpr int NT = 256;

// Frame of gram/inverse slot index i: slot 0 = text (when T > 0), then frames
// 1..fwd_max, then frames rev_lo..F-2.
struct SlotMap {
  int has_text, fwd_max, rev_lo, F;
  __device__ int frame(int i) const {
    if (has_text) { if (i == 0) return 0; --i; }
    if (i < fwd_max) return 1 + i;
    return rev_lo + (i - fwd_max);
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(NT)
gram_kernel(Layout l, SlotMap sm_map, const T* __restrict__ k, const T* __restrict__ v,
            const T* __restrict__ kt, const T* __restrict__ vt, const float* __restrict__ beta,
            const float* __restrict__ beta_t, float* __restrict__ am, float* __restrict__ bw) {
  constexpr int TU = 32;
  constexpr int RA = D / 16;
  __shared__ float ks[TU][D];
  __shared__ float kw[TU][D];
  __shared__ float vs[TU][D];
  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int f = sm_map.frame(blockIdx.x);
  const bool text = sm_map.has_text && blockIdx.x == 0;
  const long long HD = (long long)l.H * D;
  const int U = text ? l.T : l.N;
  const T* kp;
  const T* vp;
  const float* bp;
  if (text) {
    kp = kt + (long long)b * l.T * HD + (long long)h * D;
    vp = vt + (long long)b * l.T * HD + (long long)h * D;
    bp = beta_t + (long long)b * l.T * l.H + h;
  } else {
    long long tok0 = (long long)b * l.L() + (long long)f * l.N;
    kp = k + tok0 * HD + (long long)h * D;
    vp = v + tok0 * HD + (long long)h * D;
    bp = beta + tok0 * l.H + h;
  }
  const int ti = tid / 16, tj = tid % 16;
  float a_acc[RA][RA], b_acc[RA][RA];
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int y = 0; y < RA; ++y) { a_acc[x][y] = 0.f; b_acc[x][y] = 0.f; }
  for (int u0 = 0; u0 < U; u0 += TU) {
    const int nu = min(TU, U - u0);
    __syncthreads();
    for (int i = tid; i < TU * D; i += NT) {
      int r = i / D, cidx = i % D;
      float kx = 0.f, vx = 0.f, bx = 0.f;
      if (r < nu) {
        long long off = (long long)(u0 + r) * HD + cidx;
        kx = to_f32(kp[off]);
        vx = to_f32(vp[off]);
        bx = bp[(long long)(u0 + r) * l.H];
      }
      ks[r][cidx] = kx;
      kw[r][cidx] = kx * bx;
      vs[r][cidx] = vx;
    }
    __syncthreads();
    for (int u = 0; u < nu; ++u) {
      float kr[RA], vr[RA], wc[RA];
#pragma unroll
      for (int x = 0; x < RA; ++x) {
        kr[x] = ks[u][ti + 16 * x];
        vr[x] = vs[u][ti + 16 * x];
        wc[x] = kw[u][tj + 16 * x];
      }
#pragma unroll
      for (int x = 0; x < RA; ++x)
#pragma unroll
        for (int y = 0; y < RA; ++y) {
          a_acc[x][y] = fmaf(kr[x], wc[y], a_acc[x][y]);
          b_acc[x][y] = fmaf(vr[x], wc[y], b_acc[x][y]);
        }
    }
  }
  const long long slot = ((long long)b * l.H + h) * l.F + f;
  float* ao = am + slot * D * D;
  float* bo = bw + slot * D * D;
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int y = 0; y < RA; ++y) {
      ao[(ti + 16 * x) * D + tj + 16 * y] = a_acc[x][y];
      bo[(ti + 16 * x) * D + tj + 16 * y] = b_acc[x][y];
    }
}

// In-place inverse of (I + A) for one slot: Gauss-Jordan elimination without
// pivoting (every pivot of an SPD matrix with eigenvalues >= 1 is >= 1).
// Thread (tr, tc) of a 16 x 16 grid keeps the interleaved block of rows
// tr + 16a and columns tc + 16c in registers; the pivot row and column of
// each step go through double-buffered shared memory, one barrier per step.
template <int D>
__global__ void __launch_bounds__(NT)
inverse_kernel(Layout l, SlotMap sm_map, float* __restrict__ am) {
  constexpr int RA = D / 16;
  __shared__ float rowk[2][D];
  __shared__ float colk[2][D];
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;
  const int h = blockIdx.y, b = blockIdx.z;
  const int f = sm_map.frame(blockIdx.x);
  const long long slot = ((long long)b * l.H + h) * l.F + f;
  float* g = am + slot * D * D;
  float a[RA][RA];
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int y = 0; y < RA; ++y) {
      const int i = tr + 16 * x, j = tc + 16 * y;
      a[x][y] = g[i * D + j] + (i == j ? 1.f : 0.f);
    }
  // pivot k = 16 kb + kr; kb is a compile-time index into the register block
#pragma unroll
  for (int kb = 0; kb < RA; ++kb) {
#pragma unroll 1
    for (int kr = 0; kr < 16; ++kr) {
      const int k = 16 * kb + kr;
      const int buf = k & 1;
      // owners publish row k and column k of the current matrix
      if (tr == kr) {
#pragma unroll
        for (int y = 0; y < RA; ++y) rowk[buf][tc + 16 * y] = a[kb][y];
      }
      if (tc == kr) {
#pragma unroll
        for (int x = 0; x < RA; ++x) colk[buf][tr + 16 * x] = a[x][kb];
      }
      __syncthreads();
      const float rp = 1.f / rowk[buf][k];
      float rjs[RA];
#pragma unroll
      for (int y = 0; y < RA; ++y) {
        const int j = tc + 16 * y;
        rjs[y] = (j == k) ? rp : rowk[buf][j] * rp;
      }
#pragma unroll
      for (int x = 0; x < RA; ++x) {
        const int i = tr + 16 * x;
        if (i == k) {
#pragma unroll
          for (int y = 0; y < RA; ++y) a[x][y] = rjs[y];
        } else {
          const float ci = colk[buf][i];
#pragma unroll
          for (int y = 0; y < RA; ++y) {
            const int j = tc + 16 * y;
            a[x][y] = fmaf(-ci, rjs[y], (j == k) ? 0.f : a[x][y]);
          }
        }
      }
    }
  }
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int y = 0; y < RA; ++y) g[(tr + 16 * x) * D + tc + 16 * y] = a[x][y];
}

// Row-split scan. grid (D/16, 2, B*H); 16 rows of S per CTA.
template <int D>
__global__ void __launch_bounds__(NT)
scan_kernel(Layout l, int fwd_max, int rev_min, int has_text, const float* __restrict__ am,
            const float* __restrict__ bw, float* __restrict__ states) {
  constexpr int R = 16;
  constexpr int RG = NT / D;       // row groups
  constexpr int RR = R / RG;       // rows per thread
  __shared__ float x[R][D];
  const int tid = threadIdx.x;
  const int col = tid % D, rg = tid / D;
  const int row0 = blockIdx.x * R;
  const int dir = blockIdx.y;
  const int bh = blockIdx.z;
  const int J = l.J();
  const float* am_bh = am + (long long)bh * l.F * D * D;
  const float* bw_bh = bw + (long long)bh * l.F * D * D;
  float* st_bh = states + (long long)bh * 2 * J * D * D + (long long)dir * J * D * D;

  float s[RR];
  // S0 = 1/2 B_T M_T (slot 0), or 0 without text.
  if (has_text) {
    for (int i = tid; i < R * D; i += NT) x[i / D][i % D] = 0.5f * bw_bh[(row0 + i / D) * D + i % D];
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RR; ++r) s[r] = 0.f;
    for (int i = 0; i < D; ++i) {
      const float m = am_bh[i * D + col];
#pragma unroll
      for (int r = 0; r < RR; ++r) s[r] = fmaf(x[rg * RR + r][i], m, s[r]);
    }
  } else {
#pragma unroll
    for (int r = 0; r < RR; ++r) s[r] = 0.f;
  }
  auto store_for = [&](int idx) {
    for (int j = 0; j < J; ++j) {
      Group G = make_group(l, 2 + j);
      if (G.nq == 0) continue;
      int want = dir == 0 ? G.fwd_idx : G.rev_idx;
      if (want != idx) continue;
      float* dst = st_bh + (long long)j * D * D;
#pragma unroll
      for (int r = 0; r < RR; ++r) dst[(row0 + rg * RR + r) * D + col] = s[r];
    }
  };
  store_for(dir == 0 ? 0 : l.F - 1);
  const int nsteps = dir == 0 ? fwd_max : (l.F - 1 - rev_min);
  for (int t = 0; t < nsteps; ++t) {
    const int f = dir == 0 ? 1 + t : l.F - 2 - t;
    const float* mf = am_bh + (long long)f * D * D;
    const float* bf = bw_bh + (long long)f * D * D;
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RR; ++r) x[rg * RR + r][col] = s[r] + bf[(row0 + rg * RR + r) * D + col];
    __syncthreads();
#pragma unroll
    for (int r = 0; r < RR; ++r) s[r] = 0.f;
#pragma unroll 8
    for (int i = 0; i < D; ++i) {
      const float m = mf[i * D + col];
#pragma unroll
      for (int r = 0; r < RR; ++r) s[r] = fmaf(x[rg * RR + r][i], m, s[r]);
    }
    store_for(f);
  }
}

// Zero the chunk-table entries of chunks without non-boundary frames.
__global__ void zero_unused_chunks(Layout l, float* __restrict__ states) {
  const int J = l.J();
  const long long dd = (long long)l.d * l.d;
  const int bh = blockIdx.y;
  for (int j = 0; j < J; ++j) {
    Group G = make_group(l, 2 + j);
    if (G.nq != 0) continue;
    for (int dir = 0; dir < 2; ++dir) {
      float* dst = states + (((long long)bh * 2 + dir) * J + j) * dd;
      for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < dd;
           i += (long long)gridDim.x * blockDim.x)
        dst[i] = 0.f;
    }
  }
}

template <typename T, int D>
cudaError_t launch_states_t(const Layout& l, int dtype, const void* k, const void* v, const void* kt,
                            const void* vt, const float* beta, const float* beta_t, float* am,
                            float* bw, float* states, cudaStream_t st) {
  int fwd_max, rev_min;
  scan_extent(l, fwd_max, rev_min);
  SlotMap map;
  map.has_text = l.T > 0 ? 1 : 0;
  map.fwd_max = fwd_max;
  map.rev_lo = rev_min > fwd_max + 1 ? rev_min : fwd_max + 1;
  map.F = l.F;
  const int nrev = (l.F - 2) - map.rev_lo + 1;
  const int nslots = map.has_text + fwd_max + (nrev > 0 ? nrev : 0);
  if (nslots > 0) {
    dim3 grid(nslots, l.H, l.B);
    cudaError_t e;
    if (gram_tc_supported(l, dtype)) {
      e = launch_gram_tc(l, map.has_text, map.fwd_max, map.rev_lo, nslots, k, v, kt, vt, beta,
                         beta_t, am, bw, st);
    } else {
      gram_kernel<T, D><<<grid, NT, 0, st>>>(l, map, (const T*)k, (const T*)v, (const T*)kt,
                                             (const T*)vt, beta, beta_t, am, bw);
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    inverse_kernel<D><<<grid, NT, 0, st>>>(l, map, am);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  {
    dim3 grid(D / 16, 2, l.B * l.H);
    scan_kernel<D><<<grid, NT, 0, st>>>(l, fwd_max, rev_min, map.has_text, am, bw, states);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    zero_unused_chunks<<<dim3(32, l.B * l.H), 256, 0, st>>>(l, states);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_states(const Layout& l, int dtype, const void* k, const void* v,
                              const void* kt, const void* vt, const float* beta,
                              const float* beta_text, float* am, float* bw, float* states,
                              cudaStream_t st) {
  if (dtype == VDN_F32) {
    switch (l.d) {
      case 16: return launch_states_t<float, 16>(l, dtype, k, v, kt, vt, beta, beta_text, am, bw, states, st);
      case 32: return launch_states_t<float, 32>(l, dtype, k, v, kt, vt, beta, beta_text, am, bw, states, st);
      case 64: return launch_states_t<float, 64>(l, dtype, k, v, kt, vt, beta, beta_text, am, bw, states, st);
      case 128: return launch_states_t<float, 128>(l, dtype, k, v, kt, vt, beta, beta_text, am, bw, states, st);
    }
  } else {
    switch (l.d) {
      case 64: return launch_states_t<__nv_bfloat16, 64>(l, dtype, k, v, kt, vt, beta, beta_text, am, bw, states, st);
      case 128: return launch_states_t<__nv_bfloat16, 128>(l, dtype, k, v, kt, vt, beta, beta_text, am, bw, states, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace vdn
