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
//            one (b, h, direction) state and the chain needs no cross-CTA sync;
//            M_f and B_f stream into shared memory two steps ahead.
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

// Row-split scan. grid (D/16, 2, B*H); 16 rows of S per CTA, 2*D threads, each
// owning a 2 x 4 block of those rows. One thread bulk-copies M_f (D x D) and
// the CTA's 16 rows of B_f into double-buffered shared memory two steps ahead
// (cp.async.bulk completing on an mbarrier); the first step is the text slot
// (S0 = 1/2 B_T M_T) when there is text.
template <int D>
struct ScanSmem {
  float m[2][D * D];
  float bw[2][16 * D];
  float x[16 * D];
  unsigned long long full[2];
};

__device__ __forceinline__ uint32_t scan_smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <int D>
__global__ void __launch_bounds__(2 * D)
scan_kernel(Layout l, int fwd_max, int rev_min, int has_text, const float* __restrict__ am,
            const float* __restrict__ bw, float* __restrict__ states) {
  constexpr int R = 16;
  constexpr int CG = D / 4;             // column groups of 4
  extern __shared__ __align__(128) unsigned char scan_raw[];
  ScanSmem<D>& sm = *reinterpret_cast<ScanSmem<D>*>(scan_raw);
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;   // rows 2rg, 2rg+1; cols 4cg..4cg+3
  const int row0 = blockIdx.x * R;
  const int dir = blockIdx.y;
  const int bh = blockIdx.z;
  const int J = l.J();
  const float* am_bh = am + (long long)bh * l.F * D * D;
  const float* bw_bh = bw + (long long)bh * l.F * D * D;
  float* st_bh = states + (long long)bh * 2 * J * D * D + (long long)dir * J * D * D;
  const int nframes = dir == 0 ? fwd_max : (l.F - 1 - rev_min);
  const int nsteps = has_text + nframes;
  auto frame_of = [&](int t) { return (has_text && t == 0) ? 0 : (dir == 0 ? 1 + (t - has_text) : l.F - 2 - (t - has_text)); };
  constexpr uint32_t kBytes = (D * D + R * D) * 4;
  auto issue = [&](int t) {
    const int f = frame_of(t);
    const int buf = t & 1;
    const uint32_t bar = scan_smem_u32(&sm.full[buf]);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(kBytes) : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(scan_smem_u32(sm.m[buf])), "l"(am_bh + (long long)f * D * D), "r"(D * D * 4), "r"(bar)
                 : "memory");
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                 ::"r"(scan_smem_u32(sm.bw[buf])), "l"(bw_bh + (long long)f * D * D + (long long)row0 * D),
                   "r"(R * D * 4), "r"(bar)
                 : "memory");
  };
  if (tid == 0) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(scan_smem_u32(&sm.full[0])) : "memory");
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(scan_smem_u32(&sm.full[1])) : "memory");
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    if (nsteps > 0) issue(0);
    if (nsteps > 1) issue(1);
  }
  float s[2][4];
#pragma unroll
  for (int r = 0; r < 2; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) s[r][c] = 0.f;
  auto store_for = [&](int idx) {
    for (int j = 0; j < J; ++j) {
      Group G = make_group(l, 2 + j);
      if (G.nq == 0) continue;
      const int want = dir == 0 ? G.fwd_idx : G.rev_idx;
      if (want != idx) continue;
      float* dst = st_bh + (long long)j * D * D;
#pragma unroll
      for (int r = 0; r < 2; ++r)
        *reinterpret_cast<float4*>(dst + (row0 + 2 * rg + r) * D + 4 * cg) =
            make_float4(s[r][0], s[r][1], s[r][2], s[r][3]);
    }
  };
  if (!has_text) store_for(dir == 0 ? 0 : l.F - 1);
  for (int t = 0; t < nsteps; ++t) {
    const int buf = t & 1;
    const bool text = has_text && t == 0;
    // the copy lands within microseconds; the spin is bounded anyway
    {
      const uint32_t bar = scan_smem_u32(&sm.full[buf]);
      const uint32_t parity = (t >> 1) & 1;
      uint32_t ok = 0;
      for (uint32_t it = 0; it < (1u << 26) && !ok; ++it) {
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}\n"
                     : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
      }
      // (not reached in practice; if it were, the CTA carries on with stale
      // shared memory rather than leave the others waiting at the barrier)
    }
    // X = S + B_f rows (text step: X = 1/2 B_T rows)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float4 bv = *reinterpret_cast<const float4*>(&sm.bw[buf][(2 * rg + r) * D + 4 * cg]);
      float4 xv;
      if (text) {
        xv = make_float4(0.5f * bv.x, 0.5f * bv.y, 0.5f * bv.z, 0.5f * bv.w);
      } else {
        xv = make_float4(s[r][0] + bv.x, s[r][1] + bv.y, s[r][2] + bv.z, s[r][3] + bv.w);
      }
      *reinterpret_cast<float4*>(&sm.x[(2 * rg + r) * D + 4 * cg]) = xv;
    }
    __syncthreads();
    float acc[2][4];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
    const float* mb = sm.m[buf];
#pragma unroll 4
    for (int i = 0; i < D; i += 4) {
      const float4 x0 = *reinterpret_cast<const float4*>(&sm.x[(2 * rg) * D + i]);
      const float4 x1 = *reinterpret_cast<const float4*>(&sm.x[(2 * rg + 1) * D + i]);
      const float xa[4] = {x0.x, x0.y, x0.z, x0.w};
      const float xb[4] = {x1.x, x1.y, x1.z, x1.w};
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const float4 m = *reinterpret_cast<const float4*>(&mb[(i + ii) * D + 4 * cg]);
        acc[0][0] = fmaf(xa[ii], m.x, acc[0][0]);
        acc[0][1] = fmaf(xa[ii], m.y, acc[0][1]);
        acc[0][2] = fmaf(xa[ii], m.z, acc[0][2]);
        acc[0][3] = fmaf(xa[ii], m.w, acc[0][3]);
        acc[1][0] = fmaf(xb[ii], m.x, acc[1][0]);
        acc[1][1] = fmaf(xb[ii], m.y, acc[1][1]);
        acc[1][2] = fmaf(xb[ii], m.z, acc[1][2]);
        acc[1][3] = fmaf(xb[ii], m.w, acc[1][3]);
      }
    }
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[r][c] = acc[r][c];
    __syncthreads();  // everyone is done with buffer `buf` and with x
    if (tid == 0 && t + 2 < nsteps) issue(t + 2);
    if (text) store_for(dir == 0 ? 0 : l.F - 1);
    else store_for(frame_of(t));
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
    const int smem = (int)sizeof(ScanSmem<D>);
    cudaError_t e = cudaFuncSetAttribute(scan_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    scan_kernel<D><<<grid, 2 * D, smem, st>>>(l, fwd_max, rev_min, map.has_text, am, bw, states);
    e = cudaGetLastError();
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
