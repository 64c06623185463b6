// Video Delta Attention states (project page "Video Delta Attention: A
// Frame-Wise Solution"; "Faster Than It Plays", closed form
// S_t = (S_bar + B)(I + A)^-1).
//
// Three frame-parallel / lane-parallel phases:
//   gram     A_f = K_f^T Diag(beta_f) K_f and B_f = V_f^T Diag(beta_f) K_f for
//            every scanned frame and for the text (slot 0), fp32 (bf16 inputs:
//            tensor-core kernel in gram_tc.cu; fp32 inputs: CUDA-core kernel here).
//   inverse  M_f = (I + A_f)^-1 in place of A_f (register-blocked Gauss-Jordan,
//            spd_inverse.cuh; I + A_f is SPD with every pivot >= 1, so no
//            pivoting is needed). The bf16 tensor-core Gram kernel does it in
//            its own epilogue; the fp32 path launches inverse_kernel.
//   scan     S <- (S Diag(alpha_f) + B_f) M_f (alpha: optional KDA decay), forward over 1..fwd_max and reverse over
//            F-2..rev_min, from S0 = 1/2 B_T M_T. Rows of S evolve independently
//            (the update multiplies on the right), so each CTA owns 16 rows of
//            one (b, h, direction) state and the chain needs no cross-CTA sync;
//            all CTAs are resident at once and M_f streams through a small
//            cp.async ring.
//            States read by each chunk are stored into [B, H, 2, J, d, d].
#include "spd_inverse.cuh"
#include "vdn_internal.cuh"

namespace vdn {

// Device status word of this translation unit (bound checks of the checked build).
__device__ int g_vda_status = 0;

cudaError_t read_and_clear_vda_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_vda_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_vda_status, &zero, sizeof(int));
}

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
      if (r < nu && VDN_IN_BOUNDS(u0 + r < U && (text || f * l.N + u0 + r < l.L()), &g_vda_status)) {
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
  if (!VDN_IN_BOUNDS(f >= 0 && f < l.F && h < l.H && b < l.B, &g_vda_status)) return;
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

// In-place inverse of (I + A) for one slot (spd_inverse.cuh); the bf16 path
// does the same inside the tensor-core Gram kernel.
template <int D>
__global__ void __launch_bounds__(NT, 2)
inverse_kernel(Layout l, SlotMap sm_map, float* __restrict__ am) {
  constexpr int RA = D / 16;
  __shared__ float rowk[2][D];
  __shared__ float colk[2][D];
  const int tid = threadIdx.x;
  const int tr = tid / 16, tc = tid % 16;
  const int h = blockIdx.y, b = blockIdx.z;
  const int f = sm_map.frame(blockIdx.x);
  const long long slot = ((long long)b * l.H + h) * l.F + f;
  if (!VDN_IN_BOUNDS(f >= 0 && f < l.F && h < l.H && b < l.B, &g_vda_status)) return;
  float* g = am + slot * D * D;
  float a[RA][RA];
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int y = 0; y < RA; ++y) {
      const int i = tr + 16 * x, j = tc + 16 * y;
      a[x][y] = g[i * D + j] + (i == j ? 1.f : 0.f);
    }
  spd_inverse_blocks<D>(a, tr, tc, rowk, colk);
#pragma unroll
  for (int x = 0; x < RA; ++x)
#pragma unroll
    for (int y = 0; y < RA; ++y) g[(tr + 16 * x) * D + tc + 16 * y] = a[x][y];
}

// Row-split scan. grid (D/16, 2, B*H): 16 rows of S per CTA, so all
// 2 (D/16) B H CTAs are resident at once (40 KB of shared memory each) and the
// chain of dependent steps runs a single time. 128 threads (fewer for d < 32); thread (rg, cg)
// owns rows 4rg..4rg+3 and columns 4cg..4cg+3 of the CTA's block (d = 128;
// smaller d use fewer column groups and more rows per thread). Each step
// S <- (S + B_f) M_f streams M_f through a 3-deep ring of 16-row chunks with
// cp.async; the first step is the text slot (S0 = 1/2 B_T M_T) when there is text.
template <int D>
struct ScanCfg {
  static constexpr int kR = 16;                 // rows of S per CTA
  static constexpr int kCG = D / 4;             // column groups of 4
  static constexpr int kThreads = (kCG * 16 < 128) ? kCG * 16 : 128;
  static constexpr int kRG = kThreads / kCG;    // row groups
  static constexpr int kRR = kR / kRG;          // rows per thread
  static constexpr int kChunk = 16;             // rows of M per chunk
  static constexpr int kRing = 3;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int D>
__global__ void __launch_bounds__(128)
scan_kernel(Layout l, int fwd_max, int rev_min, int has_text, const float* __restrict__ am,
            const float* __restrict__ bw, const float* __restrict__ alpha, float* __restrict__ states) {
  using C = ScanCfg<D>;
  constexpr int R = C::kR, RR = C::kRR, CH = C::kChunk, NCH = D / CH;
  __shared__ __align__(16) float ring[C::kRing][CH * D];
  __shared__ __align__(16) float x[R * D];
  const int tid = threadIdx.x;
  const int cg = tid % C::kCG, rg = tid / C::kCG;
  const int row0 = blockIdx.x * R;
  const int dir = blockIdx.y;
  const int bh = blockIdx.z;
  const int J = l.J();
  const float* am_bh = am + (long long)bh * l.F * D * D;
  const float* bw_bh = bw + (long long)bh * l.F * D * D;
  float* st_bh = states + (long long)bh * 2 * J * D * D + (long long)dir * J * D * D;
  const int nframes = dir == 0 ? fwd_max : (l.F - 1 - rev_min);
  const int nsteps = has_text + nframes;
  auto frame_of = [&](int t) {
    return (has_text && t == 0) ? 0 : (dir == 0 ? 1 + (t - has_text) : l.F - 2 - (t - has_text));
  };
  // global chunk sequence q = t * NCH + c: rows 16c..16c+15 of M_{frame_of(t)}
  auto load_chunk = [&](int q) {
    const int t = q / NCH, c = q % NCH;
    (void)VDN_IN_BOUNDS(frame_of(t) >= 0 && frame_of(t) < l.F, &g_vda_status);
    const float* src = am_bh + (long long)frame_of(t) * D * D + (long long)c * CH * D;
    float* dst = ring[q % C::kRing];
    for (int i = tid * 4; i < CH * D; i += C::kThreads * 4) cp_async16(dst + i, src + i);
  };
  const int nq = nsteps * NCH;
  float s[RR][4];
#pragma unroll
  for (int r = 0; r < RR; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) s[r][c] = 0.f;
  auto store_for = [&](int idx) {
    for (int j = 0; j < J; ++j) {
      Group G = make_group(l, 2 + j);
      if (G.nq == 0) continue;
      const int want = dir == 0 ? G.fwd_idx : G.rev_idx;
      if (want != idx) continue;
      if (!VDN_IN_BOUNDS(j < J && row0 + R <= D, &g_vda_status)) continue;
      float* dst = st_bh + (long long)j * D * D;
#pragma unroll
      for (int r = 0; r < RR; ++r)
        *reinterpret_cast<float4*>(dst + (row0 + RR * rg + r) * D + 4 * cg) =
            make_float4(s[r][0], s[r][1], s[r][2], s[r][3]);
    }
  };
  if (!has_text) store_for(dir == 0 ? 0 : l.F - 1);
  // prologue: two chunks in flight
  for (int q = 0; q < 2; ++q) {
    if (q < nq) load_chunk(q);
    cp_async_commit();
  }
  for (int t = 0; t < nsteps; ++t) {
    const bool text = has_text && t == 0;
    const int f = frame_of(t);
    // X = S Diag(alpha_f) + B_f rows (text step: X = 1/2 B_T rows); B rows read
    // straight from global; alpha_f (KDA channel decay, optional) over columns
    float4 av = make_float4(1.f, 1.f, 1.f, 1.f);
    if (alpha != nullptr && !text)
      av = *reinterpret_cast<const float4*>(
          alpha + (((long long)(bh / l.H) * l.F + f) * l.H + bh % l.H) * D + 4 * cg);
#pragma unroll
    for (int r = 0; r < RR; ++r) {
      const float4 bv = *reinterpret_cast<const float4*>(bw_bh + (long long)f * D * D +
                                                         (long long)(row0 + RR * rg + r) * D + 4 * cg);
      const float4 xv = text ? make_float4(0.5f * bv.x, 0.5f * bv.y, 0.5f * bv.z, 0.5f * bv.w)
                             : make_float4(fmaf(s[r][0], av.x, bv.x), fmaf(s[r][1], av.y, bv.y),
                                           fmaf(s[r][2], av.z, bv.z), fmaf(s[r][3], av.w, bv.w));
      *reinterpret_cast<float4*>(&x[(RR * rg + r) * D + 4 * cg]) = xv;
    }
    float acc[RR][4];
#pragma unroll
    for (int r = 0; r < RR; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
    for (int c = 0; c < NCH; ++c) {
      const int q = t * NCH + c;
      cp_async_wait<1>();   // chunk q has landed (q + 1 may still be in flight)
      __syncthreads();      // ... for every thread; x is complete; slot (q + 2) % 3 is free
      if (q + 2 < nq) load_chunk(q + 2);
      cp_async_commit();
      const float* mb = ring[q % C::kRing];
#pragma unroll
      for (int i4 = 0; i4 < CH; i4 += 4) {
        float xr[RR][4];
#pragma unroll
        for (int r = 0; r < RR; ++r) {
          const float4 v = *reinterpret_cast<const float4*>(&x[(RR * rg + r) * D + c * CH + i4]);
          xr[r][0] = v.x; xr[r][1] = v.y; xr[r][2] = v.z; xr[r][3] = v.w;
        }
#pragma unroll
        for (int ii = 0; ii < 4; ++ii) {
          const float4 m = *reinterpret_cast<const float4*>(&mb[(i4 + ii) * D + 4 * cg]);
#pragma unroll
          for (int r = 0; r < RR; ++r) {
            acc[r][0] = fmaf(xr[r][ii], m.x, acc[r][0]);
            acc[r][1] = fmaf(xr[r][ii], m.y, acc[r][1]);
            acc[r][2] = fmaf(xr[r][ii], m.z, acc[r][2]);
            acc[r][3] = fmaf(xr[r][ii], m.w, acc[r][3]);
          }
        }
      }
    }
    __syncthreads();  // all reads of x done before the next step rewrites it
#pragma unroll
    for (int r = 0; r < RR; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[r][c] = acc[r][c];
    store_for(text ? (dir == 0 ? 0 : l.F - 1) : f);
  }
  cp_async_wait<0>();
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
                            const void* vt, const float* beta, const float* beta_t,
                            const float* alpha, float* am, float* bw, float* states,
                            cudaStream_t st) {
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
      // the tensor-core Gram kernel also inverts I + A_f in place (am = M_f)
      e = launch_gram_tc(l, map.has_text, map.fwd_max, map.rev_lo, nslots, k, v, kt, vt, beta,
                         beta_t, am, bw, st);
      if (e != cudaSuccess) return e;
    } else {
      gram_kernel<T, D><<<grid, NT, 0, st>>>(l, map, (const T*)k, (const T*)v, (const T*)kt,
                                             (const T*)vt, beta, beta_t, am, bw);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
      inverse_kernel<D><<<grid, NT, 0, st>>>(l, map, am);
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  {
    dim3 grid(D / ScanCfg<D>::kR, 2, l.B * l.H);
    scan_kernel<D><<<grid, ScanCfg<D>::kThreads, 0, st>>>(l, fwd_max, rev_min, map.has_text, am, bw, alpha, states);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    zero_unused_chunks<<<dim3(32, l.B * l.H), 256, 0, st>>>(l, states);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_vda_states(const Layout& l, int dtype, const void* k, const void* v,
                              const void* kt, const void* vt, const float* beta,
                              const float* beta_text, const float* alpha, float* am, float* bw,
                              float* states, cudaStream_t st) {
  if (dtype == VDN_F32) {
    switch (l.d) {
      case 16: return launch_states_t<float, 16>(l, dtype, k, v, kt, vt, beta, beta_text, alpha, am, bw, states, st);
      case 32: return launch_states_t<float, 32>(l, dtype, k, v, kt, vt, beta, beta_text, alpha, am, bw, states, st);
      case 64: return launch_states_t<float, 64>(l, dtype, k, v, kt, vt, beta, beta_text, alpha, am, bw, states, st);
      case 128: return launch_states_t<float, 128>(l, dtype, k, v, kt, vt, beta, beta_text, alpha, am, bw, states, st);
    }
  } else {
    switch (l.d) {
      case 64: return launch_states_t<__nv_bfloat16, 64>(l, dtype, k, v, kt, vt, beta, beta_text, alpha, am, bw, states, st);
      case 128: return launch_states_t<__nv_bfloat16, 128>(l, dtype, k, v, kt, vt, beta, beta_text, alpha, am, bw, states, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace vdn
