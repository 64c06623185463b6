// SIMT (CUDA-core, fp32 arithmetic) block-sparse window softmax.
//
// Used for float32 tensors (the tcgen05 kernel in window_tc.cu takes bf16).
// One CTA = 64 query rows of one query group of one (b, h); it walks the
// group's key segments (merged window + anchor frame intervals, then the text
// keys, then the audio keys of a joint layer) in 64-key tiles with an online
// softmax (project page "Local Softmax and Long-Range Linear Memory": one
// normaliser over window, anchors and text). The context query rows of a joint
// layer (text, audio) are groups whose key set is every token.
#include <type_traits>

#include "vdn_internal.cuh"

namespace vdn {

// Device status word of this translation unit (bound checks of the checked build).
__device__ int g_simt_status = 0;

cudaError_t read_and_clear_simt_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_simt_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_simt_status, &zero, sizeof(int));
}

namespace {

constexpr int BQ = 64;
constexpr int BK = 64;
constexpr int NT = 256;

template <int D>
struct SimtSmem {
  float q[BQ][D];
  float k[BK][D + 1];
  float v[BK][D];
  float p[BQ][BK + 1];
};

// Joint-layer tensors in the io dtype (null when absent).
template <typename T>
struct SimtJoint {
  const T* ka;
  const T* va;
  const T* qt;
  const T* qa;
  T* ot;
  T* oa;
  float* lse_t;
  float* lse_a;
};

template <typename T, typename TO, int D>
__global__ void __launch_bounds__(NT)
window_simt_kernel(Layout l, const T* __restrict__ q, const T* __restrict__ k,
                   const T* __restrict__ v, const T* __restrict__ kt,
                   const T* __restrict__ vt, TO* __restrict__ o, float* __restrict__ lse,
                   const SimtJoint<T> jn) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SimtSmem<D>& sm = *reinterpret_cast<SimtSmem<D>*>(smem_raw);
  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  int g, r0;
  tile_to_group(l, BQ, blockIdx.x, g, r0);
  if (g < 0) return;
  const Group G = make_group(l, g);
  const int rows_valid = min(BQ, G.q0 + G.nq - r0);
  const long long L = l.L();
  const long long HD = (long long)l.H * D;
  // rows of the query's own tensor: video L, text T, audio A
  const long long qrows = G.qsrc == kQVideo ? L : (G.qsrc == kQText ? l.T : l.A);
  const T* qsrc = G.qsrc == kQVideo ? q : (G.qsrc == kQText ? jn.qt : jn.qa);
  const T* qb = qsrc + ((long long)b * qrows) * HD + (long long)h * D;
  const T* kb = k + ((long long)b * L) * HD + (long long)h * D;
  const T* vb = v + ((long long)b * L) * HD + (long long)h * D;
  const T* ktb = kt ? kt + ((long long)b * l.T) * HD + (long long)h * D : nullptr;
  const T* vtb = vt ? vt + ((long long)b * l.T) * HD + (long long)h * D : nullptr;
  const T* kab = jn.ka ? jn.ka + ((long long)b * l.A) * HD + (long long)h * D : nullptr;
  const T* vab = jn.va ? jn.va + ((long long)b * l.A) * HD + (long long)h * D : nullptr;

  for (int i = tid; i < BQ * D; i += NT) {
    int r = i / D, cidx = i % D;
    const bool in = r < rows_valid && VDN_IN_BOUNDS(r0 + r < qrows, &g_simt_status);
    sm.q[r][cidx] = in ? to_f32(qb[(long long)(r0 + r) * HD + cidx]) : 0.f;
  }
  // Score mapping: thread (ty, tx) owns rows ty + 16m and keys tx + 16n.
  const int ty = tid / 16, tx = tid % 16;
  // Softmax / output mapping: row orow, 4 threads per row, D/4 columns each.
  const int orow = tid / 4, ocg = tid % 4;
  constexpr int OC = D / 4;
  float acc[OC];
#pragma unroll
  for (int i = 0; i < OC; ++i) acc[i] = 0.f;
  float m_run = -INFINITY, l_run = 0.f;
  const float scale = rsqrtf((float)D);

  // segments: the group's video segments, then the text, then the audio
  for (int s = 0; s < G.nseg + 2; ++s) {
    const bool text = (s == G.nseg), audio = (s == G.nseg + 1);
    const int seg_start = (text || audio) ? 0 : G.seg0[s];
    const int seg_len = text ? l.T : (audio ? l.A : G.segn[s]);
    if (seg_len == 0) continue;
    const T* ks = text ? ktb : (audio ? kab : kb);
    const T* vs = text ? vtb : (audio ? vab : vb);
    for (int k0 = 0; k0 < seg_len; k0 += BK) {
      const int kv = min(BK, seg_len - k0);
      __syncthreads();
      for (int i = tid; i < BK * D; i += NT) {
        int r = i / D, cidx = i % D;
        float kx = 0.f, vx = 0.f;
        const long long src_rows = text ? l.T : (audio ? l.A : L);
        if (r < kv && VDN_IN_BOUNDS(seg_start + k0 + r < src_rows, &g_simt_status)) {
          long long off = (long long)(seg_start + k0 + r) * HD + cidx;
          kx = to_f32(ks[off]);
          vx = to_f32(vs[off]);
        }
        sm.k[r][cidx] = kx;
        sm.v[r][cidx] = vx;
      }
      __syncthreads();
      float sc[4][4];
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) sc[a][c2] = 0.f;
#pragma unroll 4
      for (int kk = 0; kk < D; ++kk) {
        float qa[4], kc[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) qa[a] = sm.q[ty + 16 * a][kk];
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) kc[c2] = sm.k[tx + 16 * c2][kk];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int c2 = 0; c2 < 4; ++c2) sc[a][c2] = fmaf(qa[a], kc[c2], sc[a][c2]);
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c2 = 0; c2 < 4; ++c2) {
          int key = tx + 16 * c2;
          sm.p[ty + 16 * a][key] = (key < kv) ? sc[a][c2] * scale : -INFINITY;
        }
      __syncthreads();
      // online softmax on row orow, keys ocg*16 .. +16
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 16; ++i) mx = fmaxf(mx, sm.p[orow][ocg * 16 + i]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_new = fmaxf(m_run, mx);
      const float alpha = (m_run == -INFINITY) ? 0.f : expf(m_run - m_new);
      float ps = 0.f;
      float pr[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        pr[i] = expf(sm.p[orow][ocg * 16 + i] - m_new);
        ps += pr[i];
      }
      ps += __shfl_xor_sync(0xffffffffu, ps, 1);
      ps += __shfl_xor_sync(0xffffffffu, ps, 2);
      l_run = l_run * alpha + ps;
      m_run = m_new;
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 16; ++i) sm.p[orow][ocg * 16 + i] = pr[i];
      __syncthreads();
#pragma unroll
      for (int i = 0; i < OC; ++i) acc[i] *= alpha;
      for (int key = 0; key < kv; ++key) {
        const float pw = sm.p[orow][key];
#pragma unroll
        for (int i = 0; i < OC; ++i) acc[i] = fmaf(pw, sm.v[key][ocg * OC + i], acc[i]);
      }
    }
  }
  if (orow < rows_valid && VDN_IN_BOUNDS(r0 + orow < qrows, &g_simt_status)) {
    const float inv = 1.f / l_run;
    const long long rix = (long long)b * qrows + r0 + orow;
    if (G.qsrc == kQVideo) {
      TO* orow_ptr = o + rix * HD + (long long)h * D + ocg * OC;
#pragma unroll
      for (int i = 0; i < OC; ++i) orow_ptr[i] = from_f32<TO>(acc[i] * inv);
      if (lse && ocg == 0) lse[rix * l.H + h] = m_run + logf(l_run);
    } else {
      T* orow_ptr = (G.qsrc == kQText ? jn.ot : jn.oa) + rix * HD + (long long)h * D + ocg * OC;
#pragma unroll
      for (int i = 0; i < OC; ++i) orow_ptr[i] = from_f32<T>(acc[i] * inv);
      float* lp = G.qsrc == kQText ? jn.lse_t : jn.lse_a;
      if (lp && ocg == 0) lp[rix * l.H + h] = m_run + logf(l_run);
    }
  }
}

template <typename T, int D>
cudaError_t launch_simt_t(const Layout& l, const void* q, const void* k, const void* v,
                          const void* kt, const void* vt, void* o, bool out_f32, float* lse,
                          const JointArgs& ja, cudaStream_t st) {
  if (!out_f32 && std::is_same<T, float>::value) out_f32 = true;
  const SimtJoint<T> jn{(const T*)ja.k_audio, (const T*)ja.v_audio, (const T*)ja.q_text,
                        (const T*)ja.q_audio, (T*)ja.o_text, (T*)ja.o_audio, ja.lse_text,
                        ja.lse_audio};
  const int smem = (int)sizeof(SimtSmem<D>);
  dim3 grid(tiles_per_head(l, BQ), l.H, l.B);
  if (grid.x == 0) return cudaSuccess;
  if (out_f32) {
    auto kern = window_simt_kernel<T, float, D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    kern<<<grid, NT, smem, st>>>(l, (const T*)q, (const T*)k, (const T*)v, (const T*)kt,
                                 (const T*)vt, (float*)o, lse, jn);
    return cudaGetLastError();
  }
  auto kern = window_simt_kernel<T, T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<grid, NT, smem, st>>>(l, (const T*)q, (const T*)k, (const T*)v, (const T*)kt,
                               (const T*)vt, (T*)o, lse, jn);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_window_simt(const Layout& l, int dtype, const void* q, const void* k,
                               const void* v, const void* kt, const void* vt, void* o,
                               bool out_f32, float* lse, const JointArgs& ja, cudaStream_t st) {
  if (dtype == VDN_F32) {
    switch (l.d) {
      case 16: return launch_simt_t<float, 16>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
      case 32: return launch_simt_t<float, 32>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
      case 64: return launch_simt_t<float, 64>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
      case 128: return launch_simt_t<float, 128>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
    }
  } else {
    switch (l.d) {
      case 64: return launch_simt_t<__nv_bfloat16, 64>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
      case 128: return launch_simt_t<__nv_bfloat16, 128>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace vdn
