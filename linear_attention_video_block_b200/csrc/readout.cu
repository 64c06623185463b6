// Linear-branch readout, RMSNorm, gates and combine (project page, "Local
// Softmax and Long-Range Linear Memory" for the summed bidirectional readout,
// "Gating the Softmax and Linear Branch Outputs" for the gates and RMSNorm).
//
// One CTA = 64 query rows of one query group of one (b, h). All rows of a
// chunk group read the same S_sum = S_fwd + S_rev (chunk table), which is
// staged once in shared memory, transposed; boundary groups have o_lin = 0.
//   mode 0: writes o_lin = S_sum q (ungated, before RMSNorm).
//   mode 1: writes out = sigmoid(g_s) o_soft + sigmoid(g_l) RMSNorm(o_lin), and
//           optionally the two gated branches.
#include "vdn_internal.cuh"

namespace vdn {

// Device status word of this translation unit (bound checks of the checked build).
__device__ int g_ro32_status = 0;

cudaError_t read_and_clear_ro32_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_ro32_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_ro32_status, &zero, sizeof(int));
}

namespace {

constexpr int BQ = 64;
constexpr int NT = 256;

__device__ inline float sigmoidf_(float x) { return 1.f / (1.f + expf(-x)); }

template <typename T, int D>
__global__ void __launch_bounds__(NT)
readout_kernel(Layout l, int mode, const T* __restrict__ q, const float* __restrict__ states,
               const float* __restrict__ o_soft, const T* __restrict__ gs, const T* __restrict__ gl,
               const float* __restrict__ rms_w, float eps, T* __restrict__ out,
               T* __restrict__ out_soft, T* __restrict__ out_lin) {
  extern __shared__ __align__(16) float ro_smem[];
  float* st = ro_smem;            // [D][D] transposed: st[j * D + i] = S_sum[i][j]
  float* qs = st + D * D;         // [BQ][D]
  const int tid = threadIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  int g, r0;
  tile_to_group(l, BQ, blockIdx.x, g, r0);
  if (g < 0) return;
  const Group G = make_group(l, g);
  const int rows_valid = min(BQ, G.q0 + G.nq - r0);
  const bool has_lin = G.chunk >= 0 && VDN_IN_BOUNDS(G.chunk < l.J(), &g_ro32_status);
  const long long L = l.L();
  const long long HD = (long long)l.H * D;
  if (has_lin) {
    const int J = l.J();
    const float* sf = states + ((((long long)b * l.H + h) * 2 + 0) * J + G.chunk) * D * D;
    const float* sr = states + ((((long long)b * l.H + h) * 2 + 1) * J + G.chunk) * D * D;
    for (int i = tid; i < D * D; i += NT) {
      int r = i / D, cidx = i % D;
      st[cidx * D + r] = sf[i] + sr[i];
    }
    for (int i = tid; i < BQ * D; i += NT) {
      int r = i / D, cidx = i % D;
      const bool in = r < rows_valid && VDN_IN_BOUNDS(r0 + r < L, &g_ro32_status);
      qs[i] = in ? to_f32(q[((long long)b * L + r0 + r) * HD + (long long)h * D + cidx]) : 0.f;
    }
  }
  __syncthreads();
  const int row = tid / 4, cg = tid % 4;
  constexpr int OC = D / 4;
  const int c0 = cg * OC;
  float acc[OC];
#pragma unroll
  for (int i = 0; i < OC; ++i) acc[i] = 0.f;
  if (has_lin) {
    for (int j = 0; j < D; ++j) {
      const float qv = qs[row * D + j];
#pragma unroll
      for (int i = 0; i < OC; ++i) acc[i] = fmaf(st[j * D + c0 + i], qv, acc[i]);
    }
  }
  // the 4 lanes of a row reduce the sum of squares before any lane leaves
  float ss = 0.f;
#pragma unroll
  for (int i = 0; i < OC; ++i) ss = fmaf(acc[i], acc[i], ss);
  ss += __shfl_xor_sync(0xffffffffu, ss, 1);
  ss += __shfl_xor_sync(0xffffffffu, ss, 2);
  if (row >= rows_valid || !VDN_IN_BOUNDS(r0 + row < L, &g_ro32_status)) return;
  const long long base = ((long long)b * L + r0 + row) * HD + (long long)h * D + c0;
  if (mode == 0) {
#pragma unroll
    for (int i = 0; i < OC; ++i) out[base + i] = from_f32<T>(acc[i]);
    return;
  }
  const float rstd = rsqrtf(ss / (float)D + eps);
#pragma unroll
  for (int i = 0; i < OC; ++i) {
    const float w = rms_w ? rms_w[c0 + i] : 1.f;
    const float a = sigmoidf_(to_f32(gs[base + i])) * o_soft[base + i];
    const float bb = sigmoidf_(to_f32(gl[base + i])) * (acc[i] * rstd * w);
    out[base + i] = from_f32<T>(a + bb);
    if (out_soft) out_soft[base + i] = from_f32<T>(a);
    if (out_lin) out_lin[base + i] = from_f32<T>(bb);
  }
}

template <typename T, int D>
cudaError_t launch_readout_t(const Layout& l, int mode, const void* q, const float* states,
                             const float* o_soft, const void* gs, const void* gl,
                             const float* rms_w, float eps, void* out, void* out_soft,
                             void* out_lin, cudaStream_t st) {
  auto kern = readout_kernel<T, D>;
  const int smem = (D * D + BQ * D) * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles_per_head(l, BQ), l.H, l.B);
  if (grid.x == 0) return cudaSuccess;
  kern<<<grid, NT, smem, st>>>(l, mode, (const T*)q, states, o_soft, (const T*)gs,
                               (const T*)gl, rms_w, eps, (T*)out, (T*)out_soft, (T*)out_lin);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_readout(const Layout& l, int dtype, int mode, const void* q,
                           const float* states, const float* o_soft, const void* gs,
                           const void* gl, const float* rms_w, float eps, void* out,
                           void* out_soft, void* out_lin, cudaStream_t st) {
#define VDN_RO(T, D) \
  return launch_readout_t<T, D>(l, mode, q, states, o_soft, gs, gl, rms_w, eps, out, out_soft, out_lin, st)
  if (dtype == VDN_F32) {
    switch (l.d) {
      case 16: VDN_RO(float, 16);
      case 32: VDN_RO(float, 32);
      case 64: VDN_RO(float, 64);
      case 128: VDN_RO(float, 128);
    }
  } else {
    switch (l.d) {
      case 64: VDN_RO(__nv_bfloat16, 64);
      case 128: VDN_RO(__nv_bfloat16, 128);
    }
  }
#undef VDN_RO
  return cudaErrorInvalidValue;
}

}  // namespace vdn
