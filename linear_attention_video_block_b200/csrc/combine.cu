// Gated combine of the two branch outputs (project page, "Gating the Softmax
// and Linear Branch Outputs"): out = sigmoid(g_s) o_soft + sigmoid(g_l)
// RMSNorm_d(o_lin), per (token, head) row of d elements, RMSNorm with eps and
// an optional weight. This is the last step of the hybrid forward when the two
// branches have run apart (on different GPUs of a branch-specialised split)
// and their outputs have been brought back to the token shard that owns the
// gates. Token-wise, so it needs no frame structure: rows = tokens x heads.
//
// The two branch outputs arrive in float32 (the forms the branch entries
// write with _f32out): exchanged in bf16 they would each carry a rounding of
// their own into the output, beyond the tolerance of the op, while the hybrid
// entry combines float32 branches and rounds once. The gates and out are in
// the io dtype.
//
// HBM-bound: per row it reads o_soft, o_lin, g_s, g_l and writes out, once.
// Each thread owns 8 consecutive elements of a row (16-byte loads of the
// bf16 gates), so d / 8 neighbouring lanes share a row and reduce its sum of
// squares with shuffles.
#include "vdn_internal.cuh"

namespace vdn {

// Device status word of this translation unit (bound checks of the checked build).
__device__ int g_combine_status = 0;

cudaError_t read_and_clear_combine_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_combine_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_combine_status, &zero, sizeof(int));
}

namespace {

constexpr int kCombineThreads = 256;

__device__ inline float sigmoid_c(float x) { return 1.f / (1.f + expf(-x)); }

template <typename T>
struct Vec8;
template <>
struct Vec8<__nv_bfloat16> {
  static __device__ inline void load(const __nv_bfloat16* p, float* x) {
    const uint4 u = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = *reinterpret_cast<const __nv_bfloat162*>(&w[i]);
      x[2 * i] = __low2float(h);
      x[2 * i + 1] = __high2float(h);
    }
  }
  static __device__ inline void store(__nv_bfloat16* p, const float* x) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};
template <>
struct Vec8<float> {
  static __device__ inline void load(const float* p, float* x) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  }
  static __device__ inline void store(float* p, const float* x) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  }
};

template <typename T, int D>
__global__ void __launch_bounds__(kCombineThreads)
combine_kernel(long long rows, const float* __restrict__ o_soft, const float* __restrict__ o_lin,
               const T* __restrict__ gs, const T* __restrict__ gl, const float* __restrict__ rms_w,
               float eps, T* __restrict__ out) {
  constexpr int kLanes = D / 8;                      // threads per row: 2, 4, 8 or 16
  constexpr int kRowsPerBlock = kCombineThreads / kLanes;
  const int sub = threadIdx.x % kLanes;
  const int c0 = sub * 8;
  float w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) w[i] = rms_w ? rms_w[c0 + i] : 1.f;
  for (long long r0 = (long long)blockIdx.x * kRowsPerBlock; r0 < rows;
       r0 += (long long)gridDim.x * kRowsPerBlock) {
    const long long row = r0 + threadIdx.x / kLanes;
    // rows past the end still take part in the shuffles (with zeros)
    const bool live = row < rows && VDN_IN_BOUNDS(c0 + 8 <= D, &g_combine_status);
    const long long off = (live ? row : 0) * D + c0;
    float lin[8], ss = 0.f;
    if (live) Vec8<float>::load(o_lin + off, lin);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      if (!live) lin[i] = 0.f;
      ss = fmaf(lin[i], lin[i], ss);
    }
#pragma unroll
    for (int m = 1; m < kLanes; m <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, m);
    if (!live) continue;
    const float rstd = rsqrtf(ss / (float)D + eps);
    float sm[8], a[8], b[8], o[8];
    Vec8<float>::load(o_soft + off, sm);
    Vec8<T>::load(gs + off, a);
    Vec8<T>::load(gl + off, b);
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = sigmoid_c(a[i]) * sm[i] + sigmoid_c(b[i]) * (lin[i] * rstd * w[i]);
    Vec8<T>::store(out + off, o);
  }
}

template <typename T, int D>
cudaError_t launch_combine_t(long long rows, const void* o_soft, const void* o_lin, const void* gs,
                             const void* gl, const float* rms_w, float eps, void* out,
                             cudaStream_t st) {
  constexpr int kRowsPerBlock = kCombineThreads / (D / 8);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // a grid of whole waves (8 resident blocks of 256 threads per SM), grid-stride
  const long long need = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  const long long cap = (long long)sms * 8;
  const int grid = (int)(need < cap ? need : cap);
  if (grid == 0) return cudaSuccess;
  combine_kernel<T, D><<<grid, kCombineThreads, 0, st>>>(
      rows, static_cast<const float*>(o_soft), static_cast<const float*>(o_lin), static_cast<const T*>(gs),
      static_cast<const T*>(gl), rms_w, eps, static_cast<T*>(out));
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gated_combine(long long rows, int d, int dtype, const void* o_soft,
                                 const void* o_lin, const void* gs, const void* gl,
                                 const float* rms_w, float eps, void* out, cudaStream_t st) {
#define VDN_CB(T, D) return launch_combine_t<T, D>(rows, o_soft, o_lin, gs, gl, rms_w, eps, out, st)
  if (dtype == VDN_F32) {
    switch (d) {
      case 16: VDN_CB(float, 16);
      case 32: VDN_CB(float, 32);
      case 64: VDN_CB(float, 64);
      case 128: VDN_CB(float, 128);
    }
  } else if (dtype == VDN_BF16) {
    switch (d) {
      case 64: VDN_CB(__nv_bfloat16, 64);
      case 128: VDN_CB(__nv_bfloat16, 128);
    }
  }
#undef VDN_CB
  return cudaErrorInvalidValue;
}

}  // namespace vdn
