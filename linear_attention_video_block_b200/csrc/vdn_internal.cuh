// Internal declarations shared by the libvdn CUDA sources.
//
// The query-group schedule. Queries are partitioned into groups of rows that
// share one key set and one pair of VDA read states:
//   group 0          boundary frame 0          (sees every frame)
//   group 1          boundary frame F-1        (sees every frame; absent if F < 2)
//   group 2 + j      non-boundary frames of chunk j, j = 0 .. J-1 (may be empty)
//   group J + 2      text query rows  (joint layer only; dense over every key)
//   group J + 3      audio query rows (joint layer only; dense over every key)
// Tiles are enumerated in schedule order: the context groups (the heaviest:
// every key) first, then the boundary groups, then the chunks, so that the
// long tiles start early.
// Key set of a chunk group (project page "Local Softmax and Long-Range Linear
// Memory": each chunk attends to itself and both neighbour chunks, plus the
// 4-way boundary anchors and the text tokens): frames [lo, hi] with
// lo = max(0, c(j-1)), hi = min(F-1, c(j+2)-1), plus frames 0 and F-1, merged
// into at most 3 disjoint token intervals; the text keys and then the audio
// keys are separate segments seen by every group. Only the softmax launches of
// the joint layer set A or the context bits; the VDA kernels never see audio.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_bf16.h>

#include "../../include/vdn.h"

namespace vdn {

struct Layout {
  int B, F, N, T, c, H, d;
  int A = 0;       // audio tokens: softmax keys of every query, never written to VDA
  int ctx = 0;     // context query rows to compute: kCtxText | kCtxAudio
  __host__ __device__ long long L() const { return (long long)F * N; }
  __host__ __device__ int J() const { return (F + c - 1) / c; }
  __host__ __device__ int groups() const { return J() + 4; }
};

// ------------------------------------------------- argument validation
// Shared by every entry point of the C ABI (vdn_abi.cu, vda_noalloc.cu,
// host_pipeline.cu), so that their checks cannot drift apart.

inline bool layout_ok(const vdn_layout_t* l) {
  if (!l) return false;
  if (l->B < 1 || l->F < 1 || l->N < 1 || l->T < 0 || l->c < 1 || l->H < 1 || l->d < 1) return false;
  // token offsets and TMA coordinates are 32-bit signed per dimension
  const long long L = (long long)l->F * l->N;
  if (L > (1LL << 30) || l->T > (1 << 30)) return false;
  if ((long long)l->B * L * l->H * l->d > (1LL << 46)) return false;
  return true;
}

inline bool dtype_d_ok(int dtype, int d) {
  if (dtype == VDN_F32) return d == 16 || d == 32 || d == 64 || d == 128;
  if (dtype == VDN_BF16) return d == 64 || d == 128;
  return false;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline Layout to_layout(const vdn_layout_t* l) {
  Layout x;
  x.B = l->B; x.F = l->F; x.N = l->N; x.T = l->T; x.c = l->c; x.H = l->H; x.d = l->d;
  return x;
}

// VDN_OK for cudaSuccess; otherwise records e as the calling host thread's
// last CUDA error (vdn_last_cuda_error) and returns VDN_ERR_CUDA.
int cuda_status(cudaError_t e);

// vdn_hybrid_attn_fwd with two waits on the stream: before_window (the
// softmax branch's inputs q, k, v) and before_combine (the gates), so that a
// caller streaming its inputs in can start the linear branch once k, v and
// beta have arrived. Either event may be null.
int hybrid_staged(const vdn_layout_t* layout, int dtype, const void* q, const void* k, const void* v,
                  const void* k_text, const void* v_text, const float* beta, const float* beta_text,
                  const void* g_soft, const void* g_lin, const float* rms_weight, float rms_eps, void* out,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream, cudaEvent_t before_window,
                  cudaEvent_t before_combine);

// Bound checks of the checked build (-DVDN_BOUND_CHECKS): VDN_IN_BOUNDS(cond,
// status) is true when cond holds; otherwise it records VDN_ERR_BOUNDS in the
// device status word *status and is false, and the caller skips the access
// (no trap, so a failed check never takes the GPU context down). In the
// regular build it is the constant true and costs nothing.
#ifdef VDN_BOUND_CHECKS
#define VDN_IN_BOUNDS(cond, status) \
  ((cond) ? true : (atomicCAS((status), 0, (int)VDN_ERR_BOUNDS), false))
#else
#define VDN_IN_BOUNDS(cond, status) true
#endif

constexpr int kCtxText = 1;
constexpr int kCtxAudio = 2;

// Query source of a group: video tokens, text query rows or audio query rows.
enum QuerySource { kQVideo = 0, kQText = 1, kQAudio = 2 };

struct Group {
  int qsrc;        // QuerySource
  int q0;          // first query token of the group (in its source tensor)
  int nq;          // number of query tokens (0 = empty group)
  int nseg;        // video key segments
  int seg0[3];     // segment start token
  int segn[3];     // segment length in tokens
  int chunk;       // chunk index (-1 for boundary groups)
  int fwd_idx;     // forward state index: state after frames 1..fwd_idx (0 = S0)
  int rev_idx;     // reverse state index: state after frames F-2..rev_idx (F-1 = S0)
};

__host__ __device__ inline void chunk_window(const Layout& l, int j, int& lo, int& hi) {
  lo = l.c * (j - 1);
  if (lo < 0) lo = 0;
  hi = l.c * (j + 2) - 1;
  if (hi > l.F - 1) hi = l.F - 1;
}

__host__ __device__ inline Group make_group(const Layout& l, int g) {
  Group G;
  G.qsrc = kQVideo;
  G.nseg = 0;
  G.chunk = -1;
  G.fwd_idx = 0;
  G.rev_idx = l.F - 1;
  for (int s = 0; s < 3; ++s) { G.seg0[s] = 0; G.segn[s] = 0; }
  const int N = l.N, F = l.F;
  if (g >= l.J() + 2) {
    // context query rows: every video token is a key
    const bool text = g == l.J() + 2;
    G.qsrc = text ? kQText : kQAudio;
    G.q0 = 0;
    G.nq = text ? ((l.ctx & kCtxText) ? l.T : 0) : ((l.ctx & kCtxAudio) ? l.A : 0);
    G.nseg = 1;
    G.seg0[0] = 0;
    G.segn[0] = F * N;
    return G;
  }
  if (g == 0 || g == 1) {
    int f = (g == 0) ? 0 : F - 1;
    if (g == 1 && F < 2) { G.q0 = 0; G.nq = 0; return G; }
    G.q0 = f * N;
    G.nq = N;
    G.nseg = 1;
    G.seg0[0] = 0;
    G.segn[0] = F * N;
    return G;
  }
  int j = g - 2;
  int f0 = j * l.c, f1 = (j + 1) * l.c - 1;
  if (f0 < 1) f0 = 1;
  if (f1 > F - 2) f1 = F - 2;
  G.chunk = j;
  if (f1 < f0) { G.q0 = 0; G.nq = 0; return G; }
  G.q0 = f0 * N;
  G.nq = (f1 - f0 + 1) * N;
  int lo, hi;
  chunk_window(l, j, lo, hi);
  // frames {0} u [lo, hi] u {F-1}, merged
  int a = lo, b = hi;
  if (a <= 1) a = 0; else { G.seg0[G.nseg] = 0; G.segn[G.nseg] = N; G.nseg++; }
  bool tail_merged = (b >= F - 2);
  if (tail_merged) b = F - 1;
  G.seg0[G.nseg] = a * N; G.segn[G.nseg] = (b - a + 1) * N; G.nseg++;
  if (!tail_merged) { G.seg0[G.nseg] = (F - 1) * N; G.segn[G.nseg] = N; G.nseg++; }
  G.fwd_idx = (lo - 1 >= 1) ? lo - 1 : 0;
  G.rev_idx = (hi + 1 <= F - 2) ? hi + 1 : F - 1;
  return G;
}

// Group at position i of the schedule order (context groups first).
__host__ __device__ inline int sched_group(const Layout& l, int i) {
  return i < 2 ? l.J() + 2 + i : i - 2;
}

// Per-(b, h) tile enumeration over groups in schedule order: tile t of
// `rows`-row tiles.
__host__ __device__ inline int tiles_per_head(const Layout& l, int rows) {
  int n = 0;
  for (int i = 0; i < l.groups(); ++i) {
    Group G = make_group(l, sched_group(l, i));
    n += (G.nq + rows - 1) / rows;
  }
  return n;
}

__host__ __device__ inline void tile_to_group(const Layout& l, int rows, int t, int& g, int& r0) {
  for (int i = 0; i < l.groups(); ++i) {
    g = sched_group(l, i);
    Group G = make_group(l, g);
    int n = (G.nq + rows - 1) / rows;
    if (t < n) { r0 = G.q0 + t * rows; return; }
    t -= n;
  }
  g = -1;
  r0 = 0;
}

// Key tile t of a query group (tiles of `keys` keys): video segments first,
// then the text keys, then the audio keys.
enum KeySource { kKVideo = 0, kKText = 1, kKAudio = 2 };
struct KeyTile {
  int src;    // KeySource: which tensor the rows index
  int row;    // first key row of the tile
  int valid;  // keys of the tile that belong to the segment (<= keys)
};

// (The loops below run over the at most 3 video segments with compile-time
// indices, so a Group stays in registers on the device.)
__host__ __device__ inline int key_tile_count(const Group& G, int T, int A, int keys) {
  int n = 0;
#pragma unroll
  for (int s = 0; s < 3; ++s)
    if (s < G.nseg) n += (G.segn[s] + keys - 1) / keys;
  return n + (T + keys - 1) / keys + (A + keys - 1) / keys;
}

__host__ __device__ inline KeyTile key_tile(const Group& G, int T, int A, int t, int keys) {
  KeyTile k{kKText, 0, 0};
  bool found = false;
  int first = 0;  // first tile index of segment s
#pragma unroll
  for (int s = 0; s < 3; ++s) {
    const int n = (s < G.nseg) ? (G.segn[s] + keys - 1) / keys : 0;
    if (!found && t < first + n) {
      k.src = kKVideo;
      k.row = G.seg0[s] + (t - first) * keys;
      k.valid = G.segn[s] - (t - first) * keys;
      found = true;
    }
    first += n;
  }
  if (!found) {
    const int nt = (T + keys - 1) / keys;
    if (t < first + nt) {
      k.row = (t - first) * keys;
      k.valid = T - (t - first) * keys;
    } else {
      k.src = kKAudio;
      k.row = (t - first - nt) * keys;
      k.valid = A - (t - first - nt) * keys;
    }
  }
  if (k.valid > keys) k.valid = keys;
  return k;
}

// Scan extents: forward scan runs frames 1..fwd_max, reverse scan frames
// F-2 down to rev_min (rev_min = F-1 means no reverse frame).
inline void scan_extent(const Layout& l, int& fwd_max, int& rev_min) {
  fwd_max = 0;
  rev_min = l.F - 1;
  for (int j = 0; j < l.J(); ++j) {
    Group G = make_group(l, 2 + j);
    if (G.nq == 0) continue;
    if (G.fwd_idx > fwd_max) fwd_max = G.fwd_idx;
    if (G.rev_idx < rev_min) rev_min = G.rev_idx;
  }
}

template <typename T> __device__ inline float to_f32(T x);
template <> __device__ inline float to_f32<float>(float x) { return x; }
template <> __device__ inline float to_f32<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ inline T from_f32(float x);
template <> __device__ inline float from_f32<float>(float x) { return x; }
template <> __device__ inline __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// ---------------------------------------------------------------- launchers
// Each returns cudaGetLastError() after its launch(es).

// Audio keys and the context query rows of a joint layer (all null / unused
// when l.A == 0 and l.ctx == 0). Tensors [B, A, H, d] / [B, T, H, d] in the io
// dtype; the context outputs are written in the io dtype.
struct JointArgs {
  const void* k_audio = nullptr;
  const void* v_audio = nullptr;
  const void* q_text = nullptr;
  const void* q_audio = nullptr;
  void* o_text = nullptr;
  void* o_audio = nullptr;
  float* lse_text = nullptr;   // [B, T, H], nullable
  float* lse_audio = nullptr;  // [B, A, H], nullable
};

// SIMT window softmax (any supported dtype/d); o_soft in the io dtype, or in
// float32 when out_f32 (the hybrid path's intermediate).
cudaError_t launch_window_simt(const Layout& l, int dtype, const void* q, const void* k,
                               const void* v, const void* kt, const void* vt, void* o,
                               bool out_f32, float* lse, const JointArgs& ja, cudaStream_t st);
// tcgen05 window softmax (bf16, d in {64, 128}).
bool window_tc_supported(const Layout& l, int dtype);
cudaError_t launch_window_tc(const Layout& l, const void* q, const void* k, const void* v,
                             const void* kt, const void* vt, void* o, bool out_f32, float* lse,
                             const JointArgs& ja, cudaStream_t st);

// FP8 (e4m3) window softmax (d = 128; no audio keys or context rows): scores
// scaled by qk_scale / sqrt(d), output (bf16) by v_scale.
cudaError_t launch_window_fp8(const Layout& l, const void* q, const void* k, const void* v,
                              const void* kt, const void* vt, float qk_scale, float v_scale,
                              void* o, float* lse, cudaStream_t st);
cudaError_t read_and_clear_fp8_status(int* status);

// Reads and clears the device status word of the tcgen05 kernels' translation
// unit (bounded waits record VDN_ERR_TIMEOUT there).
cudaError_t read_and_clear_tc_status(int* status);

// Status words of the CUDA-core kernels' translation units (only the bound
// checks of the checked build write them).
cudaError_t read_and_clear_simt_status(int* status);
cudaError_t read_and_clear_vda_status(int* status);
cudaError_t read_and_clear_ro32_status(int* status);
cudaError_t read_and_clear_combine_status(int* status);

// Role-wait limit of each tcgen05 translation unit (0: the 4 s default).
cudaError_t set_role_wait_tc(unsigned long long ns);
cudaError_t set_role_wait_gram(unsigned long long ns);
cudaError_t set_role_wait_readout(unsigned long long ns);
cudaError_t set_role_wait_fp8(unsigned long long ns);

// tcgen05 frame Gram (bf16, d in {64, 128}) into the (am, bw) slots.
bool gram_tc_supported(const Layout& l, int dtype);
cudaError_t launch_gram_tc(const Layout& l, int has_text, int fwd_max, int rev_lo, int nslots,
                           const void* k, const void* v, const void* kt, const void* vt,
                           const float* beta, const float* beta_t, float* am, float* bw,
                           cudaStream_t st);
cudaError_t read_and_clear_gram_status(int* status);

// tcgen05 linear readout o_lin = S_sum q (bf16 q, d in {64, 128}); o_lin in
// bf16, or in float32 when out_f32.
bool readout_tc_supported(const Layout& l, int dtype);
cudaError_t launch_readout_tc(const Layout& l, const void* q, const float* states, void* o_lin,
                              bool out_f32, cudaStream_t st);
cudaError_t read_and_clear_readout_status(int* status);

// The same readout finishing the hybrid output instead of writing o_lin:
// out = sig(gs) o_soft + sig(gl) RMSNorm(o_lin) (o_soft: fp32 [B, L, H, d] from
// the window kernel; boundary frames: out = sig(gs) o_soft); out_soft and
// out_lin (nullable) receive the two gated branches.
cudaError_t launch_combine_tc(const Layout& l, const void* q, const float* states,
                              const float* o_soft, const void* gs, const void* gl,
                              const float* rms_w, float eps, void* out, void* out_soft,
                              void* out_lin, cudaStream_t st);

// out = sig(gs) o_soft + sig(gl) RMSNorm_d(o_lin) over rows x d elements: o_soft
// and o_lin float32 [rows, d], the gates and out in the io dtype (a
// token-sharded combine of the two branches computed elsewhere).
cudaError_t launch_gated_combine(long long rows, int d, int dtype, const void* o_soft,
                                 const void* o_lin, const void* gs, const void* gl,
                                 const float* rms_w, float eps, void* out, cudaStream_t st);

// VDA: Gram into (am, bw) slots [B, H, F, d, d] (slot 0 = text), inverse in place
// of am, scans into states [B, H, 2, J, d, d]. alpha (nullable) [B, F, H, d]: KDA
// channel decay applied to the state before each frame is written.
cudaError_t launch_vda_states(const Layout& l, int dtype, const void* k, const void* v,
                              const void* kt, const void* vt, const float* beta,
                              const float* beta_text, const float* alpha, float* am, float* bw,
                              float* states, cudaStream_t st);

// Readout / norm / gates. mode 0: o_lin only (ungated, pre-norm) into out.
// mode 1: out = sig(gs) o_soft + sig(gl) rms(o_lin); optional out_soft/out_lin.
// o_soft is float32 [B, L, H, d].
cudaError_t launch_readout(const Layout& l, int dtype, int mode, const void* q,
                           const float* states, const float* o_soft, const void* gs,
                           const void* gl, const float* rms_w, float eps, void* out,
                           void* out_soft, void* out_lin, cudaStream_t st);

}  // namespace vdn
