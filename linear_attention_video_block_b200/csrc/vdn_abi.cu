// libvdn C ABI: argument checks, workspace carving and launch sequencing on
// the caller's stream. Every step of the operation runs in the kernels of this
// library; the host code only validates and launches.
#include <cstdint>

#include "vdn_internal.cuh"

namespace vdn {

// The CUDA error behind the last VDN_ERR_CUDA returned on this host thread.
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return VDN_OK;
  t_last_cuda_error = e;
  return VDN_ERR_CUDA;
}

}  // namespace vdn

namespace {

using vdn::Layout;
using vdn::aligned16;
using vdn::cuda_status;
using vdn::dtype_d_ok;
using vdn::layout_ok;
using vdn::to_layout;

constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Workspace {
  float* am = nullptr;
  float* bw = nullptr;
  float* states = nullptr;
  float* o_soft = nullptr;  // float32 softmax-branch output of the hybrid path
  size_t bytes = 0;
};

// Carves the workspace; with base == nullptr only computes the size.
Workspace carve(const Layout& l, int dtype, void* base, bool need_states, bool need_osoft) {
  Workspace w;
  const size_t dd = (size_t)l.d * l.d;
  const size_t bh = (size_t)l.B * l.H;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  auto take = [&](size_t n) -> void* {
    void* r = p ? p + off : nullptr;
    off = align_up(off + n);
    return r;
  };
  w.am = static_cast<float*>(take(bh * l.F * dd * sizeof(float)));
  w.bw = static_cast<float*>(take(bh * l.F * dd * sizeof(float)));
  if (need_states) w.states = static_cast<float*>(take(bh * 2 * l.J() * dd * sizeof(float)));
  if (need_osoft) w.o_soft = static_cast<float*>(take((size_t)l.B * l.L() * l.H * l.d * sizeof(float)));
  w.bytes = off;
  return w;
}

int run_window(const Layout& l, int dtype, const void* q, const void* k, const void* v,
               const void* kt, const void* vt, void* o, bool out_f32, float* lse,
               const vdn::JointArgs& ja, cudaStream_t st) {
  if (vdn::window_tc_supported(l, dtype))
    return cuda_status(vdn::launch_window_tc(l, q, k, v, kt, vt, o, out_f32, lse, ja, st));
  return cuda_status(vdn::launch_window_simt(l, dtype, q, k, v, kt, vt, o, out_f32, lse, ja, st));
}

// Validates the joint-layer context and returns the softmax launches' layout
// (audio count and context query bits set) and tensors. ctx == nullptr: a
// video-only call.
int joint_setup(const vdn_layout_t* layout, const vdn_context_t* ctx, Layout& ls,
                vdn::JointArgs& ja) {
  ls = to_layout(layout);
  ja = vdn::JointArgs{};
  if (!ctx) return VDN_OK;
  const int A = ctx->A;
  if (A < 0 || A > (1 << 30)) return VDN_ERR_INVALID;
  if ((long long)layout->B * A * layout->H * layout->d > (1LL << 46)) return VDN_ERR_INVALID;
  if (A > 0 && (!ctx->k_audio || !ctx->v_audio)) return VDN_ERR_INVALID;
  const bool text_rows = ctx->q_text != nullptr && layout->T > 0;
  const bool audio_rows = ctx->q_audio != nullptr && A > 0;
  if (text_rows && !ctx->o_text) return VDN_ERR_INVALID;
  if (audio_rows && !ctx->o_audio) return VDN_ERR_INVALID;
  const void* ptrs[] = {A > 0 ? ctx->k_audio : nullptr, A > 0 ? ctx->v_audio : nullptr,
                        text_rows ? ctx->q_text : nullptr, text_rows ? ctx->o_text : nullptr,
                        text_rows ? ctx->lse_text : nullptr, audio_rows ? ctx->q_audio : nullptr,
                        audio_rows ? ctx->o_audio : nullptr, audio_rows ? ctx->lse_audio : nullptr};
  for (const void* p : ptrs) if (p && !aligned16(p)) return VDN_ERR_UNSUPPORTED;
  ls.A = A;
  ls.ctx = (text_rows ? vdn::kCtxText : 0) | (audio_rows ? vdn::kCtxAudio : 0);
  if (A > 0) { ja.k_audio = ctx->k_audio; ja.v_audio = ctx->v_audio; }
  if (text_rows) { ja.q_text = ctx->q_text; ja.o_text = ctx->o_text; ja.lse_text = ctx->lse_text; }
  if (audio_rows) {
    ja.q_audio = ctx->q_audio; ja.o_audio = ctx->o_audio; ja.lse_audio = ctx->lse_audio;
  }
  return VDN_OK;
}

int window_impl(const vdn_layout_t* layout, int dtype, const vdn_context_t* ctx, const void* q,
                const void* k, const void* v, const void* k_text, const void* v_text,
                void* o_soft, float* lse, cudaStream_t stream, bool out_f32 = false) {
  if (!layout_ok(layout)) return VDN_ERR_INVALID;
  if (!dtype_d_ok(dtype, layout->d)) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o_soft) return VDN_ERR_INVALID;
  if (layout->T > 0 && (!k_text || !v_text)) return VDN_ERR_INVALID;
  const void* ptrs[] = {q, k, v, o_soft, lse};
  for (const void* p : ptrs) if (p && !aligned16(p)) return VDN_ERR_UNSUPPORTED;
  if (layout->T > 0 && (!aligned16(k_text) || !aligned16(v_text))) return VDN_ERR_UNSUPPORTED;
  Layout ls;
  vdn::JointArgs ja;
  const int s = joint_setup(layout, ctx, ls, ja);
  if (s != VDN_OK) return s;
  return run_window(ls, dtype, q, k, v, layout->T ? k_text : nullptr,
                    layout->T ? v_text : nullptr, o_soft, out_f32, lse, ja, stream);
}

}  // namespace

extern "C" {

size_t vdn_workspace_bytes(const vdn_layout_t* layout, int dtype) {
  if (!layout_ok(layout) || !dtype_d_ok(dtype, layout->d)) return 0;
  const Layout l = to_layout(layout);
  return carve(l, dtype, nullptr, true, true).bytes;
}

int vdn_window_softmax_fwd(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                           const void* v, const void* k_text, const void* v_text, void* o_soft,
                           float* lse, cudaStream_t stream) {
  return window_impl(layout, dtype, nullptr, q, k, v, k_text, v_text, o_soft, lse, stream);
}

int vdn_window_softmax_fwd_f32out(const vdn_layout_t* layout, int dtype, const void* q,
                                  const void* k, const void* v, const void* k_text,
                                  const void* v_text, float* o_soft, float* lse,
                                  cudaStream_t stream) {
  return window_impl(layout, dtype, nullptr, q, k, v, k_text, v_text, o_soft, lse, stream, true);
}

int vdn_window_softmax_fwd_fp8(const vdn_layout_t* layout, const void* q, const void* k,
                               const void* v, const void* k_text, const void* v_text, float q_scale,
                               float k_scale, float v_scale, void* o_soft, float* lse,
                               cudaStream_t stream) {
  if (!layout_ok(layout)) return VDN_ERR_INVALID;
  if (layout->d != 128) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !o_soft) return VDN_ERR_INVALID;
  if (layout->T > 0 && (!k_text || !v_text)) return VDN_ERR_INVALID;
  const float sc[3] = {q_scale, k_scale, v_scale};
  for (float x : sc)
    if (!(x > 0.f) || !(x < INFINITY)) return VDN_ERR_INVALID;
  const void* ptrs[] = {q, k, v, o_soft, lse};
  for (const void* p : ptrs) if (p && !aligned16(p)) return VDN_ERR_UNSUPPORTED;
  if (layout->T > 0 && (!aligned16(k_text) || !aligned16(v_text))) return VDN_ERR_UNSUPPORTED;
  const Layout l = to_layout(layout);
  return cuda_status(vdn::launch_window_fp8(l, q, k, v, layout->T ? k_text : nullptr,
                                            layout->T ? v_text : nullptr, q_scale * k_scale, v_scale,
                                            o_soft, lse, stream));
}

int vdn_joint_softmax_fwd(const vdn_layout_t* layout, int dtype, const vdn_context_t* ctx,
                          const void* q, const void* k, const void* v, const void* k_text,
                          const void* v_text, void* o_soft, float* lse, cudaStream_t stream) {
  if (!ctx) return VDN_ERR_INVALID;
  return window_impl(layout, dtype, ctx, q, k, v, k_text, v_text, o_soft, lse, stream);
}

}  // extern "C"

namespace {

int vda_scan_impl(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                  const void* v, const void* k_text, const void* v_text, const float* beta,
                  const float* beta_text, const float* alpha, void* o_lin, float* chunk_states,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream,
                  bool out_f32 = false) {
  if (!layout_ok(layout)) return VDN_ERR_INVALID;
  if (!dtype_d_ok(dtype, layout->d)) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !beta || !o_lin) return VDN_ERR_INVALID;
  if (layout->T > 0 && (!k_text || !v_text || !beta_text)) return VDN_ERR_INVALID;
  const void* ptrs[] = {q, k, v, beta, alpha, o_lin, chunk_states, workspace};
  for (const void* p : ptrs) if (p && !aligned16(p)) return VDN_ERR_UNSUPPORTED;
  if (layout->T > 0 && (!aligned16(k_text) || !aligned16(v_text) || !aligned16(beta_text)))
    return VDN_ERR_UNSUPPORTED;
  const Layout l = to_layout(layout);
  const bool own_states = chunk_states == nullptr;
  const Workspace need = carve(l, dtype, nullptr, own_states, false);
  if (!workspace || workspace_bytes < need.bytes) return VDN_ERR_WORKSPACE;
  const Workspace w = carve(l, dtype, workspace, own_states, false);
  float* states = own_states ? w.states : chunk_states;
  const void* kt = layout->T ? k_text : nullptr;
  const void* vt = layout->T ? v_text : nullptr;
  const float* bt = layout->T ? beta_text : nullptr;
  int s = cuda_status(vdn::launch_vda_states(l, dtype, k, v, kt, vt, beta, bt, alpha, w.am, w.bw,
                                             states, stream));
  if (s != VDN_OK) return s;
  if (vdn::readout_tc_supported(l, dtype))
    return cuda_status(vdn::launch_readout_tc(l, q, states, o_lin, out_f32, stream));
  // the CUDA-core readout serves fp32 tensors, whose o_lin is float32 anyway
  return cuda_status(vdn::launch_readout(l, dtype, 0, q, states, nullptr, nullptr, nullptr, nullptr,
                                         0.f, o_lin, nullptr, nullptr, stream));
}

int hybrid_impl(const vdn_layout_t* layout, int dtype, const vdn_context_t* ctx, const void* q,
                const void* k, const void* v, const void* k_text, const void* v_text,
                const float* beta, const float* beta_text, const float* alpha, const void* g_soft,
                const void* g_lin, const float* rms_weight, float rms_eps, void* out,
                void* out_soft, void* out_lin, void* workspace, size_t workspace_bytes,
                cudaStream_t stream, cudaEvent_t before_window = nullptr,
                cudaEvent_t before_combine = nullptr) {
  if (!layout_ok(layout)) return VDN_ERR_INVALID;
  if (!dtype_d_ok(dtype, layout->d)) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !beta || !g_soft || !g_lin || !out) return VDN_ERR_INVALID;
  if (layout->T > 0 && (!k_text || !v_text || !beta_text)) return VDN_ERR_INVALID;
  if (!(rms_eps >= 0.f)) return VDN_ERR_INVALID;
  const void* ptrs[] = {q, k, v, beta, alpha, g_soft, g_lin, rms_weight, out, out_soft, out_lin, workspace};
  for (const void* p : ptrs) if (p && !aligned16(p)) return VDN_ERR_UNSUPPORTED;
  if (layout->T > 0 && (!aligned16(k_text) || !aligned16(v_text) || !aligned16(beta_text)))
    return VDN_ERR_UNSUPPORTED;
  const Layout l = to_layout(layout);
  Layout ls;  // the softmax launches' layout: with the audio keys and context rows
  vdn::JointArgs ja;
  const int js = joint_setup(layout, ctx, ls, ja);
  if (js != VDN_OK) return js;
  // Window softmax into a float32 o_soft, then the readout finishing the
  // output (tensor cores for bf16 with d in {64, 128}, CUDA cores otherwise).
  const bool tc = vdn::readout_tc_supported(l, dtype);
  const Workspace need = carve(l, dtype, nullptr, true, true);
  if (!workspace || workspace_bytes < need.bytes) return VDN_ERR_WORKSPACE;
  const Workspace w = carve(l, dtype, workspace, true, true);
  const void* kt = layout->T ? k_text : nullptr;
  const void* vt = layout->T ? v_text : nullptr;
  const float* bt = layout->T ? beta_text : nullptr;
  int s = cuda_status(vdn::launch_vda_states(l, dtype, k, v, kt, vt, beta, bt, alpha, w.am, w.bw,
                                             w.states, stream));
  if (s != VDN_OK) return s;
  if (before_window) {
    s = cuda_status(cudaStreamWaitEvent(stream, before_window, 0));
    if (s != VDN_OK) return s;
  }
  s = run_window(ls, dtype, q, k, v, kt, vt, w.o_soft, true, nullptr, ja, stream);
  if (s != VDN_OK) return s;
  if (before_combine) {
    s = cuda_status(cudaStreamWaitEvent(stream, before_combine, 0));
    if (s != VDN_OK) return s;
  }
  if (tc)
    return cuda_status(vdn::launch_combine_tc(l, q, w.states, w.o_soft, g_soft, g_lin, rms_weight,
                                              rms_eps, out, out_soft, out_lin, stream));
  return cuda_status(vdn::launch_readout(l, dtype, 1, q, w.states, w.o_soft, g_soft, g_lin,
                                         rms_weight, rms_eps, out, out_soft, out_lin, stream));
}

}  // namespace

namespace vdn {

int hybrid_staged(const vdn_layout_t* layout, int dtype, const void* q, const void* k, const void* v,
                  const void* k_text, const void* v_text, const float* beta, const float* beta_text,
                  const void* g_soft, const void* g_lin, const float* rms_weight, float rms_eps, void* out,
                  void* workspace, size_t workspace_bytes, cudaStream_t stream, cudaEvent_t before_window,
                  cudaEvent_t before_combine) {
  return hybrid_impl(layout, dtype, nullptr, q, k, v, k_text, v_text, beta, beta_text, nullptr, g_soft,
                     g_lin, rms_weight, rms_eps, out, nullptr, nullptr, workspace, workspace_bytes, stream,
                     before_window, before_combine);
}

}  // namespace vdn

extern "C" {

int vdn_vda_scan_fwd(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                     const void* v, const void* k_text, const void* v_text, const float* beta,
                     const float* beta_text, void* o_lin, float* chunk_states, void* workspace,
                     size_t workspace_bytes, cudaStream_t stream) {
  return vda_scan_impl(layout, dtype, q, k, v, k_text, v_text, beta, beta_text, nullptr, o_lin,
                       chunk_states, workspace, workspace_bytes, stream);
}

int vdn_vda_scan_fwd_f32out(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                            const void* v, const void* k_text, const void* v_text,
                            const float* beta, const float* beta_text, float* o_lin,
                            float* chunk_states, void* workspace, size_t workspace_bytes,
                            cudaStream_t stream) {
  return vda_scan_impl(layout, dtype, q, k, v, k_text, v_text, beta, beta_text, nullptr, o_lin,
                       chunk_states, workspace, workspace_bytes, stream, true);
}

int vdn_vda_scan_fwd_decay(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                           const void* v, const void* k_text, const void* v_text, const float* beta,
                           const float* beta_text, const float* alpha, void* o_lin,
                           float* chunk_states, void* workspace, size_t workspace_bytes,
                           cudaStream_t stream) {
  if (!alpha) return VDN_ERR_INVALID;
  return vda_scan_impl(layout, dtype, q, k, v, k_text, v_text, beta, beta_text, alpha, o_lin,
                       chunk_states, workspace, workspace_bytes, stream);
}

int vdn_hybrid_attn_fwd(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                        const void* v, const void* k_text, const void* v_text, const float* beta,
                        const float* beta_text, const void* g_soft, const void* g_lin,
                        const float* rms_weight, float rms_eps, void* out, void* out_soft,
                        void* out_lin, void* workspace, size_t workspace_bytes,
                        cudaStream_t stream) {
  return hybrid_impl(layout, dtype, nullptr, q, k, v, k_text, v_text, beta, beta_text, nullptr, g_soft,
                     g_lin, rms_weight, rms_eps, out, out_soft, out_lin, workspace, workspace_bytes,
                     stream);
}

int vdn_hybrid_attn_fwd_decay(const vdn_layout_t* layout, int dtype, const void* q, const void* k,
                              const void* v, const void* k_text, const void* v_text,
                              const float* beta, const float* beta_text, const float* alpha,
                              const void* g_soft, const void* g_lin, const float* rms_weight,
                              float rms_eps, void* out, void* out_soft, void* out_lin,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (!alpha) return VDN_ERR_INVALID;
  return hybrid_impl(layout, dtype, nullptr, q, k, v, k_text, v_text, beta, beta_text, alpha, g_soft,
                     g_lin, rms_weight, rms_eps, out, out_soft, out_lin, workspace, workspace_bytes,
                     stream);
}

int vdn_joint_attn_fwd(const vdn_layout_t* layout, int dtype, const vdn_context_t* ctx,
                       const void* q, const void* k, const void* v, const void* k_text,
                       const void* v_text, const float* beta, const float* beta_text,
                       const float* alpha, const void* g_soft, const void* g_lin,
                       const float* rms_weight, float rms_eps, void* out, void* out_soft,
                       void* out_lin, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  if (!ctx) return VDN_ERR_INVALID;
  return hybrid_impl(layout, dtype, ctx, q, k, v, k_text, v_text, beta, beta_text, alpha, g_soft,
                     g_lin, rms_weight, rms_eps, out, out_soft, out_lin, workspace, workspace_bytes,
                     stream);
}

int vdn_gated_combine_fwd(long long tokens, int H, int d, int dtype, const float* o_soft,
                          const float* o_lin, const void* g_soft, const void* g_lin,
                          const float* rms_weight, float rms_eps, void* out, cudaStream_t stream) {
  if (tokens < 0 || H < 1 || d < 1) return VDN_ERR_INVALID;
  if (tokens > (1LL << 36) || tokens * H * d > (1LL << 46)) return VDN_ERR_INVALID;
  if (!dtype_d_ok(dtype, d)) return VDN_ERR_UNSUPPORTED;
  if (!(rms_eps >= 0.f)) return VDN_ERR_INVALID;
  if (tokens == 0) return VDN_OK;
  if (!o_soft || !o_lin || !g_soft || !g_lin || !out) return VDN_ERR_INVALID;
  const void* ptrs[] = {o_soft, o_lin, g_soft, g_lin, rms_weight, out};
  for (const void* p : ptrs) if (p && !aligned16(p)) return VDN_ERR_UNSUPPORTED;
  return cuda_status(vdn::launch_gated_combine(tokens * H, d, dtype, o_soft, o_lin, g_soft, g_lin,
                                               rms_weight, rms_eps, out, stream));
}

int vdn_device_status(void) {
  if (cuda_status(cudaDeviceSynchronize()) != VDN_OK) return VDN_ERR_CUDA;
  cudaError_t (*const readers[])(int*) = {
      vdn::read_and_clear_tc_status,   vdn::read_and_clear_gram_status,
      vdn::read_and_clear_readout_status, vdn::read_and_clear_fp8_status,
      vdn::read_and_clear_simt_status, vdn::read_and_clear_vda_status,
      vdn::read_and_clear_ro32_status, vdn::read_and_clear_combine_status};
  constexpr int kReaders = sizeof(readers) / sizeof(readers[0]);
  int s[kReaders] = {};
  for (int i = 0; i < kReaders; ++i)
    if (cuda_status(readers[i](&s[i])) != VDN_OK) return VDN_ERR_CUDA;
  for (int i = 0; i < kReaders; ++i)
    if (s[i] != 0) return s[i];
  return VDN_OK;
}

int vdn_set_wait_limit_ns(unsigned long long ns) {
  cudaError_t (*const setters[])(unsigned long long) = {vdn::set_role_wait_tc,
                                                        vdn::set_role_wait_gram,
                                                        vdn::set_role_wait_readout,
                                                        vdn::set_role_wait_fp8};
  for (auto f : setters) {
    const int s = cuda_status(f(ns));
    if (s != VDN_OK) return s;
  }
  return VDN_OK;
}

const char* vdn_last_cuda_error(void) {
  return vdn::t_last_cuda_error == cudaSuccess ? "no CUDA error"
                                                : cudaGetErrorString(vdn::t_last_cuda_error);
}

const char* vdn_status_string(int status) {
  switch (status) {
    case VDN_OK: return "ok";
    case VDN_ERR_INVALID: return "invalid argument (layout or required pointer)";
    case VDN_ERR_UNSUPPORTED: return "unsupported dtype/head dim or misaligned pointer";
    case VDN_ERR_WORKSPACE: return "workspace missing or too small";
    case VDN_ERR_CUDA: return "CUDA error";
    case VDN_ERR_TIMEOUT: return "a kernel gave up a bounded wait";
    case VDN_ERR_BOUNDS: return "a bound check of the checked build failed";
  }
  return "unknown status";
}

}  // extern "C"
