// vdn_hybrid_attn_fwd_host: the hybrid forward on tensors in host memory, with
// the host-device copies overlapped with the computation.
//
// Every (b, h) pair is independent in both branches, so the heads are taken in
// chunks of head_chunk: chunk i is copied in (one strided 2-D copy per tensor:
// B * L rows of head_chunk * d elements out of rows of H * d), computed by the
// same kernels as vdn_hybrid_attn_fwd on a [B, L, head_chunk, d] layout, and its
// output copied back into the strided host tensor, on three streams (in,
// compute, out) with two device buffers, so that chunk i + 1 is copied in and
// chunk i - 1 copied out while chunk i computes. PCIe carries both directions
// at once; with pinned host memory the copies then hide under the kernels.
// A chunk's inputs arrive in the order its kernels need them: k, v and beta
// (the linear branch starts), then q (the window softmax), then the gates (the
// combine), each group with its own event, so that a chunk's kernels start
// before its last bytes have crossed PCIe.
#include <cstdint>
#include <mutex>

#include "vdn_internal.cuh"

namespace {

// The pipeline's three streams and ten events, created on the first call on a
// device and kept for the life of the process (creating and destroying them on
// every call costs driver round trips per call). The call is synchronous, so
// one call at a time uses them: concurrent calls on one device take turns.
struct Pipeline {
  std::mutex mu;
  bool ready = false;
  cudaStream_t s_in = nullptr, s_comp = nullptr, s_out = nullptr;
  cudaEvent_t ev_in[2] = {nullptr, nullptr}, ev_q[2] = {nullptr, nullptr}, ev_g[2] = {nullptr, nullptr},
              ev_comp[2] = {nullptr, nullptr}, ev_out[2] = {nullptr, nullptr};
};
constexpr int kMaxDevicesH = 64;
Pipeline g_pipe[kMaxDevicesH];

// Creates the streams and events of the current device's pipeline (caller
// holds its mutex).
cudaError_t pipeline_init(Pipeline& p) {
  if (p.ready) return cudaSuccess;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t r) { if (e == cudaSuccess) e = r; };
  ok(cudaStreamCreateWithFlags(&p.s_in, cudaStreamNonBlocking));
  ok(cudaStreamCreateWithFlags(&p.s_comp, cudaStreamNonBlocking));
  ok(cudaStreamCreateWithFlags(&p.s_out, cudaStreamNonBlocking));
  for (int i = 0; i < 2; ++i) {
    ok(cudaEventCreateWithFlags(&p.ev_in[i], cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&p.ev_q[i], cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&p.ev_g[i], cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&p.ev_comp[i], cudaEventDisableTiming));
    ok(cudaEventCreateWithFlags(&p.ev_out[i], cudaEventDisableTiming));
  }
  p.ready = e == cudaSuccess;
  return e;
}

constexpr size_t kAlignH = 256;
size_t align_h(size_t x) { return (x + kAlignH - 1) / kAlignH * kAlignH; }

int elem_size(int dtype) { return dtype == VDN_BF16 ? 2 : 4; }

// One device buffer of the pipeline for a chunk of hc heads.
struct ChunkBuf {
  char* q; char* k; char* v; char* gs; char* gl; char* out;  // [B, L, hc, d]
  char* kt; char* vt;                                          // [B, T, hc, d]
  float* beta; float* beta_t;                                  // [B, L, hc], [B, T, hc]
  void* ws;                                                    // hybrid workspace
  size_t bytes;
};

// Carves one chunk buffer at base (nullptr: sizes only).
ChunkBuf carve_chunk(const vdn_layout_t& lc, int dtype, char* base) {
  ChunkBuf c{};
  size_t off = 0;
  auto take = [&](size_t n) -> char* {
    char* r = base ? base + off : nullptr;
    off = align_h(off + n);
    return r;
  };
  const size_t es = elem_size(dtype);
  const size_t video = (size_t)lc.B * lc.F * lc.N * lc.H * lc.d * es;
  const size_t text = (size_t)lc.B * lc.T * lc.H * lc.d * es;
  c.q = take(video); c.k = take(video); c.v = take(video); c.gs = take(video); c.gl = take(video);
  c.out = take(video);
  c.kt = take(text); c.vt = take(text);
  c.beta = reinterpret_cast<float*>(take((size_t)lc.B * lc.F * lc.N * lc.H * 4));
  c.beta_t = reinterpret_cast<float*>(take((size_t)lc.B * lc.T * lc.H * 4));
  c.ws = take(vdn_workspace_bytes(&lc, dtype));
  c.bytes = off;
  return c;
}

// Chunk sizes. Given head_chunk > 0: uniform. Default: the first chunk's
// copy-in and the last chunk's copy-out are the only copies not hidden, so the
// chunks grow from one head (each copy-in must fit under the previous chunk's
// kernels: a head's inputs take about 3/4 of its compute time over PCIe, so a
// chunk may be about a third larger than the one before), stay at up to
// about an eighth of the heads, and shrink back to one head at the end; each
// chunk also pays the latency-bound VDA kernels, so they do not get smaller.
constexpr int kMaxChunks = 64;
int chunk_plan(const vdn_layout_t* l, int head_chunk, int* sizes) {
  const int H = l->H;
  if (head_chunk > 0) {
    const int hc = head_chunk > H ? H : head_chunk;
    int n = 0;
    for (int h0 = 0; h0 < H && n < kMaxChunks; h0 += hc) sizes[n++] = (h0 + hc <= H) ? hc : H - h0;
    if (n == kMaxChunks) return -1;
    return n;
  }
  const int cap = (H + 7) / 8;
  int head[kMaxChunks], tail[kMaxChunks], nh = 0, nt = 0, left = H;
  // grow from both ends, one head at the ends, about a third more each step
  int s = 1;
  while (left > 0 && nh + nt < kMaxChunks - 1) {
    const int a = s < left ? s : left;
    head[nh++] = a;
    left -= a;
    if (left <= 0) break;
    const int b = s < left ? s : left;
    tail[nt++] = b;
    left -= b;
    if (s >= cap) break;
    s = (s * 4 + 2) / 3 > s ? (s * 4 + 2) / 3 : s + 1;
    if (s > cap) s = cap;
  }
  int n = 0;
  for (int i = 0; i < nh; ++i) sizes[n++] = head[i];
  while (left > 0 && n < kMaxChunks - nt) {
    const int a = cap < left ? cap : left;
    sizes[n++] = a;
    left -= a;
  }
  for (int i = nt - 1; i >= 0; --i) sizes[n++] = tail[i];
  return left == 0 ? n : -1;
}

int max_chunk(const int* sizes, int n) {
  int m = 0;
  for (int i = 0; i < n; ++i) m = sizes[i] > m ? sizes[i] : m;
  return m;
}

// rows x width bytes, host rows at pitch hpitch, device rows packed.
cudaError_t copy_in(void* dst, const void* src, size_t width, size_t hpitch, size_t rows,
                    cudaStream_t st) {
  if (rows == 0 || width == 0) return cudaSuccess;
  return cudaMemcpy2DAsync(dst, width, src, hpitch, width, rows, cudaMemcpyHostToDevice, st);
}

}  // namespace

extern "C" {

size_t vdn_hybrid_host_workspace_bytes(const vdn_layout_t* layout, int dtype, int head_chunk) {
  if (vdn_workspace_bytes(layout, dtype) == 0) return 0;
  int sizes[kMaxChunks];
  const int n = chunk_plan(layout, head_chunk, sizes);
  if (n <= 0) return 0;
  vdn_layout_t lc = *layout;
  lc.H = max_chunk(sizes, n);
  // alignment slack, the RMSNorm weight, two chunk buffers
  return kAlignH + align_h((size_t)layout->d * 4) + 2 * carve_chunk(lc, dtype, nullptr).bytes;
}

int vdn_hybrid_attn_fwd_host(const vdn_layout_t* layout, int dtype, int head_chunk,
                             const void* q, const void* k, const void* v, const void* k_text,
                             const void* v_text, const float* beta, const float* beta_text,
                             const void* g_soft, const void* g_lin, const float* rms_weight,
                             float rms_eps, void* out, void* workspace, size_t workspace_bytes) {
  if (!vdn::layout_ok(layout)) return VDN_ERR_INVALID;
  const size_t need = vdn_hybrid_host_workspace_bytes(layout, dtype, head_chunk);
  if (need == 0) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !beta || !g_soft || !g_lin || !out) return VDN_ERR_INVALID;
  if (layout->T > 0 && (!k_text || !v_text || !beta_text)) return VDN_ERR_INVALID;
  if (!(rms_eps >= 0.f)) return VDN_ERR_INVALID;
  if (!workspace || workspace_bytes < need) return VDN_ERR_WORKSPACE;

  const int H = layout->H, d = layout->d, B = layout->B, T = layout->T;
  const long long L = (long long)layout->F * layout->N;
  const size_t es = elem_size(dtype);
  int sizes[kMaxChunks];
  const int n_chunks = chunk_plan(layout, head_chunk, sizes);
  const int hc_max = max_chunk(sizes, n_chunks);

  vdn_layout_t lmax = *layout;
  lmax.H = hc_max;
  char* base = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(workspace) + kAlignH - 1) &
                                       ~static_cast<uintptr_t>(kAlignH - 1));
  float* rms_w_dev = rms_weight ? reinterpret_cast<float*>(base) : nullptr;
  base += align_h((size_t)d * 4);
  const size_t buf_bytes = carve_chunk(lmax, dtype, nullptr).bytes;

  int dev = 0;
  int status = vdn::cuda_status(cudaGetDevice(&dev));
  if (status != VDN_OK) return status;
  if (dev < 0 || dev >= kMaxDevicesH) return VDN_ERR_UNSUPPORTED;
  Pipeline& pipe = g_pipe[dev];
  std::lock_guard<std::mutex> lock(pipe.mu);
  status = vdn::cuda_status(pipeline_init(pipe));
  if (status != VDN_OK) return status;
  cudaStream_t s_in = pipe.s_in, s_comp = pipe.s_comp, s_out = pipe.s_out;
  cudaEvent_t* ev_in = pipe.ev_in;
  cudaEvent_t* ev_q = pipe.ev_q;
  cudaEvent_t* ev_g = pipe.ev_g;
  cudaEvent_t* ev_comp = pipe.ev_comp;
  cudaEvent_t* ev_out = pipe.ev_out;
  auto fail = [&](cudaError_t e) {
    if (e != cudaSuccess && status == VDN_OK) status = vdn::cuda_status(e);
  };

  if (rms_weight)
    fail(cudaMemcpyAsync(rms_w_dev, rms_weight, (size_t)d * 4, cudaMemcpyHostToDevice, s_in));
  int h0 = 0;
  for (int c = 0; c < n_chunks && status == VDN_OK; h0 += sizes[c], ++c) {
    const int hc = sizes[c];
    const int slot = c & 1;
    vdn_layout_t lc = *layout;
    lc.H = hc;
    const ChunkBuf buf = carve_chunk(lc, dtype, base + slot * buf_bytes);
    // copy in, once the buffer's previous chunk has been copied out
    if (c >= 2) fail(cudaStreamWaitEvent(s_in, ev_out[slot], 0));
    const size_t w_vid = (size_t)hc * d * es, p_vid = (size_t)H * d * es, o_vid = (size_t)h0 * d * es;
    const size_t rows_v = (size_t)B * L, rows_t = (size_t)B * T;
    // the linear branch's inputs: k, v, the text, beta
    fail(copy_in(buf.k, static_cast<const char*>(k) + o_vid, w_vid, p_vid, rows_v, s_in));
    fail(copy_in(buf.v, static_cast<const char*>(v) + o_vid, w_vid, p_vid, rows_v, s_in));
    if (T > 0) {
      fail(copy_in(buf.kt, static_cast<const char*>(k_text) + o_vid, w_vid, p_vid, rows_t, s_in));
      fail(copy_in(buf.vt, static_cast<const char*>(v_text) + o_vid, w_vid, p_vid, rows_t, s_in));
      fail(copy_in(buf.beta_t, beta_text + h0, (size_t)hc * 4, (size_t)H * 4, rows_t, s_in));
    }
    fail(copy_in(buf.beta, beta + h0, (size_t)hc * 4, (size_t)H * 4, rows_v, s_in));
    fail(cudaEventRecord(ev_in[slot], s_in));
    // then q (the window softmax), then the gates (the combine)
    fail(copy_in(buf.q, static_cast<const char*>(q) + o_vid, w_vid, p_vid, rows_v, s_in));
    fail(cudaEventRecord(ev_q[slot], s_in));
    fail(copy_in(buf.gs, static_cast<const char*>(g_soft) + o_vid, w_vid, p_vid, rows_v, s_in));
    fail(copy_in(buf.gl, static_cast<const char*>(g_lin) + o_vid, w_vid, p_vid, rows_v, s_in));
    fail(cudaEventRecord(ev_g[slot], s_in));
    if (status != VDN_OK) break;
    // compute: the linear branch once k, v and beta are in, the window once q is
    fail(cudaStreamWaitEvent(s_comp, ev_in[slot], 0));
    const vdn_layout_t* lcp = &lc;
    const int s = vdn::hybrid_staged(lcp, dtype, buf.q, buf.k, buf.v, T ? buf.kt : nullptr,
                                     T ? buf.vt : nullptr, buf.beta, T ? buf.beta_t : nullptr, buf.gs,
                                     buf.gl, rms_w_dev, rms_eps, buf.out, buf.ws,
                                     vdn_workspace_bytes(lcp, dtype), s_comp, ev_q[slot], ev_g[slot]);
    if (s != VDN_OK) { status = s; break; }
    fail(cudaEventRecord(ev_comp[slot], s_comp));
    // copy out into the strided host tensor
    fail(cudaStreamWaitEvent(s_out, ev_comp[slot], 0));
    fail(cudaMemcpy2DAsync(static_cast<char*>(out) + o_vid, p_vid, buf.out, w_vid, w_vid, rows_v,
                           cudaMemcpyDeviceToHost, s_out));
    fail(cudaEventRecord(ev_out[slot], s_out));
  }
  // the call returns with the output in host memory (and nothing in flight)
  for (cudaStream_t st : {s_in, s_comp, s_out}) fail(cudaStreamSynchronize(st));
  return status;
}

}  // extern "C"
