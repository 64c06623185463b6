// vdn_vda_scan_fwd_noalloc: the linear-branch entry point without a caller
// workspace and without any allocation.
//
// Who needs it: code that cannot allocate device memory at the point where it
// runs this op, for example a plugin inside an inference engine that owns all
// device memory and hands its plugins no workspace, or a serving loop that
// forbids device allocations after start-up (cudaMalloc and cudaFree can
// synchronise the device and stall every other stream).
//
// How: the scratch that vdn_vda_scan_fwd takes from its caller (per-frame Gram
// and inverse slots, and the chunk read states when the caller does not ask
// for them) lives here in a file-scope __device__ array of kStaticScratchBytes.
// Every GPU that loads the library holds this array until the process exits.
// Host code cannot use the array's name as a device address, so the first call
// on each device looks the address up with cudaGetSymbolAddress (with that
// device current) and caches it; make that first call on a device before any
// stream capture. Nothing in the scratch has to start at zero: every entry a
// call reads is written earlier in the same call. All calls share the array
// and it keeps the last call's contents, so calls that overlap on the GPU (on
// different streams, or from several host threads) race and corrupt each
// other; serialise them.
#include <cstdint>
#include <mutex>

#include "vdn_internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = VDN_NOALLOC_SCRATCH_BYTES;
constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kStaticScratchBytes];

std::mutex g_addr_mutex;
void* g_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once).
cudaError_t scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_addr_mutex);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return cudaSuccess;
}

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Scratch layout: Gram/inverse slots am and bw [B, H, F, d, d] fp32, then the
// chunk read states [B, H, 2, J, d, d] when the caller passes none.
size_t scratch_bytes(const vdn::Layout& l, bool own_states) {
  const size_t dd = (size_t)l.d * l.d, bh = (size_t)l.B * l.H;
  size_t n = 2 * align_up(bh * l.F * dd * sizeof(float));
  if (own_states) n += align_up(bh * 2 * l.J() * dd * sizeof(float));
  return n;
}

}  // namespace

extern "C" int vdn_vda_scan_fwd_noalloc(const vdn_layout_t* layout, int dtype, const void* q,
                                        const void* k, const void* v, const void* k_text,
                                        const void* v_text, const float* beta,
                                        const float* beta_text, void* o_lin, float* chunk_states,
                                        cudaStream_t stream) {
  // the same checks as vdn_vda_scan_fwd (vdn_internal.cuh)
  if (!vdn::layout_ok(layout)) return VDN_ERR_INVALID;
  if (!vdn::dtype_d_ok(dtype, layout->d)) return VDN_ERR_UNSUPPORTED;
  if (!q || !k || !v || !beta || !o_lin) return VDN_ERR_INVALID;
  if (layout->T > 0 && (!k_text || !v_text || !beta_text)) return VDN_ERR_INVALID;
  const void* ptrs[] = {q, k, v, beta, o_lin, chunk_states};
  for (const void* p : ptrs)
    if (p && !vdn::aligned16(p)) return VDN_ERR_UNSUPPORTED;
  if (layout->T > 0 &&
      (!vdn::aligned16(k_text) || !vdn::aligned16(v_text) || !vdn::aligned16(beta_text)))
    return VDN_ERR_UNSUPPORTED;

  const vdn::Layout l = vdn::to_layout(layout);
  const bool own_states = chunk_states == nullptr;
  if (scratch_bytes(l, own_states) > kStaticScratchBytes) return VDN_ERR_WORKSPACE;

  void* base = nullptr;
  int s = vdn::cuda_status(scratch_address(&base));
  if (s != VDN_OK) return s;
  const size_t dd = (size_t)l.d * l.d, bh = (size_t)l.B * l.H;
  char* p = static_cast<char*>(base);
  float* am = reinterpret_cast<float*>(p);
  p += align_up(bh * l.F * dd * sizeof(float));
  float* bw = reinterpret_cast<float*>(p);
  p += align_up(bh * l.F * dd * sizeof(float));
  float* states = own_states ? reinterpret_cast<float*>(p) : chunk_states;

  const void* kt = layout->T ? k_text : nullptr;
  const void* vt = layout->T ? v_text : nullptr;
  const float* bt = layout->T ? beta_text : nullptr;
  s = vdn::cuda_status(
      vdn::launch_vda_states(l, dtype, k, v, kt, vt, beta, bt, nullptr, am, bw, states, stream));
  if (s != VDN_OK) return s;
  if (vdn::readout_tc_supported(l, dtype))
    return vdn::cuda_status(vdn::launch_readout_tc(l, q, states, o_lin, false, stream));
  return vdn::cuda_status(vdn::launch_readout(l, dtype, 0, q, states, nullptr, nullptr, nullptr,
                                              nullptr, 0.f, o_lin, nullptr, nullptr, stream));
}
