// Linear-branch readout o_lin = (S_fwd + S_rev) q on the 5th-generation tensor
// cores, for the standalone linear-branch entry point with bf16 tensors
// (project page "Local Softmax and Long-Range Linear Memory": both states are
// read and their outputs added; boundary frames read nothing).
//
// CTA = up to 24 consecutive 128-row query tiles of one query group of one
// (b, h); 320 threads:
//   warp 0     TMA producer: Q tiles into two shared-memory stages
//   warp 1     MMA issuer and TMEM owner: O = Q S_hi^T + Q S_lo^T into one of two
//              TMEM accumulators
//   warps 2-9  stage S_sum = S_fwd + S_rev once as two bf16 K-major operands
//              (S_hi = bf16(S_sum), S_lo = bf16(S_sum - S_hi)); then warpgroup
//              2-5 drains the accumulator of the even tiles and warpgroup 6-9
//              that of the odd tiles, so that two tiles' worth of loads and
//              stores are in flight; each warp passes its 32 TMEM rows through
//              a 16-row shared-memory staging and writes one contiguous row per
//              warp access
// Boundary-frame groups write zeros. HBM-bound: q is read once, o_lin written once
// (bf16, or float32 for the branch-specialised split's exchange).
//
// Combine variant (project page, "Gating the Softmax and Linear Branch
// Outputs"): instead of o_lin, the drain warps finish the rows of the hybrid
// output, out = sigmoid(g_s) o_soft + sigmoid(g_l) RMSNorm(o_lin), from the
// float32 softmax-branch output of the window kernel and the two gates
// (boundary frames: out = sigmoid(g_s) o_soft); optionally the two gated
// branches separately.
#include "tc_common.cuh"

namespace vdn {

__device__ int g_readout_status = 0;

cudaError_t set_role_wait_readout(unsigned long long ns) { return set_role_wait_ns(ns); }

cudaError_t read_and_clear_readout_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_readout_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_readout_status, &zero, sizeof(int));
}

namespace {

constexpr int kRows = 128;
constexpr int kTilesPerCta = 24;
constexpr int kThreads = 320;
constexpr int kDrainThreads = 256;

template <int D>
struct RCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kHalfBytes = kRows * 128;
  static constexpr int kTileBytes = kRows * D * 2;
  static constexpr int kTmemCols = 2 * D;
  // row stride of the drain staging in floats: padded so that the rows written
  // by 8 consecutive lanes fall on different banks
  static constexpr int kStgStride = D + 4;
  // S_hi, S_lo, 2 Q stages, barriers, then the drain warps' row staging
  // (8 warps x 16 rows)
  static constexpr int kSmemBytes = 1024 + 4 * kTileBytes + 256 + 8 * 16 * kStgStride * 4;
};

struct RBars {
  unsigned long long q_full[2];
  unsigned long long q_empty[2];
  unsigned long long d_full[2];
  unsigned long long d_empty[2];
  unsigned long long ssum_ready;
  unsigned long long done;
  uint32_t tmem_base;
  int abort;
};

// Inputs and outputs of the combine variant.
struct CombineArgs {
  const float* o_soft;             // [B, L, H, D] fp32 softmax branch
  const __nv_bfloat16* g_soft;     // [B, L, H, D]
  const __nv_bfloat16* g_lin;      // [B, L, H, D]
  const float* rms_w;              // [D] or null
  float eps;
  __nv_bfloat16* out;              // [B, L, H, D]
  __nv_bfloat16* out_soft;         // nullable
  __nv_bfloat16* out_lin;          // nullable
};

__device__ __forceinline__ float sigmoid_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(1.f + ex2(-1.4426950408889634f * x)));
  return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Combines 8 consecutive elements of one row: o (softmax branch, fp32), lin
// (RMS-normalised linear branch, already weighted; 0 for boundary rows) and
// the two gate words; writes out (and the gated branches when asked).
__device__ __forceinline__ void combine8(const CombineArgs& cx, long long off, const float* o,
                                         const float* lin, uint4 gs4, uint4 gl4, bool has_lin) {
  const uint32_t gsw[4] = {gs4.x, gs4.y, gs4.z, gs4.w};
  const uint32_t glw[4] = {gl4.x, gl4.y, gl4.z, gl4.w};
  uint32_t ow[4], osw[4], olw[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a0 = sigmoid_approx(bf16_lo(gsw[e])) * o[2 * e];
    const float a1 = sigmoid_approx(bf16_hi(gsw[e])) * o[2 * e + 1];
    const float b0 = has_lin ? sigmoid_approx(bf16_lo(glw[e])) * lin[2 * e] : 0.f;
    const float b1 = has_lin ? sigmoid_approx(bf16_hi(glw[e])) * lin[2 * e + 1] : 0.f;
    ow[e] = pack_bf16(a0 + b0, a1 + b1);
    osw[e] = pack_bf16(a0, a1);
    olw[e] = pack_bf16(b0, b1);
  }
  *reinterpret_cast<uint4*>(cx.out + off) = make_uint4(ow[0], ow[1], ow[2], ow[3]);
  if (cx.out_soft) *reinterpret_cast<uint4*>(cx.out_soft + off) = make_uint4(osw[0], osw[1], osw[2], osw[3]);
  if (cx.out_lin) *reinterpret_cast<uint4*>(cx.out_lin + off) = make_uint4(olw[0], olw[1], olw[2], olw[3]);
}

__device__ __forceinline__ bool rwait(unsigned long long* bar, uint32_t parity, volatile int* abort,
                                      bool watch_abort = true) {
  if (mbar_try_wait(smem_u32(bar), parity)) return true;
  return mbar_wait_impl(bar, parity, abort, &g_readout_status, watch_abort);
}

// kMode: 0 writes o_lin in bf16, 1 the combined output (CombineArgs), 2 o_lin
// in float32 (the branch output a branch-specialised split sends on).
template <int D, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
readout_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const Layout l,
                  const float* __restrict__ states, void* __restrict__ o_lin_out,
                  const CombineArgs cx) {
  constexpr bool kCombine = kMode == 1;
  __nv_bfloat16* o_lin = static_cast<__nv_bfloat16*>(o_lin_out);
  float* o_lin32 = static_cast<float*>(o_lin_out);
  using C = RCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sHi = smem;
  uint8_t* sLo = smem + C::kTileBytes;
  uint8_t* sQ = smem + 2 * C::kTileBytes;
  RBars* bars = reinterpret_cast<RBars*>(smem + 4 * C::kTileBytes);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  int g, r0;
  tile_to_group(l, kRows * kTilesPerCta, blockIdx.x, g, r0);
  if (g < 0) return;  // grid is sized by the same enumeration; uniform per CTA
  const Group G = make_group(l, g);
  const int rows = min(kRows * kTilesPerCta, G.q0 + G.nq - r0);
  const long long HD = (long long)l.H * D;

  if (G.chunk < 0) {
    // boundary frame: no linear readout
    for (int i = threadIdx.x; i < rows * (D / 8); i += kThreads) {
      const int r = i / (D / 8), c = i % (D / 8);
      if (!VDN_IN_BOUNDS(r0 + r < l.L(), &g_readout_status)) continue;
      const long long off = ((long long)b * l.L() + r0 + r) * HD + (long long)h * D + c * 8;
      if constexpr (kCombine) {
        const float4 o0 = *reinterpret_cast<const float4*>(cx.o_soft + off);
        const float4 o1 = *reinterpret_cast<const float4*>(cx.o_soft + off + 4);
        const float o[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
        const float lin[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        combine8(cx, off, o, lin, *reinterpret_cast<const uint4*>(cx.g_soft + off),
                 make_uint4(0u, 0u, 0u, 0u), false);
      } else if constexpr (kMode == 2) {
        *reinterpret_cast<float4*>(o_lin32 + off) = make_float4(0.f, 0.f, 0.f, 0.f);
        *reinterpret_cast<float4*>(o_lin32 + off + 4) = make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
        *reinterpret_cast<uint4*>(o_lin + off) = make_uint4(0u, 0u, 0u, 0u);
      }
    }
    return;
  }
  const int n_tiles = (rows + kRows - 1) / kRows;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bars->q_full[i], 1);
      mbar_init(&bars->q_empty[i], 1);
      mbar_init(&bars->d_full[i], 1);
      mbar_init(&bars->d_empty[i], 128);
    }
    mbar_init(&bars->ssum_ready, kDrainThreads);
    mbar_init(&bars->done, 1);
    bars->abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&bars->tmem_base)), "r"(C::kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t & 1, use = t >> 1;
        if (use > 0 && !rwait(&bars->q_empty[s], (use - 1) & 1, abort)) {
          ok = false;
          break;
        }
        mbar_expect_tx(&bars->q_full[s], C::kTileBytes);
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(sQ + s * C::kTileBytes + hf * C::kHalfBytes, &tm_q, &bars->q_full[s], hf * 64, h,
                      r0 + t * kRows, b);
        ++issued;
      }
      if (!ok) {
        for (int s = 0; s < 2 && s < issued; ++s) {
          const int last = issued - 1 - ((issued - 1 - s) % 2);
          rwait(&bars->q_full[s], (last >> 1) & 1, abort, false);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(D, false);
      bool ok = rwait(&bars->ssum_ready, 0, abort);
      const uint32_t hi_addr = smem_u32(sHi), lo_addr = smem_u32(sLo), q_addr = smem_u32(sQ);
      for (int t = 0; t < n_tiles && ok; ++t) {
        const int s = t & 1, use = t >> 1;
        if (!rwait(&bars->q_full[s], use & 1, abort)) { ok = false; break; }
        if (use > 0 && !rwait(&bars->d_empty[s], (use - 1) & 1, abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + s * D;
#pragma unroll
        for (int part = 0; part < 2; ++part) {
#pragma unroll
          for (int ks = 0; ks < D / 16; ++ks) {
            const uint32_t off = (uint32_t)((ks / 4) * C::kHalfBytes + (ks % 4) * 32);
            mma_ss(d_tmem, desc_k_sw128(q_addr + s * C::kTileBytes + off),
                   desc_k_sw128((part ? lo_addr : hi_addr) + off), idesc, (part > 0 || ks > 0) ? 1u : 0u);
          }
        }
        tc_commit(&bars->q_empty[s]);
        tc_commit(&bars->d_full[s]);
      }
      if (!ok) {
        // every MMA issued must finish before TMEM is freed
        tc_commit(&bars->done);
        rwait(&bars->done, 0, abort, false);
      }
    }
  } else {
    const int t256 = threadIdx.x - 64;
    const int dg = t256 / 128;  // drain warpgroup: tiles with (t & 1) == dg
    // stage S_sum (hi, lo) once
    {
      const int J = l.J();
      (void)VDN_IN_BOUNDS(G.chunk < J, &g_readout_status);
      const float* sf = states + ((((long long)b * l.H + h) * 2 + 0) * J + G.chunk) * D * D;
      const float* sr = states + ((((long long)b * l.H + h) * 2 + 1) * J + G.chunk) * D * D;
      constexpr int kChunks = D / 8;
      for (int ch = t256; ch < kRows * kChunks; ch += kDrainThreads) {
        const int n = ch / kChunks, kc = ch % kChunks;
        if (n >= D) continue;  // rows beyond d (d = 64) stay unused: the MMA reads N = d rows
        const float4 a0 = *reinterpret_cast<const float4*>(sf + n * D + kc * 8);
        const float4 a1 = *reinterpret_cast<const float4*>(sf + n * D + kc * 8 + 4);
        const float4 b0 = *reinterpret_cast<const float4*>(sr + n * D + kc * 8);
        const float4 b1 = *reinterpret_cast<const float4*>(sr + n * D + kc * 8 + 4);
        const float x[8] = {a0.x + b0.x, a0.y + b0.y, a0.z + b0.z, a0.w + b0.w,
                            a1.x + b1.x, a1.y + b1.y, a1.z + b1.z, a1.w + b1.w};
        float hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          hi[e] = __bfloat162float(__float2bfloat16_rn(x[e]));
          lo[e] = x[e] - hi[e];
        }
        const int half = kc / 8, c16 = kc % 8;
        const int off = half * C::kHalfBytes + n * 128 + ((c16 ^ (n & 7)) * 16);
        *reinterpret_cast<uint4*>(sHi + off) = make_uint4(pack_bf16(hi[0], hi[1]), pack_bf16(hi[2], hi[3]),
                                                          pack_bf16(hi[4], hi[5]), pack_bf16(hi[6], hi[7]));
        *reinterpret_cast<uint4*>(sLo + off) = make_uint4(pack_bf16(lo[0], lo[1]), pack_bf16(lo[2], lo[3]),
                                                          pack_bf16(lo[4], lo[5]), pack_bf16(lo[6], lo[7]));
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      mbar_arrive(&bars->ssum_ready);
    }
    // drain accumulators. TMEM holds one row per thread; global memory wants
    // each warp access on one row. So each warp copies its 32 rows out through
    // a shared-memory staging of 16 rows (two passes): the lanes whose rows go
    // in this pass write them, then the warp emits the staged rows one at a
    // time with its lanes on consecutive columns, several rows per batch so
    // that enough loads (the combine's o_soft and gates) are in flight. The
    // combine reads the accumulator once for the row's RMS statistic and once
    // per pass (TMEM reads are cheap; the registers are not), and stages
    // acc * rstd so that every lane can finish any row.
    const int m0 = 32 * (warp & 3);
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    static_assert(sizeof(RBars) <= 256, "barriers overlap the staging");
    float* stg = reinterpret_cast<float*>(smem + 4 * C::kTileBytes + 256) + (warp - 2) * 16 * C::kStgStride;
    float* my_stg = stg + (lane & 15) * C::kStgStride;  // this lane's staging row
    const bool cols_lane = 4 * lane < D;                  // lanes cover 4 columns each
    float w4[4] = {1.f, 1.f, 1.f, 1.f};                   // RMSNorm weight of those columns
    if constexpr (kCombine) {
      if (cx.rms_w != nullptr && cols_lane) {
        const float4 wv = *reinterpret_cast<const float4*>(cx.rms_w + 4 * lane);
        w4[0] = wv.x; w4[1] = wv.y; w4[2] = wv.z; w4[3] = wv.w;
      }
    }
    constexpr int kBatch = 8;  // rows emitted per batch
    for (int t = dg; t < n_tiles; t += 2) {
      const int s = t & 1, use = t >> 1;
      if (!__all_sync(0xffffffffu, rwait(&bars->d_full[s], use & 1, abort))) break;
      tc_fence_after();
      const uint32_t tacc = tmem + lane_base + s * D;
      const int tile_row0 = r0 + t * kRows + m0;  // global row of lane 0's row
      if constexpr (kCombine) {
        float ss4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld_x32(tacc + c0, r);
#pragma unroll
          for (int i = 0; i < 32; ++i) ss4[i & 3] = fmaf(__uint_as_float(r[i]), __uint_as_float(r[i]), ss4[i & 3]);
        }
        const float rstd = rsqrtf(((ss4[0] + ss4[1]) + (ss4[2] + ss4[3])) / (float)D + cx.eps);
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t r[32];
            tmem_ld_x32(tacc + c0, r);
            if ((lane >> 4) == pass) {
#pragma unroll
              for (int c = 0; c < 32; c += 4)
                *reinterpret_cast<float4*>(my_stg + c0 + c) =
                    make_float4(__uint_as_float(r[c]) * rstd, __uint_as_float(r[c + 1]) * rstd,
                                __uint_as_float(r[c + 2]) * rstd, __uint_as_float(r[c + 3]) * rstd);
            }
          }
          if (pass == 1) {
            tc_fence_before();
            mbar_arrive(&bars->d_empty[s]);  // the accumulator is free for tile t + 2
          }
          __syncwarp();
          const int lim = min(16, G.q0 + G.nq - (tile_row0 + 16 * pass));  // rows of the group
#pragma unroll 1
          for (int rb = 0; rb < lim; rb += kBatch) {
            float4 o4[kBatch];
            uint2 gs2[kBatch], gl2[kBatch];
            long long off[kBatch];
            bool ok[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              const int grow = tile_row0 + 16 * pass + rb + u;
              ok[u] = cols_lane && rb + u < lim && VDN_IN_BOUNDS(grow >= 0 && grow < l.L(), &g_readout_status);
              off[u] = ((long long)b * l.L() + grow) * HD + (long long)h * D + 4 * lane;
              if (ok[u]) {
                o4[u] = *reinterpret_cast<const float4*>(cx.o_soft + off[u]);
                gs2[u] = *reinterpret_cast<const uint2*>(cx.g_soft + off[u]);
                gl2[u] = *reinterpret_cast<const uint2*>(cx.g_lin + off[u]);
              }
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
              if (!ok[u]) continue;
              const float4 a4 = *reinterpret_cast<const float4*>(stg + (rb + u) * C::kStgStride + 4 * lane);
              const float o[4] = {o4[u].x, o4[u].y, o4[u].z, o4[u].w};
              const float lin[4] = {a4.x * w4[0], a4.y * w4[1], a4.z * w4[2], a4.w * w4[3]};
              const float gs[4] = {bf16_lo(gs2[u].x), bf16_hi(gs2[u].x), bf16_lo(gs2[u].y), bf16_hi(gs2[u].y)};
              const float gl[4] = {bf16_lo(gl2[u].x), bf16_hi(gl2[u].x), bf16_lo(gl2[u].y), bf16_hi(gl2[u].y)};
              float so[4], sl[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                so[e] = sigmoid_approx(gs[e]) * o[e];
                sl[e] = sigmoid_approx(gl[e]) * lin[e];
              }
              *reinterpret_cast<uint2*>(cx.out + off[u]) =
                  make_uint2(pack_bf16(so[0] + sl[0], so[1] + sl[1]), pack_bf16(so[2] + sl[2], so[3] + sl[3]));
              if (cx.out_soft)
                *reinterpret_cast<uint2*>(cx.out_soft + off[u]) =
                    make_uint2(pack_bf16(so[0], so[1]), pack_bf16(so[2], so[3]));
              if (cx.out_lin)
                *reinterpret_cast<uint2*>(cx.out_lin + off[u]) =
                    make_uint2(pack_bf16(sl[0], sl[1]), pack_bf16(sl[2], sl[3]));
            }
          }
          __syncwarp();  // the staging is rewritten by the next pass
        }
      } else {
        // o_lin only: the whole row is taken out of TMEM at once (no loads to
        // hold registers for), and the accumulator freed before the stores
        uint32_t r[D];
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 32) tmem_ld_x32(tacc + c0, r + c0);
        tc_fence_before();
        mbar_arrive(&bars->d_empty[s]);  // the accumulator is free for tile t + 2
#pragma unroll 1
        for (int pass = 0; pass < 2; ++pass) {
          if ((lane >> 4) == pass) {
#pragma unroll
            for (int c = 0; c < D; c += 4)
              *reinterpret_cast<float4*>(my_stg + c) =
                  make_float4(__uint_as_float(r[c]), __uint_as_float(r[c + 1]), __uint_as_float(r[c + 2]),
                              __uint_as_float(r[c + 3]));
          }
          __syncwarp();
          const int lim = min(16, G.q0 + G.nq - (tile_row0 + 16 * pass));  // rows of the group
#pragma unroll 1
          for (int rr = 0; rr < lim; ++rr) {
            const int grow = tile_row0 + 16 * pass + rr;
            if (!cols_lane || !VDN_IN_BOUNDS(grow >= 0 && grow < l.L(), &g_readout_status)) continue;
            const long long off = ((long long)b * l.L() + grow) * HD + (long long)h * D + 4 * lane;
            const float4 a4 = *reinterpret_cast<const float4*>(stg + rr * C::kStgStride + 4 * lane);
            if constexpr (kMode == 2)
              *reinterpret_cast<float4*>(o_lin32 + off) = a4;
            else
              *reinterpret_cast<uint2*>(o_lin + off) = make_uint2(pack_bf16(a4.x, a4.y), pack_bf16(a4.z, a4.w));
          }
          __syncwarp();  // the staging is rewritten by the next pass
        }
      }
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::kTmemCols)
                 : "memory");
  }
}

template <int D, int kMode>
cudaError_t launch_readout_t(const Layout& l, const void* q, const float* states, void* o_lin,
                             const CombineArgs& cx, cudaStream_t st) {
  CUtensorMap mq;
  if (!make_map(&mq, q, D, l.H, l.L(), l.B)) return cudaErrorInvalidValue;
  auto kern = readout_tc_kernel<D, kMode>;
  const int smem = RCfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles_per_head(l, kRows * kTilesPerCta), l.H, l.B);
  if (grid.x == 0) return cudaSuccess;
  kern<<<grid, kThreads, smem, st>>>(mq, l, states, o_lin, cx);
  return cudaGetLastError();
}

}  // namespace

bool readout_tc_supported(const Layout& l, int dtype) {
  return dtype == VDN_BF16 && (l.d == 64 || l.d == 128);
}

cudaError_t launch_readout_tc(const Layout& l, const void* q, const float* states, void* o_lin,
                              bool out_f32, cudaStream_t st) {
  const CombineArgs cx{};
  if (l.d == 128)
    return out_f32 ? launch_readout_t<128, 2>(l, q, states, o_lin, cx, st)
                   : launch_readout_t<128, 0>(l, q, states, o_lin, cx, st);
  if (l.d == 64)
    return out_f32 ? launch_readout_t<64, 2>(l, q, states, o_lin, cx, st)
                   : launch_readout_t<64, 0>(l, q, states, o_lin, cx, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_combine_tc(const Layout& l, const void* q, const float* states,
                              const float* o_soft, const void* gs, const void* gl,
                              const float* rms_w, float eps, void* out, void* out_soft,
                              void* out_lin, cudaStream_t st) {
  const CombineArgs cx{o_soft, static_cast<const __nv_bfloat16*>(gs),
                       static_cast<const __nv_bfloat16*>(gl), rms_w, eps,
                       static_cast<__nv_bfloat16*>(out), static_cast<__nv_bfloat16*>(out_soft),
                       static_cast<__nv_bfloat16*>(out_lin)};
  if (l.d == 128) return launch_readout_t<128, 1>(l, q, states, nullptr, cx, st);
  if (l.d == 64) return launch_readout_t<64, 1>(l, q, states, nullptr, cx, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
