// Frame Gram matrices of Video Delta Attention on the 5th-generation tensor
// cores (project page "Video Delta Attention: A Frame-Wise Solution"):
//   A_f = K_f^T Diag(beta_f) K_f,   B_f = V_f^T Diag(beta_f) K_f
// over the U tokens of one frame (or of the text, slot 0), fp32 results.
//
// CTA = one (b, h, slot); 256 threads:
//   warp 0     TMA producer: 32-token K and V tiles into a ring of stages
//   warp 1     MMA issuer (one lane) and TMEM owner
//   warps 2-7  scalers: write Kw = beta (.) K into a ring of two Kw slots
//              (separate from the K/V ring, so that more K/V tiles are in
//              flight in the same shared memory) as two bf16 parts,
//              Kw_hi = bf16(beta k) and Kw_lo = bf16(beta k - Kw_hi), so that the
//              products keep ~16 significant bits of beta k (a single bf16 copy
//              put the chunk states 1e-2 off); six threads per token row, the
//              betas of the next tiles in flight in a register ring, beta = 0
//              past the frame (which also masks the ragged last tile); then
//              warps 2-5 read A and B out of TMEM.
// Both MMA operands are MN-major (token = K dimension, contiguous along d):
//   d = 128: one M = 128, N = 256 MMA per Kw part (hi, lo) and 16 tokens,
//            D[j][n] += sum_u Kw[u][j] [K | V][u][n]: columns 0..127 hold
//            A_f[j][n] (A_f is symmetric), columns 128..255 hold B_f[n][j],
//            i.e. TMEM lane j holds row j of A_f and column j of B_f;
//   d = 64:  one M = 128 MMA with [K^T; V^T] stacked along M (the V tile sits
//            one leading-byte-offset after the K tile): lanes 0-63 = A, 64-127 = B.
// The work is HBM-bound: each token's k and v are read once.
//
// Epilogue: B_f goes to global memory; A_f is staged in the freed shared rings
// and all 256 threads invert I + A_f in place with the
// register-blocked Gauss-Jordan of spd_inverse.cuh (two pivots per barrier,
// packed f32x2 updates), writing M_f = (I + A_f)^-1
// to the am slot. The inverse is a latency-bound chain of d dependent pivots;
// done here, it overlaps the other CTA of the SM streaming its frame instead
// of running as a separate launch after every Gram has finished.
#include "spd_inverse.cuh"
#include "tc_common.cuh"

namespace vdn {

__device__ int g_gram_status = 0;

cudaError_t set_role_wait_gram(unsigned long long ns) { return set_role_wait_ns(ns); }

cudaError_t read_and_clear_gram_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_gram_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_gram_status, &zero, sizeof(int));
}

namespace {

constexpr int kTok = 32;        // tokens per tile (96 KB of stages: two CTAs per SM)
constexpr int kThreads = 256;
constexpr int kScalers = 192;  // warps 2-7 scale beta k; warps 2-5 also drain TMEM
constexpr int kHalfBytes = kTok * 128;  // kTok tokens x 64 bf16 (one swizzle atom column)

template <int D>
struct GCfg {
  static constexpr int kHalves = D / 64;
  static constexpr int kTileBytes = kTok * D * 2;
  static constexpr int kStageBytes = 2 * kTileBytes;          // K, V
  static constexpr int kStages = (D == 128) ? 4 : 8;
  static constexpr int kKwBytes = 2 * kTileBytes;             // Kw_hi, Kw_lo
  static constexpr int kKwSlots = 2;
  static constexpr int kTmemCols = (D == 128) ? 256 : 64;
  static constexpr int kSmemBytes = 1024 + kStages * kStageBytes + kKwSlots * kKwBytes + 256;
  // after the last MMA the K/V ring and Kw slots are free: I + A is staged there
  // (row stride kAStride floats, padded against bank conflicts) for the inverse,
  // followed by the inverse's pivot row / column buffers
  static constexpr int kAStride = D + 4;
  static_assert(D * kAStride * 4 + 8 * D * 4 <= kStages * kStageBytes + kKwSlots * kKwBytes,
                "the inverse's staging must fit in the freed rings");
};

struct GBars {
  unsigned long long full[8];        // K/V stage loaded
  unsigned long long empty[8];       // K/V stage consumed by the MMAs
  unsigned long long kw_full[2];     // Kw slot written by the scalers
  unsigned long long kw_empty[2];    // Kw slot consumed by the MMAs
  unsigned long long done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool gwait(unsigned long long* bar, uint32_t parity, volatile int* abort,
                                      bool watch_abort = true) {
  if (mbar_try_wait(smem_u32(bar), parity)) return true;
  return mbar_wait_impl(bar, parity, abort, &g_gram_status, watch_abort);
}

// kind::f16 instruction descriptor with both operands MN-major.
__host__ __device__ constexpr uint32_t idesc_mn_mn(int n) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

// Slot s -> frame: slot 0 = text (when present), then frames 1..fwd_max, then rev_lo..F-2.
struct GramSlots {
  int has_text, fwd_max, rev_lo;
  __device__ int frame(int i) const {
    if (has_text) {
      if (i == 0) return 0;
      --i;
    }
    if (i < fwd_max) return 1 + i;
    return rev_lo + (i - fwd_max);
  }
};

// Packed fp32 multiply (sm_100 f32x2 arithmetic) for the beta k split; the
// pack, unpack and fma helpers come from spd_inverse.cuh.
__device__ __forceinline__ unsigned long long sp_mul2(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
constexpr unsigned long long kMinusOne2 = 0xBF800000BF800000ull;  // (-1.f, -1.f)

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
gram_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
               const __grid_constant__ CUtensorMap tm_kt, const __grid_constant__ CUtensorMap tm_vt,
               const Layout l, const GramSlots slots, const float* __restrict__ beta,
               const float* __restrict__ beta_t, float* __restrict__ am, float* __restrict__ bw) {
  using C = GCfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sKw = smem + C::kStages * C::kStageBytes;
  GBars* bars = reinterpret_cast<GBars*>(sKw + C::kKwSlots * C::kKwBytes);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  const bool text = slots.has_text && blockIdx.x == 0;
  const int f = slots.frame(blockIdx.x);
  const int U = text ? l.T : l.N;
  const int row0 = text ? 0 : f * l.N;         // first token row in the tensor
  const int n_tiles = (U + kTok - 1) / kTok;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 1);
    }
    for (int j = 0; j < C::kKwSlots; ++j) {
      mbar_init(&bars->kw_full[j], kScalers);
      mbar_init(&bars->kw_empty[j], 1);
    }
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
      // ----------------------------------------------------------- producer
      const CUtensorMap* mk = text ? &tm_kt : &tm_k;
      const CUtensorMap* mv = text ? &tm_vt : &tm_v;
      int issued = 0;
      bool ok = true;
      for (int t = 0; t < n_tiles; ++t) {
        const int s = t % C::kStages, use = t / C::kStages;
        if (use > 0 && !gwait(&bars->empty[s], (use - 1) & 1, abort)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * C::kStageBytes;
        mbar_expect_tx(&bars->full[s], 2 * C::kTileBytes);
        for (int hf = 0; hf < C::kHalves; ++hf) {
          tma_load_4d(st + hf * kHalfBytes, mk, &bars->full[s], hf * 64, h, row0 + t * kTok, b);
          tma_load_4d(st + C::kTileBytes + hf * kHalfBytes, mv, &bars->full[s], hf * 64, h,
                      row0 + t * kTok, b);
        }
        ++issued;
      }
      if (!ok) {
        // no copy may still be landing when the CTA exits
        for (int s = 0; s < C::kStages && s < issued; ++s) {
          const int last = issued - 1 - ((issued - 1 - s) % C::kStages);
          gwait(&bars->full[s], (last / C::kStages) & 1, abort, false);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc = idesc_mn_mn(D);      // d = 64: M = 128 ([K^T; V^T]), N = 64
      constexpr uint32_t idesc256 = idesc_mn_mn(256);  // d = 128: M = 128 (Kw^T), N = 256
      bool ok = true;
      for (int t = 0; t < n_tiles && ok; ++t) {
        const int s = t % C::kStages;
        const int j = t % C::kKwSlots, juse = t / C::kKwSlots;
        // the scalers wrote Kw of tile t after its K/V stage had landed
        if (!gwait(&bars->kw_full[j], juse & 1, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * C::kStageBytes);
        const uint32_t kw = smem_u32(sKw + j * C::kKwBytes);
        const uint32_t k_addr = st;
#pragma unroll
        for (int ks = 0; ks < kTok / 16; ++ks) {
          const uint32_t koff = ks * 16 * 128;
#pragma unroll
          for (int part = 0; part < 2; ++part) {
            const uint32_t acc = (t > 0 || ks > 0 || part > 0) ? 1u : 0u;
            const uint64_t kwdesc = desc_mn_sw128(kw + part * C::kTileBytes + koff, kHalfBytes);
            if (D == 128) {
              // one N = 256 MMA: D[j][n] = sum_u Kw[u][j] [K | V][u][n] (the K and
              // V tiles of a stage are adjacent, so their four 64-column atoms
              // are one operand with a uniform atom stride)
              mma_ss(tmem, kwdesc, desc_mn_sw128(k_addr + koff, kHalfBytes), idesc256, acc);
            } else {
              // [K^T; V^T]: the two 64-wide M blocks are the K and V tiles
              mma_ss(tmem, desc_mn_sw128(k_addr + koff, C::kTileBytes), kwdesc, idesc, acc);
            }
          }
        }
        tc_commit(&bars->empty[s]);
        tc_commit(&bars->kw_empty[j]);
      }
      tc_commit(&bars->done);
      if (!ok) gwait(&bars->done, 0, abort, false);
    }
  } else {
    // ---------------------------------------------------- scalers / epilogue
    // 6 threads per token row, each scaling chunks [c_lo, c_hi) of the row's
    // D / 8 16-byte chunks (at most 3)
    const int u = threadIdx.x - 64;
    constexpr int kTpr = kScalers / kTok;         // threads per token row
    constexpr int kChunks = D / 8;                // 16-byte chunks per row
    constexpr int kCpt = (kChunks + kTpr - 1) / kTpr;
    static_assert(kTpr * kTok == kScalers, "scaler threads cover the tile's rows");
    const int r = u / kTpr, part = u % kTpr;
    const int c_lo = part * kChunks / kTpr, c_hi = (part + 1) * kChunks / kTpr;
    auto beta_of = [&](int t) -> float {
      const int tok = t * kTok + r;
      if (tok >= U) return 0.f;
      if (!VDN_IN_BOUNDS(text || row0 + tok < l.L(), &g_gram_status)) return 0.f;
      return text ? beta_t[((long long)b * l.T + tok) * l.H + h]
                  : beta[((long long)b * l.L() + row0 + tok) * l.H + h];
    };
    // beta is a strided 4-byte read per token, a DRAM round trip per tile: the
    // betas of the next kAhead tiles stay in flight in a register ring, so that
    // no tile waits for its own (fetching one tile ahead left every tile a
    // round trip long)
    constexpr int kAhead = 8;
    float bq[kAhead];
#pragma unroll
    for (int i = 0; i < kAhead; ++i) bq[i] = i < n_tiles ? beta_of(i) : 0.f;
    bool ok = true;
    for (int t0 = 0; t0 < n_tiles && ok; t0 += kAhead) {
#pragma unroll
      for (int i = 0; i < kAhead; ++i) {
        const int t = t0 + i;
        if (t >= n_tiles || !ok) break;
        const int s = t % C::kStages, use = t / C::kStages;
        const int j = t % C::kKwSlots, juse = t / C::kKwSlots;
        const float bu = bq[i];
        const unsigned long long bu2 = spd_pack(bu, bu);
        bq[i] = t + kAhead < n_tiles ? beta_of(t + kAhead) : 0.f;
        if (!__all_sync(0xffffffffu, gwait(&bars->full[s], use & 1, abort))) {
          ok = false;
          break;
        }
        // the Kw slot is free once the MMAs of tile t - kKwSlots have completed
        if (juse > 0 && !__all_sync(0xffffffffu, gwait(&bars->kw_empty[j], (juse - 1) & 1, abort))) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * C::kStageBytes;
        uint8_t* kwp = sKw + j * C::kKwBytes;
#pragma unroll
        for (int cc = 0; cc < kCpt; ++cc) {
          const int chunk = c_lo + cc;              // 0 .. D/8 - 1 within the row
          if (chunk >= c_hi) break;
          const int hf = chunk / 8, c = chunk % 8;  // (swizzle permutes chunks within a row;
                                                    //  the scaling does not care which)
          const int off = hf * kHalfBytes + r * 128 + c * 16;
          const uint4 x = *reinterpret_cast<const uint4*>(st + off);
          const uint32_t w[4] = {x.x, x.y, x.z, x.w};
          uint32_t hi4[4], lo4[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // the element pair as floats (even element in the low half), times
            // beta in one packed multiply; hi = bf16(beta k); lo = bf16(beta k - hi)
            // with the exact difference from one packed fma with -1
            const unsigned long long p2 =
                sp_mul2(spd_pack(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xFFFF0000u)), bu2);
            float p0, p1;
            spd_unpack(p2, p0, p1);
            hi4[e] = pack_bf16(p0, p1);
            const unsigned long long h2 =
                spd_pack(__uint_as_float(hi4[e] << 16), __uint_as_float(hi4[e] & 0xFFFF0000u));
            float l0, l1;
            spd_unpack(spd_fma2(h2, kMinusOne2, p2), l0, l1);
            lo4[e] = pack_bf16(l0, l1);
          }
          *reinterpret_cast<uint4*>(kwp + off) = make_uint4(hi4[0], hi4[1], hi4[2], hi4[3]);
          *reinterpret_cast<uint4*>(kwp + C::kTileBytes + off) = make_uint4(lo4[0], lo4[1], lo4[2], lo4[3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&bars->kw_full[j]);
      }
    }
    // warps 2-5 drain TMEM (warp w reaches lanes 32 (w mod 4) .. + 31)
    if (warp < 6 && ok) ok = __all_sync(0xffffffffu, gwait(&bars->done, 0, abort));
    if (warp < 6 && ok) {
      tc_fence_after();
      const int m = 32 * (warp & 3) + lane;  // TMEM lane = output row
      const uint32_t taddr = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      const long long slot = ((long long)b * l.H + h) * l.F + f;
      const bool slot_ok = VDN_IN_BOUNDS(f >= 0 && f < l.F && h < l.H && b < l.B, &g_gram_status);
      // A_f (rows of TMEM columns 0..D-1 for d = 128, lanes 0..63 for d = 64) goes
      // to the shared staging of the inverse, B_f to global memory; the staging
      // reuses ring memory last touched by the copies and the tensor cores
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      float* as = reinterpret_cast<float*>(smem);
      float* arow;
      float* bcol = bw + slot * D * D + m;  // d = 128: column m of B_f
      if (D == 128) {
        arow = as + m * C::kAStride;
      } else {
        arow = (m < 64) ? as + m * C::kAStride : bw + slot * D * D + (long long)(m - 64) * D;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < D; c0 += 32) {
        uint32_t r[32];
        tmem_ld_x32(taddr + c0, r);
        float4* dst = reinterpret_cast<float4*>(arow + c0);
#pragma unroll
        for (int i = 0; i < 8 && slot_ok; ++i)
          dst[i] = make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]),
                               __uint_as_float(r[4 * i + 2]), __uint_as_float(r[4 * i + 3]));
      }
      if (D == 128) {
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t r[32];
          tmem_ld_x32(taddr + 128 + c0, r);
          // lane m holds column m of B_f (rows c0 .. c0 + 31): each store of the
          // warp is one 128-byte row segment
#pragma unroll
          for (int i = 0; i < 32 && slot_ok; ++i) bcol[(long long)(c0 + i) * D] = __uint_as_float(r[i]);
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
  // M_f = (I + A_f)^-1 in place of A_f, by all 256 threads (spd_inverse.cuh),
  // while the other CTA on the SM streams its frame; skipped as a whole when a
  // role gave up (the staging is then incomplete)
  if (*abort) return;
  {
    constexpr int RA = D / 16;
    const float* as = reinterpret_cast<const float*>(smem);
    float (*rowk)[2][D] = reinterpret_cast<float (*)[2][D]>(smem + D * C::kAStride * 4);
    float (*colk)[2][D] = rowk + 2;
    const int tr = threadIdx.x / 16, tc = threadIdx.x % 16;
    float a[RA][RA];
#pragma unroll
    for (int x = 0; x < RA; ++x)
#pragma unroll
      for (int y = 0; y < RA; ++y) {
        const int i = tr + 16 * x, j = tc + 16 * y;
        a[x][y] = as[i * C::kAStride + j] + (i == j ? 1.f : 0.f);
      }
    spd_inverse_blocks2x<D>(a, tr, tc, rowk, colk);
    const long long slot = ((long long)b * l.H + h) * l.F + f;
    if (!VDN_IN_BOUNDS(f >= 0 && f < l.F && h < l.H && b < l.B, &g_gram_status)) return;
    float* g = am + slot * D * D;
#pragma unroll
    for (int x = 0; x < RA; ++x)
#pragma unroll
      for (int y = 0; y < RA; ++y) g[(tr + 16 * x) * D + tc + 16 * y] = a[x][y];
  }
}

template <int D>
cudaError_t launch_gram_t(const Layout& l, const GramSlots& slots, int nslots, const void* k,
                          const void* v, const void* kt, const void* vt, const float* beta,
                          const float* beta_t, float* am, float* bw, cudaStream_t st) {
  CUtensorMap mk, mv, mkt, mvt;
  if (!make_map(&mk, k, D, l.H, l.L(), l.B, kTok) || !make_map(&mv, v, D, l.H, l.L(), l.B, kTok))
    return cudaErrorInvalidValue;
  if (l.T > 0) {
    if (!make_map(&mkt, kt, D, l.H, l.T, l.B, kTok) || !make_map(&mvt, vt, D, l.H, l.T, l.B, kTok))
      return cudaErrorInvalidValue;
  } else {
    mkt = mk;
    mvt = mv;
  }
  auto kern = gram_tc_kernel<D>;
  const int smem = GCfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  kern<<<dim3(nslots, l.H, l.B), kThreads, smem, st>>>(mk, mv, mkt, mvt, l, slots, beta, beta_t, am, bw);
  return cudaGetLastError();
}

}  // namespace

bool gram_tc_supported(const Layout& l, int dtype) {
  return dtype == VDN_BF16 && (l.d == 64 || l.d == 128);
}

cudaError_t launch_gram_tc(const Layout& l, int has_text, int fwd_max, int rev_lo, int nslots,
                           const void* k, const void* v, const void* kt, const void* vt,
                           const float* beta, const float* beta_t, float* am, float* bw,
                           cudaStream_t st) {
  GramSlots slots{has_text, fwd_max, rev_lo};
  if (nslots <= 0) return cudaSuccess;
  if (l.d == 128) return launch_gram_t<128>(l, slots, nslots, k, v, kt, vt, beta, beta_t, am, bw, st);
  if (l.d == 64) return launch_gram_t<64>(l, slots, nslots, k, v, kt, vt, beta, beta_t, am, bw, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
