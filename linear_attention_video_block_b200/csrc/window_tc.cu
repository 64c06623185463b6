// Block-sparse window softmax on the 5th-generation tensor cores (sm_100a):
// tcgen05.mma with TMEM accumulators, operands staged by TMA, bf16 inputs,
// fp32 scores / softmax statistics / output accumulation.
//
// What it computes (project page "Local Softmax and Long-Range Linear Memory"):
// for every video query, softmax(q K^T / sqrt(d)) V over the keys of its
// chunk window, the boundary anchor frames and all text tokens (and, in a
// joint text-video-audio layer, all audio tokens), one normaliser. Keys are
// visited per query group as merged token segments (window/anchor intervals,
// then text, then audio) in 128-key tiles; only the last tile of each segment
// is partially masked. In a joint layer the text and audio query rows are
// extra groups of the same grid whose key set is every token (the dense
// softmax the pages keep for interactions involving text or audio); they are
// scheduled first, being the longest.
//
// CTA = 256 query rows (two 128-row Q tiles) of one query group of one
// (b, h); 320 threads (at most 200 registers each):
//   warps 0-3   softmax warpgroup of Q tile 0 (thread i owns row i = TMEM lane i)
//   warps 4-7   softmax warpgroup of Q tile 1
//   warp  8     lane 0: TMA producer (Q once, then K_t, V_t tiles into a ring
//               of shared-memory slots)
//   warp  9     MMA issuer (one elected lane) and TMEM owner
// The hybrid output is finished by the tensor-core readout (readout_tc.cu)
// from this kernel's float32 o_soft: fusing the readout, RMSNorm and gates
// into this epilogue was measured slower (the long per-CTA epilogue holds the
// SM, one CTA per SM, while a separate pass runs at full occupancy).
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d,256+2d).
// P (bf16) overwrites the first 64 columns of S and is the A operand of P.V
// straight from TMEM. MMA issue order per key tile t:
//   PV0(t), S0(t+1), PV1(t), S1(t+1)
// so softmax of one Q tile overlaps the tensor-core work of the other.
// The tcgen05.commit after S_w(t) also covers PV_w(t-1), so when softmax w sees
// S_w(t) its O accumulator is stable and can be rescaled in place (lazy
// rescaling: only when the running max grows by more than 2^8).
//
// Every mbarrier wait is bounded (%globaltimer, 4 s); a timeout records
// VDN_ERR_TIMEOUT in the status word, the roles leave their loops, the
// producer waits (bounded) for its copies in flight, the MMA issuer waits for
// its MMAs, and TMEM is freed before exit.
#include "tc_common.cuh"

namespace vdn {

// Device-side status word of this translation unit.
__device__ int g_vdn_status = 0;

cudaError_t set_role_wait_tc(unsigned long long ns) { return set_role_wait_ns(ns); }

cudaError_t read_and_clear_tc_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_vdn_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_vdn_status, &zero, sizeof(int));
}

namespace {

constexpr int kRows = 128;           // rows of a Q tile = keys of a K/V tile
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTmemCols = 512;

template <int D>
struct Cfg {
  static constexpr int kHalves = D / 64;               // 128-byte swizzle atoms per row
  static constexpr int kTileBytes = kRows * D * 2;     // one 128 x D bf16 tile
  static constexpr int kHalfBytes = kRows * 128;       // one 128-row x 64-column atom column
  static constexpr int kSlots = (D == 128) ? 4 : 8;
  static constexpr int kQBytes = 2 * kTileBytes;
  static constexpr int kSmemBytes = 1024 + kQBytes + kSlots * kTileBytes + 256;
};

struct Bars {
  unsigned long long q_full;
  unsigned long long kv_full[8];
  unsigned long long kv_empty[8];
  unsigned long long s_full[2];
  unsigned long long p_full[2][2];   // [Q tile][key half]: P of keys 0..63 / 64..127
  unsigned long long o_full;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity,
                                          volatile int* abort, bool watch_abort = true) {
  if (mbar_try_wait(smem_u32(bar), parity)) return true;
  return mbar_wait_impl(bar, parity, abort, &g_vdn_status, watch_abort);
}

// ------------------------------------------------------------------ kernel

// Outputs of the context query rows (joint layer), io dtype [B, T|A, H, D].
struct CtxOut {
  __nv_bfloat16* o_text;
  __nv_bfloat16* o_audio;
  float* lse_text;
  float* lse_audio;
};

// Packed fp32 pairs (sm_100 f32x2 arithmetic) and the 3-input max: they halve
// the instruction count of the softmax's per-element work.
__device__ __forceinline__ unsigned long long f2pack(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b,
                                                    unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ unsigned long long f2add(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
window_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                 const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
                 const __grid_constant__ CUtensorMap tm_vt, const __grid_constant__ CUtensorMap tm_ka,
                 const __grid_constant__ CUtensorMap tm_va, const __grid_constant__ CUtensorMap tm_qt,
                 const __grid_constant__ CUtensorMap tm_qa, const Layout l, void* out, int out_f32,
                 float* lse, const CtxOut cx) {
  using C = Cfg<D>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + C::kQBytes;
  Bars* bars = reinterpret_cast<Bars*>(sKV + C::kSlots * C::kTileBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  int g, r0;
  tile_to_group(l, 2 * kRows, blockIdx.x, g, r0);
  const Group G = make_group(l, g < 0 ? 0 : g);
  const int n_tiles = key_tile_count(G, l.T, l.A, kRows);
  const bool ctx_rows = G.qsrc != kQVideo;

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < C::kSlots; ++i) {
      mbar_init(&bars->kv_full[i], 1);
      mbar_init(&bars->kv_empty[i], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&bars->s_full[w], 1);
      mbar_init(&bars->p_full[w][0], 128);
      mbar_init(&bars->p_full[w][1], 128);
    }
    mbar_init(&bars->o_full, 1);
    bars->abort = (g < 0) ? 1 : 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&bars->tmem_base)), "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  volatile int* abort = &bars->abort;

  if (warp == kProducerWarp) {
    if (lane == 0 && !*abort) {
      // ------------------------------------------------------- TMA producer
      const CUtensorMap* mq = G.qsrc == kQVideo ? &tm_q : (G.qsrc == kQText ? &tm_qt : &tm_qa);
      mbar_expect_tx(&bars->q_full, 2 * C::kTileBytes);
      for (int qt = 0; qt < 2; ++qt)
        for (int hf = 0; hf < C::kHalves; ++hf)
          tma_load_4d(sQ + qt * C::kTileBytes + hf * C::kHalfBytes, mq, &bars->q_full, hf * 64,
                      h, r0 + qt * kRows, b);
      int fill = 0;
      bool ok = true;
      for (int t = 0; t < n_tiles && ok; ++t) {
        const KeyTile kt = key_tile(G, l.T, l.A, t, kRows);
        // checked build: the schedule's key rows lie inside their tensor (a copy
        // past the end would read zeros, so this is a check of the schedule)
        (void)VDN_IN_BOUNDS(kt.row >= 0 && kt.row < (kt.src == kKVideo ? l.L() : kt.src == kKText ? l.T : l.A),
                      &g_vdn_status);
        for (int kv = 0; kv < 2; ++kv, ++fill) {
          const int slot = fill % C::kSlots;
          const int use = fill / C::kSlots;
          if (use > 0 && !mbar_wait(&bars->kv_empty[slot], (use - 1) & 1, abort)) {
            ok = false;
            break;
          }
          const CUtensorMap* map = kt.src == kKVideo ? (kv ? &tm_v : &tm_k)
                                   : kt.src == kKText ? (kv ? &tm_vt : &tm_kt)
                                                      : (kv ? &tm_va : &tm_ka);
          mbar_expect_tx(&bars->kv_full[slot], C::kTileBytes);
          for (int hf = 0; hf < C::kHalves; ++hf)
            tma_load_4d(sKV + slot * C::kTileBytes + hf * C::kHalfBytes, map, &bars->kv_full[slot],
                        hf * 64, h, kt.row, b);
        }
      }
      if (!ok) {
        // leave no copy in flight into this CTA's shared memory: the last fill
        // of slot s was number (fill - 1 - ((fill - 1 - s) mod kSlots))
        mbar_wait(&bars->q_full, 0, abort, false);
        for (int s = 0; s < C::kSlots && s < fill; ++s) {
          const int last = fill - 1 - ((fill - 1 - s) % C::kSlots);
          mbar_wait(&bars->kv_full[s], (last / C::kSlots) & 1, abort, false);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && !*abort) {
      // ------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = make_idesc(kRows, false);
      constexpr uint32_t idesc_o = make_idesc(D, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t kv_addr = smem_u32(sKV);
      int use = 0;
      bool ok = mbar_wait(&bars->q_full, 0, abort);
      auto take_slot = [&](int& slot) -> bool {
        slot = use % C::kSlots;
        const bool r = mbar_wait(&bars->kv_full[slot], (use / C::kSlots) & 1, abort);
        ++use;
        tc_fence_after();
        return r;
      };
      // descriptors: the start address sits in the low 14 bits (address / 16),
      // so an operand's k-step descriptors are its base descriptor plus offset / 16
      const uint64_t qd0 = desc_k_sw128(q_addr), kvd0 = desc_k_sw128(kv_addr);
      const uint64_t vd0 = desc_mn_sw128(kv_addr, C::kHalfBytes);
      auto issue_s = [&](int w, int slot) {
        const uint32_t d_tmem = tmem + 128 * w;
        const uint64_t qd = qd0 + (uint64_t)((w * C::kTileBytes) >> 4);
        const uint64_t kd = kvd0 + (uint64_t)((slot * C::kTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks / 4) * C::kHalfBytes + (ks % 4) * 32) >> 4;
          mma_ss(d_tmem, qd + off, kd + off, idesc_s, ks > 0 ? 1u : 0u);
        }
      };
      // O_w += P_w V for one half of the key tile (keys 64 half .. 64 half + 63)
      auto issue_pv_half = [&](int w, int slot, bool acc, int half) {
        const uint32_t d_tmem = tmem + 256 + D * w;
        const uint32_t a_tmem = tmem + 128 * w;
        const uint64_t vd = vd0 + (uint64_t)((slot * C::kTileBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kRows / 32; ++kk) {
          const int ks = 4 * half + kk;
          mma_ts(d_tmem, a_tmem + ks * 8, vd + (uint64_t)(ks * 16 * 128 / 16), idesc_o,
                 (acc || ks > 0) ? 1u : 0u);
        }
      };
      // P_w(t) is published in two halves; the first half's P.V runs while the
      // softmax computes the second
      auto issue_pv = [&](int w, int slot, bool acc, int t) -> bool {
        for (int half = 0; half < 2; ++half) {
          if (!mbar_wait(&bars->p_full[w][half], t & 1, abort)) return false;
          tc_fence_after();
          issue_pv_half(w, slot, acc, half);
        }
        return true;
      };
      int ks_cur = 0;
      if (ok) ok = take_slot(ks_cur);
      if (ok) {
        issue_s(0, ks_cur);
        tc_commit(&bars->s_full[0]);
        issue_s(1, ks_cur);
        tc_commit(&bars->s_full[1]);
        tc_commit(&bars->kv_empty[ks_cur]);
      }
      for (int t = 0; t < n_tiles && ok; ++t) {
        int vs = 0, ks_next = 0;
        if (!take_slot(vs)) { ok = false; break; }
        if (!issue_pv(0, vs, t > 0, t)) { ok = false; break; }
        const bool more = t + 1 < n_tiles;
        if (more) {
          if (!take_slot(ks_next)) { ok = false; break; }
          issue_s(0, ks_next);
          tc_commit(&bars->s_full[0]);
        }
        if (!issue_pv(1, vs, t > 0, t)) { ok = false; break; }
        tc_commit(&bars->kv_empty[vs]);
        if (more) {
          issue_s(1, ks_next);
          tc_commit(&bars->s_full[1]);
          tc_commit(&bars->kv_empty[ks_next]);
        }
      }
      tc_commit(&bars->o_full);
      // every MMA issued must finish before TMEM is freed
      if (!ok) mbar_wait(&bars->o_full, 0, abort, false);
    }
  } else {
    // ----------------------------------------------------------- softmax
    const int w = warp / 4;
    const int row = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_base + 128 * w;
    const uint32_t tO = tmem + lane_base + 256 + D * w;
    const float sl2 = 1.4426950408889634f / sqrtf((float)D);  // log2(e) / sqrt(d)
    float m = -INFINITY, lsum = 0.f;
    bool ok = !*abort;
    // The only partially valid key tiles are the last tile of each segment
    // (3 video segments at most, then the text, then the audio): (tile index
    // << 8) | valid count for each (valid <= 128 fits in 8 bits; -1 when a
    // segment is empty).
    int edge[5];
    {
      int first = 0;
#pragma unroll
      for (int sgi = 0; sgi < 5; ++sgi) {
        const int len = (sgi < 3) ? ((sgi < G.nseg) ? G.segn[sgi] : 0) : (sgi == 3 ? l.T : l.A);
        const int n = (len + kRows - 1) / kRows;
        edge[sgi] = (n > 0) ? (((first + n - 1) << 8) | (len - (n - 1) * kRows)) : -1;
        first += n;
      }
    }
    const int q_end = G.q0 + G.nq;
    for (int t = 0; t < n_tiles && ok; ++t) {
      // the TMEM loads below are warp-collective: leave only as a whole warp
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[w], t & 1, abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128_split(tS, sr);
      float* s = reinterpret_cast<float*>(sr);
      int valid = kRows;
#pragma unroll
      for (int sgi = 0; sgi < 5; ++sgi)
        if (edge[sgi] >= 0 && (edge[sgi] >> 8) == t) valid = edge[sgi] & 255;
      if (valid < kRows) {
#pragma unroll
        for (int j = 0; j < kRows; ++j)
          if (j >= valid) s[j] = -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < kRows; j += 8) {
        mx4[0] = fmax3(mx4[0], s[j], s[j + 1]);
        mx4[1] = fmax3(mx4[1], s[j + 2], s[j + 3]);
        mx4[2] = fmax3(mx4[2], s[j + 4], s[j + 5]);
        mx4[3] = fmax3(mx4[3], s[j + 6], s[j + 7]);
      }
      const float mc = fmaxf(fmax3(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl2;
      if (t == 0) {
        m = mc;
      } else {
        const bool need = mc > m + 8.f;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2(m - mc) : 1.f;
#pragma unroll 1
          for (int c0 = 0; c0 < D; c0 += 32) {
            uint32_t o[32];
            tmem_ld_x32(tO + c0, o);
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st_x32(tO + c0, o);
          }
          if (need) {
            lsum *= f;
            m = mc;
          }
        }
      }
      const float nm = -m;
      const unsigned long long sl2x2 = f2pack(sl2, sl2), nmx2 = f2pack(nm, nm);
      unsigned long long sum2[2] = {0ull, 0ull};
      // P goes to TMEM in 8-column pieces as it is produced; each half of the
      // key tile (P columns 0..31 = keys 0..63, 32..63 = keys 64..127) is
      // published as soon as it is complete
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t p[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int j = 32 * half + 8 * c4 + jj;
            float xa, xc;
            f2unpack(f2fma(f2pack(s[2 * j], s[2 * j + 1]), sl2x2, nmx2), xa, xc);
            const float a = ex2(xa), c = ex2(xc);
            sum2[jj & 1] = f2add(sum2[jj & 1], f2pack(a, c));
            p[jj] = pack_bf16(a, c);
          }
          tmem_st_x8_nowait(tS + 32 * half + 8 * c4, p);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[w][half]);
      }
      {
        float s0, s1, s2, s3;
        f2unpack(sum2[0], s0, s1);
        f2unpack(sum2[1], s2, s3);
        lsum += (s0 + s1) + (s2 + s3);
      }
    }
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(&bars->o_full, 0, abort));
    if (ok) {
      tc_fence_after();
      const int grow = r0 + kRows * w + row;
      const bool store = grow < q_end;
      const float inv = 1.f / lsum;
      // rows of the query's own tensor: video [B, L, H, D], text [B, T, H, D],
      // audio [B, A, H, D]
      const long long qrows = G.qsrc == kQVideo ? l.L() : (G.qsrc == kQText ? l.T : l.A);
      const long long base = (((long long)b * qrows + grow) * l.H + h) * D;
      const bool store_ok = !store || VDN_IN_BOUNDS(grow >= 0 && grow < qrows, &g_vdn_status);
      {
        void* dst_o = out;
        float* dst_lse = lse;
        bool f32 = out_f32 != 0;
        if (ctx_rows) {
          dst_o = G.qsrc == kQText ? cx.o_text : cx.o_audio;
          dst_lse = G.qsrc == kQText ? cx.lse_text : cx.lse_audio;
          f32 = false;
        }
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld_x32(tO + c0, o);
          if (store && store_ok) {
            if (f32) {
              float4* dst = reinterpret_cast<float4*>(static_cast<float*>(dst_o) + base + c0);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                     __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
            } else {
              uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(dst_o) + base + c0);
#pragma unroll
              for (int i = 0; i < 4; ++i)
                dst[i] = make_uint4(pack_bf16(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                                    pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv),
                                    pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv),
                                    pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv));
            }
          }
        }
        if (store && store_ok && dst_lse)
          dst_lse[((long long)b * qrows + grow) * l.H + h] = (m + log2f(lsum)) * 0.6931471805599453f;
      }
    }
  }
  __syncwarp();  // elected lanes rejoin their warps
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------- host

template <int D>
cudaError_t launch_tc_t(const Layout& l, const void* q, const void* k, const void* v,
                        const void* kt, const void* vt, void* o, bool out_f32, float* lse,
                        const JointArgs& ja, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mkt, mvt, mka, mva, mqt, mqa;
  const long long L = l.L();
  if (!make_map(&mq, q, D, l.H, L, l.B) || !make_map(&mk, k, D, l.H, L, l.B) ||
      !make_map(&mv, v, D, l.H, L, l.B))
    return cudaErrorInvalidValue;
  // maps of absent tensors are copies that are never read (no tiles use them)
  mkt = mk; mvt = mv; mka = mk; mva = mv; mqt = mq; mqa = mq;
  if (l.T > 0 && (!make_map(&mkt, kt, D, l.H, l.T, l.B) || !make_map(&mvt, vt, D, l.H, l.T, l.B)))
    return cudaErrorInvalidValue;
  if (l.A > 0 && (!make_map(&mka, ja.k_audio, D, l.H, l.A, l.B) ||
                  !make_map(&mva, ja.v_audio, D, l.H, l.A, l.B)))
    return cudaErrorInvalidValue;
  if ((l.ctx & kCtxText) && l.T > 0 && !make_map(&mqt, ja.q_text, D, l.H, l.T, l.B))
    return cudaErrorInvalidValue;
  if ((l.ctx & kCtxAudio) && l.A > 0 && !make_map(&mqa, ja.q_audio, D, l.H, l.A, l.B))
    return cudaErrorInvalidValue;
  const CtxOut cx{static_cast<__nv_bfloat16*>(ja.o_text), static_cast<__nv_bfloat16*>(ja.o_audio),
                  ja.lse_text, ja.lse_audio};
  auto kern = window_tc_kernel<D>;
  const int smem = Cfg<D>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles_per_head(l, 2 * kRows), l.H, l.B);
  if (grid.x == 0) return cudaSuccess;
  kern<<<grid, kThreads, smem, st>>>(mq, mk, mv, mkt, mvt, mka, mva, mqt, mqa, l, o, out_f32 ? 1 : 0,
                                     lse, cx);
  return cudaGetLastError();
}

}  // namespace

bool window_tc_supported(const Layout& l, int dtype) {
  return dtype == VDN_BF16 && (l.d == 64 || l.d == 128);
}

cudaError_t launch_window_tc(const Layout& l, const void* q, const void* k, const void* v,
                             const void* kt, const void* vt, void* o, bool out_f32, float* lse,
                             const JointArgs& ja, cudaStream_t st) {
  if (l.d == 128) return launch_tc_t<128>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
  if (l.d == 64) return launch_tc_t<64>(l, q, k, v, kt, vt, o, out_f32, lse, ja, st);
  return cudaErrorInvalidValue;
}

}  // namespace vdn
