// Block-sparse window softmax with FP8 (e4m3) operands on the 5th-generation
// tensor cores (sm_100a, tcgen05.mma kind::f8f6f4), d = 128.
//
// Same operation and schedule as the bf16 kernel in window_tc.cu (project page
// "Local Softmax and Long-Range Linear Memory": each video query attends to its
// chunk window, the boundary anchor frames and all text tokens, one
// normaliser), for q, k, v (and the text keys / values) stored as e4m3 with one
// scale per tensor (value = e4m3 * scale; the text tensors share the scales of
// k and v). The FP8 path of the pages' serving stack ("FP8 linear attention";
// MXFP8 in the serving engine) is the motivation: half the operand bytes and
// twice the tensor-core rate of bf16.
//
// Differences from the bf16 kernel:
//   - 128 x 128 e4m3 tiles are one 128-byte swizzle atom wide (16 KB), so the
//     K/V ring has 8 slots; S = Q K^T takes 4 MMAs of K = 32.
//   - P is written to TMEM as e4m3, four keys per 32-bit column (32 columns per
//     key tile), and is the A operand of P.V (V MN-major, K = 32 per MMA).
//   - P = 2^(x - m + 6) with the reference max m raised only when a tile's max
//     exceeds it by more than 2, so P <= 2^8 (e4m3 holds up to 448) and the
//     weights keep 2^-15 of the row maximum before e4m3 underflows; the row sum
//     adds the float32 weights before rounding.
//   - Scores are scaled by q_scale * k_scale / sqrt(d), the output by v_scale.
//
// CTA = 256 query rows (two 128-row Q tiles) of one query group of one (b, h);
// 320 threads: warps 0-7 softmax (thread = row = TMEM lane), warp 8 lane 0 TMA
// producer, warp 9 MMA issuer and TMEM owner. MMA order per key tile t:
// PV0(t), S0(t+1), PV1(t), S1(t+1). Every mbarrier wait is bounded (4 s).
#include "tc_common.cuh"

namespace vdn {

__device__ int g_fp8_status = 0;

cudaError_t set_role_wait_fp8(unsigned long long ns) { return set_role_wait_ns(ns); }

cudaError_t read_and_clear_fp8_status(int* status) {
  cudaError_t e = cudaMemcpyFromSymbol(status, g_fp8_status, sizeof(int));
  if (e != cudaSuccess) return e;
  const int zero = 0;
  return cudaMemcpyToSymbol(g_fp8_status, &zero, sizeof(int));
}

namespace {

constexpr int kD = 128;
constexpr int kRows = 128;
constexpr int kThreads = 320;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kTmemCols = 512;
constexpr int kTileBytes = kRows * kD;   // 128 x 128 e4m3
constexpr int kSlots = 8;
constexpr int kQBytes = 2 * kTileBytes;
constexpr int kSmemBytes = 1024 + kQBytes + kSlots * kTileBytes + 256;
constexpr float kPShift = 6.f;            // P = 2^(x - m + kPShift)
constexpr float kLazy = 2.f;              // raise m when a tile max exceeds it by more

struct Bars8 {
  unsigned long long q_full;
  unsigned long long kv_full[kSlots];
  unsigned long long kv_empty[kSlots];
  unsigned long long s_full[2];
  unsigned long long p_full[2][2];
  unsigned long long o_full;
  uint32_t tmem_base;
  int abort;
};
static_assert(sizeof(Bars8) <= 256, "barrier area");

__device__ __forceinline__ bool wait8(unsigned long long* bar, uint32_t parity, volatile int* abort,
                                      bool watch_abort = true) {
  if (mbar_try_wait(smem_u32(bar), parity)) return true;
  return mbar_wait_impl(bar, parity, abort, &g_fp8_status, watch_abort);
}

// kind::f8f6f4 instruction descriptor: D f32, A and B e4m3 (format 0), M = 128.
__host__ __device__ constexpr uint32_t idesc_f8(int n, bool b_mn_major) {
  return (1u << 4) | (0u << 7) | (0u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_ts_f8(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n\t}\n"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ unsigned long long f2pack8(float a, float b) {
  unsigned long long r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2unpack8(unsigned long long r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ unsigned long long f2fma8(unsigned long long a, unsigned long long b,
                                                     unsigned long long c) {
  unsigned long long r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ unsigned long long f2add8(unsigned long long a, unsigned long long b) {
  unsigned long long r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ float fmax3_8(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Four weights as e4m3 in one 32-bit word, key order from the low byte up.
__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}\n"
      : "=r"(r) : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

__global__ void __launch_bounds__(kThreads, 1)
window_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_kt,
                  const __grid_constant__ CUtensorMap tm_vt, const Layout l, float qk_scale,
                  float v_scale, __nv_bfloat16* out, float* lse) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + kQBytes;
  Bars8* bars = reinterpret_cast<Bars8*>(sKV + kSlots * kTileBytes);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const int h = blockIdx.y, b = blockIdx.z;
  int g, r0;
  tile_to_group(l, 2 * kRows, blockIdx.x, g, r0);
  const Group G = make_group(l, g < 0 ? 0 : g);
  const int n_tiles = key_tile_count(G, l.T, 0, kRows);

  if (threadIdx.x == 0) {
    mbar_init(&bars->q_full, 1);
    for (int i = 0; i < kSlots; ++i) {
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
      mbar_expect_tx(&bars->q_full, 2 * kTileBytes);
      for (int qt = 0; qt < 2; ++qt)
        tma_load_4d(sQ + qt * kTileBytes, &tm_q, &bars->q_full, 0, h, r0 + qt * kRows, b);
      int fill = 0;
      bool ok = true;
      for (int t = 0; t < n_tiles && ok; ++t) {
        const KeyTile kt = key_tile(G, l.T, 0, t, kRows);
        (void)VDN_IN_BOUNDS(kt.row >= 0 && kt.row < (kt.src == kKVideo ? l.L() : l.T), &g_fp8_status);
        for (int kv = 0; kv < 2; ++kv, ++fill) {
          const int slot = fill % kSlots;
          const int use = fill / kSlots;
          if (use > 0 && !wait8(&bars->kv_empty[slot], (use - 1) & 1, abort)) {
            ok = false;
            break;
          }
          const CUtensorMap* map = kt.src == kKVideo ? (kv ? &tm_v : &tm_k) : (kv ? &tm_vt : &tm_kt);
          mbar_expect_tx(&bars->kv_full[slot], kTileBytes);
          tma_load_4d(sKV + slot * kTileBytes, map, &bars->kv_full[slot], 0, h, kt.row, b);
        }
      }
      if (!ok) {
        wait8(&bars->q_full, 0, abort, false);
        for (int s = 0; s < kSlots && s < fill; ++s) {
          const int last = fill - 1 - ((fill - 1 - s) % kSlots);
          wait8(&bars->kv_full[s], (last / kSlots) & 1, abort, false);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && !*abort) {
      // ------------------------------------------------------- MMA issuer
      constexpr uint32_t idesc_s = idesc_f8(kRows, false);
      constexpr uint32_t idesc_o = idesc_f8(kD, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t kv_addr = smem_u32(sKV);
      int use = 0;
      bool ok = wait8(&bars->q_full, 0, abort);
      auto take_slot = [&](int& slot) -> bool {
        slot = use % kSlots;
        const bool r = wait8(&bars->kv_full[slot], (use / kSlots) & 1, abort);
        ++use;
        tc_fence_after();
        return r;
      };
      // S_w = Q_w K^T: K = 128 e4m3 = one 128-byte atom, 4 MMAs of 32 bytes
      auto issue_s = [&](int w, int slot) {
        const uint32_t d_tmem = tmem + 128 * w;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          mma_ss_f8(d_tmem, desc_k_sw128(q_addr + w * kTileBytes + ks * 32),
                    desc_k_sw128(kv_addr + slot * kTileBytes + ks * 32), idesc_s, ks > 0 ? 1u : 0u);
      };
      // O_w += P_w V for keys 64 half .. 64 half + 63: two MMAs of 32 keys, P
      // from TMEM (8 columns per 32 keys), V MN-major (32 rows of 128 bytes)
      auto issue_pv_half = [&](int w, int slot, bool acc, int half) {
        const uint32_t d_tmem = tmem + 256 + kD * w;
        const uint32_t a_tmem = tmem + 128 * w;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
          const int ks = 2 * half + kk;
          mma_ts_f8(d_tmem, a_tmem + ks * 8,
                    desc_mn_sw128(kv_addr + slot * kTileBytes + ks * 32 * 128, kTileBytes),
                    idesc_o, (acc || ks > 0) ? 1u : 0u);
        }
      };
      auto issue_pv = [&](int w, int slot, bool acc, int t) -> bool {
        for (int half = 0; half < 2; ++half) {
          if (!wait8(&bars->p_full[w][half], t & 1, abort)) return false;
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
      if (!ok) wait8(&bars->o_full, 0, abort, false);
    }
  } else {
    // ----------------------------------------------------------- softmax
    const int w = warp / 4;
    const int row = threadIdx.x & 127;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t tS = tmem + lane_base + 128 * w;
    const uint32_t tO = tmem + lane_base + 256 + kD * w;
    const float sl2 = qk_scale * 1.4426950408889634f / sqrtf((float)kD);
    float m = -INFINITY, lsum = 0.f;
    bool ok = !*abort;
    int edge[4];
    {
      int first = 0;
#pragma unroll
      for (int sgi = 0; sgi < 4; ++sgi) {
        const int len = (sgi < 3) ? ((sgi < G.nseg) ? G.segn[sgi] : 0) : l.T;
        const int n = (len + kRows - 1) / kRows;
        edge[sgi] = (n > 0) ? (((first + n - 1) << 8) | (len - (n - 1) * kRows)) : -1;
        first += n;
      }
    }
    const int q_end = G.q0 + G.nq;
    for (int t = 0; t < n_tiles && ok; ++t) {
      if (!__all_sync(0xffffffffu, wait8(&bars->s_full[w], t & 1, abort))) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld_x128_split(tS, sr);
      float* s = reinterpret_cast<float*>(sr);
      int valid = kRows;
#pragma unroll
      for (int sgi = 0; sgi < 4; ++sgi)
        if (edge[sgi] >= 0 && (edge[sgi] >> 8) == t) valid = edge[sgi] & 255;
      if (valid < kRows) {
#pragma unroll
        for (int j = 0; j < kRows; ++j)
          if (j >= valid) s[j] = -INFINITY;
      }
      float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < kRows; j += 8) {
        mx4[0] = fmax3_8(mx4[0], s[j], s[j + 1]);
        mx4[1] = fmax3_8(mx4[1], s[j + 2], s[j + 3]);
        mx4[2] = fmax3_8(mx4[2], s[j + 4], s[j + 5]);
        mx4[3] = fmax3_8(mx4[3], s[j + 6], s[j + 7]);
      }
      const float mc = fmaxf(fmax3_8(mx4[0], mx4[1], mx4[2]), mx4[3]) * sl2;
      if (t == 0) {
        m = mc;
      } else {
        const bool need = mc > m + kLazy;
        if (__any_sync(0xffffffffu, need)) {
          const float f = need ? ex2(m - mc) : 1.f;
#pragma unroll 1
          for (int c0 = 0; c0 < kD; c0 += 32) {
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
      const float nm = kPShift - m;
      const unsigned long long sl2x2 = f2pack8(sl2, sl2), nmx2 = f2pack8(nm, nm);
      unsigned long long sum2[2] = {0ull, 0ull};
      // P as e4m3, four keys per TMEM column: keys 0..63 in columns 0..15,
      // published first, keys 64..127 in columns 16..31
#pragma unroll
      for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int c8 = 0; c8 < 2; ++c8) {
          uint32_t p[8];
#pragma unroll
          for (int jj = 0; jj < 8; ++jj) {
            const int k0 = 64 * half + 32 * c8 + 4 * jj;   // first key of this column
            float a0, a1, a2, a3;
            f2unpack8(f2fma8(f2pack8(s[k0], s[k0 + 1]), sl2x2, nmx2), a0, a1);
            f2unpack8(f2fma8(f2pack8(s[k0 + 2], s[k0 + 3]), sl2x2, nmx2), a2, a3);
            a0 = ex2(a0); a1 = ex2(a1); a2 = ex2(a2); a3 = ex2(a3);
            sum2[0] = f2add8(sum2[0], f2pack8(a0, a1));
            sum2[1] = f2add8(sum2[1], f2pack8(a2, a3));
            p[jj] = pack_e4m3x4(a0, a1, a2, a3);
          }
          tmem_st_x8_nowait(tS + 16 * half + 8 * c8, p);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bars->p_full[w][half]);
      }
      {
        float s0, s1, s2, s3;
        f2unpack8(sum2[0], s0, s1);
        f2unpack8(sum2[1], s2, s3);
        lsum += (s0 + s1) + (s2 + s3);
      }
    }
    if (ok) ok = __all_sync(0xffffffffu, wait8(&bars->o_full, 0, abort));
    if (ok) {
      tc_fence_after();
      const int grow = r0 + kRows * w + row;
      const bool store = grow < q_end && VDN_IN_BOUNDS(grow >= 0 && grow < l.L(), &g_fp8_status);
      const float inv = v_scale / lsum;
      const long long base = (((long long)b * l.L() + grow) * l.H + h) * kD;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t o[32];
        tmem_ld_x32(tO + c0, o);
        if (store) {
          uint4* dst = reinterpret_cast<uint4*>(out + base + c0);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16(__uint_as_float(o[8 * i]) * inv, __uint_as_float(o[8 * i + 1]) * inv),
                                pack_bf16(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv),
                                pack_bf16(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv),
                                pack_bf16(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv));
        }
      }
      if (store && lse)
        lse[((long long)b * l.L() + grow) * l.H + h] = (m - kPShift + log2f(lsum)) * 0.6931471805599453f;
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// 4-D map over a [B, rows, H, 128] e4m3 tensor: dims (128, H, rows, B), box
// (128, 1, 128, 1) = one 128-byte swizzle atom per row; rows past the end read as zero.
bool make_map_e4m3(CUtensorMap* m, const void* base, int H, long long rows, int B) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[4] = {(cuuint64_t)kD, (cuuint64_t)H, (cuuint64_t)rows, (cuuint64_t)B};
  cuuint64_t strides[3] = {(cuuint64_t)kD, (cuuint64_t)H * kD, (cuuint64_t)rows * H * kD};
  cuuint32_t box[4] = {(cuuint32_t)kD, 1, (cuuint32_t)kRows, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box,
                  estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_window_fp8(const Layout& l, const void* q, const void* k, const void* v,
                              const void* kt, const void* vt, float qk_scale, float v_scale,
                              void* o, float* lse, cudaStream_t st) {
  if (l.d != kD || l.A != 0 || l.ctx != 0) return cudaErrorInvalidValue;
  CUtensorMap mq, mk, mv, mkt, mvt;
  const long long L = l.L();
  if (!make_map_e4m3(&mq, q, l.H, L, l.B) || !make_map_e4m3(&mk, k, l.H, L, l.B) ||
      !make_map_e4m3(&mv, v, l.H, L, l.B))
    return cudaErrorInvalidValue;
  mkt = mk;  // never read without text tiles
  mvt = mv;
  if (l.T > 0 && (!make_map_e4m3(&mkt, kt, l.H, l.T, l.B) || !make_map_e4m3(&mvt, vt, l.H, l.T, l.B)))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(window_fp8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       kSmemBytes);
  if (e != cudaSuccess) return e;
  dim3 grid(tiles_per_head(l, 2 * kRows), l.H, l.B);
  if (grid.x == 0) return cudaSuccess;
  window_fp8_kernel<<<grid, kThreads, kSmemBytes, st>>>(mq, mk, mv, mkt, mvt, l, qk_scale, v_scale,
                                                       static_cast<__nv_bfloat16*>(o), lse);
  return cudaGetLastError();
}

}  // namespace vdn
