// Bidirectional block attention over the low-bit cache on the 5th-generation
// tensor cores (tcgen05 + tensor memory), for query groups of 128 rows
// (query heads per kv-head x block = 128).  Attention is computed "directly
// from low-bit KV" (MaskAhead / Q-MaskAhead abstract) at every denoising step.
//
// CTA = (unit, token split), one CTA per SM, 13 warps:
//   warps 0-3   softmax: thread r owns query row r (= TMEM lane r); loads Q
//               into TMEM, runs the online softmax on S, writes P (fp16) back
//               into TMEM, rescales O when the running max grows by > 2^8,
//               and writes the output / split partial at the end
//   warps 4-7   K producer: dequantizes 128-token K tiles into shared memory
//               (channel rows, tokens contiguous: MN-major, 128-byte swizzle)
//   warps 8-11  V producer: dequantizes V tiles (token rows, channels
//               contiguous: MN-major, 128-byte swizzle)
//   warp 12     allocates TMEM; one lane issues the MMAs:
//               S_j = Q K_j^T (A = Q from TMEM), O += P_j V_j (A = P from TMEM)
// Tensor memory (512 columns x 128 lanes x 32 bit): O [0,128), S0 [128,256),
// S1 [256,384), Q [384,448); P_j (fp16 pairs) overwrites the first 64
// columns of S_(j mod 2) once the softmax has read them.
// Hand-offs are mbarriers; MMA completion arrives through tcgen05.commit.
// Every wait is bounded (about one second of %globaltimer): on expiry the
// CTA raises DKV_FLAG_TIMEOUT, all roles leave their loops, the MMA lane waits
// (bounded) for its own MMAs, and TMEM is released before returning.
#include "dequant.cuh"
#include "dkv_internal.cuh"

namespace dkv {
namespace {

constexpr int TT = kTcTile;              // tokens per tile
constexpr int kWarps = 13;
constexpr int kThreads = kWarps * 32;
constexpr int kMmaWarp = 12;
constexpr uint32_t kTileBytes = 128 * 128 * 2;
constexpr uint32_t kColO = 0, kColS0 = 128, kColS1 = 256, kColQ = 384, kTmemCols = 512;
constexpr uint64_t kTimeoutNs = 1000000000ull;

// instruction descriptor: D f32, A f16 (K-major), B f16 (MN-major), M = N = 128
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | (1u << 16) |
                            ((128u >> 3) << 17) | ((128u >> 4) << 24);

struct Smem {
  // offsets into the 1024-byte aligned dynamic shared memory
  static constexpr uint32_t kK0 = 0, kK1 = kTileBytes, kV0 = 2 * kTileBytes, kV1 = 3 * kTileBytes;
  static constexpr uint32_t kBar = 4 * kTileBytes;  // 16 mbarriers
  static constexpr uint32_t kMisc = kBar + 16 * 8;  // tmem base, abort flag
  static constexpr uint32_t kBytes = kMisc + 16;
};
enum Bar { KFULL = 0, KEMPTY = 2, VFULL = 4, VEMPTY = 6, SFULL = 8, PFULL = 10, QREADY = 12, DONE = 13 };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of `parity`; false on abort or after ~1 s (then the
// CTA-wide abort flag and the sticky timeout flag are set).
__device__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                          uint32_t* status) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 63u) == 63u) {
      if (*abort_flag) return false;
      const uint64_t now = globaltimer();
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kTimeoutNs) {
        *abort_flag = 1;
        atomicOr(status, uint32_t(DKV_FLAG_TIMEOUT));
        return false;
      }
    }
  }
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// shared-memory matrix descriptor, 128-byte swizzle (sm100 descriptor version 1)
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = uint64_t((addr >> 4) & 0x3FFFu);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(2) << 61;
  return d;
}

// D[tmem] (+)= A[tmem] * B[smem]^T
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %3, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %4, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(accumulate), "r"(kIdesc)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}

// byte offset of the 16-byte chunk holding tokens t..t+7 (t % 8 == 0) of
// channel c in a K tile: MN-major over tokens, 1024-byte atoms of 8 channel
// rows x 64 tokens; atom (c/8, t/64) at ((c/8)*2 + t/64) * 1024
__device__ __forceinline__ uint32_t kt_off(int c, int t) {
  return uint32_t(((c >> 3) * 2 + (t >> 6)) * 1024 + (c & 7) * 128 +
                  ((((t & 63) >> 3) ^ (c & 7)) << 4));
}

// chunk of channels c..c+7 (c % 8 == 0) of token t in a V tile: MN-major over
// channels, atom (t/8, c/64) at ((t/8)*2 + c/64) * 1024
__device__ __forceinline__ uint32_t vt_off(int t, int c) {
  return uint32_t(((t >> 3) * 2 + (c >> 6)) * 1024 + (t & 7) * 128 +
                  ((((c & 63) >> 3) ^ (t & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  return h2u(__floats2half2_rn(a, b));
}

// ------------------------------------------------------------------ producers

// K tile: thread `c` (channel) fills tokens [32q, 32q+32) of the tile for q = 0..3
template <int KB>
__device__ void fill_k_tile(const AttnArgs& a, int u, int64_t tile_start, uint8_t* kt, int c) {
  const CacheView& cv = a.c;
  const int d = kHeadDim;
#pragma unroll 1
  for (int q = 0; q < 4; ++q) {
    const int64_t pos0 = tile_start + 32 * q;
    uint4 out[4];
    const uint16_t* raw = nullptr;
    bool codes = false;
    if (pos0 < a.Lq) {
      if constexpr (KB < 16) codes = true;
      else raw = cv.k_raw + (size_t(u) * cv.cap + pos0) * d;
    } else if (pos0 < a.L) {
      raw = cv.k_tail + (size_t(u) * cv.GK + (pos0 - a.Lq)) * d;
    } else if (pos0 < a.n_tok) {
      raw = a.k_act + (size_t(u) * cv.blk + (pos0 - a.L)) * d;
    }
    int64_t j = 0;
    if (codes) {
      if constexpr (KB < 16) {
        j = pos0 / cv.GK;
        const int o = int(pos0 % cv.GK);
        const size_t base = ((size_t(u) * cv.nG + j) * d + c) * cv.kw + size_t(o) * KB / 32;
        const __half2 sz = cv.k_sz[(size_t(u) * cv.nG + j) * d + c];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        if constexpr (KB == 4) {
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(cv.k_codes + base));
          out[0] = dequant4x8(w.x, s2, z2);
          out[1] = dequant4x8(w.y, s2, z2);
          out[2] = dequant4x8(w.z, s2, z2);
          out[3] = dequant4x8(w.w, s2, z2);
        } else {
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(cv.k_codes + base));
          dequant2x16(w.x, s2, z2, out[0], out[1]);
          dequant2x16(w.y, s2, z2, out[2], out[3]);
        }
      }
    } else if (raw) {
      uint32_t h[16];
#pragma unroll
      for (int t = 0; t < 16; ++t) {
        const float lo = __uint_as_float(uint32_t(__ldg(raw + size_t(2 * t) * d + c)) << 16);
        const float hi = __uint_as_float(uint32_t(__ldg(raw + size_t(2 * t + 1) * d + c)) << 16);
        h[t] = pack_h2(lo, hi);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = make_uint4(h[4 * i], h[4 * i + 1], h[4 * i + 2], h[4 * i + 3]);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(kt + kt_off(c, 32 * q + 8 * i)) = out[i];
    if constexpr (KB < 16) {
      if (codes) {
        // protected rows of this chunk: their bf16 K from the side table
        const int g0 = cv.prot_gstart[size_t(u) * (cv.nG + 1) + j];
        const int g1 = cv.prot_gstart[size_t(u) * (cv.nG + 1) + j + 1];
        for (int e = g0; e < g1; ++e) {
          const int pos = cv.prot_pos[size_t(u) * cv.P + e];
          if (pos >= pos0 && pos < pos0 + 32) {
            const int t = 32 * q + int(pos - pos0);
            __half* dst = reinterpret_cast<__half*>(kt + kt_off(c, t & ~7)) + (t & 7);
            *dst = bf16_to_half(cv.prot_k[(size_t(u) * cv.P + e) * d + c]);
          }
        }
      }
    }
  }
}

// V tile: thread `t` (token of the tile) fills its 128 channels
template <int VB>
__device__ void fill_v_tile(const AttnArgs& a, int u, int64_t tile_start, uint8_t* vt, int t) {
  const CacheView& cv = a.c;
  const int d = kHeadDim;
  const int64_t pos = tile_start + t;
  const uint16_t* raw = nullptr;
  bool codes = false;
  if (pos < a.L) {
    if constexpr (VB < 16) codes = true;
    else raw = cv.v_raw + (size_t(u) * cv.cap + pos) * d;
  } else if (pos < a.n_tok) {
    raw = a.v_act + (size_t(u) * cv.blk + (pos - a.L)) * d;
  }
#pragma unroll 1
  for (int qq = 0; qq < 4; ++qq) {
    uint4 out[4];
    if (codes) {
      if constexpr (VB < 16) {
        const size_t tok = size_t(u) * cv.cap + pos;
        const __half2 sz = cv.v_sz[tok * cv.vgroups + (qq * 32) / cv.GV];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        if constexpr (VB == 4) {
          const uint4 w = __ldg(reinterpret_cast<const uint4*>(cv.v_codes + tok * cv.vw + qq * 4));
          out[0] = dequant4x8(w.x, s2, z2);
          out[1] = dequant4x8(w.y, s2, z2);
          out[2] = dequant4x8(w.z, s2, z2);
          out[3] = dequant4x8(w.w, s2, z2);
        } else {
          const uint2 w = __ldg(reinterpret_cast<const uint2*>(cv.v_codes + tok * cv.vw + qq * 2));
          dequant2x16(w.x, s2, z2, out[0], out[1]);
          dequant2x16(w.y, s2, z2, out[2], out[3]);
        }
      }
    } else if (raw) {
#pragma unroll
      for (int i = 0; i < 4; ++i)
        out[i] = bf16x8_to_f16x8(__ldg(reinterpret_cast<const uint4*>(raw + qq * 32 + 8 * i)));
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) out[i] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
      *reinterpret_cast<uint4*>(vt + vt_off(t, 32 * qq + 8 * i)) = out[i];
  }
}

// ------------------------------------------------------------------ kernel

template <int KB, int VB>
__global__ void __launch_bounds__(kThreads, 1) attn_tc_kernel(AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~uintptr_t(1023));
  const uint32_t sm_base = smem_u32(sm);
  const uint32_t bar0 = sm_base + Smem::kBar;
  auto bar = [&](int i) { return bar0 + 8u * uint32_t(i); };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + Smem::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + Smem::kMisc + 4);

  const CacheView& cv = a.c;
  const int u = blockIdx.x / a.nsplit;
  const int sp = blockIdx.x % a.nsplit;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n_tiles = (a.n_tok + TT - 1) / TT;
  const int64_t t_begin = int64_t(sp) * a.tiles_per_split;
  const int64_t t_end = t_begin + a.tiles_per_split < n_tiles ? t_begin + a.tiles_per_split : n_tiles;
  const int nt = int(t_end - t_begin);

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(KFULL + b), 128);
      mbar_init(bar(KEMPTY + b), 1);
      mbar_init(bar(VFULL + b), 128);
      mbar_init(bar(VEMPTY + b), 1);
      mbar_init(bar(SFULL + b), 1);
      mbar_init(bar(PFULL + b), 128);
    }
    mbar_init(bar(QREADY), 128);
    mbar_init(bar(DONE), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp < 4) {
    // ------------------------------------------------------------ softmax
    const int r = threadIdx.x;  // query row = TMEM lane
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    {
      const uint4* qrow = reinterpret_cast<const uint4*>(a.q + (size_t(u) * cv.rows + r) * kHeadDim);
      uint32_t qv[32];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 y = bf16x8_to_f16x8(__ldg(qrow + h * 8 + i));
          qv[4 * i + 0] = y.x;
          qv[4 * i + 1] = y.y;
          qv[4 * i + 2] = y.z;
          qv[4 * i + 3] = y.w;
        }
        tmem_st32(lane_base + kColQ + 32 * h, qv);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(QREADY));
    }
    float m_used = -__int_as_float(0x7f800000);  // reference max (log2 units)
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt && ok; ++j) {
      const int b = j & 1;
      const uint32_t s_col = b ? kColS1 : kColS0;
      // tcgen05.ld/st are warp-collective: every branch around them is warp-uniform
      if (!__all_sync(0xffffffffu, mbar_wait(bar(SFULL + b), (j >> 1) & 1, abort_flag, cv.status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      const int64_t tile_start = (t_begin + j) * TT;
      const int valid = a.n_tok - tile_start < TT ? int(a.n_tok - tile_start) : TT;
      // pass 1: row max of this tile
      float mx = -__int_as_float(0x7f800000);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t s[32];
        tmem_ld32(lane_base + s_col + 32 * ch, s);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float x = 32 * ch + i < valid ? __uint_as_float(s[i]) * a.scale_log2
                                              : -__int_as_float(0x7f800000);
          mx = fmaxf(mx, x);
        }
      }
      // lazy rescale: keep the reference max unless the new one exceeds it by
      // 8 (P <= 2^8); decided per warp, rows whose max did not grow get alpha 1
      if (__any_sync(0xffffffffu, mx > m_used + 8.f)) {
        const float m_new = fmaxf(m_used, mx);
        const float alpha = fast_exp2(m_used - m_new);  // 0 on the first tile
        if (j > 0) {
          // O must not be in use by PV(j-1)
          const int pb = (j - 1) & 1;
          if (!__all_sync(0xffffffffu, mbar_wait(bar(VEMPTY + pb), ((j - 1) >> 1) & 1,
                                                 abort_flag, cv.status))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int ch = 0; ch < 4; ++ch) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + 32 * ch, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(lane_base + kColO + 32 * ch, o);
          }
        }
        l *= alpha;
        m_used = m_new;
      }
      // pass 2: P = 2^(x - m_used) as fp16 into the first 64 columns of S_b
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t s[32];
        tmem_ld32(lane_base + s_col + 32 * ch, s);
        tmem_ld_wait();
        uint32_t p[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const int c0 = 32 * ch + 2 * i;
          const float x0 = c0 < valid ? __uint_as_float(s[2 * i]) * a.scale_log2 - m_used
                                      : -__int_as_float(0x7f800000);
          const float x1 = c0 + 1 < valid ? __uint_as_float(s[2 * i + 1]) * a.scale_log2 - m_used
                                          : -__int_as_float(0x7f800000);
          const float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          l += p0 + p1;
          p[i] = pack_h2(p0, p1);
        }
        tmem_st16(lane_base + s_col + 16 * ch, p);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(PFULL + b));
    }
    // epilogue: wait for the last PV, then read O
    if (ok && nt > 0) {
      const int jl = nt - 1;
      ok = __all_sync(0xffffffffu,
                      mbar_wait(bar(VEMPTY + (jl & 1)), (jl >> 1) & 1, abort_flag, cv.status));
    }
    if (ok) {
      tc_fence_after();
      const float inv = 1.f / l;
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t o[32];
        tmem_ld32(lane_base + kColO + 32 * ch, o);
        tmem_ld_wait();
        if (a.nsplit == 1) {
          uint4* dst = reinterpret_cast<uint4*>(a.out + (size_t(u) * cv.rows + r) * kHeadDim + 32 * ch);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint32_t w[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[8 * i + 2 * k]) * inv,
                                                             __uint_as_float(o[8 * i + 2 * k + 1]) * inv);
              w[k] = *reinterpret_cast<const uint32_t*>(&v);
            }
            dst[i] = make_uint4(w[0], w[1], w[2], w[3]);
          }
        } else {
          float4* dst = reinterpret_cast<float4*>(
              a.part_o + ((size_t(u) * a.nsplit + sp) * cv.rows + r) * kHeadDim + 32 * ch);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            dst[i] = make_float4(__uint_as_float(o[4 * i]), __uint_as_float(o[4 * i + 1]),
                                 __uint_as_float(o[4 * i + 2]), __uint_as_float(o[4 * i + 3]));
        }
      }
      if (a.nsplit > 1) a.part_ml[(size_t(u) * a.nsplit + sp) * cv.rows + r] = make_float2(m_used, l);
    }
  } else if (warp < 8) {
    // ------------------------------------------------------------ K producer
    const int c = threadIdx.x - 128;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!mbar_wait(bar(KEMPTY + b), ((j >> 1) & 1) ^ 1, abort_flag, cv.status)) break;
      fill_k_tile<KB>(a, u, (t_begin + j) * TT, sm + (b ? Smem::kK1 : Smem::kK0), c);
      fence_async_smem();
      mbar_arrive(bar(KFULL + b));
    }
  } else if (warp < 12) {
    // ------------------------------------------------------------ V producer
    const int t = threadIdx.x - 256;
    for (int j = 0; j < nt; ++j) {
      const int b = j & 1;
      if (!mbar_wait(bar(VEMPTY + b), ((j >> 1) & 1) ^ 1, abort_flag, cv.status)) break;
      fill_v_tile<VB>(a, u, (t_begin + j) * TT, sm + (b ? Smem::kV1 : Smem::kV0), t);
      fence_async_smem();
      mbar_arrive(bar(VFULL + b));
    }
  } else if (lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = mbar_wait(bar(QREADY), 0, abort_flag, cv.status);
    tc_fence_after();
    auto issue_pv = [&](int i) -> bool {
      const int bb = i & 1;
      if (!mbar_wait(bar(PFULL + bb), (i >> 1) & 1, abort_flag, cv.status)) return false;
      if (!mbar_wait(bar(VFULL + bb), (i >> 1) & 1, abort_flag, cv.status)) return false;
      tc_fence_after();
      const uint32_t vbase = sm_base + (bb ? Smem::kV1 : Smem::kV0);
      const uint32_t p_col = bb ? kColS1 : kColS0;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tmem + kColO, tmem + p_col + 8 * kk, sdesc_sw128(vbase + 4096 * kk, 1024, 2048),
               (i > 0 || kk > 0) ? 1u : 0u);
      mma_commit(bar(VEMPTY + bb));
      return true;
    };
    for (int j = 0; j < nt && ok; ++j) {
      const int b = j & 1;
      if (!mbar_wait(bar(KFULL + b), (j >> 1) & 1, abort_flag, cv.status)) { ok = false; break; }
      tc_fence_after();
      const uint32_t kbase = sm_base + (b ? Smem::kK1 : Smem::kK0);
      const uint32_t s_col = b ? kColS1 : kColS0;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ts(tmem + s_col, tmem + kColQ + 8 * kk, sdesc_sw128(kbase + 4096 * kk, 1024, 2048),
               kk > 0 ? 1u : 0u);
      mma_commit(bar(KEMPTY + b));
      mma_commit(bar(SFULL + b));
      if (j > 0 && !issue_pv(j - 1)) { ok = false; break; }
    }
    if (ok && nt > 0) ok = issue_pv(nt - 1);
    // drain: every MMA issued above completes before TMEM is released
    mma_commit(bar(DONE));
    mbar_wait(bar(DONE), 0, abort_flag, cv.status);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

template <int KB, int VB>
cudaError_t launch_kv(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = Smem::kBytes + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<KB, VB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  attn_tc_kernel<KB, VB><<<unsigned(a.c.U) * unsigned(a.nsplit), kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int KB>
cudaError_t launch_k(const AttnArgs& a, cudaStream_t s) {
  switch (a.c.vb) {
    case 2: return launch_kv<KB, 2>(a, s);
    case 4: return launch_kv<KB, 4>(a, s);
    default: return launch_kv<KB, 16>(a, s);
  }
}

}  // namespace

bool tc_supported(const CacheView& c) { return c.rows == 128 && c.d == kHeadDim; }

cudaError_t launch_attention_tc(const AttnArgs& a, cudaStream_t s) {
  if (!tc_supported(a.c)) return cudaErrorNotSupported;
  switch (a.c.kb) {
    case 2: return launch_k<2>(a, s);
    case 4: return launch_k<4>(a, s);
    default: return launch_k<16>(a, s);
  }
}

}  // namespace dkv
