// Bidirectional block attention over the low-bit cache, warp-level mma.sync
// variant.  Block-diffusion decoding reads the whole committed cache at each
// denoising step, and Q-MaskAhead runs that attention on the low-bit cache
// itself (MaskAhead / Q-MaskAhead abstract).
//
// CTA = (unit, token split).  Each warp owns 16 query rows of the unit (rows =
// query heads of the kv-head x block tokens, contiguous in q and out).  Per
// 64-token tile all threads dequantize K into a channel-major fp16 tile and V
// into a token-major fp16 tile in shared memory (protected K rows patched
// from the side table, tail / active-block tokens converted from bf16), then
// each warp runs S = Q K^T, an online softmax in the log2 domain, and
// O += P V with m16n8k16 fp16 MMAs and fp32 accumulators.  Split partials
// (the split's O divided by its row sum in fp16, its running max and row sum)
// are merged by combine_kernel.
#include "dequant.cuh"
#include "dkv_internal.cuh"

namespace dkv {
namespace {

constexpr int T = kMmaTile;      // tokens per tile
constexpr int KT_LD = T + 8;     // K tile: [128 channels][T + 8] halves
constexpr int VT_LD = 128 + 8;   // V tile: [T tokens][136] halves

enum SegKind { SEG_CODES = 0, SEG_RAW = 1, SEG_ZERO = 2 };

__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(a));
}

__device__ __forceinline__ uint32_t bf16x2_to_h2(uint32_t w) {
  return h2u(__floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u)));
}

// Channels [32 q, 32 q + 32) of committed token j's V row (quantized V),
// dequantized to fp16 into dst[0..3]; sink positions take their bf16 row.
template <int VB>
__device__ __forceinline__ void v_quarter(const CacheView& c, int u, int64_t j, int q, uint4* dst) {
  const int d = kHeadDim;
  if (j < c.sink && DKV_IN_BOUNDS(c.sink <= c.cap, c.status)) {
    const uint4* src = reinterpret_cast<const uint4*>(
        c.v_sink + (size_t(u) * c.sink + size_t(j)) * d + q * 32);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = bf16x8_to_f16x8(src[k]);
    return;
  }
  const size_t tok = size_t(u) * c.cap + size_t(j);
  const __half2 sz = c.v_sz[tok * c.vgroups + (q * 32) / c.GV];
  const __half2 s2 = __half2half2(__low2half(sz));
  const __half2 z2 = __half2half2(__high2half(sz));
  if constexpr (VB == 3) {
    const uint32_t* vc = c.v_codes + tok * c.vw + q * 3;  // 3 words, 4-byte aligned
    uint4 o4[4];
    dequant3x32(vc[0], vc[1], vc[2], s2, z2, o4);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = o4[k];
  } else if constexpr (VB == 4) {
    const uint4 w = *reinterpret_cast<const uint4*>(c.v_codes + tok * c.vw + q * 4);
    dst[0] = dequant4x8(w.x, s2, z2);
    dst[1] = dequant4x8(w.y, s2, z2);
    dst[2] = dequant4x8(w.z, s2, z2);
    dst[3] = dequant4x8(w.w, s2, z2);
  } else {
    const uint2 w = *reinterpret_cast<const uint2*>(c.v_codes + tok * c.vw + q * 2);
    dequant2x16(w.x, s2, z2, dst[0], dst[1]);
    dequant2x16(w.y, s2, z2, dst[2], dst[3]);
  }
}

// Fill K tile columns [32*ch, 32*ch + 32) (one 32-token chunk at absolute
// position pos0) and V tile rows of the same chunk.
template <int KB, int VB>
__device__ __forceinline__ void fill_chunk(const AttnArgs& a, const UnitLen ul, int u, int64_t pos0, int ch,
                                           __half* Kt, __half* Vt, int tid, int nthr) {
  const CacheView& c = a.c;
  const int d = kHeadDim;
  // ---- K
  int kind;
  const uint16_t* kraw = nullptr;  // token-major bf16 rows (stride d)
  if (pos0 < ul.Lq) {
    if constexpr (KB < 16) {
      kind = SEG_CODES;
    } else {
      kind = SEG_RAW;
      kraw = c.k_raw + (size_t(u) * c.cap + pos0) * d;
    }
  } else if (pos0 < ul.L) {
    kind = SEG_RAW;
    kraw = c.k_tail + (size_t(u) * c.GK + (pos0 - ul.Lq)) * d;
  } else if (pos0 < ul.n_tok) {
    kind = SEG_RAW;
    kraw = a.k_act + (size_t(u) * c.blk + (pos0 - ul.L)) * d;
  } else {
    kind = SEG_ZERO;
  }
  // bounds-checking build: the chunk lies inside the segment it reads (a
  // chunk that does not is filled with zeros)
  if (!DKV_IN_BOUNDS(pos0 >= 0 && (kind == SEG_ZERO ||
                                   (kind == SEG_CODES ? pos0 + kChunk <= ul.Lq && ul.Lq <= c.cap &&
                                                            ul.Lq % c.GK == 0
                                    : pos0 < ul.Lq    ? pos0 + kChunk <= c.cap
                                    : pos0 < ul.L     ? pos0 + kChunk - ul.Lq <= c.GK
                                                     : pos0 + kChunk - ul.L <= c.blk)),
                     c.status))
    kind = SEG_ZERO;
  if (kind == SEG_CODES) {
    if constexpr (KB < 16) {
      const int64_t j = pos0 / c.GK;
      const int o = int(pos0 % c.GK);
      int g0 = c.prot_gstart[size_t(u) * (c.nG + 1) + j];
      int g1 = c.prot_gstart[size_t(u) * (c.nG + 1) + j + 1];
      if (!DKV_IN_BOUNDS(g0 >= 0 && g0 <= g1 && g1 <= c.P, c.status)) g0 = g1 = 0;
      for (int cc = tid; cc < d; cc += nthr) {
        const size_t base = ((size_t(u) * c.nG + j) * d + cc) * c.kw + size_t(o) * KB / 32;
        const __half2 sz = c.k_sz[(size_t(u) * c.nG + j) * d + cc];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        uint4* dst = reinterpret_cast<uint4*>(Kt + cc * KT_LD + ch * 32);
        if constexpr (KB == 3) {
          const uint32_t* kc = c.k_codes + base;  // 3 words, 4-byte aligned
          uint4 o4[4];
          dequant3x32(kc[0], kc[1], kc[2], s2, z2, o4);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = o4[k];
        } else if constexpr (KB == 4) {
          const uint4 w = *reinterpret_cast<const uint4*>(c.k_codes + base);
          dst[0] = dequant4x8(w.x, s2, z2);
          dst[1] = dequant4x8(w.y, s2, z2);
          dst[2] = dequant4x8(w.z, s2, z2);
          dst[3] = dequant4x8(w.w, s2, z2);
        } else {
          const uint2 w = *reinterpret_cast<const uint2*>(c.k_codes + base);
          dequant2x16(w.x, s2, z2, dst[0], dst[1]);
          dequant2x16(w.y, s2, z2, dst[2], dst[3]);
        }
        // protected rows of this chunk: bf16 values from the side table
        for (int e = g0; e < g1; ++e) {
          const int pos = c.prot_pos[size_t(u) * c.P + e];
          if (pos >= pos0 && pos < pos0 + kChunk)
            Kt[cc * KT_LD + ch * 32 + (pos - pos0)] =
                bf16_to_half(c.prot_k[(size_t(u) * c.P + e) * d + cc]);
        }
      }
    }
  } else if (kind == SEG_RAW) {
    // item = (octet o, token t), t fastest: lanes write consecutive halves
    for (int it = tid; it < kChunk * (d / 8); it += nthr) {
      const int t = it % kChunk, o = it / kChunk;
      const uint4 x = *reinterpret_cast<const uint4*>(kraw + size_t(t) * d + o * 8);
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 h = u2h(bf16x2_to_h2(w[i]));
        Kt[(o * 8 + 2 * i) * KT_LD + ch * 32 + t] = __low2half(h);
        Kt[(o * 8 + 2 * i + 1) * KT_LD + ch * 32 + t] = __high2half(h);
      }
    }
  } else {
    for (int it = tid; it < d * 4; it += nthr) {
      const int cc = it / 4, q = it % 4;
      *reinterpret_cast<uint4*>(Kt + cc * KT_LD + ch * 32 + q * 8) = make_uint4(0, 0, 0, 0);
    }
  }

  // ---- V
  const uint16_t* vraw = nullptr;
  if (pos0 < ul.L) {
    if constexpr (VB < 16) {
      kind = SEG_CODES;
    } else {
      kind = SEG_RAW;
      vraw = c.v_raw + (size_t(u) * c.cap + pos0) * d;
    }
  } else if (pos0 < ul.n_tok) {
    kind = SEG_RAW;
    vraw = a.v_act + (size_t(u) * c.blk + (pos0 - ul.L)) * d;
  } else {
    kind = SEG_ZERO;
  }
  if (!DKV_IN_BOUNDS(kind == SEG_ZERO ||
                         (pos0 < ul.L ? pos0 + kChunk <= ul.L && ul.L <= c.cap
                                     : pos0 + kChunk - ul.L <= c.blk),
                     c.status))
    kind = SEG_ZERO;
  if (kind == SEG_CODES) {
    if constexpr (VB < 16) {
      // item = (token t, quarter q of 32 channels)
      for (int it = tid; it < kChunk * 4; it += nthr) {
        const int t = it / 4, q = it % 4;
        v_quarter<VB>(c, u, pos0 + t, q, reinterpret_cast<uint4*>(Vt + (ch * 32 + t) * VT_LD + q * 32));
      }
    }
  } else if (kind == SEG_RAW) {
    for (int it = tid; it < kChunk * (d / 8); it += nthr) {
      const int t = it / (d / 8), o = it % (d / 8);
      const uint4 x = *reinterpret_cast<const uint4*>(vraw + size_t(t) * d + o * 8);
      *reinterpret_cast<uint4*>(Vt + (ch * 32 + t) * VT_LD + o * 8) = bf16x8_to_f16x8(x);
    }
  } else {
    for (int it = tid; it < kChunk * (d / 8); it += nthr) {
      const int t = it / (d / 8), o = it % (d / 8);
      *reinterpret_cast<uint4*>(Vt + (ch * 32 + t) * VT_LD + o * 8) = make_uint4(0, 0, 0, 0);
    }
  }
}


// Gather mode: the 32 slots pos0 .. pos0 + 31 of the selected-token sequence
// into K tile columns [32*ch, 32*ch + 32) and V tile rows.  Slot i < ul.L is
// committed token sel[u][i] (quantized, protected, tail or bf16 rows as
// stored), then come the active block's rows, then zeros.  sj: 32 ints of
// shared memory for this chunk.
template <int KB, int VB>
__device__ __forceinline__ void fill_chunk_gather(const AttnArgs& a, const UnitLen ul, int u,
                                                  int64_t pos0, int ch, __half* Kt, __half* Vt,
                                                  int tid, int nthr, int* sj) {
  const CacheView& c = a.c;
  const int d = kHeadDim;
  constexpr int kZero = -0x7fffffff;
  const int32_t Lc = a.lens.len[u / c.Hkv];                  // committed tokens
  const int32_t Lq = KB < 16 ? (Lc / c.GK) * c.GK : Lc;       // ... in complete K groups
  if (tid < kChunk) {
    // slot -> source: >= 0 committed token, -1 - r active-block row r, kZero none
    const int64_t i = pos0 + tid;
    int src = kZero;
    if (i < ul.L) {
      src = a.sel[size_t(u) * a.sel_ld + size_t(i)];
      if (!DKV_IN_BOUNDS(src >= 0 && src < Lc, c.status)) src = kZero;
    } else if (i < ul.n_tok) {
      src = -1 - int(i - ul.L);
    }
    sj[tid] = src;
  }
  __syncthreads();
  // ---- K: item = (octet o, slot t), t fastest
  for (int it = tid; it < kChunk * (d / 8); it += nthr) {
    const int t = it % kChunk, o = it / kChunk;
    const int src = sj[t];
    const uint16_t* row = nullptr;  // a bf16 row holding this slot's K
    uint32_t h[4] = {0u, 0u, 0u, 0u};
    if (src == kZero) {
    } else if (src < 0) {
      row = a.k_act + (size_t(u) * c.blk + size_t(-1 - src)) * d;
    } else if (KB == 16) {
      row = c.k_raw + (size_t(u) * c.cap + size_t(src)) * d;
    } else if (src >= Lq) {
      row = c.k_tail + (size_t(u) * c.GK + size_t(src - Lq)) * d;
    } else if constexpr (KB < 16) {
      const int g = src / c.GK, jo = src % c.GK;
      // a protected token keeps its bf16 vector in the side table
      const int32_t* gs = c.prot_gstart + size_t(u) * size_t(c.nG + 1) + g;
      int e = -1;
      for (int k = gs[0]; k < gs[1]; ++k)
        if (DKV_IN_BOUNDS(k >= 0 && k < c.P, c.status) && c.prot_pos[size_t(u) * c.P + k] == src) {
          e = k;
          break;
        }
      if (e >= 0) {
        row = c.prot_k + (size_t(u) * c.P + size_t(e)) * d;
      } else {
        const int bit = jo * KB, wd = bit >> 5, off = bit & 31;
#pragma unroll
        for (int ci = 0; ci < 8; ++ci) {
          const int cc = 8 * o + ci;
          const size_t gc = (size_t(u) * c.nG + size_t(g)) * d + cc;
          const uint32_t* wp = c.k_codes + gc * c.kw + wd;
          uint32_t x = wp[0];
          if (off + KB > 32) x = __funnelshift_r(x, wp[1], off);  // a 3-bit code across words
          else x >>= off;
          const __half2 sz = c.k_sz[gc];
          const __half kh =
              __hfma(__ushort2half_rn(uint16_t(x & ((1u << KB) - 1u))), __low2half(sz), __high2half(sz));
          const uint16_t kb16 = *reinterpret_cast<const uint16_t*>(&kh);
          h[ci >> 1] |= uint32_t(kb16) << (16 * (ci & 1));
        }
      }
    }
    if (row) {
      const uint4 x = bf16x8_to_f16x8(*reinterpret_cast<const uint4*>(row + o * 8));
      h[0] = x.x;
      h[1] = x.y;
      h[2] = x.z;
      h[3] = x.w;
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __half2 hh = u2h(h[i]);
      Kt[(o * 8 + 2 * i) * KT_LD + ch * 32 + t] = __low2half(hh);
      Kt[(o * 8 + 2 * i + 1) * KT_LD + ch * 32 + t] = __high2half(hh);
    }
  }
  // ---- V: item = (slot t, quarter q of 32 channels)
  for (int it = tid; it < kChunk * 4; it += nthr) {
    const int t = it / 4, q = it % 4;
    const int src = sj[t];
    uint4* dst = reinterpret_cast<uint4*>(Vt + (ch * 32 + t) * VT_LD + q * 32);
    const uint16_t* row = nullptr;
    if (src == kZero) {
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = make_uint4(0u, 0u, 0u, 0u);
      continue;
    } else if (src < 0) {
      row = a.v_act + (size_t(u) * c.blk + size_t(-1 - src)) * d;
    } else if constexpr (VB == 16) {
      row = c.v_raw + (size_t(u) * c.cap + size_t(src)) * d;
    } else {
      v_quarter<VB>(c, u, src, q, dst);
      continue;
    }
    const uint4* r4 = reinterpret_cast<const uint4*>(row + q * 32);
#pragma unroll
    for (int k = 0; k < 4; ++k) dst[k] = bf16x8_to_f16x8(r4[k]);
  }
}

constexpr int kRowsPerCta = 128;  // 8 warps; a larger query group takes several CTAs

template <int KB, int VB, bool GATHER>
__global__ void __launch_bounds__(256)
attn_mma_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ __align__(16) __half Kt[kHeadDim * KT_LD];
  __shared__ __align__(16) __half Vt[T * VT_LD];
  __shared__ int sj[2][kChunk];  // gather mode: the slots' source tokens
  pdl_wait();
  pdl_trigger();

  const CacheView& c = a.c;
  const int nrb = (c.rows + kRowsPerCta - 1) / kRowsPerCta;
  const int rb = blockIdx.x % nrb;
  const int u = (blockIdx.x / nrb) / a.nsplit;
  const int sp = (blockIdx.x / nrb) % a.nsplit;
  const int tid = threadIdx.x;
  const int nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int r0 = rb * kRowsPerCta + warp * 16 + (lane >> 2);  // rows r0, r0 + 8
  // warps past the last row only help fill the tiles
  const bool active = rb * kRowsPerCta + warp * 16 < c.rows;
  const int cq = 2 * (lane & 3);           // column pair inside an 8-wide n tile
  const UnitLen ul = unit_len(a, u);       // this unit's sequence length

  const int64_t n_tiles = (ul.n_tok + T - 1) / T;
  const int64_t t_begin = int64_t(sp) * a.tiles_per_split;
  const int64_t t_end = t_begin + a.tiles_per_split < n_tiles ? t_begin + a.tiles_per_split : n_tiles;

  // Q fragments (bf16 -> fp16), held for the whole kernel
  uint32_t qa[8][4] = {};
  if (active) {
    const uint16_t* qrow0 = a.q + (size_t(u) * c.rows + r0) * kHeadDim;
    const uint16_t* qrow1 = qrow0 + 8 * kHeadDim;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int col = kk * 16 + cq;
      qa[kk][0] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow0 + col));
      qa[kk][1] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow1 + col));
      qa[kk][2] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow0 + col + 8));
      qa[kk][3] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow1 + col + 8));
    }
  }

  float o[16][4];
#pragma unroll
  for (int i = 0; i < 16; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  float m0 = -__int_as_float(0x7f800000), m1 = m0;  // running max (log2 units)
  float l0 = 0.f, l1 = 0.f;                         // running sums (thread partial)

  // ldmatrix lane addressing
  const int lr = lane & 7, lm = lane >> 3;

  for (int64_t tile = t_begin; tile < t_end; ++tile) {
    const int64_t tile_start = tile * T;
    __syncthreads();
    if constexpr (GATHER) {
      fill_chunk_gather<KB, VB>(a, ul, u, tile_start, 0, Kt, Vt, tid, nthr, sj[0]);
      fill_chunk_gather<KB, VB>(a, ul, u, tile_start + kChunk, 1, Kt, Vt, tid, nthr, sj[1]);
    } else {
      fill_chunk<KB, VB>(a, ul, u, tile_start, 0, Kt, Vt, tid, nthr);
      fill_chunk<KB, VB>(a, ul, u, tile_start + kChunk, 1, Kt, Vt, tid, nthr);
    }
    __syncthreads();
    if (!active) continue;

    // S = Q K^T over this tile's 64 tokens
    float s[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
      for (int n2 = 0; n2 < 4; ++n2) {
        uint32_t b[4];
        const int chn = kk * 16 + lr + 8 * (lm & 1);
        const int tok = 8 * (2 * n2 + (lm >> 1));
        ldsm_x4_t(b, Kt + chn * KT_LD + tok);
        mma16816(s[2 * n2], qa[kk], b[0], b[1]);
        mma16816(s[2 * n2 + 1], qa[kk], b[2], b[3]);
      }
    }

    // scale into log2 units, mask tokens past the end
    float mx0 = -__int_as_float(0x7f800000), mx1 = mx0;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int64_t pos = tile_start + nt * 8 + cq + (i & 1);
        s[nt][i] = pos < ul.n_tok ? s[nt][i] * a.scale_log2 : -__int_as_float(0x7f800000);
      }
      mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
      mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
    }
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float al0 = fast_exp2(m0 - mn0), al1 = fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    l0 *= al0;
    l1 *= al1;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      o[i][0] *= al0;
      o[i][1] *= al0;
      o[i][2] *= al1;
      o[i][3] *= al1;
    }
    uint32_t pa[4][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) {
      const float p0 = fast_exp2(s[nt][0] - mn0), p1 = fast_exp2(s[nt][1] - mn0);
      const float p2 = fast_exp2(s[nt][2] - mn1), p3 = fast_exp2(s[nt][3] - mn1);
      l0 += p0 + p1;
      l1 += p2 + p3;
      const int kk2 = nt >> 1, hi = nt & 1;
      pa[kk2][hi * 2 + 0] = h2u(__floats2half2_rn(p0, p1));
      pa[kk2][hi * 2 + 1] = h2u(__floats2half2_rn(p2, p3));
    }
    // O += P V
#pragma unroll
    for (int kk2 = 0; kk2 < 4; ++kk2) {
#pragma unroll
      for (int n2 = 0; n2 < 8; ++n2) {
        uint32_t b[4];
        const int tok = kk2 * 16 + lr + 8 * (lm & 1);
        const int chn = 8 * (2 * n2 + (lm >> 1));
        ldsm_x4_t(b, Vt + tok * VT_LD + chn);
        mma16816(o[2 * n2], pa[kk2], b[0], b[1]);
        mma16816(o[2 * n2 + 1], pa[kk2], b[2], b[3]);
      }
    }
  }

  if (!active) return;
  l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
  l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
  l1 += __shfl_xor_sync(0xffffffffu, l1, 2);

  if (a.final_out) {
    const float i0 = 1.f / l0, i1 = 1.f / l1;
    uint16_t* out0 = a.out + (size_t(u) * c.rows + r0) * kHeadDim;
    uint16_t* out1 = out0 + 8 * kHeadDim;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      const int col = nd * 8 + cq;
      const __nv_bfloat162 v0 = __floats2bfloat162_rn(o[nd][0] * i0, o[nd][1] * i0);
      const __nv_bfloat162 v1 = __floats2bfloat162_rn(o[nd][2] * i1, o[nd][3] * i1);
      *reinterpret_cast<__nv_bfloat162*>(out0 + col) = v0;
      *reinterpret_cast<__nv_bfloat162*>(out1 + col) = v1;
    }
  } else {
    const size_t prow = (size_t(u) * a.part_stride + a.part_base + sp) * c.rows;
    // the split's output divided by its row sum, in fp16 (an empty split --
    // past the end of a shorter sequence -- has sum 0 and O 0: zeros)
    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
    __half* po0 = a.part_o + (prow + r0) * kHeadDim;
    __half* po1 = po0 + 8 * kHeadDim;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      const int col = nd * 8 + cq;
      *reinterpret_cast<__half2*>(po0 + col) = __floats2half2_rn(o[nd][0] * i0, o[nd][1] * i0);
      *reinterpret_cast<__half2*>(po1 + col) = __floats2half2_rn(o[nd][2] * i1, o[nd][3] * i1);
    }
    if ((lane & 3) == 0) {
      a.part_ml[prow + r0] = make_float2(m0, l0);
      a.part_ml[prow + r0 + 8] = make_float2(m1, l1);
    }
  }
}

// Inverse K-RPBH rotation of one output row held by a warp (lane: channels
// 4 lane .. 4 lane + 3): mix^T across the k blocks, the per-block Hadamard
// (butterflies, then 1/sqrt(b)), the inverse permutation (through `buf`, 128
// floats of this warp's shared memory).  The attention of a rotated-V cache
// sums rotated rows, so its output is the rotated output.
__device__ __forceinline__ void unrotate_row(float (&x)[4], int b, float norm,
                                          const int32_t* __restrict__ perm,
                                          const float* __restrict__ mix, float* buf, int lane) {
  const int k = kHeadDim / b, lb = b / 4;  // lanes per block
  const int i_lane = lane % lb, r = lane / lb;           // this lane's block r
  float y[4] = {0.f, 0.f, 0.f, 0.f};
  for (int rr = 0; rr < k; ++rr) {
    const float m = __ldg(mix + rr * k + r);     // mix[rr][r]: y_r = sum_rr mix[rr][r] w_rr
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] += m * __shfl_sync(0xffffffffu, x[e], rr * lb + i_lane);
  }
#pragma unroll
  for (int h = 1; h <= 2; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e & h) continue;
      const float lo = y[e], hi = y[e + h];
      y[e] = lo + hi;
      y[e + h] = lo - hi;
    }
  }
  for (int h = 4; h < b; h <<= 1) {
    const bool upper = (lane & (h >> 2)) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p = __shfl_xor_sync(0xffffffffu, y[e], h >> 2);
      y[e] = upper ? p - y[e] : y[e] + p;
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) buf[__ldg(perm + 4 * lane + e)] = y[e] * norm;
  __syncwarp();
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = buf[4 * lane + e];
}

constexpr int kCombineWarps = 4;  // rows (one per warp) per combine CTA

// One warp per (unit, row): out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// (rotated back first when V is stored rotated)
__global__ void __launch_bounds__(32 * kCombineWarps) combine_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ float rbuf[kCombineWarps][kHeadDim];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * kCombineWarps + warp;
  const int rows = a.c.rows;
  if (row >= int64_t(a.c.U) * rows) return;
  const int64_t u = row / rows, r = row % rows;
  const size_t base = size_t(u) * a.nsplit * rows + r;  // split s at base + s*rows
  // Splits merged in a fixed order, four at a time with all their loads in
  // flight: a running max M, the sum and O rescaled when it rises.  Empty
  // splits (max -inf, sum 0, O 0) get weight 1 against an equal -inf max
  // instead of 2^(-inf + inf).
  float M = -__int_as_float(0x7f800000);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
#pragma unroll 1
  for (int s0 = 0; s0 < a.nsplit; s0 += 4) {
    const int n = a.nsplit - s0 < 4 ? a.nsplit - s0 : 4;
    float2 ml[4];
    uint2 x[4];  // four fp16 channels of the split's normalised output
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i < n) {
        const size_t ps = base + size_t(s0 + i) * rows;
        ml[i] = a.part_ml[ps];
        x[i] = *reinterpret_cast<const uint2*>(a.part_o + ps * kHeadDim + lane * 4);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      if (i < n) {
        const float Mn = fmaxf(M, ml[i].x);
        const float c = M == Mn ? 1.f : fast_exp2(M - Mn);
        const float wl = (ml[i].x == Mn ? 1.f : fast_exp2(ml[i].x - Mn)) * ml[i].y;
        const float2 o01 = __half22float2(*reinterpret_cast<const __half2*>(&x[i].x));
        const float2 o23 = __half22float2(*reinterpret_cast<const __half2*>(&x[i].y));
        lsum = lsum * c + wl;
        acc.x = acc.x * c + wl * o01.x;
        acc.y = acc.y * c + wl * o01.y;
        acc.z = acc.z * c + wl * o23.x;
        acc.w = acc.w * c + wl * o23.y;
        M = Mn;
      }
    }
  }
  const float inv = 1.f / lsum;
  float x[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
  if (a.c.vrot_b)
    unrotate_row(x, a.c.vrot_b, a.c.vrot_norm, a.c.vrot_perm, a.c.vrot_mix, rbuf[warp], lane);
  const __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(x[2], x[3]);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&lo);
  pk.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(a.out + (size_t(u) * rows + r) * kHeadDim + lane * 4) = pk;
}


// ------------------------------------------------------------ Q-MaskAhead selection

// Contribution of every committed token to the block's attention output
// (MaskAhead / Q-MaskAhead abstract: the block's queries rank the cached
// entries by their expected share of the output, scored on the low-bit
// cache).  Reading: c_j = (sum over the unit's query rows i of p_ij) *
// ||v_hat_j||_2, p_ij the softmax weight of token j for row i in the whole
// call (committed tokens and active block).  The weights come from each row's
// final max and sum, merged here from the split partials of the attention
// pass (a.part_ml).  CTA = (unit, row block of 128 rows, chunk of
// tiles_per_cta 64-token tiles of the committed tokens); it writes its row
// block's share of c_j (p summed over its rows, times the norm); the top-k
// kernel adds the row blocks in order.
template <int KB, int VB>
__global__ void __launch_bounds__(256)
score_kernel(const __grid_constant__ AttnArgs a, float* __restrict__ part, int64_t ld,
             int tiles_per_cta, int nchunk) {
  __shared__ __align__(16) __half Kt[kHeadDim * KT_LD];
  __shared__ __align__(16) __half Vt[T * VT_LD];
  __shared__ float colsum[8][T];
  __shared__ float vnorm[T];
  __shared__ float2 st[kRowsPerCta];  // (final max in log2 units, 1 / final sum) per row
  pdl_wait();
  pdl_trigger();
  const CacheView& c = a.c;
  const int nrb = (c.rows + kRowsPerCta - 1) / kRowsPerCta;
  const int ck = blockIdx.x % nchunk;
  const int rb = (blockIdx.x / nchunk) % nrb;
  const int u = (blockIdx.x / nchunk) / nrb;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int r0 = rb * kRowsPerCta + warp * 16 + (lane >> 2);
  const bool active = rb * kRowsPerCta + warp * 16 < c.rows;
  const int cq = 2 * (lane & 3);
  const UnitLen ul = unit_len(a, u);  // committed tokens only (with_active = 0)
  const int64_t n_tiles = (ul.L + T - 1) / T;
  const int64_t t_begin = int64_t(ck) * tiles_per_cta;
  const int64_t t_end = t_begin + tiles_per_cta < n_tiles ? t_begin + tiles_per_cta : n_tiles;
  if (t_begin >= t_end) return;

  // this row block's final (max, sum) from the split partials
  for (int rr = tid; rr < kRowsPerCta; rr += nthr) {
    const int r = rb * kRowsPerCta + rr;
    float2 v = make_float2(0.f, 0.f);
    if (r < c.rows) {
      const size_t base = size_t(u) * a.part_stride * c.rows + r;
      float M = -__int_as_float(0x7f800000);
      for (int sp = 0; sp < a.nsplit; ++sp) M = fmaxf(M, a.part_ml[base + size_t(a.part_base + sp) * c.rows].x);
      float Ls = 0.f;
      for (int sp = 0; sp < a.nsplit; ++sp) {
        const float2 ml = a.part_ml[base + size_t(a.part_base + sp) * c.rows];
        Ls += fast_exp2(ml.x - M) * ml.y;
      }
      v = make_float2(M, 1.f / Ls);
    }
    st[rr] = v;
  }

  uint32_t qa[8][4] = {};
  if (active) {
    const uint16_t* qrow0 = a.q + (size_t(u) * c.rows + r0) * kHeadDim;
    const uint16_t* qrow1 = qrow0 + 8 * kHeadDim;
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const int col = kk * 16 + cq;
      qa[kk][0] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow0 + col));
      qa[kk][1] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow1 + col));
      qa[kk][2] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow0 + col + 8));
      qa[kk][3] = bf16x2_to_h2(*reinterpret_cast<const uint32_t*>(qrow1 + col + 8));
    }
  }
  const int lr = lane & 7, lm = lane >> 3;

  for (int64_t tile = t_begin; tile < t_end; ++tile) {
    const int64_t tile_start = tile * T;
    __syncthreads();
    fill_chunk<KB, VB>(a, ul, u, tile_start, 0, Kt, Vt, tid, nthr);
    fill_chunk<KB, VB>(a, ul, u, tile_start + kChunk, 1, Kt, Vt, tid, nthr);
    __syncthreads();
    // ||v_hat_t|| of the tile's tokens (zero rows past the end give 0)
    for (int t = tid; t < T; t += nthr) {
      float acc = 0.f;
      const __half2* vr = reinterpret_cast<const __half2*>(Vt + t * VT_LD);
#pragma unroll 8
      for (int i = 0; i < kHeadDim / 2; ++i) {
        const float2 f = __half22float2(vr[i]);
        acc = fmaf(f.x, f.x, acc);
        acc = fmaf(f.y, f.y, acc);
      }
      vnorm[t] = sqrtf(acc);
    }
    float cs[8][2];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) cs[nt][0] = cs[nt][1] = 0.f;
    if (active) {
      float sacc[8][4];
#pragma unroll
      for (int i = 0; i < 8; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
        for (int n2 = 0; n2 < 4; ++n2) {
          uint32_t b[4];
          const int chn = kk * 16 + lr + 8 * (lm & 1);
          const int tok = 8 * (2 * n2 + (lm >> 1));
          ldsm_x4_t(b, Kt + chn * KT_LD + tok);
          mma16816(sacc[2 * n2], qa[kk], b[0], b[1]);
          mma16816(sacc[2 * n2 + 1], qa[kk], b[2], b[3]);
        }
      }
      const int rl0 = warp * 16 + (lane >> 2);  // rows rl0, rl0 + 8 of the block
      const float2 s0 = st[rl0], s1 = st[rl0 + 8];
      const bool ok0 = r0 < c.rows, ok1 = r0 + 8 < c.rows;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int64_t pos = tile_start + nt * 8 + cq + i;
          if (pos < ul.L) {
            const float p0 = ok0 ? fast_exp2(sacc[nt][i] * a.scale_log2 - s0.x) * s0.y : 0.f;
            const float p1 = ok1 ? fast_exp2(sacc[nt][2 + i] * a.scale_log2 - s1.x) * s1.y : 0.f;
            cs[nt][i] = p0 + p1;
          }
        }
      }
      // sum over the warp's 16 rows: lanes that share (lane & 3) share columns
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) cs[nt][i] += __shfl_xor_sync(0xffffffffu, cs[nt][i], o);
    }
    if (lane < 4) {
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        colsum[warp][nt * 8 + cq] = cs[nt][0];
        colsum[warp][nt * 8 + cq + 1] = cs[nt][1];
      }
    }
    __syncthreads();
    for (int t = tid; t < T; t += nthr) {
      const int64_t pos = tile_start + t;
      if (pos >= ul.L) continue;
      float m = 0.f;
      for (int w = 0; w < nthr / 32; ++w) m += colsum[w][t];  // fixed order
      part[(size_t(u) * nrb + rb) * ld + size_t(pos)] = m * vnorm[t];
    }
  }
}

// Inclusive sum over the block's threads (blockDim a multiple of 32, at most
// 1024); `ws` holds 32 ints of shared memory.  Every thread calls it.
__device__ __forceinline__ int block_scan_incl(int x, int* ws) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int v = lane < nw ? ws[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    if (lane < nw) ws[lane] = v;
  }
  __syncthreads();
  return x + (warp > 0 ? ws[warp - 1] : 0);
}

// Per unit: the row blocks' shares summed in order into scores, then the
// k = min(budget, L) largest scores (ties: the lower position) selected by a
// radix select on the fp32 bit patterns (non-negative floats order like
// their bits) and written in increasing position order; -1 after them.
__global__ void __launch_bounds__(1024)
topk_kernel(const __grid_constant__ AttnArgs a, const float* __restrict__ part, int64_t ld,
            int nrb, float* __restrict__ scores, int32_t* __restrict__ sel) {
  __shared__ int hist[256];
  __shared__ int ws[32];
  __shared__ int digit_s, krem_s;
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int L = a.lens.len[u / a.c.Hkv];
  const int k = L < a.budget ? L : a.budget;
  float* sc = scores + size_t(u) * ld;
  for (int j = tid; j < L; j += nthr) {
    float v = 0.f;
    for (int rb = 0; rb < nrb; ++rb) v += part[(size_t(u) * nrb + rb) * ld + j];
    sc[j] = v;
  }
  int32_t* out = sel + size_t(u) * a.sel_ld;
  for (int i = k + tid; i < a.budget; i += nthr) out[i] = -1;
  __syncthreads();
  if (k == L) {  // everything is selected
    for (int j = tid; j < L; j += nthr) out[j] = j;
    return;
  }
  auto key_of = [&](int j) { return __float_as_uint(fmaxf(sc[j], 0.f)); };
  uint32_t prefix = 0u, pmask = 0u;
  if (tid == 0) krem_s = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += nthr) hist[i] = 0;
    __syncthreads();
    for (int j = tid; j < L; j += nthr) {
      const uint32_t key = key_of(j);
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1);
    }
    __syncthreads();
    if (tid == 0) {
      int cum = 0, krem = krem_s, dg = 0;
      for (int b = 255; b >= 0; --b) {
        if (cum + hist[b] >= krem) {
          dg = b;
          break;
        }
        cum += hist[b];
      }
      digit_s = dg;
      krem_s = krem - cum;
    }
    __syncthreads();
    prefix |= uint32_t(digit_s) << shift;
    pmask |= 255u << shift;
  }
  // prefix = the k-th largest key; krem_s of the keys equal to it are taken,
  // the lowest positions first
  const int take_eq = krem_s;
  const int chunk = (L + nthr - 1) / nthr;
  const int j0 = tid * chunk, j1 = j0 + chunk < L ? j0 + chunk : L;
  int gt = 0, eq = 0;
  for (int j = j0; j < j1; ++j) {
    const uint32_t key = key_of(j);
    gt += key > prefix;
    eq += key == prefix;
  }
  const int eq_before = block_scan_incl(eq, ws) - eq;
  int teq = take_eq - eq_before;
  teq = teq < 0 ? 0 : (teq > eq ? eq : teq);
  const int take = gt + teq;
  int off = block_scan_incl(take, ws) - take;
  for (int j = j0; j < j1; ++j) {
    const uint32_t key = key_of(j);
    if (key > prefix || (key == prefix && teq > 0)) {
      if (key == prefix) --teq;
      if (DKV_IN_BOUNDS(off < k, a.c.status)) out[off] = j;
      ++off;
    }
  }
}

template <int KB, int VB>
cudaError_t launch_scores_kv(const AttnArgs& a, float* part, int64_t ld, cudaStream_t s) {
  const int nrb = (a.c.rows + kRowsPerCta - 1) / kRowsPerCta;
  const int64_t n_tiles = (a.L + T - 1) / T;
  // chunks of tiles per (unit, row block): the count whose waves (two CTAs
  // per SM resident) times tiles per chunk is least, i.e. the grid that
  // loses the least to a partly filled last wave
  const int64_t slots = 2 * 148, cells = int64_t(a.c.U) * nrb;
  int64_t tpc = n_tiles < 1 ? 1 : n_tiles, best = -1;
  for (int64_t nc = 1; n_tiles > 0 && nc <= n_tiles && nc <= 64; ++nc) {
    const int64_t t = (n_tiles + nc - 1) / nc;
    const int64_t waves = (cells * ((n_tiles + t - 1) / t) + slots - 1) / slots;
    if (best < 0 || waves * (t + 1) < best) {
      best = waves * (t + 1);
      tpc = t;
    }
  }
  const int nchunk = int(n_tiles < 1 ? 1 : (n_tiles + tpc - 1) / tpc);
  const unsigned grid = unsigned(a.c.U) * unsigned(nrb) * unsigned(nchunk);
  const cudaError_t e = launch_pdl(score_kernel<KB, VB>, dim3(grid), dim3(256), 0, s, a, part, ld,
                                   int(tpc), nchunk);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KB>
cudaError_t launch_scores_k(const AttnArgs& a, float* part, int64_t ld, cudaStream_t s) {
  switch (a.c.vb) {
    case 2: return launch_scores_kv<KB, 2>(a, part, ld, s);
    case 3: return launch_scores_kv<KB, 3>(a, part, ld, s);
    case 4: return launch_scores_kv<KB, 4>(a, part, ld, s);
    default: return launch_scores_kv<KB, 16>(a, part, ld, s);
  }
}

template <int KB, int VB>
cudaError_t launch_kv(const AttnArgs& a, cudaStream_t s) {
  const int nrb = (a.c.rows + kRowsPerCta - 1) / kRowsPerCta;
  const int rows_cta = a.c.rows < kRowsPerCta ? a.c.rows : kRowsPerCta;
  if (a.c.rows % 16) return cudaErrorInvalidValue;
  const int threads = rows_cta * 2;  // one warp per 16 rows
  const unsigned grid = unsigned(a.c.U) * unsigned(a.nsplit) * unsigned(nrb);
  const cudaError_t e =
      a.gather ? launch_pdl(attn_mma_kernel<KB, VB, true>, dim3(grid), dim3(threads), 0, s, a)
               : launch_pdl(attn_mma_kernel<KB, VB, false>, dim3(grid), dim3(threads), 0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KB>
cudaError_t launch_k(const AttnArgs& a, cudaStream_t s) {
  switch (a.c.vb) {
    case 2: return launch_kv<KB, 2>(a, s);
    case 3: return launch_kv<KB, 3>(a, s);
    case 4: return launch_kv<KB, 4>(a, s);
    default: return launch_kv<KB, 16>(a, s);
  }
}

}  // namespace

cudaError_t launch_attention_mma(const AttnArgs& a, cudaStream_t s) {
  switch (a.c.kb) {
    case 2: return launch_k<2>(a, s);
    case 3: return launch_k<3>(a, s);
    case 4: return launch_k<4>(a, s);
    default: return launch_k<16>(a, s);
  }
}

int score_row_blocks(const CacheView& c) { return (c.rows + kRowsPerCta - 1) / kRowsPerCta; }

cudaError_t launch_scores(const AttnArgs& a, float* part, int64_t ld, cudaStream_t s) {
  if (a.c.rows % 16) return cudaErrorInvalidValue;
  switch (a.c.kb) {
    case 2: return launch_scores_k<2>(a, part, ld, s);
    case 3: return launch_scores_k<3>(a, part, ld, s);
    case 4: return launch_scores_k<4>(a, part, ld, s);
    default: return launch_scores_k<16>(a, part, ld, s);
  }
}

cudaError_t launch_topk(const AttnArgs& a, const float* part, int64_t ld, float* scores,
                        int32_t* sel, cudaStream_t s) {
  const cudaError_t e = launch_pdl(topk_kernel, dim3(unsigned(a.c.U)), dim3(1024), 0, s, a, part,
                                   ld, score_row_blocks(a.c), scores, sel);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_combine(const AttnArgs& a, cudaStream_t s) {
  const int64_t rows = int64_t(a.c.U) * a.c.rows;
  const cudaError_t e = launch_pdl(combine_kernel, dim3(unsigned((rows + kCombineWarps - 1) / kCombineWarps)),
                                   dim3(32 * kCombineWarps), 0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dkv
