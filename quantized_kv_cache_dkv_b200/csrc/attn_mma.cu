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
// (unnormalised O, running max, running sum) are merged by combine_kernel.
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
        const size_t tok = size_t(u) * c.cap + pos0 + t;
        const __half2 sz = c.v_sz[tok * c.vgroups + (q * 32) / c.GV];
        const __half2 s2 = __half2half2(__low2half(sz));
        const __half2 z2 = __half2half2(__high2half(sz));
        uint4* dst = reinterpret_cast<uint4*>(Vt + (ch * 32 + t) * VT_LD + q * 32);
        if (pos0 + t < c.sink && DKV_IN_BOUNDS(c.sink <= c.cap, c.status)) {
          // sink position: its bf16 V row
          const uint4* src = reinterpret_cast<const uint4*>(
              c.v_sink + (size_t(u) * c.sink + size_t(pos0 + t)) * d + q * 32);
#pragma unroll
          for (int k = 0; k < 4; ++k) dst[k] = bf16x8_to_f16x8(src[k]);
          continue;
        }
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

constexpr int kRowsPerCta = 128;  // 8 warps; a larger query group takes several CTAs

template <int KB, int VB>
__global__ void __launch_bounds__(256)
attn_mma_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ __align__(16) __half Kt[kHeadDim * KT_LD];
  __shared__ __align__(16) __half Vt[T * VT_LD];
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
    fill_chunk<KB, VB>(a, ul, u, tile_start, 0, Kt, Vt, tid, nthr);
    fill_chunk<KB, VB>(a, ul, u, tile_start + kChunk, 1, Kt, Vt, tid, nthr);
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
    float* po0 = a.part_o + (prow + r0) * kHeadDim;
    float* po1 = po0 + 8 * kHeadDim;
#pragma unroll
    for (int nd = 0; nd < 16; ++nd) {
      const int col = nd * 8 + cq;
      *reinterpret_cast<float2*>(po0 + col) = make_float2(o[nd][0], o[nd][1]);
      *reinterpret_cast<float2*>(po1 + col) = make_float2(o[nd][2], o[nd][3]);
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

// One warp per (unit, row): out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s
// (rotated back first when V is stored rotated)
__global__ void __launch_bounds__(128) combine_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ float rbuf[4][kHeadDim];
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * 4 + warp;
  const int rows = a.c.rows;
  if (row >= int64_t(a.c.U) * rows) return;
  const int64_t u = row / rows, r = row % rows;
  const size_t base = size_t(u) * a.nsplit * rows + r;  // split s at base + s*rows
  float M = -__int_as_float(0x7f800000);
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, a.part_ml[base + size_t(s) * rows].x);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  float lsum = 0.f;
  for (int s = 0; s < a.nsplit; ++s) {
    const float2 ml = a.part_ml[base + size_t(s) * rows];
    const float w = fast_exp2(ml.x - M);
    lsum += w * ml.y;
    const float4 x =
        *reinterpret_cast<const float4*>(a.part_o + (base + size_t(s) * rows) * kHeadDim + lane * 4);
    acc.x += w * x.x;
    acc.y += w * x.y;
    acc.z += w * x.z;
    acc.w += w * x.w;
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

template <int KB, int VB>
cudaError_t launch_kv(const AttnArgs& a, cudaStream_t s) {
  const int nrb = (a.c.rows + kRowsPerCta - 1) / kRowsPerCta;
  const int rows_cta = a.c.rows < kRowsPerCta ? a.c.rows : kRowsPerCta;
  if (a.c.rows % 16) return cudaErrorInvalidValue;
  const int threads = rows_cta * 2;  // one warp per 16 rows
  const unsigned grid = unsigned(a.c.U) * unsigned(a.nsplit) * unsigned(nrb);
  const cudaError_t e = launch_pdl(attn_mma_kernel<KB, VB>, dim3(grid), dim3(threads), 0, s, a);
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

cudaError_t launch_combine(const AttnArgs& a, cudaStream_t s) {
  const int64_t rows = int64_t(a.c.U) * a.c.rows;
  const cudaError_t e = launch_pdl(combine_kernel, dim3(unsigned((rows + 3) / 4)), dim3(128), 0, s, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace dkv
