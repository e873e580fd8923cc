// Quantize-on-commit ("KV entries are quantized only when a block is
// committed; the block still being denoised stays in full precision; keys use
// KIVI-style per-channel asymmetric quantization" -- SoloQ, block-diffusion
// paragraph; protected K entries kept in high precision with standard low-bit
// V -- "KV Cache Quantization for Diffusion Language Models", abstract).
//
// One CTA of 256 threads per (sequence, kv-head) unit.  The block's V and,
// when a K group completes, the pending K stream (bf16 tail + block) are first
// staged in shared memory with coalesced 16-byte loads.  V: one item per
// (token, channel group), threads 128..255.  K: thread c < 128 owns channel c
// of every K group that this commit completes; tokens of an incomplete group
// wait in the bf16 tail.  Group sizes are compile-time constants, so each
// group's loads and divisions are unrolled and independent.
//
// This file is compiled with -fmad=false and uses only correctly rounded fp32
// operations (__fsub_rn, __fdiv_rn, __float2half_rn, __float2int_rn), so the
// codes, scales and zero-points are bit-identical to any other IEEE fp32
// evaluation of the same formulas.
#include "dkv_internal.cuh"

namespace dkv {
namespace {

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t b) {
  return __uint_as_float(uint32_t(b) << 16);
}

// NaN, +-Inf or beyond the fp16 range
__device__ __forceinline__ bool out_of_range(float x) { return !(fabsf(x) <= 65504.f); }

__device__ __forceinline__ float sanitize(float x) {
  if (x != x) return 0.f;
  return fminf(fmaxf(x, -65504.f), 65504.f);
}

struct GroupQuant {
  float s32, z32;  // stored fp16 scale / zero, widened
  float rs;        // correctly rounded 1 / s32 (0 when s32 == 0)
  __half2 sz;      // (scale, zero)
};

// s = fp16((mx - mn) / levels), z = fp16(mn)
__device__ __forceinline__ GroupQuant make_quant(float mn, float mx, int levels) {
  const float s_f = __fdiv_rn(__fsub_rn(mx, mn), float(levels));
  const __half s = __float2half_rn(s_f);
  const __half z = __float2half_rn(mn);
  GroupQuant q;
  q.s32 = __half2float(s);
  q.z32 = __half2float(z);
  q.rs = q.s32 > 0.f ? __frcp_rn(q.s32) : 0.f;
  q.sz = __halves2half2(s, z);
  return q;
}

// q = clamp(rint((x - z) / s), 0, levels) with (x - z) / s the correctly
// rounded fp32 quotient; 0 when s == 0.  The quotient is estimated as
// (x - z) * fl(1/s), within a few ulp of it.  Inside the clamp range
// (|quotient| <= levels + 1 <= 16) those few ulp are below 2^-17, so the
// estimate rounds to the same integer unless it lies within 2^-12 of a tie
// (k + 1/2); only then is the exact division taken.  Outside the range both
// clamp alike.  The code is therefore the division-based one, bit for bit.
__device__ __noinline__ float exact_quotient(float num, float s) { return __fdiv_rn(num, s); }

__device__ __forceinline__ uint32_t code_of(float x, const GroupQuant& q, int levels) {
  if (!(q.s32 > 0.f)) return 0u;
  const float num = __fsub_rn(x, q.z32);
  float t = __fmul_rn(num, q.rs);
  if (fabsf(fabsf(__fsub_rn(t, rintf(t))) - 0.5f) < 2.44140625e-4f) t = exact_quotient(num, q.s32);
  int c = __float2int_rn(t);
  c = c < 0 ? 0 : (c > levels ? levels : c);
  return uint32_t(c);
}

constexpr int kThreads = 256;         // 128 K channels and up to 128 V groups side by side
constexpr int kRowPad = kHeadDim + 8;  // shared-memory row stride in halves (272 B)

__device__ __forceinline__ void range_check8(uint4 x, bool& range) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    range |= out_of_range(bf16_bits_to_f32(uint16_t(w[j] & 0xFFFF)));
    range |= out_of_range(bf16_bits_to_f32(uint16_t(w[j] >> 16)));
  }
}

// rows [0, n) of a [n][d] bf16 block -> shared rows of kRowPad halves
__device__ __forceinline__ void stage_rows(uint16_t* dst, const uint16_t* src, int n, int tid) {
  for (int i = tid; i < n * (kHeadDim / 8); i += kThreads) {
    const int t = i / (kHeadDim / 8), o = i % (kHeadDim / 8);
    *reinterpret_cast<uint4*>(dst + t * kRowPad + o * 8) =
        __ldg(reinterpret_cast<const uint4*>(src + size_t(t) * kHeadDim + o * 8));
  }
}

__device__ __forceinline__ float bf16_at(const uint16_t* p) { return bf16_bits_to_f32(*p); }

// Protect bits of the sink positions [0, sink) among the 32 positions
// starting at pos0.
__device__ __forceinline__ uint32_t sink_bits(int64_t pos0, int sink) {
  const int64_t n = sink - pos0;
  return n <= 0 ? 0u : (n >= 32 ? 0xFFFFFFFFu : ((1u << uint32_t(n)) - 1u));
}

// One V group: G consecutive channels of one token (x: shared memory, 16-byte
// aligned).  Rolled loops over 8-channel chunks and code words keep the code
// small (each warp runs it once, so its instructions come from the cache).
template <int VB>
__device__ __forceinline__ void quant_v_group(const uint16_t* x, int G, uint32_t* codes,
                                              __half2* sz, bool& range) {
  constexpr int levels = (1 << VB) - 1;
  constexpr int per = 32 / VB;
  float mn2[2] = {__int_as_float(0x7f800000), __int_as_float(0x7f800000)};
  float mx2[2] = {-__int_as_float(0x7f800000), -__int_as_float(0x7f800000)};
#pragma unroll 1
  for (int i8 = 0; i8 < G; i8 += 8) {
    const uint4 q8 = *reinterpret_cast<const uint4*>(x + i8);
    const uint32_t w[4] = {q8.x, q8.y, q8.z, q8.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float f = bf16_bits_to_f32(uint16_t(w[j >> 1] >> (16 * (j & 1))));
      range |= out_of_range(f);
      f = sanitize(f);
      mn2[j & 1] = fminf(mn2[j & 1], f);
      mx2[j & 1] = fmaxf(mx2[j & 1], f);
    }
  }
  const GroupQuant q = make_quant(fminf(mn2[0], mn2[1]), fmaxf(mx2[0], mx2[1]), levels);
#pragma unroll 1
  for (int w = 0; w < G / per; ++w) {
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < per; ++e)
      word |= code_of(sanitize(bf16_at(x + w * per + e)), q, levels) << (e * VB);
    codes[w] = word;
  }
  *sz = q.sz;
}

// K-RPBH rotation of one V row held by a warp ("SoloQ", K-RPBH paragraph:
// random permutation, per-block Hadamard, k x k orthogonal mix of the same
// in-block coordinate across the k = d/b blocks).  On entry x[e] holds input
// channel perm[4 lane + e] (the caller's gather applies the permutation); on
// exit rotated channel 4 lane + e.  The fp32 order is fixed because the codes
// depend on the last bit: butterflies (lo, hi) -> (lo + hi, lo - hi) over
// strides 1, 2, 4, ..., b/2; one multiply by fp32(1/sqrt(b)); the mix as a
// left-to-right sum over the k blocks of rounded products, starting from 0.
__device__ __forceinline__ void rotate_row(float (&x)[4], int b, float norm,
                                        const float* __restrict__ mix, int lane) {
  const int k = kHeadDim / b, lb = b / 4;  // lanes per block
#pragma unroll
  for (int h = 1; h <= 2; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (e & h) continue;
      const float lo = x[e], hi = x[e + h];
      x[e] = __fadd_rn(lo, hi);
      x[e + h] = __fsub_rn(lo, hi);
    }
  }
  for (int h = 4; h < b; h <<= 1) {
    const bool upper = (lane & (h >> 2)) != 0;  // channel 4 lane + e has bit h set
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float p = __shfl_xor_sync(0xffffffffu, x[e], h >> 2);
      x[e] = upper ? __fsub_rn(p, x[e]) : __fadd_rn(x[e], p);
    }
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = __fmul_rn(x[e], norm);
  const int r = lane / lb, i_lane = lane % lb;  // output block r, in-block lane
  float w[4] = {0.f, 0.f, 0.f, 0.f};
  for (int cc = 0; cc < k; ++cc) {
    const float m = __ldg(mix + r * k + cc);  // mix[r][cc]
#pragma unroll
    for (int e = 0; e < 4; ++e)
      w[e] = __fadd_rn(w[e], __fmul_rn(m, __shfl_sync(0xffffffffu, x[e], cc * lb + i_lane)));
  }
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = w[e];
}

// Per-token quantization of a rotated V row held by a warp (channels 4 lane +
// e): groups of G consecutive channels (G/4 lanes), the same quantizer as
// quant_v_group, codes packed along channels.
template <int VB>
__device__ __forceinline__ void quant_v_rotated(float (&w)[4], int G, uint32_t* codes, __half2* sz,
                                             int lane, bool& range) {
  constexpr int levels = (1 << VB) - 1;
  constexpr int lw = 8 / VB;  // lanes per code word (32 / VB channels)
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    range |= out_of_range(w[e]);
    w[e] = sanitize(w[e]);
  }
  float mn = fminf(fminf(w[0], w[1]), fminf(w[2], w[3]));
  float mx = fmaxf(fmaxf(w[0], w[1]), fmaxf(w[2], w[3]));
  for (int o = 1; o < G / 4; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  const GroupQuant q = make_quant(mn, mx, levels);
  uint32_t word = 0;
#pragma unroll
  for (int e = 0; e < 4; ++e) word |= code_of(w[e], q, levels) << (e * VB);
  word <<= (lane % lw) * 4 * VB;
#pragma unroll
  for (int o = 1; o < lw; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
  if (lane % lw == 0) codes[lane / lw] = word;
  if (lane % (G / 4) == 0) sz[lane / (G / 4)] = q.sz;
}

// One K group of channel ch: G tokens of the pending stream (rows of sk),
// protected tokens (bits of gm) left out of min/max and given code 0.  Rolled
// loops as above.
template <int KB>
__device__ __forceinline__ GroupQuant quant_k_group(const uint16_t* sk, int G, int row0, int ch,
                                                    const uint32_t (&gm)[4], int check_row,
                                                    uint32_t* codes, bool& range) {
  constexpr int levels = (1 << KB) - 1;
  constexpr int per = 32 / KB;
  float mn2[2] = {__int_as_float(0x7f800000), __int_as_float(0x7f800000)};
  float mx2[2] = {-__int_as_float(0x7f800000), -__int_as_float(0x7f800000)};
#pragma unroll 1
  for (int t8 = 0; t8 < G; t8 += 8) {
    const uint32_t m8 = (gm[t8 >> 5] >> (t8 & 31)) & 0xFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int t = t8 + i;
      float f = bf16_at(sk + (row0 + t) * kRowPad + ch);
      if (row0 + t >= check_row) range |= out_of_range(f);
      f = sanitize(f);
      if (!((m8 >> i) & 1u)) {
        mn2[i & 1] = fminf(mn2[i & 1], f);
        mx2[i & 1] = fmaxf(mx2[i & 1], f);
      }
    }
  }
  float mn = fminf(mn2[0], mn2[1]);
  float mx = fmaxf(mx2[0], mx2[1]);
  if (mn > mx) mn = mx = 0.f;  // every token protected
  const GroupQuant q = make_quant(mn, mx, levels);
#pragma unroll 1
  for (int w = 0; w < G / per; ++w) {
    const uint32_t mw = (gm[(w * per) >> 5] >> ((w * per) & 31));  // per <= 16 bits of mask
    uint32_t word = 0;
#pragma unroll
    for (int e = 0; e < per; ++e) {
      const uint32_t cq =
          code_of(sanitize(bf16_at(sk + (row0 + w * per + e) * kRowPad + ch)), q, levels);
      if (!((mw >> e) & 1u)) word |= cq << (e * KB);  // protected slot: code 0
    }
    codes[w] = word;
  }
  return q;
}

// Shared memory: the V block [blk][kRowPad] (quantized V), then the pending
// K stream [max(k_group, blk)][kRowPad] (quantized K, when a group completes).
// Threads [0, 128): K (channel = thread); threads [128, 256): V groups.
template <int KB, int VB>
__global__ void __launch_bounds__(kThreads)
commit_kernel(CacheView c, const uint16_t* __restrict__ k, const uint16_t* __restrict__ v,
              const uint32_t* __restrict__ pw, int64_t p0, int truncated) {
  extern __shared__ __align__(16) uint16_t sbuf[];
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x;
  const int tid = threadIdx.x;
  const int d = kHeadDim;
  const int blk = c.blk;
  const uint16_t* ku = k + size_t(u) * blk * d;
  const uint16_t* vu = v + size_t(u) * blk * d;
  const int nbw = blk / 32;
  bool range = false;
  uint16_t* sv = sbuf;
  uint16_t* sk = sbuf + (VB < 16 ? blk * kRowPad : 0);
  const int GK = c.GK;
  const int n_tail = KB < 16 ? int(p0 % GK) : 0;
  const bool completes = KB < 16 && n_tail + blk >= GK;
  // bounds-checking build: the block lands inside the unit's capacity, an
  // incomplete group stays inside the tail, the completed groups inside the
  // group arrays (the condition is the same for every thread of the block)
  if (!DKV_IN_BOUNDS(p0 >= 0 && p0 + blk <= c.cap && blk % 32 == 0 &&
                         (KB == 16 || (completes ? (p0 + blk) / GK <= c.nG && (n_tail + blk) % GK == 0
                                                 : n_tail + blk <= GK)) &&
                         (VB == 16 || c.sink <= c.cap),
                     c.status))
    return;

  // a roll-back to p0 (a multiple of the K group) recorded since the last
  // commit: the side table keeps the entries of the groups before p0, the
  // tail is empty; applied here, before any thread reads either
  if (KB < 16 && truncated) {
    if (tid == 0) c.prot_count[u] = c.prot_gstart[size_t(u) * size_t(c.nG + 1) + size_t(p0 / GK)];
    if (tid < c.twords) c.tail_mask[size_t(u) * c.twords + tid] = 0u;
  }

  // ------------------------------------------------------------------ stage
  if constexpr (VB < 16) stage_rows(sv, vu, blk, tid);
  if (completes) {
    stage_rows(sk, c.k_tail + size_t(u) * GK * d, n_tail, tid);
    stage_rows(sk + n_tail * kRowPad, ku, blk, tid);
  }
  __syncthreads();

  // ------------------------------------------------------------------ V
  if constexpr (VB == 16) {
    const uint4* src = reinterpret_cast<const uint4*>(vu);
    uint4* dst = reinterpret_cast<uint4*>(c.v_raw + (size_t(u) * c.cap + p0) * d);
    for (int i = tid; i < blk * d / 8; i += kThreads) {
      const uint4 x = src[i];
      range_check8(x, range);
      dst[i] = x;
    }
  } else if (tid >= 128 && c.vrot_b) {
    // rotated V (no sink): warp wv rotates and quantizes tokens wv, wv + 4, ...
    const int lane = tid & 31;
    int pm[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pm[e] = __ldg(c.vrot_perm + 4 * lane + e);
    for (int t = (tid - 128) >> 5; t < blk; t += 4) {
      float x[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float f = bf16_at(sv + t * kRowPad + pm[e]);
        range |= out_of_range(f);
        x[e] = sanitize(f);
      }
      rotate_row(x, c.vrot_b, c.vrot_norm, c.vrot_mix, lane);
      const size_t tok = size_t(u) * c.cap + size_t(p0 + t);
      quant_v_rotated<VB>(x, c.GV, c.v_codes + tok * c.vw, c.v_sz + tok * c.vgroups, lane, range);
    }
  } else if (tid >= 128) {
    // sink positions keep their V row in bf16 too
    const int64_t ns = c.sink - p0 < blk ? c.sink - p0 : blk;
    for (int i = tid - 128; i < ns * (kHeadDim / 8); i += 128) {
      const int t = i / (kHeadDim / 8), o = i % (kHeadDim / 8);
      reinterpret_cast<uint4*>(c.v_sink + (size_t(u) * c.sink + size_t(p0 + t)) * d)[o] =
          *reinterpret_cast<const uint4*>(sv + t * kRowPad + o * 8);
    }
    const int GV = c.GV;
    const int ngr = d / GV;
    for (int it = tid - 128; it < blk * ngr; it += 128) {
      const int t = it / ngr, gi = it % ngr;
      const uint16_t* x = sv + t * kRowPad + gi * GV;
      uint32_t* codes = c.v_codes + (size_t(u) * c.cap + p0 + t) * c.vw + gi * GV * VB / 32;
      __half2* sz = c.v_sz + (size_t(u) * c.cap + p0 + t) * ngr + gi;
      quant_v_group<VB>(x, GV, codes, sz, range);
    }
  }

  // ------------------------------------------------------------------ K
  if constexpr (KB == 16) {
    const uint4* src = reinterpret_cast<const uint4*>(ku);
    uint4* dst = reinterpret_cast<uint4*>(c.k_raw + (size_t(u) * c.cap + p0) * d);
    for (int i = tid; i < blk * d / 8; i += kThreads) {
      const uint4 x = src[i];
      range_check8(x, range);
      dst[i] = x;
    }
  } else {
    uint16_t* tail = c.k_tail + size_t(u) * GK * d;
    uint32_t* tmask = c.tail_mask + size_t(u) * c.twords;
    if (!completes) {
      // the group stays incomplete: append the block to the bf16 tail
      const uint4* src = reinterpret_cast<const uint4*>(ku);
      uint4* dst = reinterpret_cast<uint4*>(tail + size_t(n_tail) * d);
      for (int i = tid; i < blk * d / 8; i += kThreads) {
        const uint4 x = src[i];
        range_check8(x, range);
        dst[i] = x;
      }
      if (tid < nbw)
        tmask[n_tail / 32 + tid] =
            (pw ? pw[size_t(u) * nbw + tid] : 0u) | sink_bits(p0 + 32 * tid, c.sink);
    } else if (tid < 128) {
      // pending stream = tail[0, n_tail) ++ block[0, blk) (staged in sk);
      // quantize every complete group (k_group and block divide one another,
      // so nothing is left over)
      const int npend = n_tail + blk;
      const int nfull = npend / GK;
      const int ch = tid;  // channel
      int count = c.prot_count[u];
      const int64_t j0 = (p0 - n_tail) / GK;
      for (int gi = 0; gi < nfull; ++gi) {
        const int64_t j = j0 + gi;
        uint32_t gm[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          if (w < GK / 32) {
            const int pwi = gi * GK / 32 + w;  // word of the pending stream
            if (pwi < n_tail / 32)
              gm[w] = tmask[pwi];
            else
              gm[w] = pw ? pw[size_t(u) * nbw + (pwi - n_tail / 32)] : 0u;
            gm[w] |= sink_bits(j * GK + 32 * w, c.sink);
          }
        }
        // side table full: keep the first `room` protected tokens by position
        int want = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) want += __popc(gm[w]);
        const int room = c.P - count;
        if (want > room) {
          int kept = 0;
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint32_t m = gm[w], nm = 0u;
            while (m && kept < room) {
              const uint32_t low = m & (0u - m);
              nm |= low;
              m ^= low;
              ++kept;
            }
            gm[w] = nm;
          }
          if (tid == 0) atomicOr(c.status, uint32_t(DKV_FLAG_CAPACITY));
        }
        uint32_t* codes = c.k_codes + ((size_t(u) * c.nG + j) * d + ch) * c.kw;
        const GroupQuant q = quant_k_group<KB>(sk, GK, gi * GK, ch, gm, n_tail, codes, range);
        c.k_sz[(size_t(u) * c.nG + j) * d + ch] = q.sz;
        // side-table entries, ascending positions
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t m = gm[w];
          while (m) {
            const int b = __ffs(m) - 1;
            m &= m - 1u;
            const int t = w * 32 + b;
            if (!DKV_IN_BOUNDS(count < c.P, c.status)) break;
            if (tid == 0) c.prot_pos[size_t(u) * c.P + count] = int32_t(j * GK + t);
            c.prot_k[(size_t(u) * c.P + count) * d + ch] = sk[(gi * GK + t) * kRowPad + ch];
            ++count;
          }
        }
        if (tid == 0) c.prot_gstart[size_t(u) * (c.nG + 1) + j + 1] = count;
      }
      // every K thread has read prot_count and the tail mask before either
      // is rewritten (named barrier over the 128 K threads only)
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (tid == 0) c.prot_count[u] = count;
      if (tid < c.twords) tmask[tid] = 0u;
    }
  }
  if (range) atomicOr(c.status, uint32_t(DKV_FLAG_RANGE));
}

// The active block's V rows rotated like committed rows and rounded to bf16
// (attention sums them with the rotated cache rows).  One warp per row.
__global__ void __launch_bounds__(256) rotate_rows_kernel(CacheView c,
                                                          const uint16_t* __restrict__ src,
                                                          uint16_t* __restrict__ dst,
                                                          int64_t n_rows) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t row = int64_t(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (row >= n_rows) return;
  const uint16_t* s = src + row * kHeadDim;
  float x[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) x[e] = bf16_bits_to_f32(__ldg(s + __ldg(c.vrot_perm + 4 * lane + e)));
  rotate_row(x, c.vrot_b, c.vrot_norm, c.vrot_mix, lane);
  const __nv_bfloat162 lo = __floats2bfloat162_rn(x[0], x[1]);
  const __nv_bfloat162 hi = __floats2bfloat162_rn(x[2], x[3]);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&lo);
  pk.y = *reinterpret_cast<const uint32_t*>(&hi);
  *reinterpret_cast<uint2*>(dst + row * kHeadDim + 4 * lane) = pk;
}

// Roll back to new_len (a multiple of the K group): the side table keeps the
// entries stored before group new_len / GK; the tail is empty.
__global__ void truncate_kernel(CacheView c, int64_t new_len) {
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= c.U) return;
  c.prot_count[u] = c.prot_gstart[size_t(u) * (c.nG + 1) + new_len / c.GK];
  for (int w = 0; w < c.twords; ++w) c.tail_mask[size_t(u) * c.twords + w] = 0u;
}

template <int KB, int VB>
cudaError_t launch_kv(const CacheView& c, const uint16_t* k, const uint16_t* v,
                      const uint32_t* pw, int64_t p0, bool truncated, cudaStream_t s) {
  const int krows = KB < 16 ? (c.GK > c.blk ? c.GK : c.blk) : 0;
  const int vrows = VB < 16 ? c.blk : 0;
  const size_t smem = size_t(krows + vrows) * kRowPad * 2;
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(commit_kernel<KB, VB>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
  }
  const cudaError_t e = launch_pdl(commit_kernel<KB, VB>, dim3(c.U), dim3(kThreads), smem, s, c, k,
                                   v, pw, p0, truncated ? 1 : 0);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KB>
cudaError_t launch_k(const CacheView& c, const uint16_t* k, const uint16_t* v,
                     const uint32_t* pw, int64_t p0, bool truncated, cudaStream_t s) {
  switch (c.vb) {
    case 2: return launch_kv<KB, 2>(c, k, v, pw, p0, truncated, s);
    case 4: return launch_kv<KB, 4>(c, k, v, pw, p0, truncated, s);
    default: return launch_kv<KB, 16>(c, k, v, pw, p0, truncated, s);
  }
}

}  // namespace

cudaError_t launch_truncate(const CacheView& c, int64_t new_len, cudaStream_t s) {
  const cudaError_t e = launch_pdl(truncate_kernel, dim3((c.U + 127) / 128), dim3(128), 0, s, c,
                                   new_len);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_rotate_v_rows(const CacheView& c, const uint16_t* src, uint16_t* dst,
                                 cudaStream_t s) {
  const int64_t n_rows = int64_t(c.U) * c.blk;
  const cudaError_t e = launch_pdl(rotate_rows_kernel, dim3(unsigned((n_rows + 7) / 8)), dim3(256),
                                   0, s, c, src, dst, n_rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_commit(const CacheView& c, const uint16_t* k, const uint16_t* v,
                          const uint32_t* pw, int64_t p0, bool truncated, cudaStream_t s) {
  switch (c.kb) {
    case 2: return launch_k<2>(c, k, v, pw, p0, truncated, s);
    case 4: return launch_k<4>(c, k, v, pw, p0, truncated, s);
    default: return launch_k<16>(c, k, v, pw, p0, truncated, s);
  }
}

}  // namespace dkv
