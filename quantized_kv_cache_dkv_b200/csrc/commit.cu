// Quantize-on-commit.  In block-diffusion decoding the cache is quantized at
// the moment a block is committed and never before; the block under
// denoising keeps its full precision; K is quantized per channel with an
// asymmetric (min / max) grid, as KIVI does (SoloQ, block-diffusion
// paragraph).  A chosen set of K entries keeps high precision while V is
// stored at low bit width (KProtect, "KV Cache Quantization for Diffusion
// Language Models", abstract).
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

constexpr int kThreads = 256;
// CTAs per (sequence, kv-head) unit, chosen per launch from the unit count
// (1, 2 or 4, so that all CTAs fit one wave of four per SM): slice sl of nsl
// takes K channels [sl 128/nsl, (sl + 1) 128/nsl) and V tokens
// [sl blk/nsl, (sl + 1) blk/nsl).
constexpr int kMaxSlices = 4;
constexpr int kPendStride = 128 + 8;  // tokens per staged channel row (pending <= 128), padded

__device__ __forceinline__ void range_check8(uint4 x, bool& range) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    range |= out_of_range(bf16_bits_to_f32(uint16_t(w[j] & 0xFFFF)));
    range |= out_of_range(bf16_bits_to_f32(uint16_t(w[j] >> 16)));
  }
}

// Protect bits of the sink positions [0, sink) among the 32 positions
// starting at pos0.
__device__ __forceinline__ uint32_t sink_bits(int64_t pos0, int sink) {
  const int64_t n = sink - pos0;
  return n <= 0 ? 0u : (n >= 32 ? 0xFFFFFFFFu : ((1u << uint32_t(n)) - 1u));
}

// K-RPBH rotation of one V row held by a warp (SoloQ, K-RPBH paragraph:
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
// quant_v_group, codes packed along channels.  At 3 bits the 12 code bits of
// a lane sit at stream bits 12 (lane % 8) of its 32-channel block, whose 96
// bits fill three words (lanes 2 and 5 straddle a word boundary).
template <int VB>
__device__ __forceinline__ void quant_v_rotated(float (&w)[4], int G, uint32_t* codes, __half2* sz,
                                             int lane, bool& range) {
  constexpr int levels = (1 << VB) - 1;
  constexpr int lw = VB == 3 ? 8 : 8 / VB;  // lanes per code word (32 / VB channels; 3 words at 3 bits)
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
  if constexpr (VB == 3) {
    const int pos = 12 * (lane & 7), wi = pos >> 5, off = pos & 31;
    uint32_t part[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      part[k] = wi == k ? word << off : 0u;
      if (off > 20 && wi + 1 == k) part[k] |= word >> (32 - off);
#pragma unroll
      for (int o = 1; o < 8; o <<= 1) part[k] |= __shfl_xor_sync(0xffffffffu, part[k], o);
    }
    if ((lane & 7) == 0) {
#pragma unroll
      for (int k = 0; k < 3; ++k) codes[(lane >> 3) * 3 + k] = part[k];
    }
  } else {
    word <<= (lane % lw) * 4 * VB;
#pragma unroll
    for (int o = 1; o < lw; o <<= 1) word |= __shfl_xor_sync(0xffffffffu, word, o);
    if (lane % lw == 0) codes[lane / lw] = word;
  }
  if (lane % (G / 4) == 0) sz[lane / (G / 4)] = q.sz;
}

// Packs n codes (code(e), e = 0..n-1, each < 2^B) little-endian into the
// bit stream of words[]: code e at bits [B e, B e + B).  n B is 32 (one
// word) or, at 3 bits, 96 (three words; codes 10 and 21 straddle words).
template <int B, int n, class F>
__device__ __forceinline__ void pack_codes(F code, uint32_t (&words)[n * B / 32]) {
  uint64_t lo = 0, hi = 0;  // bits [0, 64) and [64, 128) of the stream
#pragma unroll
  for (int e = 0; e < n; ++e) {
    const uint64_t cq = code(e);
    const int pos = B * e;
    if (pos + B <= 64) {
      lo |= cq << pos;
    } else if (pos >= 64) {
      hi |= cq << (pos - 64);
    } else {
      lo |= cq << pos;
      hi |= cq >> (64 - pos);
    }
  }
  words[0] = uint32_t(lo);
  if constexpr (n * B / 32 > 1) words[1] = uint32_t(lo >> 32);
  if constexpr (n * B / 32 > 2) words[2] = uint32_t(hi);
}

// Codes of n values (val(e), called with compile-time e only; val_slow(e),
// the same value for a run-time e; code 0 where bit e of `zero` is set) packed
// little-endian as in pack_codes, with code_of's arithmetic split in two
// passes: the unrolled pass takes the reciprocal estimate for every value and
// notes those near a tie; a rolled pass then replaces their codes with the
// exact division's (rare).  The unrolled loop holds no call, so the values
// need not stay live across one.  The unrolled pass clamps the estimate to
// [0, levels] before rounding it: rounding to nearest is monotone and both
// bounds are integers, so this gives clamp(rint(t)); the only ties that can
// change a code (k + 1/2, k = 0 .. levels - 1) lie inside the range, where
// the clamp leaves t as it is.  Adding 1.5 * 2^23 rounds t in [0, 15] to an
// integer (round to nearest even, as rint) in the low mantissa bits, and
// subtracting it back gives rint(t) exactly, so t - rint(t) is exact and
// |t - rint(t)| > 1/2 - 2^-12 is the same tie test as code_of's.
template <int B, int n, class V, class VS>
__device__ __forceinline__ void quantize_pack(V val, VS val_slow, uint32_t zero, const GroupQuant& q,
                                              int levels, uint32_t (&words)[n * B / 32]) {
  uint64_t lo = 0, hi = 0;  // bits [0, 64) and [64, 128) of the stream
  auto put = [&](int e, uint64_t cq) {
    const int pos = B * e;
    if (pos + B <= 64) {
      lo |= cq << pos;
    } else if (pos >= 64) {
      hi |= cq << (pos - 64);
    } else {
      lo |= cq << pos;
      hi |= cq >> (64 - pos);
    }
  };
  if (q.s32 > 0.f) {
    uint32_t tie = 0u;
    const float lv = float(levels);
    constexpr float kRound = 12582912.f;  // 1.5 * 2^23
#pragma unroll
    for (int e = 0; e < n; ++e) {
      if ((zero >> e) & 1u) continue;
      const float t = fminf(fmaxf(__fmul_rn(__fsub_rn(val(e), q.z32), q.rs), 0.f), lv);
      const float y = __fadd_rn(t, kRound);
      if (fabsf(__fsub_rn(t, __fsub_rn(y, kRound))) > 0.499755859375f) tie |= 1u << e;
      put(e, uint64_t(__float_as_uint(y) & uint32_t(levels)));
    }
#pragma unroll 1
    while (tie) {
      const int e = __ffs(tie) - 1;
      tie &= tie - 1u;
      int c = __float2int_rn(exact_quotient(__fsub_rn(val_slow(e), q.z32), q.s32));
      c = c < 0 ? 0 : (c > levels ? levels : c);
      // replace the estimate's code at bits [B e, B e + B)
      const int pos = B * e;
      const uint64_t m = (uint64_t(1) << B) - 1;
      if (pos + B <= 64) {
        lo = (lo & ~(m << pos)) | (uint64_t(c) << pos);
      } else if (pos >= 64) {
        hi = (hi & ~(m << (pos - 64))) | (uint64_t(c) << (pos - 64));
      } else {
        lo = (lo & ~(m << pos)) | (uint64_t(c) << pos);
        hi = (hi & ~(m >> (64 - pos))) | (uint64_t(c) >> (64 - pos));
      }
    }
  }
  words[0] = uint32_t(lo);
  if constexpr (n * B / 32 > 1) words[1] = uint32_t(lo >> 32);
  if constexpr (n * B / 32 > 2) words[2] = uint32_t(hi);
}

// min / max over the `lanes` consecutive lanes of one group (lanes a power
// of two dividing 32, the group aligned to it)
__device__ __forceinline__ void group_minmax(float& mn, float& mx, int lanes) {
  for (int o = 1; o < lanes; o <<= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
}

// Protect words of K group gi of the pending stream (the tail's slots, then
// the block), with the sink positions, cut to the side table's room: the
// first `room` protected tokens by position stay protected.  Returns how
// many stay; `cut` is set when some did not fit.
__device__ __forceinline__ int group_mask(const CacheView& c, const uint32_t* tmask,
                                          const uint32_t* pwu, int n_tail, int gi, int64_t j,
                                          int room, uint32_t (&gm)[4], bool& cut) {
  const int GK = c.GK;
  int want = 0;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    gm[w] = 0u;
    if (w < GK / 32) {
      const int pwi = gi * GK / 32 + w;  // word of the pending stream
      gm[w] = pwi < n_tail / 32 ? tmask[pwi] : (pwu ? pwu[pwi - n_tail / 32] : 0u);
      gm[w] |= sink_bits(j * GK + 32 * w, c.sink);
      want += __popc(gm[w]);
    }
  }
  if (want <= room) return want;
  cut = true;
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
  return kept;
}

// Quantize-on-commit of one block.  Grid: nsl CTAs per unit.  Every
// thread produces one packed code word: K item (group, channel, word) covers
// the 32/KB tokens of one word of one channel's group, V item (token, word)
// the 32/VB channels of one word of one token.  A group's min / max is
// reduced across the lanes holding its words (shuffles), so no thread runs a
// serial loop over a whole group.  Values are read straight from global
// memory (the K tail / the caller's block).  The K side table's running count
// is taken from the group index written by earlier commits (entries before
// the first group this commit completes), which no CTA of this launch
// writes, so the CTAs of one unit need no ordering among themselves.
template <int KB, int VB>
__global__ void __launch_bounds__(kThreads, 4)  // four CTAs per SM: one wave up to 592 CTAs
commit_kernel(const __grid_constant__ CacheView c, const uint16_t* __restrict__ k,
              const uint16_t* __restrict__ v, const uint32_t* __restrict__ pw,
              const __grid_constant__ CommitArgs ca, int nsl) {
  // the pending K stream of this CTA's 32 channels, channel-major (a
  // thread's tokens are contiguous), filled by coalesced row loads
  __shared__ __align__(16) uint16_t sk[kHeadDim * kPendStride];
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x / nsl, sl = blockIdx.x % nsl;
  const int sch = kHeadDim / nsl;  // K channels of this CTA
  // the unit's sequence: does it commit, at which position, after a roll-back?
  const int sq = u / c.Hkv;
  if (!((ca.commit[sq >> 5] >> (sq & 31)) & 1u)) return;
  const int64_t p0 = ca.p0.len[sq];
  const bool truncated = (ca.trunc[sq >> 5] >> (sq & 31)) & 1u;
  const int tid = threadIdx.x, lane = tid & 31;
  const int d = kHeadDim;
  const int blk = c.blk;
  const uint16_t* ku = k + size_t(u) * blk * d;
  const uint16_t* vu = v + size_t(u) * blk * d;
  const int nbw = blk / 32;
  const uint32_t* pwu = pw ? pw + size_t(u) * nbw : nullptr;
  bool range = false;
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
  const int tpc = blk / nsl;  // V (and raw K) tokens of this CTA
  const int t_lo = sl * tpc;

  // ------------------------------------------------------------------ K
  int nK = 0;  // K items of this CTA (a multiple of 32)
  // One thread codes kper tokens of one (group, channel) into kwpt packed
  // words: one word (32 / KB tokens) at 2 and 4 bits; at 3 bits 32 tokens,
  // whose codes fill exactly 3 words.  kthr threads share a group.
  constexpr int kper = KB < 16 ? (KB == 3 ? 32 : 32 / KB) : 1;
  constexpr int kwpt = KB == 3 ? 3 : 1;
  const int kthr = GK / kper;
  int nfull = 0;
  int64_t j0 = 0;
  int count0 = 0;
  if constexpr (KB == 16) {
    const uint4* src = reinterpret_cast<const uint4*>(ku + size_t(t_lo) * d);
    uint4* dst = reinterpret_cast<uint4*>(c.k_raw + (size_t(u) * c.cap + p0 + t_lo) * d);
    for (int i = tid; i < tpc * d / 8; i += kThreads) {
      const uint4 x = src[i];
      range_check8(x, range);
      dst[i] = x;
    }
  } else if (!completes) {
    // the group stays incomplete: this CTA's channels of the block go to the
    // bf16 tail; the slice-0 CTA writes the tail's protect words
    uint16_t* tail = c.k_tail + size_t(u) * GK * d;
    for (int i = tid; i < blk * (sch / 8); i += kThreads) {
      const int t = i / (sch / 8), o = i % (sch / 8);
      const uint4 x = *reinterpret_cast<const uint4*>(ku + size_t(t) * d + sch * sl + 8 * o);
      range_check8(x, range);
      *reinterpret_cast<uint4*>(tail + size_t(n_tail + t) * d + sch * sl + 8 * o) = x;
    }
    if (sl == 0 && tid < nbw)
      c.tail_mask[size_t(u) * c.twords + n_tail / 32 + tid] =
          (pwu ? pwu[tid] : 0u) | sink_bits(p0 + 32 * tid, c.sink);
    // a roll-back recorded since the last commit (p0 is then a multiple of
    // the K group): the side table's count restarts at the group index
    if (sl == 0 && tid == 0 && truncated)
      c.prot_count[u] = c.prot_gstart[size_t(u) * size_t(c.nG + 1) + size_t(p0 / GK)];
  } else {
    // pending stream = tail[0, n_tail) ++ block[0, blk); every complete group
    // is quantized (k_group and block divide one another: nothing is left)
    nfull = (n_tail + blk) / GK;
    j0 = (p0 - n_tail) / GK;
    count0 = c.prot_gstart[size_t(u) * size_t(c.nG + 1) + size_t(j0)];
    nK = nfull * sch * kthr;
    // stage: item (token t, octet o) = 8 channels of one row, 16-byte loads;
    // the block's values are range-checked (the tail's were on entry)
    const int npend = n_tail + blk;
    for (int i = tid; i < npend * (sch / 8); i += kThreads) {
      const int t = i / (sch / 8), o = i % (sch / 8);
      const uint16_t* src = t < n_tail ? c.k_tail + (size_t(u) * GK + t) * d
                                       : ku + size_t(t - n_tail) * d;
      const uint4 x = *reinterpret_cast<const uint4*>(src + sch * sl + 8 * o);
      if (t >= n_tail) range_check8(x, range);
      const uint32_t w4[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int e = 0; e < 8; ++e)
        sk[(8 * o + e) * kPendStride + t] = uint16_t(w4[e >> 1] >> (16 * (e & 1)));
    }
  }
  __syncthreads();

  // ------------------------------------------------------------------ V
  // likewise for V: vper channels of one token into vwpt words per thread
  constexpr int vper = VB < 16 ? (VB == 3 ? 32 : 32 / VB) : 1;
  constexpr int vwpt = VB == 3 ? 3 : 1;
  const int vthr = kHeadDim / vper;  // threads per token
  const int nV = (VB < 16 && !c.vrot_b) ? tpc * vthr : 0;
  if constexpr (VB == 16) {
    const uint4* src = reinterpret_cast<const uint4*>(vu + size_t(t_lo) * d);
    uint4* dst = reinterpret_cast<uint4*>(c.v_raw + (size_t(u) * c.cap + p0 + t_lo) * d);
    for (int i = tid; i < tpc * d / 8; i += kThreads) {
      const uint4 x = src[i];
      range_check8(x, range);
      dst[i] = x;
    }
  } else {
    // sink positions keep their V row in bf16 too
    const int64_t s_end = c.sink - p0 < int64_t(t_lo + tpc) ? c.sink - p0 : int64_t(t_lo + tpc);
    for (int i = tid; i < (s_end - t_lo) * (kHeadDim / 8); i += kThreads) {
      const int t = t_lo + i / (kHeadDim / 8), o = i % (kHeadDim / 8);
      reinterpret_cast<uint4*>(c.v_sink + (size_t(u) * c.sink + size_t(p0 + t)) * d)[o] =
          reinterpret_cast<const uint4*>(vu + size_t(t) * d)[o];
    }
    if (c.vrot_b) {
      // rotated V (no sink): warp wv rotates and quantizes tokens t_lo + wv, + 8, ...
      int pm[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) pm[e] = __ldg(c.vrot_perm + 4 * lane + e);
      for (int t = t_lo + (tid >> 5); t < t_lo + tpc; t += kThreads / 32) {
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float f = bf16_bits_to_f32(__ldg(vu + size_t(t) * d + pm[e]));
          range |= out_of_range(f);
          x[e] = sanitize(f);
        }
        rotate_row(x, c.vrot_b, c.vrot_norm, c.vrot_mix, lane);
        const size_t tok = size_t(u) * c.cap + size_t(p0 + t);
        quant_v_rotated<VB>(x, c.GV, c.v_codes + tok * c.vw, c.v_sz + tok * c.vgroups, lane, range);
      }
    }
  }

  // one code word per item; items are warp-aligned (nK, nV multiples of 32)
  for (int it = tid; it < nK + nV; it += kThreads) {
    if constexpr (KB < 16) {
      if (it < nK) {
        constexpr int levels = (1 << KB) - 1;
        const int w = it % kthr, cl = (it / kthr) % sch, gi = it / (kthr * sch);
        const int ch = sch * sl + cl;
        const int64_t j = j0 + gi;
        const uint32_t* tmask = c.tail_mask + size_t(u) * c.twords;
        // side-table entries stored before group gi (groups of this commit
        // in order; the same arithmetic in every thread)
        int before = count0;
        bool cut = false;
        uint32_t gm[4];
        for (int g = 0; g < gi; ++g)
          before += group_mask(c, tmask, pwu, n_tail, g, j0 + g, c.P - before, gm, cut);
        const int kept = group_mask(c, tmask, pwu, n_tail, gi, j, c.P - before, gm, cut);
        if (cut && cl == 0 && w == 0) atomicOr(c.status, uint32_t(DKV_FLAG_CAPACITY));
        // this thread's tokens: t = w kper + e of the group, pending index
        // gi GK + t (tail slot below n_tail, else block row)
        const int tw = w * kper;
        // (a select chain, not a dynamic index: gm stays in registers)
        const int wi = tw >> 5;
        const uint32_t gw = wi == 0 ? gm[0] : (wi == 1 ? gm[1] : (wi == 2 ? gm[2] : gm[3]));
        const uint32_t mw = (gw >> (tw & 31)) & ((kper == 32 ? 0u : (1u << kper)) - 1u);
        uint32_t raw2[kper / 2];  // the tokens' bf16 bits, two per word (values are
                                  // re-derived from them, not held as floats)
        float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
        {
          // this thread's kper tokens: kper / 8 16-byte reads of its channel row
          const uint4* row = reinterpret_cast<const uint4*>(sk + cl * kPendStride + gi * GK + tw);
#pragma unroll
          for (int o = 0; o < kper / 8; ++o) {
            const uint4 x8 = row[o];
            raw2[4 * o] = x8.x;
            raw2[4 * o + 1] = x8.y;
            raw2[4 * o + 2] = x8.z;
            raw2[4 * o + 3] = x8.w;
          }
        }
        auto raw = [&](int e) { return uint16_t(raw2[e >> 1] >> (16 * (e & 1))); };
        // the values, converted once where they fit in registers (2 and 4 bits)
        float fv[kper <= 16 ? kper : 1];
        auto val_slow = [&](int e) { return sanitize(bf16_bits_to_f32(raw(e))); };
        auto val = [&](int e) {
          if constexpr (kper <= 16) return fv[e];
          else return val_slow(e);
        };
        if constexpr (kper <= 16) {
#pragma unroll
          for (int e = 0; e < kper; ++e) fv[e] = sanitize(bf16_bits_to_f32(raw(e)));
        }
#pragma unroll
        for (int e = 0; e < kper; ++e) {
          const float f = val(e);
          if (!((mw >> e) & 1u)) {
            mn = fminf(mn, f);
            mx = fmaxf(mx, f);
          }
        }
        group_minmax(mn, mx, kthr);
        if (mn > mx) mn = mx = 0.f;  // every token protected
        const GroupQuant q = make_quant(mn, mx, levels);
        uint32_t words[kwpt];
        quantize_pack<KB, kper>(val, val_slow, mw, q, levels, words);  // protected tokens: code 0
        const size_t gidx = (size_t(u) * c.nG + size_t(j)) * d + ch;
#pragma unroll
        for (int i = 0; i < kwpt; ++i) c.k_codes[gidx * c.kw + w * kwpt + i] = words[i];
        if (w == 0) c.k_sz[gidx] = q.sz;
        // protected tokens of this word: side-table entry = entries before the
        // group + protected tokens of the group before this one
        if (mw) {
          int rank = before;
#pragma unroll
          for (int ww = 0; ww < 4; ++ww)
            if (32 * ww < tw) rank += __popc(gm[ww] & (32 * ww + 32 <= tw ? 0xFFFFFFFFu
                                                                           : ((1u << (tw & 31)) - 1u)));
#pragma unroll
          for (int e = 0; e < kper; ++e) {
            if (!((mw >> e) & 1u)) continue;
            if (DKV_IN_BOUNDS(rank < c.P, c.status)) {
              c.prot_k[(size_t(u) * c.P + rank) * d + ch] = raw(e);
              if (ch == 0) c.prot_pos[size_t(u) * c.P + rank] = int32_t(j * GK + tw + e);
            }
            ++rank;
          }
        }
        if (ch == 0 && w == 0) {
          c.prot_gstart[size_t(u) * (c.nG + 1) + size_t(j) + 1] = before + kept;
          if (gi == nfull - 1) c.prot_count[u] = before + kept;
        }
        continue;
      }
    }
    if constexpr (VB < 16) {
      constexpr int levels = (1 << VB) - 1;
      const int iv = it - nK;
      const int w = iv % vthr, t = t_lo + iv / vthr;
      const int wpg = c.GV / vper;  // threads per V group
      const uint16_t* src = vu + size_t(t) * d + w * vper;
      uint32_t raw2[vper / 2];  // the channels' bf16 bits, two per word
#pragma unroll
      for (int o = 0; o < vper / 8; ++o) {
        const uint4 q8 = *reinterpret_cast<const uint4*>(src + 8 * o);
        raw2[4 * o] = q8.x;
        raw2[4 * o + 1] = q8.y;
        raw2[4 * o + 2] = q8.z;
        raw2[4 * o + 3] = q8.w;
      }
      auto bits = [&](int e) { return uint16_t(raw2[e >> 1] >> (16 * (e & 1))); };
      // the values, converted once where they fit in registers (2 and 4 bits)
      float fv[vper <= 16 ? vper : 1];
      auto val_slow = [&](int e) { return sanitize(bf16_bits_to_f32(bits(e))); };
      auto val = [&](int e) {
        if constexpr (vper <= 16) return fv[e];
        else return val_slow(e);
      };
      float mn = __int_as_float(0x7f800000), mx = -__int_as_float(0x7f800000);
#pragma unroll
      for (int e = 0; e < vper; ++e) {
        const float r = bf16_bits_to_f32(bits(e));
        range |= out_of_range(r);
        const float f = sanitize(r);
        if constexpr (vper <= 16) fv[e] = f;
        mn = fminf(mn, f);
        mx = fmaxf(mx, f);
      }
      group_minmax(mn, mx, wpg);
      const GroupQuant q = make_quant(mn, mx, levels);
      uint32_t words[vwpt];
      quantize_pack<VB, vper>(val, val_slow, 0u, q, levels, words);
      const size_t tok = size_t(u) * c.cap + size_t(p0 + t);
#pragma unroll
      for (int i = 0; i < vwpt; ++i) c.v_codes[tok * c.vw + w * vwpt + i] = words[i];
      if (w % wpg == 0) c.v_sz[tok * c.vgroups + w / wpg] = q.sz;
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

// Roll back the sequences with a trunc bit to their length ca.p0 (a multiple
// of the K group): the side table keeps the entries stored before group
// len / GK; the tail is empty.
__global__ void truncate_kernel(const __grid_constant__ CacheView c,
                                const __grid_constant__ CommitArgs ca) {
  pdl_wait();
  pdl_trigger();
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= c.U) return;
  const int sq = u / c.Hkv;
  if (!((ca.trunc[sq >> 5] >> (sq & 31)) & 1u)) return;
  c.prot_count[u] = c.prot_gstart[size_t(u) * (c.nG + 1) + ca.p0.len[sq] / c.GK];
  for (int w = 0; w < c.twords; ++w) c.tail_mask[size_t(u) * c.twords + w] = 0u;
}

template <int KB, int VB>
cudaError_t launch_kv(const CacheView& c, const uint16_t* k, const uint16_t* v,
                      const uint32_t* pw, const CommitArgs& ca, cudaStream_t s) {
  // one wave of at most four CTAs per SM (148 SMs): four slices for small batches, one for large
  const int nsl = c.U >= 296 ? 1 : (c.U >= 148 ? 2 : kMaxSlices);
  const cudaError_t e = launch_pdl(commit_kernel<KB, VB>, dim3(unsigned(c.U) * unsigned(nsl)),
                                   dim3(kThreads), 0, s, c, k, v, pw, ca, nsl);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

template <int KB>
cudaError_t launch_k(const CacheView& c, const uint16_t* k, const uint16_t* v,
                     const uint32_t* pw, const CommitArgs& ca, cudaStream_t s) {
  switch (c.vb) {
    case 2: return launch_kv<KB, 2>(c, k, v, pw, ca, s);
    case 3: return launch_kv<KB, 3>(c, k, v, pw, ca, s);
    case 4: return launch_kv<KB, 4>(c, k, v, pw, ca, s);
    default: return launch_kv<KB, 16>(c, k, v, pw, ca, s);
  }
}

}  // namespace

cudaError_t launch_truncate(const CacheView& c, const CommitArgs& ca, cudaStream_t s) {
  const cudaError_t e = launch_pdl(truncate_kernel, dim3((c.U + 127) / 128), dim3(128), 0, s, c, ca);
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
                          const uint32_t* pw, const CommitArgs& ca, cudaStream_t s) {
  switch (c.kb) {
    case 2: return launch_k<2>(c, k, v, pw, ca, s);
    case 3: return launch_k<3>(c, k, v, pw, ca, s);
    case 4: return launch_k<4>(c, k, v, pw, ca, s);
    default: return launch_k<16>(c, k, v, pw, ca, s);
  }
}

}  // namespace dkv
