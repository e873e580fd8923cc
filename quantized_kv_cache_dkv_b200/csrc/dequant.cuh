// Packed-code -> fp16 conversion used by the attention kernels.
//
// A 4-bit word holds 8 codes (element e at bits 4e), a 2-bit word 16 codes
// (element e at bits 2e).  Codes are moved into the low mantissa bits of the
// fp16 constant 1024 (bit pattern 0x6400, whose ulp is 1), giving 1024 + c or
// 1024 + 2^k c exactly; one fp16 fma removes the offset and the 2^k factor
// exactly, and a second fp16 fma gives q * s + z with a single rounding.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace dkv {

__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t mask, uint32_t bits) {
  uint32_t r;  // (a & mask) | bits
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "r"(mask), "r"(bits));
  return r;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
  return r;
}

__device__ __forceinline__ __half2 u2h(uint32_t x) { return *reinterpret_cast<__half2*>(&x); }
__device__ __forceinline__ uint32_t h2u(__half2 x) { return *reinterpret_cast<uint32_t*>(&x); }

__device__ __forceinline__ __half2 h2c(float a) { return __float2half2_rn(a); }

constexpr uint32_t kMagic1024 = 0x64006400u;

// (1024 + 2^k c) -> c, exactly
__device__ __forceinline__ __half2 unbias(uint32_t x, float inv, float off) {
  return __hfma2(u2h(x), h2c(inv), h2c(off));
}

// 8 four-bit codes -> 8 halves q*s+z, element order
__device__ __forceinline__ uint4 dequant4x8(uint32_t w, __half2 s2, __half2 z2) {
  const uint32_t w8 = w >> 8;
  const __half2 n04 = unbias(and_or(w, 0x000F000Fu, kMagic1024), 1.f, -1024.f);
  const __half2 n15 = unbias(and_or(w, 0x00F000F0u, kMagic1024), 0.0625f, -64.f);
  const __half2 n26 = unbias(and_or(w8, 0x000F000Fu, kMagic1024), 1.f, -1024.f);
  const __half2 n37 = unbias(and_or(w8, 0x00F000F0u, kMagic1024), 0.0625f, -64.f);
  const uint32_t v04 = h2u(__hfma2(n04, s2, z2));
  const uint32_t v15 = h2u(__hfma2(n15, s2, z2));
  const uint32_t v26 = h2u(__hfma2(n26, s2, z2));
  const uint32_t v37 = h2u(__hfma2(n37, s2, z2));
  uint4 r;
  r.x = prmt(v04, v15, 0x5410);  // e0 e1
  r.y = prmt(v26, v37, 0x5410);  // e2 e3
  r.z = prmt(v04, v15, 0x7632);  // e4 e5
  r.w = prmt(v26, v37, 0x7632);  // e6 e7
  return r;
}

// 16 two-bit codes -> 16 halves q*s+z, element order (lo = e0..e7, hi = e8..e15)
__device__ __forceinline__ void dequant2x16(uint32_t w, __half2 s2, __half2 z2, uint4& lo,
                                            uint4& hi) {
  const uint32_t w8 = w >> 8;
  uint32_t v[8];
  v[0] = h2u(__hfma2(unbias(and_or(w, 0x00030003u, kMagic1024), 1.f, -1024.f), s2, z2));
  v[1] = h2u(__hfma2(unbias(and_or(w, 0x000C000Cu, kMagic1024), 0.25f, -256.f), s2, z2));
  v[2] = h2u(__hfma2(unbias(and_or(w, 0x00300030u, kMagic1024), 0.0625f, -64.f), s2, z2));
  v[3] = h2u(__hfma2(unbias(and_or(w, 0x00C000C0u, kMagic1024), 0.015625f, -16.f), s2, z2));
  v[4] = h2u(__hfma2(unbias(and_or(w8, 0x00030003u, kMagic1024), 1.f, -1024.f), s2, z2));
  v[5] = h2u(__hfma2(unbias(and_or(w8, 0x000C000Cu, kMagic1024), 0.25f, -256.f), s2, z2));
  v[6] = h2u(__hfma2(unbias(and_or(w8, 0x00300030u, kMagic1024), 0.0625f, -64.f), s2, z2));
  v[7] = h2u(__hfma2(unbias(and_or(w8, 0x00C000C0u, kMagic1024), 0.015625f, -16.f), s2, z2));
  // v[i] = (e_i, e_{i+8})
  lo.x = prmt(v[0], v[1], 0x5410);
  lo.y = prmt(v[2], v[3], 0x5410);
  lo.z = prmt(v[4], v[5], 0x5410);
  lo.w = prmt(v[6], v[7], 0x5410);
  hi.x = prmt(v[0], v[1], 0x7632);
  hi.y = prmt(v[2], v[3], 0x7632);
  hi.z = prmt(v[4], v[5], 0x7632);
  hi.w = prmt(v[6], v[7], 0x7632);
}

// The same conversions without the element reordering (no prmt): 4-bit
// halves come out as (e0, e4), (e1, e5), (e2, e6), (e3, e7); 2-bit halves as
// a = (e0, e8), (e1, e9), (e2, e10), (e3, e11) and b = (e4, e12), ...,
// (e7, e15).  A tile stored in this order holds its tokens permuted within
// groups of 8 (4-bit) or 16 (2-bit) tokens.
__device__ __forceinline__ uint4 dequant4x8_raw(uint32_t w, __half2 s2, __half2 z2) {
  const uint32_t w8 = w >> 8;
  uint4 r;
  r.x = h2u(__hfma2(unbias(and_or(w, 0x000F000Fu, kMagic1024), 1.f, -1024.f), s2, z2));
  r.y = h2u(__hfma2(unbias(and_or(w, 0x00F000F0u, kMagic1024), 0.0625f, -64.f), s2, z2));
  r.z = h2u(__hfma2(unbias(and_or(w8, 0x000F000Fu, kMagic1024), 1.f, -1024.f), s2, z2));
  r.w = h2u(__hfma2(unbias(and_or(w8, 0x00F000F0u, kMagic1024), 0.0625f, -64.f), s2, z2));
  return r;
}

__device__ __forceinline__ void dequant2x16_raw(uint32_t w, __half2 s2, __half2 z2, uint4& a,
                                                uint4& b) {
  const uint32_t w8 = w >> 8;
  a.x = h2u(__hfma2(unbias(and_or(w, 0x00030003u, kMagic1024), 1.f, -1024.f), s2, z2));
  a.y = h2u(__hfma2(unbias(and_or(w, 0x000C000Cu, kMagic1024), 0.25f, -256.f), s2, z2));
  a.z = h2u(__hfma2(unbias(and_or(w, 0x00300030u, kMagic1024), 0.0625f, -64.f), s2, z2));
  a.w = h2u(__hfma2(unbias(and_or(w, 0x00C000C0u, kMagic1024), 0.015625f, -16.f), s2, z2));
  b.x = h2u(__hfma2(unbias(and_or(w8, 0x00030003u, kMagic1024), 1.f, -1024.f), s2, z2));
  b.y = h2u(__hfma2(unbias(and_or(w8, 0x000C000Cu, kMagic1024), 0.25f, -256.f), s2, z2));
  b.z = h2u(__hfma2(unbias(and_or(w8, 0x00300030u, kMagic1024), 0.0625f, -64.f), s2, z2));
  b.w = h2u(__hfma2(unbias(and_or(w8, 0x00C000C0u, kMagic1024), 0.015625f, -16.f), s2, z2));
}

// Four three-bit codes at bits 0-2, 3-5, 6-8 and 9-11 of t -> two pairs of
// halves q*s+z, (c0, c1) and (c2, c3).  t << 13 brings c1 to bits 16-18 and
// c3 to bits 22-24, so one mask-and-or per pair forms 1024 + c0 | 1024 + c1
// and 1024 + 64 c2 | 1024 + 64 c3 (exact in fp16); the unbias fma removes the
// offset and the factor 64 exactly, and the second fma gives q*s+z with one
// rounding.
__device__ __forceinline__ void dequant3x4(uint32_t t, __half2 s2, __half2 z2, uint32_t& p01,
                                           uint32_t& p23) {
  const uint32_t t13 = t << 13;
  const uint32_t a = and_or(t13, 0x00070000u, and_or(t, 0x00000007u, kMagic1024));
  const uint32_t b = and_or(t13, 0x01C00000u, and_or(t, 0x000001C0u, kMagic1024));
  p01 = h2u(__hfma2(unbias(a, 1.f, -1024.f), s2, z2));
  p23 = h2u(__hfma2(unbias(b, 0.015625f, -16.f), s2, z2));
}

// 32 three-bit codes packed little-endian into the 96-bit stream w2:w1:w0
// (code e at bits 3e; codes 10 and 21 straddle two words) -> 32 halves q*s+z
// in element order (out[k] = e 8k..8k+7).  Codes 4g..4g+3 sit at stream bits
// 12g..12g+11, which a shift (a funnel shift across a word boundary) moves to
// bits 0-11.
__device__ __forceinline__ void dequant3x32(uint32_t w0, uint32_t w1, uint32_t w2, __half2 s2,
                                            __half2 z2, uint4 (&out)[4]) {
  const uint32_t t[8] = {w0,      w0 >> 12, __funnelshift_r(w0, w1, 24), w1 >> 4,
                         w1 >> 16, __funnelshift_r(w1, w2, 28), w2 >> 8, w2 >> 20};
  uint32_t p[16];
#pragma unroll
  for (int g = 0; g < 8; ++g) dequant3x4(t[g], s2, z2, p[2 * g], p[2 * g + 1]);
#pragma unroll
  for (int k = 0; k < 4; ++k) out[k] = make_uint4(p[4 * k], p[4 * k + 1], p[4 * k + 2], p[4 * k + 3]);
}

// 8 bf16 -> 8 fp16 (exact inside fp16's normal range)
__device__ __forceinline__ uint4 bf16x8_to_f16x8(uint4 x) {
  auto cvt = [](uint32_t w) -> uint32_t {
    const float a = __uint_as_float(w << 16);
    const float b = __uint_as_float(w & 0xFFFF0000u);
    return h2u(__floats2half2_rn(a, b));
  };
  uint4 r;
  r.x = cvt(x.x);
  r.y = cvt(x.y);
  r.z = cvt(x.z);
  r.w = cvt(x.w);
  return r;
}

__device__ __forceinline__ __half bf16_to_half(uint16_t b) {
  return __float2half_rn(__uint_as_float(uint32_t(b) << 16));
}

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace dkv
