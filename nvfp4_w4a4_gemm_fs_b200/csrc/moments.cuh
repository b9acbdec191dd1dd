// Exact integer channel moments of bf16 values, shared by the statistics kernel and the fused
// statistics + quantise kernel (FourSight §5.2 "running channel moments"; this library fixes them as
// s1 = sum rint(x 2^16), s2 = sum rint(x^2 2^14) over values with |x| < 2^15).
#pragma once

#include "common.cuh"

namespace fs {
namespace moments {

constexpr double kS1Scale = 65536.0;
constexpr double kS2Scale = 16384.0;
constexpr float kRangeLimit = 32768.0f;

// Exact integer moments without 64-bit conversions, branch-free, for |x| < 2^15.
//
// Magic rounding: for |t| < 2^22, fl32(t + 1.5*2^23) lies in [2^23, 2^24) where the float spacing
// is 1, so the addition rounds t to the nearest integer (ties to even) and the integer is the
// bit pattern minus that of 1.5*2^23; with 1.5*2^31 the spacing is 2^8 and the addition rounds to
// a multiple of 2^8 for |t| < 2^30.
//   s1 term rint(x*2^16) = rint(x)*2^16 + rint((x - rint(x))*2^16)   (rint(x)*2^16 is even, so
//     the split keeps ties-to-even; |x - rint(x)| <= 1/2 and both parts are exact in fp32);
//   s2 term rint(y*2^14), y = x^2 (exact for bf16 x, y < 2^30) = yh*2^14 + rint(yl*2^14) with
//     yh the multiple of 2^8 nearest y and yl = y - yh, |yl| <= 2^7 (yh*2^14 is a multiple of
//     2^22, so again the split keeps ties-to-even).
// The raw bit patterns are summed in wrapping 32-bit registers for a few rows; subtracting
// count * magic-bits recovers the exact small sums, which are then added to 64-bit totals.
constexpr float kMagic = 12582912.0f;          // 1.5 * 2^23
constexpr float kMagic8 = 3221225472.0f;       // 1.5 * 2^31 (rounds to multiples of 2^8)
constexpr uint32_t kMagicBits = 0x4B400000u;
constexpr uint32_t kMagic8Bits = 0x4F400000u;

struct SmallSums {
  uint32_t a1, b1, c2, d2;   // raw-bit sums: rint(x), rint(frac*2^16), yh/2^8, rint(yl*2^14)
  float amax;
};

__device__ __forceinline__ void add_bf16(SmallSums& a, float x, bool& bad) {
  const float ax = fabsf(x);
  const bool ok = ax < kRangeLimit;              // false for NaN too
  bad |= !ok;
  x = ok ? x : 0.0f;
  a.amax = fmaxf(a.amax, ok ? ax : 0.0f);
  const float t1 = __fadd_rn(x, kMagic);
  a.a1 += __float_as_uint(t1);
  const float frac = __fsub_rn(x, __fsub_rn(t1, kMagic));
  a.b1 += __float_as_uint(__fmaf_rn(frac, 65536.0f, kMagic));
  const float y = __fmul_rn(x, x);
  const float u = __fadd_rn(y, kMagic8);
  a.c2 += __float_as_uint(u);
  const float yl = __fsub_rn(y, __fsub_rn(u, kMagic8));
  a.d2 += __float_as_uint(__fmaf_rn(yl, 16384.0f, kMagic));
}

// Two elements of one channel at once with the packed fp32 instructions of sm_100a: each lane of
// add/sub/mul/fma.rn.f32x2 is the IEEE single-precision RN operation add_bf16 performs on an
// in-range element, in the same order, so the raw-bit terms are identical; the two lanes' bits are
// summed with one 3-input add per term.
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
  return (static_cast<uint64_t>(__float_as_uint(hi)) << 32) | __float_as_uint(lo);
}
__device__ __forceinline__ uint64_t add_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint32_t lanes_sum(uint64_t v) {
  return static_cast<uint32_t>(v) + static_cast<uint32_t>(v >> 32);
}
__device__ __forceinline__ void add_bf16_pair_in_range(uint32_t& a1, uint32_t& b1, uint32_t& c2, uint32_t& d2,
                                                       float x0, float x1) {
  constexpr uint64_t kM2 = (static_cast<uint64_t>(kMagicBits) << 32) | kMagicBits;
  constexpr uint64_t kM8x2 = (static_cast<uint64_t>(kMagic8Bits) << 32) | kMagic8Bits;
  constexpr uint64_t k2p16 = 0x4780000047800000ull;    // 65536.0f in both lanes
  constexpr uint64_t k2p14 = 0x4680000046800000ull;    // 16384.0f in both lanes
  const uint64_t X = pack_f32x2(x0, x1);
  const uint64_t T1 = add_f32x2(X, kM2);
  a1 += lanes_sum(T1);
  const uint64_t F = sub_f32x2(X, sub_f32x2(T1, kM2));
  b1 += lanes_sum(fma_f32x2(F, k2p16, kM2));
  const uint64_t Y = mul_f32x2(X, X);
  const uint64_t U = add_f32x2(Y, kM8x2);
  c2 += lanes_sum(U);
  const uint64_t YL = sub_f32x2(Y, sub_f32x2(U, kM8x2));
  d2 += lanes_sum(fma_f32x2(YL, k2p14, kM2));
}

}  // namespace moments
}  // namespace fs
