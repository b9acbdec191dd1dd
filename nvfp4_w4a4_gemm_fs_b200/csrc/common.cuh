// Shared host/device helpers of the SpliceGEMM library (sm_100a).
//
// Host side: status/last-error bookkeeping and argument checks.
// Device side: the NVFP4 block-quantiser arithmetic of FourSight §9.3.1 Eq. 9 and §5.1
// "Data preparation", written so that every rounding decision matches the IEEE fp32
// operation order the library documents (t = fl32(fl32(a_b*g)/6), v = fl32(fl32(x*g)/sf)).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <cstdarg>
#include <cstdio>
#include <string>
#include <algorithm>

#include "foursight.h"
#include "per_device.h"

namespace fs {

// ------------------------------------------------------------------------------------------
// Host: status handling
// ------------------------------------------------------------------------------------------
void set_last_error(const char* fmt, ...);
fs_status fail(fs_status s, const char* fmt, ...);
fs_status cuda_status(cudaError_t e, const char* what);

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }
inline int side_cols(int p) { return (p + 15) / 16 * 16; }
inline int64_t sf_bytes(int64_t rows, int K) { return round_up(rows, 128) * round_up(K / 16, 4); }
// Index of the current device (cudaGetDevice), -1 if it cannot be read.
int current_device();
// Streaming multiprocessors of the current device (queried once per device).
int sm_count();
// Sets a kernel's dynamic shared-memory limit once per device (the attribute belongs to the
// device's context); `cache` is the caller's static per-device flag.
fs_status set_max_dynamic_smem(PerDevice<int>& cache, const void* kernel, int bytes, const char* who);

#define FS_CHECK_LAUNCH(what)                                         \
  do {                                                                \
    cudaError_t e_ = cudaGetLastError();                              \
    if (e_ != cudaSuccess) return ::fs::cuda_status(e_, what);        \
  } while (0)

// Device error words written by kernels whose bounded waits gave up.
enum : uint32_t { ERR_NONE = 0, ERR_TIMEOUT = 1 };

// ------------------------------------------------------------------------------------------
// Device: small numeric helpers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Round-to-nearest-even float -> bf16 bits.
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  __nv_bfloat16 h = __float2bfloat16_rn(x);
  return *reinterpret_cast<uint16_t*>(&h);
}

// UE4M3 code of a finite t >= 0: round to nearest, ties to the even code, saturating at 448.
// Subnormals are multiples of 2^-9 below 2^-6; normals carry 3 mantissa bits, exponent bias 7.
__device__ __forceinline__ uint32_t ue4m3_rne(float t) {
  if (t >= 448.0f) return 0x7Eu;
  if (t < 0.015625f) return static_cast<uint32_t>(__float2int_rn(t * 512.0f));  // 0..8 (8 == 2^-6)
  uint32_t b = __float_as_uint(t);
  b += 0x7FFFFu + ((b >> 20) & 1u);            // round the 23-bit fraction to 3 bits, ties to even
  const uint32_t c = (((b >> 23) - 120u) << 3) | ((b >> 20) & 7u);
  return c > 0x7Eu ? 0x7Eu : c;
}

// Value of a UE4M3 code (0x00..0x7E).
__device__ __forceinline__ float ue4m3_value(uint32_t c) {
  const uint32_t e = c >> 3, m = c & 7u;
  if (e == 0) return static_cast<float>(m) * 0.001953125f;                       // m * 2^-9
  return __uint_as_float(((e + 120u) << 23) | (m << 20));                        // (1+m/8) 2^(e-7)
}

// Exact quotient rounding for divisors with at most 4 significant bits.
//
// For q = y / d with y an fp32 value and d = o * 2^k (o odd, o <= 15), RN32(q) equals
// RN32(RN64(y * RN64(1/d))).  Reason: the float64 product is within 2^-52 |q| of q, while q
// either is exactly an fp32 value or lies at least 2^-28 |q| away from every fp32 rounding
// midpoint (y has 24 significant bits, so y - M*d, for an fp32 midpoint M with 25 bits, is a
// non-zero multiple of M's last unit unless y/d == M, which would need y to span more than
// 24 bits).  The fp64 error therefore never moves the result across a rounding boundary.
// Used for the per-block step t = fl32(a_b*g)/6 (6 = 3*2).
__device__ __forceinline__ float div_small_divisor(float y, double inv_d) {
  return __double2float_rn(__dmul_rn(static_cast<double>(y), inv_d));
}
constexpr double kInvSix = 1.0 / 6.0;   // RN64(1/6): compile-time IEEE division

// Correctly rounded y / d in fp32 by Markstein's correction (P. Markstein, "Computation of
// elementary functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990):
// with r = RN(1/d), a quotient q within one ulp of y/d and the remainder e = y - d*q (exact when
// formed by one fused multiply-add), RN(q + e*r) is the correctly rounded quotient.  The first
// correction brings q0 = RN(y*r) within one ulp; the second rounds correctly.  Used per element
// (v = fl32(x*g) / sf), where it replaces an IEEE division by five fp32 operations.  Requires
// finite y and d > 0 (d = 1, r = 0 yields +-0 with the sign of y, the zero-scale rule).  The
// quotient takes the sign of y explicitly: for y = -0 the remainder y - d*q0 = (-0) + (+0) is +0, and the
// corrections would otherwise return +0.
__device__ __forceinline__ float div_markstein(float y, float d, float r) {
  const float q0 = __fmul_rn(y, r);
  const float e0 = __fmaf_rn(-q0, d, y);
  const float q1 = __fmaf_rn(e0, r, q0);
  const float e1 = __fmaf_rn(-q1, d, y);
  const float q2 = __fmaf_rn(e1, r, q1);
  return __uint_as_float((__float_as_uint(q2) & 0x7FFFFFFFu) | (__float_as_uint(y) & 0x80000000u));
}

// Fast path of v = fl32(fl32(x*g)/sf) for the E2M1 decision, valid for bf16 x (at most 8
// significant bits), a power-of-two g in [2^-100, 2^100] and a UE4M3 scale sf (at most 4
// significant bits; sf_rcp = RN(1/sf), or 0 for the zero scale).
//
// The E2M1 code depends only on where q = x*g/sf lies relative to the rounding midpoints
// mu/4, mu in {1,3,5,7,10,14,20}.  x*g - (mu/4)*sf is a difference of an 8-bit and a 7-bit
// integer multiple of powers of two, so unless it is zero, |q - mu/4| >= 2^-8.3 * mu/4.
// q' = RN(x * RN(g*sf_rcp)) is within 2^-22.9 of q, relatively, and rounding q' to 12
// significant bits returns mu/4 exactly when q == mu/4 (a tie, which the E2M1 conversion then
// breaks to even) and moves no other value across a midpoint.  The fp32 rounding of q in the
// exact formula cannot create a tie either (q is at least 2^-8.3 away), so both give the same
// code, the sign of zero included (the rounding keeps the sign bit).
__device__ __forceinline__ float snap12(float v) {
  return __uint_as_float((__float_as_uint(v) + 0x800u) & 0xFFFFF000u);
}
__device__ __forceinline__ bool pow2_gain_in_fast_range(float g) {
  const uint32_t b = __float_as_uint(g);
  const uint32_t e = b >> 23;                   // g > 0 here, sign bit clear
  return (b & 0x7FFFFFu) == 0 && e >= 127u - 100u && e <= 127u + 100u;
}

// Packs two fp32 values into one byte of E2M1 codes (round to nearest even, saturating at 6),
// `lo` into the low nibble.  The PTX conversion places its first source in the high nibble.
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %2;\n\tcvt.u32.u8 %0, t;\n\t}"
      : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Packs eight fp32 values into one 32-bit word of E2M1 codes (element 0 in the low nibble).
__device__ __forceinline__ uint32_t e2m1x8(float v0, float v1, float v2, float v3, float v4, float v5, float v6,
                                           float v7) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r) : "f"(v0), "f"(v1), "f"(v2), "f"(v3), "f"(v4), "f"(v5), "f"(v6), "f"(v7));
  return r;
}

// Power-of-two encode gain: largest g = 2^E with amax*g <= 2688 = 0.65625*2^12, E clamped to
// [-126,127]; 1 for amax == 0 or non-finite.  With amax = f*2^e, f in [0.5,1): E = 12-e when
// f <= 0.65625, else 11-e.
__device__ __forceinline__ float gain_pow2(float amax) {
  if (!(amax > 0.0f) || !isfinite(amax)) return 1.0f;
  uint32_t b = __float_as_uint(amax);
  int bias = 0;
  if ((b >> 23) == 0) {                         // subnormal: scale by 2^64 first (exact)
    b = __float_as_uint(amax * 18446744073709551616.0f);
    bias = 64;
  }
  const int e = static_cast<int>(b >> 23) - 126 - bias;     // amax = f * 2^e, f in [0.5, 1)
  const uint32_t frac = b & 0x7FFFFFu;                       // f = (1 + frac/2^23) / 2
  int E = (frac <= 0x280000u) ? 12 - e : 11 - e;             // f <= 0.65625 <=> frac <= 0.3125*2^23
  E = E < -126 ? -126 : (E > 127 ? 127 : E);
  return __uint_as_float(static_cast<uint32_t>(E + 127) << 23);
}

// fl32(2688/amax) saturated to the largest finite float (the quotient overflows for every
// subnormal amax); 1 for amax == 0 or non-finite.
__device__ __forceinline__ float gain_exact(float amax) {
  if (!(amax > 0.0f) || !isfinite(amax)) return 1.0f;
  return fminf(__fdiv_rn(2688.0f, amax), 3.40282346638528859812e+38f);
}

// Byte offset of (row r, 16-block b) in the tiled scale array; kb4 = roundup(K/16,4)/4.
__device__ __host__ __forceinline__ int64_t sf_offset(int64_t r, int b, int kb4) {
  return ((r >> 7) * kb4 + (b >> 2)) * 512 + (r & 31) * 16 + ((r & 127) >> 5) * 4 + (b & 3);
}

// Bounded spin limit shared by the kernels that wait on barriers (about a second at 2 GHz).
constexpr uint32_t kSpinLimit = 1u << 28;

}  // namespace fs
