// Arithmetic building blocks for sm_100a written for throughput: packed
// two-lane fp32 operations (fma/add/mul .f32x2, two results per instruction),
// the three-input maximum, 2^x on the FMA pipe, and the register layouts of
// the warp-wide TMEM loads used for column sums.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace avq {
namespace fm {

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }

// max(a, b, c) in one instruction (PTX max.f32 with three sources, sm_100+).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x for two values on the FMA pipe instead of the special-function unit.
// Range reduction to the nearest integer (Cody and Waite): j = round(x) by
// adding and subtracting 1.5 * 2^23 (exact round-to-nearest for |x| < 2^22),
// f = x - j in [-1/2, 1/2]; 2^f by a cubic whose coefficients were fitted to
// minimise the largest relative error on [-1/2, 1/2] (Lawson's iteratively
// reweighted least squares): 7.5e-5.  2^j is then added to the exponent
// field as an integer, j * 2^23 (the rounding constant's own high bits fall
// off the top of the 32-bit word).  Inputs below -126 are clamped there, so
// that the exponent field of the result never goes below zero (j >= -126 and
// 2^f >= 2^-1/2 keep it at 0 or above: a non-negative number below 2^-125);
// inputs must stay below 127.5.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  x.x = fmaxf(x.x, -126.0f);
  x.y = fmaxf(x.y, -126.0f);
  const float2 j = add2(x, f2(kRound, kRound));
  const float2 jf = add2(j, f2(-kRound, -kRound));
  const float2 f = add2(x, f2(-jf.x, -jf.y));
  float2 p = fma2(f2(0.05517166493f, 0.05517166493f), f, f2(0.24261112188f, 0.24261112188f));
  p = fma2(p, f, f2(0.69326098622f, 0.69326098622f));
  p = fma2(p, f, f2(0.99992807358f, 0.99992807358f));
  const uint32_t r0 = __float_as_uint(p.x) + (__float_as_uint(j.x) << 23);
  const uint32_t r1 = __float_as_uint(p.y) + (__float_as_uint(j.y) << 23);
  return f2(__uint_as_float(r0), __uint_as_float(r1));
}

// tcgen05.ld of shape 16x256b, 4 repetitions: 16 TMEM lanes x 32 columns.
// Thread t of the warp receives, for repetition k (columns 8k .. 8k+7):
//   r[4k + 0], r[4k + 1]: lane (t / 4),     columns 8k + 2 (t % 4) + {0, 1}
//   r[4k + 2], r[4k + 3]: lane (t / 4) + 8, the same two columns
// (lanes relative to the 16-lane base in the address).
__device__ __forceinline__ void tmem_ld_16x256b_x4(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

}  // namespace fm
}  // namespace avq
