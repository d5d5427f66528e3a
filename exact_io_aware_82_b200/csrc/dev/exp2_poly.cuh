// 2^x on the FMA pipe, two values at a time, for softmax weights that are rounded to bf16
// right after (relative error 7.5e-5, about 2^-13.7, against bf16's rounding of 2^-9).
//
// The multi-function unit that runs ex2.approx has a sixteenth of the FMA pipe's throughput;
// at d = 128 one softmax exponential per score keeps it as busy as the tensor core is with the
// two products, so computing part of the exponentials here lets the two units share the work.
//
// Method (Cody-Waite range reduction, then a polynomial): x = j + f with j the integer nearest
// x (adding 1.5 * 2^23 rounds it into the low mantissa bits of t), f in [-1/2, 1/2];
// 2^f ~ c0 + f (c1 + f (c2 + f c3)); 2^j is added to the result's exponent field as
// bits(t) * 2^23, whose low 32 bits are j * 2^23 because bits(t) = 0x4B400000 + j.  The
// coefficients minimise the largest relative error on [-1/2, 1/2] (Lawson's algorithm on
// Chebyshev nodes, fp32), as fit_exp2_poly.py computes and tests/test_exp2_poly.py checks.
// x is clamped at -126 so that j never takes the exponent below its field; an input of -inf
// therefore gives about 2^-126, not 0: callers use it only on scores no mask has removed.
#pragma once

#include <cstdint>

namespace attn {
namespace dev {

constexpr float kExp2C0 = 9.999280572e-01f;
constexpr float kExp2C1 = 6.932609677e-01f;
constexpr float kExp2C2 = 2.426111251e-01f;
constexpr float kExp2C3 = 5.517166853e-02f;

__device__ __forceinline__ uint64_t pack2(float a, float b) {
  uint64_t x;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(a), "f"(b));
  return x;
}
__device__ __forceinline__ float2 unpack2(uint64_t x) {
  float2 r;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(x));
  return r;
}
// a * b + c and a + b, element-wise on two fp32 values (one instruction each on sm_100)
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t add2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t sub2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// 2^x for both halves of x (packed pair); see the header comment for the method and range.
__device__ __forceinline__ float2 exp2_poly2(uint64_t x) {
  float2 xc = unpack2(x);
  xc.x = fmaxf(xc.x, -126.f);
  xc.y = fmaxf(xc.y, -126.f);
  const uint64_t xs = pack2(xc.x, xc.y);
  const uint64_t magic = pack2(12582912.f, 12582912.f);
  const uint64_t t = add2(xs, magic);  // 1.5 * 2^23 + j
  const uint64_t f = sub2(xs, sub2(t, magic));
  uint64_t p = fma2(f, pack2(kExp2C3, kExp2C3), pack2(kExp2C2, kExp2C2));
  p = fma2(p, f, pack2(kExp2C1, kExp2C1));
  p = fma2(p, f, pack2(kExp2C0, kExp2C0));
  const float2 tt = unpack2(t), pp = unpack2(p);
  float2 r;
  r.x = __uint_as_float(__float_as_uint(tt.x) * (1u << 23) + __float_as_uint(pp.x));
  r.y = __uint_as_float(__float_as_uint(tt.y) * (1u << 23) + __float_as_uint(pp.y));
  return r;
}

}  // namespace dev
}  // namespace attn
