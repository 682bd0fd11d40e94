// swiglu_math.cuh -- fp32 arithmetic of the fused SwiGLU activation (device code).
//
// The exponential is the library's own fixed sequence (the quantized output must be
// reproducible bit for bit by a CPU implementation of the same steps), so no vendor math
// function is called. Everything works on pairs with the packed fp32x2 instructions, which
// give each lane the IEEE result of the scalar operation.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {

// Library exponential e(v) on a pair: clamp v to [-87, 88]; k = the integer nearest the
// exact product v * fl(log2 e), ties to even; Cody-Waite reduction f = v - k*ln2_hi -
// k*ln2_lo; degree-7 Taylor polynomial p of e^f (coefficients 1/n! rounded to fp32) by fused
// multiply-add; result p * 2^k.
//  * k comes from one FMA, t = v * fl(log2 e) + 1.5*2^23: for |v * log2 e| < 2^22 the fused
//    sum rounds the exact product to an integer with ties to even, and -k = 1.5*2^23 - t
//    exactly.
//  * p * 2^k is formed by adding k to p's exponent field: bits(t) * 2^23 = k * 2^23 modulo
//    2^32 (bits(t) = 0x4B400000 + k, and 0x4B400000 * 2^23 = 0 mod 2^32), and on the
//    clamped range p * 2^k is a normal number (e^-87 > 2^-126, e^88 < 2^128), where the
//    product by a power of two is exact, so the integer add gives the product's bits.
// CLAMP = false skips the clamp; callers use it only when every v of the pair is NaN or lies
// in [-87, 87] already.
template <bool CLAMP>
__device__ __forceinline__ F2 exp_pair(F2 v) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  if constexpr (CLAMP) {
    v.x = fminf(fmaxf(v.x, -87.0f), 88.0f);
    v.y = fminf(fmaxf(v.y, -87.0f), 88.0f);
  }
  const F2 t = fma2_rn(v, F2{0x1.715476p+0f, 0x1.715476p+0f}, F2{kRound, kRound});
  const F2 nk = add2f_rn(F2{kRound, kRound}, F2{-t.x, -t.y});
  F2 f = fma2_rn(nk, F2{0x1.62e4p-1f, 0x1.62e4p-1f}, v);
  f = fma2_rn(nk, F2{0x1.7f7d1cp-20f, 0x1.7f7d1cp-20f}, f);
  F2 p{0x1.a01a02p-13f, 0x1.a01a02p-13f};                   // 1/7!
  p = fma2_rn(p, f, F2{0x1.6c16c2p-10f, 0x1.6c16c2p-10f});  // 1/6!
  p = fma2_rn(p, f, F2{0x1.111112p-7f, 0x1.111112p-7f});    // 1/5!
  p = fma2_rn(p, f, F2{0x1.555556p-5f, 0x1.555556p-5f});    // 1/4!
  p = fma2_rn(p, f, F2{0x1.555556p-3f, 0x1.555556p-3f});    // 1/3!
  p = fma2_rn(p, f, F2{0.5f, 0.5f});                        // 1/2!
  p = fma2_rn(p, f, F2{1.0f, 1.0f});                        // 1/1!
  p = fma2_rn(p, f, F2{1.0f, 1.0f});                        // 1/0!
  return F2{__uint_as_float(__float_as_uint(t.x) * 8388608u + __float_as_uint(p.x)),
            __uint_as_float(__float_as_uint(t.y) * 8388608u + __float_as_uint(p.y))};
}

// Quotient a / b for a pair, given v = -a and 1 <= b < 2^128, from the hardware reciprocal
// approximation and one residual correction (Markstein's FMA quotient refinement, IBM J.
// Res. Dev. 34(1), 1990): ny ~ -1/b, q0 = v*ny (= a*(1/b) up to rounding), e = q0*b - a
// (exact by FMA), q1 = q0 - e/b taken as q0 + e*ny. The flush-to-zero form of the
// reciprocal is used: with SCALED it is taken of b * 2^-32 (a normal number) and scaled back
// by 2^-32, which covers b up to 2^128; without, b must stay below 2^126 so 1/b is normal.
// Taking the residual with this sign keeps the quotient of a signed zero signed. An
// infinite dividend makes e NaN; SAFE then returns q0 (= +-inf, the quotient) in that lane,
// and callers that know every dividend is finite (or NaN) skip that select.
template <bool SCALED, bool SAFE>
__device__ __forceinline__ F2 div_pair(F2 v, F2 b) {
  F2 ny;
  if constexpr (SCALED) {
    const F2 bs = mul2f_rn(b, F2{-0x1p-32f, -0x1p-32f});
    F2 y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.x) : "f"(bs.x));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.y) : "f"(bs.y));
    ny = mul2f_rn(y, F2{0x1p-32f, 0x1p-32f});
  } else {
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(ny.x) : "f"(-b.x));
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(ny.y) : "f"(-b.y));
  }
  const F2 q0 = mul2f_rn(v, ny);
  const F2 e = fma2_rn(q0, b, v);
  const F2 q1 = fma2_rn(e, ny, q0);
  if constexpr (SAFE) return F2{e.x == e.x ? q1.x : q0.x, e.y == e.y ? q1.y : q0.y};
  return q1;
}

// silu(gate) = gate / (1 + e(-gate)) for a pair, from v = -gate. The division forms are
// used only where the divisor is den = 1 + e(-gate) for a 16-bit gate, a set of 2^16 values
// per input type; a GPU test runs every bf16 and fp16 gate through each form on the gates
// it is used for and compares silu with the oracle's IEEE quotient.
//   CLAMP = false, SAFE = false: every gate NaN or |gate| <= 87 (then den <= 1 + e(87) <
//                                2^126 and the reciprocal needs no scaling)
//   CLAMP = true,  SAFE = false: every gate finite or NaN
//   CLAMP = true,  SAFE = true : any gate
template <bool CLAMP, bool SAFE>
__device__ __forceinline__ F2 silu_pair_neg(F2 v) {
  const F2 den = add2f_rn(F2{1.0f, 1.0f}, exp_pair<CLAMP>(v));
  return div_pair<CLAMP, SAFE>(v, den);
}

// Two packed 16-bit inputs -> their negations as two fp32 (exact).
template <int DTYPE>
__device__ __forceinline__ F2 unpack2_neg(uint32_t w) {
  if constexpr (DTYPE == 0) {  // bfloat16: the upper half of an fp32, sign bit flipped
    return F2{__uint_as_float(w * 65536u + 0x80000000u), __uint_as_float((w & 0xFFFF0000u) ^ 0x80000000u)};
  } else {
    F2 r;
    unpack2<1>(w ^ 0x80008000u, r.x, r.y);
    return r;
  }
}

}  // namespace nvfp4
