// swiglu_math.cuh -- fp32 arithmetic of the fused SwiGLU activation (device code).
//
// The exponential is the library's own fixed sequence (the quantized output must be
// reproducible bit for bit by a CPU implementation of the same steps), so no vendor math
// function is called.
#pragma once

#include "ptx.cuh"

namespace nvfp4 {

// Library fp32 exponential on a pair of values: clamp to [-87, 88]; k = rint(v * log2 e);
// Cody-Waite reduction f = v - k*ln2_hi - k*ln2_lo; degree-7 Taylor polynomial of e^f
// (coefficients 1/n! rounded to fp32) by fused multiply-add; times 2^k built from exponent
// bits. Packed fp32x2 instructions give each lane the same IEEE results as scalar code.
// rint is taken as (z + 1.5*2^23) - 1.5*2^23: for |z| < 2^22 the sum is rounded to an
// integer with ties to even, which is exactly rint(z), and its low mantissa bits are k.
__device__ __forceinline__ F2 exp2_f32(F2 v) {
  constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
  v.x = fminf(fmaxf(v.x, -87.0f), 88.0f);
  v.y = fminf(fmaxf(v.y, -87.0f), 88.0f);
  const F2 z = mul2f_rn(v, F2{0x1.715476p+0f, 0x1.715476p+0f});
  const F2 t = add2f_rn(z, F2{kRound, kRound});
  const F2 k = add2f_rn(t, F2{-kRound, -kRound});
  const F2 nk{-k.x, -k.y};
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
  // 2^k: k sits in the low bits of t (t's bits = 0x4B400000 + k), so (k + 127) << 23 is
  // (bits(t) - 0x4B400000 + 127) << 23 = bits(t) * 2^23 - 0x4B3FFF81 * 2^23 (mod 2^32),
  // one integer multiply-add.
  constexpr uint32_t kBias = 0x4B3FFF81u << 23;
  const F2 two_k{__uint_as_float(__float_as_uint(t.x) * 8388608u - kBias),
                 __uint_as_float(__float_as_uint(t.y) * 8388608u - kBias)};
  return mul2f_rn(p, two_k);
}

// Quotient a / b for a pair, given v = -a and 1 <= b < 2^128, from the hardware reciprocal
// approximation and one residual correction (Markstein's FMA quotient refinement, IBM J.
// Res. Dev. 34(1), 1990): ny ~ -1/b, q0 = v*ny (= a*(1/b) up to rounding), e = q0*b - a
// (exact by FMA), q1 = q0 - e/b taken as q0 + e*ny. The reciprocal is taken of b * 2^-32,
// which is a normal number, so the flush-to-zero form of the instruction applies, and scaled
// back by 2^-32. Taking the residual with this sign keeps the quotient of a signed zero
// signed. An infinite dividend makes e NaN; SAFE then returns q0 (= +-inf, the quotient) in
// that lane, and callers that know every dividend is finite (or NaN) skip that select.
// It is used only where the divisor is den = 1 + e(-gate) for a 16-bit gate, a set of 2^16
// values per input type; a GPU test runs every bf16 and fp16 gate through both forms and
// compares silu with the oracle's IEEE quotient.
template <bool SAFE>
__device__ __forceinline__ F2 div2_rcp_fma(F2 v, F2 b) {
  const F2 bs = mul2f_rn(b, F2{-0x1p-32f, -0x1p-32f});
  F2 y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.x) : "f"(bs.x));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y.y) : "f"(bs.y));
  const F2 ny = mul2f_rn(y, F2{0x1p-32f, 0x1p-32f});
  const F2 q0 = mul2f_rn(v, ny);
  const F2 e = fma2_rn(q0, b, v);
  const F2 q1 = fma2_rn(e, ny, q0);
  if constexpr (SAFE) return F2{e.x == e.x ? q1.x : q0.x, e.y == e.y ? q1.y : q0.y};
  return q1;
}

// silu(gate) = gate / (1 + e(-gate)) for a pair of elements. SAFE = false requires both
// gates finite or NaN (no infinity).
template <bool SAFE>
__device__ __forceinline__ F2 silu2_f32(F2 gate) {
  const F2 v{-gate.x, -gate.y};
  const F2 den = add2f_rn(F2{1.0f, 1.0f}, exp2_f32(v));
  return div2_rcp_fma<SAFE>(v, den);
}

// y = silu(gate) * up for a pair of elements.
template <bool SAFE>
__device__ __forceinline__ F2 swiglu2_f32(F2 gate, F2 up) { return mul2f_rn(silu2_f32<SAFE>(gate), up); }

}  // namespace nvfp4
