// GELU in the two forms the encoder offers, for FP32 values in registers.
// Shared by the GEMM epilogues and the single-launch small-batch forward, so
// that both apply the same function.
#pragma once

#include "sm100.cuh"

namespace enc {
namespace act {

using sm100::f2_fma;
using sm100::f2_mul;
using sm100::f2_pack;
using sm100::f2_unpack;

// GELU(v) = v * Phi(v) = 0.5 v (1 + erf(v / sqrt 2)), with erf from the
// rational approximation of Abramowitz & Stegun, Handbook of Mathematical
// Functions, formula 7.1.28: for z >= 0,
//   erf(z) = 1 - 1 / (1 + a1 z + a2 z^2 + a3 z^3 + a4 z^4 + a5 z^5 + a6 z^6)^16,
// |error| <= 3e-7, and erf(-z) = -erf(z).  The 16th power is four squarings, so
// an element costs one reciprocal (special-function unit) and a dozen FMA-pipe
// operations, which keeps the FFN1 epilogue behind its MMAs.  For large z the
// power overflows to +inf and the reciprocal gives 0, i.e. erf = 1.  The error
// is far below the FP16 rounding of the stored result.
// Two elements are evaluated at once with the packed FP32 instructions of
// sm_100 (fma/mul .f32x2): the polynomial, the squarings and the final
// scaling cost one instruction per pair; the reciprocal and the sign stay per
// element.
__device__ __forceinline__ void gelu_erf_pair(float& v0, float& v1) {
  const uint64_t v = f2_pack(v0, v1);
  const uint64_t z = f2_mul(f2_pack(fabsf(v0), fabsf(v1)), f2_pack(0.70710678118654752f, 0.70710678118654752f));
  uint64_t q = f2_fma(z, f2_pack(0.0000430638f, 0.0000430638f), f2_pack(0.0002765672f, 0.0002765672f));
  q = f2_fma(z, q, f2_pack(0.0001520143f, 0.0001520143f));
  q = f2_fma(z, q, f2_pack(0.0092705272f, 0.0092705272f));
  q = f2_fma(z, q, f2_pack(0.0422820123f, 0.0422820123f));
  q = f2_fma(z, q, f2_pack(0.0705230784f, 0.0705230784f));
  q = f2_fma(z, q, f2_pack(1.0f, 1.0f));
  q = f2_mul(q, q);
  q = f2_mul(q, q);
  q = f2_mul(q, q);
  q = f2_mul(q, q);
  float q0, q1, r0, r1;
  f2_unpack(q, q0, q1);
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(q0));
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r1) : "f"(q1));
  // erf(|z|) = 1 - r >= 0; give it the sign of v
  const uint64_t e = f2_fma(f2_pack(r0, r1), f2_pack(-1.0f, -1.0f), f2_pack(1.0f, 1.0f));
  float e0, e1;
  f2_unpack(e, e0, e1);
  e0 = copysignf(e0, v0);
  e1 = copysignf(e1, v1);
  const uint64_t hv = f2_mul(v, f2_pack(0.5f, 0.5f));
  f2_unpack(f2_fma(hv, f2_pack(e0, e1), hv), v0, v1);
}

// tanh form of GELU: 0.5 v (1 + tanh(u)), u = sqrt(2/pi) (v + 0.044715 v^3), with
// tanh(u) = 1 - 2 / (exp(2u) + 1) (one exponential and one reciprocal on the
// special-function unit; exp overflowing to +inf gives tanh = 1, underflowing
// to 0 gives -1).
__device__ __forceinline__ float gelu_tanh(float v) {
  const float u = 0.7978845608028654f * fmaf(0.044715f * v, v * v, v);
  float e, r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(u * 2.8853900817779268f));   // exp(2u) = 2^(2u log2 e)
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(e + 1.0f));
  const float th = fmaf(-2.0f, r, 1.0f);
  const float hv = 0.5f * v;
  return fmaf(hv, th, hv);
}

}  // namespace act
}  // namespace enc
