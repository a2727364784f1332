// SwiGLU activation of the fused expert FFN: h = silu(gate) * up with
// silu(g) = g / (1 + exp(-g)), evaluated in fp32 from bf16 gate and up values
// and rounded once to bf16. (The "Mega MoE" kernel fuses both expert GEMMs
// with the SwiGLU activation: "DeepGEMM" overview, section "swapAB与Mega MoE";
// the pages give no formula, this is the standard definition.)
//
// exp is one fixed sequence of IEEE fp32 operations, so that the result does
// not depend on a math library: the argument is clamped to [-87, 88], reduced
// by Cody and Waite's method ("Software Manual for the Elementary Functions",
// 1980): n = nearest integer to x * log2(e), r = x - n * ln2 with ln2 split
// into 355/512 (so that n * 355/512 is exact) and its remainder, then
// exp(r) = sum_{k<=7} r^k / k! by Horner's rule with fused multiply-adds, and
// the result is p * 2^n. Every step is written with an explicit
// round-to-nearest intrinsic so that the compiler cannot contract or reorder
// it.
#pragma once

#include <cstdint>

namespace fg {

__device__ __forceinline__ float exp_fixed(float x) {
  x = fminf(fmaxf(x, -87.0f), 88.0f);
  const float n = rintf(__fmul_rn(x, 1.44269504088896341f));
  float r = __fmaf_rn(-n, 0.693359375f, x);
  r = __fmaf_rn(-n, -2.12194440e-4f, r);
  float p = 1.0f / 5040.0f;
  p = __fmaf_rn(p, r, 1.0f / 720.0f);
  p = __fmaf_rn(p, r, 1.0f / 120.0f);
  p = __fmaf_rn(p, r, 1.0f / 24.0f);
  p = __fmaf_rn(p, r, 1.0f / 6.0f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  const float two_n = __int_as_float((static_cast<int>(n) + 127) << 23);  // n in [-126, 127]
  return __fmul_rn(p, two_n);
}

__device__ __forceinline__ float silu_fixed(float g) {
  return __fdiv_rn(g, __fadd_rn(1.0f, exp_fixed(-g)));
}

// bf16 round trip of an fp32 value (nearest even), as a float.
__device__ __forceinline__ float round_bf16(float v) {
  uint32_t out;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(0.0f), "f"(v));
  return __uint_as_float(out << 16);
}

}  // namespace fg
