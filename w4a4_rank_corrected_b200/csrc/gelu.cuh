// GELU between the two linears of a Flux MLP pair, fused into the first
// linear's epilogue.  The pages name "fused GELU/MLP kernels" as part of the
// original engine's speed ("Bringing Nunchaku 4-bit diffusion inference to
// Diffusers", Vietnamese rendering, section "Introducing Nunchaku Lite").
//
// The tanh form of GELU, 0.5 y (1 + tanh(u)) with u = sqrt(2/pi) (y +
// 0.044715 y^3), is the same function as y * sigma(2u) = y / (1 + e^(-2u))
// (1 + tanh(u) = 2 / (1 + e^(-2u))), which has no cancellation for negative
// y.  Here e^(-2u) = 2^(-2u log2 e) comes from the hardware's base-2
// exponential and the reciprocal from its reciprocal instruction (both the
// approximate forms, a few 1e-7 relative), so one GELU costs about seven
// operations: cheap enough for a GEMM epilogue that writes 56 million
// outputs per Flux MLP layer.  (A division-based form whose every step is a
// correctly rounded fp32 operation was measured first: it made the first
// linear of the pair four times slower.)  The result is rounded to bf16 and
// agrees with the correctly rounded exact GELU except next to a bf16
// rounding boundary, where the two may differ by one unit in the last
// place.
#pragma once
#include <cuda_bf16.h>

namespace svdq_dev {

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// GELU (tanh form) of an fp32 value: y / (1 + 2^(-2 log2(e) u)).
__device__ __forceinline__ float gelu_tanh_fast(float y) {
  // -2 log2(e) sqrt(2/pi) and the same times 0.044715
  constexpr float c0 = -2.3022082f;
  constexpr float c1 = -0.10294324f;
  const float y2 = y * y;
  const float z = y * fmaf(c1, y2, c0);   // -2 log2(e) u
  return y * rcp_approx(1.0f + ex2_approx(z));
}

// bf16 in, bf16 out: the MLP pair's glue.
__device__ __forceinline__ float gelu_bf16_value(float y_bf16) {
  return __bfloat162float(__float2bfloat16_rn(gelu_tanh_fast(y_bf16)));
}

}  // namespace svdq_dev
