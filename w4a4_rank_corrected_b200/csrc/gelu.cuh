// GELU between the two linears of a Flux MLP pair, fused into the first
// linear's epilogue.  The pages name "fused GELU/MLP kernels" as part of the
// original engine's speed ("Bringing Nunchaku 4-bit diffusion inference to
// Diffusers", Vietnamese rendering, section "Introducing Nunchaku Lite").
//
// The tanh form of GELU, 0.5 y (1 + tanh(u)) with u = sqrt(2/pi) (y +
// 0.044715 y^3), is evaluated as h = y / (1 + e^(-2u)) (the same function:
// 1 + tanh(u) = 2 / (1 + e^(-2u)); nothing cancels for negative y), every
// step one IEEE round-to-nearest fp32 operation in a fixed order, and e^x
// from basic fp32 operations only:
//   t = fp32(x log2 e), clamped to [-126, 128]; n = t rounded to the nearest
//   integer (ties to even); f = t - n (exact); 2^f by the degree-7 Taylor
//   series of e^(f ln 2) in Horner form, each multiply and add rounded;
//   the result scaled by 2^n (exact, or inf at n = 128).
// So the kernel's GELU is a fixed sequence of correctly rounded operations
// that any implementation of the same steps reproduces bit for bit.
#pragma once
#include <cmath>
#include <cuda_bf16.h>

namespace svdq_dev {

// (ln 2)^k / k!, k = 0..7, each rounded once from double to float.
struct GeluConsts {
  float taylor[8];
  float log2e;        // fp32(log2(e))
  float sqrt_2_pi;    // fp32(sqrt(2 / pi))
  float cubic;        // fp32(0.044715)
};

// The constants in double, each rounded once to float: ln(2)^k by pow, k!
// exactly, sqrt(2 / pi) from the double pi.
__host__ inline GeluConsts gelu_consts_host() {
  GeluConsts c;
  const double ln2 = std::log(2.0);
  double fact = 1.0;
  for (int k = 0; k < 8; ++k) {
    if (k > 0) fact *= (double)k;
    c.taylor[k] = (float)(std::pow(ln2, (double)k) / fact);
  }
  c.log2e = (float)1.4426950408889634;
  c.sqrt_2_pi = (float)std::sqrt(2.0 / 3.141592653589793);
  c.cubic = (float)0.044715;
  return c;
}

__device__ __forceinline__ float exp_f32_steps(float x, const GeluConsts& c) {
  float t = __fmul_rn(x, c.log2e);
  t = fminf(fmaxf(t, -126.0f), 128.0f);
  const float n = rintf(t);
  const float f = __fsub_rn(t, n);
  float p = c.taylor[7];
#pragma unroll
  for (int k = 6; k >= 0; --k) {
    p = __fmul_rn(p, f);
    p = __fadd_rn(p, c.taylor[k]);
  }
  const int ni = (int)n;
  if (ni == 128) return __fmul_rn(__fmul_rn(p, 1.7014118346046923e38f), 2.0f);  // 2^127 * 2
  return __fmul_rn(p, __int_as_float((ni + 127) << 23));
}

__device__ __forceinline__ float gelu_tanh_steps(float y, const GeluConsts& c) {
  const float y2 = __fmul_rn(y, y);
  const float y3 = __fmul_rn(y2, y);
  const float v = __fmul_rn(c.cubic, y3);
  const float w = __fadd_rn(y, v);
  const float u = __fmul_rn(c.sqrt_2_pi, w);
  const float e = exp_f32_steps(__fmul_rn(-2.0f, u), c);
  const float d = __fadd_rn(1.0f, e);
  return __fdiv_rn(y, d);
}

// bf16 in, bf16 out: the MLP pair's glue.
__device__ __forceinline__ float gelu_bf16_value(float y_bf16, const GeluConsts& c) {
  return __bfloat162float(__float2bfloat16_rn(gelu_tanh_steps(y_bf16, c)));
}

}  // namespace svdq_dev
