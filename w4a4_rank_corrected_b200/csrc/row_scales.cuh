// Per-token (per-row) activation tensor scales: the dynamic alternative to
// the static calibrated scale, for inputs outside the calibration range.
// The pages fix only the static form (NVFP4: one fp32 tensor scale; hardware
// table of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"); here
// each row of X_hat is its own tensor for the same NVFP4 recipe:
//   A_m  = max_k |fp32(x_mk * smooth_k)|            (exact: a maximum)
//   g_m  = fp32(2688 / A_m), gs_m = fp32(448 / A_m) (1 and 1 when A_m = 0)
//   lr_m = fp32(g_m * g_w)     the low-rank branch's pre-scale for row m
//   al_m = fp32(1 / lr_m)      the GEMM epilogue's output scale for row m
// One pass over X, memory-bound: one warp per row, 16-byte loads.
#pragma once
#include "ptx.cuh"

namespace svdq_dev {

struct RowScale {
  float g, gs, lr, alpha;
};

__global__ void __launch_bounds__(256)
    row_scales_kernel(const uint16_t* __restrict__ X, int64_t ldx, const float* __restrict__ smooth,
                      int M, int K, float g_w, RowScale* __restrict__ out) {
  const int warps = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int m = blockIdx.x * warps + (threadIdx.x >> 5); m < M; m += gridDim.x * warps) {
    const uint4* xr = reinterpret_cast<const uint4*>(X + (size_t)m * ldx);
    const float4* s4 = reinterpret_cast<const float4*>(smooth);
    uint32_t amax = 0;   // bit pattern of a non-negative float: integer order = value order
    for (int j = lane; j < K / 8; j += 32) {
      const uint4 x = __ldg(xr + j);
      const float4 s0 = __ldg(s4 + 2 * j), s1 = __ldg(s4 + 2 * j + 1);
      const float v[8] = {__fmul_rn(bf16_lo_f32(x.x), s0.x), __fmul_rn(bf16_hi_f32(x.x), s0.y),
                          __fmul_rn(bf16_lo_f32(x.y), s0.z), __fmul_rn(bf16_hi_f32(x.y), s0.w),
                          __fmul_rn(bf16_lo_f32(x.z), s1.x), __fmul_rn(bf16_hi_f32(x.z), s1.y),
                          __fmul_rn(bf16_lo_f32(x.w), s1.z), __fmul_rn(bf16_hi_f32(x.w), s1.w)};
#pragma unroll
      for (int e = 0; e < 8; ++e) amax = max(amax, __float_as_uint(fabsf(v[e])));
    }
    amax = __reduce_max_sync(0xffffffffu, amax);
    if (lane == 0) {
      const float a = __uint_as_float(amax);
      RowScale rs;
      rs.g = a == 0.0f ? 1.0f : __fdiv_rn(2688.0f, a);
      rs.gs = a == 0.0f ? 1.0f : __fdiv_rn(448.0f, a);
      rs.lr = __fmul_rn(rs.g, g_w);
      rs.alpha = __fdiv_rn(1.0f, rs.lr);
      out[m] = rs;
    }
  }
}

}  // namespace svdq_dev
