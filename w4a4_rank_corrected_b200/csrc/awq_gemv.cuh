// AWQ W4A16 linear: 4-bit weights, 16-bit activations -- the second kernel
// family of the pages, for the memory-bound, precision-sensitive modulation
// and adaptive-normalization projections ("Bringing Nunchaku 4-bit diffusion
// inference to Diffusers", Russian rendering, "Technical details and
// hardware support"; Korean rendering, the kernel-family list).
//
// Y = X W^T + bias with W stored as asymmetric INT4 per group of `group`
// input channels: w = (q - z) * scale, q and z integers 0..15, scale fp16.
// At the batch sizes of those layers (a few conditioning vectors) the layer
// is a matrix-vector product bound by the weight stream, so it runs on the
// CUDA cores: one warp per output row at a time, each lane streaming 16
// bytes (32 codes) of the row per step, dequantizing in registers (exact in
// fp32: a small integer times an fp16 scale) and accumulating the M dot
// products in fp32; X is staged once per CTA in shared memory as fp32, each
// 32-value chunk padded to 36 floats (lane l reads chunk l: with a 144-byte
// chunk stride the 32 lanes' 16-byte reads fall on distinct bank groups,
// where the unpadded 128-byte stride put all of them on the same banks and
// cost 8x in shared-memory wavefronts); the lanes' partial sums meet in a
// warp reduction.  A persistent grid (a few
// CTAs per SM) keeps enough loads in flight to cover the memory latency.
#pragma once
#include <cuda_fp16.h>
#include "ptx.cuh"

namespace svdq_dev {

constexpr int AWQ_THREADS = 256;
constexpr int AWQ_MAX_M = 8;
constexpr int AWQ_CHUNK_PAD = 36;   // floats per staged 32-value chunk of X

template <int MT>
__global__ void __launch_bounds__(AWQ_THREADS)
    awq_gemv_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ zeros,
                    const uint16_t* __restrict__ scales, const uint16_t* __restrict__ bias, int N,
                    int K, int group, const uint16_t* __restrict__ X, int64_t ldx,
                    uint16_t* __restrict__ Y, int64_t ldy) {
  extern __shared__ float xs[];   // [MT][K / 32][36] fp32 (chunks padded)
  const int KP = (K >> 5) * AWQ_CHUNK_PAD;
  for (int i = threadIdx.x; i < MT * K; i += blockDim.x) {
    const int m = i / K, k = i - m * K;
    xs[m * KP + (k >> 5) * AWQ_CHUNK_PAD + (k & 31)] = bf16_lo_f32(X[(size_t)m * ldx + k]);
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int warps = blockDim.x >> 5;
  const int chunks = K >> 5;                 // 32 codes (16 bytes) per chunk
  const int G = K / group;
  const int cpg = group >> 5;                // chunks per group
  for (int n = blockIdx.x * warps + (threadIdx.x >> 5); n < N; n += gridDim.x * warps) {
    const uint4* row = reinterpret_cast<const uint4*>(q + (size_t)n * (K / 2));
    float acc[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    for (int c0 = lane; c0 < chunks; c0 += 4 * 32) {
      // up to four chunks per lane in flight before any arithmetic
      uint4 w[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        w[u] = c < chunks ? __ldcs(row + c) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + 32 * u;
        if (c >= chunks) break;
        const int gi = c / cpg;
        const float sc = __half2float(__ushort_as_half(scales[(size_t)n * G + gi]));
        const float nzs = -(float)zeros[(size_t)n * G + gi] * sc;   // exact: z * fp16
        const uint32_t words[4] = {w[u].x, w[u].y, w[u].z, w[u].w};
        float v[32];
#pragma unroll
        for (int t = 0; t < 4; ++t)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // the code as a float without a conversion instruction: the bits
            // of 2^23 + q, minus 2^23 (exact); then (q - z) scale = q scale -
            // z scale, exact in one fused operation (every term is a small
            // integer times the fp16 scale)
            const float qf =
                __uint_as_float(0x4B000000u | ((words[t] >> (4 * j)) & 15u)) - 8388608.0f;
            v[8 * t + j] = fmaf(qf, sc, nzs);
          }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
          const float4* x4 = reinterpret_cast<const float4*>(xs + m * KP + c * AWQ_CHUNK_PAD);
          float a = acc[m];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const float4 xv = x4[j];
            a = fmaf(xv.x, v[4 * j], a);
            a = fmaf(xv.y, v[4 * j + 1], a);
            a = fmaf(xv.z, v[4 * j + 2], a);
            a = fmaf(xv.w, v[4 * j + 3], a);
          }
          acc[m] = a;
        }
      }
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
      float a = acc[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      acc[m] = a;
    }
    if (lane < MT) {
      float a = acc[0];
#pragma unroll
      for (int m = 1; m < MT; ++m)
        if (lane == m) a = acc[m];
      if (bias) a += bf16_lo_f32(bias[n]);
      Y[(size_t)lane * ldy + n] = (uint16_t)(__float_as_uint(__bfloat162float(__float2bfloat16_rn(a))) >> 16);
    }
  }
}

}  // namespace svdq_dev
