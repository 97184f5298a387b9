// AWQ W4A16 linear: 4-bit weights, 16-bit activations -- the second kernel
// family of the pages, for the memory-bound, precision-sensitive modulation
// and adaptive-normalization projections ("Bringing Nunchaku 4-bit diffusion
// inference to Diffusers", Russian rendering, "Technical details and
// hardware support"; Korean rendering, the kernel-family list).
//
// Y = X W^T + bias with W stored as asymmetric INT4 per group of `group`
// input channels: w = (q - z) * scale, q and z integers 0..15, scale fp16.
// At the batch sizes of those layers (M <= 8 conditioning vectors) the
// layer is bound by the weight stream: about 22 bytes, 45 weights, per SM
// clock at the HBM rate.  A CUDA-core dot product spends an FMA per weight
// and batch row plus the code's conversion -- more issue slots than an SM
// has at that rate.  So the contraction runs on the tensor core with
// register operands (mma.sync m16n8k16, bf16 in, fp32 accumulate): a warp's
// 16 x 16 weight tile is dequantized in registers and meets the batch
// (padded to 8 columns) in one instruction.  The dequantized weights never
// touch shared or tensor memory (the weight stream's rate would saturate
// either), which is why this is not a tcgen05 kernel.
//
//   * codes arrive pre-tiled (svdq_awq_tile_codes): per 16-row block and
//     four 16-deep k-steps, 512 bytes in which lane l's 16 bytes are its
//     four 32-bit words, one per k-step; the eight codes of a word are that
//     lane's eight A-fragment elements, nibbles j and j + 4 forming register
//     j of the fragment (low and high half);
//   * a pair of codes becomes the bf16 pair (128 + q, 128 + q') with one
//     shift and one bitwise op (the nibble lands in the low mantissa bits
//     of 128.0), then q - z exactly with one bf16x2 subtraction of
//     (128 + z, 128 + z);
//   * per group the MMA accumulators (two, for even and odd k-steps) hold
//     sum_k (q_k - z) x_k (products exact, fp32 accumulation); the group's
//     fp16 scale multiplies it into the running sum (one FMA per output);
//   * X is staged once per CTA in shared memory (16-byte loads), per k-step
//     and batch row 16 values in B-fragment order (lane c's four values
//     adjacent: one 8-byte load);
//   * a CTA's eight warps cover 8 / S row blocks, S warps splitting K per
//     block (S chosen by the host so the grid has enough warps); their
//     partial sums meet in shared memory, bias is added and Y is rounded
//     once to bf16.  A warp works in 128-deep slots (two 512-byte blocks of
//     codes, one group's scales and zeros; the group size is a multiple of
//     128) and keeps four slots in flight ahead of the one it computes.
#pragma once
#include <cuda_fp16.h>
#include "ptx.cuh"

namespace svdq_dev {

constexpr int AWQ_THREADS = 256;
constexpr int AWQ_WARPS = AWQ_THREADS / 32;
constexpr int AWQ_MAX_M = 8;
constexpr int AWQ_PF = 4;                                // 1 KB slots in flight per warp
constexpr uint32_t AWQ_SMEM_MAX = 216u * 1024u;
constexpr int AWQ_RED_FLOATS = 2 * AWQ_WARPS * 32 * 4;   // two buffers of partial fragments

// Shared memory of one CTA: the partial-sum buffers, then X (bf16 [K/16][M][16]).
__host__ __device__ inline size_t awq_smem_bytes(int M, int K) {
  return (size_t)AWQ_RED_FLOATS * 4 + (size_t)K * (size_t)M * 2;
}

// Byte offset of lane l's word for k-step ks of row block rb in the tiled codes.
__host__ __device__ inline size_t awq_tile_word_offset(int rb, int ks, int lane, int K) {
  return (((size_t)rb * (size_t)(K / 64) + (size_t)(ks >> 2)) * 32 + (size_t)lane) * 16 +
         (size_t)(ks & 3) * 4;
}

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
      "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t bf16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The codes of nibbles j and j + 4 (the word shifted right by 4 j) as the
// bf16 pair (128 + q_j, 128 + q_{j+4}).
__device__ __forceinline__ uint32_t awq_pair128(uint32_t shifted) {
  return (shifted & 0x000F000Fu) | 0x43004300u;
}

struct AwqSlot {   // one 128-deep slot in flight: codes, and its group's scales and zeros
  uint4 w0, w1;    // the slot's two 512-byte blocks (this lane's 16 bytes of each)
  uint32_t s;      // fp16 bits: row g (low half), row g + 8 (high half)
  uint32_t z;      // zeros: row g (bits 0..7), row g + 8 (bits 16..23)
};

template <int MT>
__global__ void __launch_bounds__(AWQ_THREADS, 2)
    awq_gemv_kernel(const uint8_t* __restrict__ q, const uint8_t* __restrict__ zeros,
                    const uint16_t* __restrict__ scales, const uint16_t* __restrict__ bias, int N,
                    int K, int group, int S, const uint16_t* __restrict__ X, int64_t ldx,
                    uint16_t* __restrict__ Y, int64_t ldy) {
  extern __shared__ __align__(16) uint8_t awq_smem[];
  float* red = reinterpret_cast<float*>(awq_smem);                            // [2][8][32][4]
  uint16_t* xs = reinterpret_cast<uint16_t*>(awq_smem + AWQ_RED_FLOATS * 4);  // [K/16][MT][16]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, c = lane & 3;
  const int G = K / group;
  const int spg = group >> 7;                 // 128-deep slots per group
  const int R = AWQ_WARPS / S;                // row blocks per CTA per round
  const int rb_total = (N + 15) >> 4;
  const int rounds = (rb_total + R - 1) / R;
  const int my_rounds =
      (int)blockIdx.x < rounds ? (rounds - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int sub = warp % S, rloc = warp / S;
  const int gps = (G + S - 1) / S;            // groups per K slice
  const int g0 = min(G, sub * gps), g1 = min(G, g0 + gps);
  const int nsl = (g1 - g0) * spg;            // this warp's slots per round
  const int total = my_rounds * nsl;
  const int sk0 = g0 * spg;                   // first slot of this warp's K slice

  // ---- fetch side of this warp's sequence of (round, slot): pointers
  // advanced per slot, recomputed once per round ----
  int f_round = 0, f_sl = 0, f_ing = 0;       // round, slot in the round, slot in the group
  bool f_ok = false, f_ok0 = false, f_ok1 = false;
  const uint4* f_q = reinterpret_cast<const uint4*>(q);
  const uint16_t *f_s0 = scales, *f_s1 = scales;
  const uint8_t *f_z0 = zeros, *f_z1 = zeros;
  auto f_start_round = [&]() {
    const int rb = ((int)blockIdx.x + f_round * (int)gridDim.x) * R + rloc;
    const int n0 = rb * 16 + g;
    f_ok = rb < rb_total;
    f_ok0 = n0 < N;
    f_ok1 = n0 + 8 < N;
    f_q = reinterpret_cast<const uint4*>(q + awq_tile_word_offset(f_ok ? rb : 0, 8 * sk0, lane, K));
    const size_t r0 = f_ok0 ? (size_t)n0 * G + g0 : 0, r1 = f_ok1 ? (size_t)(n0 + 8) * G + g0 : 0;
    f_s0 = scales + r0;
    f_s1 = scales + r1;
    f_z0 = zeros + r0;
    f_z1 = zeros + r1;
    f_ing = 0;
  };
  auto fetch = [&](AwqSlot& sl) {
    if (f_ok) {
      sl.w0 = __ldcs(f_q);
      sl.w1 = __ldcs(f_q + 32);               // the next 512-byte block
    } else {
      sl.w0 = sl.w1 = make_uint4(0, 0, 0, 0);
    }
    sl.s = (f_ok0 ? (uint32_t)__ldg(f_s0) : 0u) | ((f_ok1 ? (uint32_t)__ldg(f_s1) : 0u) << 16);
    sl.z = (f_ok0 ? (uint32_t)__ldg(f_z0) : 0u) | ((f_ok1 ? (uint32_t)__ldg(f_z1) : 0u) << 16);
    f_q += 64;
    if (++f_ing == spg) {
      f_ing = 0;
      ++f_s0, ++f_s1, ++f_z0, ++f_z1;
    }
    if (++f_sl == nsl) {
      f_sl = 0;
      ++f_round;
      f_start_round();
    }
  };
  if (nsl > 0) f_start_round();
  AwqSlot ring[AWQ_PF];
#pragma unroll
  for (int j = 0; j < AWQ_PF; ++j)
    if (j < total) fetch(ring[j]);            // in flight while X is staged

  // ---- X into shared memory, each k-step's 16 values in B-fragment order:
  // value j of a k-step goes to 4 ((j % 8) / 2) + 2 (j / 8) + j % 2, so each
  // aligned pair stays a pair.  16-byte loads, four in flight per thread.
  {
    const int cpr = K >> 3;                   // 8-value chunks per row
    uint32_t* xs32 = reinterpret_cast<uint32_t*>(xs);
    for (int i0 = threadIdx.x; i0 < MT * cpr; i0 += 4 * AWQ_THREADS) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * AWQ_THREADS;
        if (i < MT * cpr) {
          const int m = i / cpr, ch = i - m * cpr;
          v[u] = __ldg(reinterpret_cast<const uint4*>(X + (size_t)m * ldx) + ch);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * AWQ_THREADS;
        if (i < MT * cpr) {
          const int m = i / cpr, ch = i - m * cpr;
          const int ks = ch >> 1, hi8 = ch & 1;   // the chunk is values 8 hi8 .. 8 hi8 + 7
          uint32_t* dst = xs32 + ((size_t)ks * MT + m) * 8 + hi8;
          dst[0] = v[u].x;
          dst[2] = v[u].y;
          dst[4] = v[u].z;
          dst[6] = v[u].w;
        }
      }
    }
  }
  __syncthreads();

  float acc[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  float ce[4] = {0.0f, 0.0f, 0.0f, 0.0f}, co[4] = {0.0f, 0.0f, 0.0f, 0.0f};   // even / odd k-steps
  int c_round = 0, c_sl = 0, c_ing = 0;
  // this lane's B fragment: batch row g, values 4c .. 4c+3 of each k-step's
  // 16; a lane past the batch keeps zeros
  const bool has_b = g < MT;
  const uint2* xl0 = reinterpret_cast<const uint2*>(xs + (size_t)(has_b ? g : 0) * 16 + 4 * c) +
                     (size_t)sk0 * 8 * MT * 4;
  const uint2* xl = xl0;
  uint32_t b0 = 0, b1 = 0;
  // a warp without slots still takes one step per round (the CTA's barrier
  // is passed by every warp once per round)
  const int steps = nsl > 0 ? total : my_rounds;
  for (int base = 0; base < steps; base += AWQ_PF) {
#pragma unroll
    for (int j = 0; j < AWQ_PF; ++j) {
      const int item = base + j;
      if (item < steps) {
        bool round_end = true;
        if (nsl > 0) {
          const AwqSlot sl = ring[j];
          if (item + AWQ_PF < total) fetch(ring[j]);
          // (128 + z) in both halves, for each of this lane's two rows
          const uint32_t zz0 = ((sl.z & 0xFFu) * 0x00010001u) | 0x43004300u;
          const uint32_t zz1 = ((sl.z >> 16) * 0x00010001u) | 0x43004300u;
          const uint32_t words[8] = {sl.w0.x, sl.w0.y, sl.w0.z, sl.w0.w,
                                     sl.w1.x, sl.w1.y, sl.w1.z, sl.w1.w};
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const uint32_t wd = words[t];
            uint32_t a[4];
            a[0] = bf16x2_sub(awq_pair128(wd), zz0);         // row g,     k 2c, 2c+1
            a[1] = bf16x2_sub(awq_pair128(wd >> 4), zz1);    // row g + 8, k 2c, 2c+1
            a[2] = bf16x2_sub(awq_pair128(wd >> 8), zz0);    // row g,     k 2c+8, 2c+9
            a[3] = bf16x2_sub(awq_pair128(wd >> 12), zz1);   // row g + 8, k 2c+8, 2c+9
            if (has_b) {
              const uint2 xv = xl[t * MT * 4];   // k-step t of the slot: MT rows of 16 values
              b0 = xv.x;
              b1 = xv.y;
            }
            if (t & 1)
              mma_bf16_16816(co, a, b0, b1);
            else
              mma_bf16_16816(ce, a, b0, b1);
          }
          xl += 8 * MT * 4;
          if (++c_ing == spg) {
            c_ing = 0;
            // the group's sum of (q - z) x, times its scale
            const float s0 = __half2float(__ushort_as_half((unsigned short)(sl.s & 0xFFFFu)));
            const float s1 = __half2float(__ushort_as_half((unsigned short)(sl.s >> 16)));
            acc[0] = fmaf(s0, ce[0] + co[0], acc[0]);
            acc[1] = fmaf(s0, ce[1] + co[1], acc[1]);
            acc[2] = fmaf(s1, ce[2] + co[2], acc[2]);
            acc[3] = fmaf(s1, ce[3] + co[3], acc[3]);
#pragma unroll
            for (int e = 0; e < 4; ++e) ce[e] = co[e] = 0.0f;
          }
          round_end = ++c_sl == nsl;
          if (round_end) {
            c_sl = 0;
            xl = xl0;
          }
        }
        if (round_end) {
          // the S warps of each row block add their partial sums
          float* buf = red + (c_round & 1) * (AWQ_WARPS * 32 * 4);
          *reinterpret_cast<float4*>(buf + (warp * 32 + lane) * 4) =
              make_float4(acc[0], acc[1], acc[2], acc[3]);
          acc[0] = acc[1] = acc[2] = acc[3] = 0.0f;
          named_barrier_sync(1, AWQ_THREADS);
          const int rbase = ((int)blockIdx.x + c_round * (int)gridDim.x) * R;
          for (int o = threadIdx.x; o < R * 16 * MT; o += AWQ_THREADS) {
            const int rl = o / (16 * MT), rem = o - rl * (16 * MT);
            const int row = rem / MT, m = rem - row * MT;
            const int src = (row & 7) * 4 + (m >> 1);      // the fragment's lane
            const int idx = (row >> 3) * 2 + (m & 1);      // and element
            float y = 0.0f;
            for (int s2 = 0; s2 < S; ++s2) y += buf[((rl * S + s2) * 32 + src) * 4 + idx];
            const int n = (rbase + rl) * 16 + row;
            if (rbase + rl < rb_total && n < N) {
              if (bias) y += bf16_lo_f32(bias[n]);
              Y[(size_t)m * ldy + n] =
                  (uint16_t)(__float_as_uint(__bfloat162float(__float2bfloat16_rn(y))) >> 16);
            }
          }
          ++c_round;
        }
      }
    }
  }
}

}  // namespace svdq_dev
