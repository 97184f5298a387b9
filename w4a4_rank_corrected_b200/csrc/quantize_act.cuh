// Activation kernel of the SVDQuant W4A4 linear: smoothing, NVFP4
// quantization and the fused low-rank down-projection, in one pass over X.
//
// The fusion is the one described for the Nunchaku engine in the Korean
// rendering of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"
// (section "SVDQuant and the Nunchaku engine"): the low-rank down projection
// is merged into the quantization kernel so the 16-bit branch costs no extra
// pass over the activations.  The B200 design:
//
//   * one CTA owns 64 rows x a contiguous slice of K (64-column chunks).  The
//     host picks how many CTAs split K (a thread-block cluster of 1, 2, 4 or
//     8) so that the whole grid is resident in one wave;
//   * warp 0 streams X chunks [64 x 64] bf16, the matching chunk of the
//     low-rank operand and 64 smoothing factors into a deep shared-memory
//     ring with TMA (128-byte swizzle);
//   * W quantize warps (W = number of ring stages, up to 8): warp w owns ring
//     stage w and processes every chunk that lands there, whole.  Lane l
//     handles rows l and l + 32 (all four 16-groups): it copies its rows and
//     the chunk's smoothing factors into registers and hands the stage back
//     before quantizing, so the next chunk for that stage is already loading
//     while this one is processed; the warps work on different chunks at the
//     same time instead of in lockstep.  Per group: multiply by the
//     smoothing factors, take the maximum in registers, form the E4M3 block
//     scale with one multiply and the hardware conversion, look up g/scale in
//     a 127-entry table (the IEEE quotients, computed once per CTA), form the
//     E2M1 codes with the hardware conversion; per row: 32 code bytes and one
//     32-bit word of scales straight into the MMA tile layout;
//   * warp 1 issues tcgen05 bf16 MMAs (M = 64) on the SAME shared-memory X
//     tile: X [64 x 64] times L1' [2r x 64]^T into a 64 x 2r fp32 accumulator
//     in tensor memory.  L1' holds smooth * L1 split into bf16 hi and lo
//     halves, so X L1' = X_hat L1 to ~2^-16 relative (X itself is exact);
//   * at the end the accumulator is read back (tcgen05.ld), hi + lo columns
//     are summed, the partial sums of a K split are reduced across the
//     cluster through distributed shared memory in a fixed order
//     (deterministic), and the result times lr_scale is stored as a bf16
//     hi/lo pair for the GEMM's up-projection.
#pragma once
#include "ptx.cuh"

namespace svdq_dev {

constexpr int QA_BM = 64;
constexpr int QA_MAX_STAGES = 8;
constexpr int QA_QWARPS = QA_MAX_STAGES;                 // one per ring stage (at most)
constexpr int QA_THREADS = 32 * (2 + QA_QWARPS);
constexpr uint32_t QA_X_BYTES = QA_BM * 128;  // 64 rows x 64 bf16
constexpr uint32_t QA_RING_BUDGET = 180 * 1024;

struct QAParams {
  const float* smooth;
  uint8_t* codes_x;
  uint8_t* sf_x;
  uint16_t* xl1;
  int M, K, r, klr;
  int chunks_per_split;
  int num_splits;
  int stages;
  uint32_t stage_bytes;
  uint32_t tmem_cols;
  float g_x, gs_x, lr_scale;
  uint64_t timeout_ns;
};

__host__ __device__ inline uint32_t qa_stage_bytes(int r) {
  const uint32_t b = QA_X_BYTES + 256u * (uint32_t)r + 256u;
  return (b + 1023u) & ~1023u;
}
__host__ __device__ inline int qa_stages(int r) {
  int st = (int)(QA_RING_BUDGET / qa_stage_bytes(r));
  return st > QA_MAX_STAGES ? QA_MAX_STAGES : (st < 2 ? 2 : st);
}
__host__ __device__ inline uint32_t qa_smem_bytes(int r) {
  return 1024u + (uint32_t)qa_stages(r) * qa_stage_bytes(r) + 1024u;
}

__device__ __forceinline__ int64_t sf_tile_off(int row, int g, int K) {
  return ((int64_t)(row >> 7) * (K >> 6) + (g >> 2)) * 512 + (row & 31) * 16 +
         ((row & 127) >> 5) * 4 + (g & 3);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// hi = bf16(v), lo = bf16(v - hi): v ~= hi + lo to ~2^-16 relative.
__device__ __forceinline__ void split_hi_lo(float v, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(v));
  lo = __fsub_rn(v, hi);
}

// Store 16 consecutive fp32 values (times lr_scale) as a bf16 hi part at
// dst_hi and a bf16 lo part at dst_lo.
__device__ __forceinline__ void store_hi_lo16(const float (&v)[16], float scale, uint16_t* dst_hi,
                                              uint16_t* dst_lo) {
  uint32_t ph[8], pl[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    float h0, l0, h1, l1;
    split_hi_lo(__fmul_rn(v[2 * j], scale), h0, l0);
    split_hi_lo(__fmul_rn(v[2 * j + 1], scale), h1, l1);
    ph[j] = pack_bf16x2(h0, h1);
    pl[j] = pack_bf16x2(l0, l1);
  }
  uint4* dh = reinterpret_cast<uint4*>(dst_hi);
  uint4* dl = reinterpret_cast<uint4*>(dst_lo);
  dh[0] = make_uint4(ph[0], ph[1], ph[2], ph[3]);
  dh[1] = make_uint4(ph[4], ph[5], ph[6], ph[7]);
  dl[0] = make_uint4(pl[0], pl[1], pl[2], pl[3]);
  dl[1] = make_uint4(pl[4], pl[5], pl[6], pl[7]);
}

__global__ void __launch_bounds__(QA_THREADS, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const QAParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int r = p.r;
  const bool has_lr = r > 0;
  const int ST = p.stages;
  const uint32_t SB = p.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + ST * SB);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * ST;
  const uint32_t acc_full = full0 + 16 * ST;
  const uint32_t drain_bar = acc_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * ST + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* qlut = reinterpret_cast<float*>(smem + ST * SB + 512);  // 128 floats

  const uint32_t warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x;
  const int rb = blockIdx.y;
  const int kchunks = p.K >> 6;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(kchunks, c_begin + p.chunks_per_split);
  const int nchunks = max(0, c_end - c_begin);
  const unsigned int kid = 1;  // kernel id in error codes

  if (threadIdx.x == 0) {
    for (int i = 0; i < ST; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1 + (has_lr ? 1 : 0));
    }
    mbar_init(acc_full, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_x);
    if (has_lr) prefetch_tensormap(&tm_l1);
  }
  if (warp == 1 && has_lr) {
    tmem_alloc(smem_u32(tmem_holder), p.tmem_cols);
    tmem_relinquish();
  }
  if (threadIdx.x >= 64 && threadIdx.x < 64 + 128) {
    // q = g / e4m3(code) for every finite non-negative scale code
    const uint32_t code = threadIdx.x - 64;
    qlut[code] = (code == 0 || code == 127) ? 0.0f : __fdiv_rn(p.g_x, e4m3_to_f32(code));
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_lr ? *tmem_holder : 0u;
  // Everything above overlaps the tail of the previous kernel in the stream;
  // from here on this kernel reads and writes memory that kernel may touch.
  grid_dependency_wait();
  grid_launch_dependents();

  int issued = 0;  // producer: chunks whose loads were issued
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      const uint32_t tx = QA_X_BYTES + (has_lr ? 256u * r : 0u) + 256u;
      int st = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nchunks; ++i) {
        if (!mbar_wait(empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (1u << 8) | kid)) break;
        const uint32_t sb = smem_u32(smem + st * SB);
        const int c = c_begin + i;
        mbar_arrive_expect_tx(full0 + 8 * st, tx);
        tma_load_2d(sb, &tm_x, c * 64, rb * QA_BM, full0 + 8 * st);
        if (has_lr) tma_load_2d(sb + QA_X_BYTES, &tm_l1, c * 64, 0, full0 + 8 * st);
        bulk_load(sb + QA_X_BYTES + 256u * r, p.smooth + c * 64, 256, full0 + 8 * st);
        issued = i + 1;
        if (++st == ST) { st = 0; ph ^= 1; }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- down-projection ----
    if (has_lr && lane == 0) {
      const uint32_t idesc = idesc_bf16(QA_BM, 2 * r);
      int st = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nchunks; ++i) {
        if (!mbar_wait(full0 + 8 * st, ph, p.timeout_ns, abort_flag, (2u << 8) | kid)) break;
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + st * SB);
        const uint64_t da = sdesc_sw128(sb), db = sdesc_sw128(sb + QA_X_BYTES);
        for (int kk = 0; kk < 4; ++kk)  // K = 16 bf16 = 32 bytes per MMA
          mma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        tc_commit(empty0 + 8 * st);
        if (++st == ST) { st = 0; ph ^= 1; }
      }
      tc_commit(acc_full);
    }
  } else {
    // ---------------------------------------------- NVFP4 quantization ----
    // warp qw owns ring stage qw: chunks qw, qw + ST, qw + 2 ST, ...
    const int qw = warp - 2;
    const float gs = p.gs_x;
    if (qw < ST) {
      const uint32_t sb = smem_u32(smem + qw * SB);
      const uint8_t* sbp = smem + qw * SB;
      uint32_t ph = 0;
      for (int i = qw; i < nchunks; i += ST, ph ^= 1) {
        if (!mbar_wait_warp(full0 + 8 * qw, ph, p.timeout_ns, abort_flag, (3u << 8) | kid)) break;
        const int c = c_begin + i;
        // copy this lane's two rows and the chunk's smoothing factors into
        // registers, then hand the stage back so the next chunk can land
        // while this one is quantized
        uint4 xr[2][8];
        float4 sv[16];
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int row_t = lane + 32 * hr;
#pragma unroll
          for (int j = 0; j < 8; ++j)
            xr[hr][j] = *reinterpret_cast<const uint4*>(sbp + row_t * 128 + ((j ^ (row_t & 7)) << 4));
        }
        {
          const float4* sp = reinterpret_cast<const float4*>(sbp + QA_X_BYTES + 256u * r);
#pragma unroll
          for (int j = 0; j < 16; ++j) sv[j] = sp[j];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8 * qw);
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int row_t = lane + 32 * hr;
          const int row = rb * QA_BM + row_t;
          uint32_t cw[8];
          uint32_t sfw = 0;
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint4 x0 = xr[hr][2 * g], x1 = xr[hr][2 * g + 1];
            const float4 s0 = sv[4 * g], s1 = sv[4 * g + 1], s2 = sv[4 * g + 2], s3 = sv[4 * g + 3];
            float v[16];
            v[0] = __fmul_rn(bf16_lo_f32(x0.x), s0.x);
            v[1] = __fmul_rn(bf16_hi_f32(x0.x), s0.y);
            v[2] = __fmul_rn(bf16_lo_f32(x0.y), s0.z);
            v[3] = __fmul_rn(bf16_hi_f32(x0.y), s0.w);
            v[4] = __fmul_rn(bf16_lo_f32(x0.z), s1.x);
            v[5] = __fmul_rn(bf16_hi_f32(x0.z), s1.y);
            v[6] = __fmul_rn(bf16_lo_f32(x0.w), s1.z);
            v[7] = __fmul_rn(bf16_hi_f32(x0.w), s1.w);
            v[8] = __fmul_rn(bf16_lo_f32(x1.x), s2.x);
            v[9] = __fmul_rn(bf16_hi_f32(x1.x), s2.y);
            v[10] = __fmul_rn(bf16_lo_f32(x1.y), s2.z);
            v[11] = __fmul_rn(bf16_hi_f32(x1.y), s2.w);
            v[12] = __fmul_rn(bf16_lo_f32(x1.z), s3.x);
            v[13] = __fmul_rn(bf16_hi_f32(x1.z), s3.y);
            v[14] = __fmul_rn(bf16_lo_f32(x1.w), s3.z);
            v[15] = __fmul_rn(bf16_hi_f32(x1.w), s3.w);
            float m0 = fmaxf(fabsf(v[0]), fabsf(v[1])), m1 = fmaxf(fabsf(v[2]), fabsf(v[3]));
            float m2 = fmaxf(fabsf(v[4]), fabsf(v[5])), m3 = fmaxf(fabsf(v[6]), fabsf(v[7]));
            float m4 = fmaxf(fabsf(v[8]), fabsf(v[9])), m5 = fmaxf(fabsf(v[10]), fabsf(v[11]));
            float m6 = fmaxf(fabsf(v[12]), fabsf(v[13])), m7 = fmaxf(fabsf(v[14]), fabsf(v[15]));
            const float a = fmaxf(fmaxf(fmaxf(m0, m1), fmaxf(m2, m3)), fmaxf(fmaxf(m4, m5), fmaxf(m6, m7)));
            const uint32_t code = cvt_e4m3x2(__fmul_rn(a, gs), 0.0f) & 0xFF;
            const float q = qlut[code];
            float t0[8], t1[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              t0[e] = __fmul_rn(v[e], q);
              t1[e] = __fmul_rn(v[8 + e], q);
            }
            cw[2 * g] = cvt_e2m1x8(t0);
            cw[2 * g + 1] = cvt_e2m1x8(t1);
            sfw |= code << (8 * g);
          }
          if (row < p.M) {
            uint4* dst = reinterpret_cast<uint4*>(p.codes_x + (size_t)row * (p.K >> 1) + (size_t)c * 32);
            dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
            dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
          }
          *reinterpret_cast<uint32_t*>(p.sf_x + sf_tile_off(row, 4 * c, p.K)) = sfw;
        }
      }
      (void)sb;
    }

    // ----------------------------------------- low-rank epilogue (X L1) ----
    if (has_lr) {
      const bool ok = mbar_wait_warp(acc_full, 0, p.timeout_ns, abort_flag, (4u << 8) | kid);
      tc_fence_after();
      // M = 64 accumulator: row m sits in lane (m % 16) + 32 (m / 16).  Warp w
      // reads its lane quarter w % 4; lanes 0..15 hold rows 16 (w % 4) + lane.
      const int quad = warp & 3;
      const int hc = (warp - 2) >> 2;          // 0..1: which chunks of 16 columns
      const int lrow_t = quad * 16 + lane;
      const int lrow = rb * QA_BM + lrow_t;
      const bool own = lane < 16;
      const int S = p.num_splits;
      float* P = reinterpret_cast<float*>(smem);  // [64][r+1], reuses the ring
      const int pstride = r + 1;
      // every quantize warp is done reading the ring before it is reused
      asm volatile("bar.sync 1, %0;" ::"n"(32 * QA_QWARPS) : "memory");
      for (int ci = hc; ci < r / 16; ci += QA_QWARPS / 4) {  // QA_QWARPS / 4 warps per quarter
        uint32_t hi[16], lo[16];
        const uint32_t base = tmem + ((uint32_t)(quad * 32) << 16);
        if (ok) {
          tmem_ld16(base + 16 * ci, hi);
          tmem_ld16(base + r + 16 * ci, lo);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 16; ++j) hi[j] = lo[j] = 0u;
        }
        float part[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) part[j] = __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
        if (own) {
          if (S > 1) {
#pragma unroll
            for (int j = 0; j < 16; ++j) P[lrow_t * pstride + 16 * ci + j] = part[j];
          } else if (lrow < p.M) {
            store_hi_lo16(part, p.lr_scale, p.xl1 + (size_t)lrow * p.klr + 16 * ci,
                          p.xl1 + (size_t)lrow * p.klr + r + 16 * ci);
          }
        }
      }
      if (S == 1 && hc == 0 && own && lrow < p.M) {
        for (int cpad = 2 * r; cpad < p.klr; cpad += 8)
          *reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + cpad) = make_uint4(0, 0, 0, 0);
      }
    }
  }

  // ------------------------------------ cross-CTA reduction of X L1 parts ----
  if (has_lr && p.num_splits > 1) {
    tc_fence_before();
    __syncthreads();
    cluster_sync();  // every rank's partial sums are in its shared memory
    if (blockIdx.x == 0 && warp >= 2) {
      const int t = threadIdx.x - 64;           // 0..255
      const int lrow_t = t >> 2;                // 64 rows x 4 threads
      const int lrow = rb * QA_BM + lrow_t;
      const int pstride = r + 1;
      const uint32_t Pbase = smem_u32(smem);
      if (lrow < p.M) {
        for (int ci = (t & 3); ci < r / 16; ci += 4) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
          for (int s = 0; s < p.num_splits; ++s) {
            const uint32_t rbase = map_to_rank(Pbase, (uint32_t)s);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              acc[j] += ld_cluster_f32(rbase + 4u * (uint32_t)(lrow_t * pstride + 16 * ci + j));
          }
          store_hi_lo16(acc, p.lr_scale, p.xl1 + (size_t)lrow * p.klr + 16 * ci,
                        p.xl1 + (size_t)lrow * p.klr + r + 16 * ci);
        }
        if ((t & 3) == 0)
          for (int cpad = 2 * r; cpad < p.klr; cpad += 8)
            *reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + cpad) = make_uint4(0, 0, 0, 0);
      }
    }
    cluster_sync();  // keep every rank's shared memory alive until read
  }

  // ------------------------------------------------------------ teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // drain: loads still in flight, then tensor-core work still in flight
    if (warp == 0 && lane == 0) {
      for (int i = max(0, issued - ST); i < issued; ++i)
        mbar_wait_drain(full0 + 8 * (i % ST), (i / ST) & 1, p.timeout_ns);
    }
    if (warp == 1 && lane == 0 && has_lr) {
      tc_commit(drain_bar);
      mbar_wait_drain(drain_bar, 0, p.timeout_ns);
    }
    __syncthreads();
  }
  if (warp == 1 && has_lr) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace svdq_dev
