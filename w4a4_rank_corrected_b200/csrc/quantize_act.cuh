// Activation kernel of the SVDQuant W4A4 linear: smoothing, NVFP4
// quantization and the fused low-rank down-projection, in one pass over X.
//
// The fusion is the one described for the Nunchaku engine in the Korean
// rendering of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"
// (section "SVDQuant and the Nunchaku engine"): the low-rank down projection
// is merged into the quantization kernel so the 16-bit branch costs no extra
// pass over the activations.  The B200 design:
//
//   * one CTA owns 128 rows x a contiguous slice of K (64-column chunks);
//     when there are too few row blocks to fill the GPU, the K range is split
//     over a thread-block cluster of up to 8 CTAs;
//   * warp 0 streams X chunks [128 x 64] bf16, the matching chunk of the
//     low-rank operand and 64 smoothing factors into a 4-deep shared-memory
//     ring with TMA (128-byte swizzle);
//   * warps 2..9 read each chunk from shared memory, multiply by the
//     smoothing factors, take the per-16 maximum in registers (one thread
//     owns whole groups), form the E4M3 scale and the E2M1 codes with the
//     hardware conversions, and store codes (16 bytes per thread) and scales
//     (directly in the MMA tile layout);
//   * warp 1 issues tcgen05 bf16 MMAs on the SAME shared-memory X tile:
//     X [128 x 64] times L1' [2r x 64]^T into a 128 x 2r fp32 accumulator in
//     tensor memory.  L1' holds smooth * L1 split into bf16 hi and lo halves,
//     so X L1' = X_hat L1 to ~2^-16 relative (X itself is exact in bf16);
//   * at the end the accumulator is read back (tcgen05.ld), hi + lo columns
//     are summed, partial sums of the K split are reduced across the cluster
//     through distributed shared memory in a fixed order (deterministic), and
//     the result, times lr_scale, is stored as a bf16 hi/lo pair for the
//     GEMM's up-projection.
#pragma once
#include "ptx.cuh"

namespace svdq_dev {

constexpr int QA_STAGES = 4;
constexpr int QA_QWARPS = 8;
constexpr int QA_THREADS = 32 * (2 + QA_QWARPS);
constexpr uint32_t QA_X_BYTES = 128 * 128;  // 128 rows x 64 bf16

struct QAParams {
  const float* smooth;
  uint8_t* codes_x;
  uint8_t* sf_x;
  uint16_t* xl1;
  int M, K, r, klr;
  int chunks_per_split;
  int num_splits;
  uint32_t stage_bytes;
  uint32_t tmem_cols;
  float g_x, lr_scale;
  uint64_t timeout_ns;
};

__host__ __device__ inline uint32_t qa_stage_bytes(int r) {
  const uint32_t b = QA_X_BYTES + 256u * (uint32_t)r + 256u;
  return (b + 1023u) & ~1023u;
}
__host__ __device__ inline uint32_t qa_smem_bytes(int r) {
  return 1024u + QA_STAGES * qa_stage_bytes(r) + 256u;
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

__global__ void __launch_bounds__(QA_THREADS, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const QAParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int r = p.r;
  const bool has_lr = r > 0;
  const uint32_t SB = p.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + QA_STAGES * SB);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * QA_STAGES;
  const uint32_t acc_full = full0 + 16 * QA_STAGES;
  const uint32_t drain_bar = acc_full + 8;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * QA_STAGES + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x;
  const int rb = blockIdx.y;
  const int kchunks = p.K >> 6;
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(kchunks, c_begin + p.chunks_per_split);
  const int nchunks = max(0, c_end - c_begin);
  const unsigned int kid = 1;  // kernel id in error codes

  if (threadIdx.x == 0) {
    for (int i = 0; i < QA_STAGES; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, QA_QWARPS + (has_lr ? 1 : 0));
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = has_lr ? *tmem_holder : 0u;

  int issued = 0;  // producer: chunks whose loads were issued
  if (warp == 0) {
    // ---------------------------------------------------- TMA producer ----
    if (lane == 0) {
      const uint32_t tx = QA_X_BYTES + (has_lr ? 256u * r : 0u) + 256u;
      for (int i = 0; i < nchunks; ++i) {
        const int st = i % QA_STAGES;
        const uint32_t ph = (i / QA_STAGES) & 1;
        if (!mbar_wait(empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (1u << 8) | kid)) break;
        const uint32_t sb = smem_u32(smem + st * SB);
        const int c = c_begin + i;
        mbar_arrive_expect_tx(full0 + 8 * st, tx);
        tma_load_2d(sb, &tm_x, c * 64, rb * 128, full0 + 8 * st);
        if (has_lr) tma_load_2d(sb + QA_X_BYTES, &tm_l1, c * 64, 0, full0 + 8 * st);
        bulk_load(sb + QA_X_BYTES + 256u * r, p.smooth + c * 64, 256, full0 + 8 * st);
        issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------- down-projection ----
    if (has_lr && lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 2 * r);
      for (int i = 0; i < nchunks; ++i) {
        const int st = i % QA_STAGES;
        const uint32_t ph = (i / QA_STAGES) & 1;
        if (!mbar_wait(full0 + 8 * st, ph, p.timeout_ns, abort_flag, (2u << 8) | kid)) break;
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + st * SB);
        const uint64_t da = sdesc_sw128(sb), db = sdesc_sw128(sb + QA_X_BYTES);
        for (int kk = 0; kk < 4; ++kk)  // K = 16 bf16 = 32 bytes per MMA
          mma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (i | kk) != 0 ? 1u : 0u);
        tc_commit(empty0 + 8 * st);
      }
      tc_commit(acc_full);
    }
  } else {
    // ---------------------------------------------- NVFP4 quantization ----
    const int qw = warp - 2;
    const int row_t = qw * 16 + (lane >> 1);
    const int h = lane & 1;
    const int row = rb * 128 + row_t;
    const float g = p.g_x;
    for (int i = 0; i < nchunks; ++i) {
      const int st = i % QA_STAGES;
      const uint32_t ph = (i / QA_STAGES) & 1;
      if (!mbar_wait(full0 + 8 * st, ph, p.timeout_ns, abort_flag, (3u << 8) | kid)) break;
      const uint8_t* sb = smem + st * SB;
      const int c = c_begin + i;
      uint4 xw[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int phys = (4 * h + jj) ^ (row_t & 7);  // 128-byte swizzle
        xw[jj] = *reinterpret_cast<const uint4*>(sb + row_t * 128 + phys * 16);
      }
      const float4* sp = reinterpret_cast<const float4*>(sb + QA_X_BYTES + 256u * r) + 8 * h;
      float v[2][16];
      float amax[2];
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const uint32_t w[8] = {xw[2 * gi].x,     xw[2 * gi].y,     xw[2 * gi].z,
                               xw[2 * gi].w,     xw[2 * gi + 1].x, xw[2 * gi + 1].y,
                               xw[2 * gi + 1].z, xw[2 * gi + 1].w};
        float a = 0.0f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const float4 s4 = sp[4 * gi + q4];
          const float sv[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int idx = 4 * q4 + e;
            const uint32_t word = w[idx >> 1];
            const float x = (idx & 1) ? bf16_hi_f32(word) : bf16_lo_f32(word);
            const float xs = __fmul_rn(x, sv[e]);
            v[gi][idx] = xs;
            a = fmaxf(a, fabsf(xs));
          }
        }
        amax[gi] = __fmul_rn(__fdiv_rn(a, 6.0f), g);
      }
      const uint32_t sf2 = cvt_e4m3x2(amax[0], amax[1]);
      uint32_t cw[4];
#pragma unroll
      for (int gi = 0; gi < 2; ++gi) {
        const uint32_t code = (sf2 >> (8 * gi)) & 0xFF;
        const float q = code == 0 ? 0.0f : __fdiv_rn(g, e4m3_to_f32(code));
        float t0[8], t1[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          t0[e] = __fmul_rn(v[gi][e], q);
          t1[e] = __fmul_rn(v[gi][8 + e], q);
        }
        cw[2 * gi] = cvt_e2m1x8(t0);
        cw[2 * gi + 1] = cvt_e2m1x8(t1);
      }
      if (row < p.M) {
        uint4* dst = reinterpret_cast<uint4*>(p.codes_x + (size_t)row * (p.K >> 1) + c * 32 + h * 16);
        *dst = make_uint4(cw[0], cw[1], cw[2], cw[3]);
      }
      // scales of groups 4c+2h and 4c+2h+1 are adjacent bytes of one word
      *reinterpret_cast<uint16_t*>(p.sf_x + sf_tile_off(row, 4 * c + 2 * h, p.K)) = (uint16_t)sf2;
      __syncwarp();
      if (lane == 0) mbar_arrive(empty0 + 8 * st);
    }

    // ----------------------------------------- low-rank epilogue (X L1) ----
    if (has_lr) {
      const bool ok = mbar_wait(acc_full, 0, p.timeout_ns, abort_flag, (4u << 8) | kid);
      tc_fence_after();
      const int quad = warp & 3;            // tensor-memory lane quarter
      const int hc = (warp - 2) >> 2;       // which half of the 16-wide chunks
      const int lrow_t = quad * 32 + lane;
      const int lrow = rb * 128 + lrow_t;
      const int S = p.num_splits;
      float* P = reinterpret_cast<float*>(smem);  // [128][r+1], reuses the ring
      const int pstride = r + 1;
      // every quantize warp is done reading the ring before it is reused
      asm volatile("bar.sync 1, %0;" ::"n"(32 * QA_QWARPS) : "memory");
      for (int ci = hc; ci < r / 16; ci += 2) {
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
        if (S > 1) {
#pragma unroll
          for (int j = 0; j < 16; ++j) P[lrow_t * pstride + 16 * ci + j] = part[j];
        } else if (lrow < p.M) {
          uint32_t ph2[8], pl2[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float h0, l0, h1, l1;
            split_hi_lo(__fmul_rn(part[2 * j], p.lr_scale), h0, l0);
            split_hi_lo(__fmul_rn(part[2 * j + 1], p.lr_scale), h1, l1);
            ph2[j] = pack_bf16x2(h0, h1);
            pl2[j] = pack_bf16x2(l0, l1);
          }
          uint4* dh = reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + 16 * ci);
          uint4* dl = reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + r + 16 * ci);
          dh[0] = make_uint4(ph2[0], ph2[1], ph2[2], ph2[3]);
          dh[1] = make_uint4(ph2[4], ph2[5], ph2[6], ph2[7]);
          dl[0] = make_uint4(pl2[0], pl2[1], pl2[2], pl2[3]);
          dl[1] = make_uint4(pl2[4], pl2[5], pl2[6], pl2[7]);
        }
      }
      if (S == 1 && hc == 0 && lrow < p.M) {
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
      const int quad = warp & 3;
      const int hc = (warp - 2) >> 2;
      const int lrow_t = quad * 32 + lane;
      const int lrow = rb * 128 + lrow_t;
      const int pstride = r + 1;
      const uint32_t Pbase = smem_u32(smem);
      if (lrow < p.M) {
        for (int ci = hc; ci < r / 16; ci += 2) {
          float acc[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) acc[j] = 0.0f;
          for (int s = 0; s < p.num_splits; ++s) {
            const uint32_t rbase = map_to_rank(Pbase, (uint32_t)s);
#pragma unroll
            for (int j = 0; j < 16; ++j)
              acc[j] += ld_cluster_f32(rbase + 4u * (uint32_t)(lrow_t * pstride + 16 * ci + j));
          }
          uint32_t ph2[8], pl2[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            float h0, l0, h1, l1;
            split_hi_lo(__fmul_rn(acc[2 * j], p.lr_scale), h0, l0);
            split_hi_lo(__fmul_rn(acc[2 * j + 1], p.lr_scale), h1, l1);
            ph2[j] = pack_bf16x2(h0, h1);
            pl2[j] = pack_bf16x2(l0, l1);
          }
          uint4* dh = reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + 16 * ci);
          uint4* dl = reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + r + 16 * ci);
          dh[0] = make_uint4(ph2[0], ph2[1], ph2[2], ph2[3]);
          dh[1] = make_uint4(ph2[4], ph2[5], ph2[6], ph2[7]);
          dl[0] = make_uint4(pl2[0], pl2[1], pl2[2], pl2[3]);
          dl[1] = make_uint4(pl2[4], pl2[5], pl2[6], pl2[7]);
        }
        if (hc == 0)
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
      for (int i = max(0, issued - QA_STAGES); i < issued; ++i)
        mbar_wait_drain(full0 + 8 * (i % QA_STAGES), (i / QA_STAGES) & 1, p.timeout_ns);
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
