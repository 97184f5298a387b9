// 4-bit GEMM kernel of the SVDQuant W4A4 linear with the fused low-rank
// up-projection, bias and bf16 store.
//
// The fusion follows the Nunchaku engine as described in the Korean
// rendering of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"
// (section "SVDQuant and the Nunchaku engine"): the low-rank up projection is
// merged into the 4-bit compute kernel.  The B200 design:
//
//   * CTA pairs (thread-block clusters of 2) share one tensor-core MMA
//     (tcgen05 cta_group::2): a pair computes a 256 x 192 output tile, each
//     CTA holds its 128 rows of the activation codes and half (96 rows) of
//     the weight codes in its own shared memory and its 128 rows of the fp32
//     accumulator in its own tensor memory;
//   * two accumulators (tensor-memory columns [0, 192) and [192, 384)): the
//     MMA works on tile t + 1 while the epilogue drains tile t, so the
//     tensor core never waits for a tile boundary.  The per-stage scale
//     factors take the columns after them ([384, 480), double-buffered);
//   * warp 0 of each CTA (the whole warp waits, one elected lane issues)
//     streams, per 256-deep K step, its A and B code tiles (TMA, 128-byte
//     swizzle) and the scale atoms (its own 128 rows of activation scales,
//     all 192 (padded to 256) rows of weight scales) into a 5-deep ring;
//     every load is counted on the leader CTA's barrier (cta_group::2 form,
//     no multicast);
//   * warp 1 of the leader (converged; an elected lane issues each
//     instruction) copies the scale atoms into both CTAs' tensor memory
//     (tcgen05.cp cta_group::2) and issues
//     tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 (M = 256,
//     N = 192, K = 64); after the K loop it streams the low-rank operands
//     (xl1 hi|lo and L2, bf16) through the same ring into the SAME
//     accumulator with kind::f16 MMAs (xl1 was pre-multiplied by
//     g_x g_w = 1/alpha); completions are multicast to both CTAs;
//   * warps 2..13 of each CTA: warp w drains tensor-memory lane quarter
//     w % 4, columns [64 c, 64 c + 64) with c = (w - 2) / 4, releases the
//     accumulator to the leader, then computes Y = bf16(alpha * acc + bias)
//     (bias staged per tile in shared memory).  The four warps of one column
//     group write a 128-row x 64-column box into a 16 KB shared-memory
//     buffer (128-byte swizzle: a thread's row of 128 bytes lands in eight
//     different bank groups across each eight rows) that one thread stores
//     with TMA.
//
// Weight scales: each 192-row tile of the weight has its own two atom rows
// (128 + 64 rows, padded with 64 zero rows), so a tile's scales are two
// whole 512-byte atoms per 64-deep K step.  In row terms: weight row n sits
// at row (n / 192) * 256 + n % 192 of the atom layout.
#pragma once
#include "ptx.cuh"

namespace svdq_dev {

constexpr int G_STAGES = 5;
constexpr int G_EPI_WARPS = 12;
constexpr int G_THREADS = 32 * (2 + G_EPI_WARPS);
constexpr int G_BM = 128;                    // rows per CTA (pair tile: 256)
constexpr int G_BN = 192;                    // columns per pair tile (MMA N)
constexpr int G_BN_CTA = 96;                 // weight rows held per CTA
constexpr int G_SFB_ROWS = 256;              // weight-scale rows per tile (padded)
constexpr uint32_t G_A_BYTES = 128 * 128;    // 128 rows x 128 B
constexpr uint32_t G_B_BYTES = 96 * 128;     // 96 rows x 128 B
constexpr uint32_t G_SFA_BYTES = 4 * 512;    // 4 atoms (K = 256)
constexpr uint32_t G_SFB_BYTES = 8 * 512;    // 2 atom rows x 4 atoms
constexpr uint32_t G_STAGE_BYTES = G_A_BYTES + G_B_BYTES + G_SFA_BYTES + G_SFB_BYTES;
constexpr uint32_t G_TMEM_COLS = 512;
constexpr uint32_t G_ACC_STRIDE = G_BN;      // accumulator b at columns [192 b, 192 b + 192)
constexpr uint32_t G_SF_TMEM = 2 * G_BN;     // 384: scale buffers after the accumulators
constexpr uint32_t G_SF_TMEM_STRIDE = 48;    // 16 cols SFA + 32 cols SFB per stage
static_assert(G_SF_TMEM + 2 * G_SF_TMEM_STRIDE <= G_TMEM_COLS, "tensor memory plan");
constexpr uint32_t G_BIAS_BYTES = 2 * G_BN * 4;   // two fp32 bias tiles
constexpr int G_OUT_COLS = 64;                    // columns per output box (128 bytes)
constexpr int G_OUT_BOXES = G_BN / G_OUT_COLS;    // 3
constexpr uint32_t G_OUT_BOX_BYTES = G_BM * 128;  // one box: 128 rows x 128 bytes
constexpr uint32_t G_OUT_BYTES = G_OUT_BOXES * G_OUT_BOX_BYTES;
constexpr uint32_t G_FP4_TX = 2 * G_STAGE_BYTES;  // bytes per FP4 stage, both CTAs
constexpr uint32_t G_LR_TX = 2 * (G_A_BYTES + G_B_BYTES);
static_assert(G_EPI_WARPS == 4 * G_OUT_BOXES, "one warp per lane quarter and column box");

__host__ __device__ inline uint32_t gemm_smem_bytes() {
  return 1024u + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES + G_BIAS_BYTES + 256u;  // + barriers
}
static_assert(1024u + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES + G_BIAS_BYTES + 256u <= 232448u,
              "GEMM shared memory above the 227 KB a CTA may use");
static_assert((G_STAGES * G_STAGE_BYTES) % 1024 == 0, "output boxes need 1024-byte alignment");

struct GemmParams {
  const uint16_t* bias;
  int M, N, K, r, klr;
  float alpha;
  uint64_t timeout_ns;
};

__global__ void __launch_bounds__(G_THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_sfa,
                     const __grid_constant__ CUtensorMap tm_sfb,
                     const __grid_constant__ CUtensorMap tm_alr,
                     const __grid_constant__ CUtensorMap tm_blr,
                     const __grid_constant__ CUtensorMap tm_y, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t out_s = smem_u32(smem + G_STAGES * G_STAGE_BYTES);  // [3][128 rows][128 B]
  float* bias_s =
      reinterpret_cast<float*>(smem + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES);  // [2][192]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES +
                                               G_BIAS_BYTES);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * G_STAGES;
  const uint32_t acc_full0 = full0 + 16 * G_STAGES;   // two: one per accumulator
  const uint32_t acc_empty0 = acc_full0 + 16;         // two
  const uint32_t drain_bar = acc_full0 + 32;
  const uint32_t bias_bar0 = acc_full0 + 40;          // two: one per bias buffer
  const uint32_t peer_bar = acc_full0 + 56;           // the pair CTA's final load count
  // per output box: "staged" (its 4 warps wrote it) and "free" (the store
  // issued from it has finished reading it)
  const uint32_t out_staged0 = acc_full0 + 64;        // three
  const uint32_t out_free0 = out_staged0 + 8 * G_OUT_BOXES;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * G_STAGES + 8 + 2 * G_OUT_BOXES);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  volatile int* peer_issued = reinterpret_cast<volatile int*>(tmem_holder + 2);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();      // 0 = leader of the pair
  const bool leader = rank == 0;
  const int M = p.M, N = p.N, K = p.K, r = p.r;
  const bool has_lr = r > 0;
  const int num_m = (M + 2 * G_BM - 1) / (2 * G_BM);
  const int num_n = (N + G_BN - 1) / G_BN;
  const int num_tiles = num_m * num_n;
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  // Each pair takes a contiguous run of tiles in M-major order (tile t is
  // M block t / num_n, N block t % num_n): consecutive tiles share their
  // activation rows, which then mostly come from L2.
  const int t_begin = (int)(((long long)pair * num_tiles) / num_pairs);
  const int t_end = (int)(((long long)(pair + 1) * num_tiles) / num_pairs);
  const int k64 = K >> 6;
  const int kb_total = (k64 + 3) >> 2;
  const int lr_chunks = has_lr ? (p.klr >> 6) : 0;
  const unsigned int kid = 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G_STAGES; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full0 + 8 * b, 1);
      mbar_init(acc_empty0 + 8 * b, 2 * G_EPI_WARPS);
      mbar_init(bias_bar0 + 8 * b, 32 * G_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    mbar_init(peer_bar, 1);
    for (int h = 0; h < G_OUT_BOXES; ++h) {
      mbar_init(out_staged0 + 8 * h, 4);
      mbar_init(out_free0 + 8 * h, 1);
    }
    *abort_flag = 0;
    *peer_issued = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    prefetch_tensormap(&tm_sfa);
    prefetch_tensormap(&tm_sfb);
    prefetch_tensormap(&tm_y);
    if (has_lr) {
      prefetch_tensormap(&tm_alr);
      prefetch_tensormap(&tm_blr);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(tmem_holder), G_TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  const uint32_t lead_full0 = map_to_rank(full0, 0);
  const uint32_t lead_acc_empty0 = map_to_rank(acc_empty0, 0);
  // The prologue above overlaps the previous kernel; the activation codes,
  // scales and low-rank operand it produced are read only after this.
  grid_dependency_wait();
  grid_launch_dependents();

  int issued = 0;
  if (warp == 0) {
    // ---------------------------------------------- TMA producer (warp) ----
    int it = 0;
    bool stop = false;
    for (int tile = t_begin; tile < t_end && !stop; ++tile) {
      const int mb = tile / num_n, nb = tile % num_n;
      const int row0 = mb * 2 * G_BM + (int)rank * G_BM;     // this CTA's A rows
      const int brow0 = nb * G_BN + (int)rank * G_BN_CTA;    // this CTA's B rows
      const int sfa_blk = mb * 2 + (int)rank;                // 128-row scale block
      for (int kb = 0; kb < kb_total; ++kb, ++it) {
        const int st = it % G_STAGES;
        const uint32_t ph = (it / G_STAGES) & 1;
        if (!mbar_wait_warp(empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (1u << 8) | kid)) {
          stop = true;
          break;
        }
        if (elect_one()) {
          const uint32_t sb = smem_u32(smem + st * G_STAGE_BYTES);
          if (leader) mbar_arrive_expect_tx(full0 + 8 * st, G_FP4_TX);
          const uint32_t fb = lead_full0 + 8 * st;
          tma_load_2d_pair(sb, &tm_a, kb * 128, row0, fb);
          tma_load_2d_pair(sb + G_A_BYTES, &tm_b, kb * 128, brow0, fb);
          // scale atoms: rows of 256 bytes = half atoms; 4 atoms = 8 rows
          tma_load_2d_pair(sb + G_A_BYTES + G_B_BYTES, &tm_sfa, 0, (sfa_blk * k64 + 4 * kb) * 2,
                           fb);
          for (int hh = 0; hh < 2; ++hh)
            tma_load_2d_pair(sb + G_A_BYTES + G_B_BYTES + G_SFA_BYTES + hh * 2048, &tm_sfb, 0,
                             ((2 * nb + hh) * k64 + 4 * kb) * 2, fb);
        }
        __syncwarp();
        issued = it + 1;
      }
      for (int c = 0; c < lr_chunks && !stop; ++c, ++it) {
        const int st = it % G_STAGES;
        const uint32_t ph = (it / G_STAGES) & 1;
        if (!mbar_wait_warp(empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (1u << 8) | kid)) {
          stop = true;
          break;
        }
        if (elect_one()) {
          const uint32_t sb = smem_u32(smem + st * G_STAGE_BYTES);
          if (leader) mbar_arrive_expect_tx(full0 + 8 * st, G_LR_TX);
          const uint32_t fb = lead_full0 + 8 * st;
          tma_load_2d_pair(sb, &tm_alr, c * 64, row0, fb);
          tma_load_2d_pair(sb + G_A_BYTES, &tm_blr, c * 64, brow0, fb);
        }
        __syncwarp();
        issued = it + 1;
      }
    }
    // The peer CTA's loads complete on the leader's barriers: it tells the
    // leader how many stages it issued (remote store, then a remote arrive
    // that releases it), so an aborted leader can drain them all.
    if (!leader && lane == 0) {
      st_cluster_u32(map_to_rank(smem_u32((const void*)peer_issued), 0), (uint32_t)issued);
      mbar_arrive_release_cluster(map_to_rank(peer_bar, 0));
    }
    __syncwarp();
  } else if (warp == 1) {
    // -------------------------------------- MMA issuer (leader, warp) ----
    if (leader) {
      const uint32_t id_fp4 = idesc_nvfp4(2 * G_BM, G_BN);
      const uint32_t id_lr = idesc_bf16(2 * G_BM, G_BN);
      int it = 0, tcount = 0;
      bool stop = false;
      // `ready`: the stage `it` was already seen full by a non-blocking test
      // made right after the previous stage was issued (its latency then
      // overlaps the tensor-core work instead of preceding the next issue)
      bool ready = false;
      for (int tile = t_begin; tile < t_end && !stop; ++tile, ++tcount) {
        const int ab = tcount & 1;                 // accumulator of this tile
        const uint32_t acc = tmem + (uint32_t)ab * G_ACC_STRIDE;
        // the accumulator is free once the epilogue has drained the tile
        // that used it two tiles ago
        if (!mbar_wait_warp(acc_empty0 + 8 * ab, ((tcount >> 1) & 1) ^ 1, p.timeout_ns, abort_flag,
                            (2u << 8) | kid))
          break;
        tc_fence_after();
        for (int kb = 0; kb < kb_total; ++kb, ++it) {
          const int st = it % G_STAGES;
          const uint32_t ph = (it / G_STAGES) & 1;
          // the stage's TMA bytes have landed (complete_tx); the MMAs and
          // scale copies below read them through the async proxy
          if (!ready &&
              !mbar_wait_warp(full0 + 8 * st, ph, p.timeout_ns, abort_flag, (3u << 8) | kid)) {
            stop = true;
            break;
          }
          const uint32_t sb = smem_u32(smem + st * G_STAGE_BYTES);
          const uint32_t sfa_s = sb + G_A_BYTES + G_B_BYTES;
          const uint32_t sfb_s = sfa_s + G_SFA_BYTES;
          const uint32_t sfa_t = tmem + G_SF_TMEM + (it & 1) * G_SF_TMEM_STRIDE;
          const uint32_t sfb_t = sfa_t + 16;
          // Every stage runs all four 64-deep steps, fixed and fully
          // unrolled: a loop bounded at run time (or a per-step guard) around
          // elect.sync here cut the issue rate by up to half.  A short last
          // stage (K % 256 != 0) reads zero codes past K (TMA fill) against
          // finite scales, which adds exactly zero.
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              tmem_copy_32x128b_x4_pair(sfa_t + 4 * kk, sdesc_sf_block(sfa_s + 512 * kk));
              tmem_copy_32x128b_x4_pair(sfb_t + 8 * kk, sdesc_sf_block(sfb_s + 512 * kk));
              tmem_copy_32x128b_x4_pair(sfb_t + 8 * kk + 4,
                                        sdesc_sf_block(sfb_s + 2048 + 512 * kk));
            }
          }
          __syncwarp();
          const uint64_t da = sdesc_sw128(sb), db = sdesc_sw128(sb + G_A_BYTES);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {  // K = 64 E2M1 = 32 bytes per MMA
            if (elect_one())
              mma_nvfp4_pair(acc, da + 2 * kk, db + 2 * kk, id_fp4, sfa_t + 4 * kk,
                             sfb_t + 8 * kk, (kb | kk) > 0 ? 1u : 0u);
            __syncwarp();
          }
          ready = mbar_test_warp(full0 + 8 * ((it + 1) % G_STAGES), ((it + 1) / G_STAGES) & 1);
          if (elect_one()) tc_commit_pair(empty0 + 8 * st, 0x3);
          __syncwarp();
        }
        for (int c = 0; c < lr_chunks && !stop; ++c, ++it) {
          const int st = it % G_STAGES;
          const uint32_t ph = (it / G_STAGES) & 1;
          if (!ready &&
              !mbar_wait_warp(full0 + 8 * st, ph, p.timeout_ns, abort_flag, (3u << 8) | kid)) {
            stop = true;
            break;
          }
          const uint32_t sb = smem_u32(smem + st * G_STAGE_BYTES);
          const uint64_t da = sdesc_sw128(sb), db = sdesc_sw128(sb + G_A_BYTES);
          // four 16-deep bf16 steps; columns [2r, klr) of both operands are
          // zeros, so a partial last chunk adds exactly zero
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            if (elect_one()) mma_bf16_pair(acc, da + 2 * kk, db + 2 * kk, id_lr, 1u);
            __syncwarp();
          }
          ready = mbar_test_warp(full0 + 8 * ((it + 1) % G_STAGES), ((it + 1) / G_STAGES) & 1);
          if (elect_one()) tc_commit_pair(empty0 + 8 * st, 0x3);
          __syncwarp();
        }
        if (elect_one()) tc_commit_pair(acc_full0 + 8 * ab, 0x3);
        __syncwarp();
      }
    }
  } else {
    // -------------------------------------------------------- epilogue ----
    const int quad = warp & 3;                 // tensor-memory lane quarter
    const int cg = (warp - 2) >> 2;            // column box: [64 cg, 64 cg + 64)
    const int et = threadIdx.x - 64;           // 0 .. 32 G_EPI_WARPS - 1
    const float alpha = p.alpha;
    const int row_t = quad * 32 + lane;        // this thread's row of the CTA's 128
    const uint32_t obuf = out_s + cg * G_OUT_BOX_BYTES;
    const uint32_t staged = out_staged0 + 8 * cg, freed = out_free0 + 8 * cg;
    // one thread per column box issues its bulk stores
    const bool issuer = ((warp - 2) & 3) == 0 && lane == 0;
    int tcount = 0;
    bool ok = true;
    for (int tile = t_begin; tile < t_end && ok; ++tile, ++tcount) {
      const int mb = tile / num_n, nb = tile % num_n;
      const int ab = tcount & 1;
      // stage this tile's bias (fp32) while the main loop runs.  Buffer
      // tcount&1 was last read for tile tcount-2, which every thread had
      // finished before arriving on the other buffer's barrier.
      float* bt = bias_s + (tcount & 1) * G_BN;
      const uint32_t bb = bias_bar0 + 8 * (tcount & 1);
      if (et < G_BN) {
        const int n = nb * G_BN + et;
        bt[et] = (p.bias && n < N) ? bf16_lo_f32(p.bias[n]) : 0.0f;
      }
      mbar_arrive(bb);
      if (!mbar_wait_warp(bb, (tcount >> 1) & 1, p.timeout_ns, abort_flag, (5u << 8) | kid)) break;
      if (!mbar_wait_warp(acc_full0 + 8 * ab, (tcount >> 1) & 1, p.timeout_ns, abort_flag,
                          (4u << 8) | kid))
        break;
      tc_fence_after();
      const uint32_t tbase =
          tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)ab * G_ACC_STRIDE + cg * G_OUT_COLS;
      uint32_t acc[2][32];
      tmem_ld32(tbase, acc[0]);
      tmem_ld32(tbase + 32, acc[1]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_acc_empty0 + 8 * ab);   // accumulator free again
      const int row0 = mb * 2 * G_BM + (int)rank * G_BM;   // first row of this CTA's box
      // the box buffer is free once the store issued from it has read it
      if (tcount > 0) {
        if (issuer) {
          bulk_wait_read_all();
          mbar_arrive(freed);
        }
        __syncwarp();
        if (!mbar_wait_warp(freed, (tcount - 1) & 1, p.timeout_ns, abort_flag, (7u << 8) | kid)) {
          ok = false;
          break;
        }
      }
      // 64 columns of this thread's row: 8 chunks of 16 bytes, chunk j at
      // slot j ^ (row % 8) of the row's 128 bytes (the 128-byte swizzle)
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int ch = j >> 2;
        const int cb = 8 * (j & 3);
        const int c0 = cg * G_OUT_COLS + ch * 32 + cb;
        uint32_t o[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float y0 = fmaf(alpha, __uint_as_float(acc[ch][cb + 2 * q]), bt[c0 + 2 * q]);
          const float y1 = fmaf(alpha, __uint_as_float(acc[ch][cb + 2 * q + 1]), bt[c0 + 2 * q + 1]);
          o[q] = pack_bf16x2(y0, y1);
        }
        st_shared_v4(obuf + row_t * 128 + ((j ^ (row_t & 7)) << 4), o[0], o[1], o[2], o[3]);
      }
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(staged);
      if (issuer) {
        const int x = nb * G_BN + cg * G_OUT_COLS;
        // a box wholly past N or M has nothing to write
        if (mbar_wait(staged, tcount & 1, p.timeout_ns, abort_flag, (8u << 8) | kid)) {
          if (x < N && row0 < M) {
            tma_store_2d(&tm_y, obuf, x, row0);
          }
          bulk_commit_group();
        } else {
          ok = false;
        }
      }
      ok = __all_sync(0xffffffffu, ok) != 0;   // the issuer's verdict, warp-wide
    }
    // no store may still be reading shared memory (or writing Y) at exit
    if (issuer) bulk_wait_all();
  }

  // ------------------------------------------------------------ teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // The leader's barriers count both CTAs' loads.  Drain the stages either
    // CTA issued: the peer reports its count (bounded wait); a stage only the
    // peer issued was never armed here, so arm it with the peer's bytes.
    if (leader && warp == 0 && lane == 0) {
      mbar_wait_drain_cluster(peer_bar, 0, p.timeout_ns);
      const int peer = *peer_issued;
      const int hi = max(issued, peer);
      for (int i = max(0, hi - G_STAGES); i < hi; ++i) {
        const uint32_t fb = full0 + 8 * (i % G_STAGES);
        if (i >= issued) {
          // the stage's kind follows from its position in the tile sequence
          const int per_tile = kb_total + lr_chunks;
          const bool lr_stage = (i % per_tile) >= kb_total;
          mbar_arrive_expect_tx(fb, (lr_stage ? G_LR_TX : G_FP4_TX) / 2);
        }
        mbar_wait_drain(fb, (i / G_STAGES) & 1, p.timeout_ns);
      }
    }
    if (leader && warp == 1) {
      // the commit must come from the lane that issued the MMAs: elect.sync
      // over the full warp picks the same lane every time
      if (elect_one()) {
        tc_commit_pair(drain_bar, 0x1);
        mbar_wait_drain(drain_bar, 0, p.timeout_ns);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  cluster_sync();  // the pair is done with shared and tensor memory
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, G_TMEM_COLS);
  }
}

}  // namespace svdq_dev
