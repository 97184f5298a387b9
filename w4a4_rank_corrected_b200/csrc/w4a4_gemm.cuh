// 4-bit GEMM kernel of the SVDQuant W4A4 linear with the fused low-rank
// up-projection, bias and bf16 store.
//
// The fusion follows the Nunchaku engine as described in the Korean
// rendering of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"
// (section "SVDQuant and the Nunchaku engine"): the low-rank up projection is
// merged into the 4-bit compute kernel.  The B200 design:
//
//   * CTA pairs (thread-block clusters of 2) share one tensor-core MMA
//     (tcgen05 cta_group::2): a pair computes a 256 x 256 output tile, each
//     CTA holds its 128 rows of the activation codes and half (128 rows) of
//     the weight codes in its own shared memory and its 128 rows of the fp32
//     accumulator in its own tensor memory.  Per unit of MMA work each SM
//     moves half the weight bytes through shared memory that a single-SM
//     128 x 256 tile would, which is what keeps the tensor core fed;
//   * warp 0 of each CTA (the whole warp waits, one elected lane issues)
//     streams, per 256-deep K step, its A and B code tiles
//     (TMA, 128-byte swizzle) and the scale atoms (TMA; its own 128 rows of
//     activation scales, all 256 rows of weight scales) into a 5-deep ring;
//     every load is counted on the leader CTA's barrier (cta_group::2 form,
//     no multicast);
//   * each pair works through a contiguous run of output tiles in M-major
//     order; for K <= 3072 the activation scales of the current 256-row
//     block stay in tensor memory (192 columns beside the 256-column
//     accumulator) and are loaded and copied only when the run enters a new
//     row block, which takes a third of the scale copies off the MMA
//     issuer's path (each copy beyond about one per MMA stalls it);
//   * warp 1 of the leader (converged; an elected lane issues each
//     instruction) copies the scale atoms into both CTAs' tensor
//     memory (tcgen05.cp cta_group::2) and issues
//     tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.block16 (M = 256,
//     N = 256, K = 64); after the K loop it streams the low-rank operands
//     (xl1 hi|lo and L2, bf16) through the same ring into the SAME
//     accumulator with kind::f16 MMAs (xl1 was pre-multiplied by
//     g_x g_w = 1/alpha); completions are multicast to both CTAs;
//   * warps 2..9 of each CTA drain its accumulator (four 32-column
//     tcgen05.ld, one wait), release it to the leader, and only then compute
//     Y = bf16(alpha * acc + bias) (bias staged per tile in shared memory),
//     overlapping the next tile's main loop.  Each group of four warps owns
//     128 columns and writes them as two 128-row x 64-column boxes through a
//     16 KB shared-memory buffer (128-byte swizzle, so the row-per-thread
//     writes are free of bank conflicts) that one thread stores with TMA:
//     one bulk store per box instead of a 16-byte global store per thread
//     and row, which scattered each warp instruction over 32 rows and held
//     the MMA issuer back.
#pragma once
#include "gelu.cuh"
#include "ptx.cuh"
#include "row_scales.cuh"

namespace svdq_dev {

constexpr int G_STAGES = 5;
constexpr int G_EPI_WARPS = 8;
constexpr int G_THREADS = 32 * (2 + G_EPI_WARPS);
constexpr int G_BM = 128;                    // rows per CTA (pair tile: 256)
constexpr int G_BN = 256;                    // columns per pair tile (MMA N)
constexpr int G_BN_CTA = 128;                // weight rows held per CTA
constexpr uint32_t G_A_BYTES = 128 * 128;    // 128 rows x 128 B
constexpr uint32_t G_B_BYTES = 128 * 128;    // 128 rows x 128 B
constexpr uint32_t G_SFA_BYTES = 4 * 512;    // 4 atoms (K = 256)
constexpr uint32_t G_SFB_BYTES = 8 * 512;    // 2 row blocks x 4 atoms
constexpr uint32_t G_STAGE_BYTES = G_A_BYTES + G_B_BYTES + G_SFA_BYTES + G_SFB_BYTES;
constexpr uint32_t G_TMEM_COLS = 512;
constexpr uint32_t G_SF_TMEM = 256;          // scale buffers after the accumulator
constexpr uint32_t G_SF_TMEM_STRIDE = 48;    // 16 cols SFA + 32 cols SFB
// Resident activation scales: 4 columns per 64-deep K step, all of K, for
// K <= 3072 (192 columns); then the weight scales double-buffer after them.
constexpr int G_SFA_RES_MAX_K64 = 48;
constexpr uint32_t G_SFB_RES_TMEM = G_SF_TMEM + 4 * G_SFA_RES_MAX_K64;  // 448
constexpr uint32_t G_SFB_RES_STRIDE = 32;
constexpr uint32_t G_BIAS_BYTES = 2 * G_BN * 4;   // two fp32 bias tiles
constexpr int G_OUT_COLS = 64;                    // columns per output box (128 bytes)
constexpr uint32_t G_OUT_HALF_BYTES = G_BM * 128; // one box: 128 rows x 128 bytes
constexpr uint32_t G_OUT_BYTES = 2 * G_OUT_HALF_BYTES;
constexpr uint32_t G_FP4_TX = 2 * G_STAGE_BYTES;  // bytes per FP4 stage, both CTAs
constexpr uint32_t G_FP4_TX_NOSFA = 2 * (G_STAGE_BYTES - G_SFA_BYTES);
constexpr uint32_t G_LR_TX = 2 * (G_A_BYTES + G_B_BYTES);

__host__ __device__ inline uint32_t gemm_smem_bytes() {
  return 1024u + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES + G_BIAS_BYTES + 256u;  // + barriers
}
static_assert(1024u + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES + G_BIAS_BYTES + 256u <= 232448u,
              "GEMM shared memory above the 227 KB a CTA may use");
static_assert((G_STAGES * G_STAGE_BYTES) % 1024 == 0, "output boxes need 1024-byte alignment");
static_assert((2 * G_STAGES + 12) * 8 <= 256, "barriers and words past the 256-byte barrier area");

struct GemmParams {
  const uint16_t* bias;
  int M, N, K, r, klr;
  float alpha;
  uint64_t timeout_ns;
  int gelu;          // 1: the epilogue writes GELU(bf16(y)) (first linear of an MLP pair)
  const RowScale* row_scales;   // per-row output scale alpha_m (dynamic mode) or NULL
  // split-K (few output tiles): each tile's K stages are split into ksplit
  // parts ("units"); every unit stores its fp32 partial accumulator instead
  // of Y, and splitk_reduce_kernel adds them in part order and writes Y
  int ksplit;                   // 1: no split
  float* partials;              // [tiles][ksplit][2 CTAs][128 rows][256 cols] fp32
};

// The 256-deep stages [lo, hi) of part `part` of a K split in `ksplit` parts.
__device__ __forceinline__ void split_stages(int part, int ksplit, int kb_total, int& lo, int& hi) {
  lo = (int)(((long long)part * kb_total) / ksplit);
  hi = (int)(((long long)(part + 1) * kb_total) / ksplit);
}

__global__ void __launch_bounds__(G_THREADS, 1)
    w4a4_gemm_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                     const __grid_constant__ CUtensorMap tm_sfa,
                     const __grid_constant__ CUtensorMap tm_sfb,
                     const __grid_constant__ CUtensorMap tm_alr,
                     const __grid_constant__ CUtensorMap tm_blr,
                     const __grid_constant__ CUtensorMap tm_y,
                     const __grid_constant__ CUtensorMap tm_part, const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t out_s = smem_u32(smem + G_STAGES * G_STAGE_BYTES);  // [2][128 rows][128 B]
  float* bias_s =
      reinterpret_cast<float*>(smem + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES);  // [2][256]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + G_STAGES * G_STAGE_BYTES + G_OUT_BYTES +
                                               G_BIAS_BYTES);
  const uint32_t full0 = smem_u32(bars);
  const uint32_t empty0 = full0 + 8 * G_STAGES;
  const uint32_t acc_full = full0 + 16 * G_STAGES;
  const uint32_t acc_empty = acc_full + 8;
  const uint32_t drain_bar = acc_full + 16;
  const uint32_t bias_bar0 = acc_full + 24;  // two: one per bias buffer
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * G_STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  // per output buffer: "staged" (its 4 warps wrote it) and "free" (the
  // store issued from it has finished reading it)
  const uint32_t out_staged0 = smem_u32(bars + 2 * G_STAGES + 6);
  const uint32_t out_free0 = out_staged0 + 16;
  // the pair CTA's final load count (error path): a barrier and a word
  const uint32_t peer_bar = smem_u32(bars + 2 * G_STAGES + 10);
  volatile int* peer_issued = reinterpret_cast<volatile int*>(bars + 2 * G_STAGES + 11);

  const uint32_t warp = warp_id(), lane = lane_id();
  const uint32_t rank = cluster_ctarank();      // 0 = leader of the pair
  const bool leader = rank == 0;
  const int M = p.M, N = p.N, K = p.K, r = p.r;
  const bool has_lr = r > 0;
  const int num_m = (M + 2 * G_BM - 1) / (2 * G_BM);
  const int num_n = (N + G_BN - 1) / G_BN;
  const int num_tiles = num_m * num_n;
  const int ksplit = p.ksplit > 1 ? p.ksplit : 1;
  const int num_units = num_tiles * ksplit;   // unit u: tile u / ksplit, part u % ksplit
  const int pair = blockIdx.x >> 1, num_pairs = gridDim.x >> 1;
  // Each pair takes a contiguous run of tiles in M-major order (tile t is
  // M block t / num_n, N block t % num_n), so consecutive tiles mostly share
  // their activation rows and those rows' scales stay in tensor memory.
  const int t_begin = (int)(((long long)pair * num_units) / num_pairs);   // this pair's units
  const int t_end = (int)(((long long)(pair + 1) * num_units) / num_pairs);
  const int k64 = K >> 6;
  const bool sfa_res = ksplit == 1 && k64 <= G_SFA_RES_MAX_K64;
  const int kb_total = (k64 + 3) >> 2;
  const int lr_chunks = has_lr ? (p.klr >> 6) : 0;
  const unsigned int kid = 2;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G_STAGES; ++i) {
      mbar_init(full0 + 8 * i, 1);
      mbar_init(empty0 + 8 * i, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * G_EPI_WARPS);
    mbar_init(drain_bar, 1);
    mbar_init(bias_bar0, 32 * G_EPI_WARPS);
    mbar_init(bias_bar0 + 8, 32 * G_EPI_WARPS);
    for (int h = 0; h < 2; ++h) {
      mbar_init(out_staged0 + 8 * h, G_EPI_WARPS / 2);
      mbar_init(out_free0 + 8 * h, 1);
    }
    mbar_init(peer_bar, 1);
    *peer_issued = 0;
    *abort_flag = 0;
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
  const uint32_t lead_acc_empty = map_to_rank(acc_empty, 0);
  // The prologue above overlaps the previous kernel; the activation codes,
  // scales and low-rank operand it produced are read only after this.
  grid_dependency_wait();
  grid_launch_dependents();

  int issued = 0;
  if (warp == 0) {
    // ---------------------------------------------- TMA producer (warp) ----
    int it = 0;
    bool stop = false;
    for (int u = t_begin; u < t_end && !stop; ++u) {
      const int tile = u / ksplit, part = u - tile * ksplit;
      int kb_lo, kb_hi;
      split_stages(part, ksplit, kb_total, kb_lo, kb_hi);
      const int lr_here = part == ksplit - 1 ? lr_chunks : 0;   // the low-rank stage: last part
      const int mb = tile / num_n, nb = tile % num_n;
      const bool load_sfa = !sfa_res || u == t_begin || nb == 0;
      const int row0 = mb * 2 * G_BM + (int)rank * G_BM;     // this CTA's A rows
      const int brow0 = nb * G_BN + (int)rank * G_BN_CTA;    // this CTA's B rows
      const int sfa_blk = mb * 2 + (int)rank;                // 128-row scale block
      for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
        const int st = it % G_STAGES;
        const uint32_t ph = (it / G_STAGES) & 1;
        if (!mbar_wait_warp(empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (1u << 8) | kid)) {
          stop = true;
          break;
        }
        if (elect_one()) {
          const uint32_t sb = smem_u32(smem + st * G_STAGE_BYTES);
          if (leader) mbar_arrive_expect_tx(full0 + 8 * st, load_sfa ? G_FP4_TX : G_FP4_TX_NOSFA);
          const uint32_t fb = lead_full0 + 8 * st;
          tma_load_2d_pair(sb, &tm_a, kb * 128, row0, fb);
          tma_load_2d_pair(sb + G_A_BYTES, &tm_b, kb * 128, brow0, fb);
          // scale atoms: rows of 256 bytes = half atoms; 4 atoms = 8 rows
          if (load_sfa)
            tma_load_2d_pair(sb + G_A_BYTES + G_B_BYTES, &tm_sfa, 0,
                             (sfa_blk * k64 + 4 * kb) * 2, fb);
          for (int hh = 0; hh < 2; ++hh)
            tma_load_2d_pair(sb + G_A_BYTES + G_B_BYTES + G_SFA_BYTES + hh * 2048, &tm_sfb, 0,
                             ((2 * nb + hh) * k64 + 4 * kb) * 2, fb);
        }
        __syncwarp();
        issued = it + 1;
      }
      for (int c = 0; c < lr_here && !stop; ++c, ++it) {
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
    // The other CTA's loads complete on the leader's barriers: it reports
    // how many stages it issued (remote store, then a remote arrive that
    // releases it), so an aborted leader can drain every one of them.
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
      for (int u = t_begin; u < t_end && !stop; ++u, ++tcount) {
        // (the accumulator is free only once every MMA of the previous tile
        // has completed, so resident scales may be overwritten after this)
        if (!mbar_wait_warp(acc_empty, (tcount & 1) ^ 1, p.timeout_ns, abort_flag, (2u << 8) | kid))
          break;
        tc_fence_after();
        const int tile = u / ksplit, part = u - tile * ksplit;
        int kb_lo, kb_hi;
        split_stages(part, ksplit, kb_total, kb_lo, kb_hi);
        const int lr_here = part == ksplit - 1 ? lr_chunks : 0;
        const bool load_sfa = !sfa_res || u == t_begin || tile % num_n == 0;
        uint32_t accumulate = 0;
        for (int kb = kb_lo; kb < kb_hi; ++kb, ++it) {
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
          const uint32_t sfa_t = sfa_res ? tmem + G_SF_TMEM + 16 * kb
                                         : tmem + G_SF_TMEM + (it & 1) * G_SF_TMEM_STRIDE;
          const uint32_t sfb_t = sfa_res ? tmem + G_SFB_RES_TMEM + (it & 1) * G_SFB_RES_STRIDE
                                         : sfa_t + 16;
          // Every stage runs all four 64-deep steps, fixed and fully
          // unrolled: a loop bounded at run time (or a per-step guard) around
          // elect.sync here cut the issue rate by up to half.  A short last
          // stage (K % 256 != 0) reads zero codes past K (TMA fill) against
          // finite scales, which adds exactly zero.
          if (elect_one()) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              if (load_sfa)
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
              mma_nvfp4_pair(tmem, da + 2 * kk, db + 2 * kk, id_fp4, sfa_t + 4 * kk,
                             sfb_t + 8 * kk, kk > 0 ? 1u : accumulate);
            __syncwarp();
          }
          accumulate = 1;
          ready = mbar_test_warp(full0 + 8 * ((it + 1) % G_STAGES), ((it + 1) / G_STAGES) & 1);
          if (elect_one()) tc_commit_pair(empty0 + 8 * st, 0x3);
          __syncwarp();
        }
        for (int c = 0; c < lr_here && !stop; ++c, ++it) {
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
            if (elect_one()) mma_bf16_pair(tmem, da + 2 * kk, db + 2 * kk, id_lr, 1u);
            __syncwarp();
          }
          ready = mbar_test_warp(full0 + 8 * ((it + 1) % G_STAGES), ((it + 1) / G_STAGES) & 1);
          if (elect_one()) tc_commit_pair(empty0 + 8 * st, 0x3);
          __syncwarp();
        }
        if (elect_one()) tc_commit_pair(acc_full, 0x3);
        __syncwarp();
      }
    }
  } else {
    // -------------------------------------------------------- epilogue ----
    const int quad = warp & 3;                 // tensor-memory lane quarter
    const int half = (warp - 2) >> 2;          // columns [128 half, 128 half + 128)
    const int et = threadIdx.x - 64;           // 0..255
    const int row_t = quad * 32 + lane;        // this thread's row of the CTA's 128
    const uint32_t obuf = out_s + half * G_OUT_HALF_BYTES;
    const uint32_t staged = out_staged0 + 8 * half, freed = out_free0 + 8 * half;
    // one thread per group of four warps issues the group's bulk stores
    const bool issuer = ((warp - 2) & 3) == 0 && lane == 0;
    int use = 0;                               // boxes this group has staged
    int tcount = 0;
    for (int u = t_begin; u < t_end; ++u, ++tcount) {
      const int tile = u / ksplit, part = u - tile * ksplit;
      const int mb = tile / num_n, nb = tile % num_n;
      // stage this tile's bias (fp32) while the main loop runs.  Buffer
      // tcount&1 was last read for tile tcount-2, which every thread had
      // finished before arriving on the other buffer's barrier.
      float* bt = bias_s + (tcount & 1) * G_BN;
      const uint32_t bb = bias_bar0 + 8 * (tcount & 1);
      {
        const int n = nb * G_BN + et;
        bt[et] = (p.bias && n < N) ? bf16_lo_f32(p.bias[n]) : 0.0f;
      }
      mbar_arrive(bb);
      if (!mbar_wait_warp(bb, (tcount >> 1) & 1, p.timeout_ns, abort_flag, (5u << 8) | kid)) break;
      if (!mbar_wait_warp(acc_full, tcount & 1, p.timeout_ns, abort_flag, (4u << 8) | kid)) break;
      tc_fence_after();
      const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16) + half * 128;
      uint32_t acc[4][32];
      tmem_ld32(tbase, acc[0]);
      tmem_ld32(tbase + 32, acc[1]);
      tmem_ld32(tbase + 64, acc[2]);
      tmem_ld32(tbase + 96, acc[3]);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(lead_acc_empty);   // accumulator free again
      const int row0 = mb * 2 * G_BM + (int)rank * G_BM;   // first row of this CTA's box
      // the output scale: static, or this row's own (dynamic mode)
      const float alpha = (p.row_scales && row0 + row_t < M) ? p.row_scales[row0 + row_t].alpha
                                                             : p.alpha;
      bool ok = true;
      if (ksplit > 1) {
        // split-K: this unit's fp32 partial instead of Y, through the same
        // staging buffer and bulk stores: four 128-row x 32-column boxes per
        // half (rows past M are written but never read)
        const int prow = ((tile * ksplit + part) * 2 + (int)rank) * G_BM;
#pragma unroll
        for (int sb = 0; sb < 4; ++sb, ++use) {
          if (use > 0) {
            if (issuer) {
              bulk_wait_read_all();
              mbar_arrive(freed);
            }
            __syncwarp();
            if (!mbar_wait_warp(freed, (use - 1) & 1, p.timeout_ns, abort_flag, (7u << 8) | kid)) {
              ok = false;
              break;
            }
          }
#pragma unroll
          for (int j = 0; j < 8; ++j)
            st_shared_v4(obuf + row_t * 128 + ((j ^ (row_t & 7)) << 4), acc[sb][4 * j],
                         acc[sb][4 * j + 1], acc[sb][4 * j + 2], acc[sb][4 * j + 3]);
          fence_proxy_async_shared();
          __syncwarp();
          if (lane == 0) mbar_arrive(staged);
          if (issuer) {
            if (mbar_wait(staged, use & 1, p.timeout_ns, abort_flag, (8u << 8) | kid)) {
              if (row0 < M) {
                tma_store_2d(&tm_part, obuf, half * 128 + sb * 32, prow);
                bulk_commit_group();
              }
            } else {
              ok = false;
            }
          }
          ok = __all_sync(0xffffffffu, ok) != 0;
          if (!ok) break;
        }
        if (!ok) break;
        continue;
      }
#pragma unroll
      for (int sb = 0; sb < 2; ++sb, ++use) {
        // the buffer is free once the store issued from it has read it
        if (use > 0) {
          if (issuer) {
            bulk_wait_read_all();
            mbar_arrive(freed);
          }
          __syncwarp();
          if (!mbar_wait_warp(freed, (use - 1) & 1, p.timeout_ns, abort_flag, (7u << 8) | kid)) {
            ok = false;
            break;
          }
        }
        // 64 columns of this thread's row: 8 chunks of 16 bytes, chunk j at
        // slot j ^ (row % 8) of the row's 128 bytes (the 128-byte swizzle)
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int ch = 2 * sb + (j >> 2);
          const int cb = 8 * (j & 3);
          const int c0 = half * 128 + ch * 32 + cb;
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float y0 = fmaf(alpha, __uint_as_float(acc[ch][cb + 2 * q]), bt[c0 + 2 * q]);
            float y1 = fmaf(alpha, __uint_as_float(acc[ch][cb + 2 * q + 1]), bt[c0 + 2 * q + 1]);
            if (p.gelu) {
              // the layer's bf16 output, then the MLP pair's GELU of it
              y0 = gelu_bf16_value(__bfloat162float(__float2bfloat16_rn(y0)));
              y1 = gelu_bf16_value(__bfloat162float(__float2bfloat16_rn(y1)));
            }
            o[q] = pack_bf16x2(y0, y1);
          }
          st_shared_v4(obuf + row_t * 128 + ((j ^ (row_t & 7)) << 4), o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_shared();
        __syncwarp();
        if (lane == 0) mbar_arrive(staged);
        if (issuer) {
          const int x = nb * G_BN + half * 128 + sb * G_OUT_COLS;
          // a box wholly past N or M has nothing to write
          if (mbar_wait(staged, use & 1, p.timeout_ns, abort_flag, (8u << 8) | kid)) {
            if (x < N && row0 < M) {
              tma_store_2d(&tm_y, obuf, x, row0);
              bulk_commit_group();
            }
          } else {
            ok = false;
          }
        }
        ok = __all_sync(0xffffffffu, ok) != 0;   // the issuer's verdict, warp-wide
        if (!ok) break;
      }
      if (!ok) break;
    }
    // no store may still be reading shared memory (or writing Y) at exit
    if (issuer) bulk_wait_all();
  }

  // ------------------------------------------------------------ teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // The leader's barriers count both CTAs' loads.  Drain the stages either
    // CTA issued: the other CTA reports its count (bounded wait); a stage
    // that only it issued was never armed here, so arm it with its bytes.
    // Then drain the tensor-core work in flight.
    if (leader && warp == 0 && lane == 0) {
      mbar_wait_drain_cluster(peer_bar, 0, p.timeout_ns);
      const int peer = *peer_issued;
      const int hi = max(issued, peer);
      for (int i = max(0, hi - G_STAGES); i < hi; ++i) {
        const uint32_t fb = full0 + 8 * (i % G_STAGES);
        if (i >= issued) {
          // the stage's bytes follow from its place in the unit sequence
          // (the same rule the producers use)
          int u = t_begin, j = i;
          bool lr_stage = false;
          while (u < t_end) {
            const int tl = u / ksplit, pt = u - tl * ksplit;
            int lo, hi2;
            split_stages(pt, ksplit, kb_total, lo, hi2);
            const int n_fp4 = hi2 - lo, n_lr = pt == ksplit - 1 ? lr_chunks : 0;
            if (j < n_fp4 + n_lr) {
              lr_stage = j >= n_fp4;
              break;
            }
            j -= n_fp4 + n_lr;
            ++u;
          }
          const bool with_sfa = !sfa_res || u == t_begin || (u / ksplit) % num_n == 0;
          mbar_arrive_expect_tx(fb, (lr_stage ? G_LR_TX : with_sfa ? G_FP4_TX : G_FP4_TX_NOSFA) / 2);
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

// Split-K reduction: Y[m][n] = bf16(alpha * sum_p partial_p[m][n] + bias[n]),
// the parts added in part order (so Y does not depend on which unit of the
// GEMM finished first).  One thread per 8 consecutive outputs of a row: all
// parts' 32 bytes are loaded before the sum (up to 8 parts in flight).
// Launched right after the GEMM with programmatic dependent launch.
__global__ void __launch_bounds__(256)
    splitk_reduce_kernel(const float* __restrict__ partials, int M, int N, int ksplit,
                         float alpha, const uint16_t* __restrict__ bias, uint16_t* __restrict__ Y,
                         int64_t ldy) {
  grid_dependency_wait();
  const int num_n = (N + G_BN - 1) / G_BN;
  const int groups = N >> 3;   // N % 8 == 0
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < (long long)M * groups;
       i += (long long)gridDim.x * blockDim.x) {
    const int m = (int)(i / groups), n = (int)(i - (long long)m * groups) * 8;
    const int tile = (m / (2 * G_BM)) * num_n + n / G_BN;
    const int rank = (m % (2 * G_BM)) / G_BM, row = m % G_BM, col = n % G_BN;
    const float* src = partials + (((size_t)tile * ksplit * 2 + rank) * G_BM + row) * G_BN + col;
    const size_t stride = (size_t)2 * G_BM * G_BN;
    float4 v[2 * 8];
#pragma unroll
    for (int pp = 0; pp < 8; ++pp)
      if (pp < ksplit) {
        v[2 * pp] = ld_cg_f4(src + pp * stride);
        v[2 * pp + 1] = ld_cg_f4(src + pp * stride + 4);
      }
    float y[8] = {v[0].x, v[0].y, v[0].z, v[0].w, v[1].x, v[1].y, v[1].z, v[1].w};
#pragma unroll
    for (int pp = 1; pp < 8; ++pp)
      if (pp < ksplit) {
        y[0] += v[2 * pp].x;
        y[1] += v[2 * pp].y;
        y[2] += v[2 * pp].z;
        y[3] += v[2 * pp].w;
        y[4] += v[2 * pp + 1].x;
        y[5] += v[2 * pp + 1].y;
        y[6] += v[2 * pp + 1].z;
        y[7] += v[2 * pp + 1].w;
      }
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float b0 = bias ? bf16_lo_f32(bias[n + 2 * q]) : 0.0f;
      const float b1 = bias ? bf16_lo_f32(bias[n + 2 * q + 1]) : 0.0f;
      o[q] = pack_bf16x2(fmaf(alpha, y[2 * q], b0), fmaf(alpha, y[2 * q + 1], b1));
    }
    *reinterpret_cast<uint4*>(Y + (size_t)m * ldy + n) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  grid_launch_dependents();
}

}  // namespace svdq_dev
