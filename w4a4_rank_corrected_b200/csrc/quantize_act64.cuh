// Activation kernel of the SVDQuant W4A4 linear, 64-row tiles: the form for
// token counts too small to give every SM a 128-row tile (below about 15k
// rows), where K is split across a cluster of CTAs with the low-rank partial
// sums reduced on chip.  Same arithmetic as the 128-row kernel
// (quantize_act.cuh): smoothing, NVFP4 quantization and the fused low-rank
// down-projection, in one pass over X.
//
// The fusion is the one described for the Nunchaku engine in the Korean
// rendering of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"
// (section "SVDQuant and the Nunchaku engine"): the low-rank down projection
// is merged into the quantization kernel so the 16-bit branch costs no extra
// pass over the activations.  The B200 design:
//
//   * one CTA owns 64 rows x a contiguous slice of K (64-column chunks).  The
//     host picks how many CTAs split K (a thread-block cluster of up to 8)
//     so that the whole grid is resident in one wave;
//   * the slice's smoothing factors are loaded once (bulk copy) and stay in
//     shared memory;
//   * warp 0 streams X chunks [64 rows x 128 columns] bf16, as two 64 x 64
//     boxes (TMA, 128-byte swizzle) under one barrier pair, into a ring of 4
//     or 8 stages: the ring holds only X, so up to 128 KB of activations per
//     SM are in flight;
//   * warp 2 streams the matching chunks of the low-rank operand L1' into a
//     separate ring of up to 8 stages (they come from L2: every row block
//     reads the same L1', so each row block starts its K slice at a
//     different chunk to spread those reads);
//   * Q64_QWARPS quantize warps: unit u = (chunk u / 4, box (u % 4) / 2,
//     rows 32 (u % 2) .. + 31) goes to warp u % Q64_QWARPS; lane l handles one
//     row.  A warp copies
//     its row segment (128 bytes per lane) into registers, hands the X stage
//     back, then quantizes: per 16-group multiply by the smoothing factors,
//     take the maximum, form the E4M3 block scale with one multiply and the
//     hardware conversion, look up g/scale in a 127-entry table (the IEEE
//     quotients, computed once per CTA), form the E2M1 codes with the
//     hardware conversion; per row 32 code bytes and one 32-bit word of
//     scales go straight into the MMA tile layout;
//   * warp 1 (converged: every lane waits, an elected lane issues) issues
//     tcgen05 bf16 MMAs (M = 64) on the SAME shared-memory X
//     tile: X [64 x 64] times L1' [2r x 64]^T into a 64 x 2r fp32 accumulator
//     in tensor memory.  L1' holds smooth * L1 split into bf16 hi and lo
//     halves, so X L1' = X_hat L1 to ~2^-16 relative (X itself is exact);
//   * at the end the accumulator is read back (tcgen05.ld) and hi + lo
//     columns are summed.  In a K split every rank but 0 pushes its partial
//     sums into rank 0's shared memory with st.async (the bytes are counted
//     on a barrier there), rank 0 adds them in rank order (deterministic) and
//     stores the result times lr_scale as a bf16 hi/lo pair for the GEMM's
//     up-projection.
#pragma once
#include "ptx.cuh"
#include "row_scales.cuh"

namespace svdq_dev {

constexpr int Q64_BM = 64;
constexpr int Q64_QWARPS = 16;
constexpr int Q64_QWARP0 = 3;                               // first quantize warp
constexpr int Q64_THREADS = 32 * (Q64_QWARP0 + Q64_QWARPS);
// A chunk is 128 columns of the slice: two 64-column TMA boxes (128-byte
// swizzle rows) that share one barrier pair, so each barrier round trip of
// the producer moves 16 KB of X.
constexpr int Q64_BOXES = 2;
constexpr uint32_t Q64_BOX_BYTES = Q64_BM * 128;             // 64 rows x 64 bf16
constexpr uint32_t Q64_X_BYTES = Q64_BOXES * Q64_BOX_BYTES;   // one X stage
// X ring depth: a multiple of Q64_QWARPS / 4 = 4.  A chunk has 4 units (two
// row halves x two boxes); warp w's units cover chunks w / 4, w / 4 + 4,
// w / 4 + 8, ...; with the depth a multiple of 4, the previous use of the
// stage a warp is about to wait on was that same warp's own earlier chunk,
// which it has already seen land, so the stage's barrier is never two
// phases behind a parity wait (which would pass at once).
constexpr int Q64_UNITS = 2 * Q64_BOXES;                     // units per chunk
constexpr int Q64_XST_STEP = Q64_QWARPS / Q64_UNITS;
constexpr int Q64_MAX_XST = 2 * Q64_XST_STEP;
constexpr int Q64_MIN_XST = Q64_XST_STEP;
constexpr int Q64_MAX_LST = 8;
static_assert(Q64_QWARPS % Q64_UNITS == 0 && Q64_MAX_XST % Q64_XST_STEP == 0,
              "ring depth must be a multiple of the chunk stride of a warp's units");
constexpr uint32_t Q64_SMEM_BUDGET = 224 * 1024;  // + 1.5 KB: within the 227 KB per CTA

// Shared-memory plan of one CTA (offsets from the 1024-aligned base).
struct Q64Layout {
  int xst, lst;              // ring depths (X, low-rank operand)
  uint32_t l1_bytes;         // one low-rank stage: two boxes of 2r rows x 128 bytes
  uint32_t l1_off, s_off, red_off, lut_off, bar_off;
  uint32_t total;            // bytes to request (incl. alignment slack)
};

__host__ __device__ inline Q64Layout q64_layout(int r, int chunks_per_split, int num_splits) {
  Q64Layout L;
  L.l1_bytes = (uint32_t)Q64_BOXES * 256u * (uint32_t)r;
  const uint32_t s_bytes = (uint32_t)Q64_BOXES * 256u * (uint32_t)chunks_per_split;
  const uint32_t red_bytes =
      (r > 0 && num_splits > 1) ? (uint32_t)(num_splits - 1) * Q64_BM * (uint32_t)r * 4u : 0u;
  const uint32_t fixed = s_bytes + red_bytes + 512u + 512u;
  // the deeper X ring if the low-rank ring still gets a stage, else the
  // shallower one; the low-rank ring takes what is left, up to 8 stages
  L.xst = 0;
  L.lst = 0;
  for (int xst = Q64_MAX_XST; xst >= Q64_MIN_XST; xst -= Q64_XST_STEP) {
    const uint32_t used = fixed + (uint32_t)xst * Q64_X_BYTES;
    if (used > Q64_SMEM_BUDGET) continue;
    int lst = 0;
    if (r > 0) {
      lst = (int)((Q64_SMEM_BUDGET - used) / L.l1_bytes);
      lst = lst > Q64_MAX_LST ? Q64_MAX_LST : lst;
      if (lst < 1) continue;
    }
    L.xst = xst;
    L.lst = lst;
    break;
  }
  L.l1_off = (uint32_t)L.xst * Q64_X_BYTES;
  L.s_off = L.l1_off + (uint32_t)L.lst * L.l1_bytes;
  L.red_off = L.s_off + s_bytes;
  L.lut_off = L.red_off + red_bytes;
  L.bar_off = L.lut_off + 512u;
  L.total = 1024u + L.bar_off + 512u;
  return L;
}

struct Q64Params {
  const float* smooth;
  uint8_t* codes_x;
  uint8_t* sf_x;
  uint16_t* xl1;
  const RowScale* row_scales;   // per-row scales (dynamic mode) or NULL (static)
  int M, K, r, klr;
  int chunks_per_split;
  int num_splits;
  Q64Layout L;
  uint32_t tmem_cols;
  float g_x, gs_x, lr_scale;
  uint64_t timeout_ns;
};

__device__ __forceinline__ int64_t q64_sf_tile_off(int row, int g, int K) {
  return ((int64_t)(row >> 7) * (K >> 6) + (g >> 2)) * 512 + (row & 31) * 16 +
         ((row & 127) >> 5) * 4 + (g & 3);
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

__global__ void __launch_bounds__(Q64_THREADS, 1)
    quantize_act64_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1, const Q64Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int r = p.r;
  const bool has_lr = r > 0;
  const Q64Layout& L = p.L;
  const int XST = L.xst, LST = L.lst;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  const uint32_t x_full0 = smem_u32(bars);
  const uint32_t x_empty0 = x_full0 + 8 * XST;
  const uint32_t l_full0 = x_empty0 + 8 * XST;
  const uint32_t l_empty0 = l_full0 + 8 * LST;
  const uint32_t acc_full = l_empty0 + 8 * LST;
  const uint32_t s_bar = acc_full + 8;
  const uint32_t red_bar = acc_full + 16;
  const uint32_t drain_bar = acc_full + 24;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 2 * XST + 2 * LST + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* qlut = reinterpret_cast<float*>(smem + L.lut_off);  // 128 floats
  const float* s_sm = reinterpret_cast<const float*>(smem + L.s_off);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x;  // = rank in the cluster when S > 1
  const int rb = blockIdx.y;
  const int S = p.num_splits;
  const bool reduce = has_lr && S > 1;
  const int kchunks = ((p.K >> 6) + Q64_BOXES - 1) / Q64_BOXES;   // 128-column chunks
  const int c_begin = split * p.chunks_per_split;
  const int c_end = min(kchunks, c_begin + p.chunks_per_split);
  const int nchunks = max(0, c_end - c_begin);
  // Row blocks walk their K slice from different starting chunks, so the
  // CTAs do not all ask L2 for the same low-rank tile at the same moment.
  const int rot = nchunks > 0 ? rb % nchunks : 0;
  const unsigned int kid = 1;  // kernel id in error codes

  if (threadIdx.x == 0) {
    for (int i = 0; i < XST; ++i) {
      mbar_init(x_full0 + 8 * i, 1);
      mbar_init(x_empty0 + 8 * i, Q64_UNITS + (has_lr ? 1 : 0));  // its 4 units + the MMA
    }
    for (int i = 0; i < LST; ++i) {
      mbar_init(l_full0 + 8 * i, 1);
      mbar_init(l_empty0 + 8 * i, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(s_bar, 1);
    mbar_init(red_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
    // rank 0 of a K split expects the other ranks' partial sums
    if (reduce && split == 0)
      mbar_arrive_expect_tx(red_bar, (uint32_t)(S - 1) * Q64_BM * (uint32_t)r * 4u);
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
  // every rank's barriers exist before any rank stores into another's
  // shared memory (the matching wait comes before the epilogue)
  if (reduce) cluster_arrive();
  const uint32_t tmem = has_lr ? *tmem_holder : 0u;
  // Everything above overlaps the tail of the previous kernel in the stream;
  // from here on this kernel reads and writes memory that kernel may touch.
  grid_dependency_wait();
  grid_launch_dependents();

  int x_issued = 0, l_issued = 0;  // producers: chunks whose loads were issued
  if (warp == 0) {
    // ------------------------------------------------ X producer (TMA) ----
    // One lane runs the loop (its warp shares an SM sub-partition with busy
    // quantize warps, so the fewer instructions per load the better); the
    // rest of the warp waits at the __syncwarp below.
    if (lane == 0) {
      if (nchunks > 0) {
        const int ncols = min(p.K - c_begin * 128, nchunks * 128);  // a multiple of 64
        mbar_arrive_expect_tx(s_bar, 4u * (uint32_t)ncols);
        bulk_load(smem_u32(smem + L.s_off), p.smooth + c_begin * 128, 4u * (uint32_t)ncols, s_bar);
      }
      int st = 0;
      uint32_t ph = 0;
      int cl = rot;  // local chunk of load i: (i + rot) mod nchunks
      for (int i = 0; i < nchunks; ++i) {
        // every stage starts free: the first XST loads go out back to back
        // (a satisfied try_wait still costs a round trip per load)
        if (i >= XST &&
            !mbar_wait(x_empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (1u << 8) | kid))
          break;
        mbar_arrive_expect_tx(x_full0 + 8 * st, Q64_X_BYTES);
        // (a box past K reads zeros: the TMA fill)
        for (int b = 0; b < Q64_BOXES; ++b)
          tma_load_2d(smem_u32(smem + st * Q64_X_BYTES + b * Q64_BOX_BYTES), &tm_x,
                      (c_begin + cl) * 128 + 64 * b, rb * Q64_BM, x_full0 + 8 * st);
        x_issued = i + 1;
        if (++st == XST) { st = 0; ph ^= 1; }
        if (++cl == nchunks) cl = 0;
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ---------------------------------- low-rank operand producer (TMA) ----
    if (has_lr && lane == 0) {
      int st = 0;
      uint32_t ph = 0;
      int cl = rot;
      for (int i = 0; i < nchunks; ++i) {
        if (i >= LST &&
            !mbar_wait(l_empty0 + 8 * st, ph ^ 1, p.timeout_ns, abort_flag, (5u << 8) | kid))
          break;
        mbar_arrive_expect_tx(l_full0 + 8 * st, L.l1_bytes);
        for (int b = 0; b < Q64_BOXES; ++b)
          tma_load_2d(smem_u32(smem + L.l1_off + st * L.l1_bytes + b * (L.l1_bytes / Q64_BOXES)),
                      &tm_l1, (c_begin + cl) * 128 + 64 * b, 0, l_full0 + 8 * st);
        l_issued = i + 1;
        if (++st == LST) { st = 0; ph ^= 1; }
        if (++cl == nchunks) cl = 0;
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------ down-projection (warp) ----
    if (has_lr) {
      const uint32_t idesc = idesc_bf16(Q64_BM, 2 * r);
      int xs = 0, ls = 0;
      uint32_t xph = 0, lph = 0;
      for (int i = 0; i < nchunks; ++i) {
        // both tiles have landed (complete_tx); the MMAs read them through
        // the async proxy
        if (!mbar_wait_warp(x_full0 + 8 * xs, xph, p.timeout_ns, abort_flag, (2u << 8) | kid)) break;
        if (!mbar_wait_warp(l_full0 + 8 * ls, lph, p.timeout_ns, abort_flag, (2u << 8) | kid)) break;
        // the chunk's eight MMAs and both releases from one elected lane: this
        // warp shares its sub-partition with busy quantize warps, and each
        // stage's release waits for its MMAs, so the fewer issue slots the
        // chunk costs here the sooner the X ring turns over (an elect and a
        // warp sync per MMA left this warp about 1.8 us behind the
        // quantize warps at the end of a 4608 x 3072 launch)
        if (elect_one()) {
#pragma unroll
          for (int b = 0; b < Q64_BOXES; ++b) {
            const uint64_t da = sdesc_sw128(smem_u32(smem + xs * Q64_X_BYTES + b * Q64_BOX_BYTES));
            const uint64_t db = sdesc_sw128(
                smem_u32(smem + L.l1_off + ls * L.l1_bytes + b * (L.l1_bytes / Q64_BOXES)));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // K = 16 bf16 = 32 bytes per MMA
              mma_bf16(tmem, da + 2 * kk, db + 2 * kk, idesc, (i | b | kk) != 0 ? 1u : 0u);
          }
          tc_commit(x_empty0 + 8 * xs);
          tc_commit(l_empty0 + 8 * ls);
        }
        __syncwarp();
        if (++xs == XST) { xs = 0; xph ^= 1; }
        if (++ls == LST) { ls = 0; lph ^= 1; }
      }
      if (elect_one()) tc_commit(acc_full);
      __syncwarp();
    }
  } else {
    // ---------------------------------------------- NVFP4 quantization ----
    const int qw = warp - Q64_QWARP0;
    bool ok = nchunks == 0 || mbar_wait_warp(s_bar, 0, p.timeout_ns, abort_flag, (3u << 8) | kid);
    for (int u = qw; ok && u < Q64_UNITS * nchunks; u += Q64_QWARPS) {
      const int i = u / Q64_UNITS;
      const int box = (u % Q64_UNITS) >> 1;
      const int cl = i + rot < nchunks ? i + rot : i + rot - nchunks;  // local chunk
      const int st = i % XST;
      const uint32_t ph = (uint32_t)(i / XST) & 1u;
      if (!mbar_wait_warp(x_full0 + 8 * st, ph, p.timeout_ns, abort_flag, (3u << 8) | kid)) break;
      const int row_t = 32 * (u & 1) + lane;
      const int row = rb * Q64_BM + row_t;
      // this row's tensor scales: the static ones, or (dynamic mode) its own
      const bool dyn = p.row_scales != nullptr;
      float g_row = p.g_x, gs = p.gs_x;
      if (dyn && row < p.M) {
        g_row = p.row_scales[row].g;
        gs = p.row_scales[row].gs;
      }
      const int col0 = (c_begin + cl) * 128 + 64 * box;   // first column of the unit
      const uint8_t* xrow = smem + st * Q64_X_BYTES + box * Q64_BOX_BYTES + row_t * 128;
      // copy this lane's row segment into registers, then hand the stage
      // back so the next chunk can land while this one is quantized
      uint4 xr[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        xr[j] = *reinterpret_cast<const uint4*>(xrow + ((j ^ (row_t & 7)) << 4));
      // Hand the stage back only after the reads are done and ordered before
      // the next fill.  The fill is a TMA write (async proxy) after these
      // generic-proxy reads of the same bytes: each lane folds its loaded
      // words into one value (its loads have landed), the warp reduces those,
      // every lane fences the generic proxy against the async proxy, and
      // lane 0 releases.  Without the proxy fence an occasional refill
      // overwrote a stage while a warp's reads of it were still being served
      // (a few percent of launches had one unit wrong).
      uint32_t dep = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) dep ^= xr[j].x ^ xr[j].y ^ xr[j].z ^ xr[j].w;
      dep = __reduce_or_sync(0xffffffffu, dep);
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive_after(x_empty0 + 8 * st, dep);
      if (col0 >= p.K) continue;  // the zero box past K: nothing to store
      const float4* sp = reinterpret_cast<const float4*>(s_sm + cl * 128 + 64 * box);
      uint32_t cw[8];
      uint32_t sfw = 0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        // 16 products x * s as 8 lane-pairs (one f32x2 multiply each)
        const uint4 x0 = xr[2 * g], x1 = xr[2 * g + 1];
        const ulonglong2* sp2 = reinterpret_cast<const ulonglong2*>(sp + 4 * g);
        const ulonglong2 s0 = sp2[0], s1 = sp2[1], s2 = sp2[2], s3 = sp2[3];
        uint64_t v[8];
        v[0] = fmul_f32x2(bf16x2_to_f32x2(x0.x), s0.x);
        v[1] = fmul_f32x2(bf16x2_to_f32x2(x0.y), s0.y);
        v[2] = fmul_f32x2(bf16x2_to_f32x2(x0.z), s1.x);
        v[3] = fmul_f32x2(bf16x2_to_f32x2(x0.w), s1.y);
        v[4] = fmul_f32x2(bf16x2_to_f32x2(x1.x), s2.x);
        v[5] = fmul_f32x2(bf16x2_to_f32x2(x1.y), s2.y);
        v[6] = fmul_f32x2(bf16x2_to_f32x2(x1.z), s3.x);
        v[7] = fmul_f32x2(bf16x2_to_f32x2(x1.w), s3.y);
        float m[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float lo, hi;
          unpack_f32x2(v[e], lo, hi);
          m[e] = fmaxf(fabsf(lo), fabsf(hi));
        }
        const float a = fmaxf(fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3])),
                              fmaxf(fmaxf(m[4], m[5]), fmaxf(m[6], m[7])));
        const uint32_t code = cvt_e4m3x2(__fmul_rn(a, gs), 0.0f) & 0xFF;
        const float q = !dyn ? qlut[code]
                             : (code == 0 ? 0.0f : __fdiv_rn(g_row, e4m3_to_f32(code)));
        const uint64_t qq = pack_f32x2(q, q);
        float t0[8], t1[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          unpack_f32x2(fmul_f32x2(v[e], qq), t0[2 * e], t0[2 * e + 1]);
          unpack_f32x2(fmul_f32x2(v[4 + e], qq), t1[2 * e], t1[2 * e + 1]);
        }
        cw[2 * g] = cvt_e2m1x8(t0);
        cw[2 * g + 1] = cvt_e2m1x8(t1);
        sfw |= code << (8 * g);
      }
      if (row < p.M) {
        uint4* dst = reinterpret_cast<uint4*>(p.codes_x + (size_t)row * (p.K >> 1) + (col0 >> 1));
        dst[0] = make_uint4(cw[0], cw[1], cw[2], cw[3]);
        dst[1] = make_uint4(cw[4], cw[5], cw[6], cw[7]);
      }
      *reinterpret_cast<uint32_t*>(p.sf_x + q64_sf_tile_off(row, col0 >> 4, p.K)) = sfw;
    }
  }

  // ----------------------------------------- low-rank epilogue (X L1) ----
  if (reduce) cluster_wait();
  if (has_lr && warp >= Q64_QWARP0) {
    const bool ok = mbar_wait_warp(acc_full, 0, p.timeout_ns, abort_flag, (4u << 8) | kid);
    tc_fence_after();
    // M = 64 accumulator: row m sits in lane (m % 16) + 32 (m / 16).  Warp w
    // reads its lane quarter w % 4; lanes 0..15 hold rows 16 (w % 4) + lane.
    const int quad = warp & 3;
    const int slot = (warp - Q64_QWARP0) >> 2;   // 0 .. Q64_QWARPS / 4 - 1
    const int lrow_t = quad * 16 + lane;
    const int lrow = rb * Q64_BM + lrow_t;
    const bool own = lane < 16;
    const uint32_t red_base = smem_u32(smem + L.red_off);
    const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16);
    for (int ci = slot; ci < r / 16; ci += Q64_QWARPS / 4) {
      uint32_t hi[16], lo[16];
      if (ok) {
        tmem_ld16(tbase + 16 * ci, hi);
        tmem_ld16(tbase + r + 16 * ci, lo);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 16; ++j) hi[j] = lo[j] = 0u;
      }
      float part[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) part[j] = __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
      if (!reduce) {
        if (own && lrow < p.M)
          store_hi_lo16(part, p.row_scales ? p.row_scales[lrow].lr : p.lr_scale,
                        p.xl1 + (size_t)lrow * p.klr + 16 * ci,
                        p.xl1 + (size_t)lrow * p.klr + r + 16 * ci);
      } else if (split != 0) {
        // partial sums [row][r] of rank `split` into rank 0's buffer split-1
        if (own) {
          const uint32_t dst = map_to_rank(
              red_base + 4u * (uint32_t)(((split - 1) * Q64_BM + lrow_t) * r + 16 * ci), 0);
          const uint32_t bar = map_to_rank(red_bar, 0);
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            st_async_v4(dst + 4u * j, part[j], part[j + 1], part[j + 2], part[j + 3], bar);
        }
      } else {
        const bool got = mbar_wait_warp(red_bar, 0, p.timeout_ns, abort_flag, (6u << 8) | kid);
        if (own && lrow < p.M) {
          if (got) {
            for (int sr = 1; sr < S; ++sr) {
              const float4* q4 = reinterpret_cast<const float4*>(
                  smem + L.red_off + 4u * (uint32_t)(((sr - 1) * Q64_BM + lrow_t) * r + 16 * ci));
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float4 t = q4[j];
                part[4 * j] += t.x;
                part[4 * j + 1] += t.y;
                part[4 * j + 2] += t.z;
                part[4 * j + 3] += t.w;
              }
            }
          }
          store_hi_lo16(part, p.row_scales ? p.row_scales[lrow].lr : p.lr_scale,
                        p.xl1 + (size_t)lrow * p.klr + 16 * ci,
                        p.xl1 + (size_t)lrow * p.klr + r + 16 * ci);
        }
      }
    }
    // zero columns [2r, klr) of the rows this CTA finishes
    if (split == 0 && slot == 0 && own && lrow < p.M) {
      for (int cpad = 2 * r; cpad < p.klr; cpad += 8)
        *reinterpret_cast<uint4*>(p.xl1 + (size_t)lrow * p.klr + cpad) = make_uint4(0, 0, 0, 0);
    }
  }

  // ------------------------------------------------------------ teardown ----
  tc_fence_before();
  __syncthreads();
  if (*abort_flag) {
    // drain: loads still in flight, then tensor-core work still in flight
    if (warp == 0 && lane == 0) {
      for (int i = max(0, x_issued - XST); i < x_issued; ++i)
        mbar_wait_drain(x_full0 + 8 * (i % XST), (i / XST) & 1, p.timeout_ns);
      if (nchunks > 0) mbar_wait_drain(s_bar, 0, p.timeout_ns);
    }
    if (warp == 2 && lane == 0) {
      for (int i = max(0, l_issued - LST); i < l_issued; ++i)
        mbar_wait_drain(l_full0 + 8 * (i % LST), (i / LST) & 1, p.timeout_ns);
    }
    if (warp == 1 && has_lr) {
      // from the lane that issued the MMAs (elect.sync picks it again)
      if (elect_one()) {
        tc_commit(drain_bar);
        mbar_wait_drain(drain_bar, 0, p.timeout_ns);
      }
      __syncwarp();
    }
    __syncthreads();
  }
  // no rank leaves while another may still store into its shared memory
  if (reduce) cluster_sync();
  if (warp == 1 && has_lr) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace svdq_dev
