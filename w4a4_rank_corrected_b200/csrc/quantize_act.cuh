// Activation kernel of the SVDQuant W4A4 linear, 128-row tiles: smoothing,
// NVFP4 quantization and the fused low-rank down-projection, in one pass
// over X.  This is the form for large token counts (one 128-row tile per SM
// or more, about 15k rows and up); smaller batches use the 64-row kernel
// (quantize_act64.cuh), which splits K within a cluster.
//
// The fusion is the one described for the Nunchaku engine in the Korean
// rendering of "Bringing Nunchaku 4-bit diffusion inference to Diffusers"
// (section "SVDQuant and the Nunchaku engine"): the low-rank down projection
// is merged into the quantization kernel so the 16-bit branch costs no extra
// pass over the activations.  The B200 design:
//
//   * one CTA owns 128 rows x all of K, walked in chunks of 128 columns.
//     128 rows per CTA (one full scale-factor atom row) means every byte of
//     the low-rank operand that reaches an SM serves 128 rows of X, and the
//     scales of a chunk are two whole 512-byte atoms;
//   * the slice's smoothing factors are loaded once (bulk copy) and stay in
//     shared memory;
//   * warp 0 streams X chunks [128 rows x 128 columns] bf16, as two
//     128 x 64 boxes (TMA, 128-byte swizzle) under one barrier pair, into a
//     ring of 2 or 4 stages; warp 2 streams the matching chunks of the
//     low-rank operand L1' into a separate ring (they come from L2: every
//     row block reads the same L1', so each row block starts its K slice at
//     a different chunk to spread those reads);
//   * QA_QWARPS quantize warps: unit u = (chunk u / 8, box (u % 8) / 4,
//     rows 32 (u % 4) .. + 31) goes to warp u % QA_QWARPS; lane l handles one
//     row.  A warp copies its row segment (128 bytes per lane) into
//     registers, hands the X stage back, then quantizes: per 16-group
//     multiply by the smoothing factors, take the maximum, form the E4M3
//     block scale with one multiply and the hardware conversion, look up
//     g/scale in a 127-entry table (the IEEE quotients, computed once per
//     CTA), form the E2M1 codes with the hardware conversion.  The 32 code
//     bytes and the 32-bit scale word of each row go into a shared-memory
//     staging slot laid out exactly as the global tiles (codes with the
//     64-byte swizzle of their TMA box, scales in the MMA atom layout);
//   * warp 3 (one lane) writes each finished chunk out: one TMA tile store
//     of the 128 x 64-byte code box and one bulk copy of the chunk's two
//     512-byte scale atoms -- coalesced, asynchronous stores instead of one
//     scattered 16-byte store per lane and row;
//   * warp 1 (converged: every lane waits, an elected lane issues) issues
//     tcgen05 bf16 MMAs (M = 128) on the SAME shared-memory X tile: X
//     [128 x 64] times L1' [2r x 64]^T into a 128 x 2r fp32 accumulator in
//     tensor memory.  L1' holds smooth * L1 split into bf16 hi and lo
//     halves, so X L1' = X_hat L1 to ~2^-16 relative (X itself is exact);
//   * at the end the accumulator is read back (tcgen05.ld), hi + lo columns
//     are summed and stored times lr_scale as a bf16 hi/lo pair for the
//     GEMM's up-projection.  (A K split of this kernel across CTAs was tried:
//     its cross-CTA reduction of the partial sums cost more at the end of
//     the kernel than the split gained, so small batches use the 64-row
//     kernel instead.)
#pragma once
#include "ptx.cuh"
#include "row_scales.cuh"

namespace svdq_dev {

constexpr int QA_BM = 128;                                 // rows per CTA
constexpr int QA_QWARPS = 16;
constexpr int QA_QWARP0 = 4;                               // first quantize warp
constexpr int QA_THREADS = 32 * (QA_QWARP0 + QA_QWARPS);
// A chunk is 128 columns of the slice: two 64-column TMA boxes (128-byte
// swizzle rows) that share one barrier pair, so each barrier round trip of
// the producer moves 32 KB of X.
constexpr int QA_BOXES = 2;
constexpr uint32_t QA_BOX_BYTES = QA_BM * 128;             // 128 rows x 64 bf16
constexpr uint32_t QA_X_BYTES = QA_BOXES * QA_BOX_BYTES;   // one X stage
constexpr int QA_UNITS = QA_BOXES * (QA_BM / 32);          // units per chunk (8)
// Ring depths (X, staging) are multiples of the chunk stride of a warp's
// units, QA_QWARPS / QA_UNITS = 2: warp w's units cover chunks w / 8,
// w / 8 + 2, w / 8 + 4, ...  So the previous use of any stage a warp is about
// to wait on was that same warp's own earlier chunk, which it has already
// seen complete, and no stage barrier is ever two phases behind a parity
// wait (which would pass at once).
constexpr int QA_XST_STEP = QA_QWARPS / QA_UNITS;
constexpr int QA_MAX_XST = 2 * QA_XST_STEP;
constexpr int QA_MIN_XST = QA_XST_STEP;
constexpr int QA_MAX_LST = 8;
constexpr int QA_MAX_NSTG = 2 * QA_XST_STEP;
constexpr int QA_MIN_NSTG = QA_XST_STEP;
static_assert(QA_QWARPS % QA_UNITS == 0 && QA_MAX_XST % QA_XST_STEP == 0 &&
                  QA_MAX_NSTG % QA_XST_STEP == 0,
              "ring depths must be multiples of the chunk stride of a warp's units");
constexpr uint32_t QA_CODES_STG = QA_BM * 64;              // 128 rows x 64 code bytes
constexpr uint32_t QA_SF_STG = QA_BOXES * 512;             // two scale atoms
constexpr uint32_t QA_STG_BYTES = QA_CODES_STG + QA_SF_STG;  // 9 KB, 1024-aligned slots
static_assert(QA_STG_BYTES % 1024 == 0, "staging slots keep 1024-byte alignment");
constexpr uint32_t QA_SMEM_BUDGET = 224 * 1024;  // + 1.5 KB: within the 227 KB per CTA

// Shared-memory plan of one CTA (offsets from the 1024-aligned base).
struct QALayout {
  int xst, lst, nstg;        // ring depths (X, low-rank operand, output staging)
  uint32_t l1_bytes;         // one low-rank stage: two boxes of 2r rows x 128 bytes
  uint32_t l1_off, stg_off, s_off, lut_off, bar_off;
  uint32_t total;            // bytes to request (incl. alignment slack)
};

__host__ __device__ inline QALayout qa_layout(int r, int chunks_per_split) {
  QALayout L;
  L.l1_bytes = (uint32_t)QA_BOXES * 256u * (uint32_t)r;
  const uint32_t s_bytes = (uint32_t)QA_BOXES * 256u * (uint32_t)chunks_per_split;
  const uint32_t fixed = s_bytes + 512u + 512u;
  const int lmax = chunks_per_split < QA_MAX_LST ? (chunks_per_split > 0 ? chunks_per_split : 1)
                                                 : QA_MAX_LST;
  // Preference: the deeper X ring, then two staging slots and two low-rank
  // stages, then as many low-rank stages as fit (up to the chunk count),
  // then deeper staging; a shallower plan only when nothing deeper fits.
  L.xst = 0;
  L.lst = 0;
  L.nstg = 0;
  for (int pass = 0; pass < 2 && L.xst == 0; ++pass) {
    const int lmin = (r > 0) ? (pass == 0 ? (lmax < 2 ? lmax : 2) : 1) : 0;
    for (int xst = QA_MAX_XST; xst >= QA_MIN_XST && L.xst == 0; xst -= QA_XST_STEP) {
      const uint32_t used = fixed + (uint32_t)xst * QA_X_BYTES + QA_MIN_NSTG * QA_STG_BYTES;
      if (used + (uint32_t)lmin * L.l1_bytes > QA_SMEM_BUDGET) continue;
      int lst = 0;
      if (r > 0) {
        lst = (int)((QA_SMEM_BUDGET - used) / L.l1_bytes);
        lst = lst > lmax ? lmax : lst;
      }
      int nstg = QA_MIN_NSTG;
      if (used + (uint32_t)lst * L.l1_bytes + (QA_MAX_NSTG - QA_MIN_NSTG) * QA_STG_BYTES <=
          QA_SMEM_BUDGET)
        nstg = QA_MAX_NSTG;
      L.xst = xst;
      L.lst = lst;
      L.nstg = nstg;
    }
  }
  L.l1_off = (uint32_t)L.xst * QA_X_BYTES;
  L.stg_off = L.l1_off + (uint32_t)L.lst * L.l1_bytes;      // multiple of 1024
  L.s_off = L.stg_off + (uint32_t)L.nstg * QA_STG_BYTES;
  L.lut_off = L.s_off + s_bytes;
  L.bar_off = L.lut_off + 512u;
  L.total = 1024u + L.bar_off + 512u;
  return L;
}

struct QAParams {
  const float* smooth;
  uint8_t* sf_x;
  uint16_t* xl1;
  const RowScale* row_scales;   // per-row scales (dynamic mode) or NULL (static)
  int M, K, r, klr;
  int chunks_per_split;
  int num_splits;
  QALayout L;
  uint32_t tmem_cols;
  float g_x, gs_x, lr_scale;
  uint64_t timeout_ns;
};

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// hi = bf16(v), lo = bf16(v - hi): v ~= hi + lo to ~2^-16 relative.
__device__ __forceinline__ void split_hi_lo(float v, float& hi, float& lo) {
  hi = __bfloat162float(__float2bfloat16_rn(v));
  lo = __fsub_rn(v, hi);
}

// Store 4 consecutive fp32 values (times lr_scale) as a bf16 hi part at
// dst_hi and a bf16 lo part at dst_lo (8 bytes each).
__device__ __forceinline__ void store_hi_lo4(const float (&v)[4], float scale, uint16_t* dst_hi,
                                             uint16_t* dst_lo) {
  float h[4], l[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) split_hi_lo(__fmul_rn(v[j], scale), h[j], l[j]);
  *reinterpret_cast<uint2*>(dst_hi) = make_uint2(pack_bf16x2(h[0], h[1]), pack_bf16x2(h[2], h[3]));
  *reinterpret_cast<uint2*>(dst_lo) = make_uint2(pack_bf16x2(l[0], l[1]), pack_bf16x2(l[2], l[3]));
}

__global__ void __launch_bounds__(QA_THREADS, 1)
    quantize_act_kernel(const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_l1,
                        const __grid_constant__ CUtensorMap tm_codes, const QAParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int r = p.r;
  const bool has_lr = r > 0;
  const QALayout& L = p.L;
  const int XST = L.xst, LST = L.lst, NSTG = L.nstg;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar_off);
  const uint32_t x_full0 = smem_u32(bars);
  const uint32_t x_empty0 = x_full0 + 8 * XST;
  const uint32_t l_full0 = x_empty0 + 8 * XST;
  const uint32_t l_empty0 = l_full0 + 8 * LST;
  const uint32_t staged0 = l_empty0 + 8 * LST;
  const uint32_t free0 = staged0 + 8 * NSTG;
  const uint32_t acc_full = free0 + 8 * NSTG;
  const uint32_t s_bar = acc_full + 8;
  const uint32_t drain_bar = acc_full + 24;
  uint32_t* tmem_holder =
      reinterpret_cast<uint32_t*>(bars + 2 * XST + 2 * LST + 2 * NSTG + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_holder + 1);
  float* qlut = reinterpret_cast<float*>(smem + L.lut_off);  // 128 floats
  const float* s_sm = reinterpret_cast<const float*>(smem + L.s_off);

  const uint32_t warp = warp_id(), lane = lane_id();
  const int split = blockIdx.x;  // always 0: one CTA walks all of K
  const int rb = blockIdx.y;
  const int kchunks = ((p.K >> 6) + QA_BOXES - 1) / QA_BOXES;   // 128-column chunks
  const int k64 = p.K >> 6;
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
      mbar_init(x_empty0 + 8 * i, QA_UNITS + (has_lr ? 1 : 0));  // its 8 units + the MMA
    }
    for (int i = 0; i < LST; ++i) {
      mbar_init(l_full0 + 8 * i, 1);
      mbar_init(l_empty0 + 8 * i, 1);
    }
    for (int i = 0; i < NSTG; ++i) {
      mbar_init(staged0 + 8 * i, QA_UNITS);
      mbar_init(free0 + 8 * i, 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(s_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    mbar_fence_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tm_x);
    prefetch_tensormap(&tm_codes);
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
        mbar_arrive_expect_tx(x_full0 + 8 * st, QA_X_BYTES);
        // (a box past K or rows past M read zeros: the TMA fill)
        for (int b = 0; b < QA_BOXES; ++b)
          tma_load_2d(smem_u32(smem + st * QA_X_BYTES + b * QA_BOX_BYTES), &tm_x,
                      (c_begin + cl) * 128 + 64 * b, rb * QA_BM, x_full0 + 8 * st);
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
        for (int b = 0; b < QA_BOXES; ++b)
          tma_load_2d(smem_u32(smem + L.l1_off + st * L.l1_bytes + b * (L.l1_bytes / QA_BOXES)),
                      &tm_l1, (c_begin + cl) * 128 + 64 * b, 0, l_full0 + 8 * st);
        l_issued = i + 1;
        if (++st == LST) { st = 0; ph ^= 1; }
        if (++cl == nchunks) cl = 0;
      }
    }
    __syncwarp();
  } else if (warp == 3) {
    // ------------------------------------------ code / scale stores (TMA) ----
    // A chunk's slot is written out once its 8 units have staged it; the
    // slot is handed back when the stores have read it.
    if (lane == 0) {
      int cl = rot;
      for (int i = 0; i < nchunks; ++i) {
        const int slot = i % NSTG;
        if (!mbar_wait(staged0 + 8 * slot, (uint32_t)(i / NSTG) & 1u, p.timeout_ns, abort_flag,
                       (8u << 8) | kid))
          break;
        const int c = c_begin + cl;
        const uint32_t src = smem_u32(smem + L.stg_off + slot * QA_STG_BYTES);
        // codes: one 128-row x 64-byte box (columns past K/2, rows past M
        // are clipped by the TMA)
        tma_store_2d(&tm_codes, src, c * 64, rb * QA_BM);
        // scales: the chunk's two 512-byte atoms (only the first when the
        // chunk's second 64 columns lie past K), contiguous in the tiles
        const int atoms = (2 * c + 1 < k64) ? 2 : 1;
        bulk_store(p.sf_x + ((size_t)rb * k64 + 2 * c) * 512, src + QA_CODES_STG,
                   512u * (uint32_t)atoms);
        bulk_commit_group();
        bulk_wait_read_all();
        mbar_arrive(free0 + 8 * slot);
        if (++cl == nchunks) cl = 0;
      }
      // no store may still be reading shared memory (or writing) at exit
      bulk_wait_all();
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------ down-projection (warp) ----
    if (has_lr) {
      const uint32_t idesc = idesc_bf16(QA_BM, 2 * r);
      int xs = 0, ls = 0;
      uint32_t xph = 0, lph = 0;
      for (int i = 0; i < nchunks; ++i) {
        // both tiles have landed (complete_tx); the MMAs read them through
        // the async proxy
        if (!mbar_wait_warp(x_full0 + 8 * xs, xph, p.timeout_ns, abort_flag, (2u << 8) | kid)) break;
        if (!mbar_wait_warp(l_full0 + 8 * ls, lph, p.timeout_ns, abort_flag, (2u << 8) | kid)) break;
        // the chunk's MMAs and both releases from one elected lane (fewer
        // issue slots on a sub-partition shared with the quantize warps, so
        // the X ring turns over sooner)
        if (elect_one()) {
#pragma unroll
          for (int b = 0; b < QA_BOXES; ++b) {
            const uint64_t da = sdesc_sw128(smem_u32(smem + xs * QA_X_BYTES + b * QA_BOX_BYTES));
            const uint64_t db = sdesc_sw128(
                smem_u32(smem + L.l1_off + ls * L.l1_bytes + b * (L.l1_bytes / QA_BOXES)));
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
    const int qw = warp - QA_QWARP0;
    bool ok = nchunks == 0 || mbar_wait_warp(s_bar, 0, p.timeout_ns, abort_flag, (3u << 8) | kid);
    for (int u = qw; ok && u < QA_UNITS * nchunks; u += QA_QWARPS) {
      const int i = u / QA_UNITS;
      const int box = (u % QA_UNITS) >> 2;
      const int quarter = u & 3;
      const int cl = i + rot < nchunks ? i + rot : i + rot - nchunks;  // local chunk
      const int st = i % XST;
      const uint32_t ph = (uint32_t)(i / XST) & 1u;
      if (!mbar_wait_warp(x_full0 + 8 * st, ph, p.timeout_ns, abort_flag, (3u << 8) | kid)) break;
      const int row_t = 32 * quarter + lane;
      const int col0 = (c_begin + cl) * 128 + 64 * box;   // first column of the unit
      const bool live = col0 < p.K;                       // else the zero box past K
      // this row's tensor scales: the static ones, or (dynamic mode) its own
      const int row = rb * QA_BM + row_t;
      const bool dyn = p.row_scales != nullptr;
      float g_row = p.g_x, gs = p.gs_x;
      if (dyn && row < p.M) {
        g_row = p.row_scales[row].g;
        gs = p.row_scales[row].gs;
      }
      uint4 xr[8];
      if (live) {
        // copy this lane's row segment into registers, then hand the stage
        // back so the next chunk can land while this one is quantized
        const uint8_t* xrow = smem + st * QA_X_BYTES + box * QA_BOX_BYTES + row_t * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          xr[j] = *reinterpret_cast<const uint4*>(xrow + ((j ^ (row_t & 7)) << 4));
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) xr[j] = make_uint4(0, 0, 0, 0);
      }
      // Hand the stage back only after the reads are done and ordered before
      // the next fill.  The fill is a TMA write (async proxy) after these
      // generic-proxy reads of the same bytes: each lane folds its loaded
      // words into one value (its loads have landed), the warp reduces those,
      // every lane fences the generic proxy against the async proxy, and
      // lane 0 releases.  Without the proxy fence an occasional refill
      // overwrote a stage while a warp's reads of it were still being served.
      uint32_t dep = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) dep ^= xr[j].x ^ xr[j].y ^ xr[j].z ^ xr[j].w;
      dep = __reduce_or_sync(0xffffffffu, dep);
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive_after(x_empty0 + 8 * st, dep);
      uint32_t cw[8];
      uint32_t sfw = 0;
      if (live) {
        const float4* sp = reinterpret_cast<const float4*>(s_sm + cl * 128 + 64 * box);
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
      }
      // stage the unit's codes and scales; the slot must have been read out
      // by the stores of the chunk that used it before
      const int slot = i % NSTG;
      if (i >= NSTG &&
          !mbar_wait_warp(free0 + 8 * slot, (uint32_t)(i / NSTG - 1) & 1u, p.timeout_ns, abort_flag,
                          (9u << 8) | kid))
        break;
      if (live) {
        const uint32_t sbase = smem_u32(smem + L.stg_off + slot * QA_STG_BYTES);
        // codes row of 64 bytes, 16-byte chunk c at slot c ^ ((row / 2) % 4)
        // (the 64-byte swizzle of the store's tensor map); this unit holds
        // chunks 2 box and 2 box + 1
        const uint32_t rowb = sbase + (uint32_t)row_t * 64u;
        const uint32_t sw = (uint32_t)(row_t >> 1) & 3u;
        st_shared_v4(rowb + (((2u * box) ^ sw) << 4), cw[0], cw[1], cw[2], cw[3]);
        st_shared_v4(rowb + (((2u * box + 1u) ^ sw) << 4), cw[4], cw[5], cw[6], cw[7]);
        // scale word of the row in the chunk's atom `box`
        st_shared_u32(sbase + QA_CODES_STG + (uint32_t)box * 512u + lane * 16u + quarter * 4u, sfw);
      }
      fence_proxy_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(staged0 + 8 * slot);
    }
  }

  // ----------------------------------------- low-rank epilogue (X L1) ----
  if (has_lr && warp >= QA_QWARP0) {
    const bool ok = mbar_wait_warp(acc_full, 0, p.timeout_ns, abort_flag, (4u << 8) | kid);
    tc_fence_after();
    // M = 128 accumulator: row m sits in tensor-memory lane m; warp w reads
    // its lane quarter w % 4.  The four warps of one quarter split the r
    // columns: slot (w - QA_QWARP0) / 4 takes columns [slot r/4, slot r/4 +
    // r/4), in groups of four.
    const int quad = warp & 3;
    const int slot = (warp - QA_QWARP0) >> 2;
    const int cw4 = r / 16;                       // groups of 4 columns per slot
    const int row_t = quad * 32 + lane;
    const int row = rb * QA_BM + row_t;
    const uint32_t tbase = tmem + ((uint32_t)(quad * 32) << 16);
#pragma unroll
    for (int g = 0; g < 8; ++g) {
      if (g < cw4) {
        const int col = slot * 4 * cw4 + 4 * g;   // first of the group's 4 columns
        uint32_t hi[4], lo[4];
        if (ok && nchunks > 0) {
          tmem_ld4(tbase + col, hi);
          tmem_ld4(tbase + r + col, lo);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) hi[j] = lo[j] = 0u;
        }
        float sum[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) sum[j] = __uint_as_float(hi[j]) + __uint_as_float(lo[j]);
        if (row < p.M)
          store_hi_lo4(sum, p.row_scales ? p.row_scales[row].lr : p.lr_scale,
                       p.xl1 + (size_t)row * p.klr + col,
                       p.xl1 + (size_t)row * p.klr + r + col);
      }
    }
    // zero columns [2r, klr) of this row block
    if (slot == 0 && row < p.M) {
      for (int cpad = 2 * r; cpad < p.klr; cpad += 8)
        *reinterpret_cast<uint4*>(p.xl1 + (size_t)row * p.klr + cpad) = make_uint4(0, 0, 0, 0);
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
  if (warp == 1 && has_lr) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

}  // namespace svdq_dev
