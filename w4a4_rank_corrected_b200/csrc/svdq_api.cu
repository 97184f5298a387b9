// C ABI of the B200 SVDQuant W4A4 linear: argument checks, tensor-map
// (TMA descriptor) encoding and kernel launches.  See include/svdq.h for the
// contract of every entry point.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/svdq.h"
#include "ptx.cuh"
#include "quantize_act.cuh"
#include "quantize_act64.cuh"
#include "row_scales.cuh"
#include "awq_gemv.cuh"
#include "w4a4_gemm.cuh"

namespace svdq_dev {

// Never satisfied wait: exercises the bounded-wait error path.
__global__ void selftest_timeout_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0)
    mbar_wait(smem_u32(&bar), 0, timeout_ns, &abort_flag, (7u << 8) | 3u);
  __syncthreads();
}

// The epilogue's GELU on arbitrary bf16 inputs, one value per thread.
__global__ void debug_gelu_kernel(const uint16_t* in, uint16_t* out, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float y = __uint_as_float((uint32_t)in[i] << 16);
  const float h = gelu_bf16_value(y);
  out[i] = (uint16_t)(__float_as_uint(h) >> 16);
}

// The hardware conversions of the activation kernel, one value per thread.
__global__ void debug_convert_kernel(const float* in, uint8_t* e2m1, uint8_t* e4m3, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float x = in[i];
  if (e2m1) {
    const float v[8] = {x, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    e2m1[i] = (uint8_t)(cvt_e2m1x8(v) & 0xF);
  }
  if (e4m3) e4m3[i] = (uint8_t)(cvt_e4m3x2(fabsf(x), 0.0f) & 0xFF);
}
}  // namespace svdq_dev

using namespace svdq_dev;

namespace {

constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;  // 1 s per wait

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceInfo {
  bool checked = false;
  bool ok = false;
  int num_sms = 0;
  bool attrs_set = false;
  // max co-resident clusters of the 64-row activation kernel per cluster
  // size S (1..8; every shared-memory plan holds one CTA per SM, so r does
  // not matter); -1 = not queried yet
  int q64_clusters[9];
  int gemm_pairs = -1;  // max co-resident CTA pairs of the GEMM kernel
  DeviceInfo() {
    for (int& v : q64_clusters) v = -1;
  }
};
constexpr int kMaxDevices = 64;
DeviceInfo g_dev[kMaxDevices];
std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;

svdq_status device_check(int* sms) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return SVDQ_ERR_UNSUPPORTED_ARCH;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.checked) {
    int major = 0, minor = 0, n = 0;
    const bool q = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) == cudaSuccess &&
                   cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) == cudaSuccess &&
                   cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess;
    cudaGetLastError();
    d.checked = true;
    d.ok = q && major == 10 && minor == 0;
    d.num_sms = n;
  }
  if (!d.ok) return SVDQ_ERR_UNSUPPORTED_ARCH;
  if (!d.attrs_set) {
    const uint32_t qa_max = 1024u + QA_SMEM_BUDGET + 512u;  // every qa_layout fits
    const uint32_t q64_max = 1024u + Q64_SMEM_BUDGET + 512u;
    if (cudaFuncSetAttribute(quantize_act_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)qa_max) != cudaSuccess ||
        cudaFuncSetAttribute(quantize_act64_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)q64_max) != cudaSuccess ||
        cudaFuncSetAttribute(w4a4_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)gemm_smem_bytes()) != cudaSuccess) {
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    d.attrs_set = true;
  }
  if (!g_encode) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult qres;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &qres) !=
            cudaSuccess ||
        qres != cudaDriverEntryPointSuccess || !fn) {
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
    g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  }
  if (sms) *sms = d.num_sms;
  return SVDQ_OK;
}

// 2D tensor map over a row-major [rows][inner] matrix (128-byte swizzle
// unless `swizzle` says otherwise).
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
              uint64_t rows, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
              CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_128B) {
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return g_encode(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }
inline size_t rup(size_t x, size_t m) { return (x + m - 1) / m * m; }

svdq_status check_weight(const svdq_weight* w) {
  if (!w) return SVDQ_ERR_INVALID_ARG;
  svdq_sizes sz;
  if (svdq_query_sizes(w->N, w->K, w->r, &sz) != SVDQ_OK) return SVDQ_ERR_INVALID_ARG;
  if (!w->smooth || !w->codes_w || !w->sf_w) return SVDQ_ERR_INVALID_ARG;
  if (w->r > 0 && (!w->l1_mma || !w->l2_mma)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(w->smooth) || !aligned16(w->codes_w) || !aligned16(w->sf_w) ||
      (w->bias && !aligned16(w->bias)) || (w->l1_mma && !aligned16(w->l1_mma)) ||
      (w->l2_mma && !aligned16(w->l2_mma)))
    return SVDQ_ERR_MISALIGNED;
  return SVDQ_OK;
}

int klr_of(int r) { return (int)rup((size_t)2 * r, 64); }

cudaLaunchAttribute pdl_attr() {
  cudaLaunchAttribute a;
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
  return a;
}

// Largest K split S (cluster size when the low-rank branch needs the
// cross-CTA reduction) such that the whole grid is resident in one wave and
// the split's shared-memory plan keeps a deep enough activation ring.
int choose_splits64(int tiles, int kchunks, int r, int sms) {
  int dev = 0;
  cudaGetDevice(&dev);
  int best = 1;
  for (int S = 2; S <= 8; ++S) {
    if (S > kchunks || tiles * S > sms) break;
    const int cps = (kchunks + S - 1) / S;
    const Q64Layout L = q64_layout(r, cps, S);
    if (L.xst < Q64_MIN_XST) break;
    if (r > 0) {
      std::lock_guard<std::mutex> lk(g_mu);   // the caches are shared by host threads
      int& cached = g_dev[dev].q64_clusters[S];
      if (cached < 0) {
        cudaLaunchConfig_t cfg;
        std::memset(&cfg, 0, sizeof(cfg));
        cfg.gridDim = dim3((unsigned)S, 1, 1);
        cfg.blockDim = dim3(Q64_THREADS, 1, 1);
        cfg.dynamicSmemBytes = L.total;
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = (unsigned)S;
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, quantize_act64_kernel, &cfg) != cudaSuccess) {
          cudaGetLastError();
          n = 0;
        }
        cached = n;
      }
      if (tiles > cached) continue;
    }
    best = S;
  }
  return best;
}

svdq_status launch_quantize64(const svdq_weight* w, const uint16_t* X, int M, int64_t ldx,
                              uint8_t* codes_x, uint8_t* sf_x, uint16_t* xl1, cudaStream_t s,
                              int sms, const RowScale* rs) {
  const int K = w->K, r = w->r;
  // 64-row tiles covering whole 128-row scale atoms (padding rows get zero
  // scales)
  const int tiles = 2 * ((M + 127) / 128);
  const int KC = (K / 64 + Q64_BOXES - 1) / Q64_BOXES;  // 128-column chunks
  int S = choose_splits64(tiles, KC, r, sms);
  const int cps = (KC + S - 1) / S;
  S = (KC + cps - 1) / cps;
  const Q64Layout L = q64_layout(r, cps, S);
  if (L.xst < Q64_MIN_XST) return SVDQ_ERR_INVALID_ARG;  // K too large for one CTA's slice

  CUtensorMap tm_x, tm_l1;
  std::memset(&tm_l1, 0, sizeof(tm_l1));
  if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M,
                (uint64_t)ldx * 2, 64, Q64_BM))
    return SVDQ_ERR_CUDA;
  if (r > 0 && !make_map(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->l1_mma, (uint64_t)K,
                         (uint64_t)(2 * r), (uint64_t)K * 2, 64, (uint32_t)(2 * r)))
    return SVDQ_ERR_CUDA;

  Q64Params p;
  p.row_scales = rs;
  p.smooth = w->smooth;
  p.codes_x = codes_x;
  p.sf_x = sf_x;
  p.xl1 = xl1;
  p.M = M;
  p.K = K;
  p.r = r;
  p.klr = klr_of(r);
  p.chunks_per_split = cps;
  p.num_splits = S;
  p.L = L;
  uint32_t cols = 32;
  while (cols < (uint32_t)(2 * r)) cols <<= 1;
  p.tmem_cols = cols;
  p.g_x = w->g_x;
  p.gs_x = w->gs_x;
  p.lr_scale = w->lr_scale;
  p.timeout_ns = kDefaultTimeoutNs;

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)S, (unsigned)tiles, 1);
  cfg.blockDim = dim3(Q64_THREADS, 1, 1);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0] = pdl_attr();
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (r > 0 && S > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)S;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  if (cudaLaunchKernelEx(&cfg, quantize_act64_kernel, tm_x, tm_l1, p) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// The 128-row kernel: one CTA per 128-row block, all of K.
svdq_status launch_quantize128(const svdq_weight* w, const uint16_t* X, int M, int64_t ldx,
                               uint8_t* codes_x, uint8_t* sf_x, uint16_t* xl1, cudaStream_t s,
                               const RowScale* rs) {
  const int K = w->K, r = w->r;
  // 128-row tiles: one scale-factor atom row each (padding rows get zero
  // scales)
  const int tiles = (M + QA_BM - 1) / QA_BM;
  const int KC = (K / 64 + QA_BOXES - 1) / QA_BOXES;  // 128-column chunks
  const int S = 1;
  const int cps = KC;
  const QALayout L = qa_layout(r, cps);
  if (L.xst < QA_MIN_XST || L.nstg < QA_MIN_NSTG || (r > 0 && L.lst < 1))
    return SVDQ_ERR_INVALID_ARG;  // K too large for one CTA's slice

  CUtensorMap tm_x, tm_l1, tm_codes;
  std::memset(&tm_l1, 0, sizeof(tm_l1));
  if (!make_map(&tm_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M,
                (uint64_t)ldx * 2, 64, QA_BM))
    return SVDQ_ERR_CUDA;
  // codes are stored in 128-row x 64-byte boxes, 64-byte swizzle
  if (!make_map(&tm_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes_x, (uint64_t)K / 2, (uint64_t)M,
                (uint64_t)K / 2, 64, QA_BM, CU_TENSOR_MAP_SWIZZLE_64B))
    return SVDQ_ERR_CUDA;
  if (r > 0 && !make_map(&tm_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->l1_mma, (uint64_t)K,
                         (uint64_t)(2 * r), (uint64_t)K * 2, 64, (uint32_t)(2 * r)))
    return SVDQ_ERR_CUDA;

  QAParams p;
  p.row_scales = rs;
  p.smooth = w->smooth;
  p.sf_x = sf_x;
  p.xl1 = xl1;
  p.M = M;
  p.K = K;
  p.r = r;
  p.klr = klr_of(r);
  p.chunks_per_split = cps;
  p.num_splits = S;
  p.L = L;
  uint32_t cols = 32;
  while (cols < (uint32_t)(2 * r)) cols <<= 1;
  p.tmem_cols = cols;
  p.g_x = w->g_x;
  p.gs_x = w->gs_x;
  p.lr_scale = w->lr_scale;
  p.timeout_ns = kDefaultTimeoutNs;

  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)S, (unsigned)tiles, 1);
  cfg.blockDim = dim3(QA_THREADS, 1, 1);
  cfg.dynamicSmemBytes = p.L.total;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0] = pdl_attr();
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, quantize_act_kernel, tm_x, tm_l1, tm_codes, p) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// Which activation kernel: the 128-row kernel once 128-row blocks alone
// nearly fill the machine (>= 120 blocks on 148 SMs: every byte of the
// low-rank operand then serves 128 rows and no K split is needed); below
// that the 64-row kernel, whose K split within a cluster keeps every SM
// busy.
svdq_status launch_quantize(const svdq_weight* w, const uint16_t* X, int M, int64_t ldx,
                            uint8_t* codes_x, uint8_t* sf_x, uint16_t* xl1, cudaStream_t s,
                            int sms, const RowScale* rs = nullptr) {
  const int tiles128 = (M + QA_BM - 1) / QA_BM;
  if (tiles128 * 148 >= 120 * sms)
    return launch_quantize128(w, X, M, ldx, codes_x, sf_x, xl1, s, rs);
  return launch_quantize64(w, X, M, ldx, codes_x, sf_x, xl1, s, sms, rs);
}

// The per-row scales of the dynamic mode: one warp per row, 8 rows per CTA.
svdq_status launch_row_scales(const svdq_weight* w, const uint16_t* X, int M, int64_t ldx,
                              RowScale* rs, cudaStream_t s, int sms) {
  const int blocks = std::max(1, std::min((M + 7) / 8, 16 * sms));
  row_scales_kernel<<<blocks, 256, 0, s>>>(X, ldx, w->smooth, M, w->K, w->g_w, rs);
  if (cudaGetLastError() != cudaSuccess) return SVDQ_ERR_CUDA;
  return SVDQ_OK;
}

int gemm_max_pairs(int sms) {
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(g_mu);   // the caches are shared by host threads
  int& cached = g_dev[dev].gemm_pairs;
  if (cached < 0) {
    cudaLaunchConfig_t cfg;
    std::memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(2, 1, 1);
    cfg.blockDim = dim3(G_THREADS, 1, 1);
    cfg.dynamicSmemBytes = gemm_smem_bytes();
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, w4a4_gemm_kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = sms / 2;
    }
    cached = std::min(n, sms / 2);
  }
  return std::max(1, cached);
}

// Split-K for few output tiles and long K: with at most 16 tiles of
// 256 x 256 (the GEMM has 74 CTA pairs on a B200) and at least 24 stages of
// 256 along K, each tile's K is split into min(8, 64 / tiles, stages / 6)
// parts.  The split adds a second kernel and a round trip of fp32 partials
// through L2, about 5 us; measured, it pays at K = 12288 (M = 64: 16.5 against
// 21.2 us whole-K; M = 256: 18.5 against 22.0 us), breaks even at 24 tiles and
// loses at K = 3072 (12.4 against 9.2 us).  The rule depends on the shapes
// only, so the workspace size does too.
constexpr int kSplitTileLimit = 16;
constexpr int kSplitMinStages = 24;
constexpr int kSplitUnits = 64;
constexpr int kSplitMax = 8;
int gemm_tiles(int M, int N) { return ((M + 2 * G_BM - 1) / (2 * G_BM)) * ((N + G_BN - 1) / G_BN); }
int gemm_ksplit(int M, int N, int K) {
  const int tiles = gemm_tiles(M, N), kb_total = (K / 64 + 3) / 4;
  if (tiles > kSplitTileLimit || kb_total < kSplitMinStages) return 1;
  return std::max(1, std::min(std::min(kSplitMax, kSplitUnits / tiles), kb_total / 6));
}
// partials [tiles][ksplit][2][128][256] fp32
size_t gemm_split_ws_bytes(int M, int N, int K) {
  if (M <= 0 || gemm_ksplit(M, N, K) <= 1) return 0;
  return (size_t)gemm_tiles(M, N) * gemm_ksplit(M, N, K) * 2 * G_BM * G_BN * 4;
}

svdq_status launch_gemm(const svdq_weight* w, const uint8_t* codes_x, const uint8_t* sf_x,
                        const uint16_t* xl1, int M, uint16_t* Y, int64_t ldy, cudaStream_t s,
                        int sms, bool gelu = false, const RowScale* rs = nullptr,
                        void* split_ws = nullptr) {
  const int N = w->N, K = w->K, r = w->r, klr = klr_of(r);
  CUtensorMap ta, tb, tsa, tsb, talr, tblr, ty, tpart;
  std::memset(&talr, 0, sizeof(talr));
  std::memset(&tblr, 0, sizeof(tblr));
  std::memset(&tpart, 0, sizeof(tpart));
  // scale buffers as rows of 256 bytes (half a 512-byte atom), unswizzled
  const uint64_t sfa_rows = rup((size_t)M, 128) * (K / 16) / 256;
  const uint64_t sfb_rows = rup((size_t)N, 256) * (K / 16) / 256;
  if (!make_map(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, codes_x, (uint64_t)K / 2, (uint64_t)M,
                (uint64_t)K / 2, 128, G_BM) ||
      !make_map(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->codes_w, (uint64_t)K / 2, (uint64_t)N,
                (uint64_t)K / 2, 128, G_BN_CTA) ||
      !make_map(&tsa, CU_TENSOR_MAP_DATA_TYPE_UINT8, sf_x, 256, sfa_rows, 256, 256, 8,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_map(&tsb, CU_TENSOR_MAP_DATA_TYPE_UINT8, w->sf_w, 256, sfb_rows, 256, 256, 8,
                CU_TENSOR_MAP_SWIZZLE_NONE) ||
      // Y is written in 128-row x 64-column boxes (128-byte swizzle)
      !make_map(&ty, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Y, (uint64_t)N, (uint64_t)M,
                (uint64_t)ldy * 2, G_OUT_COLS, G_BM))
    return SVDQ_ERR_CUDA;
  if (r > 0) {
    if (!make_map(&talr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xl1, (uint64_t)klr, (uint64_t)M,
                  (uint64_t)klr * 2, 64, G_BM) ||
        !make_map(&tblr, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, w->l2_mma, (uint64_t)klr, (uint64_t)N,
                  (uint64_t)klr * 2, 64, G_BN_CTA))
      return SVDQ_ERR_CUDA;
  }
  GemmParams p;
  p.bias = w->bias;
  p.M = M;
  p.N = N;
  p.K = K;
  p.r = r;
  p.klr = klr;
  p.alpha = w->alpha;
  p.timeout_ns = kDefaultTimeoutNs;
  p.gelu = gelu ? 1 : 0;
  p.row_scales = rs;
  const int tiles = gemm_tiles(M, N);
  // (the split is for the plain layer: not with GELU or per-row scales)
  p.ksplit = (split_ws && !gelu && !rs) ? gemm_ksplit(M, N, K) : 1;
  p.partials = p.ksplit > 1 ? static_cast<float*>(split_ws) : nullptr;
  // the partials as a 2-D fp32 tensor [tiles * ksplit * 256 rows][256], stored
  // in 128-row x 32-column boxes (128-byte swizzle, as the Y boxes)
  if (p.ksplit > 1 &&
      !make_map(&tpart, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, p.partials, (uint64_t)G_BN,
                (uint64_t)tiles * p.ksplit * 2 * G_BM, (uint64_t)G_BN * 4, 32, G_BM))
    return SVDQ_ERR_CUDA;
  const int pairs = std::max(1, std::min(tiles * p.ksplit, gemm_max_pairs(sms)));
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(2 * pairs), 1, 1);
  cfg.blockDim = dim3(G_THREADS, 1, 1);
  cfg.dynamicSmemBytes = gemm_smem_bytes();
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0] = pdl_attr();
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, w4a4_gemm_kernel, ta, tb, tsa, tsb, talr, tblr, ty, tpart, p) !=
      cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  if (p.ksplit > 1) {
    // the partials -> Y, chained to the GEMM by programmatic dependent launch
    const long long threads = (long long)M * (N / 8);
    cudaLaunchConfig_t rc;
    std::memset(&rc, 0, sizeof(rc));
    rc.gridDim = dim3((unsigned)std::max(1LL, std::min((threads + 255) / 256, 4LL * sms)), 1, 1);
    rc.blockDim = dim3(256, 1, 1);
    rc.stream = s;
    cudaLaunchAttribute ra = pdl_attr();
    rc.attrs = &ra;
    rc.numAttrs = 1;
    if (cudaLaunchKernelEx(&rc, splitk_reduce_kernel, (const float*)p.partials, M, N, p.ksplit,
                           p.alpha, p.bias, Y, ldy) != cudaSuccess) {
      cudaGetLastError();
      return SVDQ_ERR_CUDA;
    }
  }
  return SVDQ_OK;
}

size_t ws_codes(int M, int K) { return rup((size_t)M * (K / 2), 256); }
size_t ws_sf(int M, int K) { return rup(rup((size_t)M, 128) * (K / 16), 256); }
size_t ws_xl1(int M, int r) { return rup((size_t)M * klr_of(r) * 2, 256); }

}  // namespace

extern "C" const char* svdq_status_string(svdq_status s) {
  switch (s) {
    case SVDQ_OK: return "ok";
    case SVDQ_ERR_INVALID_ARG: return "invalid argument";
    case SVDQ_ERR_UNSUPPORTED_ARCH: return "unsupported device (an sm_100 B200 is required)";
    case SVDQ_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
    case SVDQ_ERR_WORKSPACE: return "workspace too small";
    case SVDQ_ERR_CUDA: return "CUDA runtime error";
    case SVDQ_ERR_TIMEOUT: return "a kernel wait timed out";
    case SVDQ_ERR_NUMERIC: return "non-finite input";
  }
  return "unknown status";
}

extern "C" const char* svdq_version(void) { return "svdq-b200 0.1"; }

extern "C" size_t svdq_act_workspace_bytes(int M, int K, int r) {
  if (M < 0 || K <= 0 || K % 64 || r < 0 || r > 128 || (r && r % 16)) return 0;
  return ws_codes(M, K) + ws_sf(M, K) + (r > 0 ? ws_xl1(M, r) : 0);
}

extern "C" svdq_status svdq_quantize_act(const svdq_weight* w, const uint16_t* X, int M,
                                         int64_t ldx, uint8_t* codes_x, uint8_t* sf_x,
                                         uint16_t* xl1, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx < w->K) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !codes_x || !sf_x || (w->r > 0 && !xl1)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || ldx % 8 || !aligned16(codes_x) || !aligned16(sf_x) ||
      (xl1 && !aligned16(xl1)))
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_quantize(w, X, M, ldx, codes_x, sf_x, xl1, (cudaStream_t)stream, sms);
}

extern "C" svdq_status svdq_gemm(const svdq_weight* w, const uint8_t* codes_x,
                                 const uint8_t* sf_x, const uint16_t* xl1, int M, uint16_t* Y,
                                 int64_t ldy, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldy < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!codes_x || !sf_x || !Y || (w->r > 0 && !xl1)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(codes_x) || !aligned16(sf_x) || !aligned16(Y) || ldy % 8 ||
      (xl1 && !aligned16(xl1)))
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_gemm(w, codes_x, sf_x, xl1, M, Y, ldy, (cudaStream_t)stream, sms);
}

extern "C" size_t svdq_gemm_workspace_bytes(int M, int N, int K) {
  if (M < 0 || N <= 0 || K <= 0 || K % 64) return 0;
  return gemm_split_ws_bytes(M, N, K);
}

extern "C" svdq_status svdq_gemm_splitk(const svdq_weight* w, const uint8_t* codes_x,
                                        const uint8_t* sf_x, const uint16_t* xl1, int M,
                                        uint16_t* Y, int64_t ldy, void* workspace,
                                        size_t ws_bytes, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldy < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!codes_x || !sf_x || !Y || (w->r > 0 && !xl1)) return SVDQ_ERR_INVALID_ARG;
  const size_t need = gemm_split_ws_bytes(M, w->N, w->K);
  if (need && (!workspace || ws_bytes < need)) return SVDQ_ERR_WORKSPACE;
  if (!aligned16(codes_x) || !aligned16(sf_x) || !aligned16(Y) || ldy % 8 ||
      (xl1 && !aligned16(xl1)) || (reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_gemm(w, codes_x, sf_x, xl1, M, Y, ldy, (cudaStream_t)stream, sms, false, nullptr,
                     need ? workspace : nullptr);
}

extern "C" size_t svdq_forward_workspace_bytes(const svdq_weight* w, int M) {
  if (!w || M < 0) return 0;
  const size_t a = svdq_act_workspace_bytes(M, w->K, w->r);
  if (!a && M > 0) return 0;
  const size_t g = gemm_split_ws_bytes(M, w->N, w->K);
  return g ? rup(a, 256) + g : a;
}

extern "C" svdq_status svdq_gemm_gelu(const svdq_weight* w, const uint8_t* codes_x,
                                      const uint8_t* sf_x, const uint16_t* xl1, int M,
                                      uint16_t* H, int64_t ldh, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldh < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!codes_x || !sf_x || !H || (w->r > 0 && !xl1)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(codes_x) || !aligned16(sf_x) || !aligned16(H) || ldh % 8 ||
      (xl1 && !aligned16(xl1)))
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_gemm(w, codes_x, sf_x, xl1, M, H, ldh, (cudaStream_t)stream, sms, true);
}

extern "C" size_t svdq_mlp_workspace_bytes(int M, int K1, int N1, int r1, int r2) {
  const size_t a = svdq_act_workspace_bytes(M, K1, r1), b = svdq_act_workspace_bytes(M, N1, r2);
  if (!a || !b) return 0;
  return std::max(a, b);
}

extern "C" svdq_status svdq_mlp_forward(const svdq_weight* w1, const svdq_weight* w2,
                                        const uint16_t* X, int M, int64_t ldx, uint16_t* H,
                                        int64_t ldh, uint16_t* Y, int64_t ldy, void* workspace,
                                        size_t ws_bytes, void* stream) {
  svdq_status st = check_weight(w1);
  if (st != SVDQ_OK) return st;
  if ((st = check_weight(w2)) != SVDQ_OK) return st;
  if (w2->K != w1->N) return SVDQ_ERR_INVALID_ARG;
  if (M < 0 || ldx < w1->K || ldh < w1->N || ldy < w2->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !H || !Y || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (ws_bytes < svdq_mlp_workspace_bytes(M, w1->K, w1->N, w1->r, w2->r)) return SVDQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return SVDQ_ERR_MISALIGNED;
  if (!aligned16(X) || !aligned16(H) || !aligned16(Y) || ldx % 8 || ldh % 8 || ldy % 8)
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  for (int layer = 0; layer < 2; ++layer) {
    const svdq_weight* w = layer == 0 ? w1 : w2;
    const uint16_t* in = layer == 0 ? X : H;
    const int64_t ldin = layer == 0 ? ldx : ldh;
    uint8_t* codes_x = static_cast<uint8_t*>(workspace);
    uint8_t* sf_x = codes_x + ws_codes(M, w->K);
    uint16_t* xl1 = w->r > 0 ? reinterpret_cast<uint16_t*>(sf_x + ws_sf(M, w->K)) : nullptr;
    if ((st = launch_quantize(w, in, M, ldin, codes_x, sf_x, xl1, s, sms)) != SVDQ_OK) return st;
    if ((st = launch_gemm(w, codes_x, sf_x, xl1, M, layer == 0 ? H : Y, layer == 0 ? ldh : ldy, s,
                          sms, layer == 0)) != SVDQ_OK)
      return st;
  }
  return SVDQ_OK;
}

extern "C" svdq_status svdq_debug_gelu(const uint16_t* in, uint16_t* out, int64_t n,
                                       void* stream) {
  if (n < 0 || (n > 0 && (!in || !out))) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  svdq_status st = device_check(nullptr);
  if (st != SVDQ_OK) return st;
  const int64_t blocks = (n + 255) / 256;
  if (blocks > 0x7FFFFFFF) return SVDQ_ERR_INVALID_ARG;
  debug_gelu_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(in, out, n);
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

extern "C" svdq_status svdq_act_row_scales(const svdq_weight* w, const uint16_t* X, int M,
                                           int64_t ldx, void* row_scales, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx < w->K) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !row_scales) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || ldx % 8 || !aligned16(row_scales)) return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_row_scales(w, X, M, ldx, static_cast<RowScale*>(row_scales), (cudaStream_t)stream,
                           sms);
}

extern "C" svdq_status svdq_quantize_act_dynamic(const svdq_weight* w, const uint16_t* X, int M,
                                                 int64_t ldx, const void* row_scales,
                                                 uint8_t* codes_x, uint8_t* sf_x, uint16_t* xl1,
                                                 void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx < w->K) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !row_scales || !codes_x || !sf_x || (w->r > 0 && !xl1)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(X) || ldx % 8 || !aligned16(codes_x) || !aligned16(sf_x) ||
      !aligned16(row_scales) || (xl1 && !aligned16(xl1)))
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_quantize(w, X, M, ldx, codes_x, sf_x, xl1, (cudaStream_t)stream, sms,
                         static_cast<const RowScale*>(row_scales));
}

extern "C" svdq_status svdq_gemm_dynamic(const svdq_weight* w, const uint8_t* codes_x,
                                         const uint8_t* sf_x, const uint16_t* xl1,
                                         const void* row_scales, int M, uint16_t* Y, int64_t ldy,
                                         void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldy < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!codes_x || !sf_x || !Y || !row_scales || (w->r > 0 && !xl1)) return SVDQ_ERR_INVALID_ARG;
  if (!aligned16(codes_x) || !aligned16(sf_x) || !aligned16(Y) || ldy % 8 ||
      !aligned16(row_scales) || (xl1 && !aligned16(xl1)))
    return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  return launch_gemm(w, codes_x, sf_x, xl1, M, Y, ldy, (cudaStream_t)stream, sms, false,
                     static_cast<const RowScale*>(row_scales));
}

extern "C" size_t svdq_dyn_workspace_bytes(int M, int K, int r) {
  const size_t a = svdq_act_workspace_bytes(M, K, r);
  if (!a) return 0;
  return a + rup((size_t)M * sizeof(RowScale), 256);
}

extern "C" svdq_status svdq_linear_forward_dynamic(const svdq_weight* w, const uint16_t* X, int M,
                                                   int64_t ldx, uint16_t* Y, int64_t ldy,
                                                   void* workspace, size_t ws_bytes, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx < w->K || ldy < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (ws_bytes < svdq_dyn_workspace_bytes(M, w->K, w->r)) return SVDQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return SVDQ_ERR_MISALIGNED;
  if (!aligned16(X) || !aligned16(Y) || ldx % 8 || ldy % 8) return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint8_t* codes_x = base;
  uint8_t* sf_x = codes_x + ws_codes(M, w->K);
  uint16_t* xl1 = w->r > 0 ? reinterpret_cast<uint16_t*>(sf_x + ws_sf(M, w->K)) : nullptr;
  RowScale* rs = reinterpret_cast<RowScale*>(base + svdq_act_workspace_bytes(M, w->K, w->r));
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = launch_row_scales(w, X, M, ldx, rs, s, sms)) != SVDQ_OK) return st;
  if ((st = launch_quantize(w, X, M, ldx, codes_x, sf_x, xl1, s, sms, rs)) != SVDQ_OK) return st;
  return launch_gemm(w, codes_x, sf_x, xl1, M, Y, ldy, s, sms, false, rs);
}

template <int MT>
svdq_status launch_awq(const uint8_t* q, const uint8_t* zeros, const uint16_t* scales,
                       const uint16_t* bias, int N, int K, int group, const uint16_t* X,
                       int64_t ldx, uint16_t* Y, int64_t ldy, cudaStream_t s, int sms) {
  const size_t smem = awq_smem_bytes(MT, K);
  if (cudaFuncSetAttribute(awq_gemv_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, awq_gemv_kernel<MT>, AWQ_THREADS,
                                                    smem) != cudaSuccess ||
      per_sm <= 0) {
    cudaGetLastError();
    per_sm = 1;
  }
  // S warps per 16-row block split K: the smallest split that gives every
  // resident warp slot a block (while each K slice keeps a group)
  const int rb_total = (N + 15) / 16, G = K / group;
  const long long slots = (long long)per_sm * sms * AWQ_WARPS;
  int S = 1;
  while (S < AWQ_WARPS && (long long)rb_total * S < slots && 2 * S <= G) S *= 2;
  const int R = AWQ_WARPS / S;
  const int rounds = (rb_total + R - 1) / R;
  const int blocks = std::max(1, std::min(rounds, per_sm * sms));
  awq_gemv_kernel<MT><<<blocks, AWQ_THREADS, smem, s>>>(q, zeros, scales, bias, N, K, group, S,
                                                        X, ldx, Y, ldy);
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

extern "C" svdq_status svdq_awq_linear(const uint8_t* q, const uint8_t* zeros,
                                       const uint16_t* scales, const uint16_t* bias, int N, int K,
                                       int group, const uint16_t* X, int M, int64_t ldx,
                                       uint16_t* Y, int64_t ldy, void* stream) {
  if (N <= 0 || K <= 0 || group <= 0 || group % 128 || K % group) return SVDQ_ERR_INVALID_ARG;
  if (M < 0 || M > AWQ_MAX_M || ldx < K || ldy < N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!q || !zeros || !scales || !X || !Y) return SVDQ_ERR_INVALID_ARG;
  if (awq_smem_bytes(M, K) > AWQ_SMEM_MAX) return SVDQ_ERR_INVALID_ARG;   // X staged in smem
  if (!aligned16(q) || !aligned16(X) || ldx % 8) return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  svdq_status st = device_check(&sms);
  if (st != SVDQ_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  switch (M) {
    case 1: return launch_awq<1>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    case 2: return launch_awq<2>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    case 3: return launch_awq<3>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    case 4: return launch_awq<4>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    case 5: return launch_awq<5>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    case 6: return launch_awq<6>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    case 7: return launch_awq<7>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
    default: return launch_awq<8>(q, zeros, scales, bias, N, K, group, X, ldx, Y, ldy, s, sms);
  }
}

extern "C" svdq_status svdq_linear_forward(const svdq_weight* w, const uint16_t* X, int M,
                                           int64_t ldx, uint16_t* Y, int64_t ldy,
                                           void* workspace, size_t ws_bytes, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx < w->K || ldy < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (ws_bytes < svdq_act_workspace_bytes(M, w->K, w->r)) return SVDQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return SVDQ_ERR_MISALIGNED;
  if (!aligned16(X) || !aligned16(Y) || ldx % 8 || ldy % 8) return SVDQ_ERR_MISALIGNED;
  int sms = 0;
  if ((st = device_check(&sms)) != SVDQ_OK) return st;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  uint8_t* codes_x = base;
  uint8_t* sf_x = codes_x + ws_codes(M, w->K);
  uint16_t* xl1 = w->r > 0 ? reinterpret_cast<uint16_t*>(sf_x + ws_sf(M, w->K)) : nullptr;
  cudaStream_t s = (cudaStream_t)stream;
  if ((st = launch_quantize(w, X, M, ldx, codes_x, sf_x, xl1, s, sms)) != SVDQ_OK) return st;
  // split-K for few output tiles when the workspace has room for it
  const size_t a = rup(svdq_act_workspace_bytes(M, w->K, w->r), 256);
  const size_t g = gemm_split_ws_bytes(M, w->N, w->K);
  void* split_ws = (g && ws_bytes >= a + g) ? static_cast<void*>(base + a) : nullptr;
  return launch_gemm(w, codes_x, sf_x, xl1, M, Y, ldy, s, sms, false, nullptr, split_ws);
}

extern "C" svdq_status svdq_linear_forward_host(const svdq_weight* w, const uint16_t* X_host,
                                                int M, int64_t ldx_host, uint16_t* Y_host,
                                                int64_t ldy_host, uint16_t* X_dev,
                                                uint16_t* Y_dev, void* workspace,
                                                size_t ws_bytes, void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx_host < w->K || ldy_host < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X_host || !Y_host || !X_dev || !Y_dev || !workspace) return SVDQ_ERR_INVALID_ARG;
  if (ws_bytes < svdq_act_workspace_bytes(M, w->K, w->r)) return SVDQ_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0) return SVDQ_ERR_MISALIGNED;
  if (!aligned16(X_dev) || !aligned16(Y_dev) || w->K % 8 || w->N % 8) return SVDQ_ERR_MISALIGNED;
  if ((st = device_check(nullptr)) != SVDQ_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t xrow = (size_t)w->K * 2, yrow = (size_t)w->N * 2;
  if (cudaMemcpy2DAsync(X_dev, xrow, X_host, (size_t)ldx_host * 2, xrow, (size_t)M,
                        cudaMemcpyHostToDevice, s) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  st = svdq_linear_forward(w, X_dev, M, w->K, Y_dev, w->N, workspace, ws_bytes, stream);
  if (st != SVDQ_OK) return st;
  if (cudaMemcpy2DAsync(Y_host, (size_t)ldy_host * 2, Y_dev, yrow, yrow, (size_t)M,
                        cudaMemcpyDeviceToHost, s) != cudaSuccess) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  return SVDQ_OK;
}

// Scratch of svdq_linear_forward_static: one per device, module-resident, so
// that the call itself never allocates.  Calls that overlap in time (two
// streams, two host threads) share it and race.
__device__ __align__(256) unsigned char g_static_ws[SVDQ_STATIC_WORKSPACE_BYTES];

namespace {
// Device address of g_static_ws on the current device.  Looked up on every
// call (cudaGetSymbolAddress reserves nothing and costs a table lookup), so
// no address outlives the module it belongs to, for instance across a
// device reset that reloads the library's device code.
svdq_status static_ws_address(void** out) {
  void* a = nullptr;
  if (cudaGetSymbolAddress(&a, g_static_ws) != cudaSuccess || !a) {
    cudaGetLastError();
    return SVDQ_ERR_CUDA;
  }
  *out = a;
  return SVDQ_OK;
}
}  // namespace

extern "C" svdq_status svdq_linear_forward_static(const svdq_weight* w, const uint16_t* X,
                                                  int M, int64_t ldx, uint16_t* Y, int64_t ldy,
                                                  void* stream) {
  svdq_status st = check_weight(w);
  if (st != SVDQ_OK) return st;
  if (M < 0 || ldx < w->K || ldy < w->N) return SVDQ_ERR_INVALID_ARG;
  if (M == 0) return SVDQ_OK;
  if (!X || !Y) return SVDQ_ERR_INVALID_ARG;
  const size_t need = svdq_act_workspace_bytes(M, w->K, w->r);
  if (need == 0 || need > SVDQ_STATIC_WORKSPACE_BYTES) return SVDQ_ERR_WORKSPACE;
  if (!aligned16(X) || !aligned16(Y) || ldx % 8 || ldy % 8) return SVDQ_ERR_MISALIGNED;
  if ((st = device_check(nullptr)) != SVDQ_OK) return st;
  void* ws = nullptr;
  if ((st = static_ws_address(&ws)) != SVDQ_OK) return st;
  return svdq_linear_forward(w, X, M, ldx, Y, ldy, ws, SVDQ_STATIC_WORKSPACE_BYTES, stream);
}

extern "C" svdq_status svdq_device_error(void* stream, int* code) {
  if (!code) return SVDQ_ERR_INVALID_ARG;
  *code = 0;
  svdq_status st = device_check(nullptr);
  if (st != SVDQ_OK) return st;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return SVDQ_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_svdq_error, sizeof(v)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_svdq_error, &zero, sizeof(zero)) != cudaSuccess)
    return SVDQ_ERR_CUDA;
  *code = (int)v;
  return v ? SVDQ_ERR_TIMEOUT : SVDQ_OK;
}

extern "C" svdq_status svdq_selftest_timeout(int timeout_us, void* stream) {
  if (timeout_us <= 0 || timeout_us > 10000000) return SVDQ_ERR_INVALID_ARG;
  svdq_status st = device_check(nullptr);
  if (st != SVDQ_OK) return st;
  selftest_timeout_kernel<<<1, 32, 0, (cudaStream_t)stream>>>((uint64_t)timeout_us * 1000ull);
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}

extern "C" svdq_status svdq_debug_convert(const float* in, uint8_t* e2m1_out, uint8_t* e4m3_out,
                                          int64_t n, void* stream) {
  if (n < 0 || (n > 0 && !in)) return SVDQ_ERR_INVALID_ARG;
  if (n == 0) return SVDQ_OK;
  svdq_status st = device_check(nullptr);
  if (st != SVDQ_OK) return st;
  const int64_t blocks = (n + 255) / 256;
  if (blocks > 0x7FFFFFFF) return SVDQ_ERR_INVALID_ARG;
  debug_convert_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(in, e2m1_out, e4m3_out, n);
  return cudaGetLastError() == cudaSuccess ? SVDQ_OK : SVDQ_ERR_CUDA;
}
