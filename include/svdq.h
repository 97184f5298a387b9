/*
 * svdq.h -- C ABI of the B200-native SVDQuant W4A4 (NVFP4) linear layer.
 *
 * What the layer computes ("Bringing Nunchaku 4-bit diffusion inference to
 * Diffusers", section "Background: SVDQuant and Nunchaku"; the Hacker News
 * thread on "SVDQuant: 4-Bit Quantization Powers 12B Flux on a 16GB 4090
 * GPU with 3x Speedup"): activation outliers are smoothed into the weight,
 * the smoothed weight W~ is split into a 16-bit rank-r branch L1 L2 plus a
 * residual R, and only R (and the activation) is held in 4 bits:
 *
 *     Y = Q(X_hat) Q(R)^T + (X_hat L1) L2 + bias,   Q = NVFP4.
 *
 * NVFP4 (the svdq_w4a4 precision on Blackwell, hardware-support table of
 * the same article): E2M1 values, one E4M3 scale per 16 consecutive
 * elements along K, one fp32 tensor scale.
 *
 * Kernel fusion follows the Korean rendering of the article (section
 * "SVDQuant and the Nunchaku engine"): the low-rank down-projection runs
 * inside the activation-quantization kernel and the up-projection inside
 * the 4-bit GEMM kernel, so the 16-bit branch adds no separate pass over
 * memory.
 *
 * Conventions for every call:
 *   - All pointers are caller-owned.  The library never allocates, frees or
 *     retains device or host memory and never synchronizes a stream (except
 *     svdq_device_error, whose job is to read the kernels' error word).
 *   - "device" pointers must be global memory of the current CUDA device;
 *     "host" pointers are ordinary host memory.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Matrices are row-major; ld* is the row stride in elements.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  GPU calls
 *     are asynchronous; errors found on the host are returned before any
 *     launch; a device-side fault surfaces on the caller's next synchronize.
 *   - Inputs must be finite; NaN/Inf activations give unspecified codes.
 *   - The GPU entry points require an sm_100 device (B200); any other device
 *     gives SVDQ_ERR_UNSUPPORTED_ARCH and launches nothing (the article's
 *     rule: validate GPU capability and refuse rather than compute wrongly).
 */
#ifndef SVDQ_H
#define SVDQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum svdq_status {
  SVDQ_OK = 0,
  SVDQ_ERR_INVALID_ARG = 1,      /* null pointer, bad shape or rank        */
  SVDQ_ERR_UNSUPPORTED_ARCH = 2, /* no CUDA device, or not sm_100          */
  SVDQ_ERR_MISALIGNED = 3,       /* pointer / leading dimension alignment  */
  SVDQ_ERR_WORKSPACE = 4,        /* workspace smaller than required        */
  SVDQ_ERR_CUDA = 5,             /* a CUDA runtime call or launch failed   */
  SVDQ_ERR_TIMEOUT = 6,          /* a kernel gave up waiting (see below)   */
  SVDQ_ERR_NUMERIC = 7           /* pack: non-finite weight or statistics  */
} svdq_status;

/* Human-readable name of a status code (static string, never NULL). */
const char* svdq_status_string(svdq_status s);

/* Library version, e.g. "svdq-b200 0.1". */
const char* svdq_version(void);

/* ---------------------------------------------------------------- sizes --
 * Buffer sizes (bytes) for an N x K weight with rank r.
 *   r must be 0 or a multiple of 16 in [16, 128]; K a multiple of 64;
 *   N a multiple of 16.
 *   klr = round_up(2 r, 64): the padded K extent of the low-rank operands.
 */
typedef struct svdq_sizes {
  int N, K, r, klr;
  size_t smooth_bytes;   /* fp32 [K]                                       */
  size_t l1_bytes;       /* bf16 [K][r]       plain factor L1              */
  size_t l2_bytes;       /* bf16 [r][N]       plain factor L2              */
  size_t l1_mma_bytes;   /* bf16 [2r][K]      kernel operand, see pack     */
  size_t l2_mma_bytes;   /* bf16 [N][klr]     kernel operand, see pack     */
  size_t codes_w_bytes;  /* u8   [N][K/2]     E2M1 codes of R              */
  size_t sf_w_bytes;     /* u8   MMA tiles    E4M3 scales of R (rows padded to 256) */
  size_t bias_bytes;     /* bf16 [N]                                       */
} svdq_sizes;

svdq_status svdq_query_sizes(int N, int K, int r, svdq_sizes* out);

/* ------------------------------------------------------------------ pack --
 * svdq_pack_weight: the offline quantization of one linear (host only,
 * synchronous, re-entrant; OpenMP threads).
 * Source: "Bringing Nunchaku 4-bit diffusion inference to Diffusers",
 * section "Background: SVDQuant and Nunchaku" (and its Korean rendering,
 * "SVDQuant and the Nunchaku engine"): outliers are moved from the
 * activations into the weight, the hardest part of each weight becomes a
 * small 16-bit low-rank branch, the residual is quantized to 4 bit.  The
 * formula of each step is a reading of that prose (the page prints none).
 * Steps, in that order:
 *   1. smoothing: lambda_j = (x_absmax_j / max_n |W_nj|)^alpha (lambda = 1
 *      where either maximum is 0); stored as smooth_j = fp32(1/lambda_j), the
 *      activation multiplier (x_hat = fp32(x * smooth_j)); W~ = W / smooth
 *      in float64.
 *   2. low-rank branch: top-r SVD of W~ (randomized subspace iteration with
 *      Rayleigh-Ritz, seeded): L1 = V sqrt(S) [K x r], L2 = sqrt(S) U^T
 *      [r x N], each rounded once to bf16.
 *   3. residual R = fp32(W~ - (L1 L2)^T) (float64 sum over rank ascending).
 *   4. NVFP4 of R with A_w = max|R|: g_w = 2688/A_w, gs_w = 448/A_w; per
 *      16 along K: sf = E4M3(a * gs_w), code = E2M1(R * fp32(g_w / sf)).
 *   5. activation tensor scale from calibration:
 *      A_x = max_j fp32(x_absmax_j * smooth_j); g_x = 2688/A_x,
 *      gs_x = 448/A_x (g = gs = 1 when A = 0).
 *   6. lr_scale = fp32(g_x * g_w), alpha = fp32(1 / lr_scale).
 *   7. kernel operands: l1_mma[i][k] = bf16 hi part and l1_mma[r+i][k] =
 *      bf16 lo part of smooth_k * L1[k][i] (exact product in float64, hi =
 *      bf16(p), lo = bf16(p - hi)); l2_mma[n][i] = l2_mma[n][r+i] = L2[i][n],
 *      zero beyond 2r.
 *   8. bias: carried through unchanged as bf16 (it enters only the GEMM
 *      epilogue, Y = bf16(alpha * acc + bias), and takes no part in the
 *      smoothing, the SVD or the quantization).
 * Arguments:
 *   W         host fp32 [N][K] (out x in, the PyTorch Linear layout)
 *   x_absmax  host fp32 [K], per-input-channel max |x| of calibration data
 *   bias_bf16 host bf16 [N] or NULL (no bias)
 *   smooth_alpha  smoothing exponent (0.5 in the workloads here)
 *   seed      seed of the SVD's random start (the result is deterministic
 *             for a given seed and build)
 *   out       host buffers sized by svdq_query_sizes; every pointer field
 *             except bias must be non-NULL (l1, l2, l1_mma, l2_mma may be
 *             NULL when r == 0); the scalars are written.  out->bias, when
 *             non-NULL, receives bias_bf16 (zeros when bias_bf16 is NULL).
 * Errors: INVALID_ARG for shapes/NULLs (also bias_bf16 given with
 * out->bias NULL), NUMERIC for non-finite input.
 */
typedef struct svdq_packed_host {
  float*    smooth;      /* [K]        */
  uint16_t* l1;          /* [K][r]     */
  uint16_t* l2;          /* [r][N]     */
  uint16_t* l1_mma;      /* [2r][K]    */
  uint16_t* l2_mma;      /* [N][klr]   */
  uint8_t*  codes_w;     /* [N][K/2], even k in the low nibble             */
  uint8_t*  sf_w;        /* MMA tile layout (svdq_sf_tile_offset)          */
  uint16_t* bias;        /* [N] bf16, or NULL                              */
  float amax_x, amax_w;  /* static activation absmax A_x, residual absmax A_w */
  float g_x, gs_x, g_w, alpha, lr_scale;
} svdq_packed_host;

svdq_status svdq_pack_weight(const float* W, const float* x_absmax,
                             const uint16_t* bias_bf16, int N, int K, int r,
                             float smooth_alpha, uint64_t seed,
                             svdq_packed_host* out);

/* ---------------------------------------------------------------- layout --
 * Byte offset of the E4M3 scale of (row, group g = k/16) in the MMA tile
 * layout used for sf_w and sf_x: atoms of 128 rows x 4 scales (512 bytes),
 * atom (row/128, g/4) at ((row/128) * (K/64) + g/4) * 512, and inside the
 * atom byte (row%32)*16 + ((row%128)/32)*4 + g%4.  Returns -1 on bad args.
 * This is the scale arrangement the block-scaled tensor-core MMA reads; the
 * pages fix only "one E4M3 scale per 16 elements" (NVFP4, hardware-support
 * table of "Bringing Nunchaku 4-bit diffusion inference to Diffusers").
 */
int64_t svdq_sf_tile_offset(int row, int g, int K);

/* svdq_unswizzle_scales: host permutation from the MMA tile layout back to
 * plain row-major scales, sf_rowmajor[row][g] = sf_mma[svdq_sf_tile_offset(
 * row, g, K)] for row < rows, g < K/16.  Used to compare device scales with
 * a row-major reference.  Host pointers; sf_mma holds at least
 * round_up(rows, 128) * K/16 bytes, sf_rowmajor rows * K/16 bytes.
 * Errors: INVALID_ARG for NULLs, rows < 0, K not a multiple of 64. */
svdq_status svdq_unswizzle_scales(const uint8_t* sf_mma, int rows, int K,
                                  uint8_t* sf_rowmajor);

/* -------------------------------------------------------------- forward --
 * Device-side weight: a plain struct of device pointers (filled by the
 * caller after copying the packed host buffers to the GPU).
 */
typedef struct svdq_weight {
  int N, K, r;
  float g_x, gs_x, g_w, alpha, lr_scale;
  const float*    smooth;   /* device fp32 [K], 16-byte aligned            */
  const uint16_t* l1_mma;   /* device bf16 [2r][K]        (NULL if r == 0) */
  const uint16_t* l2_mma;   /* device bf16 [N][klr]       (NULL if r == 0) */
  const uint16_t* bias;     /* device bf16 [N] or NULL                     */
  const uint8_t*  codes_w;  /* device u8 [N][K/2]                          */
  const uint8_t*  sf_w;     /* device u8, MMA tiles, rows padded to 256    */
} svdq_weight;

/* Bytes of the activation workspace for M tokens: codes_x [M][K/2],
 * sf_x (MMA tiles, rows padded to 128) and xl1 [M][klr] bf16, each region
 * 256-byte aligned.  0 on bad arguments. */
size_t svdq_act_workspace_bytes(int M, int K, int r);

/* svdq_quantize_act: activation kernel (one launch).
 * Source: the Korean rendering of "Bringing Nunchaku 4-bit diffusion
 * inference to Diffusers", section "SVDQuant and the Nunchaku engine": the
 * low-rank down projection is fused with the quantization kernel, which
 * removes the 16-bit branch's extra memory traffic; NVFP4 per the
 * hardware-support table of the same article.  For every row of X:
 * x_hat = fp32(x * smooth); NVFP4 with the static tensor scales g_x, gs_x
 * (per 16-group max, sf = E4M3(a * gs_x), codes = E2M1(x_hat * g_x / sf),
 * two per byte); and, fused, the
 * down-projection X_hat L1 on the tensor cores, written pre-multiplied by
 * lr_scale as a bf16 hi/lo pair: xl1[m][i] + xl1[m][r+i] ~= lr_scale *
 * (X_hat L1)[m][i], zeros in columns [2r, klr).
 *   X        device bf16 [M][ldx], 16-byte aligned, ldx % 8 == 0, ldx >= K
 *   codes_x  device u8 [M][K/2]
 *   sf_x     device u8, MMA tiles, round_up(M,128) * K/16 bytes (pad rows 0)
 *   xl1      device bf16 [M][klr] (may be NULL if r == 0)
 * Reads X exactly once.  Two kernel forms by batch size: 128-row tiles over
 * all of K when there are enough rows to give most SMs a tile of their own
 * (about 15k rows and up), else 64-row tiles with K split within a cluster.
 * Returns SVDQ_ERR_INVALID_ARG when one CTA's share of K does not fit its
 * shared-memory plan (for large M: K above roughly 36000 at r <= 32, 24000
 * at r = 128).
 */
svdq_status svdq_quantize_act(const svdq_weight* w, const uint16_t* X, int M,
                              int64_t ldx, uint8_t* codes_x, uint8_t* sf_x,
                              uint16_t* xl1, void* stream);

/* svdq_gemm: the 4-bit GEMM kernel (one launch).
 * Source: the Korean rendering of "Bringing Nunchaku 4-bit diffusion
 * inference to Diffusers", section "SVDQuant and the Nunchaku engine": the
 * low-rank up projection is fused with the 4-bit compute kernel; W4A4 (both
 * operands 4-bit) per "Background: SVDQuant and Nunchaku".  Block-scaled FP4 x FP4
 * tensor-core MMA into an fp32 accumulator in tensor memory, the low-rank
 * up-projection xl1 * L2 accumulated into the same accumulator, epilogue
 * Y = bf16(alpha * acc + bias).
 *   Y  device bf16 [M][ldy], 16-byte aligned, ldy % 8 == 0, ldy >= N
 */
svdq_status svdq_gemm(const svdq_weight* w, const uint8_t* codes_x,
                      const uint8_t* sf_x, const uint16_t* xl1, int M,
                      uint16_t* Y, int64_t ldy, void* stream);

/* Bytes of the workspace of svdq_gemm_splitk for an M x N x K layer (the
 * partials: tiles x parts x 256 x 256 fp32); 0 when the GEMM does not split
 * (32 or more 256 x 256 output tiles, or a single 256-deep K stage). */
size_t svdq_gemm_workspace_bytes(int M, int N, int K);

/* svdq_gemm_splitk: svdq_gemm for layers with few output tiles (small M,
 * where whole-K tiles would leave most SMs idle; the pages' small-batch
 * latency concern, Vietnamese rendering, "End-to-end latency and memory").
 * Each tile's K stages are split into up to 8 parts ("units") run by
 * different CTA pairs (about 64 units in all); every unit stores its fp32
 * partial accumulator in the workspace, and a second kernel (chained by
 * programmatic dependent launch, the whole GPU wide) adds the partials in
 * part order -- Y is deterministic -- and applies alpha, bias and the bf16
 * store.  The low-rank branch is accumulated by the last K part.  Same
 * result as svdq_gemm up to the fp32 summation order.  Two launches.
 *   workspace  device, 256-byte aligned, >= svdq_gemm_workspace_bytes(M, N, K)
 *              (may be NULL when that is 0); contents need not be preserved
 * Errors as svdq_gemm, plus SVDQ_ERR_WORKSPACE. */
svdq_status svdq_gemm_splitk(const svdq_weight* w, const uint8_t* codes_x,
                             const uint8_t* sf_x, const uint16_t* xl1, int M,
                             uint16_t* Y, int64_t ldy, void* workspace, size_t ws_bytes,
                             void* stream);

/* Bytes of a svdq_linear_forward workspace that also holds the split-K
 * partials (svdq_act_workspace_bytes rounded up to 256, plus
 * svdq_gemm_workspace_bytes); equal to svdq_act_workspace_bytes when the
 * GEMM does not split.  0 on bad arguments. */
size_t svdq_forward_workspace_bytes(const svdq_weight* w, int M);

/* svdq_gemm_gelu: svdq_gemm for the first linear of an MLP pair, with the
 * pair's GELU fused into the epilogue.  Source: the fused GELU/MLP kernels
 * the pages name as part of the original engine's speed ("Bringing Nunchaku
 * 4-bit diffusion inference to Diffusers", Vietnamese rendering, section
 * "Introducing Nunchaku Lite").  Writes H = bf16(GELU(bf16(alpha * acc +
 * bias))) instead of Y: the tanh form of GELU, evaluated as y / (1 +
 * 2^(-2 log2(e) u)), u = sqrt(2/pi) (y + 0.044715 y^3), with the hardware's
 * approximate base-2 exponential and reciprocal (a few 1e-7 relative before
 * the bf16 rounding; within one bf16 unit of the correctly rounded GELU, see
 * svdq_debug_gelu).  Arguments and errors as svdq_gemm (H in place of Y). */
svdq_status svdq_gemm_gelu(const svdq_weight* w, const uint8_t* codes_x,
                           const uint8_t* sf_x, const uint16_t* xl1, int M,
                           uint16_t* H, int64_t ldh, void* stream);

/* Bytes of the workspace of svdq_mlp_forward (the larger of the two
 * layers' forward workspaces).  0 on bad arguments. */
size_t svdq_mlp_workspace_bytes(int M, int K1, int N1, int r1, int r2);

/* svdq_mlp_forward: a Flux MLP pair, fc1 -> GELU -> fc2, in four launches on
 * one stream: the activation kernel of fc1, the GEMM of fc1 with the GELU
 * epilogue (svdq_gemm_gelu), the activation kernel of fc2 on H, the GEMM of
 * fc2.  w2->K must equal w1->N.
 *   X  device bf16 [M][ldx]   (fc1 input)
 *   H  device bf16 [M][ldh]   (GELU(fc1 output), caller-owned, also fc2's input)
 *   Y  device bf16 [M][ldy]   (fc2 output)
 *   workspace  >= svdq_mlp_workspace_bytes, 256-byte aligned.
 * Errors as svdq_linear_forward. */
svdq_status svdq_mlp_forward(const svdq_weight* w1, const svdq_weight* w2,
                             const uint16_t* X, int M, int64_t ldx, uint16_t* H,
                             int64_t ldh, uint16_t* Y, int64_t ldy, void* workspace,
                             size_t ws_bytes, void* stream);

/* svdq_linear_forward: the whole layer, Y = Q(X_hat) Q(R)^T + (X_hat L1) L2
 * + bias ("Background: SVDQuant and Nunchaku"; the runtime SVDQW4A4Linear
 * layer that replaces nn.Linear in "Loading natively in Diffusers"):
 * svdq_quantize_act then svdq_gemm on one stream, with the intermediates in
 * `workspace` (device, >= svdq_act_workspace_bytes, 256-byte aligned).  With
 * a workspace of svdq_forward_workspace_bytes(w, M) the GEMM runs split-K
 * (svdq_gemm_splitk) when the layer has few output tiles. */
svdq_status svdq_linear_forward(const svdq_weight* w, const uint16_t* X,
                                int M, int64_t ldx, uint16_t* Y, int64_t ldy,
                                void* workspace, size_t ws_bytes,
                                void* stream);

/* ------------------------------------------------ dynamic (per-token) --
 * The dynamic alternative to the static activation tensor scale, for inputs
 * outside the calibration range.  The pages fix only the static form (one
 * fp32 tensor scale, NVFP4 of the hardware-support table of "Bringing
 * Nunchaku 4-bit diffusion inference to Diffusers"); here each row (token)
 * of X_hat is its own tensor for the same recipe:
 *   A_m = max_k |fp32(x_mk smooth_k)|, g_m = fp32(2688 / A_m),
 *   gs_m = fp32(448 / A_m) (both 1 when A_m = 0), lr_m = fp32(g_m g_w),
 *   alpha_m = fp32(1 / lr_m);
 * row m is quantized with g_m, gs_m (q = fp32(g_m / e4m3(sf)) per group),
 * its low-rank operand is pre-scaled by lr_m, and the GEMM scales its
 * output row by alpha_m.  Row scales: 16 bytes per row, {g, gs, lr, alpha}
 * as fp32, device memory, 16-byte aligned.
 */
/* One pass over X: the row scales of every row (memory-bound). */
svdq_status svdq_act_row_scales(const svdq_weight* w, const uint16_t* X, int M, int64_t ldx,
                                void* row_scales, void* stream);
/* svdq_quantize_act with each row's own scales (from svdq_act_row_scales). */
svdq_status svdq_quantize_act_dynamic(const svdq_weight* w, const uint16_t* X, int M,
                                      int64_t ldx, const void* row_scales, uint8_t* codes_x,
                                      uint8_t* sf_x, uint16_t* xl1, void* stream);
/* svdq_gemm with each output row scaled by its alpha_m. */
svdq_status svdq_gemm_dynamic(const svdq_weight* w, const uint8_t* codes_x,
                              const uint8_t* sf_x, const uint16_t* xl1,
                              const void* row_scales, int M, uint16_t* Y, int64_t ldy,
                              void* stream);
/* Workspace of svdq_linear_forward_dynamic: the static forward's plus 16
 * bytes per row (rounded to 256).  0 on bad arguments. */
size_t svdq_dyn_workspace_bytes(int M, int K, int r);
/* The layer with per-token scales: row scales, activation kernel, GEMM on
 * one stream.  Arguments and errors as svdq_linear_forward (workspace >=
 * svdq_dyn_workspace_bytes). */
svdq_status svdq_linear_forward_dynamic(const svdq_weight* w, const uint16_t* X, int M,
                                        int64_t ldx, uint16_t* Y, int64_t ldy,
                                        void* workspace, size_t ws_bytes, void* stream);

/* svdq_linear_forward_host: svdq_linear_forward for activations and outputs
 * that live in host memory (the drop-in layer's view of a host batch):
 * copies X_host to X_dev, runs the layer, copies Y_dev back to Y_host, all
 * enqueued on `stream` in that order (one cudaMemcpy2DAsync per copy; no
 * synchronization; the host buffers must stay valid until the stream
 * reaches the end of the call, and should be pinned for the copies to be
 * asynchronous).
 *   X_host  host bf16 [M][ldx_host], ldx_host >= K
 *   Y_host  host bf16 [M][ldy_host], ldy_host >= N
 *   X_dev   device bf16 [M][K] (contiguous, 16-byte aligned)
 *   Y_dev   device bf16 [M][N] (contiguous, 16-byte aligned)
 *   workspace, ws_bytes, stream: as svdq_linear_forward.
 * Errors: those of svdq_linear_forward; SVDQ_ERR_CUDA if a copy cannot be
 * enqueued (nothing after it is enqueued). */
svdq_status svdq_linear_forward_host(const svdq_weight* w, const uint16_t* X_host,
                                     int M, int64_t ldx_host, uint16_t* Y_host,
                                     int64_t ldy_host, uint16_t* X_dev,
                                     uint16_t* Y_dev, void* workspace,
                                     size_t ws_bytes, void* stream);

/* svdq_linear_forward_static: the same forward as svdq_linear_forward, with
 * the intermediates in a fixed scratch area that the library holds in device
 * memory (SVDQ_STATIC_WORKSPACE_BYTES per device, reserved when the library's
 * module loads).  The paper has no counterpart: it is a convenience for
 * callers that cannot allocate device memory while a forward runs, such as a
 * plain C host with no device allocator of its own, or a runtime that plans
 * all memory ahead and forbids allocation inside its step.
 *   - Never allocates or frees device memory and calls no allocating library
 *     routine.  Each call looks the scratch address up on the current device
 *     (cudaGetSymbolAddress, which reserves nothing); make the first call on
 *     a device before any stream capture, since that lookup may load the
 *     library's device code on the device.
 *   - M is limited by the scratch size: svdq_act_workspace_bytes(M, K, r)
 *     must be <= SVDQ_STATIC_WORKSPACE_BYTES, else SVDQ_ERR_WORKSPACE and
 *     nothing is launched (e.g. K = 3072, r = 32 allows M <= 9033).
 *   - Nothing in the scratch needs to start at zero: the activation kernel
 *     writes every byte the GEMM reads, padding rows included.
 *   - One scratch area per device: calls that overlap in time (different
 *     streams, or threads without ordering) race on it.  Calls in order on
 *     one stream are safe.
 * Arguments, layouts and the other errors are those of svdq_linear_forward. */
#define SVDQ_STATIC_WORKSPACE_BYTES ((size_t)16 << 20)
svdq_status svdq_linear_forward_static(const svdq_weight* w, const uint16_t* X,
                                       int M, int64_t ldx, uint16_t* Y,
                                       int64_t ldy, void* stream);

/* ------------------------------------------------------ AWQ W4A16 linear --
 * The second kernel family of the pages: 4-bit weights with 16-bit
 * activations, for the memory-bound, precision-sensitive modulation and
 * adaptive-normalization projections ("Bringing Nunchaku 4-bit diffusion
 * inference to Diffusers", Russian rendering, section "Technical details and
 * hardware support"; the Korean rendering's kernel-family list).  The pages
 * fix only "INT4 weights, 16-bit activations"; the format is AWQ's
 * asymmetric INT4 per group of `group` input channels:
 *   range [wmin, wmax] of the group widened to include 0,
 *   scale = fp16(max(wmax - wmin, 1e-5) / 15), z = clamp(rint(-wmin/scale), 0, 15),
 *   q = clamp(rint(w / scale) + z, 0, 15) (rint: ties to even, in double),
 *   dequantized weight (q - z) * scale.
 * (AWQ's activation-aware per-channel scale search is an offline step and
 * is not part of these calls.)
 *
 * svdq_awq_pack (host, synchronous): W fp32 [N][K] -> q_packed u8 [N][K/2]
 * (even k in the low nibble), zeros u8 [N][K/group], scales fp16 bit
 * patterns [N][K/group].  group a multiple of 32 dividing K (128 is AWQ's
 * usual group).  Errors: INVALID_ARG, NUMERIC (non-finite W). */
svdq_status svdq_awq_pack(const float* W, int N, int K, int group, uint8_t* q_packed,
                          uint8_t* zeros, uint16_t* scales);

/* svdq_awq_tile_codes (host, synchronous): the codes in the layout the
 * GPU layer reads (a permutation only: the layer is the awq_w4a16 family of
 * "Bringing Nunchaku 4-bit diffusion inference to Diffusers", Russian
 * rendering, "Technical details and hardware support").  q_rowmajor as svdq_awq_pack writes it ([N][K/2], even k
 * in the low nibble); q_tiled: ceil(N/16) * 16 * K / 2 bytes.  Per 16-row
 * block rb and 64-deep block of K, 512 bytes = 32 lanes x 16 bytes; lane
 * l = 4 g + c holds one 32-bit word per 16-deep k-step ks (4 per block, at
 * byte ((rb * K/64 + ks/4) * 32 + l) * 16 + (ks % 4) * 4), and nibble j of
 * that word is the code of row 16 rb + g + 8 (j % 2), column
 * 16 ks + 2 c + 8 ((j % 4) / 2) + j / 4 (the elements a warp's tensor-core
 * fragment takes from lane l); rows past N hold code 0.  K % 64 == 0.
 * Errors: INVALID_ARG. */
svdq_status svdq_awq_tile_codes(const uint8_t* q_rowmajor, int N, int K, uint8_t* q_tiled);

/* svdq_awq_linear (GPU): Y = X dequant(W)^T + bias, one bf16 rounding.  Per
 * group the sum of (q - z) x is accumulated in fp32 (products exact), then
 * scaled by the group's fp16 scale and added in fp32.  For the batch sizes
 * of modulation layers: 1 <= M <= 8 (a memory-bound product over the weight
 * stream), group a multiple of 128 dividing K, and 8 KB + M * K * 2 bytes
 * <= 216 KB (X is staged in shared memory).
 *   q      device, tiled as svdq_awq_tile_codes writes it (16-byte aligned)
 *   zeros, scales  device, as svdq_awq_pack writes them ([N][K/group])
 *   bias   device bf16 [N] or NULL
 *   X      device bf16 [M][ldx], 16-byte aligned, ldx >= K, ldx % 8 == 0
 *   Y      device bf16 [M][ldy], ldy >= N
 * Errors: INVALID_ARG (shapes, M > 8, NULLs), MISALIGNED, UNSUPPORTED_ARCH. */
svdq_status svdq_awq_linear(const uint8_t* q, const uint8_t* zeros, const uint16_t* scales,
                            const uint16_t* bias, int N, int K, int group, const uint16_t* X,
                            int M, int64_t ldx, uint16_t* Y, int64_t ldy, void* stream);

/* ------------------------------------------------------------- failure --
 * Every wait inside the kernels is bounded (about one second).  A kernel
 * that gives up records a code in a device-side word and exits cleanly
 * (outstanding copies drained, tensor memory released); the CUDA context
 * stays usable.  svdq_device_error synchronizes `stream`, returns the
 * recorded code in *code (0 = none) and clears it.  Returns SVDQ_ERR_TIMEOUT
 * when a code was set, SVDQ_OK otherwise.
 */
svdq_status svdq_device_error(void* stream, int* code);

/* Test hook: launches a one-CTA kernel whose mbarrier wait can never be
 * satisfied, with the wait limit set to `timeout_us`; it must end with the
 * device error code set (exercises the bounded-wait path without a hang). */
svdq_status svdq_selftest_timeout(int timeout_us, void* stream);

/* Diagnostic: device float32 -> E2M1 (n codes, one per byte) and float32 ->
 * E4M3 (one per byte, inputs >= 0) with the same hardware conversions the
 * activation kernel uses.  in/out device pointers, n >= 0. */
svdq_status svdq_debug_convert(const float* in, uint8_t* e2m1_out,
                               uint8_t* e4m3_out, int64_t n, void* stream);

/* Diagnostic: the epilogue GELU of svdq_gemm_gelu on n bf16 values
 * (device in/out, bf16 bit patterns). */
svdq_status svdq_debug_gelu(const uint16_t* in, uint16_t* out, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* SVDQ_H */
