// Host-side offline pack of one SVDQuant W4A4 linear (NVFP4).
//
// Steps follow "Bringing Nunchaku 4-bit diffusion inference to Diffusers",
// section "Background: SVDQuant and Nunchaku": smooth activation outliers
// into the weight, keep a 16-bit rank-r branch from the SVD of the smoothed
// weight, quantize the residual to 4 bit (NVFP4 per the hardware-support
// table).  The points the article leaves open are fixed as documented in
// include/svdq.h (smoothing exponent, the sqrt(S) split, the NVFP4 scale
// recipe, the residual's summation order).
//
// Everything here is plain C++ on the host (OpenMP over rows/columns).  The
// SVD is a randomized subspace iteration with Rayleigh-Ritz: a few products
// with the N x K matrix instead of a dense decomposition.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "../../include/svdq.h"

namespace svdq_host {

// ------------------------------------------------------------ formats ----

// float64 -> bf16 bits with one round-to-nearest-even step taken directly on
// the float64 mantissa (no intermediate float rounding).  Magnitudes below
// 2^-126 become a signed zero.
uint16_t bf16_from_double(double x) {
  uint64_t b;
  std::memcpy(&b, &x, 8);
  const uint64_t sign = b >> 63;
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
  uint64_t keep = mag >> 45;
  const uint64_t rem = mag & ((1ull << 45) - 1);
  const uint64_t half = 1ull << 44;
  if (rem > half || (rem == half && (keep & 1))) keep += 1;
  const uint64_t rb = keep << 45;
  double r;
  std::memcpy(&r, &rb, 8);
  float f = (std::fabs(r) < std::ldexp(1.0, -126)) ? 0.0f : (float)r;  // exact
  uint32_t fb;
  std::memcpy(&fb, &f, 4);
  return (uint16_t)((fb >> 16) | (sign << 15));
}

double bf16_to_double(uint16_t h) {
  uint32_t fb = (uint32_t)h << 16;
  float f;
  std::memcpy(&f, &fb, 4);
  return (double)f;
}

// E2M1 magnitude code of |v| by the midpoints of the grid
// {0, .5, 1, 1.5, 2, 3, 4, 6}; a midpoint goes to the even code.
static inline uint8_t e2m1_code(float v) {
  const float m = std::fabs(v);
  uint8_t c;
  if (m <= 0.25f) c = 0;
  else if (m < 0.75f) c = 1;
  else if (m <= 1.25f) c = 2;
  else if (m < 1.75f) c = 3;
  else if (m <= 2.5f) c = 4;
  else if (m < 3.5f) c = 5;
  else if (m <= 5.0f) c = 6;
  else c = 7;
  return (uint8_t)(c | (std::signbit(v) ? 8 : 0));
}

// Non-negative float -> E4M3 (fn) code, nearest-even, saturating at 448.
static inline uint8_t e4m3_code(float y) {
  if (!(y > 0.0f)) return 0;
  if (y >= 448.0f) return 0x7E;
  const double d = (double)y;
  if (d < std::ldexp(1.0, -6)) {                 // subnormal range, step 2^-9
    const double n = std::nearbyint(d * 512.0);  // ties to even
    return (uint8_t)n;                           // n == 8 is the first normal
  }
  int e;
  const double fr = std::frexp(d, &e);           // d = fr * 2^e, fr in [.5,1)
  int ex = e - 1;                                // d = (2 fr) 2^ex
  double n = std::nearbyint((2.0 * fr - 1.0) * 8.0);
  if (n == 8.0) { n = 0.0; ex += 1; }
  const int code = ((ex + 7) << 3) | (int)n;
  return (uint8_t)std::min(code, 0x7E);
}

static inline float e4m3_value(uint8_t c) {
  const int e = c >> 3, m = c & 7;
  if (e == 0) return (float)std::ldexp((double)m, -9);
  return (float)std::ldexp(1.0 + m / 8.0, e - 7);
}

static inline float tensor_scale(float amax) {
  return amax > 0.0f ? 2688.0f / amax : 1.0f;
}
static inline float block_scale_factor(float amax) {
  return amax > 0.0f ? 448.0f / amax : 1.0f;
}

// --------------------------------------------------------------- rng ----

struct SplitMix {
  uint64_t s;
  uint64_t next() {
    uint64_t z = (s += 0x9E3779B97F4A7C15ull);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }
  double uniform() { return ((next() >> 11) + 0.5) * (1.0 / 9007199254740992.0); }
  double normal() {
    const double u = uniform(), v = uniform();
    return std::sqrt(-2.0 * std::log(u)) * std::cos(6.283185307179586 * v);
  }
};

// -------------------------------------------------- dense helpers ----
// A is N x K row-major (float64).  Tall matrices are row-major n x l.

static void mul_A_B(const double* A, int N, int K, const double* B, int l, double* C) {
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    double* c = C + (size_t)n * l;
    for (int j = 0; j < l; ++j) c[j] = 0.0;
    const double* a = A + (size_t)n * K;
    for (int k = 0; k < K; ++k) {
      const double av = a[k];
      const double* b = B + (size_t)k * l;
      for (int j = 0; j < l; ++j) c[j] += av * b[j];
    }
  }
}

static void mul_At_B(const double* A, int N, int K, const double* Q, int l, double* Z) {
  const int KB = 64;
#pragma omp parallel for schedule(static)
  for (int kb = 0; kb < K; kb += KB) {
    const int ke = std::min(K, kb + KB);
    for (int k = kb; k < ke; ++k)
      for (int j = 0; j < l; ++j) Z[(size_t)k * l + j] = 0.0;
    for (int n = 0; n < N; ++n) {
      const double* a = A + (size_t)n * K;
      const double* q = Q + (size_t)n * l;
      for (int k = kb; k < ke; ++k) {
        const double av = a[k];
        double* z = Z + (size_t)k * l;
        for (int j = 0; j < l; ++j) z[j] += av * q[j];
      }
    }
  }
}

// Orthonormalize the l columns of the n x l row-major matrix Y in place
// (Gram-Schmidt, two passes).  Columns that vanish become zero.
static void orthonormalize(double* Y, int n, int l) {
  std::vector<double> col((size_t)l * n);
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < l; ++j) col[(size_t)j * n + i] = Y[(size_t)i * l + j];
  for (int j = 0; j < l; ++j) {
    double* v = &col[(size_t)j * n];
    double orig = 0.0;
    for (int i = 0; i < n; ++i) orig += v[i] * v[i];
    orig = std::sqrt(orig);
    for (int pass = 0; pass < 2; ++pass) {
      for (int p = 0; p < j; ++p) {
        const double* q = &col[(size_t)p * n];
        double d = 0.0;
        for (int i = 0; i < n; ++i) d += q[i] * v[i];
        for (int i = 0; i < n; ++i) v[i] -= d * q[i];
      }
    }
    double nrm = 0.0;
    for (int i = 0; i < n; ++i) nrm += v[i] * v[i];
    nrm = std::sqrt(nrm);
    if (nrm <= 1e-13 * orig || nrm == 0.0) {
      for (int i = 0; i < n; ++i) v[i] = 0.0;
    } else {
      for (int i = 0; i < n; ++i) v[i] /= nrm;
    }
  }
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < l; ++j) Y[(size_t)i * l + j] = col[(size_t)j * n + i];
}

// Cyclic Jacobi eigen-decomposition of the symmetric l x l matrix C.
// On return C holds the eigenvalues on its diagonal and V (row-major) the
// eigenvectors as columns.
static void jacobi_eigen(std::vector<double>& C, int l, std::vector<double>& V) {
  V.assign((size_t)l * l, 0.0);
  for (int i = 0; i < l; ++i) V[(size_t)i * l + i] = 1.0;
  double diag = 0.0;
  for (int i = 0; i < l; ++i) diag += C[(size_t)i * l + i] * C[(size_t)i * l + i];
  for (int sweep = 0; sweep < 60; ++sweep) {
    double off = 0.0;
    for (int p = 0; p < l; ++p)
      for (int q = p + 1; q < l; ++q) off += C[(size_t)p * l + q] * C[(size_t)p * l + q];
    if (off <= 1e-30 * diag || off == 0.0) break;
    for (int p = 0; p < l; ++p) {
      for (int q = p + 1; q < l; ++q) {
        const double apq = C[(size_t)p * l + q];
        if (std::fabs(apq) < 1e-300) continue;
        const double app = C[(size_t)p * l + p], aqq = C[(size_t)q * l + q];
        const double theta = (aqq - app) / (2.0 * apq);
        const double t = (theta >= 0 ? 1.0 : -1.0) / (std::fabs(theta) + std::sqrt(theta * theta + 1.0));
        const double c = 1.0 / std::sqrt(t * t + 1.0), s = t * c;
        for (int k = 0; k < l; ++k) {          // columns p, q
          const double ckp = C[(size_t)k * l + p], ckq = C[(size_t)k * l + q];
          C[(size_t)k * l + p] = c * ckp - s * ckq;
          C[(size_t)k * l + q] = s * ckp + c * ckq;
        }
        for (int k = 0; k < l; ++k) {          // rows p, q
          const double cpk = C[(size_t)p * l + k], cqk = C[(size_t)q * l + k];
          C[(size_t)p * l + k] = c * cpk - s * cqk;
          C[(size_t)q * l + k] = s * cpk + c * cqk;
        }
        for (int k = 0; k < l; ++k) {
          const double vkp = V[(size_t)k * l + p], vkq = V[(size_t)k * l + q];
          V[(size_t)k * l + p] = c * vkp - s * vkq;
          V[(size_t)k * l + q] = s * vkp + c * vkq;
        }
      }
    }
  }
}

// Top-r singular triplets of the N x K matrix A: U [N x r], sigma [r],
// V [K x r] (row-major).
static void truncated_svd(const double* A, int N, int K, int r, uint64_t seed,
                          std::vector<double>& U, std::vector<double>& sig,
                          std::vector<double>& V) {
  const int mn = std::min(N, K);
  const int l = std::min(mn, r + std::max(r, 16));
  const int iters = 4;
  SplitMix rng{seed ^ 0x5D5D5D5Dull};
  std::vector<double> Om((size_t)K * l), Y((size_t)N * l), Z((size_t)K * l);
  for (auto& x : Om) x = rng.normal();
  mul_A_B(A, N, K, Om.data(), l, Y.data());
  orthonormalize(Y.data(), N, l);
  for (int it = 0; it < iters; ++it) {
    mul_At_B(A, N, K, Y.data(), l, Z.data());
    orthonormalize(Z.data(), K, l);
    mul_A_B(A, N, K, Z.data(), l, Y.data());
    orthonormalize(Y.data(), N, l);
  }
  // Rayleigh-Ritz: B = Q^T A  (l x K), kept as Z = B^T (K x l); C = B B^T.
  mul_At_B(A, N, K, Y.data(), l, Z.data());
  std::vector<double> C((size_t)l * l, 0.0), W;
#pragma omp parallel for schedule(static)
  for (int i = 0; i < l; ++i)
    for (int j = 0; j < l; ++j) {
      double acc = 0.0;
      for (int k = 0; k < K; ++k) acc += Z[(size_t)k * l + i] * Z[(size_t)k * l + j];
      C[(size_t)i * l + j] = acc;
    }
  jacobi_eigen(C, l, W);
  std::vector<int> order(l);
  for (int i = 0; i < l; ++i) order[i] = i;
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) {
    return C[(size_t)a * l + a] > C[(size_t)b * l + b];
  });
  U.assign((size_t)N * r, 0.0);
  V.assign((size_t)K * r, 0.0);
  sig.assign(r, 0.0);
  for (int t = 0; t < r; ++t) {
    const int c = order[t];
    const double lam = C[(size_t)c * l + c];
    sig[t] = lam > 0 ? std::sqrt(lam) : 0.0;
  }
  const double smax = sig.empty() ? 0.0 : sig[0];
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int t = 0; t < r; ++t) {
      const int c = order[t];
      double acc = 0.0;
      for (int i = 0; i < l; ++i) acc += Y[(size_t)n * l + i] * W[(size_t)i * l + c];
      U[(size_t)n * r + t] = acc;
    }
#pragma omp parallel for schedule(static)
  for (int k = 0; k < K; ++k)
    for (int t = 0; t < r; ++t) {
      const int c = order[t];
      if (!(sig[t] > 1e-13 * smax) || sig[t] == 0.0) { V[(size_t)k * r + t] = 0.0; continue; }
      double acc = 0.0;
      for (int i = 0; i < l; ++i) acc += Z[(size_t)k * l + i] * W[(size_t)i * l + c];
      V[(size_t)k * r + t] = acc / sig[t];
    }
  for (int t = 0; t < r; ++t)
    if (!(sig[t] > 1e-13 * smax)) sig[t] = 0.0;
}

int64_t sf_tile_offset(int row, int g, int K) {
  const int64_t kb = K / 64;
  return ((int64_t)(row / 128) * kb + g / 4) * 512 + (row % 32) * 16 + ((row % 128) / 32) * 4 + (g % 4);
}

// NVFP4 of rows x K float32 (row-major): codes two per byte (even k low
// nibble) and E4M3 scales in the MMA tile layout.
static void quantize_nvfp4_rows(const float* T, int rows, int K, float g, float gs,
                                uint8_t* codes, uint8_t* sf_tiled) {
#pragma omp parallel for schedule(static)
  for (int n = 0; n < rows; ++n) {
    const float* t = T + (size_t)n * K;
    for (int gi = 0; gi < K / 16; ++gi) {
      float a = 0.0f;
      for (int j = 0; j < 16; ++j) a = std::max(a, std::fabs(t[gi * 16 + j]));
      const uint8_t s = e4m3_code(a * gs);
      const float q = (s == 0) ? 0.0f : g / e4m3_value(s);
      sf_tiled[sf_tile_offset(n, gi, K)] = s;
      for (int j = 0; j < 16; j += 2) {
        const uint8_t lo = e2m1_code(t[gi * 16 + j] * q);
        const uint8_t hi = e2m1_code(t[gi * 16 + j + 1] * q);
        codes[(size_t)n * (K / 2) + (gi * 16 + j) / 2] = (uint8_t)(lo | (hi << 4));
      }
    }
  }
}

}  // namespace svdq_host

using namespace svdq_host;

static inline size_t round_up(size_t x, size_t m) { return (x + m - 1) / m * m; }

extern "C" svdq_status svdq_query_sizes(int N, int K, int r, svdq_sizes* out) {
  if (!out || N <= 0 || K <= 0 || N % 16 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (r < 0 || r > 128 || (r != 0 && r % 16)) return SVDQ_ERR_INVALID_ARG;
  if (r > std::min(N, K)) return SVDQ_ERR_INVALID_ARG;
  out->N = N;
  out->K = K;
  out->r = r;
  out->klr = (int)round_up((size_t)2 * r, 64);
  out->smooth_bytes = (size_t)K * 4;
  out->l1_bytes = (size_t)K * r * 2;
  out->l2_bytes = (size_t)r * N * 2;
  out->l1_mma_bytes = (size_t)2 * r * K * 2;
  out->l2_mma_bytes = (size_t)N * out->klr * 2;
  out->codes_w_bytes = (size_t)N * (K / 2);
  out->sf_w_bytes = round_up((size_t)N, 256) * (K / 16);
  out->bias_bytes = (size_t)N * 2;
  return SVDQ_OK;
}

extern "C" int64_t svdq_sf_tile_offset(int row, int g, int K) {
  if (row < 0 || g < 0 || K <= 0 || K % 64 || g >= K / 16) return -1;
  return sf_tile_offset(row, g, K);
}

extern "C" svdq_status svdq_unswizzle_scales(const uint8_t* sf_mma, int rows, int K,
                                             uint8_t* sf_rowmajor) {
  if (rows < 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  if (rows == 0) return SVDQ_OK;
  if (!sf_mma || !sf_rowmajor) return SVDQ_ERR_INVALID_ARG;
  const int G = K / 16;
  for (int m = 0; m < rows; ++m)
    for (int g = 0; g < G; ++g) sf_rowmajor[(size_t)m * G + g] = sf_mma[sf_tile_offset(m, g, K)];
  return SVDQ_OK;
}

extern "C" svdq_status svdq_pack_weight(const float* W, const float* x_absmax,
                                        const uint16_t* bias_bf16, int N, int K, int r,
                                        float smooth_alpha, uint64_t seed,
                                        svdq_packed_host* out) {
  svdq_sizes sz;
  svdq_status st = svdq_query_sizes(N, K, r, &sz);
  if (st != SVDQ_OK) return st;
  if (!W || !x_absmax || !out || !out->smooth || !out->codes_w || !out->sf_w)
    return SVDQ_ERR_INVALID_ARG;
  if (r > 0 && (!out->l1 || !out->l2 || !out->l1_mma || !out->l2_mma))
    return SVDQ_ERR_INVALID_ARG;
  if (bias_bf16 && !out->bias) return SVDQ_ERR_INVALID_ARG;
  if (!(smooth_alpha >= 0.0f) || !std::isfinite(smooth_alpha)) return SVDQ_ERR_INVALID_ARG;
  for (int k = 0; k < K; ++k)
    if (!std::isfinite(x_absmax[k]) || x_absmax[k] < 0) return SVDQ_ERR_NUMERIC;
  for (size_t i = 0; i < (size_t)N * K; ++i)
    if (!std::isfinite(W[i])) return SVDQ_ERR_NUMERIC;

  // 1. smoothing factors, stored as the activation multiplier 1/lambda
  std::vector<double> wmax(K, 0.0);
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      wmax[k] = std::max(wmax[k], (double)std::fabs(W[(size_t)n * K + k]));
  float* s = out->smooth;
  for (int k = 0; k < K; ++k) {
    const double cx = x_absmax[k];
    double lam = 1.0;
    if (cx > 0.0 && wmax[k] > 0.0) {
      const double ratio = cx / wmax[k];
      lam = (smooth_alpha == 0.5f) ? std::sqrt(ratio) : std::pow(ratio, (double)smooth_alpha);
    }
    s[k] = (float)(1.0 / lam);
  }
  std::vector<double> Wt((size_t)N * K);
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k)
      Wt[(size_t)n * K + k] = (double)W[(size_t)n * K + k] / (double)s[k];

  // 2. low-rank branch
  std::vector<double> L1d((size_t)K * r), L2d((size_t)r * N);
  if (r > 0) {
    std::vector<double> U, sig, V;
    truncated_svd(Wt.data(), N, K, r, seed, U, sig, V);
    for (int k = 0; k < K; ++k)
      for (int i = 0; i < r; ++i) {
        const uint16_t h = bf16_from_double(V[(size_t)k * r + i] * std::sqrt(sig[i]));
        out->l1[(size_t)k * r + i] = h;
        L1d[(size_t)k * r + i] = bf16_to_double(h);
      }
    for (int i = 0; i < r; ++i)
      for (int n = 0; n < N; ++n) {
        const uint16_t h = bf16_from_double(std::sqrt(sig[i]) * U[(size_t)n * r + i]);
        out->l2[(size_t)i * N + n] = h;
        L2d[(size_t)i * N + n] = bf16_to_double(h);
      }
  }

  // 3. residual, float64 sum over the rank in ascending order, one rounding
  std::vector<float> R((size_t)N * K);
  float amax = 0.0f;
#pragma omp parallel for schedule(static) reduction(max : amax)
  for (int n = 0; n < N; ++n)
    for (int k = 0; k < K; ++k) {
      double acc = 0.0;
      for (int i = 0; i < r; ++i) acc += L1d[(size_t)k * r + i] * L2d[(size_t)i * N + n];
      const float v = (float)(Wt[(size_t)n * K + k] - acc);
      R[(size_t)n * K + k] = v;
      amax = std::max(amax, std::fabs(v));
    }

  // 4. NVFP4 of R
  const float g_w = tensor_scale(amax);
  std::memset(out->sf_w, 0, sz.sf_w_bytes);
  quantize_nvfp4_rows(R.data(), N, K, g_w, block_scale_factor(amax), out->codes_w, out->sf_w);

  // 5. static activation tensor scale
  float ax = 0.0f;
  for (int k = 0; k < K; ++k) ax = std::max(ax, std::fabs(x_absmax[k] * s[k]));
  const float g_x = tensor_scale(ax);

  // 6. output scale and its inverse for the low-rank branch
  const float lr_scale = g_x * g_w;
  out->amax_x = ax;
  out->amax_w = amax;
  out->g_x = g_x;
  out->gs_x = block_scale_factor(ax);
  out->g_w = g_w;
  out->lr_scale = lr_scale;
  out->alpha = 1.0f / lr_scale;

  // 7. kernel operands of the low-rank branch
  if (r > 0) {
    for (int i = 0; i < r; ++i)
      for (int k = 0; k < K; ++k) {
        const double p = (double)s[k] * L1d[(size_t)k * r + i];  // exact
        const uint16_t hi = bf16_from_double(p);
        const uint16_t lo = bf16_from_double(p - bf16_to_double(hi));
        out->l1_mma[(size_t)i * K + k] = hi;
        out->l1_mma[(size_t)(r + i) * K + k] = lo;
      }
    std::memset(out->l2_mma, 0, sz.l2_mma_bytes);
    for (int n = 0; n < N; ++n)
      for (int i = 0; i < r; ++i) {
        const uint16_t v = out->l2[(size_t)i * N + n];
        out->l2_mma[(size_t)n * sz.klr + i] = v;
        out->l2_mma[(size_t)n * sz.klr + r + i] = v;
      }
  }

  // 8. bias: carried through as bf16 for the GEMM epilogue
  if (out->bias) {
    if (bias_bf16)
      std::memcpy(out->bias, bias_bf16, (size_t)N * 2);
    else
      std::memset(out->bias, 0, (size_t)N * 2);
  }
  return SVDQ_OK;
}

// ----------------------------------------------------------------- AWQ ----
// binary16 (1 sign, 5 exponent bits with bias 15, 10 fraction bits;
// subnormals k * 2^-24) nearest to a double, ties to even.
static uint16_t half_from_double(double x) {
  const uint16_t sign = std::signbit(x) ? 0x8000 : 0;
  const double a = std::fabs(x);
  if (a == 0.0) return sign;
  if (!(a < 65520.0)) return (uint16_t)(sign | 0x7C00);   // rounds past 65504
  if (a < std::ldexp(1.0, -14)) {
    const double k = std::rint(std::ldexp(a, 24));          // 0 .. 1024 (1024: smallest normal)
    return (uint16_t)(sign | (uint16_t)k);
  }
  int e = 0;
  const double m = std::frexp(a, &e);                      // a = m 2^e, m in [0.5, 1)
  double r = std::rint(std::ldexp(m, 11));                 // 1024 .. 2048
  int ex = e - 1;
  if (r == 2048.0) {
    r = 1024.0;
    ex += 1;
  }
  if (ex > 15) return (uint16_t)(sign | 0x7C00);
  return (uint16_t)(sign | ((ex + 15) << 10) | ((int)r - 1024));
}

static double half_to_double(uint16_t h) {
  const int e = (h >> 10) & 31, f = h & 1023;
  const double v = e == 0 ? std::ldexp((double)f, -24) : std::ldexp(1.0 + f / 1024.0, e - 15);
  return (h & 0x8000) ? -v : v;
}

// The AWQ GEMV's code layout: per 16-row block and 64-deep block of K, 512
// bytes = 32 lanes x 16 bytes; lane l = 4 g + c holds one 32-bit word per
// 16-deep k-step ks (4 per block), and nibble j of the word is the code of
//   row 16 rb + g + 8 (j % 2),  column 16 ks + 2 c + 8 ((j % 4) / 2) + j / 4
// (the m16n8k16 A-fragment element of register j % 4, half j / 4).  Rows
// past N hold code 0.
extern "C" svdq_status svdq_awq_tile_codes(const uint8_t* q_rowmajor, int N, int K,
                                           uint8_t* q_tiled) {
  if (!q_rowmajor || !q_tiled || N <= 0 || K <= 0 || K % 64) return SVDQ_ERR_INVALID_ARG;
  const int RB = (N + 15) / 16, KS = K / 16;
#pragma omp parallel for schedule(static)
  for (int rb = 0; rb < RB; ++rb)
    for (int ks = 0; ks < KS; ++ks)
      for (int l = 0; l < 32; ++l) {
        const int g = l >> 2, c = l & 3;
        uint32_t word = 0;
        for (int j = 0; j < 8; ++j) {
          const int n = 16 * rb + g + 8 * (j & 1);
          const int k = 16 * ks + 2 * c + 8 * ((j & 3) >> 1) + (j >> 2);
          uint32_t code = 0;
          if (n < N) {
            const uint8_t b = q_rowmajor[(size_t)n * (K / 2) + k / 2];
            code = (k & 1) ? (b >> 4) : (b & 15u);
          }
          word |= code << (4 * j);
        }
        const size_t off = (((size_t)rb * (K / 64) + (ks >> 2)) * 32 + l) * 16 + (ks & 3) * 4;
        std::memcpy(q_tiled + off, &word, 4);
      }
  return SVDQ_OK;
}

extern "C" svdq_status svdq_awq_pack(const float* W, int N, int K, int group, uint8_t* q_packed,
                                     uint8_t* zeros, uint16_t* scales) {
  if (!W || !q_packed || !zeros || !scales || N <= 0 || K <= 0 || group <= 0 || group % 32 ||
      K % group)
    return SVDQ_ERR_INVALID_ARG;
  for (size_t i = 0; i < (size_t)N * K; ++i)
    if (!std::isfinite(W[i])) return SVDQ_ERR_NUMERIC;
  const int G = K / group;
#pragma omp parallel for schedule(static)
  for (int n = 0; n < N; ++n) {
    for (int gi = 0; gi < G; ++gi) {
      const float* w = W + (size_t)n * K + (size_t)gi * group;
      double wmin = 0.0, wmax = 0.0;   // the range includes 0
      for (int j = 0; j < group; ++j) {
        wmin = std::min(wmin, (double)w[j]);
        wmax = std::max(wmax, (double)w[j]);
      }
      const uint16_t hb = half_from_double(std::max(wmax - wmin, 1e-5) / 15.0);
      const double scale = half_to_double(hb);
      const double z = std::min(15.0, std::max(0.0, std::rint(-wmin / scale)));
      scales[(size_t)n * G + gi] = hb;
      zeros[(size_t)n * G + gi] = (uint8_t)z;
      for (int j = 0; j < group; j += 2) {
        const double q0 = std::min(15.0, std::max(0.0, std::rint((double)w[j] / scale) + z));
        const double q1 = std::min(15.0, std::max(0.0, std::rint((double)w[j + 1] / scale) + z));
        q_packed[(size_t)n * (K / 2) + ((size_t)gi * group + j) / 2] =
            (uint8_t)((int)q0 | ((int)q1 << 4));
      }
    }
  }
  return SVDQ_OK;
}
