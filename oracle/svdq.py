"""SVDQuant W4A4 linear layer, restated step by step (CPU, numpy, float64).

What the pages fix ("Bringing Nunchaku 4-bit diffusion inference to
Diffusers", section "Background: SVDQuant and Nunchaku", and its Russian and
Korean renderings; the Hacker News thread on "SVDQuant: 4-Bit Quantization
Powers 12B Flux ..."):
  1. activation outliers are migrated into the weights (smoothing);
  2. the hardest part of each smoothed weight is kept as a small 16-bit
     low-rank branch (a top-r SVD: "basically a LoRA");
  3. only the residual is quantized to 4 bit; weights AND activations are
     4-bit (W4A4), NVFP4 on Blackwell (hardware-support table);
  4. the forward pass is  Y = Q(X_hat) Q(R)^T + (X_hat L1) L2 (+ bias).

Readings of what the pages leave open:
  R1 smoothing: lambda_j = (cx_j / wmax_j) ** alpha with alpha = 0.5, where
     cx_j = max_m |X_mj| over the calibration batch and wmax_j =
     max_n |W_nj|; lambda_j = 1 if either maximum is 0.  The stored factor
     is the activation multiplier s_j = fp32(1 / lambda_j); the smoothed
     activation is x_hat = fp32(x * s_j) (one float32 rounding) and the
     smoothed weight is W~_nj = W_nj / s_j (float64), so s_j cancels
     exactly in X_hat W~^T up to the rounding of x_hat.  For alpha = 0.5 the
     power is a square root (correctly rounded everywhere).
  R2 low-rank split: W~ = U S V^T (top r), L1 = V sqrt(S) [K x r],
     L2 = sqrt(S) U^T [r x N], each rounded once from float64 to bf16.
     The SVD is not unique, so parity of the rest of the path is defined
     GIVEN the stored L1, L2.
  R3 residual: R_nk = fp32( W~_nk - sum_{i ascending} L1_ki * L2_in ), the
     sum in float64.
  R4 NVFP4 recipe for a tensor T with tensor absmax A (fp32):
       g   = fp32(2688 / A)            element encode scale (2688 = 6 * 448)
       gs  = fp32(448 / A)             block-scale encode scale (= g / 6)
       (g = gs = 1 if A = 0)
       per group G of 16 consecutive elements along K:
       a   = max_{t in G} |t|
       sf  = E4M3_rn_satfinite( fp32(a * gs) )
       q   = 0 if sf == 0 else fp32( g / e4m3(sf) )
       code= E2M1_rn_satfinite( fp32(t * q) )
     dequantized value = e2m1(code) * e4m3(sf) / g.
  R5 activation tensor scale is static (from calibration):
     A_x = max_j fp32(cx_j * s_j), which equals max |x_hat| over the
     calibration batch (rounding is monotone); g_x, gs_x follow R4.
     Run-time values beyond it saturate (satfinite).
  R6 reference output: Y_ref = D / (g_x g_w) + (X_hat L1) L2 + bias in
     float64, D = deq(codes_x, sf_x) deq(codes_w, sf_w)^T (the codes are
     the method's own 4-bit encodings; 1/(g_x g_w) undoes both tensor
     scales).
  R7 packed layouts: codes are two per byte, the even k in the low nibble;
     block scales in the MMA tile layout (see `sf_to_mma_tiles`).
  R11f GELU between the MLP pair's layers, in a form a fused kernel and this
     oracle evaluate bit-identically: the tanh form of GELU,
       0.5 y (1 + tanh(u)),  u = sqrt(2/pi) (y + 0.044715 y^3),
     rewritten through 1 + tanh(u) = 2 / (1 + e^(-2u)) as
       h = y / (1 + e^(-2u))      (no cancellation for any y),
     every step one float32 operation in the order written in `gelu_tanh_f32`,
     e^x from `exp_f32` (basic float32 operations only), h rounded to bf16.
  R5d dynamic per-token activation scale (an alternative to R5 for inputs
     outside the calibration range; not the pages' path): each row m of
     X_hat is its own tensor for R4, with A_m = max_k |x_hat_mk| taken at
     run time; the output undoes g_x,m = fp32(2688 / A_m) row by row.  A row
     whose x_hat is all zero has A_m = 0, so g = gs = 1 and all codes 0.

Parity pins: tests/test_oracle_formats.py, tests/test_oracle_svdq.py.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np

from .formats import (bf16_bits_to_f64, e2m1_decode, e2m1_encode,
                      e4m3_decode, e4m3_encode_nonneg, f64_to_bf16_bits)

F32 = np.float32
NVFP4_GROUP = 16
NVFP4_AMAX_TARGET = F32(6.0 * 448.0)      # 2688


# ------------------------------------------------------------ smoothing ----

def smoothing_factors(x_absmax: np.ndarray, W: np.ndarray,
                      alpha: float = 0.5) -> np.ndarray:
    """Step 1 (smoothing), reading R1.  Returns s = fp32(1/lambda), [K]."""
    cx = np.asarray(x_absmax, dtype=F32).astype(np.float64)
    wmax = np.abs(np.asarray(W, dtype=F32)).max(axis=0).astype(np.float64)
    ok = (cx > 0) & (wmax > 0)
    ratio = np.where(ok, cx / np.where(ok, wmax, 1.0), 1.0)
    if alpha == 0.5:
        lam = np.sqrt(ratio)
    else:
        lam = np.power(ratio, alpha)
    lam = np.where(ok, lam, 1.0)
    return (1.0 / lam).astype(F32)


def smooth_weight(W: np.ndarray, s: np.ndarray) -> np.ndarray:
    """W~ = W diag(lambda) = W / s  (float64), [N, K]."""
    return np.asarray(W, dtype=F32).astype(np.float64) / np.asarray(s, F32).astype(np.float64)[None, :]


def smooth_activation(X_bf16: np.ndarray, s: np.ndarray) -> np.ndarray:
    """x_hat = fp32(x * s_j): one float32 rounding, [M, K] float32."""
    x = bf16_bits_to_f64(X_bf16).astype(F32)
    return (x * np.asarray(s, F32)[None, :]).astype(F32)


# ------------------------------------------------------- low-rank branch ----

def lowrank_factors(W_tilde: np.ndarray, r: int, round_bf16: bool = True):
    """Step 2: top-r SVD of W~ (numpy LAPACK, float64), reading R2.
    Returns (L1 [K, r], L2 [r, N]) as bf16 bit patterns, or as float64 when
    round_bf16 is False (used by the full-rank pin)."""
    U, S, Vt = np.linalg.svd(W_tilde, full_matrices=False)
    root = np.sqrt(S[:r])
    L1 = Vt[:r, :].T * root[None, :]
    L2 = root[:, None] * U[:, :r].T
    if not round_bf16:
        return L1, L2
    return f64_to_bf16_bits(L1), f64_to_bf16_bits(L2)


def lowrank_product_t(L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """(L1 L2)^T as [N, K], float64, summed over i in ascending order."""
    L1d = bf16_bits_to_f64(L1) if L1.dtype == np.uint16 else np.asarray(L1, np.float64)
    L2d = bf16_bits_to_f64(L2) if L2.dtype == np.uint16 else np.asarray(L2, np.float64)
    K, r = L1d.shape
    N = L2d.shape[1]
    acc = np.zeros((N, K), dtype=np.float64)
    for i in range(r):
        acc += np.outer(L2d[i, :], L1d[:, i])
    return acc


def residual64(W_tilde: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """Step 3 before the float32 cast: W~ - (L1 L2)^T, float64 [N, K]."""
    return W_tilde - lowrank_product_t(L1, L2)


def residual(W_tilde: np.ndarray, L1: np.ndarray, L2: np.ndarray) -> np.ndarray:
    """Step 3, reading R3: R = fp32(W~ - (L1 L2)^T)."""
    return residual64(W_tilde, L1, L2).astype(F32)


# ----------------------------------------------------------------- NVFP4 ----

def tensor_encode_scale(amax) -> np.float32:
    """g = fp32(2688 / A); g = 1 when A = 0 (reading R4)."""
    amax = F32(amax)
    if amax == 0:
        return F32(1.0)
    return F32(NVFP4_AMAX_TARGET / amax)


def block_scale_factor(amax) -> np.float32:
    """gs = fp32(448 / A); gs = 1 when A = 0 (reading R4)."""
    amax = F32(amax)
    if amax == 0:
        return F32(1.0)
    return F32(F32(448.0) / amax)


def nvfp4_quantize(T: np.ndarray, amax) -> Tuple[np.ndarray, np.ndarray]:
    """Reading R4.  T: float32 [rows, K] (K % 16 == 0), amax: the fp32
    tensor absmax A that fixes the tensor scales.  Returns (codes uint8
    [rows, K] one code per byte, sf uint8 [rows, K/16] E4M3 codes)."""
    T = np.asarray(T, dtype=F32)
    rows, K = T.shape
    assert K % NVFP4_GROUP == 0
    g = tensor_encode_scale(amax)
    gs = block_scale_factor(amax)
    grp = T.reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    a = np.abs(grp).max(axis=2).astype(F32)
    sf = e4m3_encode_nonneg((a * gs).astype(F32))
    dec = e4m3_decode(sf).astype(F32)
    with np.errstate(divide="ignore"):
        q = np.where(sf == 0, F32(0.0), (g / np.where(sf == 0, F32(1.0), dec)).astype(F32)).astype(F32)
    v = (grp * q[:, :, None]).astype(F32)
    codes = e2m1_encode(v).reshape(rows, K)
    return codes, sf


def nvfp4_dequantize(codes: np.ndarray, sf: np.ndarray) -> np.ndarray:
    """e2m1(code) * e4m3(sf), float64 [rows, K] (without the 1/g)."""
    rows, K = codes.shape
    vals = e2m1_decode(codes).reshape(rows, K // NVFP4_GROUP, NVFP4_GROUP)
    return (vals * e4m3_decode(sf)[:, :, None]).reshape(rows, K)


# ------------------------------------------------------ packed layouts ----

def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """[rows, K] codes -> [rows, K/2] bytes, even k in the low nibble."""
    codes = np.asarray(codes, dtype=np.uint8)
    return (codes[:, 0::2] & 0xF) | ((codes[:, 1::2] & 0xF) << 4)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    rows, half = packed.shape
    out = np.empty((rows, 2 * half), dtype=np.uint8)
    out[:, 0::2] = packed & 0xF
    out[:, 1::2] = packed >> 4
    return out


def sf_to_mma_tiles(sf: np.ndarray, row_multiple: int = 128) -> np.ndarray:
    """Block scales [rows, K/16] -> the MMA tile layout (flat uint8).

    Rows are padded with zero scales to a multiple of `row_multiple` (a
    multiple of 128).  The tensor is cut into atoms of 128 rows x 4 scales
    (64 elements of K), 512 bytes each; atom (row block b, k block c) sits
    at byte ((b * (K/64)) + c) * 512.  Inside an atom, row m (0..127) and
    scale j (0..3) sit at byte (m % 32) * 16 + (m // 32) * 4 + j, so the
    four scales of one row form one 32-bit word and 32 rows x 16 bytes form
    one 512-byte block.  This is the scale-factor arrangement the block-
    scaled tensor-core MMA consumes (one atom per 128 rows per 64 k)."""
    sf = np.asarray(sf, dtype=np.uint8)
    rows, nsf = sf.shape
    assert nsf % 4 == 0 and row_multiple % 128 == 0
    prow = -(-rows // row_multiple) * row_multiple
    padded = np.zeros((prow, nsf), dtype=np.uint8)
    padded[:rows] = sf
    nb, kb = prow // 128, nsf // 4
    # index names: b row block, q = m // 32, p = m % 32, c k block, j scale
    t = padded.reshape(nb, 4, 32, kb, 4)          # [b, q, p, c, j]
    t = t.transpose(0, 3, 2, 1, 4)                # [b, c, p, q, j]
    return np.ascontiguousarray(t).reshape(-1)


def sf_from_mma_tiles(tiled: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Inverse of `sf_to_mma_tiles` for the first `rows` rows."""
    nsf = K // NVFP4_GROUP
    kb = nsf // 4
    nb = -(-rows // 128)
    t = np.asarray(tiled, np.uint8)[:nb * kb * 512].reshape(nb, kb, 32, 4, 4)  # [b, c, p, q, j]
    t = t.transpose(0, 3, 2, 1, 4).reshape(nb * 128, nsf)                     # [b, q, p, c, j]
    return np.ascontiguousarray(t[:rows])


# --------------------------------------------------------- whole layer ----

@dataclass
class OraclePack:
    """What the offline pack produces (oracle side)."""
    s: np.ndarray            # fp32 [K]
    L1: np.ndarray           # bf16 bits [K, r]
    L2: np.ndarray           # bf16 bits [r, N]
    R: np.ndarray            # fp32 [N, K]
    g_w: np.float32
    g_x: np.float32
    A_w: np.float32          # tensor absmax of R
    A_x: np.float32          # static activation absmax (reading R5)
    codes_w: np.ndarray      # uint8 [N, K] (one code per byte)
    sf_w: np.ndarray         # uint8 [N, K/16]


def activation_absmax(x_absmax: np.ndarray, s: np.ndarray) -> np.float32:
    """Reading R5: A_x = max_j fp32(cx_j * s_j)."""
    a = (np.asarray(x_absmax, F32) * np.asarray(s, F32)).astype(F32)
    return F32(np.abs(a).max()) if a.size else F32(0)


def activation_tensor_scale(x_absmax: np.ndarray, s: np.ndarray) -> np.float32:
    """g_x = fp32(2688 / A_x) (readings R4, R5)."""
    return tensor_encode_scale(activation_absmax(x_absmax, s))


def quantize_weight(W: np.ndarray, s: np.ndarray, L1: np.ndarray,
                    L2: np.ndarray):
    """Steps 2-3 for given smoothing factors and low-rank factors:
    R, A_w, codes_w, sf_w."""
    Wt = smooth_weight(W, s)
    R = residual(Wt, L1, L2)
    A_w = F32(np.abs(R).max()) if R.size else F32(0)
    codes, sf = nvfp4_quantize(R, A_w)
    return R, A_w, codes, sf


def pack(W: np.ndarray, x_absmax: np.ndarray, r: int,
         alpha: float = 0.5, L1: Optional[np.ndarray] = None,
         L2: Optional[np.ndarray] = None) -> OraclePack:
    """The whole offline pack.  When L1/L2 are given they are used as the
    low-rank branch (parity given the stored factors, reading R2)."""
    s = smoothing_factors(x_absmax, W, alpha)
    if L1 is None or L2 is None:
        if r > 0:
            L1, L2 = lowrank_factors(smooth_weight(W, s), r)
        else:
            K, N = W.shape[1], W.shape[0]
            L1 = np.zeros((K, 0), np.uint16)
            L2 = np.zeros((0, N), np.uint16)
    R, A_w, codes, sf = quantize_weight(W, s, L1, L2)
    A_x = activation_absmax(x_absmax, s)
    return OraclePack(s, L1, L2, R, tensor_encode_scale(A_w), tensor_encode_scale(A_x),
                      A_w, A_x, codes, sf)


def quantize_activation(X_bf16: np.ndarray, s: np.ndarray, A_x):
    """The activation step: smoothing then NVFP4 with the static tensor
    absmax A_x.  Returns (x_hat fp32, codes [M, K], sf [M, K/16])."""
    xh = smooth_activation(X_bf16, s)
    codes, sf = nvfp4_quantize(xh, A_x)
    return xh, codes, sf


def lowrank_down(x_hat: np.ndarray, L1: np.ndarray) -> np.ndarray:
    """X_hat L1 in float64, [M, r]."""
    return x_hat.astype(np.float64) @ bf16_bits_to_f64(L1)


def linear_reference(X_bf16: np.ndarray, p: OraclePack,
                     bias_bf16: Optional[np.ndarray] = None,
                     rows: Optional[np.ndarray] = None,
                     deq_w: Optional[np.ndarray] = None):
    """Reading R6: the float64 reference output Y_ref [M, N] (or only the
    listed rows).  `deq_w` may pass nvfp4_dequantize(p.codes_w, p.sf_w)
    computed once for many calls.  Returns (Y_ref, codes_x, sf_x, xl1)."""
    X = X_bf16 if rows is None else X_bf16[rows]
    xh, cx, sfx = quantize_activation(X, p.s, p.A_x)
    if deq_w is None:
        deq_w = nvfp4_dequantize(p.codes_w, p.sf_w)
    D = nvfp4_dequantize(cx, sfx) @ deq_w.T
    Y = D / (np.float64(p.g_x) * np.float64(p.g_w))
    xl1 = lowrank_down(xh, p.L1)
    if p.L1.shape[1]:
        Y = Y + xl1 @ bf16_bits_to_f64(p.L2)
    if bias_bf16 is not None:
        Y = Y + bf16_bits_to_f64(bias_bf16)[None, :]
    return Y, cx, sfx, xl1


# --------------------------------- dynamic per-token activation scale ----

def activation_absmax_rows(x_hat: np.ndarray) -> np.ndarray:
    """Reading R5d: A_m = max_k |x_hat_mk| per row, fp32 (exact)."""
    xh = np.asarray(x_hat, F32)
    if xh.shape[1] == 0:
        return np.zeros(xh.shape[0], F32)
    return np.abs(xh).max(axis=1).astype(F32)


def quantize_activation_dynamic(X_bf16: np.ndarray, s: np.ndarray):
    """Reading R5d: smoothing, then R4 on each row with that row's own
    absmax.  Returns (x_hat fp32, codes [M, K], sf [M, K/16], A fp32 [M])."""
    xh = smooth_activation(X_bf16, s)
    A = activation_absmax_rows(xh)
    M, K = xh.shape
    codes = np.zeros((M, K), np.uint8)
    sf = np.zeros((M, K // NVFP4_GROUP), np.uint8)
    for m in range(M):
        codes[m:m + 1], sf[m:m + 1] = nvfp4_quantize(xh[m:m + 1], A[m])
    return xh, codes, sf, A


def linear_reference_dynamic(X_bf16: np.ndarray, p: OraclePack,
                             bias_bf16: Optional[np.ndarray] = None,
                             rows: Optional[np.ndarray] = None,
                             deq_w: Optional[np.ndarray] = None):
    """Reading R6 with R5d in place of R5: row m of the 4-bit product is
    divided by g_x,m g_w.  Returns (Y_ref, codes_x, sf_x, xl1, A_rows)."""
    X = X_bf16 if rows is None else X_bf16[rows]
    xh, cx, sfx, A = quantize_activation_dynamic(X, p.s)
    if deq_w is None:
        deq_w = nvfp4_dequantize(p.codes_w, p.sf_w)
    g_rows = np.array([tensor_encode_scale(a) for a in A], np.float64)
    D = nvfp4_dequantize(cx, sfx) @ deq_w.T
    Y = D / (g_rows[:, None] * np.float64(p.g_w))
    xl1 = lowrank_down(xh, p.L1)
    if p.L1.shape[1]:
        Y = Y + xl1 @ bf16_bits_to_f64(p.L2)
    if bias_bf16 is not None:
        Y = Y + bf16_bits_to_f64(bias_bf16)[None, :]
    return Y, cx, sfx, xl1, A


# ------------------------------------------- GELU of the MLP pair (R11f) ----

_LOG2E = F32(1.4426950408889634)          # log2(e), rounded to float32
_EXP2_TAYLOR = [F32(np.log(2.0) ** k / np.prod(np.arange(1, k + 1, dtype=np.float64)))
                for k in range(8)]        # (ln 2)^k / k!, k = 0..7, float32
_SQRT_2_OVER_PI = F32(np.sqrt(2.0 / np.pi))
_GELU_CUBIC = F32(0.044715)


def exp_f32(x: np.ndarray) -> np.ndarray:
    """e^x in float32 from basic float32 operations (reading R11f):
    t = fp32(x log2 e), clamped to [-126, 128]; n = t rounded to the nearest
    integer (ties to even); f = t - n (exact, |f| <= 1/2); 2^f from the
    degree-7 Taylor series of e^(f ln 2) in Horner form (each multiply and
    add rounded to float32); the result is 2^f scaled by 2^n (exact; 2^128
    overflows to inf).  Relative error a few 1e-6 at |x| ~ 80, from the
    rounding of t; far below a bf16 ulp."""
    x = np.asarray(x, F32)
    t = (x * _LOG2E).astype(F32)
    t = np.clip(t, F32(-126.0), F32(128.0)).astype(F32)
    n = np.rint(t).astype(F32)
    f = (t - n).astype(F32)
    p = np.full(x.shape, _EXP2_TAYLOR[7], F32)
    for k in range(6, -1, -1):
        p = (p * f).astype(F32)
        p = (p + _EXP2_TAYLOR[k]).astype(F32)
    with np.errstate(over="ignore"):
        return np.ldexp(p, n.astype(np.int32)).astype(F32)


def gelu_tanh_f32(y: np.ndarray) -> np.ndarray:
    """GELU, tanh form, reading R11f: h = y / (1 + e^(-2u)) with
    u = sqrt(2/pi) (y + 0.044715 y^3), each step one float32 rounding:
    y2 = y y, y3 = y2 y, v = 0.044715 y3, w = y + v, u = c w, E = exp(-2u),
    d = 1 + E, h = y / d.  For finite y: h = y exactly for large y (E
    underflows to 2^-126), and h = -0 once e^(-2u) passes 2^128 (where the
    true value is below 2^-120 in magnitude: an absolute error under
    2^-120).  Tiny inputs keep gradual underflow: for y below 2^-126 the
    result is y / 2 rounded in the float32 subnormal range."""
    y = np.asarray(y, F32)
    with np.errstate(over="ignore", divide="ignore", invalid="ignore"):
        return _gelu_steps(y)


def _gelu_steps(y: np.ndarray) -> np.ndarray:
    y2 = (y * y).astype(F32)
    y3 = (y2 * y).astype(F32)
    v = (_GELU_CUBIC * y3).astype(F32)
    w = (y + v).astype(F32)
    u = (_SQRT_2_OVER_PI * w).astype(F32)
    E = exp_f32((F32(-2.0) * u).astype(F32))
    d = (F32(1.0) + E).astype(F32)
    return (y / d).astype(F32)


def gelu_bf16(Y_bf16: np.ndarray) -> np.ndarray:
    """The MLP pair's glue on bf16 bits: bf16(gelu_tanh_f32(y))."""
    y = bf16_bits_to_f64(Y_bf16).astype(F32)
    return f64_to_bf16_bits(gelu_tanh_f32(y).astype(np.float64))


# ------------------------------------------------------------ tolerance ----

def bf16_half_ulp(y: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at |y| (8 significant bits)."""
    a = np.abs(np.asarray(y, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.where(a > 0, 2.0 ** (e - 8), 2.0 ** -134)


def output_errors(Y: np.ndarray, Y_ref: np.ndarray):
    """(relative Frobenius error, max |Y - Y_ref| / rms(Y_ref),
    max excess of |Y - Y_ref| over 1e-2 rms + half a bf16 ulp)."""
    Y = np.asarray(Y, np.float64)
    Y_ref = np.asarray(Y_ref, np.float64)
    diff = Y - Y_ref
    fro = np.linalg.norm(diff) / max(np.linalg.norm(Y_ref), 1e-300)
    rms = np.sqrt(np.mean(Y_ref ** 2)) if Y_ref.size else 0.0
    maxabs = np.abs(diff).max() / max(rms, 1e-300) if diff.size else 0.0
    bound = 1e-2 * rms + bf16_half_ulp(np.maximum(np.abs(Y), np.abs(Y_ref)))
    excess = (np.abs(diff) - bound).max() if diff.size else -1.0
    return float(fro), float(maxabs), float(excess)
