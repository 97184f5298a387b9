"""Number formats used by NVFP4, written from their definitions.

* E2M1 ("FP4"): 1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit.  The
  eight magnitudes are 0, 0.5 (subnormal), 1, 1.5, 2, 3, 4, 6; there is no
  infinity or NaN.  Code = sign<<3 | magnitude index.
* E4M3 (the "fn" variant used for NVFP4 block scales): 4 exponent bits
  (bias 7), 3 mantissa bits, subnormals m * 2^-9, largest finite 448,
  code 0x7F = NaN, no infinity.  Block scales are non-negative, so only codes
  0..126 occur.
* bfloat16: the top 16 bits of an IEEE float32.

Rounding is round-to-nearest, ties to the even code ("rn"), and
"satfinite": a magnitude beyond the largest finite value becomes that value.
With nearest-point rounding over the finite values this is automatic.  The
sign of a value that rounds to zero is kept (-0.1 -> code 0x8).

Parity: pinned in tests/test_oracle_formats.py against independent
implementations (ml_dtypes float4_e2m1fn, torch float8_e4m3fn), against
brute force in exact rational arithmetic, and against hand-worked fixtures.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

# ---------------------------------------------------------------- E2M1 ----

E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """E2M1 code (0..15, one per uint8) -> float64 value."""
    codes = np.asarray(codes).astype(np.int64)
    mag = E2M1_MAGNITUDES[codes & 7]
    return np.where((codes >> 3) & 1, -mag, mag)


def e2m1_encode(v: np.ndarray, chunk: int = 1 << 20) -> np.ndarray:
    """float32 -> E2M1 code, round to nearest (ties to the even code),
    saturating at +-6, sign kept for values that round to zero.

    Nearest-point search over the eight magnitudes; when two magnitudes are
    equally near, the one whose code is even (mantissa bit 0) wins."""
    v = np.asarray(v, dtype=np.float32)
    flat = v.reshape(-1)
    out = np.empty(flat.shape, dtype=np.uint8)
    for s in range(0, flat.size, chunk):
        part = flat[s:s + chunk]
        # satfinite: every magnitude at or beyond 6 becomes 6
        mag = np.minimum(np.abs(part.astype(np.float64)), 6.0)
        d = np.abs(mag[:, None] - E2M1_MAGNITUDES[None, :])
        dmin = d.min(axis=1, keepdims=True)
        is_min = d == dmin
        idx = np.arange(8)[None, :]
        # among the nearest candidates prefer an even code; at most two tie
        even_pick = np.where(is_min & (idx % 2 == 0), idx, 99).min(axis=1)
        any_pick = np.where(is_min, idx, 99).min(axis=1)
        best = np.where(even_pick < 99, even_pick, any_pick)
        sign = np.signbit(part).astype(np.uint8)
        out[s:s + chunk] = (best.astype(np.uint8) | (sign << 3))
    return out.reshape(v.shape)


# ---------------------------------------------------------------- E4M3 ----

def _e4m3_table() -> np.ndarray:
    vals = []
    for code in range(127):  # 0x7F is NaN
        e, m = code >> 3, code & 7
        if e == 0:
            vals.append(m * 2.0 ** -9)
        else:
            vals.append((1.0 + m / 8.0) * 2.0 ** (e - 7))
    return np.array(vals, dtype=np.float64)


E4M3_VALUES = _e4m3_table()        # index = code, strictly increasing
E4M3_MAX = 448.0


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 code (0..126, non-negative scales) -> float64 value."""
    codes = np.asarray(codes).astype(np.int64)
    if np.any(codes > 126):
        raise ValueError("E4M3 block scale codes must be in 0..126")
    return E4M3_VALUES[codes]


def e4m3_encode_nonneg(a: np.ndarray) -> np.ndarray:
    """Non-negative float32 -> E4M3 code, round to nearest (ties to even
    code), saturating at 448."""
    a = np.asarray(a, dtype=np.float32).astype(np.float64)
    if np.any(a < 0) or np.any(~np.isfinite(a)):
        raise ValueError("block scale input must be finite and >= 0")
    hi = np.searchsorted(E4M3_VALUES, a, side="left")     # first value >= a
    hi = np.minimum(hi, 126)
    lo = np.maximum(hi - 1, 0)
    d_hi = np.abs(E4M3_VALUES[hi] - a)
    d_lo = np.abs(a - E4M3_VALUES[lo])
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi)
    code = np.where(a >= E4M3_MAX, 126, code)
    return code.astype(np.uint8)


# ------------------------------------------------------------ bfloat16 ----

def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float64 -> bfloat16, ONE rounding (nearest, ties to even) straight
    from the float64 value, with gradual underflow: below the smallest
    normal bf16 (2^-126) the values are the multiples of 2^-133 (7 mantissa
    bits, exponent field 0), so |x| rounds to the nearest such multiple,
    ties to the even one; the result keeps the sign (a value that rounds to
    zero gives a signed zero)."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    bits = x.view(np.uint64)
    sign = (bits >> np.uint64(63)).astype(np.uint64)
    mag_bits = bits & np.uint64(0x7FFFFFFFFFFFFFFF)
    # normal range: keep sign+exponent(11)+7 mantissa bits, drop the low 45
    keep = mag_bits >> np.uint64(45)
    rem = mag_bits & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rem > half) | ((rem == half) & ((keep & np.uint64(1)) == np.uint64(1)))
    keep = keep + up.astype(np.uint64)
    rounded = (keep << np.uint64(45)).view(np.float64)
    f = rounded.astype(np.float32)       # exact: 8 significant bits
    fb = f.view(np.uint32) >> np.uint32(16)
    # subnormal range: the count of 2^-133 steps, rounded half to even
    # (np.rint); a count of 128 is the smallest normal, 0x0080, as it should
    mag = np.abs(x)
    tiny = mag < 2.0 ** -126
    steps = np.rint(np.where(tiny, mag, 0.0) * 2.0 ** 133).astype(np.uint32)
    fb = np.where(tiny, steps, fb)
    fb = fb.astype(np.uint16) | (sign.astype(np.uint16) << np.uint16(15))
    return fb


def bf16_round_exact(x: float) -> Fraction:
    """Brute force (exact rationals): nearest bf16 value to x, ties to even,
    with the subnormal grid (multiples of 2^-133) below 2^-126.  Used only by
    the pins."""
    fx = Fraction(x)
    if fx == 0:
        return Fraction(0)
    s = -1 if fx < 0 else 1
    a = abs(fx)
    if a < Fraction(2) ** -126:
        scaled = a * Fraction(2) ** 133
        lo = int(scaled)
        frac = scaled - lo
        if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
            lo += 1
        return s * Fraction(lo) * Fraction(2) ** -133
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    # a in [1, 2): 8 significant bits -> steps of 2^-7
    scaled = a * 128
    lo = int(scaled)
    frac = scaled - lo
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return s * Fraction(lo, 128) * Fraction(2) ** e
