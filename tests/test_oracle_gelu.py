"""Pins for the oracle's float32 GELU of the MLP pair (reading R11f): its own
exp against numpy's float64 exp, the GELU against a 40-digit evaluation of
the tanh form (mpmath) and against torch's float64 GELU where that formula
is well conditioned, exact special values, and the bf16 glue against the
correctly rounded 40-digit value on every finite bf16 input."""
import mpmath
import numpy as np
import pytest

from oracle import formats as F
from oracle import svdq as O

mpmath.mp.dps = 40
TINY = 2.0 ** -120


def _gelu_exact(y: float) -> float:
    yv = mpmath.mpf(float(y))
    u = mpmath.sqrt(2 / mpmath.pi) * (yv + mpmath.mpf("0.044715") * yv ** 3)
    return float(yv / (1 + mpmath.exp(-2 * u)))


def test_exp_f32_against_float64_exp():
    x = np.concatenate([np.linspace(-87.0, 88.0, 100001), [0.0, 1.0, -1.0]]).astype(np.float32)
    got = O.exp_f32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    assert np.max(np.abs(got - ref) / ref) < 8e-6
    assert O.exp_f32(np.float32(0.0)) == 1.0
    assert O.exp_f32(np.float32(-200.0)) == np.float32(2.0 ** -126)   # the clamp
    assert np.isinf(O.exp_f32(np.float32(100.0)))


def test_gelu_f32_against_40_digits():
    rng = np.random.default_rng(0)
    y = np.concatenate([np.linspace(-10.0, 12.0, 2201), rng.uniform(-10.0, 3.0, 800),
                        [-1e-3, 1e-3, -0.7517916, 9.99]]).astype(np.float32)
    got = O.gelu_tanh_f32(y).astype(np.float64)
    ref = np.array([_gelu_exact(v) for v in y])
    big = np.abs(ref) >= TINY
    assert np.max(np.abs(got[big] - ref[big]) / np.abs(ref[big])) < 2e-5
    assert np.max(np.abs(got[~big] - ref[~big]), initial=0.0) < TINY


def test_gelu_f32_against_torch_where_well_conditioned():
    """torch evaluates 0.5 y (1 + tanh u); for y >= -4 the sum 1 + tanh u
    keeps at least ~1e-6 of 1, so its float64 value is good to ~1e-10."""
    torch = pytest.importorskip("torch")
    y = np.linspace(-4.0, 16.0, 200001).astype(np.float32)
    got = O.gelu_tanh_f32(y).astype(np.float64)
    ref = torch.nn.functional.gelu(torch.from_numpy(y.astype(np.float64)), approximate="tanh").numpy()
    nz = np.abs(ref) > 1e-30
    assert np.max(np.abs(got[nz] - ref[nz]) / np.abs(ref[nz])) < 2e-5


def test_gelu_f32_special_values():
    g = O.gelu_tanh_f32
    assert g(np.float32(0.0)) == 0 and not np.signbit(g(np.float32(0.0)))
    assert g(np.float32(-0.0)) == 0 and np.signbit(g(np.float32(-0.0)))
    big = np.array([10.0, 11.5, 100.0, 3e38], np.float32)
    assert np.array_equal(g(big), big)                     # e^(-2u) below 2^-126
    neg = np.array([-11.0, -50.0, -3e38], np.float32)
    out = g(neg)
    assert np.all(out == 0) and np.all(np.signbit(out))    # below 2^-120: flushed
    # odd part: gelu(y) - gelu(-y) = y
    y = np.linspace(-6.0, 6.0, 1201).astype(np.float32)
    diff = g(y).astype(np.float64) - g(-y).astype(np.float64)
    assert np.max(np.abs(diff - y) / np.maximum(np.abs(y), 1.0)) < 3e-6


def test_gelu_bf16_glue_is_the_rounded_exact_value():
    """Every finite bf16 input: the glue's bf16 output is the exact GELU
    rounded to nearest bf16, except where the exact value sits within the
    float32 evaluation's error (2e-5 relative) of a rounding boundary."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        x = F.bf16_bits_to_f64(bits)
    bits = bits[np.isfinite(x) & (np.abs(x) <= 20.0) & (x != 0)]   # zeros: special values
    x = F.bf16_bits_to_f64(bits)
    out = O.gelu_bf16(bits)
    ref = np.array([_gelu_exact(v) for v in x])
    ref_bits = F.f64_to_bf16_bits(ref)
    # true values below 2^-120 may come out as a zero of the input's sign
    flushed = (np.abs(ref) < TINY) & ((out & 0x7FFF) == 0)
    differ = (out != ref_bits) & ~flushed
    # a disagreement is allowed only next to a bf16 rounding boundary
    lo = F.f64_to_bf16_bits(ref * (1 - 2e-5))
    hi = F.f64_to_bf16_bits(ref * (1 + 2e-5))
    near = (lo != ref_bits) | (hi != ref_bits)
    assert not np.any(differ & ~near), x[differ & ~near][:5]
    assert np.count_nonzero(differ) <= 40
