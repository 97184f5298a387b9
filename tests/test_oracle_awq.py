"""Pins for the AWQ W4A16 oracle (oracle/awq.py), CPU only: the fp16
rounding against exact-rational brute force and torch's conversion,
hand-worked groups (tests/golden/awq_worked_examples.json), the rounding
against a brute-force nearest-level search, the error bound, and the layer
against a brute-force triple loop."""
import json
import os
import random
from fractions import Fraction

import numpy as np
import pytest

from oracle import awq as A
from oracle import formats as F


def _fp16_exact(x: float) -> Fraction:
    """Nearest binary16 value to x (ties to even; subnormals 2^-24 apart)."""
    fx = Fraction(x)
    if fx == 0:
        return Fraction(0)
    s = -1 if fx < 0 else 1
    a = abs(fx)
    if a < Fraction(2) ** -14:
        step = Fraction(2) ** -24
    else:
        e = 0
        t = a
        while t >= 2:
            t /= 2
            e += 1
        while t < 1:
            t *= 2
            e -= 1
        step = Fraction(2) ** (e - 10)
    n = a / step
    lo = int(n)
    frac = n - lo
    if frac > Fraction(1, 2) or (frac == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    return s * lo * step


def test_fp16_round_brute_force_and_torch():
    rnd = random.Random(3)
    xs = [rnd.uniform(-1, 1) * 2.0 ** rnd.randint(-27, 14) for _ in range(3000)]
    xs += [(k + 0.5) * 2.0 ** -24 for k in range(40)] + [(1 + (k + 0.5) / 1024) for k in range(40)]
    x = np.array(xs)
    got = A.fp16_round(x)
    for xi, gi in zip(x, got):
        assert float(_fp16_exact(float(xi))) == gi, xi
    torch = pytest.importorskip("torch")
    f = x.astype(np.float32)
    ref = torch.from_numpy(f).to(torch.float16).to(torch.float64).numpy()
    # float32 inputs: one rounding either way
    assert np.array_equal(A.fp16_round(f.astype(np.float64)), ref)


def test_awq_hand_worked_groups(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "awq_worked_examples.json")))
    for case in g["cases"]:
        W = np.array([case["w"]], np.float32)
        q, z, sb = A.awq_quantize(W, group=g["group"])
        assert int(sb[0, 0]) == case["scale_f16_bits"], case
        assert int(z[0, 0]) == case["z"], case
        assert q[0].tolist() == case["q"], case


def test_awq_codes_are_the_nearest_level():
    """For weights inside the representable range, the code is the level
    (q - z) scale nearest to w (brute force over the 16 levels)."""
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((16, 256)) * 0.02).astype(np.float32)
    W[3, :128] = 0.01          # a constant group
    W[5, 128:] = 0.0           # an all-zero group
    q, z, sb = A.awq_quantize(W)
    scale = sb.view(np.float16).astype(np.float64)
    for n in range(16):
        for gi in range(2):
            levels = (np.arange(16) - float(z[n, gi])) * scale[n, gi]
            w = W[n, gi * 128:(gi + 1) * 128].astype(np.float64)
            inside = (w >= levels[0]) & (w <= levels[-1])
            best = np.argmin(np.abs(w[:, None] - levels[None, :]), axis=1)
            dist_best = np.abs(w - levels[best])
            dist_got = np.abs(w - levels[q[n, gi * 128:(gi + 1) * 128]])
            assert np.all(dist_got[inside] <= dist_best[inside] + 1e-15)


def test_awq_error_bound_and_exact_zero():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((32, 512)) * 0.05).astype(np.float32)
    W[0, :128] = 0.0
    q, z, sb = A.awq_quantize(W)
    deq = A.awq_dequantize(q, z, sb)
    scale = np.repeat(sb.view(np.float16).astype(np.float64), 128, axis=1)
    # the range and the zero point are rounded, so a weight can sit up to
    # one step from its level at the ends; inside, half a step
    assert np.all(np.abs(deq - W) <= scale * 1.0 + 1e-12)
    assert np.mean(np.abs(deq - W) <= scale * 0.5 + 1e-12) > 0.99
    assert np.all(deq[0, :128] == 0.0)           # zero is exactly representable


def test_awq_layer_against_triple_loop():
    rng = np.random.default_rng(2)
    M, K, N = 3, 256, 5
    X = F.f64_to_bf16_bits(rng.standard_normal((M, K)))
    W = (rng.standard_normal((N, K)) * 0.03).astype(np.float32)
    b = F.f64_to_bf16_bits(rng.standard_normal(N) * 0.01)
    q, z, sb = A.awq_quantize(W)
    Y = A.awq_linear_reference(X, q, z, sb, b)
    x = F.bf16_bits_to_f64(X)
    scale = sb.view(np.float16).astype(np.float64)
    for m in range(M):
        for n in range(N):
            acc = 0.0
            for k in range(K):
                acc += x[m, k] * (float(q[n, k]) - float(z[n, k // 128])) * scale[n, k // 128]
            acc += float(F.bf16_bits_to_f64(b)[n])
            assert abs(Y[m, n] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_awq_nibble_order():
    q = np.array([[1, 2, 3, 4]], np.uint8)
    assert A.pack_nibbles_awq(q).tolist() == [[0x21, 0x43]]
