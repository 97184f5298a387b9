"""Pins for the oracle's SVDQuant steps (CPU only).

Each check ties the oracle to the mathematics rather than to itself: hand
values, closed forms (a matrix with a known spectrum), exact invariants,
brute-force loops, and special cases that reduce to plain NVFP4."""
import itertools

import numpy as np
import pytest

import svdq_inputs as SI
from oracle import formats as F
from oracle import svdq as O


def test_smoothing_hand_values():
    cx = np.array([4.0, 0.0, 1.0, 9.0, 2.0], np.float32)
    W = np.zeros((3, 5), np.float32)
    W[0, 0], W[1, 1], W[2, 3], W[0, 4] = -1.0, 2.0, 1.0, 8.0
    W[1, 2] = 0.0                               # column 2 all zero
    s = O.smoothing_factors(cx, W, 0.5)
    # lambda = sqrt(cx / wmax): 2, guard 1, guard 1, 3, 0.5
    expect = np.array([0.5, 1.0, 1.0, np.float32(1.0 / 3.0), 2.0], np.float32)
    assert np.array_equal(s, expect)


def test_smoothing_is_exact_in_float64():
    """X_hat W~^T equals X W^T up to the one float32 rounding of x_hat."""
    X, W, _ = SI.random_layer(7, 32, 128, 48)
    cx = SI.channel_absmax(X)
    s = O.smoothing_factors(cx, W)
    xh = O.smooth_activation(X, s).astype(np.float64)
    Wt = O.smooth_weight(W, s)
    lhs = xh @ Wt.T
    rhs = F.bf16_bits_to_f64(X) @ W.astype(np.float64).T
    denom = np.abs(F.bf16_bits_to_f64(X)) @ np.abs(W.astype(np.float64)).T
    assert np.all(np.abs(lhs - rhs) <= 2.0 ** -23 * denom + 1e-300)
    # outlier channels get lambda > 1 (their activations shrink)
    lam = 1.0 / s.astype(np.float64)
    big = np.argsort(cx)[-4:]
    assert np.all(lam[big] > np.median(lam))


def _known_spectrum(N, K, sig, seed=0):
    rng = np.random.default_rng(seed)
    U, _ = np.linalg.qr(rng.standard_normal((N, len(sig))))
    V, _ = np.linalg.qr(rng.standard_normal((K, len(sig))))
    return (U * sig[None, :]) @ V.T


def test_lowrank_closed_form_tail():
    """Eckart-Young: the best rank-r approximation leaves exactly the tail
    energy sqrt(sum_{i>r} sigma_i^2) of a matrix with a known spectrum."""
    sig = np.array([50, 40, 30, 20, 10, 5, 4, 3, 2, 1, 0.5, 0.25], np.float64)
    Wt = _known_spectrum(40, 64, sig)
    for r in (1, 3, 6, 10):
        L1, L2 = O.lowrank_factors(Wt, r, round_bf16=False)
        resid = np.linalg.norm(O.residual64(Wt, L1, L2))
        tail = np.sqrt(np.sum(sig[r:] ** 2))
        assert abs(resid - tail) <= 1e-10 * np.linalg.norm(sig)
        # balanced split: column norms of L1 equal row norms of L2 (= sqrt sigma)
        assert np.allclose(np.linalg.norm(L1, axis=0), np.sqrt(sig[:r]))
        assert np.allclose(np.linalg.norm(L2, axis=1), np.sqrt(sig[:r]))
    # bf16 factors: the tail plus a bf16-sized perturbation of the kept part
    L1b, L2b = O.lowrank_factors(Wt, 6)
    resid_b = np.linalg.norm(O.residual64(Wt, L1b, L2b))
    tail = np.sqrt(np.sum(sig[6:] ** 2))
    assert tail <= resid_b <= 1.01 * tail + 2.0 ** -7 * np.linalg.norm(sig[:6])


def test_residual_invariant_and_full_rank():
    X, W, _ = SI.random_layer(11, 16, 128, 64)
    s = O.smoothing_factors(SI.channel_absmax(X), W)
    Wt = O.smooth_weight(W, s)
    L1, L2 = O.lowrank_factors(Wt, 16)
    R64 = O.residual64(Wt, L1, L2)
    recon = O.lowrank_product_t(L1, L2) + R64
    assert np.linalg.norm(Wt - recon) <= 1e-12 * np.linalg.norm(Wt)
    # full rank with unrounded factors: nothing is left for the 4-bit part
    L1f, L2f = O.lowrank_factors(Wt, 64, round_bf16=False)
    assert np.linalg.norm(O.residual64(Wt, L1f, L2f)) <= 1e-12 * np.linalg.norm(Wt)
    # the float32 residual is the float64 one rounded once
    assert np.array_equal(O.residual(Wt, L1, L2), R64.astype(np.float32))


def test_dequant_gemm_brute_force():
    """The vectorized dequantize-then-matmul equals a triple loop over
    (m, n, k) that decodes every code and scale on its own."""
    rng = np.random.default_rng(2)
    for (M, N, K) in [(3, 5, 64), (4, 2, 128), (2, 3, 256)]:
        cx = rng.integers(0, 16, (M, K)).astype(np.uint8)
        cw = rng.integers(0, 16, (N, K)).astype(np.uint8)
        sx = rng.integers(0, 127, (M, K // 16)).astype(np.uint8)
        sw = rng.integers(0, 127, (N, K // 16)).astype(np.uint8)
        fast = O.nvfp4_dequantize(cx, sx) @ O.nvfp4_dequantize(cw, sw).T
        for m, n in itertools.product(range(M), range(N)):
            acc = 0.0
            for k in range(K):
                a = float(F.e2m1_decode(cx[m, k])) * float(F.e4m3_decode(sx[m, k // 16]))
                b = float(F.e2m1_decode(cw[n, k])) * float(F.e4m3_decode(sw[n, k // 16]))
                acc += a * b
            assert abs(fast[m, n] - acc) <= 1e-15 * max(1.0, abs(acc))


def test_r0_unit_smoothing_is_plain_nvfp4():
    """With r = 0 and lambda = 1 the layer is plain W4A4 NVFP4."""
    rng = np.random.default_rng(4)
    M, K, N = 8, 64, 16
    x = rng.standard_normal((M, K)).astype(np.float32)
    X = SI.f32_to_bf16_bits(x)
    W = (rng.standard_normal((N, K)) * 0.1).astype(np.float32)
    wmax = np.abs(W).max(axis=0)
    cx = wmax.copy()                                  # cx == wmax -> lambda = 1
    p = O.pack(W, cx, 0)
    assert np.all(p.s == 1.0)
    Y, _, _, _ = O.linear_reference(X, p)
    xf = F.bf16_bits_to_f64(X).astype(np.float32)
    gx = O.tensor_encode_scale(np.abs(cx).max())
    cxq, sxq = O.nvfp4_quantize(xf, np.abs(cx).max())
    gw = O.tensor_encode_scale(np.abs(W).max())
    cwq, swq = O.nvfp4_quantize(W, np.abs(W).max())
    D = O.nvfp4_dequantize(cxq, sxq) @ O.nvfp4_dequantize(cwq, swq).T
    assert np.array_equal(Y, D / (np.float64(gx) * np.float64(gw)))


def test_zero_input_gives_bias():
    X, W, b = SI.random_layer(5, 4, 64, 32)
    p = O.pack(W, SI.channel_absmax(X), 16)
    Y, cx, _, xl1 = O.linear_reference(np.zeros_like(X), p, b)
    assert np.array_equal(Y, np.broadcast_to(F.bf16_bits_to_f64(b), Y.shape))
    assert np.all((cx & 7) == 0) and np.all(xl1 == 0)


def test_static_activation_scale_equals_runtime_max():
    X, W, _ = SI.random_layer(9, 64, 256, 32)
    cx = SI.channel_absmax(X)
    s = O.smoothing_factors(cx, W)
    runtime = np.abs(O.smooth_activation(X, s)).max()
    assert O.activation_tensor_scale(cx, s) == O.tensor_encode_scale(runtime)


def test_layer_approximates_exact_linear():
    """The whole W4A4 + low-rank layer approximates the exact float64
    X W^T + b, and the low-rank branch is what makes it good: a dropped or
    sign-flipped term, or a transposed operand, breaks this."""
    wl = SI.make_workload("single_256", M=64)
    X, lt = wl.X_bf16, wl.layers[0]
    W, b = lt.W, lt.bias_bf16
    cx = SI.channel_absmax(X)
    exact = F.bf16_bits_to_f64(X) @ W.astype(np.float64).T + F.bf16_bits_to_f64(b)[None, :]
    err = {}
    for r in (0, 32):
        p = O.pack(W, cx, r)
        Y, _, _, _ = O.linear_reference(X, p, b)
        err[r] = np.linalg.norm(Y - exact) / np.linalg.norm(exact)
    assert err[32] < 0.15
    assert err[32] < 0.8 * err[0]
