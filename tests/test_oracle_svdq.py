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


# ------------------------------- dynamic per-token activation scale (R5d) ----

def _rows_with_common_max(seed, M, K):
    """bf16 X whose column 0 holds the same large value in every row, so
    every row of x_hat reaches the batch maximum there."""
    rng = np.random.default_rng(seed)
    x = rng.uniform(-1.0, 1.0, (M, K)).astype(np.float32)
    x[:, 0] = 64.0
    s = rng.uniform(0.5, 2.0, K).astype(np.float32)
    return SI.f32_to_bf16_bits(x), s


def test_dynamic_scale_reduces_to_static_when_row_max_is_batch_max():
    """If every row's absmax equals the static (calibration) absmax, R5d and
    R5 quantize identically."""
    X, s = _rows_with_common_max(11, 12, 128)
    xh = O.smooth_activation(X, s)
    A_static = O.activation_absmax(SI.channel_absmax(X), s)
    assert np.all(O.activation_absmax_rows(xh) == A_static)
    _, c_st, sf_st = O.quantize_activation(X, s, A_static)
    _, c_dy, sf_dy, _ = O.quantize_activation_dynamic(X, s)
    assert np.array_equal(c_st, c_dy) and np.array_equal(sf_st, sf_dy)


def test_dynamic_scale_is_per_row_and_power_of_two_invariant():
    """Scaling one row by 2^k (exact in bf16 and fp32) leaves its codes and
    scales unchanged, scales its A_m by 2^k, leaves every other row alone, and
    scales that row of Y - bias by exactly 2^k."""
    X, W, b = SI.random_layer(12, 16, 128, 32)
    p = O.pack(W, SI.channel_absmax(X), 16)
    Y0, c0, s0, _, A0 = O.linear_reference_dynamic(X, p, b)
    bias = F.bf16_bits_to_f64(b)[None, :]
    for m, k in ((3, 5), (7, -3)):
        x = SI.bf16_bits_to_f32(X).copy()
        x[m] *= np.float32(2.0 ** k)
        X2 = SI.f32_to_bf16_bits(x)
        Y2, c2, s2, _, A2 = O.linear_reference_dynamic(X2, p, b)
        assert np.array_equal(c2, c0) and np.array_equal(s2, s0)
        assert A2[m] == A0[m] * np.float32(2.0 ** k)
        others = np.arange(16) != m
        assert np.array_equal(A2[others], A0[others])
        assert np.array_equal(Y2[others], Y0[others])
        np.testing.assert_allclose(Y2[m] - bias[0], (2.0 ** k) * (Y0[m] - bias[0]),
                                   rtol=1e-12, atol=1e-12 * np.abs(Y0[m]).max())


def test_dynamic_scale_row_max_takes_the_top_code():
    """The element at a row's maximum lands on E2M1 +-6 with block scale
    E4M3 448: the per-row scale uses the whole 4-bit range."""
    X, W, _ = SI.random_layer(13, 24, 256, 16)
    s = O.smoothing_factors(SI.channel_absmax(X), W)
    xh, codes, sf, A = O.quantize_activation_dynamic(X, s)
    for m in range(xh.shape[0]):
        k = int(np.argmax(np.abs(xh[m])))
        assert abs(float(F.e2m1_decode(codes[m, k]))) == 6.0
        assert float(F.e4m3_decode(sf[m, k // 16])) == 448.0
        assert A[m] == np.abs(xh[m, k])


def test_dynamic_scale_zero_row():
    X, W, b = SI.random_layer(14, 6, 64, 16)
    X = X.copy()
    X[2] = 0
    p = O.pack(W, SI.channel_absmax(X), 16)
    Y, cx, sfx, xl1, A = O.linear_reference_dynamic(X, p, b)
    assert A[2] == 0 and np.all(cx[2] == 0) and np.all(sfx[2] == 0) and np.all(xl1[2] == 0)
    assert np.array_equal(Y[2], F.bf16_bits_to_f64(b))


def test_dynamic_scale_beats_static_outside_calibration():
    """Inputs 16x beyond the calibration range saturate the static scale;
    the per-row scale tracks them."""
    wl = SI.make_workload("single_256", M=64)
    X, lt = wl.X_bf16, wl.layers[0]
    W, b = lt.W, lt.bias_bf16
    p = O.pack(W, SI.channel_absmax(X), 32)
    Xbig = SI.f32_to_bf16_bits(SI.bf16_bits_to_f32(X) * np.float32(16.0))
    exact = F.bf16_bits_to_f64(Xbig) @ W.astype(np.float64).T + F.bf16_bits_to_f64(b)[None, :]
    Ys, _, _, _ = O.linear_reference(Xbig, p, b)
    Yd, _, _, _, _ = O.linear_reference_dynamic(Xbig, p, b)
    es = np.linalg.norm(Ys - exact) / np.linalg.norm(exact)
    ed = np.linalg.norm(Yd - exact) / np.linalg.norm(exact)
    assert ed < 0.15 and ed < 0.5 * es
