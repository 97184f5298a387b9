"""Host pack (svdq_pack_weight, C++) against the oracle (CPU only).

Bit-exact: smoothing factors, the activation and weight tensor scales, the
E2M1 codes and E4M3 scales of the residual (the oracle recomputes R from its
own smoothed weight and the library's stored low-rank factors, reading R2).
Quality: the library's randomized SVD against the optimal tail energy, and
the hi/lo kernel operands against their definition."""
import numpy as np
import pytest

import svdq_inputs as SI
import w4a4_rank_corrected_b200 as S
from oracle import formats as F
from oracle import svdq as O


def _check_pack(W, cx, r, svd_quality=True):
    p = S.svdq_pack_weight(W, cx, r)
    s = O.smoothing_factors(cx, W)
    assert np.array_equal(p.smooth, s)
    assert np.float32(p.g_x) == O.activation_tensor_scale(cx, s)
    assert np.float32(p.amax_x) == O.activation_absmax(cx, s)
    assert np.float32(p.gs_x) == O.block_scale_factor(O.activation_absmax(cx, s))
    R, A_w, codes, sf = O.quantize_weight(W, p.smooth, p.l1, p.l2)
    assert np.float32(p.amax_w) == A_w
    assert np.float32(p.g_w) == O.tensor_encode_scale(A_w)
    assert np.array_equal(p.codes_w, O.pack_nibbles(codes))
    assert np.array_equal(p.sf_w, O.sf_to_mma_tiles(sf, row_multiple=256))
    assert np.float32(p.lr_scale) == np.float32(np.float32(p.g_x) * np.float32(p.g_w))
    assert np.float32(p.alpha) == np.float32(np.float32(1.0) / np.float32(p.lr_scale))
    if r == 0:
        return p
    # kernel operands: hi + lo of smooth * L1 (transposed), L2 twice
    L1 = F.bf16_bits_to_f64(p.l1)
    target = (p.smooth.astype(np.float64)[:, None] * L1).T          # [r, K]
    hi = F.bf16_bits_to_f64(p.l1_mma[:r])
    lo = F.bf16_bits_to_f64(p.l1_mma[r:2 * r])
    assert np.array_equal(p.l1_mma[:r], F.f64_to_bf16_bits(target))
    assert np.all(np.abs(hi + lo - target) <= 2.0 ** -16 * np.abs(target) + 1e-38)
    assert np.array_equal(p.l2_mma[:, :r], p.l2.T)
    assert np.array_equal(p.l2_mma[:, r:2 * r], p.l2.T)
    assert np.all(p.l2_mma[:, 2 * r:] == 0)
    if svd_quality:
        Wt = O.smooth_weight(W, s)
        sig = np.linalg.svd(Wt, compute_uv=False)
        tail = np.sqrt(np.sum(sig[r:] ** 2))
        resid = np.linalg.norm(O.residual64(Wt, p.l1, p.l2))
        slack = 2.0 ** -7 * np.sqrt(np.sum(sig[:r] ** 2))
        assert tail <= resid + 1e-9 * tail
        assert resid <= 1.01 * tail + slack, (resid, tail)
        # the kept part captures the outlier energy: far below the r=0 error
        assert resid < 0.9 * np.linalg.norm(Wt)
    return p


@pytest.mark.parametrize("N,K,r,seed", [(48, 192, 16, 1), (272, 320, 32, 2), (64, 128, 64, 3),
                                        (256, 256, 0, 4), (128, 1024, 128, 5)])
def test_pack_ragged_shapes(N, K, r, seed):
    X, W, _ = SI.random_layer(seed, 40, K, N)
    _check_pack(W, SI.channel_absmax(X), r)


def test_pack_single_256_workload():
    wl = SI.make_workload("single_256")
    _check_pack(wl.layers[0].W, SI.channel_absmax(wl.X_bf16), 32)


def test_pack_full_rank_leaves_little():
    """r = min(N, K): only the bf16 rounding of the factors is left."""
    X, W, _ = SI.random_layer(6, 16, 64, 32)
    cx = SI.channel_absmax(X)
    p = S.svdq_pack_weight(W, cx, 32)
    Wt = O.smooth_weight(W, p.smooth)
    resid = np.linalg.norm(O.residual64(Wt, p.l1, p.l2))
    assert resid <= 2.0 ** -7 * np.linalg.norm(Wt)


def test_pack_is_deterministic():
    X, W, _ = SI.random_layer(8, 16, 256, 96)
    cx = SI.channel_absmax(X)
    a = S.svdq_pack_weight(W, cx, 32, seed=3)
    b = S.svdq_pack_weight(W, cx, 32, seed=3)
    for f in ("smooth", "l1", "l2", "codes_w", "sf_w", "l1_mma", "l2_mma"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f


def test_pack_balanced_sqrt_sigma_split():
    """Reading R2: L1 = V sqrt(S), L2 = sqrt(S) U^T.  So the i-th column of L1
    and the i-th row of L2 both have norm sqrt(sigma_i) (V, U orthonormal),
    and L1^T L1 = L2 L2^T = diag(sigma), up to the bf16 rounding of the
    factors and the randomized SVD's accuracy.  A pack that put all of S into
    one factor (column norms 1 on the other) fails."""
    X, W, _ = SI.random_layer(12, 64, 512, 384)
    cx = SI.channel_absmax(X)
    r = 32
    p = S.svdq_pack_weight(W, cx, r)
    L1 = F.bf16_bits_to_f64(p.l1)
    L2 = F.bf16_bits_to_f64(p.l2)
    sig = np.linalg.svd(O.smooth_weight(W, p.smooth), compute_uv=False)[:r]
    c1 = np.linalg.norm(L1, axis=0)
    r2 = np.linalg.norm(L2, axis=1)
    assert np.allclose(c1, r2, rtol=2.0 ** -7), np.max(np.abs(c1 / r2 - 1))
    # (the randomized SVD resolves the near-degenerate tail of the spectrum
    # to about 1 %, so each sigma_i gets 2 % and their sum 1 %)
    assert np.allclose(c1 ** 2, sig, rtol=2e-2)
    assert abs((c1 ** 2).sum() / sig.sum() - 1) <= 1e-2
    G1, G2 = L1.T @ L1, L2 @ L2.T
    off = ~np.eye(r, dtype=bool)
    assert np.max(np.abs(G1[off])) <= 2e-2 * sig[0]
    assert np.max(np.abs(G2[off])) <= 2e-2 * sig[0]


def test_pack_carries_bias():
    X, W, b = SI.random_layer(13, 16, 128, 64)
    cx = SI.channel_absmax(X)
    p = S.svdq_pack_weight(W, cx, 16, bias_bf16=b)
    assert np.array_equal(p.bias, b)
    q = S.svdq_pack_weight(W, cx, 16)
    assert q.bias is None
    # the rest of the pack does not depend on the bias
    for f in ("smooth", "l1", "l2", "codes_w", "sf_w"):
        assert np.array_equal(getattr(p, f), getattr(q, f)), f
