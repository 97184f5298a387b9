"""Shared helpers of the GPU parity tests (imported only by tests)."""
import numpy as np

import svdq_inputs as SI
from oracle import formats as F
from oracle import svdq as O

TOL_FRO = 2e-3   # relative Frobenius error of the bf16 output vs the float64 oracle


def torch_mod():
    import torch
    return torch


def to_dev_bf16(bits: np.ndarray):
    torch = torch_mod()
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev_bf16(t) -> np.ndarray:
    torch = torch_mod()
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def prepare(W, cx, r, bias=None, seed=0):
    """Library pack (host C++), the oracle pack that takes the library's
    stored low-rank factors as given (the SVD is not unique), and the
    device copy.  The oracle recomputes the residual codes itself; they
    must equal the library's bit for bit."""
    import w4a4_rank_corrected_b200 as S
    lp = S.svdq_pack_weight(W, cx, r, seed=seed)
    if r:
        op = O.pack(W, cx, r, L1=lp.l1, L2=lp.l2)
    else:
        op = O.pack(W, cx, 0)
    assert np.array_equal(lp.smooth, op.s)
    assert np.array_equal(lp.codes_w, O.pack_nibbles(op.codes_w))
    assert np.array_equal(lp.sf_w, O.sf_to_mma_tiles(op.sf_w, row_multiple=256))
    return lp, op, lp.to_device("cuda", bias)


def check_output(Y_bits: np.ndarray, Y_ref: np.ndarray, tol_fro: float = TOL_FRO):
    """rel-Fro <= tol_fro, and per element |Y - Y_ref| <= 1e-2 rms(Y_ref)
    plus half a bf16 ulp (the output format's own rounding)."""
    Y = F.bf16_bits_to_f64(Y_bits)
    fro, maxabs, excess = O.output_errors(Y, Y_ref)
    assert fro <= tol_fro, (fro, maxabs)
    assert excess <= 0.0, (fro, maxabs, excess)
    return fro, maxabs


def check_activation(codes_dev, sf_dev, xl1_dev, X_bits, op, M, K, r, rows=None):
    """Bit-exact codes and scales; xl1 hi+lo against lr_scale * X_hat L1."""
    torch = torch_mod()
    idx = np.arange(M) if rows is None else np.asarray(rows)
    xh, codes, sf = O.quantize_activation(X_bits[idx], op.s, op.A_x)
    got_codes = codes_dev.cpu().numpy()[idx]
    assert np.array_equal(got_codes, O.pack_nibbles(codes)), "activation codes differ"
    tiles = sf_dev.cpu().numpy()
    got_sf = O.sf_from_mma_tiles(tiles, M, K)[idx]
    assert np.array_equal(got_sf, sf), "activation scales differ"
    if rows is None:  # the whole tile buffer, padding rows (zero scales) included
        exp = O.sf_to_mma_tiles(sf)
        assert tiles.size >= exp.size
        assert np.array_equal(tiles[:exp.size], exp), "scale tiles differ"
    if r:
        lr_scale = np.float64(np.float32(op.g_x) * np.float32(op.g_w))
        want = O.lowrank_down(xh, op.L1) * lr_scale
        xl = from_dev_bf16(xl1_dev)[idx]
        hi = F.bf16_bits_to_f64(xl[:, :r])
        lo = F.bf16_bits_to_f64(xl[:, r:2 * r])
        scale = (np.abs(xh.astype(np.float64)) @ np.abs(F.bf16_bits_to_f64(op.L1))) * lr_scale
        err = np.abs(hi + lo - want)
        assert np.all(err <= 2e-5 * scale + 1e-30), float((err / (scale + 1e-30)).max())
        assert np.all(xl[:, 2 * r:] == 0)


def rows_sample(M, n=64, seed=0):
    rng = np.random.default_rng(seed)
    pick = rng.choice(M, size=min(n, M), replace=False)
    return np.unique(np.concatenate([pick, [0, M - 1]]))
