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


def check_activation(codes_dev, sf_dev, xl1_dev, X_bits, op, M, K, r, rows=None,
                     chunk_rows=2048):
    """Bit-exact codes and scales; xl1 hi+lo against lr_scale * X_hat L1.
    With rows=None every row is compared (in chunks of rows, to bound the
    oracle's memory), and the whole scale-tile buffer, padding rows
    included, must equal the oracle's tiles."""
    torch = torch_mod()
    codes_all = codes_dev.cpu().numpy()
    tiles = sf_dev.cpu().numpy()
    got_sf_all = O.sf_from_mma_tiles(tiles, M, K)
    xl_all = from_dev_bf16(xl1_dev) if r else None
    lr_scale = np.float64(np.float32(op.g_x) * np.float32(op.g_w))
    L1 = F.bf16_bits_to_f64(op.L1) if r else None
    if rows is None:
        blocks = [np.arange(a, min(M, a + chunk_rows)) for a in range(0, M, chunk_rows)]
        sf_full = np.zeros((M, K // 16), np.uint8)
    else:
        blocks = [np.asarray(rows)]
        sf_full = None
    for idx in blocks:
        xh, codes, sf = O.quantize_activation(X_bits[idx], op.s, op.A_x)
        assert np.array_equal(codes_all[idx], O.pack_nibbles(codes)), \
            f"activation codes differ in rows {idx[0]}..{idx[-1]}"
        assert np.array_equal(got_sf_all[idx], sf), \
            f"activation scales differ in rows {idx[0]}..{idx[-1]}"
        if sf_full is not None:
            sf_full[idx] = sf
        if r:
            want = O.lowrank_down(xh, op.L1) * lr_scale
            xl = xl_all[idx]
            hi = F.bf16_bits_to_f64(xl[:, :r])
            lo = F.bf16_bits_to_f64(xl[:, r:2 * r])
            scale = (np.abs(xh.astype(np.float64)) @ np.abs(L1)) * lr_scale
            err = np.abs(hi + lo - want)
            assert np.all(err <= 2e-5 * scale + 1e-30), float((err / (scale + 1e-30)).max())
            assert np.all(xl[:, 2 * r:] == 0)
    if sf_full is not None:  # the whole tile buffer, padding rows (zero scales) included
        exp = O.sf_to_mma_tiles(sf_full)
        assert tiles.size >= exp.size
        assert np.array_equal(tiles[:exp.size], exp), "scale tiles differ"


def rows_every_block(M, per_block=1, extra=64, seed=0, block=128):
    """Row indices with at least `per_block` rows in every `block`-row block
    (so every GEMM row tile and activation row block is looked at), plus
    `extra` random rows and the first and last row."""
    rng = np.random.default_rng(seed)
    pick = [0, M - 1]
    for b0 in range(0, M, block):
        n = min(block, M - b0)
        pick.extend((b0 + rng.choice(n, size=min(per_block, n), replace=False)).tolist())
    pick.extend(rng.choice(M, size=min(extra, M), replace=False).tolist())
    return np.unique(np.array(pick))


def rows_sample(M, n=64, seed=0):
    rng = np.random.default_rng(seed)
    pick = rng.choice(M, size=min(n, M), replace=False)
    return np.unique(np.concatenate([pick, [0, M - 1]]))
