"""Pins for the oracle's number formats (CPU only).

Each check compares the oracle against something other than itself: an
independent library conversion (ml_dtypes float4_e2m1fn, torch
float8_e4m3fn), exact rational brute force, or hand-worked fixtures."""
import json
import os
import random

import numpy as np
import pytest

from oracle import formats as F
from oracle import svdq as O


def _dense_f32_sweep(lo_exp=-12, hi_exp=4, per_binade=4096, seed=0):
    """Every float32 with few mantissa bits plus random ones, both signs,
    across the binades [2^lo_exp, 2^hi_exp), and exact zeros."""
    rng = np.random.default_rng(seed)
    vals = [0.0, -0.0]
    for e in range(lo_exp, hi_exp):
        m = np.arange(0, 1 << 10) / (1 << 10)           # 10-bit grid: hits every tie
        vals.extend(((1 + m) * 2.0 ** e).tolist())
        vals.extend(((1 + rng.random(per_binade)) * 2.0 ** e).tolist())
    v = np.array(vals, dtype=np.float32)
    return np.concatenate([v, -v])


def test_e2m1_decode_matches_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml.float4_e2m1fn).astype(np.float64)
    got = F.e2m1_decode(codes)
    assert np.array_equal(np.signbit(ref), np.signbit(got))
    assert np.array_equal(ref, got)


def test_e2m1_encode_matches_ml_dtypes():
    ml = pytest.importorskip("ml_dtypes")
    v = _dense_f32_sweep()
    v = np.concatenate([v, np.array([7.0, 100.0, 1e30, -1e30, 5.999, 6.001], np.float32)])
    ref = v.astype(ml.float4_e2m1fn).view(np.uint8) & 0xF
    got = F.e2m1_encode(v)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, (v[bad[:5]], ref[bad[:5]], got[bad[:5]])


def test_e2m1_round_trip_all_codes():
    codes = np.arange(16, dtype=np.uint8)
    vals = F.e2m1_decode(codes).astype(np.float32)
    back = F.e2m1_encode(vals)
    assert np.array_equal(back, codes)          # +0 and -0 stay distinct


def test_e2m1_tie_table():
    ties = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}
    for x, code in ties.items():
        assert F.e2m1_encode(np.float32(x)) == code
        assert F.e2m1_encode(np.float32(-x)) == code | 8


def test_e4m3_decode_matches_torch():
    torch = pytest.importorskip("torch")
    codes = torch.arange(127, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(ref, F.e4m3_decode(np.arange(127)))
    assert F.E4M3_VALUES.max() == 448.0


def test_e4m3_encode_matches_torch_below_saturation():
    torch = pytest.importorskip("torch")
    v = _dense_f32_sweep(lo_exp=-14, hi_exp=9)
    v = np.abs(v)
    v = v[v < 464.0]                    # torch's cast is non-saturating above
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = F.e4m3_encode_nonneg(v)
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, (v[bad[:5]], ref[bad[:5]], got[bad[:5]])


def test_e4m3_satfinite_and_round_trip():
    big = np.array([448.0, 463.99, 464.0, 479.0, 500.0, 1e6, 3e38], np.float32)
    assert np.all(F.e4m3_encode_nonneg(big) == 126)
    codes = np.arange(127)
    assert np.array_equal(F.e4m3_encode_nonneg(F.e4m3_decode(codes).astype(np.float32)), codes)


def test_bf16_from_f64_brute_force():
    rnd = random.Random(1)
    xs = []
    for _ in range(3000):
        m = rnd.random() + 1.0
        e = rnd.randint(-40, 40)
        xs.append(rnd.choice([-1, 1]) * m * 2.0 ** e)
    # exact ties and near-ties at bf16 precision
    for k in range(200):
        base = (1 + k / 128.0) * 2.0 ** rnd.randint(-20, 20)
        half = 2.0 ** -8 * 2.0 ** np.floor(np.log2(base))
        xs.extend([base + half, base + half * (1 + 2 ** -40), base + half * (1 - 2 ** -40)])
    # the subnormal range and its edge: ties and near-ties of the 2^-133 grid
    for k in range(300):
        n = rnd.randint(0, 130)
        xs.extend([(n + 0.5) * 2.0 ** -133, (n + 0.5 + 2 ** -30) * 2.0 ** -133,
                   (n + rnd.random()) * 2.0 ** -133, -(n + rnd.random()) * 2.0 ** -133])
    xs.extend([2.0 ** -126, 2.0 ** -126 * (1 - 2 ** -9), 2.0 ** -134, 2.0 ** -135, 1e-300])
    x = np.array(xs, np.float64)
    got = F.bf16_bits_to_f64(F.f64_to_bf16_bits(x))
    for xi, gi in zip(x, got):
        assert float(F.bf16_round_exact(float(xi))) == gi, xi


def test_bf16_from_f32_matches_torch_including_subnormals():
    """An independent conversion: torch's float32 -> bfloat16 (round to
    nearest even, with subnormals), on every float32 with a 16-bit
    significand prefix near each binade edge plus the whole subnormal
    range's grid points and ties."""
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(4)
    hi = rng.integers(0, 1 << 16, 20000, dtype=np.uint32)
    lo = np.array([0, 0x7FFF, 0x8000, 0x8001, 0xFFFF], np.uint32)
    bits = (hi[:, None] << 16 | lo[None, :]).reshape(-1)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = F.f64_to_bf16_bits(f.astype(np.float64))
    bad = np.nonzero(ref != got)[0]
    assert bad.size == 0, (f[bad[:5]], ref[bad[:5]], got[bad[:5]])


def _load_golden(golden_dir):
    with open(os.path.join(golden_dir, "nvfp4_worked_examples.json")) as f:
        return json.load(f)


def test_nvfp4_hand_worked_groups(golden_dir):
    gold = _load_golden(golden_dir)
    for ex in gold["groups"]:
        t = np.array(ex["t"], np.float32)[None, :]
        codes, sf = O.nvfp4_quantize(t, np.float32(ex["amax"]))
        assert int(sf[0, 0]) == ex["sf"], ex["name"]
        assert codes[0].tolist() == ex["codes"], ex["name"]


def test_nvfp4_hand_worked_tensor_scales(golden_dir):
    gold = _load_golden(golden_dir)
    for ex in gold["tensor_scales"]:
        assert O.tensor_encode_scale(np.float32(ex["amax"])) == np.float32(ex["g"])
        assert O.block_scale_factor(np.float32(ex["amax"])) == np.float32(ex["gs"])


def test_nvfp4_error_bound_random():
    """|v - e2m1(code)| is at most half the E2M1 spacing at |v| (0.25 below
    2, 0.5 below 4, 1 below 6), plus the saturation excess above 6, where
    v = t * q is the scaled value of reading R4."""
    rng = np.random.default_rng(3)
    T = (rng.standard_normal((64, 256)) * np.exp(rng.standard_normal((64, 1)) * 3)).astype(np.float32)
    A = np.abs(T).max()
    g = O.tensor_encode_scale(A)
    codes, sf = O.nvfp4_quantize(T, A)
    dec = F.e4m3_decode(sf).astype(np.float32)
    q = np.where(sf == 0, 0, g / np.where(sf == 0, 1, dec)).astype(np.float32)
    v = (T.reshape(64, 16, 16) * q[:, :, None]).astype(np.float64).reshape(64, 256)
    err = np.abs(v - F.e2m1_decode(codes))
    av = np.abs(v)
    bound = np.where(av <= 2, 0.25, np.where(av <= 4, 0.5, 1.0)) + np.maximum(av - 6, 0)
    assert np.all(err <= bound + 1e-12)
    # the group maximum lands within one E4M3 rounding of 6: a normal
    # (unsaturated) scale is within 2^-4 relative of a*gs = a*g/6 (up to
    # float32 rounding), so v_max = a g / sf lies in [6/(1+2^-4), 6/(1-2^-4)]
    vmax = av.reshape(64, 16, 16).max(axis=2)
    normal = (sf > 8) & (sf < 126)      # code 8 may be reached from a subnormal y
    assert normal.sum() > 500
    assert np.all(vmax[normal] <= 6 / (1 - 2.0 ** -4) + 1e-6)
    assert np.all(vmax[normal] >= 6 / (1 + 2.0 ** -4) - 1e-6)


def test_pack_nibbles_low_nibble_even():
    codes = np.array([[1, 2, 3, 4, 15, 0]], np.uint8)
    packed = O.pack_nibbles(codes)
    assert packed.tolist() == [[0x21, 0x43, 0x0F]]
    assert np.array_equal(O.unpack_nibbles(packed), codes)


def test_sf_tile_layout_properties():
    rng = np.random.default_rng(5)
    rows, K = 300, 256
    sf = rng.integers(0, 127, (rows, K // 16)).astype(np.uint8)
    t = O.sf_to_mma_tiles(sf)
    assert t.size == 384 * (K // 16)                    # rows padded to 128
    assert np.array_equal(O.sf_from_mma_tiles(t, rows, K), sf)
    # bijection on the padded index space: tag every (row, scale) uniquely
    tags = np.arange(384 * 16, dtype=np.int64).reshape(384, 16)
    lo = O.sf_to_mma_tiles((tags % 251).astype(np.uint8))
    assert sorted(np.unique(lo).tolist()) == sorted(np.unique(tags % 251).tolist())
    # each row's 4 scales of one 64-wide k block are one aligned 32-bit word
    words = t.reshape(-1, 4)
    row0 = sf[0, 0:4]
    assert any(np.array_equal(w, row0) for w in words[:128])
    # padding rows are zero
    t2 = O.sf_to_mma_tiles(np.full((1, 4), 7, np.uint8))
    assert (t2 != 0).sum() == 4
