"""Pins for the oracle's tolerance helpers (CPU only).

`bf16_half_ulp` is checked against brute force over every finite bf16
value (the gap between the two neighbours that bracket |y|, halved), and
`output_errors` against planted pairs whose three figures were worked out
by hand.  A slip such as 2**(e-7) for 2**(e-8), or the bound taken at
|Y_ref| instead of max(|Y|, |Y_ref|), fails here."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import formats as F
from oracle import svdq as O


def _bf16_positive_values():
    """Every non-negative finite bf16 value, sorted (exact in float64)."""
    bits = np.arange(0, 0x7F80, dtype=np.uint16)           # +0 .. largest finite
    return np.sort(F.bf16_bits_to_f64(bits))


_VALS = _bf16_positive_values()


def _brute_half_ulp(y: float) -> float:
    """Half the gap [lo, hi) of consecutive bf16 values with lo <= |y| < hi."""
    a = abs(y)
    i = int(np.searchsorted(_VALS, a, side="right")) - 1
    lo, hi = _VALS[i], _VALS[i + 1]
    return float((Fraction(hi) - Fraction(lo)) / 2)


def test_half_ulp_matches_brute_force_across_binades():
    rng = np.random.default_rng(5)
    ys = [0.0, 2.0 ** -140, 2.0 ** -133, 2.0 ** -127, 2.0 ** -126, 3 * 2.0 ** -127, 1.0,
          1.5, 1.9999, 2.0, 3.0, 255.9, 256.0, 1e30, -1.0, -3.75, 2.0 ** 100]
    ys += list(rng.standard_normal(200) * 10.0 ** rng.integers(-30, 30, 200))
    ys += list(2.0 ** rng.integers(-125, 120, 100).astype(np.float64))   # exact powers of two
    got = O.bf16_half_ulp(np.array(ys))
    for y, g in zip(ys, got):
        assert g == _brute_half_ulp(y), (y, g, _brute_half_ulp(y))


def test_half_ulp_hand_values():
    # ulp of bf16 (8 significant bits) at 1 is 2^-7, so half of it is 2^-8
    assert O.bf16_half_ulp(np.array([1.0]))[0] == 2.0 ** -8
    assert O.bf16_half_ulp(np.array([3.5]))[0] == 2.0 ** -7       # binade [2, 4)
    assert O.bf16_half_ulp(np.array([-1000.0]))[0] == 2.0 ** 1    # [512, 1024): ulp 4
    assert O.bf16_half_ulp(np.array([0.0]))[0] == 2.0 ** -134     # subnormal spacing 2^-133


def test_output_errors_planted_pair():
    # Y_ref = [3, 4, 0, 0]: |Y_ref| = 5, rms = sqrt(25 / 4) = 2.5
    Y_ref = np.array([3.0, 4.0, 0.0, 0.0])
    Y = np.array([3.5, 4.0, 0.0, 0.0])                             # one error of 0.5
    fro, maxabs, excess = O.output_errors(Y, Y_ref)
    assert fro == pytest.approx(0.1, abs=1e-15)                    # 0.5 / 5
    assert maxabs == pytest.approx(0.2, abs=1e-15)                 # 0.5 / 2.5
    # bound at element 0: 1e-2 * 2.5 + half ulp at max(3.5, 3) = 2^-7
    assert excess == pytest.approx(0.5 - (0.025 + 2.0 ** -7), abs=1e-15)


def test_output_errors_bound_uses_larger_magnitude():
    # the error sits exactly between the half ulp at |Y_ref| and at |Y|:
    # Y_ref = 1.99 (binade [1, 2): half ulp 2^-8), Y = 2.0 (binade [2, 4): 2^-7)
    Y_ref = np.array([1.99, 0.0, 0.0, 0.0])
    rms = np.sqrt(1.99 ** 2 / 4)
    Y = np.array([1.99 + 1e-2 * rms + 2.0 ** -8 + 2.0 ** -9, 0.0, 0.0, 0.0])
    assert Y[0] >= 2.0
    _, _, excess = O.output_errors(Y, Y_ref)
    # within the bound taken at max(|Y|, |Y_ref|) = |Y| (half ulp 2^-7) ...
    assert excess == pytest.approx(2.0 ** -8 + 2.0 ** -9 - 2.0 ** -7, abs=1e-12)
    assert excess < 0
    # ... and the same error measured against Y_ref's half ulp would exceed it
    assert 2.0 ** -8 + 2.0 ** -9 > 2.0 ** -8


def test_output_errors_exact_output_has_no_excess():
    rng = np.random.default_rng(0)
    Y_ref = rng.standard_normal(1000)
    Y = F.bf16_bits_to_f64(F.f64_to_bf16_bits(Y_ref))             # correctly rounded output
    fro, maxabs, excess = O.output_errors(Y, Y_ref)
    assert excess <= -1e-2 * np.sqrt(np.mean(Y_ref ** 2)) + 1e-18
    assert 1e-3 < fro < 2e-3                                       # bf16 rounding alone


def test_sf_atom_golden_offsets(golden_dir):
    """The oracle's MMA scale-tile layout against hand-derived offsets of the
    documented 512-byte scale-factor atom (tests/golden/sf_atom_offsets.json)."""
    g = json.load(open(os.path.join(golden_dir, "sf_atom_offsets.json")))
    K, rows = g["K"], g["rows"]
    G = K // 16
    r_idx, g_idx = np.meshgrid(np.arange(rows), np.arange(G), indexing="ij")
    tiles_row = O.sf_to_mma_tiles((r_idx & 0x7F).astype(np.uint8))
    tiles_grp = O.sf_to_mma_tiles(g_idx.astype(np.uint8) + 1)
    assert tiles_row.size == 384 * G               # rows padded to 128
    for e in g["entries"]:
        off = e["offset"]
        assert tiles_row[off] == (e["row"] & 0x7F), e
        assert tiles_grp[off] == e["g"] + 1, e
    # the inverse picks the same bytes back
    sf = ((r_idx * 7 + g_idx * 3) % 127).astype(np.uint8)
    tiled = O.sf_to_mma_tiles(sf)
    for e in g["entries"]:
        assert tiled[e["offset"]] == sf[e["row"], e["g"]]
    assert np.array_equal(O.sf_from_mma_tiles(tiled, rows, K), sf)
    # padding rows carry zero scales
    pad = np.ones((rows, G), np.uint8)
    tp = O.sf_to_mma_tiles(pad)
    assert int(tp.sum()) == rows * G

