"""The C ABI on the CPU: the library loads, exports every entry point that
include/svdq.h declares, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import w4a4_rank_corrected_b200 as S
from oracle import svdq as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "svdq.h")


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(svdq_[a-z0-9_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(S.lib, n), n


def test_status_strings_and_version():
    seen = set()
    for code in range(8):
        s = S.svdq_status_string(code)
        assert s and s not in seen
        seen.add(s)
    assert S.lib.svdq_version().startswith(b"svdq-b200")


def test_query_sizes():
    sz = S.svdq_query_sizes(9216, 3072, 32)
    assert (sz.N, sz.K, sz.r, sz.klr) == (9216, 3072, 32, 64)
    assert sz.codes_w_bytes == 9216 * 1536
    assert sz.sf_w_bytes == 9216 * 192
    sz = S.svdq_query_sizes(48, 192, 16)
    assert sz.klr == 64 and sz.sf_w_bytes == 256 * 12
    for bad in [(9216, 3000, 32), (9210, 3072, 32), (9216, 3072, 40), (9216, 3072, 144),
                (0, 64, 0), (32, 64, 48)]:
        with pytest.raises(S.SvdqError) as e:
            S.svdq_query_sizes(*bad)
        assert e.value.status == 1


def test_sf_tile_offset_matches_oracle_layout():
    rng = np.random.default_rng(0)
    rows, K = 300, 512
    sf = rng.integers(0, 127, (rows, K // 16)).astype(np.uint8)
    tiled = O.sf_to_mma_tiles(sf)
    for _ in range(2000):
        r_, g = int(rng.integers(rows)), int(rng.integers(K // 16))
        assert tiled[S.svdq_sf_tile_offset(r_, g, K)] == sf[r_, g]
    assert S.svdq_sf_tile_offset(0, K // 16, K) == -1
    assert S.svdq_sf_tile_offset(0, 0, 100) == -1


def test_workspace_bytes():
    M, K, r = 4608, 3072, 32
    ws = S.svdq_act_workspace_bytes(M, K, r)
    assert ws >= M * K // 2 + M * K // 16 + M * 64 * 2
    assert ws % 256 == 0
    assert S.svdq_act_workspace_bytes(100, 3000, 32) == 0


def test_split_k_workspace_rule():
    """svdq_gemm_workspace_bytes restated: at most 16 output tiles of
    256 x 256 and at least 24 stages of 256 along K split each tile's K into
    min(8, 64 // tiles, stages // 6) parts; partials are
    [tiles][parts][2][128][256] fp32."""
    def rule(M, N, K):
        tiles = -(-M // 256) * -(-N // 256)
        stages = -(-(K // 64) // 4)
        if tiles > 16 or stages < 24:
            return 0
        parts = max(1, min(8, 64 // tiles, stages // 6))
        if parts <= 1:
            return 0
        return tiles * parts * 2 * 128 * 256 * 4
    for M, N, K in [(64, 3072, 3072), (4608, 9216, 3072), (256, 12288, 3072), (512, 3072, 12288),
                    (1, 16, 64), (129, 272, 320), (300, 784, 768), (257, 3072, 3072),
                    (2048, 3072, 12288), (64, 128, 12288), (64, 3072, 12288), (200, 256, 6144),
                    (64, 4096, 6144), (16, 640, 6144)]:
        assert S.svdq_gemm_workspace_bytes(M, N, K) == rule(M, N, K), (M, N, K)
    assert S.svdq_gemm_workspace_bytes(64, 3072, 12288) == 12 * 5 * 262144
    assert S.svdq_gemm_workspace_bytes(64, 3072, 3072) == 0
    # the forward workspace adds it after the activation workspace (256-aligned)
    w = _fake_weight(N=3072, K=12288, r=32)
    a = S.svdq_act_workspace_bytes(64, 12288, 32)
    assert S.lib.svdq_forward_workspace_bytes(ctypes.byref(w), 64) == \
        -(-a // 256) * 256 + rule(64, 3072, 12288)
    assert S.lib.svdq_forward_workspace_bytes(ctypes.byref(w), 4608) == \
        S.svdq_act_workspace_bytes(4608, 12288, 32)
    # a split GEMM refuses a short workspace before touching the device
    C, SF, XL = 0x30000000, 0x40000000, 0x50000000
    need = S.svdq_gemm_workspace_bytes(64, 3072, 12288)
    assert S.lib.svdq_gemm_splitk(ctypes.byref(w), C, SF, XL, 64, 0x60000000, 3072,
                                  0x70000000, need - 1, None) == 4
    assert S.lib.svdq_gemm_splitk(ctypes.byref(w), C, SF, XL, 64, 0x60000000, 3072,
                                  None, 0, None) == 4


def _fake_weight(N=256, K=256, r=32, base=0x10000000):
    w = S.SvdqWeight()
    w.N, w.K, w.r = N, K, r
    w.g_x = w.gs_x = w.g_w = w.alpha = w.lr_scale = 1.0
    w.smooth, w.l1_mma, w.l2_mma = base, base + 0x1000, base + 0x2000
    w.bias, w.codes_w, w.sf_w = base + 0x3000, base + 0x4000, base + 0x8000
    return w


def test_argument_validation_before_any_launch():
    L = S.lib
    w = _fake_weight()
    X, C, SF, XL = 0x20000000, 0x30000000, 0x40000000, 0x50000000
    # null weight / null pointers / bad shapes
    assert L.svdq_quantize_act(None, X, 16, 256, C, SF, XL, None) == 1
    assert L.svdq_quantize_act(ctypes.byref(w), None, 16, 256, C, SF, XL, None) == 1
    assert L.svdq_quantize_act(ctypes.byref(w), X, -1, 256, C, SF, XL, None) == 1
    assert L.svdq_quantize_act(ctypes.byref(w), X, 16, 128, C, SF, XL, None) == 1  # ldx < K
    bad = _fake_weight(K=200)
    assert L.svdq_quantize_act(ctypes.byref(bad), X, 16, 256, C, SF, XL, None) == 1
    # misalignment
    assert L.svdq_quantize_act(ctypes.byref(w), X + 2, 16, 256, C, SF, XL, None) == 3
    assert L.svdq_quantize_act(ctypes.byref(w), X, 16, 260, C, SF, XL, None) == 3
    assert L.svdq_gemm(ctypes.byref(w), C, SF, XL, 16, 0x60000008, 256, None) == 3
    mis = _fake_weight(base=0x10000004)
    assert L.svdq_gemm(ctypes.byref(mis), C, SF, XL, 16, 0x60000000, 256, None) == 3
    # workspace
    need = S.svdq_act_workspace_bytes(16, 256, 32)
    assert L.svdq_linear_forward(ctypes.byref(w), X, 16, 256, 0x60000000, 256,
                                 0x70000000, need - 1, None) == 4
    assert L.svdq_linear_forward(ctypes.byref(w), X, 16, 256, 0x60000000, 256,
                                 0x70000010, need, None) == 3
    # M == 0 is a no-op
    assert L.svdq_linear_forward(ctypes.byref(w), X, 0, 256, 0x60000000, 256,
                                 0x70000000, need, None) == 0


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


@pytest.mark.skipif(_has_gpu(), reason="would launch on fake pointers")
def test_gpu_entry_points_refuse_without_b200():
    L = S.lib
    w = _fake_weight()
    need = S.svdq_act_workspace_bytes(16, 256, 32)
    assert L.svdq_linear_forward(ctypes.byref(w), 0x20000000, 16, 256, 0x60000000, 256,
                                 0x70000000, need, None) == 2
    assert L.svdq_selftest_timeout(1000, None) == 2
    code = ctypes.c_int(0)
    assert L.svdq_device_error(None, ctypes.byref(code)) == 2


def test_unswizzle_scales_matches_oracle_layout():
    rng = np.random.default_rng(3)
    rows, K = 300, 512
    sf = rng.integers(0, 127, (rows, K // 16)).astype(np.uint8)
    tiled = O.sf_to_mma_tiles(sf)
    assert np.array_equal(S.svdq_unswizzle_scales(tiled, rows, K), sf)
    L = S.lib
    out = np.empty((rows, K // 16), np.uint8)
    assert L.svdq_unswizzle_scales(tiled.ctypes.data, rows, 100, out.ctypes.data) == 1
    assert L.svdq_unswizzle_scales(None, rows, K, out.ctypes.data) == 1
    assert L.svdq_unswizzle_scales(tiled.ctypes.data, -1, K, out.ctypes.data) == 1
    assert L.svdq_unswizzle_scales(None, 0, K, None) == 0


def test_host_forward_argument_validation():
    L = S.lib
    w = _fake_weight()
    Xh, Yh, Xd, Yd, WS = 0x20000000, 0x30000000, 0x40000000, 0x50000000, 0x70000000
    need = S.svdq_act_workspace_bytes(16, 256, 32)
    f = L.svdq_linear_forward_host
    assert f(None, Xh, 16, 256, Yh, 256, Xd, Yd, WS, need, None) == 1
    assert f(ctypes.byref(w), None, 16, 256, Yh, 256, Xd, Yd, WS, need, None) == 1
    assert f(ctypes.byref(w), Xh, 16, 255, Yh, 256, Xd, Yd, WS, need, None) == 1   # ldx < K
    assert f(ctypes.byref(w), Xh, 16, 256, Yh, 200, Xd, Yd, WS, need, None) == 1   # ldy < N
    assert f(ctypes.byref(w), Xh, 16, 256, Yh, 256, None, Yd, WS, need, None) == 1
    assert f(ctypes.byref(w), Xh, 16, 256, Yh, 256, Xd, Yd, WS, need - 1, None) == 4
    assert f(ctypes.byref(w), Xh, 16, 256, Yh, 256, Xd + 8, Yd, WS, need, None) == 3
    assert f(ctypes.byref(w), Xh, 16, 256, Yh, 256, Xd, Yd, WS + 16, need, None) == 3
    assert f(ctypes.byref(w), Xh, 0, 256, Yh, 256, Xd, Yd, WS, need, None) == 0
    # host rows may be strided and unaligned: only the device side is checked
    if not _has_gpu():
        assert f(ctypes.byref(w), Xh + 2, 16, 300, Yh + 2, 260, Xd, Yd, WS, need, None) == 2


def test_pack_rejects_bad_input():
    W = np.zeros((32, 64), np.float32)
    cx = np.ones(64, np.float32)
    with pytest.raises(S.SvdqError) as e:
        S.svdq_pack_weight(W, cx, 48)
    assert e.value.status == 1
    # a bias given without an output buffer for it
    out = S.SvdqPackedHost()
    sm = np.empty(64, np.float32)
    cw = np.empty((32, 32), np.uint8)
    sfw = np.empty(256 * 4, np.uint8)
    out.smooth, out.codes_w, out.sf_w, out.bias = sm.ctypes.data, cw.ctypes.data, sfw.ctypes.data, None
    bias = np.zeros(32, np.uint16)
    assert S.lib.svdq_pack_weight(W.ctypes.data, cx.ctypes.data, bias.ctypes.data, 32, 64, 0,
                                  0.5, 0, ctypes.byref(out)) == 1
    W[3, 5] = np.nan
    with pytest.raises(S.SvdqError) as e:
        S.svdq_pack_weight(W, cx, 16)
    assert e.value.status == 7


def test_split_k_argument_checks():
    """svdq_gemm_splitk checks its workspace's size and alignment before
    touching a device; a shape that does not split needs no workspace."""
    L = S.lib
    w = _fake_weight(N=3072, K=12288, r=32)
    C, SF, XL, Y = 0x30000000, 0x40000000, 0x50000000, 0x60000000
    need = S.svdq_gemm_workspace_bytes(64, 3072, 12288)
    assert need > 0
    assert L.svdq_gemm_splitk(ctypes.byref(w), C, SF, XL, 64, Y, 3072, 0x70000010, need,
                              None) == 3                                  # not 256-aligned
    assert L.svdq_gemm_splitk(ctypes.byref(w), C, SF, XL, 0, Y, 3072, None, 0, None) == 0
    assert L.svdq_gemm_splitk(ctypes.byref(w), C, SF, XL, 64, Y, 3000, 0x70000000, need,
                              None) == 1                                  # ldy < N
    assert S.svdq_gemm_workspace_bytes(64, 3072, 100) == 0                # K % 64
