"""AWQ W4A16 linear: host pack against the oracle (CPU, bit-exact), the
entry points' argument checks (CPU), and the GPU kernel against the
oracle's float64 layer (GPU)."""
import ctypes

import numpy as np
import pytest

import svdq_inputs as SI
import w4a4_rank_corrected_b200 as S
from oracle import awq as A
from oracle import formats as F


@pytest.mark.parametrize("N,K,group,seed", [(16, 128, 128, 0), (100, 3072, 128, 1),
                                            (33, 512, 64, 2), (8, 256, 32, 3)])
def test_awq_pack_matches_oracle(N, K, group, seed):
    rng = np.random.default_rng(seed)
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    W[0, :group] = 0.0                       # an all-zero group
    W[1, :group] = 0.01                      # a constant group
    W[2, :] *= 50.0                          # a large row
    aw = S.svdq_awq_pack(W, group)
    q, z, sb = A.awq_quantize(W, group)
    assert np.array_equal(aw.scales, sb)
    assert np.array_equal(aw.zeros, z)
    assert np.array_equal(aw.q, A.pack_nibbles_awq(q))


@pytest.mark.parametrize("N,K,seed", [(16, 64, 0), (40, 256, 1), (1000, 1536, 2)])
def test_awq_tile_codes_layout(N, K, seed):
    """The tiled code layout read back the way a warp's m16n8k16 A fragment
    takes it: lane l = 4 g + c, register r holds (row g + 8 (r % 2),
    columns 2 c + 8 (r // 2) + {0, 1}) of each 16 x 16 tile; in the word,
    register r's low half is nibble r and its high half nibble r + 4."""
    rng = np.random.default_rng(seed)
    q = rng.integers(0, 16, (N, K), dtype=np.uint8)
    tiled = S.svdq_awq_tile_codes(A.pack_nibbles_awq(q), N, K)
    N16 = (N + 15) // 16 * 16
    assert tiled.shape == (N16 * K // 2,)
    words = tiled.view(np.uint32)
    back = np.full((N16, K), 255, np.int32)
    for rb in range(N16 // 16):
        for ks in range(K // 16):
            for lane in range(32):
                g, c = divmod(lane, 4)
                w = int(words[((rb * (K // 64) + ks // 4) * 32 + lane) * 4 + ks % 4])
                for r in range(4):
                    for half in range(2):
                        nib = (w >> (4 * (r + 4 * half))) & 15
                        row = 16 * rb + g + 8 * (r % 2)
                        col = 16 * ks + 2 * c + 8 * (r // 2) + half
                        assert back[row, col] == 255
                        back[row, col] = nib
    assert np.array_equal(back[:N], q)
    assert np.all(back[N:] == 0)


def test_awq_argument_validation():
    L = S.lib
    W = np.zeros((4, 128), np.float32)
    q = np.empty((4, 64), np.uint8)
    z = np.empty((4, 1), np.uint8)
    sc = np.empty((4, 1), np.uint16)
    assert L.svdq_awq_pack(W.ctypes.data, 4, 128, 48, q.ctypes.data, z.ctypes.data, sc.ctypes.data) == 1
    assert L.svdq_awq_pack(None, 4, 128, 128, q.ctypes.data, z.ctypes.data, sc.ctypes.data) == 1
    W[0, 0] = np.inf
    assert L.svdq_awq_pack(W.ctypes.data, 4, 128, 128, q.ctypes.data, z.ctypes.data, sc.ctypes.data) == 7
    Q, Z, SC, X, Y = 0x10000000, 0x20000000, 0x30000000, 0x40000000, 0x50000000
    f = L.svdq_awq_linear
    assert f(Q, Z, SC, None, 64, 128, 128, X, 9, 128, Y, 64, None) == 1        # M > 8
    assert f(Q, Z, SC, None, 64, 128, 100, X, 1, 128, Y, 64, None) == 1       # group
    assert f(Q, Z, SC, None, 64, 128, 64, X, 1, 128, Y, 64, None) == 1        # group % 128
    assert f(Q, Z, SC, None, 64, 128, 128, X, 1, 100, Y, 64, None) == 1       # ldx < K
    assert f(Q + 8, Z, SC, None, 64, 128, 128, X, 1, 128, Y, 64, None) == 3   # alignment
    assert f(Q, Z, SC, None, 64, 16384, 128, X, 8, 16384, Y, 64, None) == 1   # X too big to stage
    assert f(Q, Z, SC, None, 64, 128, 128, X, 0, 128, Y, 64, None) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("M,K,N", [(1, 3072, 18432), (4, 3072, 18432), (3, 128, 64),
                                   (8, 1536, 1000), (2, 12288, 3072)])
def test_awq_linear_parity(M, K, N):
    """The GPU layer against the oracle's float64 layer (same packed codes):
    rel-Fro <= 2e-3 and per element 1e-2 rms + half a bf16 ulp."""
    import torch
    from gpu_common import check_output, from_dev_bf16, to_dev_bf16
    rng = np.random.default_rng(M * 7 + K + N)
    X = SI.f32_to_bf16_bits((rng.standard_normal((M, K))).astype(np.float32))
    W = (rng.standard_normal((N, K)) * 0.02).astype(np.float32)
    b = SI.f32_to_bf16_bits((rng.standard_normal(N) * 0.01).astype(np.float32))
    aw = S.svdq_awq_pack(W, 128, bias_bf16=b).to_device("cuda")
    Y = S.svdq_awq_linear(aw, to_dev_bf16(X))
    torch.cuda.synchronize()
    q, z, sb = A.awq_quantize(W, 128)
    Y_ref = A.awq_linear_reference(X, q, z, sb, b)
    check_output(from_dev_bf16(Y), Y_ref)
    assert S.svdq_device_error() == 0


def test_awq_code_to_bf16_trick_is_exact():
    """The GEMV's dequantization, restated on the host: the bit pattern
    0x4300 | q is the bf16 number 128 + q for every 4-bit q, and the bf16
    difference (128 + q) - (128 + z) is q - z exactly (no rounding: every
    operand and result is an integer of at most 8 significant bits)."""
    import torch
    q = torch.arange(16, dtype=torch.int32)
    as_bf16 = (q | 0x4300).to(torch.int16).view(torch.bfloat16)
    assert torch.equal(as_bf16.float(), 128.0 + q.float())
    for z in range(16):
        zz = torch.full((16,), 0x4300 | z, dtype=torch.int16).view(torch.bfloat16)
        d = (as_bf16 - zz)                    # bf16 subtraction, round to nearest
        assert torch.equal(d.float(), (q - z).float())


def test_awq_tile_codes_validation():
    L = S.lib
    q = np.zeros((16, 32), np.uint8)
    out = np.zeros(16 * 32, np.uint8)
    assert L.svdq_awq_tile_codes(q.ctypes.data, 16, 64, out.ctypes.data) == 0
    assert L.svdq_awq_tile_codes(q.ctypes.data, 16, 96, out.ctypes.data) == 1      # K % 64
    assert L.svdq_awq_tile_codes(None, 16, 64, out.ctypes.data) == 1
    assert L.svdq_awq_tile_codes(q.ctypes.data, 0, 64, out.ctypes.data) == 1
    with pytest.raises(ValueError):
        S.svdq_awq_tile_codes(q[:, :16], 16, 64)                                   # shape
