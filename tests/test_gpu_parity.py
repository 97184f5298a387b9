"""GPU parity of the CUDA path against the CPU oracle (needs a B200).

Bar: bit-exact E2M1 codes and E4M3 scales (activation and weight); bf16
output with relative Frobenius error <= 2e-3 against the float64 oracle and
every element within 1e-2 rms(Y_ref) plus half a bf16 ulp.  Shapes span
several tiles with ragged tails; the full-size workloads run in the launch
configuration that bench.py times, with codes and scales compared on every
row and the output on at least one row of every 128-row block."""
import numpy as np
import pytest

import svdq_inputs as SI
from oracle import formats as F
from oracle import svdq as O

from gpu_common import (check_activation, check_output, from_dev_bf16, prepare, rows_every_block,
                        rows_sample, to_dev_bf16)

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import w4a4_rank_corrected_b200 as S
    assert S.svdq_device_error() == 0
    yield
    assert S.svdq_device_error() == 0, "a kernel recorded a timed-out wait"


def _S():
    import w4a4_rank_corrected_b200 as S
    return S


# ---------------------------------------------------------- conversions ----

def _binade(e: int) -> np.ndarray:
    """Every float32 in [2^e, 2^(e+1))."""
    bits = ((e + 127) << 23) | np.arange(1 << 23, dtype=np.uint32)
    return bits.astype(np.uint32).view(np.float32)


def test_hardware_conversions_match_oracle_exhaustive():
    """The device conversions the activation kernel uses against the
    oracle's encoders on EVERY float32 of the binades that reach a non-zero
    code: E2M1 on [2^-3, 2^4) with both signs (below 2^-2 everything rounds
    to a signed zero; from 6 on everything saturates), E4M3 on [2^-11, 2^10)
    (non-negative: block scales; the smallest subnormal is 2^-9, the
    largest finite 448).  Plus zeros, the sub-binade tails and saturation."""
    S = _S()
    for e in range(-3, 4):
        for sign in (1.0, -1.0):
            v = _binade(e) * np.float32(sign)
            e2, _ = S.svdq_debug_convert(torch.from_numpy(v).cuda())
            got = e2.cpu().numpy()
            want = F.e2m1_encode(v)
            bad = np.nonzero(got != want)[0]
            assert bad.size == 0, (e, sign, v[bad[:4]], got[bad[:4]], want[bad[:4]])
    for e in range(-11, 10):
        v = _binade(e)
        _, e4 = S.svdq_debug_convert(torch.from_numpy(v).cuda())
        got = e4.cpu().numpy()
        want = F.e4m3_encode_nonneg(v)
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (e, v[bad[:4]], got[bad[:4]], want[bad[:4]])
    edge = np.array([0.0, -0.0, 2.0 ** -40, 2.0 ** -12, 1e-30, 6.0, 7.0, 448.0, 464.0, 1e30,
                     3.0e38], np.float32)
    edge = np.concatenate([edge, -edge])
    e2, e4 = S.svdq_debug_convert(torch.from_numpy(edge).cuda())
    assert np.array_equal(e2.cpu().numpy(), F.e2m1_encode(edge))
    assert np.array_equal(e4.cpu().numpy(), F.e4m3_encode_nonneg(np.abs(edge)))


def test_bounded_wait_reports_and_recovers():
    S = _S()
    S.svdq_selftest_timeout(20000)
    code = S.svdq_device_error()
    assert code == (7 << 8) | 3
    assert S.svdq_device_error() == 0
    x = torch.ones(1024, device="cuda")
    assert float((x * 2).sum()) == 2048.0        # the context is still usable


# ----------------------------------------------------- activation kernel ----

QUANT_CASES = [  # M, K, N, r
    (1, 64, 32, 16), (100, 192, 48, 16), (129, 256, 64, 32), (256, 3072, 64, 32),
    (300, 1024, 64, 0), (64, 3072, 128, 128), (517, 640, 96, 48), (1000, 1536, 64, 64),
]


@pytest.mark.parametrize("M,K,N,r", QUANT_CASES)
def test_quantize_act_parity(M, K, N, r):
    S = _S()
    X, W, b = SI.random_layer(M * 7 + K, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    codes, sf, xl1 = S.svdq_quantize_act(dw, Xd)
    torch.cuda.synchronize()
    check_activation(codes, sf, xl1, X, op, M, K, r)


def test_quantize_act_strided_input():
    """X as a column slice of a wider tensor (ldx > K), like the V slice of a
    fused QKV output."""
    S = _S()
    M, K, N, r = 200, 256, 64, 16
    X, W, b = SI.random_layer(3, M, 3 * K, N)
    Xs = np.ascontiguousarray(X[:, 2 * K:])
    lp, op, dw = prepare(W[:, :K].copy(), SI.channel_absmax(Xs), r, b)
    Xd = to_dev_bf16(X)[:, 2 * K:]
    assert Xd.stride(0) == 3 * K
    codes, sf, xl1 = S.svdq_quantize_act(dw, Xd)
    torch.cuda.synchronize()
    check_activation(codes, sf, xl1, Xs, op, M, K, r)


# ------------------------------------------------------------ full layer ----

def test_linear_strided_output_writes_only_its_window():
    """Y as a window of a wider, taller buffer (ldy > N, 8 columns in, rows
    below M): the layer writes exactly rows [0, M) x columns [0, N) of the
    window, bit-identical to a contiguous Y, and leaves the rest alone.  The
    shape has a partial last column box (N = 272) and a partial row box
    (M = 200)."""
    S = _S()
    M, K, N, r = 200, 256, 272, 16
    X, W, b = SI.random_layer(31, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    Y0 = S.svdq_linear_forward(dw, Xd)
    ld = N + 72                       # a multiple of 8 elements
    sentinel = -3.0
    big = torch.full((M + 130, ld), sentinel, dtype=torch.bfloat16, device="cuda")
    Yv = big[:M, 8:8 + N]
    assert Yv.stride(0) == ld and Yv.data_ptr() % 16 == 0
    S.svdq_linear_forward(dw, Xd, Y=Yv)
    torch.cuda.synchronize()
    assert np.array_equal(from_dev_bf16(Yv), from_dev_bf16(Y0))
    mask = torch.ones_like(big, dtype=torch.bool)
    mask[:M, 8:8 + N] = False
    assert bool((big[mask] == sentinel).all()), "the layer wrote outside its output window"
    assert S.svdq_device_error() == 0


LAYER_CASES = [  # M, K, N, r
    (1, 64, 16, 16), (100, 192, 48, 16), (129, 320, 272, 32), (200, 1024, 512, 0),
    (64, 512, 256, 128), (300, 768, 784, 48), (257, 3072, 3072, 32),
]


@pytest.mark.parametrize("M,K,N,r", LAYER_CASES)
def test_linear_forward_parity(M, K, N, r):
    S = _S()
    X, W, b = SI.random_layer(M + 13 * K + N, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Y = S.svdq_linear_forward(dw, to_dev_bf16(X))
    torch.cuda.synchronize()
    Y_ref, _, _, _ = O.linear_reference(X, op, b)
    check_output(from_dev_bf16(Y), Y_ref)


SPLIT_CASES = [  # M, K, N, r: few output tiles and long K, so the GEMM splits K
    (64, 12288, 3072, 32), (200, 6144, 256, 0), (300, 8192, 512, 32), (16, 6144, 640, 128),
]


@pytest.mark.parametrize("M,K,N,r", SPLIT_CASES)
def test_gemm_splitk_parity_and_determinism(M, K, N, r):
    """Split-K GEMM: within tolerance of the oracle, bit-identical across
    calls (the partials are added in part order), with a workspace that
    starts out as garbage."""
    S = _S()
    need = S.svdq_gemm_workspace_bytes(M, N, K)
    assert need > 0
    X, W, b = SI.random_layer(M + 7 * K + N, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    codes, sf, xl1 = S.svdq_quantize_act(dw, to_dev_bf16(X))
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")
    Y1 = S.svdq_gemm_splitk(dw, codes, sf, xl1, M, workspace=ws).clone()
    Y2 = S.svdq_gemm_splitk(dw, codes, sf, xl1, M, workspace=ws)
    Y0 = S.svdq_gemm(dw, codes, sf, xl1, M)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))
    Y_ref, _, _, _ = O.linear_reference(X, op, b)
    check_output(from_dev_bf16(Y1), Y_ref)
    check_output(from_dev_bf16(Y0), Y_ref)
    # the forward with a workspace that has room for the partials splits too
    Yf = S.svdq_linear_forward(dw, to_dev_bf16(X))
    torch.cuda.synchronize()
    assert torch.equal(Yf.view(torch.int16), Y1.view(torch.int16))
    assert S.svdq_device_error() == 0


def test_zero_input_gives_bias_exactly():
    S = _S()
    M, K, N, r = 130, 256, 512, 32
    X, W, b = SI.random_layer(21, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Y = S.svdq_linear_forward(dw, torch.zeros((M, K), dtype=torch.bfloat16, device="cuda"))
    got = from_dev_bf16(Y)
    assert np.array_equal(got, np.broadcast_to(b, got.shape))


def test_low_rank_branch_alone():
    """All activation codes zero: the GEMM output is the up-projection plus
    bias only (checks the low-rank MMA, its operands and the shared
    accumulator on their own)."""
    S = _S()
    M, K, N, r = 192, 512, 512, 32
    X, W, b = SI.random_layer(22, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    codes, sf, xl1 = S.svdq_quantize_act(dw, to_dev_bf16(X))
    codes.zero_()
    Y = S.svdq_gemm(dw, codes, sf, xl1, M)
    torch.cuda.synchronize()
    xh = O.smooth_activation(X, op.s)
    Y_ref = O.lowrank_down(xh, op.L1) @ F.bf16_bits_to_f64(op.L2) + F.bf16_bits_to_f64(b)[None, :]
    check_output(from_dev_bf16(Y), Y_ref)


def test_fp4_branch_alone():
    """r = 0 and no bias: the plain block-scaled FP4 GEMM."""
    S = _S()
    M, K, N = 256, 1024, 512
    X, W, _ = SI.random_layer(23, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), 0, None)
    Y = S.svdq_linear_forward(dw, to_dev_bf16(X))
    torch.cuda.synchronize()
    Y_ref, _, _, _ = O.linear_reference(X, op, None)
    check_output(from_dev_bf16(Y), Y_ref)


def test_forward_is_deterministic():
    S = _S()
    M, K, N, r = 4608, 3072, 1024, 32
    X, W, b = SI.random_layer(24, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    Y1 = S.svdq_linear_forward(dw, Xd).clone()
    Y2 = S.svdq_linear_forward(dw, Xd)
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def test_activation_kernel_repeats_bit_identical():
    """Twenty launches of the activation kernel at the Flux shape give the same
    codes, scales and low-rank operand bit for bit: guards the hand-back of
    ring stages (generic reads, then a TMA refill) against reordering races,
    which showed up as one unit of wrong codes in a few percent of launches."""
    S = _S()
    M, K, N, r = 4608, 3072, 1024, 32
    X, W, b = SI.random_layer(24, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    c0, s0, x0 = (t.clone() for t in S.svdq_quantize_act(dw, Xd))
    for _ in range(20):
        c, sf, xl1 = S.svdq_quantize_act(dw, Xd)
        assert torch.equal(c, c0) and torch.equal(sf, s0)
        assert torch.equal(xl1.view(torch.int16), x0.view(torch.int16))


@pytest.mark.parametrize("M,K,N,r", [(15361, 320, 64, 48), (16000, 3072, 128, 32),
                                     (15500, 192, 64, 0), (20000, 1024, 256, 128)])
def test_activation_kernel_128_row_tiles(M, K, N, r):
    """Batches of about 15k rows and more take the 128-row activation kernel
    (the others the 64-row one): bit-exact codes and scales on every row,
    the low-rank operand within tolerance, ragged M and K tails, r from 0 to
    128; and the whole layer on one row of every 128-row block."""
    S = _S()
    X, W, b = SI.random_layer(M + K, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    codes, sf, xl1 = S.svdq_quantize_act(dw, Xd)
    Y = S.svdq_linear_forward(dw, Xd)
    torch.cuda.synchronize()
    check_activation(codes, sf, xl1, X, op, M, K, r)
    rows = rows_every_block(M, extra=16, seed=M)
    Y_ref, _, _, _ = O.linear_reference(X, op, b, rows=rows)
    check_output(from_dev_bf16(Y)[rows], Y_ref)


# ---------------------------------------------------- full-size workloads ----

def _workload_layer(name, M=None):
    wl = SI.make_workload(name, M=M)
    lt = wl.layers[0]
    return wl.X_bf16, lt.W, lt.bias_bf16, lt.spec.r


@pytest.mark.parametrize("name", ["single_256", "flux_qkv", "sweep_r16", "sweep_r32", "sweep_r64",
                                  "sweep_r128", "sweep_m64", "sweep_m512"])
def test_workload_parity(name):
    """Each workload at full size: activation codes and scales bit-exact on
    every row, the output on every row for M <= 1024 and otherwise on at
    least one row of every 128-row block."""
    S = _S()
    X, W, b, r = _workload_layer(name)
    M, K = X.shape
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    codes, sf, xl1 = S.svdq_quantize_act(dw, Xd)
    ws = S.new_workspace(M, K, r)
    Y = S.svdq_linear_forward(dw, Xd, workspace=ws)
    torch.cuda.synchronize()
    check_activation(codes, sf, xl1, X, op, M, K, r)
    idx = np.arange(M) if M <= 1024 else rows_every_block(M, seed=len(name))
    Y_ref, _, _, _ = O.linear_reference(X, op, b, rows=idx)
    check_output(from_dev_bf16(Y)[idx], Y_ref)


def _layer_check(S, lt, Xin_dev, Xin_bits, seed):
    """One layer of a chain, calibrated on and compared with the oracle fed
    its actual bf16 input: codes and scales on every row, the output on at
    least one row of every 128-row block."""
    M, K, r = Xin_bits.shape[0], lt.spec.K, lt.spec.r
    lp, op, dw = prepare(lt.W, SI.channel_absmax(Xin_bits), r, lt.bias_bf16)
    codes, sf, xl1 = S.svdq_quantize_act(dw, Xin_dev)
    Y = S.svdq_linear_forward(dw, Xin_dev)
    torch.cuda.synchronize()
    check_activation(codes, sf, xl1, Xin_bits, op, M, K, r)
    rows = rows_every_block(M, seed=seed)
    Yr, _, _, _ = O.linear_reference(Xin_bits, op, lt.bias_bf16, rows=rows)
    check_output(from_dev_bf16(Y)[rows], Yr)
    return Y


def test_mlp_pair_parity():
    """fc1 -> GELU (tanh, bf16, on the GPU) -> fc2 (K = 12288)."""
    S = _S()
    wl = SI.make_workload("flux_mlp")
    X = wl.X_bf16
    fc1, fc2 = wl.layers
    Y1 = _layer_check(S, fc1, to_dev_bf16(X), X, seed=5)
    H = torch.nn.functional.gelu(Y1, approximate="tanh")
    _layer_check(S, fc2, H, from_dev_bf16(H), seed=6)


def test_flux_block_parity():
    """Config 4 (M = 18432): qkv -> out on the V slice of the qkv output
    (strided input, ldx = 9216) -> fc1 -> GELU (tanh, bf16, on the GPU) ->
    fc2 (K = 12288)."""
    S = _S()
    wl = SI.make_workload("flux_block")
    X = wl.X_bf16
    qkv, out, fc1, fc2 = wl.layers
    M, H = X.shape
    Yq = _layer_check(S, qkv, to_dev_bf16(X), X, seed=9)
    V = Yq[:, 2 * H:]                       # strided view, ldx = 3 H
    assert V.stride(0) == 3 * H
    Yo = _layer_check(S, out, V, from_dev_bf16(V), seed=10)
    Y1 = _layer_check(S, fc1, Yo, from_dev_bf16(Yo), seed=11)
    G = torch.nn.functional.gelu(Y1, approximate="tanh")
    _layer_check(S, fc2, G, from_dev_bf16(G), seed=12)


def test_host_streamer_matches_forward():
    """The host-buffer path (C ABI svdq_linear_forward_host, two streams,
    two buffer sets) gives the device forward's output bit for bit, batch
    after batch."""
    S = _S()
    M, K, N, r = 300, 512, 384, 32
    X0, W, b = SI.random_layer(91, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X0), r, b)
    hs = S.HostStreamer(dw, M, "cuda")
    outs, refs = [], []
    for i in range(4):
        X, _, _ = SI.random_layer(200 + i, M, K, N)
        Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).pin_memory()
        Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
        hs.submit(Xh, Yh)
        outs.append((Xh, Yh))
        refs.append(from_dev_bf16(S.svdq_linear_forward(dw, to_dev_bf16(X))))
    hs.synchronize()
    torch.cuda.synchronize()
    for (Xh, Yh), ref in zip(outs, refs):
        got = Yh.view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(got, ref)


def test_host_forward_strided_host_buffers():
    """svdq_linear_forward_host with host rows wider than the tensor (ldx_host
    > K, ldy_host > N): the device forward's output bit for bit, written into
    exactly the [M, N] window of the host buffer."""
    S = _S()
    M, K, N, r = 257, 320, 272, 16
    X, W, b = SI.random_layer(93, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xwide = np.zeros((M, K + 24), np.uint16)
    Xwide[:, :K] = X
    Xh = torch.from_numpy(Xwide.view(np.int16)).view(torch.bfloat16).pin_memory()[:, :K]
    Yh_full = torch.full((M, N + 40), -2.0, dtype=torch.bfloat16).pin_memory()
    Yh = Yh_full[:, :N]
    Xd = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    Yd = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    # the same workspace size as the reference call below (with room for the
    # split-K partials), so both take the same GEMM path
    ws = S.new_forward_workspace(dw, M)
    S.svdq_linear_forward_host(dw, Xh, Yh, Xd, Yd, ws)
    torch.cuda.synchronize()
    ref = from_dev_bf16(S.svdq_linear_forward(dw, to_dev_bf16(X)))
    got = Yh_full.view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got[:, :N], ref)
    assert np.all(got[:, N:] == np.uint16(0xC000))     # bf16(-2.0): untouched


def test_forward_on_side_stream_without_workspace():
    """A forward on a non-current stream whose workspace and output the
    binding allocates: the binding ties them to that stream, so work queued
    meanwhile on the current stream cannot reuse their memory."""
    S = _S()
    M, K, N, r = 1024, 1024, 768, 32
    X, W, b = SI.random_layer(95, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    ref = from_dev_bf16(S.svdq_linear_forward(dw, Xd))
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    outs = []
    for _ in range(3):
        Y = S.svdq_linear_forward(dw, Xd, stream=side)
        outs.append(Y)
        # churn the allocator on the current stream while the side stream runs
        junk = [torch.full((M * K,), 7, dtype=torch.uint8, device="cuda") for _ in range(4)]
        del junk
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for Y in outs:
        assert np.array_equal(from_dev_bf16(Y), ref)
    assert S.svdq_device_error() == 0


# ------------------------------------------------- fused GELU (MLP pair) ----

def test_epilogue_gelu_on_every_bf16():
    """The GEMM epilogue's GELU (hardware approximate exponential and
    reciprocal) against the oracle's GELU on every finite bf16 input: the
    same bf16 value, except next to a bf16 rounding boundary (where the
    exact value lies within 2e-6 relative of one), where the two differ by
    at most one unit in the last place; and +-inf map as the oracle maps
    them."""
    S = _S()
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        x = F.bf16_bits_to_f64(bits)
    bits = bits[~np.isnan(x)]
    got = from_dev_bf16(S.svdq_debug_gelu(to_dev_bf16(bits)))
    want = O.gelu_bf16(bits)
    ref = O.gelu_tanh_f32(F.bf16_bits_to_f64(bits).astype(np.float32)).astype(np.float64)
    with np.errstate(invalid="ignore", over="ignore"):
        lo = F.f64_to_bf16_bits(ref * (1 - 2e-6))
        hi = F.f64_to_bf16_bits(ref * (1 + 2e-6))
    near = (lo != want) | (hi != want)
    with np.errstate(invalid="ignore"):
        both_nan = np.isnan(F.bf16_bits_to_f64(got)) & np.isnan(F.bf16_bits_to_f64(want))
    differ = (got != want) & ~both_nan          # GELU(-inf) is NaN on both sides
    assert not np.any(differ & ~near), bits[differ & ~near][:5]
    # where they differ: adjacent bf16 values (one ulp) of the same sign
    d = np.abs(got[differ].astype(np.int32) - want[differ].astype(np.int32))
    assert np.all(d == 1), d.max() if d.size else 0
    assert np.count_nonzero(differ) <= 200


@pytest.mark.parametrize("M,K,N,r", [(129, 320, 272, 32), (300, 768, 784, 16),
                                     (4608, 3072, 12288, 32)])
def test_gemm_gelu_equals_gemm_then_gelu(M, K, N, r):
    """The fused epilogue writes exactly GELU of what the plain GEMM writes:
    H == gelu(Y) bit for bit (the same bf16 y, the same GELU steps)."""
    S = _S()
    X, W, b = SI.random_layer(M + N, M, K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    codes, sf, xl1 = S.svdq_quantize_act(dw, to_dev_bf16(X))
    Y = S.svdq_gemm(dw, codes, sf, xl1, M)
    H = S.svdq_gemm_gelu(dw, codes, sf, xl1, M)
    torch.cuda.synchronize()
    assert torch.equal(H.view(torch.int16), S.svdq_debug_gelu(Y).view(torch.int16))
    assert S.svdq_device_error() == 0


def test_mlp_pair_fused_parity():
    """svdq_mlp_forward on the Flux MLP pair (config 2): fc1 with the GELU
    epilogue, fc2 on its output.  H equals the epilogue GELU of fc1's bf16
    output bit for bit and the oracle's GELU of it within one bf16 unit;
    fc2's codes and scales bit-exact against the oracle fed the GPU's H on
    every row; fc1's output and Y within tolerance on at least one row of
    every 128-row block."""
    S = _S()
    wl = SI.make_workload("flux_mlp")
    X = wl.X_bf16
    fc1, fc2 = wl.layers
    M = X.shape[0]
    # fc2 is calibrated on the unfused chain's GELU output (the same values)
    lp1, op1, dw1 = prepare(fc1.W, SI.channel_absmax(X), 32, fc1.bias_bf16)
    Y1 = S.svdq_linear_forward(dw1, to_dev_bf16(X))
    Hcal = from_dev_bf16(S.svdq_debug_gelu(Y1))
    lp2, op2, dw2 = prepare(fc2.W, SI.channel_absmax(Hcal), 32, fc2.bias_bf16)
    H, Y = S.svdq_mlp_forward(dw1, dw2, to_dev_bf16(X))
    torch.cuda.synchronize()
    Hb = from_dev_bf16(H)
    # the fused GELU is exactly the oracle's GELU of fc1's bf16 output, and
    # that output is within tolerance of fc1's float64 reference
    assert np.array_equal(Hb, Hcal)
    Ho = O.gelu_bf16(from_dev_bf16(Y1))
    assert np.max(np.abs(Hb.astype(np.int32) - Ho.astype(np.int32))) <= 1
    assert np.count_nonzero(Hb != Ho) <= 1e-3 * Hb.size
    rows = rows_every_block(M, seed=21)
    Y1r, _, _, _ = O.linear_reference(X, op1, fc1.bias_bf16, rows=rows)
    check_output(from_dev_bf16(Y1)[rows], Y1r)
    codes2, sf2, xl2 = S.svdq_quantize_act(dw2, H)
    torch.cuda.synchronize()
    check_activation(codes2, sf2, xl2, Hb, op2, M, fc2.spec.K, 32)
    Y2r, _, _, _ = O.linear_reference(Hb, op2, fc2.bias_bf16, rows=rows)
    check_output(from_dev_bf16(Y)[rows], Y2r)
    assert S.svdq_device_error() == 0


# ------------------------------------------- dynamic per-token scales ----

def _check_dynamic(S, dw, op, X, b, rows=None):
    M, K = X.shape
    Xd = to_dev_bf16(X)
    rs = S.svdq_act_row_scales(dw, Xd)
    codes, sf, xl1 = S.svdq_quantize_act_dynamic(dw, Xd, rs)
    Y = S.svdq_linear_forward_dynamic(dw, Xd)
    torch.cuda.synchronize()
    xh, cq, sq, A = O.quantize_activation_dynamic(X, op.s)
    # the row scales: g, gs bit-exact against the oracle's R4 of each row
    r_ = rs.cpu().numpy()
    g_ref = np.array([O.tensor_encode_scale(a) for a in A], np.float32)
    gs_ref = np.array([O.block_scale_factor(a) for a in A], np.float32)
    assert np.array_equal(r_[:, 0], g_ref) and np.array_equal(r_[:, 1], gs_ref)
    assert np.array_equal(codes.cpu().numpy(), O.pack_nibbles(cq)), "dynamic codes differ"
    assert np.array_equal(O.sf_from_mma_tiles(sf.cpu().numpy(), M, K), sq), "dynamic scales differ"
    idx = np.arange(M) if rows is None else rows
    Y_ref, _, _, _, _ = O.linear_reference_dynamic(X, op, b, rows=idx)
    check_output(from_dev_bf16(Y)[idx], Y_ref)
    return from_dev_bf16(Y)


@pytest.mark.parametrize("name", ["flux_qkv", "sweep_r32", "sweep_m64"])
def test_dynamic_scale_parity(name):
    """Per-token activation scales (reading R5d) on configs 1 and 3: row
    scales, codes and scales bit-exact against the oracle on every row; the
    output against the oracle's per-row reference (one row of every 128-row
    block, or every row for small M)."""
    S = _S()
    X, W, b, r = _workload_layer(name)
    M = X.shape[0]
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    _check_dynamic(S, dw, op, X, b, rows=None if M <= 1024 else rows_every_block(M, seed=3))
    assert S.svdq_device_error() == 0


def test_dynamic_scale_beyond_calibration():
    """Inputs 16x beyond the calibration range.  Per-token scales are
    invariant to a power-of-two scaling of X: the codes and scales of 16 X
    equal those of X bit for bit, and the output error against the exact
    X W^T + b stays at the in-range 4-bit floor.  The static scale
    saturates (E4M3 at 448, E2M1 at 6): its error at 16x is at least 1.5x
    the in-range one (the unquantized low-rank branch, most of the output,
    is untouched by the saturation).  Large M takes the 128-row kernel."""
    S = _S()
    for M in (512, 16384):
        K, N, r = 3072, 512, 32
        Xc, W, b = SI.random_layer(60 + M, M, K, N)
        lp, op, dw = prepare(W, SI.channel_absmax(Xc), r, b)       # calibrated on Xc
        Xb = SI.f32_to_bf16_bits(SI.bf16_bits_to_f32(Xc) * np.float32(16.0))
        rows = rows_every_block(M, extra=8, seed=M)
        Yd = _check_dynamic(S, dw, op, Xb, b, rows=rows)
        c1, s1, _ = S.svdq_quantize_act_dynamic(dw, to_dev_bf16(Xc), S.svdq_act_row_scales(dw, to_dev_bf16(Xc)))
        c16, s16, _ = S.svdq_quantize_act_dynamic(dw, to_dev_bf16(Xb), S.svdq_act_row_scales(dw, to_dev_bf16(Xb)))
        assert torch.equal(c1, c16) and torch.equal(s1, s16)
        Ys1 = from_dev_bf16(S.svdq_linear_forward(dw, to_dev_bf16(Xc)))
        Ys16 = from_dev_bf16(S.svdq_linear_forward(dw, to_dev_bf16(Xb)))
        w64 = W.astype(np.float64).T
        bias = F.bf16_bits_to_f64(b)[None, :]
        ex1 = SI.bf16_bits_to_f32(Xc).astype(np.float64)[rows] @ w64 + bias
        ex16 = SI.bf16_bits_to_f32(Xb).astype(np.float64)[rows] @ w64 + bias
        rel = lambda Y, ex: np.linalg.norm(F.bf16_bits_to_f64(Y[rows]) - ex) / np.linalg.norm(ex)
        e_s1, e_s16, e_d16 = rel(Ys1, ex1), rel(Ys16, ex16), rel(Yd, ex16)
        assert e_d16 <= 1.1 * e_s1, (e_d16, e_s1)
        assert e_s16 >= 1.5 * e_s1, (e_s16, e_s1)
    assert S.svdq_device_error() == 0
