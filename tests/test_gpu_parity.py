"""GPU parity of the CUDA path against the CPU oracle (needs a B200).

Bar: bit-exact E2M1 codes and E4M3 scales (activation and weight); bf16
output with relative Frobenius error <= 2e-3 against the float64 oracle and
every element within 1e-2 rms(Y_ref) plus half a bf16 ulp.  Shapes span
several tiles with ragged tails; the full-size workloads run in the launch
configuration that bench.py times and are compared on sampled rows."""
import numpy as np
import pytest

import svdq_inputs as SI
from oracle import formats as F
from oracle import svdq as O

from gpu_common import (check_activation, check_output, from_dev_bf16, prepare, rows_sample,
                         to_dev_bf16)

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

def _sweep():
    vals = [0.0, -0.0, 6.0, 7.0, 448.0, 449.0, 464.0, 1e30, 2.0 ** -10, 2.0 ** -9, 3 * 2.0 ** -10]
    for e in range(-12, 10):
        m = np.arange(0, 1 << 11) / (1 << 11)
        vals.extend(((1 + m) * 2.0 ** e).tolist())
    v = np.array(vals, np.float32)
    rng = np.random.default_rng(0)
    v = np.concatenate([v, -v, (rng.standard_normal(200000) * 10).astype(np.float32)])
    return v


def test_hardware_conversions_match_oracle():
    S = _S()
    v = _sweep()
    e2, e4 = S.svdq_debug_convert(torch.from_numpy(v).cuda())
    assert np.array_equal(e2.cpu().numpy(), F.e2m1_encode(v))
    assert np.array_equal(e4.cpu().numpy(), F.e4m3_encode_nonneg(np.abs(v)))


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


# ---------------------------------------------------- full-size workloads ----

def _workload_layer(name, M=None):
    wl = SI.make_workload(name, M=M)
    lt = wl.layers[0]
    return wl.X_bf16, lt.W, lt.bias_bf16, lt.spec.r


@pytest.mark.parametrize("name", ["single_256", "flux_qkv", "sweep_r16", "sweep_r32", "sweep_r64",
                                  "sweep_r128", "sweep_m64", "sweep_m512"])
def test_workload_parity(name):
    """Each workload at full size: activation codes/scales bit-exact on every
    row (or sampled rows for M > 1024), output on sampled rows."""
    S = _S()
    X, W, b, r = _workload_layer(name)
    M, K = X.shape
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Xd = to_dev_bf16(X)
    codes, sf, xl1 = S.svdq_quantize_act(dw, Xd)
    ws = torch.empty(S.svdq_act_workspace_bytes(M, K, r), dtype=torch.uint8, device="cuda")
    Y = S.svdq_linear_forward(dw, Xd, workspace=ws)
    torch.cuda.synchronize()
    rows = None if M <= 1024 else rows_sample(M, 128, seed=len(name))
    check_activation(codes, sf, xl1, X, op, M, K, r, rows=rows)
    idx = np.arange(M) if rows is None else rows
    Y_ref, _, _, _ = O.linear_reference(X, op, b, rows=idx)
    check_output(from_dev_bf16(Y)[idx], Y_ref)


def test_mlp_pair_parity():
    """fc1 -> GELU (tanh, bf16, on the GPU) -> fc2 (K = 12288).  Each layer is
    compared with the oracle fed that layer's actual bf16 input."""
    S = _S()
    wl = SI.make_workload("flux_mlp")
    X = wl.X_bf16
    fc1, fc2 = wl.layers
    lp1, op1, dw1 = prepare(fc1.W, SI.channel_absmax(X), 32, fc1.bias_bf16)
    Y1 = S.svdq_linear_forward(dw1, to_dev_bf16(X))
    H = torch.nn.functional.gelu(Y1, approximate="tanh")
    Hb = from_dev_bf16(H)
    lp2, op2, dw2 = prepare(fc2.W, SI.channel_absmax(Hb), 32, fc2.bias_bf16)
    Y2 = S.svdq_linear_forward(dw2, H)
    torch.cuda.synchronize()
    rows = rows_sample(X.shape[0], 64, seed=5)
    Y1r, _, _, _ = O.linear_reference(X, op1, fc1.bias_bf16, rows=rows)
    check_output(from_dev_bf16(Y1)[rows], Y1r)
    Y2r, _, _, _ = O.linear_reference(Hb, op2, fc2.bias_bf16, rows=rows)
    check_output(from_dev_bf16(Y2)[rows], Y2r)


def test_flux_block_parity():
    """Config 4 (M = 18432): qkv -> out on the V slice of the qkv output
    (strided input, ldx = 9216) -> fc1 -> GELU (tanh, bf16, on the GPU) ->
    fc2 (K = 12288).  Each layer is calibrated on, and compared with the
    oracle fed, its actual bf16 input; codes and scales bit-exact and the
    output within tolerance on sampled rows."""
    S = _S()
    wl = SI.make_workload("flux_block")
    X = wl.X_bf16
    qkv, out, fc1, fc2 = wl.layers
    M, H = X.shape
    rows = rows_sample(M, 48, seed=9)

    def layer(lt, Xin_dev, Xin_bits):
        lp, op, dw = prepare(lt.W, SI.channel_absmax(Xin_bits), lt.spec.r, lt.bias_bf16)
        codes, sf, xl1 = S.svdq_quantize_act(dw, Xin_dev)
        Y = S.svdq_linear_forward(dw, Xin_dev)
        torch.cuda.synchronize()
        check_activation(codes, sf, xl1, Xin_bits, op, M, lt.spec.K, lt.spec.r, rows=rows)
        Yr, _, _, _ = O.linear_reference(Xin_bits, op, lt.bias_bf16, rows=rows)
        check_output(from_dev_bf16(Y)[rows], Yr)
        return Y

    Yq = layer(qkv, to_dev_bf16(X), X)
    V = Yq[:, 2 * H:]                       # strided view, ldx = 3 H
    assert V.stride(0) == 3 * H
    Yo = layer(out, V, from_dev_bf16(V))
    Y1 = layer(fc1, Yo, from_dev_bf16(Yo))
    G = torch.nn.functional.gelu(Y1, approximate="tanh")
    layer(fc2, G, from_dev_bf16(G))


def test_host_streamer_matches_forward():
    """The overlapped host-buffer path (three streams, two buffer sets) gives
    the device forward's output bit for bit, batch after batch."""
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
