"""svdq_linear_forward_static: the forward with the library's fixed device
scratch instead of a caller-given workspace.  Its output must equal
svdq_linear_forward's bit for bit (same kernels, same arithmetic), call after
call, whatever the previous call left in the scratch."""
import numpy as np
import pytest

import svdq_inputs as SI

S = pytest.importorskip("w4a4_rank_corrected_b200")


def _fake_weight(N=256, K=3072, r=32, base=0x10000000):
    w = S.SvdqWeight()
    w.N, w.K, w.r = N, K, r
    w.g_x = w.gs_x = w.g_w = w.alpha = w.lr_scale = 1.0
    w.smooth, w.l1_mma, w.l2_mma = base, base + 0x1000, base + 0x2000
    w.bias, w.codes_w, w.sf_w = base + 0x3000, base + 0x4000, base + 0x8000
    return w


def _max_rows(K, r):
    M = 0
    step = 1 << 14
    while step:
        if S.svdq_act_workspace_bytes(M + step, K, r) <= S.SVDQ_STATIC_WORKSPACE_BYTES:
            M += step
        else:
            step >>= 1
    return M


def test_static_forward_rejects_before_any_launch():
    """Errors that return before the device is touched (runs without a GPU)."""
    L = S.lib
    w = _fake_weight()
    X, Y = 0x20000000, 0x30000000
    Mmax = _max_rows(3072, 32)
    assert Mmax == 9033   # the example the header gives
    over = L.svdq_linear_forward_static(w, X, Mmax + 1, 3072, Y, 256, None)
    assert over == 4  # SVDQ_ERR_WORKSPACE
    assert L.svdq_linear_forward_static(w, X, 0, 3072, Y, 256, None) == 0
    assert L.svdq_linear_forward_static(w, None, 8, 3072, Y, 256, None) == 1
    assert L.svdq_linear_forward_static(w, X, 8, 3000, Y, 256, None) == 1
    assert L.svdq_linear_forward_static(w, X + 2, 8, 3072, Y, 256, None) == 3
    assert L.svdq_linear_forward_static(w, X, 8, 3076, Y, 256, None) == 3
    assert L.svdq_linear_forward_static(None, X, 8, 3072, Y, 256, None) == 1


@pytest.mark.gpu
def test_static_forward_matches_workspace_forward():
    import torch
    from gpu_common import from_dev_bf16, prepare, to_dev_bf16, check_output
    from oracle import svdq as O
    K, N, r = 1024, 640, 32
    rng_rows = [1000, 300]  # the second call is smaller: stale scratch must not leak in
    X0, W, b = SI.random_layer(77, max(rng_rows), K, N)
    lp, op, dw = prepare(W, SI.channel_absmax(X0), r, b)
    for i, M in enumerate(rng_rows):
        X, _, _ = SI.random_layer(100 + i, M, K, N)
        Xd = to_dev_bf16(X)
        Y_ws = S.svdq_linear_forward(dw, Xd)
        Y_st = S.svdq_linear_forward_static(dw, Xd)
        torch.cuda.synchronize()
        a, c = from_dev_bf16(Y_ws), from_dev_bf16(Y_st)
        assert np.array_equal(a, c), f"call {i}: static-scratch forward differs"
        rows = np.arange(0, M, 7)
        Y_ref, _, _, _ = O.linear_reference(X, op, b, rows=rows)
        check_output(c[rows], Y_ref)
    assert S.svdq_device_error() == 0


@pytest.mark.gpu
def test_static_forward_size_limit_on_device():
    import torch
    K, N, r = 3072, 256, 32
    X, W, b = SI.random_layer(5, 64, K, N)
    from gpu_common import prepare
    lp, op, dw = prepare(W, SI.channel_absmax(X), r, b)
    Mmax = _max_rows(K, r)
    Xbig = torch.zeros((Mmax + 1, K), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(S.SvdqError):
        S.svdq_linear_forward_static(dw, Xbig)
    # the largest allowed M runs: zero input gives the bias in every row
    Y = S.svdq_linear_forward_static(dw, Xbig[:Mmax])
    torch.cuda.synchronize()
    got = Y.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, np.broadcast_to(b, got.shape))
