"""The multi-GPU host logic of bench.py on CPU: two gloo ranks.

The layer shards as independent token batches (replicas, no data-path
collective); the only cross-rank steps are the timing barrier and the
max-over-ranks of the elapsed time.  Both run here over gloo."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import svdq_inputs as SI
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w, lr = bench.dist_env()
        assert (r, w, lr) == (rank, world, rank)
        dist.barrier()
        elapsed = 10.0 + rank * 2.5
        got = bench.max_over_ranks(elapsed, world)
        spec = SI.workload_specs()["single_256"]
        X = bench.rank_activations(spec, rank, 32, 3072)
        out[rank] = (got, X.shape, float(np.abs(X.view(np.int16)).mean()), int(X[0, 0]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_reduction_and_batches():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 12.5          # max over ranks, same on every rank
    assert out[0][1] == out[1][1] == (32, 3072)    # same shape per rank (weak scaling)
    assert out[0][3] != out[1][3]                  # but each rank has its own tokens


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_layer_setup_shapes():
    """bench --layer: every layer of every workload gets an input of its own
    (M, K) shape, weights of (N, K), seeded (two calls agree)."""
    import bench
    import svdq_inputs as SI
    for name in ("flux_mlp",):
        spec = SI.workload_specs()[name]
        for i, ls in enumerate(spec.layers):
            ls2, W, b, X = bench.layer_setup(spec, i)
            assert ls2 == ls
            assert X.shape == (ls.M, ls.K) and X.dtype == np.uint16
            assert W.shape == (ls.N, ls.K) and b.shape == (ls.N,)
            _, _, _, X2 = bench.layer_setup(spec, i)
            assert np.array_equal(X, X2)
