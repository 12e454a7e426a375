"""Host side of the benchmark's multi-process path, on CPU with gloo.

With N > 1 GPUs every rank runs its own independent problem; the only
cross-rank steps are a barrier around each timed region and the maximum of
the per-rank device times.  These run here as two gloo ranks on 127.0.0.1:
the reported time is the slowest rank's, every rank takes the same
collective steps, and `value` counts the units of all ranks.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, times, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank), "W8_BENCH_BACKEND": "gloo"})
    import bench
    ws, r, local = bench.dist_setup()
    assert (ws, r, local) == (world, rank, rank)
    bench.barrier(ws)
    t = bench.max_over_ranks(ws, times[rank], torch.device("cpu"))
    bench.barrier(ws)
    # the aggregate is units of all ranks over the slowest rank's time
    units_per_rank = 1000
    value = ws * units_per_rank / t
    out[rank] = (t, value)
    dist.destroy_process_group()


@pytest.mark.parametrize("times", [(0.25, 0.5), (0.75, 0.125)])
def test_two_gloo_ranks_report_the_slowest_rank(times):
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    slowest = max(times)
    for r in range(world):
        t, value = out[r]
        assert t == slowest
        assert value == pytest.approx(world * 1000 / slowest)


def test_single_rank_needs_no_process_group():
    import bench
    os.environ.pop("WORLD_SIZE", None)
    ws, rank, local = bench.dist_setup()
    assert (ws, rank, local) == (1, 0, 0)
    assert bench.max_over_ranks(1, 0.5, torch.device("cpu")) == 0.5
    bench.barrier(1)


def test_tensor_peak_follows_the_region_length():
    import bench
    assert bench.tensor_peak(0.14, 1617.4, 1370.6) == (1617.4, "bf16_tflops (burst)")
    assert bench.tensor_peak(5.0, 1617.4, 1370.6) == (1370.6, "bf16_tflops_sustained")
    assert bench.tensor_peak(5.0, 1617.4, 0.0)[0] == 1617.4


def test_cpu_baseline_slabs_give_the_oracles_whole_result():
    # the CPU baseline drives the unchanged oracle over column slabs on
    # several threads; the joined result must be the whole-matrix one
    import numpy as np
    import bench
    import oracle
    import synthetic
    W = synthetic.weights(128, 700, 1, 5, outlier_frac=0.01)
    X = synthetic.activations(3, 128, 1, 6)
    runner = bench.SlabRunner(4)
    q, s = bench.oracle_quantize_threads(W, runner)
    q0, s0 = oracle.quantize(W)
    assert np.array_equal(q, q0) and np.array_equal(s.view(np.uint16), s0.view(np.uint16))
    parts = bench.oracle_linear_timer(X, q, s, runner)()
    runner.close()
    assert np.array_equal(np.concatenate(parts, axis=1), oracle.linear(X, q0, s0))
