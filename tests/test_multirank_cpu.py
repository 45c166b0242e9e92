"""The multi-GPU path of the benchmark on CPU: two gloo ranks.

The layer runs as independent replicas (every token's quantisation and output
row are independent, weights are replicated), so the only cross-rank steps are
the max-over-ranks of the timings and the whole-job value, which counts the
work of all ranks."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import sys
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    # rank r pretends its 10 steps took 10 * (2 + r) ms, its kernels 1 + r and 0.5 ms
    out = bench.combine_ranks([10.0 * (2 + rank), 1.0 + rank, 0.5], 10, 1e12, world)
    dist.barrier()
    dist.destroy_process_group()
    q.put((rank, out))


def test_two_rank_combination_is_max_time_and_summed_work():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r]["times_ms"] == [30.0, 2.0, 0.5], "each timing is the max over ranks"
        assert res[r]["ms_per_step"] == pytest.approx(3.0)
        # 2 ranks x 1e12 ops per step in 3 ms -> 666.7 TOPS for the whole job
        assert res[r]["value"] == pytest.approx(2 * 1e12 / 3e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    out = bench.combine_ranks([20.0, 1.0, 0.5], 10, 1e12, 1)
    assert out["ms_per_step"] == pytest.approx(2.0)
    assert out["value"] == pytest.approx(500.0)
