"""Multi-rank logic of the benchmark on CPU: two gloo ranks, no GPU.

Each rank calibrates its own layer (seed = rank) with no collective on the data path; the
only collective is the max over ranks of the measured times, from which the whole-job
throughput is computed.
"""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    from scale_calibration_lh_b200 import synth

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # Rank-dependent "times": the max over ranks must come back on every rank.
        vals = bench.rank_max([1.0 + rank, 10.0 - rank, 0.5 * rank])
        layer = synth.make_layer("dense", rank, tokens=32, cin=32, rows=4)
        units, ops, acc_bytes = bench.algorithmic(layer)
        out[rank] = (vals, float(layer.w_f32().sum()), units, ops, acc_bytes)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_and_independent_layers():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    r0, r1 = out[0], out[1]
    assert r0[0] == r1[0] == [2.0, 10.0, 0.5]
    assert r0[1] != r1[1]  # each rank draws its own layer
    assert r0[2:] == r1[2:] == (4 * 2, 126 * 184, 32 * 32 * 2 + 2 * 1024)


def test_weak_scaling_value_and_single_process_identity():
    import bench

    assert bench.rank_max([3.0, 4.0]) == [3.0, 4.0]
    v1 = bench.weak_scaling_value(1000, 1, 2.0)
    v2 = bench.weak_scaling_value(1000, 2, 2.0)
    assert v1 == pytest.approx(500000.0) and v2 == pytest.approx(2 * v1)


def test_reference_arm_other_ranks_exit_silently(capsys):
    import argparse

    import bench

    args = argparse.Namespace(workload="dense", steps=1, warmup=3)
    bench.run_reference(args, rank=1, world=2)
    assert capsys.readouterr().out == ""
