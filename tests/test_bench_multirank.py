"""The multi-process paths of bench.py on CPU with the gloo backend
(world size 2): rank aggregation (max over ranks, whole-job throughput) and
the reference arm, which rank 0 alone runs."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    world_, rank_, local_ = bench.dist_setup(world)
    try:
        assert (world_, rank_) == (world, rank)
        dev = torch.device("cpu")
        bench.barrier(world_, dev)
        # the slower rank (rank 1 here) sets the job's step time
        t = bench.max_over_ranks(10.0 + 5.0 * rank, world_, dev)
        results[rank] = (t, bench.job_throughput(2.0e12, t, world_))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    for rank in range(world):
        t, v = res[rank]
        assert t == 15.0
        assert v == pytest.approx(2 * 2.0e12 / 15e-3 / 1e12)


def _ref_worker(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    world_, rank_, _ = bench.dist_setup(world)
    calls = []
    try:
        class Args:
            workload, steps, warmup, ref_blocks = "tiny", 1, 3, 2
        import io
        import contextlib
        buf = io.StringIO()
        with contextlib.redirect_stdout(buf):
            bench.run_reference(Args, world_, rank_)
        results[rank] = buf.getvalue()
    finally:
        dist.destroy_process_group()


def test_reference_arm_runs_on_rank0_only_gloo():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_ref_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    import json
    line = json.loads(res[0].strip())
    assert line["impl"] == "reference" and line["n_gpus"] == 2 and line["value"] > 0
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert res[1] == ""


def test_job_throughput_single():
    assert bench.job_throughput(8.3e12, 10.0, 1) == pytest.approx(830.0)
