"""The N > 1 host path of bench.py on CPU: two gloo ranks (one process each)
reduce their timed regions and work exactly as the GPU ranks do over NCCL:
max over ranks of the time, sum over ranks of the work; every replica draws
its own noise seed."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        ms = [12.5, 20.0][rank]
        work = [3e12, 5e12][rank]
        ms_max, work_all = bench.reduce_over_ranks(ms, work, world, torch.device("cpu"))
        dist.barrier()
        results[rank] = (ms_max, work_all, bench.whole_job_tflops(work_all, ms_max), bench.replica_seed(7, rank))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_time_sum_work():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:   # no fork of a multi-threaded process
        results = m.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    assert set(res) == {0, 1}
    for rank in (0, 1):
        ms_max, work_all, value, _ = res[rank]
        assert ms_max == 20.0 and work_all == 8e12
        assert value == pytest.approx(8e12 / 20e-3 / 1e12)
    assert res[0][3] != res[1][3]                     # replicas draw different noise


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_over_ranks(3.0, 4.0, 1, torch.device("cpu")) == (3.0, 4.0)


def test_reference_arm_non_zero_rank_exits_quietly():
    """Under torchrun the reference arm runs on rank 0 only; rank 1 prints nothing and exits 0."""
    import subprocess
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", MASTER_ADDR="127.0.0.1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1"],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0
    assert r.stdout.strip() == ""
