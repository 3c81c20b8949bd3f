"""The N > 1 host path of bench.py on CPU: two gloo ranks (one process each)
reduce their timed regions and work exactly as the GPU ranks do over NCCL:
max over ranks of the time, sum over ranks of the work; every replica draws
its own noise seed.  The replica test runs the bench's own per-rank pieces on
a small chain workload: the replica inputs (same step 0, rank-specific drift),
the executed work of each rank's skip masks, the cross-rank reduction and the
JSON line rank 0 prints."""
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


def _replica_worker(rank, world, port, results):
    sys.path.insert(0, ROOT)
    import bench
    from block_sparse_attention_flash_b200 import inputs
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        wl = inputs.Workload("replica", 1, 2, 64, 4, 8, 16, 64, "lite", seed=11)
        qkv = bench.replica_chain(wl, rank, 3, torch.device("cpu"))
        sums = torch.tensor([float(t.float().sum()) for step in qkv for t in step], dtype=torch.float64)
        gathered = [torch.zeros_like(sums) for _ in range(world)]
        dist.all_gather(gathered, sums)
        # each rank's skip masks: rank r skips the first r + 1 k-blocks of every row after step 0
        nb = wl.nblocks
        skips = [torch.zeros(1, wl.H, nb, nb, dtype=torch.uint8) for _ in range(3)]
        for s in (1, 2):
            skips[s][..., : rank + 1] = 1
        flops = [bench.executed_flops(skips[s], wl.N, wl.block, wl.d) for s in (1, 2)]
        kern_ms = [[1.0, 1.5], [2.0, 2.5]][rank]
        ms_max, work_all = bench.reduce_over_ranks(sum(kern_ms), sum(flops), world, torch.device("cpu"))
        line = None
        if rank == 0:
            line = bench.assemble_line(wl, world, 2, 1, ms_max, work_all, kern_ms, flops)
        dist.barrier()
        results[rank] = ([g.tolist() for g in gathered], flops, ms_max, work_all, line)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_run_the_replica_path():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        results = m.dict()
        mp.spawn(_replica_worker, args=(world, port, results), nprocs=world, join=True)
        res = dict(results)
    gathered, flops0, ms_max, work_all, line = res[0]
    _, flops1, _, _, line1 = res[1]
    # step 0 is the workload's draw on every rank; the drift steps differ between replicas
    assert gathered[0][:3] == gathered[1][:3]
    assert gathered[0][3:] != gathered[1][3:]
    # 8 k-blocks of 64 tokens per row: rank 0 executes 7 of 8, rank 1 6 of 8
    dense = 4.0 * 64 * 512 * 512 * 2
    assert flops0 == [pytest.approx(dense * 7 / 8)] * 2 and flops1 == [pytest.approx(dense * 6 / 8)] * 2
    assert ms_max == 4.5 and work_all == pytest.approx(sum(flops0) + sum(flops1))
    assert line1 is None                                  # only rank 0 prints
    assert line["n_gpus"] == 2 and line["scaling"] == "weak" and line["steps"] == 2
    assert line["value"] == round(work_all / 4.5e-3 / 1e12, 2)   # summed work / slowest rank
    assert line["ms_per_step"] == pytest.approx(2.25)
    assert line["density"] == pytest.approx(7 / 8)         # rank 0's own launches
    assert line["config"]["parallelism"] == "replicas x2"


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
