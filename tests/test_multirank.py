"""Host logic of the multi-GPU benchmark path, on CPU ranks over gloo (world size 2).

Verification shards by batch row with no data-path collective: each rank verifies its own
batch, and the job's time is the slowest rank's. These tests run that reduction and the
throughput arithmetic as two processes."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, times, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        ms_max = bench.max_over_ranks(times[rank], torch.device("cpu"), world)
        value = bench.job_value(512, 8, world, 100, ms_max)
        out.put((rank, ms_max, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(times):
    world = len(times)
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, times, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = [out.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return sorted(res)


def test_max_over_ranks_takes_slowest_rank():
    res = _run([12.5, 40.0])
    assert [r[1] for r in res] == [40.0, 40.0]  # every rank sees the job time


def test_job_value_counts_all_ranks_units():
    res = _run([10.0, 20.0])
    # 2 ranks x 512 rows x 8 positions x 100 steps in the slowest rank's 20 ms
    expect = 2 * 512 * 8 * 100 / 0.020
    for _, _, v in res:
        assert v == pytest.approx(expect)


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.25, torch.device("cpu"), 1) == 3.25
    assert bench.job_value(64, 5, 1, 10, 2.0) == pytest.approx(64 * 5 * 10 / 0.002)
