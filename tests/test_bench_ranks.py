"""Host-side logic of bench.py under several ranks (CPU, gloo, world size 2):
the max-over-ranks time, the whole-job throughput, and which ranks print."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, ws, port, times, out):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=timedelta(seconds=60))
    try:
        dist.barrier()
        got = bench.max_over_ranks(times[rank], ws, "cpu")
        got2 = bench.max_over_ranks(times[rank] * 2, ws, "cpu")  # a second collective, same order on all ranks
        dist.barrier()
        out.put((rank, got, got2))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ws = 2
    times = [3.25, 7.5]
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, ws, port, times, out)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res == [(0, 7.5, 15.0), (1, 7.5, 15.0)]


def test_single_process_keeps_its_time():
    assert bench.max_over_ranks(4.0, 1, "cpu") == 4.0


def test_job_throughput_scales_with_ranks():
    # 1e12 operations per rank and step in 1 ms: 1000 TOPS per rank
    assert bench.job_tops(1e12, 1, 1.0) == pytest.approx(1000.0)
    assert bench.job_tops(1e12, 8, 1.0) == pytest.approx(8000.0)


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        steps, warmup = 1, 3
    assert bench.run_reference(A(), 2, 1) is None
