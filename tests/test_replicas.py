"""The multi-GPU bench mode is independent replicas: every rank runs the same
workload, the job's time is the slowest rank's, and the throughput counts every
rank's units.  Checked here with two gloo ranks on the CPU (no GPU, no NCCL)."""
import multiprocessing as mp
import os
import socket
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, times, q):
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world)
    try:
        import bench
        ms = bench.max_over_ranks(times[rank], world)
        bench.barrier(world)
        q.put((rank, ms, bench.replica_throughput(1, 100, ms, world)))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_count_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    times = [40.0, 55.0]  # ms of 100 steps of one token each, per rank
    procs = [ctx.Process(target=_rank, args=(r, 2, port, times, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        got = sorted(q.get(timeout=120) for _ in procs)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for rank, ms, tput in got:
        assert ms == 55.0
        assert abs(tput - 2 * 100 / 0.055) < 1e-9


def test_one_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1) == 12.5
    assert abs(bench.replica_throughput(4, 10, 20.0, 1) - 4 * 10 / 0.020) < 1e-9
