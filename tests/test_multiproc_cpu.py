"""The multi-rank host logic of bench.py on CPU: two gloo ranks (world size 2).

The path has no data-path exchange (every output row is independent), so N GPUs run N
replicas; what N > 1 adds is host logic: every rank must agree on the slowest rank's step
time (max over ranks), and the whole-job rate counts every rank's bytes over that time.
"""
import datetime
import os
import socket

import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=2,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = [0.071, 0.074][rank]                    # this rank's step time
        ms_max = bench.max_over_ranks(ms, 2)
        bench.barrier(2)
        q.put((rank, ms_max, bench.job_gbs(262_416_896, ms_max, 2)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_agree_on_the_slowest_step_and_the_job_rate():
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms_max, gbs in out:
        assert ms_max == 0.074                       # both ranks see the slower rank's time
        assert abs(gbs - 2 * 262_416_896 / 0.074 / 1e6) < 1e-6


def test_single_rank_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(0.5, 1) == 0.5
    assert bench.job_gbs(1e9, 1.0, 1) == 1000.0      # 1 GB in 1 ms = 1000 GB/s
