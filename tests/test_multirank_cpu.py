"""The multi-GPU host logic of bench.py on CPU: two gloo ranks (world size 2)
check that every rank gets its own independent problem (weak scaling, no
data-path collective), that timings reduce to the maximum over ranks on every
rank, and that the job throughput counts all ranks' work."""
import os
import socket
from datetime import timedelta

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        import bench
        import synth
        w = bench.rank_workload(synth.WORKLOADS[1], rank)
        x = synth.make_inputs(w)
        timings = bench.max_over_ranks([1.0 + rank, 10.0 - 3 * rank, 2.5], dist, torch.device("cpu"))
        out.put((rank, w.seed, float(x["q"].double().sum()), timings))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_independent_problems_and_max_timing():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, seed0, sum0, t0), (r1, seed1, sum1, t1) = res
    assert (r0, r1) == (0, 1)
    assert seed0 != seed1 and sum0 != sum1          # each rank times its own problem
    assert t0 == t1 == [2.0, 10.0, 2.5]             # the slowest rank sets each timing


def test_job_throughput_counts_every_rank():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.job_tflops(1, 2e12, 1000.0) == pytest.approx(2.0)
    assert bench.job_tflops(4, 2e12, 1000.0) == pytest.approx(8.0)
    assert bench.max_over_ranks([3.0, 1.0]) == [3.0, 1.0]
