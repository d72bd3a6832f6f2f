"""The multi-rank path of bench.py on CPU: two gloo ranks on 127.0.0.1.

Each rank runs its own batch element (independent attention problems, no data-path collective);
the only collective is the max over ranks of the step timings, and the whole-job throughput is
every rank's flops over that slowest time."""
import datetime
import os
import socket

import numpy as np


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from mxfp4_bit_attention_b200 import inputs
        t = bench.reduce_max(10.0 + 3.0 * rank, dist, device="cpu")
        w = bench.rank_workload(inputs.WORKLOADS["tiny"], rank)
        g = inputs.generate(w)
        results.put((rank, t, w.seed, w.B, g["q"][:4].copy()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_and_own_independent_problems():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    results = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(2):
        rank, t, seed, B, q = results.get(timeout=120)
        got[rank] = (t, seed, B, q)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0][0] == got[1][0] == 13.0          # every rank sees the slowest rank's time
    assert got[0][1] != got[1][1]                  # each rank its own seeded problem ...
    assert got[0][2] == got[1][2] == 1             # ... of one batch element
    assert not np.array_equal(got[0][3], got[1][3])


def test_whole_job_throughput_counts_every_rank():
    import bench
    one = bench.whole_job_tflops(1, 1.0e14, 100.0)
    assert abs(one - 1000.0) < 1e-9
    assert abs(bench.whole_job_tflops(4, 1.0e14, 100.0) - 4 * one) < 1e-9
