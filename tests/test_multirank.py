"""The N > 1 bench logic on CPU: two gloo ranks, each timing its own replica;
the job's time is the slowest rank's and its throughput counts every rank's
tokens (weak scaling, no data-path collective).  The reference arm runs on
rank 0 only."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, ws, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    import bench
    ms = 10.0 + 5.0 * rank                       # rank 1 is the slower one
    slowest = bench.max_over_ranks(ms, ws, device="cpu")
    value = bench.job_throughput(131144, ws, slowest)
    bench.barrier(ws)
    # the reference arm: rank 0 prints, the others return without work
    class A:
        gpus, steps, warmup, workload = ws, 1, 0, "msa_128k_1m"
    ran = []

    class StubLeg:                               # the oracle itself is not what this test is about
        def __init__(self, parts=None):
            pass

        def run(self, seconds=0.0):
            ran.append(1)
            return {"value": 1.0, "unit": "tokens/s", "cores": 1, "kind": "oracle", "sample": "stub",
                    "extrapolated_step_s": 1.0}
    orig = bench.OracleLeg
    bench.OracleLeg = StubLeg
    try:
        bench.run_reference(A, rank, ws)
    finally:
        bench.OracleLeg = orig
    q.put((rank, slowest, value, len(ran)))
    dist.destroy_process_group()


def test_two_ranks_weak_scaling_and_reference_on_rank0():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, value, ran in res:
        assert slowest == 15.0
        assert value == pytest.approx(2 * 131144 / 0.015)
        assert ran == (1 if rank == 0 else 0)
