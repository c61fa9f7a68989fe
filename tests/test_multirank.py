"""Multi-rank host logic of bench.py on CPU (gloo, 2 ranks): the per-step time
is the slowest rank's, the whole-job throughput sums the ranks' independent
workloads, and the reference arm runs on rank 0 only."""
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


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from gsa_inputs import CONFIGS
        per_rank_ms = [12.0, 17.5][rank]
        ms = bench.max_over_ranks(per_rank_ms, dist)
        value = bench.throughput(world, 1000, ms)

        class A:
            steps, warmup, ref_windows = 1, 0, 8
        cfg = CONFIGS["tiny_fp32"]
        ref = bench.run_reference(A, cfg, rank, world)
        dist.barrier()
        q.put((rank, ms, value, ref is None, None if ref is None else ref["impl"]))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_reference_arm():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, ms0, v0, none0, impl0), (r1, ms1, v1, none1, impl1) = res
    assert ms0 == ms1 == 17.5                       # slowest rank
    assert v0 == v1 == pytest.approx(2 * 1000 / 0.0175)
    assert not none0 and impl0 == "reference"       # rank 0 runs the oracle arm
    assert none1                                    # other ranks do no work
