"""The multi-GPU path is replicas only (each rank its own sequences, no data
collective): what the bench does across ranks is a barrier, the max of the
ranks' times and rank 0 alone reporting. That plumbing runs here on two gloo
ranks on CPU (127.0.0.1); the library itself is never called."""
import os
import socket
import sys
import types

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    sys.path.insert(0, ROOT)
    import torch.distributed as dist
    import bench
    try:
        w, r, _ = bench.dist_init()
        bench.barrier(w)
        m = bench.all_max(10.0 + 5.0 * r, w)          # each rank's "time"; all must agree on the max
        args = types.SimpleNamespace(workload="tiny_fp32", steps=1, warmup=0)
        line = bench.run_reference(args, w, r)       # the reference arm: rank 0 alone runs and reports
        bench.barrier(w)
        q.put((r, w, m, None if line is None else line.get("impl")))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_two_cpu_ranks_agree_on_the_max_time_and_only_rank0_reports():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(2):
            r, w, m, impl = q.get(timeout=180)
            results[r] = (w, m, impl)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert results[0] == (2, 15.0, "reference")
    assert results[1] == (2, 15.0, None)
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.all_max(3.5, 1) == 3.5
    bench.barrier(1)
