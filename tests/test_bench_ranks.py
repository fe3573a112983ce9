"""bench.py's multi-rank host logic on CPU: two gloo ranks, each with its own
timings, must both see the element-wise max, and the job value counts every
rank's units over that time (replicas: no data-path collective)."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import importlib.util
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
        bench = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(bench)
        tot, conv = bench.max_over_ranks([10.0 + rank, 3.0 - rank], world, torch.device("cpu"))
        out[rank] = (tot, conv, bench.job_value(1000, world, tot / 5))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_gloo_world2():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        res = dict(out)
    for r in range(world):
        tot, conv, value = res[r]
        assert tot == 11.0 and conv == 3.0
        assert value == pytest.approx(1000 * world / (11.0 / 5 / 1e3))
