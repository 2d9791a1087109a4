"""The multi-rank path of the benchmark on CPU: two gloo ranks, each with its
own graph (weak scaling, no data-path collective), reduced to one whole-job
figure = edges of all ranks / slowest rank's step time."""

import importlib.util
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B = _bench()
        import workloads as W
        rowptr, col, vec = W.graph_for("tiny", rank)  # each rank its own graph
        local_ms = [3.0, 5.0][rank]
        value, ms, edges = B.job_throughput(len(col), local_ms, world, torch.device("cpu"))
        mx = B.reduce_over_ranks(rank + 10.0, "max", world, torch.device("cpu"))
        q.put((rank, value, ms, edges, mx, len(col), int(col[:16].sum()), float(vec[0, 0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_job_throughput():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in procs:
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    e0, e1 = res[0][5], res[1][5]
    for r in (0, 1):
        _, value, ms, edges, mx, *_ = res[r]
        assert ms == 5.0 and edges == e0 + e1 and mx == 11.0
        assert np.isclose(value, (e0 + e1) / 5e-3)
    # distinct seeded graphs of the same workload on the two ranks
    assert (res[0][6], res[0][7]) != (res[1][6], res[1][7])


def test_single_rank_reduction_is_identity():
    B = _bench()
    assert B.reduce_over_ranks(7.5, "max", 1, None) == 7.5
    value, ms, edges = B.job_throughput(1000, 2.0, 1, None)
    assert (ms, edges) == (2.0, 1000.0) and np.isclose(value, 1000 / 2e-3)
