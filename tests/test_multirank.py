"""Multi-rank paths on CPU with gloo ranks.

* Replicas: two ranks, each with its own graph (weak scaling, no data-path
  collective), reduced to one whole-job figure = edges of all ranks / slowest
  rank's step time.
* One graph sharded by receiver ranges (2 and 3 ranks): the assembled results
  of forward, backward and double backward equal the single-rank fp64 oracle.
* Failure on the host: a rank that leaves between operations makes the peer's
  next collective end with an error within the process group's timeout.
"""

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


# ---- one graph sharded over ranks by receiver ranges (host logic + collectives) ----

class _OracleOps:
    """The fp64 oracle on a rank's local graph: stands in for the library on CPU ranks."""

    def __init__(self, prob, vec_local):
        self.prob, self.vec = prob, vec_local

    def forward(self, lg, x, theta):
        import torch
        from oracle import conv
        return torch.as_tensor(conv.forward(self.prob, lg.rowptr, lg.col, self.vec, x.numpy(), theta.numpy()))

    def backward(self, lg, x, theta, g):
        import torch
        from oracle import conv
        r = conv.backward(self.prob, lg.rowptr, lg.col, self.vec, x.numpy(), theta.numpy(), g.numpy())
        return tuple(torch.as_tensor(r[k]) for k in ("dx", "dtheta", "dvec"))

    def double_backward(self, lg, x, theta, g, gg_x, gg_vec, gg_theta):
        import torch
        from oracle import conv
        n = lambda t: None if t is None else t.numpy()
        r = conv.double_backward(self.prob, lg.rowptr, lg.col, self.vec, x.numpy(), theta.numpy(), g.numpy(),
                                 n(gg_x), n(gg_vec), n(gg_theta))
        return tuple(torch.as_tensor(r[k]) for k in ("d_g", "d_x", "d_vec", "d_theta"))


SHARD_CASE = dict(irr="4x0e+4x1o+2x2e", lsh=2, R=3, N=90, box=11.0)


def _shard_inputs():
    import workloads as W
    from oracle import conv
    c = SHARD_CASE
    rowptr, col, vec = W.radius_graph(c["N"], c["box"], 5.0, 13)
    prob = conv.Problem(c["irr"], c["lsh"], c["irr"], c["R"], "bessel", (5.0,))
    N, E = len(rowptr) - 1, len(col)
    x = W.normal((N, prob.dim_in), 1)
    th = W.theta([(c["R"] * p.c_in * p.c_out, 0.3) for p in prob.paths], 2)
    g = W.normal((N, prob.dim_out), 3)
    ggx, ggv, ggt = W.normal((N, prob.dim_in), 4), W.normal((E, 3), 5), W.normal(th.shape, 6) * 0.1
    return prob, (rowptr, col, vec), (x, th, g, ggx, ggv, ggt)


def _shard_rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from equivariant_gnn_tensor_receiver_b200.sharded import ShardedConv
        prob, (rowptr, col, vec), (x, th, g, ggx, ggv, ggt) = _shard_inputs()
        sc = ShardedConv(rowptr, col, rank, world, None)
        lg = sc.local
        sc.ops = _OracleOps(prob, vec[lg.edges])
        T = lambda a: torch.as_tensor(np.ascontiguousarray(a))
        lo, hi = lg.lo, lg.hi
        out = sc.forward(T(x[lo:hi]), T(th))
        dx, dth, dvec = sc.backward(T(x[lo:hi]), T(th), T(g[lo:hi]))
        d_g, d_x, d_vec, d_th = sc.double_backward(T(x[lo:hi]), T(th), T(g[lo:hi]), T(ggx[lo:hi]), T(ggv[lg.edges]),
                                                   T(ggt))
        q.put((rank, lo, hi, lg.edges[0] if lg.E else 0, lg.E,
               {k: v.numpy() for k, v in dict(out=out, dx=dx, dth=dth, dvec=dvec, d_g=d_g, d_x=d_x, d_vec=d_vec,
                                              d_th=d_th).items()}))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_receiver_sharded_graph_matches_single_rank(world):
    """One graph over `world` gloo ranks by receiver ranges: all-gather of x,
    reduce-scatter of the sender-side gradients, all-reduce of the Theta
    gradients.  The assembled results equal the single-rank oracle (fp64)."""
    import torch.multiprocessing as mp
    from oracle import conv
    from equivariant_gnn_tensor_receiver_b200.sharded import receiver_ranges
    prob, (rowptr, col, vec), (x, th, g, ggx, ggv, ggt) = _shard_inputs()
    ranges = receiver_ranges(rowptr, world)
    assert ranges[0][0] == 0 and ranges[-1][1] == len(rowptr) - 1
    assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ref = dict(out=conv.forward(prob, rowptr, col, vec, x, th))
    rb = conv.backward(prob, rowptr, col, vec, x, th, g)
    rd = conv.double_backward(prob, rowptr, col, vec, x, th, g, ggx, ggv, ggt)
    ref.update(dx=rb["dx"], dth=rb["dtheta"], dvec=rb["dvec"], d_g=rd["d_g"], d_x=rd["d_x"], d_vec=rd["d_vec"],
               d_th=rd["d_theta"])
    got = {k: np.zeros_like(v) for k, v in ref.items()}
    for rank, lo, hi, e0, ne, r in res:
        for k in ("out", "dx", "d_g", "d_x"):
            got[k][lo:hi] = r[k]
        for k in ("dvec", "d_vec"):
            got[k][e0:e0 + ne] = r[k]
        for k in ("dth", "d_th"):  # all-reduced: identical on every rank
            got[k] = r[k]
    for k in ref:
        scale = max(np.abs(ref[k]).max(), 1e-30)
        assert np.abs(got[k] - ref[k]).max() / scale < 1e-12, k


def _shard_rank_leaves(rank, world, port, q):
    """Rank 1 leaves before the backward's collectives (between operations,
    nothing in flight); rank 0's next collective must end with an error within
    the process group's timeout instead of waiting for good."""
    import datetime
    import time

    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=3))
    from equivariant_gnn_tensor_receiver_b200.sharded import ShardedConv
    prob, (rowptr, col, vec), (x, th, g, ggx, ggv, ggt) = _shard_inputs()
    sc = ShardedConv(rowptr, col, rank, world, None)
    lg = sc.local
    sc.ops = _OracleOps(prob, vec[lg.edges])
    T = lambda a: torch.as_tensor(np.ascontiguousarray(a))
    lo, hi = lg.lo, lg.hi
    sc.forward(T(x[lo:hi]), T(th))  # both ranks complete one operation
    if rank == 1:
        q.put((rank, "left", 0.0))
        q.close()
        q.join_thread()  # flush the message, then vanish
        os._exit(0)  # no destroy_process_group: the peer simply disappears
    t0 = time.monotonic()
    try:
        sc.backward(T(x[lo:hi]), T(th), T(g[lo:hi]))
        q.put((rank, "completed", time.monotonic() - t0))
    except Exception as e:  # gloo reports the lost peer or the timeout
        q.put((rank, "error:" + type(e).__name__, time.monotonic() - t0))
    q.close()
    q.join_thread()
    os._exit(0)


def test_sharded_rank_that_leaves_is_detected_by_the_peer():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_shard_rank_leaves, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict((r, (s, t)) for r, s, t in (q.get(timeout=120) for _ in procs))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert res[1][0] == "left"
    status, waited = res[0]
    assert status.startswith("error:"), status
    assert waited < 60.0
