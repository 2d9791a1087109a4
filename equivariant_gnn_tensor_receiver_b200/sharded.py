"""One graph sharded over the ranks of a process group by receiver ranges.

The streaming schedule ("Sobek", arXiv 2607.18074, abstract) keeps its state
on the receiver side, so the natural split of one graph over GPUs is by
receivers: rank q owns the contiguous receiver range [r_lo(q), r_hi(q)) (edge
counts balanced), computes every edge that ends in it, and produces the
receiver-side outputs of that range.  What crosses ranks:

  forward          x rows of the senders of its edges: all-gather of the
                   owned x rows (every rank then reads the rows it needs).
  backward         dx: an edge contributes to its *sender*, which another
                   rank may own: each rank adds its contributions into a
                   [N][dim_in] buffer and a reduce-scatter sums them onto the
                   owners.  dTheta: all-reduce.  dvec stays with the edge.
  double backward  d_g: receiver-side, local.  d_x: reduce-scatter as dx.
                   d_Theta: all-reduce.  d_vec: local.

Each rank runs the single-GPU operator on its local graph: its owned
receivers first (local ids 0 .. n_own-1), then the senders it needs that it
does not own (halo nodes, empty segments).  The per-rank arithmetic comes from
``ops`` (the CUDA library's entry points on a GPU; any implementation with the
same three calls works), the exchanges from ``torch.distributed`` (NCCL over
NVLink on GPUs, gloo on CPUs).  Collectives go through the group in the same
order on every rank; ranges are padded to the largest one so that the
reduce-scatter and all-gather see equal chunks.
"""

from __future__ import annotations

import numpy as np


def receiver_ranges(rowptr, world: int):
    """Contiguous receiver ranges [lo, hi) per rank with balanced edge counts
    (every range cut at the receiver whose CSR offset crosses q * E / world)."""
    rowptr = np.asarray(rowptr, dtype=np.int64)
    N, E = len(rowptr) - 1, int(rowptr[-1])
    cuts = [0]
    for q in range(1, world):
        cuts.append(int(np.searchsorted(rowptr, q * E / world, side="left")))
    cuts.append(N)
    cuts = np.maximum.accumulate(np.minimum(np.array(cuts), N))
    return [(int(cuts[q]), int(cuts[q + 1])) for q in range(world)]


class LocalGraph:
    """The part of a receiver-CSR graph one rank computes (host arrays).

    nodes[i]   global id of local node i (owned receivers first, then halo senders)
    rowptr     local CSR over len(nodes) receivers (halo nodes: empty segments)
    col        local sender ids of the rank's edges
    edges      global CSR positions of those edges (for dvec / gg_vec)
    """

    def __init__(self, rowptr, col, lo: int, hi: int):
        rowptr = np.asarray(rowptr, dtype=np.int64)
        col = np.asarray(col, dtype=np.int64)
        e0, e1 = int(rowptr[lo]), int(rowptr[hi])
        self.lo, self.hi, self.n_own = lo, hi, hi - lo
        self.edges = np.arange(e0, e1, dtype=np.int64)
        send = col[e0:e1]
        halo = np.unique(send[(send < lo) | (send >= hi)])
        self.nodes = np.concatenate([np.arange(lo, hi, dtype=np.int64), halo])
        local = {int(g): i for i, g in enumerate(self.nodes)}
        self.col = np.fromiter((local[int(s)] for s in send), dtype=np.int64, count=len(send))
        self.rowptr = np.concatenate([rowptr[lo:hi + 1] - e0, np.full(len(halo), e1 - e0, dtype=np.int64)])
        self.N = len(self.nodes)
        self.E = e1 - e0


class ShardedConv:
    """Receiver-sharded forward / backward / double backward of one graph.

    ops: object with forward(lg, x, theta) -> out[lg.N], backward(lg, x, theta,
    g) -> (dx[lg.N], dtheta, dvec[lg.E]) and double_backward(lg, x, theta, g,
    gg_x, gg_vec, gg_theta) -> (d_g[lg.N], d_x[lg.N], d_vec[lg.E], d_theta),
    on torch tensors of the group's device.  Node arrays passed in and out are
    the rank's owned rows [lo, hi); theta is replicated.
    """

    def __init__(self, rowptr, col, rank: int, world: int, ops, device="cpu", group=None):
        import torch
        self.rank, self.world, self.ops, self.group = rank, world, ops, group
        self.device = torch.device(device)
        rowptr = np.asarray(rowptr, dtype=np.int64)
        self.N = len(rowptr) - 1
        self.ranges = receiver_ranges(rowptr, world)
        lo, hi = self.ranges[rank]
        self.local = LocalGraph(rowptr, col, lo, hi)
        self.chunk = max(h - l for l, h in self.ranges)  # padded rows per rank in the exchanges
        self._nodes = torch.as_tensor(self.local.nodes, device=self.device)
        # position of every global node in the padded, rank-major exchange layout
        pad_pos = np.empty(self.N, dtype=np.int64)
        for q, (l, h) in enumerate(self.ranges):
            pad_pos[l:h] = q * self.chunk + np.arange(h - l)
        self._pad_nodes = torch.as_tensor(pad_pos[self.local.nodes], device=self.device)

    # ---- exchanges -------------------------------------------------------------
    def gather_rows(self, own):
        """All-gather of the ranks' owned rows -> the rows of this rank's local nodes."""
        import torch
        import torch.distributed as dist
        own = own.contiguous()
        buf = torch.zeros((self.chunk,) + tuple(own.shape[1:]), dtype=own.dtype, device=self.device)
        buf[:own.shape[0]] = own
        full = torch.empty((self.world * self.chunk,) + tuple(own.shape[1:]), dtype=own.dtype, device=self.device)
        if self.world > 1:
            dist.all_gather_into_tensor(full, buf, group=self.group)
        else:
            full.copy_(buf)
        return full.index_select(0, self._pad_nodes)

    def scatter_rows(self, local_rows):
        """Contributions to local nodes (owned and halo) -> the sums for this rank's owned rows."""
        import torch
        import torch.distributed as dist
        full = torch.zeros((self.world * self.chunk,) + tuple(local_rows.shape[1:]), dtype=local_rows.dtype,
                           device=self.device)
        full.index_add_(0, self._pad_nodes, local_rows)
        out = torch.empty((self.chunk,) + tuple(local_rows.shape[1:]), dtype=local_rows.dtype, device=self.device)
        if self.world > 1:
            dist.reduce_scatter_tensor(out, full, group=self.group)
        else:
            out.copy_(full[:self.chunk])
        return out[:self.local.n_own]

    def all_sum(self, t):
        import torch.distributed as dist
        t = t.contiguous()
        if self.world > 1:
            dist.all_reduce(t, group=self.group)
        return t

    # ---- operator --------------------------------------------------------------
    def forward(self, x_own, theta):
        x = self.gather_rows(x_own)
        out = self.ops.forward(self.local, x, theta)
        return out[:self.local.n_own]

    def backward(self, x_own, theta, g_own):
        import torch
        x = self.gather_rows(x_own)
        g = torch.zeros((self.local.N,) + tuple(g_own.shape[1:]), dtype=g_own.dtype, device=self.device)
        g[:self.local.n_own] = g_own  # halo nodes receive no edges here
        dx, dtheta, dvec = self.ops.backward(self.local, x, theta, g)
        return self.scatter_rows(dx), self.all_sum(dtheta), dvec

    def double_backward(self, x_own, theta, g_own, gg_x_own=None, gg_vec=None, gg_theta=None):
        """gg_vec: the rank's own edges (local CSR order = global order of its range)."""
        import torch
        x = self.gather_rows(x_own)
        gg_x = self.gather_rows(gg_x_own) if gg_x_own is not None else None
        g = torch.zeros((self.local.N,) + tuple(g_own.shape[1:]), dtype=g_own.dtype, device=self.device)
        g[:self.local.n_own] = g_own
        d_g, d_x, d_vec, d_theta = self.ops.double_backward(self.local, x, theta, g, gg_x, gg_vec, gg_theta)
        return d_g[:self.local.n_own], self.scatter_rows(d_x), d_vec, self.all_sum(d_theta)


class LibraryOps:
    """The CUDA library's entry points on one rank's local graph (device tensors)."""

    def __init__(self, plan, edge_vec_local):
        import torch

        from . import api
        self.api, self.plan = api, plan
        self._graphs = {}
        self._vec = edge_vec_local.to(torch.float32).contiguous()

    def _graph(self, lg):
        import torch
        key = id(lg)
        if key not in self._graphs:
            dev = self._vec.device
            self._graphs[key] = self.api.Graph(torch.as_tensor(lg.rowptr, dtype=torch.int32, device=dev),
                                               torch.as_tensor(lg.col, dtype=torch.int32, device=dev), self._vec)
        return self._graphs[key]

    def forward(self, lg, x, theta):
        return self.api.forward(self.plan, self._graph(lg), x.contiguous(), theta)

    def backward(self, lg, x, theta, g):
        r = self.api.backward(self.plan, self._graph(lg), x.contiguous(), theta, g.contiguous())
        return r["dx"], r["dtheta"], r["dvec"]

    def double_backward(self, lg, x, theta, g, gg_x, gg_vec, gg_theta):
        c = lambda t: None if t is None else t.contiguous()
        r = self.api.double_backward(self.plan, self._graph(lg), x.contiguous(), theta, g.contiguous(), c(gg_x),
                                     c(gg_vec), c(gg_theta))
        return r["d_g"], r["d_x"], r["d_vec"], r["d_theta"]
