"""Convenience layer over the C ABI: allocates outputs and workspace with torch
(the caching allocator owns all device memory) and caches the sender-sorted
view of a graph.  No arithmetic of the operator happens here."""

from __future__ import annotations

import torch

from . import _lib as L


class Graph:
    """Receiver-CSR graph on the device: rowptr[N+1], col[E] (senders), edge_vec[E, 3]."""

    def __init__(self, rowptr, col, edge_vec):
        self.rowptr = rowptr.to(torch.int32).contiguous()
        self.col = col.to(torch.int32).contiguous()
        self.edge_vec = edge_vec.to(torch.float32).contiguous()
        self.N = self.rowptr.numel() - 1
        self.E = self.col.numel()
        self._t = None

    def transposed(self, plan, stream=None):
        """(perm, s_rowptr, s_recv), computed once."""
        if self._t is None:
            dev = self.rowptr.device
            perm = torch.empty(max(self.E, 1), dtype=torch.int32, device=dev)
            s_rowptr = torch.empty(self.N + 1, dtype=torch.int32, device=dev)
            s_recv = torch.empty(max(self.E, 1), dtype=torch.int32, device=dev)
            ws = workspace(plan, L.OP_TRANSPOSE, self.N, self.E, dev)
            L.tpconv_graph_transpose(plan, self.N, self.E, self.rowptr, self.col, perm, s_rowptr, s_recv, ws,
                                     stream)
            self._t = (perm, s_rowptr, s_recv)
        return self._t


def workspace(plan, op, N, E, device):
    n = L.tpconv_workspace_size(plan, op, N, E)
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


def forward(plan, graph: Graph, x, theta, out=None, ws=None, stream=None):
    dev = x.device
    if out is None:
        out = torch.empty(graph.N, plan.dim_out, dtype=torch.float32, device=dev)
    if ws is None:
        ws = workspace(plan, L.OP_FORWARD, graph.N, graph.E, dev)
    L.tpconv_forward(plan, graph.N, graph.E, graph.rowptr, graph.col, graph.edge_vec, x, theta, out, ws, stream)
    return out


def backward(plan, graph: Graph, x, theta, g, want=("dx", "dtheta", "dvec"), ws=None, stream=None):
    dev = x.device
    E = graph.E
    outs = {
        "dx": torch.empty(graph.N, plan.dim_in, dtype=torch.float32, device=dev) if "dx" in want else None,
        "dtheta": torch.empty(plan.theta_numel, dtype=torch.float32, device=dev) if "dtheta" in want else None,
        "dvec": torch.empty(E, 3, dtype=torch.float32, device=dev) if "dvec" in want else None,
        "dY": torch.empty(E, plan.n_sh, dtype=torch.float32, device=dev) if "dY" in want else None,
        "db": torch.empty(E, plan.R, dtype=torch.float32, device=dev) if "db" in want else None,
    }
    perm = s_rowptr = s_recv = None
    if outs["dx"] is not None or outs["dtheta"] is not None:
        perm, s_rowptr, s_recv = graph.transposed(plan, stream)
    if ws is None:
        ws = workspace(plan, L.OP_BACKWARD, graph.N, graph.E, dev)
    L.tpconv_backward(plan, graph.N, E, graph.rowptr, graph.col, perm, s_rowptr, s_recv, graph.edge_vec, x, theta,
                      g, outs["dx"], outs["dtheta"], outs["dvec"], outs["dY"], outs["db"], ws, stream)
    return {k: v for k, v in outs.items() if v is not None}


def double_backward(plan, graph: Graph, x, theta, g, gg_x=None, gg_vec=None, gg_theta=None,
                    want=("d_g", "d_x", "d_vec", "d_theta"), ws=None, stream=None):
    dev = x.device
    outs = {
        "d_g": torch.empty(graph.N, plan.dim_out, dtype=torch.float32, device=dev) if "d_g" in want else None,
        "d_x": torch.empty(graph.N, plan.dim_in, dtype=torch.float32, device=dev) if "d_x" in want else None,
        "d_vec": torch.empty(graph.E, 3, dtype=torch.float32, device=dev) if "d_vec" in want else None,
        "d_theta": torch.empty(plan.theta_numel, dtype=torch.float32, device=dev) if "d_theta" in want else None,
    }
    perm, s_rowptr, s_recv = graph.transposed(plan, stream)
    if ws is None:
        ws = workspace(plan, L.OP_DOUBLE_BACKWARD, graph.N, graph.E, dev)
    L.tpconv_double_backward(plan, graph.N, graph.E, graph.rowptr, graph.col, perm, s_rowptr, s_recv,
                             graph.edge_vec, x, theta, g, gg_x, gg_vec, gg_theta, outs["d_g"], outs["d_x"],
                             outs["d_vec"], outs["d_theta"], ws, stream)
    return {k: v for k, v in outs.items() if v is not None}


# ---------------------------------------------------------------------------
# torch autograd glue: every product below runs in the library (C ABI); the
# Functions only route tensors.  d(out)/d(x, theta, edge_vec) is the library's
# backward; the backward of that backward is its double backward, so forces
# (-d energy / d positions) can themselves be differentiated.
# ---------------------------------------------------------------------------
class _ConvFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, theta, edge_vec, plan, graph):
        ctx.plan, ctx.graph = plan, graph
        ctx.save_for_backward(x, theta, edge_vec)
        return forward(plan, graph, x.contiguous(), theta.contiguous())

    @staticmethod
    def backward(ctx, g):
        x, theta, edge_vec = ctx.saved_tensors
        dx, dtheta, dvec = _ConvBwdFn.apply(x, theta, edge_vec, g.contiguous(), ctx.plan, ctx.graph)
        return dx, dtheta, dvec, None, None


class _ConvBwdFn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, theta, edge_vec, g, plan, graph):
        ctx.plan, ctx.graph = plan, graph
        ctx.save_for_backward(x, theta, edge_vec, g)
        r = backward(plan, graph, x.contiguous(), theta.contiguous(), g, want=("dx", "dtheta", "dvec"))
        return r["dx"], r["dtheta"], r["dvec"]

    @staticmethod
    def backward(ctx, gg_x, gg_theta, gg_vec):
        x, theta, edge_vec, g = ctx.saved_tensors
        c = lambda t: None if t is None else t.contiguous()
        r = double_backward(ctx.plan, ctx.graph, x.contiguous(), theta.contiguous(), g, c(gg_x), c(gg_vec),
                            c(gg_theta))
        return r["d_x"], r["d_theta"], r["d_vec"], r["d_g"], None, None


class TPConv(torch.nn.Module):
    """The streaming CG tensor-product convolution as a torch module.

    Holds Theta ([P][R][C_in][C_out], or [P][R][C] with ``family="channelwise"``;
    one normal block per path with standard deviation 1/sqrt(R C_in), 1/sqrt(R)
    channel-wise) as a parameter; ``forward(x, graph)`` returns
    out[N][dim_out] for the receiver-sorted ``Graph`` (its ``edge_vec`` may
    require grad).  Differentiable twice in x, Theta and the edge vectors.
    """

    def __init__(self, irreps_in, l_sh_max, irreps_out, R, device="cuda", **plan_options):
        super().__init__()
        self.plan = L.Plan(irreps_in, l_sh_max, irreps_out, R, **plan_options)
        cw = self.plan.family == "channelwise"
        blocks = [torch.randn(self.plan.R * p["c_in"] * (1 if cw else p["c_out"]))
                  / (self.plan.R * (1 if cw else p["c_in"])) ** 0.5 for p in self.plan.paths]
        self.theta = torch.nn.Parameter(torch.cat(blocks).to(device=device, dtype=torch.float32))

    def forward(self, x, graph: Graph):
        return _ConvFn.apply(x, self.theta, graph.edge_vec, self.plan, graph)
