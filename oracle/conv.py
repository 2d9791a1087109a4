"""The edge-conditioned CG tensor-product convolution, conventional schedule.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

Operator ("Sobek", arXiv 2607.18074, abstract: radial projection, spherical-
harmonic coupling, graph aggregation with fully connected multiplicity
mixing; the exact formula is a reading):

    out[r, i3, w, m3] = sum_{e : recv(e) = r} sum_{p -> i3} sum_u
                        W_e[p][u, w] * T_e[p, u, m3]
    W_e[p]            = sum_k b_k(|v_e|) Theta[p][k]              (C_in x C_out)
    T_e[p, u, m3]     = sum_{m1, m2} C_p[m1, m2, m3] x[send(e), i1, u, m1] Y_{l2, m2}(v_e)

Second operator family ("channelwise"; the abstract counts two operator
families without naming them, the reading taken is the channel-wise product):
every path keeps each channel on its own, W_e[p] = diag(sum_k b_k Theta[p][k])
with Theta[p] of shape R x C (C_in = C_out = C), so

    out[r, i3, u, m3] = sum_e sum_{p -> i3} w_e[p, u] * T_e[p, u, m3],
    w_e[p, u]         = sum_k b_k(|v_e|) Theta[p][k, u].

The abstract names the conventional schedule as the one that materialises
edge-specific weights, messages and adjoints; this module is exactly that
schedule (edge chunks keep host memory bounded): W_e and the message of every
edge are formed explicitly and scatter-added to receivers.  Backward and
double backward are the explicit adjoints; the abstract states that the
operator extends through forward, backward and double backward.

Graph: CSR by receiver -- ``rowptr[N+1]``, ``col[E]`` = sender of edge e,
``vec[E, 3]`` = pos[sender] - pos[receiver] (minimum image), all in CSR order.
"""

from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import irreps as _irreps
from . import radial as _radial
from . import so3 as _so3

EDGE_CHUNK = 2048


@dataclass
class Problem:
    irreps_in: str
    l_sh_max: int
    irreps_out: str
    R: int
    radial: str = "bessel"            # "gaussian" | "bessel"
    radial_params: tuple = (5.0,)     # (r_min, r_max) | (r_cut,)
    family: str = "full"              # "full" | "channelwise"
    paths: list = field(init=False)
    dim_in: int = field(init=False)
    dim_out: int = field(init=False)
    n_sh: int = field(init=False)
    theta_numel: int = field(init=False)

    def __post_init__(self):
        self.paths = _irreps.paths(self.irreps_in, self.l_sh_max, self.irreps_out, self.R, self.family)
        self.dim_in = _irreps.dim(_irreps.parse(self.irreps_in))
        self.dim_out = _irreps.dim(_irreps.parse(self.irreps_out))
        self.n_sh = (self.l_sh_max + 1) ** 2
        self.theta_numel = _irreps.theta_numel(self.paths, self.R, self.family)

    @property
    def channelwise(self) -> bool:
        return self.family == "channelwise"

    def theta_size(self, p) -> int:
        return self.R * p.c_in * (1 if self.channelwise else p.c_out)

    def theta_block(self, theta, p):
        """Theta[p]: (R, C_in, C_out), or (R, C) for the channel-wise family."""
        blk = theta[p.theta_off:p.theta_off + self.theta_size(p)]
        return blk.reshape(self.R, p.c_in) if self.channelwise else blk.reshape(self.R, p.c_in, p.c_out)


# Edge weights and their uses, per family.  Full: W (E, C_in, C_out); channel-wise:
# the diagonal w (E, C) of the same matrix.

def _weights(prob, b, Th):
    return np.einsum('ek,ku->eu', b, Th) if prob.channelwise else np.einsum('ek,kuw->euw', b, Th)


def _message(prob, W, T):
    """msg[e, w, m3] = sum_u W[e, u, w] T[e, u, m3]."""
    return W[:, :, None] * T if prob.channelwise else np.einsum('euw,euk->ewk', W, T, optimize=True)


def _weight_adjoint(prob, T, gr):
    """dW = d<g, msg>/dW  (full: (E, C_in, C_out); channel-wise: its diagonal (E, C))."""
    if prob.channelwise:
        return np.einsum('euk,euk->eu', T, gr)
    return np.einsum('euk,ewk->euw', T, gr, optimize=True)


def _message_adjoint(prob, W, gr):
    """dT[e, u, m3] = sum_w W[e, u, w] g_r[w, m3]."""
    return W[:, :, None] * gr if prob.channelwise else np.einsum('euw,ewk->euk', W, gr, optimize=True)


def receivers_of(rowptr) -> np.ndarray:
    rowptr = np.asarray(rowptr, dtype=np.int64)
    return np.repeat(np.arange(len(rowptr) - 1), np.diff(rowptr))


def geometry(prob: Problem, vec, order: int = 0):
    """Y (E, n_sh) and b (E, R); with order >= 1 also their Jacobians in v
    (E, n_sh, 3), (E, R, 3); with order 2 also Hessians (E, n_sh, 3, 3), (E, R, 3, 3)."""
    vec = np.asarray(vec, dtype=np.float64)
    Y = _so3.sh_all(prob.l_sh_max, vec)
    b, Jb, Hb = _radial.vector_derivs(prob.radial, vec, prob.R, prob.radial_params)
    if order == 0:
        return Y, b
    JY = _so3.sh_all_grad(prob.l_sh_max, vec)
    if order == 1:
        return Y, b, JY, Jb
    HY = _so3.sh_all_hess(prob.l_sh_max, vec)
    return Y, b, JY, Jb, HY, Hb


def _chunks(E, size=EDGE_CHUNK):
    for e0 in range(0, E, size):
        yield e0, min(E, e0 + size)


def _in_block(prob, x, send, p):
    n1 = 2 * p.l1 + 1
    return x[send, p.in_off:p.in_off + p.c_in * n1].reshape(len(send), p.c_in, n1)


def _out_block(prob, g, recv, p):
    n3 = 2 * p.l3 + 1
    return g[recv, p.out_off:p.out_off + p.c_out * n3].reshape(len(recv), p.c_out, n3)


def _sh_block(Y, l2):
    return Y[:, l2 * l2:(l2 + 1) * (l2 + 1)]


def forward_core(prob: Problem, N: int, send, recv, x, Y, b, theta):
    """out[N, dim_out]; every edge's weights and message are materialised."""
    out = np.zeros((N, prob.dim_out))
    E = len(send)
    for e0, e1 in _chunks(E):
        s, r = send[e0:e1], recv[e0:e1]
        for p in prob.paths:
            C = _so3.real_cg(p.l1, p.l2, p.l3)
            W = _weights(prob, b[e0:e1], prob.theta_block(theta, p))              # edge weights
            xs = _in_block(prob, x, s, p)
            T = np.einsum('ijk,eui,ej->euk', C, xs, _sh_block(Y[e0:e1], p.l2), optimize=True)
            msg = _message(prob, W, T)                                             # edge message
            n3 = 2 * p.l3 + 1
            np.add.at(out[:, p.out_off:p.out_off + p.c_out * n3], r, msg.reshape(len(r), -1))
    return out


def backward_core(prob: Problem, N: int, send, recv, x, Y, b, theta, g):
    """Adjoint of ``forward_core`` for cotangent g:  (dx, dtheta, dY, db)."""
    dx = np.zeros_like(x, dtype=np.float64)
    dtheta = np.zeros(prob.theta_numel)
    E = len(send)
    dY = np.zeros((E, prob.n_sh))
    db = np.zeros((E, prob.R))
    for e0, e1 in _chunks(E):
        s, r = send[e0:e1], recv[e0:e1]
        for p in prob.paths:
            C = _so3.real_cg(p.l1, p.l2, p.l3)
            Th = prob.theta_block(theta, p)
            W = _weights(prob, b[e0:e1], Th)
            xs = _in_block(prob, x, s, p)
            Ys = _sh_block(Y[e0:e1], p.l2)
            T = np.einsum('ijk,eui,ej->euk', C, xs, Ys, optimize=True)
            gr = _out_block(prob, g, r, p)
            dW = _weight_adjoint(prob, T, gr)                                     # weight adjoint
            n = prob.theta_size(p)
            # dTheta[k] = sum_e b_ek dW_e and db_ek = <Theta[k], dW_e>
            dtheta[p.theta_off:p.theta_off + n] += np.einsum('ek,e...->k...', b[e0:e1], dW).reshape(-1)
            if prob.channelwise:
                db[e0:e1] += np.einsum('ku,eu->ek', Th, dW)
            else:
                db[e0:e1] += np.einsum('kuw,euw->ek', Th, dW, optimize=True)
            dT = _message_adjoint(prob, W, gr)                                    # message adjoint
            dxs = np.einsum('ijk,ej,euk->eui', C, Ys, dT, optimize=True)
            n1 = 2 * p.l1 + 1
            np.add.at(dx[:, p.in_off:p.in_off + p.c_in * n1], s, dxs.reshape(len(s), -1))
            dY[e0:e1, p.l2 * p.l2:(p.l2 + 1) ** 2] += np.einsum('ijk,eui,euk->ej', C, xs, dT,
                                                                 optimize=True)
    return dx, dtheta, dY, db


def forward(prob: Problem, rowptr, col, vec, x, theta):
    N = len(rowptr) - 1
    recv = receivers_of(rowptr)
    send = np.asarray(col, dtype=np.int64)
    Y, b = geometry(prob, vec)
    return forward_core(prob, N, send, recv, np.asarray(x, np.float64), Y, b,
                        np.asarray(theta, np.float64))


def backward(prob: Problem, rowptr, col, vec, x, theta, g):
    """Gradients of <g, out>: dict(dx, dtheta, dvec, dY, db)."""
    N = len(rowptr) - 1
    recv = receivers_of(rowptr)
    send = np.asarray(col, dtype=np.int64)
    Y, b, JY, Jb = geometry(prob, vec, order=1)
    dx, dth, dY, db = backward_core(prob, N, send, recv, np.asarray(x, np.float64), Y, b,
                                    np.asarray(theta, np.float64), np.asarray(g, np.float64))
    dvec = np.einsum('em,emi->ei', dY, JY) + np.einsum('ek,eki->ei', db, Jb)
    return dict(dx=dx, dtheta=dth, dvec=dvec, dY=dY, db=db)


def double_backward(prob: Problem, rowptr, col, vec, x, theta, g,
                    gg_x=None, gg_vec=None, gg_theta=None):
    """Second-order terms for cotangents (gg_x, gg_vec, gg_theta) on (dx, dvec, dtheta).

    With Phi(g, x, Y, b, Theta) = <g, out> (linear in each slot),
    Ydot = J_Y gg_vec and bdot = J_b gg_vec, the scalar
        Psi = Phi(g, gg_x, Y, b, Th) + Phi(g, x, Y, b, gg_Th)
            + Phi(g, x, Ydot, b, Th) + Phi(g, x, Y, bdot, Th)
    equals <gg_x, dx> + <gg_theta, dtheta> + <gg_vec, dvec>.  Returned:
        d_g     = dPsi/dg,
        d_x     = dPsi/dx,
        d_theta = dPsi/dTheta,
        d_vec   = J_Y^T dPsi/dY + J_b^T dPsi/db
                  + sum_m dY_m Hess(Y_m) gg_vec + sum_k db_k Hess(b_k) gg_vec,
    where dY, db are the first-order adjoints.  A cotangent given as None is zero.
    """
    N = len(rowptr) - 1
    recv = receivers_of(rowptr)
    send = np.asarray(col, dtype=np.int64)
    x = np.asarray(x, np.float64)
    theta = np.asarray(theta, np.float64)
    g = np.asarray(g, np.float64)
    E = len(send)
    Y, b, JY, Jb, HY, Hb = geometry(prob, vec, order=2)

    d_g = np.zeros((N, prob.dim_out))
    d_x = np.zeros_like(x)
    d_theta = np.zeros(prob.theta_numel)
    dPsi_dY = np.zeros((E, prob.n_sh))
    dPsi_db = np.zeros((E, prob.R))
    d_vec = np.zeros((E, 3))

    def F(xx, YY, bb, th):
        return forward_core(prob, N, send, recv, xx, YY, bb, th)

    def B(xx, YY, bb, th):
        return backward_core(prob, N, send, recv, xx, YY, bb, th, g)

    if gg_x is not None:                       # term 1: x -> gg_x
        gg_x = np.asarray(gg_x, np.float64)
        d_g += F(gg_x, Y, b, theta)
        _, dth1, dY1, db1 = B(gg_x, Y, b, theta)
        d_theta += dth1
        dPsi_dY += dY1
        dPsi_db += db1
    if gg_theta is not None:                   # term 2: Theta -> gg_theta
        gg_theta = np.asarray(gg_theta, np.float64)
        d_g += F(x, Y, b, gg_theta)
        dx2, _, dY2, db2 = B(x, Y, b, gg_theta)
        d_x += dx2
        dPsi_dY += dY2
        dPsi_db += db2
    if gg_vec is not None:                     # terms 3, 4: Y -> Ydot, b -> bdot
        gg_vec = np.asarray(gg_vec, np.float64)
        Yd = np.einsum('emi,ei->em', JY, gg_vec)
        bd = np.einsum('eki,ei->ek', Jb, gg_vec)
        d_g += F(x, Yd, b, theta) + F(x, Y, bd, theta)
        dx3, dth3, _, db3 = B(x, Yd, b, theta)
        dx4, dth4, dY4, _ = B(x, Y, bd, theta)
        d_x += dx3 + dx4
        d_theta += dth3 + dth4
        dPsi_db += db3
        dPsi_dY += dY4
        _, _, dY0, db0 = B(x, Y, b, theta)
        d_vec += np.einsum('em,emij,ej->ei', dY0, HY, gg_vec)
        d_vec += np.einsum('ek,ekij,ej->ei', db0, Hb, gg_vec)
    d_vec += np.einsum('em,emi->ei', dPsi_dY, JY) + np.einsum('ek,eki->ei', dPsi_db, Jb)
    return dict(d_g=d_g, d_x=d_x, d_vec=d_vec, d_theta=d_theta)
