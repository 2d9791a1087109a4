"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds none of the operator's arithmetic: it only draws graphs,
edge vectors and dense arrays from ``numpy.random.Generator(PCG64(seed))``.
Both the CPU oracle and the CUDA library consume what it returns.

Graphs are returned in receiver-sorted CSR form:
    rowptr[N+1] (int32), col[E] (int32, sender of each edge),
    vec[E, 3]  (float64, pos[sender] - pos[receiver], minimum image)
with edges of one receiver ordered by sender index (radius graphs) or by
draw order (random graphs).

Workload recipes (one per configuration of the layer):
    tiny   N=64, E=512, senders/receivers uniform, vec = uniform direction *
           U[0.5, 5]; 8x0e+8x1o, SH l<=2, R=4 Gaussian on [0.5, 5].
    mace   4096 atoms uniform in a periodic cube at 0.1 atoms/A^3, all pairs
           within 5 A; 64x0e+64x1o+64x2e, SH l<=3, R=8 Bessel (cosine cutoff).
    sweep  N=20000, periodic cube sized for mean degree d in {25..400}, 5 A
           cutoff; 32x0e+32x1o+32x2e, SH l<=2, R=8 Bessel.
    wide   N=8192, mean degree 32, 5 A cutoff; 128x0e+128x1o+128x2e+128x3o,
           SH l<=3, R=8 Bessel.
    dbl    graph and irreps of ``mace`` (double backward).
    capacity  irreps of ``mace`` on 1 222 309 atoms at the same density and
           cutoff (cube side 230.35 A): about 64 M edges, node-side state of
           107.6 GB if held at once, so it runs in receiver chunks.
Features x, cotangents g, gg ~ N(0, 1); Theta ~ N(0, std^2) with
std = 1/sqrt(R * C_in) per path block.
"""

from __future__ import annotations

import math

import numpy as np

CONFIGS = {
    "tiny": dict(irreps_in="8x0e+8x1o", irreps_out="8x0e+8x1o", l_sh_max=2, R=4,
                 radial="gaussian", radial_params=(0.5, 5.0)),
    "mace": dict(irreps_in="64x0e+64x1o+64x2e", irreps_out="64x0e+64x1o+64x2e", l_sh_max=3, R=8,
                 radial="bessel", radial_params=(5.0,)),
    "sweep": dict(irreps_in="32x0e+32x1o+32x2e", irreps_out="32x0e+32x1o+32x2e", l_sh_max=2, R=8,
                  radial="bessel", radial_params=(5.0,)),
    "wide": dict(irreps_in="128x0e+128x1o+128x2e+128x3o", irreps_out="128x0e+128x1o+128x2e+128x3o",
                 l_sh_max=3, R=8, radial="bessel", radial_params=(5.0,)),
}
CONFIGS["dbl"] = dict(CONFIGS["mace"])
CONFIGS["capacity"] = dict(CONFIGS["mace"])
CAPACITY_ATOMS = 1222309


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def _to_csr(N, send, recv, vec, order_key=None):
    """Stable sort by receiver (then by ``order_key`` inside a receiver)."""
    if order_key is None:
        perm = np.argsort(recv, kind="stable")
    else:
        perm = np.lexsort((order_key, recv))
    recv, send, vec = recv[perm], send[perm], vec[perm]
    counts = np.bincount(recv, minlength=N)
    rowptr = np.zeros(N + 1, dtype=np.int64)
    np.cumsum(counts, out=rowptr[1:])
    return rowptr.astype(np.int32), send.astype(np.int32), np.ascontiguousarray(vec, dtype=np.float64)


def random_graph(N: int, E: int, seed: int, r_min: float = 0.5, r_max: float = 5.0):
    """Senders and receivers uniform on [0, N); vec = random direction * U[r_min, r_max]."""
    g = rng(seed)
    send = g.integers(0, N, size=E)
    recv = g.integers(0, N, size=E)
    d = g.normal(size=(E, 3))
    d /= np.linalg.norm(d, axis=1, keepdims=True)
    vec = d * g.uniform(r_min, r_max, size=(E, 1))
    return _to_csr(N, send, recv, vec)


def box_for_degree(N: int, r_cut: float, degree: float) -> float:
    """Side of a periodic cube in which N uniform points have the given mean degree."""
    return (N * (4.0 / 3.0) * math.pi * r_cut ** 3 / degree) ** (1.0 / 3.0)


def radius_graph(N: int, box: float, r_cut: float, seed: int, node_batch: int = 65536):
    """All ordered pairs (s -> r), s != r, with minimum-image |pos_s - pos_r| < r_cut."""
    g = rng(seed)
    pos = g.uniform(0.0, box, size=(N, 3))
    if r_cut >= box / 2:
        raise ValueError("cutoff must be below half the box for minimum image")
    nc = int(box // r_cut)
    sends, recvs, vecs = [], [], []
    if nc < 3:
        for i0 in range(0, N, 1024):
            i1 = min(N, i0 + 1024)
            d = pos[None, :, :] - pos[i0:i1, None, :]          # (recv, send, 3)
            d -= box * np.round(d / box)
            r2 = (d * d).sum(-1)
            rr, ss = np.nonzero(r2 < r_cut * r_cut)
            rr = rr + i0
            keep = rr != ss
            recvs.append(rr[keep])
            sends.append(ss[keep])
            vecs.append(d[rr[keep] - i0, ss[keep]])
    else:
        cell = np.minimum((pos / (box / nc)).astype(np.int64), nc - 1)
        cid = (cell[:, 0] * nc + cell[:, 1]) * nc + cell[:, 2]
        order = np.argsort(cid, kind="stable")
        counts = np.bincount(cid, minlength=nc ** 3)
        start = np.zeros(nc ** 3 + 1, dtype=np.int64)
        np.cumsum(counts, out=start[1:])
        offs = [(a, b, c) for a in (-1, 0, 1) for b in (-1, 0, 1) for c in (-1, 0, 1)]
        for i0 in range(0, N, node_batch):
            ri = np.arange(i0, min(N, i0 + node_batch))
            for (a, b, c) in offs:
                nb = (((cell[ri, 0] + a) % nc) * nc + (cell[ri, 1] + b) % nc) * nc + (cell[ri, 2] + c) % nc
                cnt = counts[nb]
                rep = np.repeat(ri, cnt)
                first = np.repeat(start[nb], cnt)
                within = np.arange(cnt.sum()) - np.repeat(np.cumsum(cnt) - cnt, cnt)
                sj = order[first + within]
                d = pos[sj] - pos[rep]
                d -= box * np.round(d / box)
                r2 = (d * d).sum(-1)
                keep = (r2 < r_cut * r_cut) & (sj != rep)
                recvs.append(rep[keep])
                sends.append(sj[keep])
                vecs.append(d[keep])
    send = np.concatenate(sends)
    recv = np.concatenate(recvs)
    vec = np.concatenate(vecs)
    return _to_csr(N, send, recv, vec, order_key=send)


def normal(shape, seed: int, std: float = 1.0) -> np.ndarray:
    return rng(seed).normal(0.0, std, size=shape)


def theta(segments, seed: int) -> np.ndarray:
    """Concatenated N(0, std^2) blocks; ``segments`` = [(numel, std), ...]."""
    g = rng(seed)
    return np.concatenate([g.normal(0.0, s, size=n) for n, s in segments]) if segments else np.zeros(0)


def graph_for(name: str, seed: int, degree: float | None = None):
    """The graph of a named workload (see module docstring)."""
    if name == "tiny":
        return random_graph(64, 512, seed)
    if name in ("mace", "dbl"):
        return radius_graph(4096, (4096 / 0.1) ** (1.0 / 3.0), 5.0, seed)
    if name == "sweep":
        return radius_graph(20000, box_for_degree(20000, 5.0, degree or 25), 5.0, seed)
    if name == "wide":
        return radius_graph(8192, box_for_degree(8192, 5.0, 32), 5.0, seed)
    if name == "capacity":
        return radius_graph(CAPACITY_ATOMS, (CAPACITY_ATOMS / 0.1) ** (1.0 / 3.0), 5.0, seed)
    raise ValueError(name)
