"""The allocation-free forward entry point (``tpconv_forward_static``), through
the C ABI, against ``tpconv_forward`` with a caller workspace and against the
fp64 oracle.

Collected last (file name) so that it also runs after the other GPU tests have
used the device.  Tolerance: the fp32 bar of the parity tests (max-norm
relative error <= 1e-5); the two entry points run the same kernels in the same
order, so their results are expected to agree exactly.  The cases run in an
order that leaves the fixed scratch full of another plan's data before each
call: the chunked mace-like layer first, then the tiny layer on what it left.
"""

import numpy as np
import pytest

import workloads as W
from oracle import conv

pytestmark = pytest.mark.gpu

TOL_FP32 = 1e-5


@pytest.fixture(scope="module")
def T():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import equivariant_gnn_tensor_receiver_b200 as T
    T.lib()
    return T


def rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    d = np.abs(b).max()
    return np.abs(a - b).max() / (d if d > 0 else 1.0)


def inputs(name, cap):
    import equivariant_gnn_tensor_receiver_b200 as T
    import torch
    c = W.CONFIGS[name]
    rowptr, col, vec = W.graph_for(name, 0)
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"], workspace_cap=cap)
    N, E = len(rowptr) - 1, len(col)
    d = lambda a, t: torch.as_tensor(np.ascontiguousarray(a), dtype=t, device="cuda")
    x = d(W.normal((N, plan.dim_in), 21), torch.float32)
    th = d(W.theta([(plan.R * p["c_in"] * p["c_out"], 1 / np.sqrt(plan.R * p["c_in"])) for p in plan.paths], 22),
           torch.float32)
    return plan, N, E, d(rowptr, torch.int32), d(col, torch.int32), d(vec, torch.float32), x, th


def oracle_rows(name, rows, rowptr, col, vec, x, th):
    """The oracle's out for the listed receivers (exact from their own edges)."""
    c = W.CONFIGS[name]
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"],
                        tuple(c["radial_params"]))
    rowptr, col = rowptr.cpu().numpy(), col.cpu().numpy()
    N = len(rowptr) - 1
    recv = np.repeat(np.arange(N), np.diff(rowptr))
    em = np.isin(recv, rows)
    sub = np.concatenate([[0], np.cumsum(np.bincount(recv[em], minlength=N))])
    v = vec.double().cpu().numpy()[em]
    ref = conv.forward(prob, sub, col[em], v, x.double().cpu().numpy(), th.double().cpu().numpy())
    return ref[rows]


@pytest.mark.parametrize("name,cap", [("mace", 32 << 20), ("tiny", 0)])
def test_static_forward_matches_workspace_forward(T, name, cap):
    import torch
    L = T._lib
    plan, N, E, rowptr, col, vec, x, th = inputs(name, cap)
    need = L.tpconv_workspace_size(plan, L.OP_FORWARD, N, E)
    assert need <= L.STATIC_SCRATCH_BYTES  # fits the library's fixed scratch
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    ref = torch.empty(N, plan.dim_out, dtype=torch.float32, device="cuda")
    L.tpconv_forward(plan, N, E, rowptr, col, vec, x, th, ref, ws)
    torch.cuda.synchronize()
    ref_h = ref.cpu().numpy()
    assert np.abs(ref_h).max() > 0
    rows = np.arange(N) if N <= 64 else np.random.default_rng(5).choice(N, 24, replace=False)
    exact = oracle_rows(name, rows, rowptr, col, vec, x, th)
    for _ in range(2):  # two calls in a row: the second reuses the scratch the first left behind
        out = torch.full((N, plan.dim_out), float("nan"), dtype=torch.float32, device="cuda")
        L.tpconv_forward_static(plan, N, E, rowptr, col, vec, x, th, out)
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        assert rel(got, ref_h) <= TOL_FP32
        assert rel(got[rows], exact) <= TOL_FP32


def test_static_forward_rejects_oversized_problem(T):
    import torch
    L = T._lib
    plan, N, E, rowptr, col, vec, x, th = inputs("mace", 0)  # no cap: one chunk of 4096 nodes
    assert L.tpconv_workspace_size(plan, L.OP_FORWARD, N, E) > L.STATIC_SCRATCH_BYTES
    out = torch.zeros(N, plan.dim_out, dtype=torch.float32, device="cuda")
    with pytest.raises(L.TPConvError) as e:
        L.tpconv_forward_static(plan, N, E, rowptr, col, vec, x, th, out)
    assert e.value.status == L.TPCONV_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert float(out.abs().max()) == 0.0  # rejected before any device work
