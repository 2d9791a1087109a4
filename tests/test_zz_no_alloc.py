"""The allocation-free forward entry point (``tpconv_forward_static``) against
``tpconv_forward`` with a caller workspace, through the C ABI.

Collected last (file name) so that it also runs after the other GPU tests have
used the device.  Tolerance: the fp32 bar of the parity tests (max-norm
relative error <= 1e-5); both calls run the same kernels in the same order, so
the results are expected to agree exactly.
"""

import numpy as np
import pytest

import workloads as W

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


@pytest.mark.parametrize("name,cap", [("tiny", 0), ("mace", 32 << 20)])
def test_static_forward_matches_workspace_forward(T, name, cap):
    import torch
    L = T._lib
    plan, N, E, rowptr, col, vec, x, th = inputs(name, cap)
    need = L.tpconv_workspace_size(plan, L.OP_FORWARD, N, E)
    assert need <= 64 << 20  # fits the library's fixed scratch
    ws = torch.empty(max(need, 256), dtype=torch.uint8, device="cuda")
    ref = torch.empty(N, plan.dim_out, dtype=torch.float32, device="cuda")
    L.tpconv_forward(plan, N, E, rowptr, col, vec, x, th, ref, ws)
    torch.cuda.synchronize()
    ref_h = ref.cpu().numpy()
    assert np.abs(ref_h).max() > 0
    for _ in range(2):  # two calls in a row: the second reuses the scratch the first left behind
        out = torch.full((N, plan.dim_out), float("nan"), dtype=torch.float32, device="cuda")
        L.tpconv_forward_static(plan, N, E, rowptr, col, vec, x, th, out)
        torch.cuda.synchronize()
        assert rel(out.cpu().numpy(), ref_h) <= TOL_FP32


def test_static_forward_rejects_oversized_problem(T):
    import torch
    L = T._lib
    plan, N, E, rowptr, col, vec, x, th = inputs("mace", 0)  # no cap: one chunk of 4096 nodes
    assert L.tpconv_workspace_size(plan, L.OP_FORWARD, N, E) > 64 << 20
    out = torch.zeros(N, plan.dim_out, dtype=torch.float32, device="cuda")
    with pytest.raises(L.TPConvError) as e:
        L.tpconv_forward_static(plan, N, E, rowptr, col, vec, x, th, out)
    assert e.value.status == L.TPCONV_ERR_WORKSPACE_TOO_SMALL
    torch.cuda.synchronize()
    assert float(out.abs().max()) == 0.0  # rejected before any device work
