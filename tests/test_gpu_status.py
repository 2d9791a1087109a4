"""Device-side failure detection and determinism of the tensor-core kernels,
through the C ABI.

* Every wait of the tensor-core kernels (Theta contractions, Theta gradient)
  on their own pipelines is bounded.  With the limit set to 1 ns the waits run
  out on purpose: the kernels record it, drain their own copies and MMAs, free
  tensor memory and return; ``tpconv_get_device_status`` reports
  TPCONV_ERR_TIMEOUT, validate mode returns it from the call, and the next call
  with the default limit is correct again (the context stays usable).  No
  kernel is made to fault or hang: the expiry is an ordinary, bounded exit.
* The Theta gradient sums its split-K partial tiles in a fixed order (no
  atomics), so repeated calls give bitwise identical dTheta and d_Theta.
"""

import numpy as np
import pytest

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def T():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import equivariant_gnn_tensor_receiver_b200 as T
    T.lib()
    return T


def setup(T, validate=False, gemm="fp32"):
    import torch
    c = W.CONFIGS["mace"]
    rowptr, col, vec = W.graph_for("mace", 0)
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"], gemm=gemm, validate=validate)
    N, E = len(rowptr) - 1, len(col)
    d = lambda a, t=torch.float32: torch.as_tensor(np.ascontiguousarray(a), dtype=t, device="cuda")
    G = T.Graph(d(rowptr, torch.int32), d(col, torch.int32), d(vec))
    x = d(W.normal((N, plan.dim_in), 201))
    th = d(W.theta([(plan.R * p["c_in"] * p["c_out"], 1 / np.sqrt(plan.R * p["c_in"])) for p in plan.paths], 202))
    g = d(W.normal((N, plan.dim_out), 203))
    ggx = d(W.normal((N, plan.dim_in), 204))
    ggv = d(W.normal((E, 3), 205))
    return plan, G, x, th, g, ggx, ggv


def test_theta_gradient_is_bitwise_repeatable(T):
    import torch
    plan, G, x, th, g, ggx, ggv = setup(T)
    a = T.backward(plan, G, x, th, g, want=("dtheta",))["dtheta"].clone()
    b = T.backward(plan, G, x, th, g, want=("dtheta",))["dtheta"].clone()
    c = T.double_backward(plan, G, x, th, g, ggx, ggv, None, want=("d_theta",))["d_theta"].clone()
    d = T.double_backward(plan, G, x, th, g, ggx, ggv, None, want=("d_theta",))["d_theta"].clone()
    torch.cuda.synchronize()
    assert float(a.abs().max()) > 0 and float(c.abs().max()) > 0
    assert torch.equal(a, b)
    assert torch.equal(c, d)


def test_expired_device_wait_is_reported_and_recovered(T):
    import torch
    L = T._lib
    plan, G, x, th, g, ggx, ggv = setup(T)
    good = T.forward(plan, G, x, th).clone()
    good_dth = T.backward(plan, G, x, th, g, want=("dtheta",))["dtheta"].clone()
    assert L.tpconv_get_device_status(plan) == L.TPCONV_OK
    try:
        L.tpconv_set_wait_limit(1)
        T.forward(plan, G, x, th)
        st_fwd = L.tpconv_get_device_status(plan)
        T.backward(plan, G, x, th, g, want=("dtheta",))
        st_bwd = L.tpconv_get_device_status(plan)
    finally:
        L.tpconv_set_wait_limit(0)
    assert st_fwd == L.TPCONV_ERR_TIMEOUT
    assert st_bwd == L.TPCONV_ERR_TIMEOUT
    # the record was cleared by the query, and the context is still usable
    assert L.tpconv_get_device_status(plan) == L.TPCONV_OK
    again = T.forward(plan, G, x, th)
    again_dth = T.backward(plan, G, x, th, g, want=("dtheta",))["dtheta"]
    torch.cuda.synchronize()
    assert L.tpconv_get_device_status(plan) == L.TPCONV_OK
    assert torch.equal(again, good)
    assert torch.equal(again_dth, good_dth)


def test_validate_mode_returns_timeout_from_the_call(T):
    L = T._lib
    plan, G, x, th, g, ggx, ggv = setup(T, validate=True)
    T.forward(plan, G, x, th)  # default limit: OK
    try:
        L.tpconv_set_wait_limit(1)
        with pytest.raises(L.TPConvError) as e:
            T.forward(plan, G, x, th)
    finally:
        L.tpconv_set_wait_limit(0)
    assert e.value.status == L.TPCONV_ERR_TIMEOUT
    out = T.forward(plan, G, x, th)  # and runs normally again
    assert float(out.abs().max()) > 0
