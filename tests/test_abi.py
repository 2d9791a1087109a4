"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/tpconv.h declares, plans match the oracle's path table,
the device CG table (Racah construction) agrees with the oracle's independent
null-space construction, errors are reported, workspace is edge-independent."""

import ctypes
import os
import re

import numpy as np
import pytest

import workloads as W
from oracle import conv, so3

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def T():
    from equivariant_gnn_tensor_receiver_b200 import build
    build.build(verbose=False)
    import equivariant_gnn_tensor_receiver_b200 as T
    return T


def test_exports_every_declared_symbol(T):
    hdr = open(os.path.join(ROOT, "include", "tpconv.h")).read()
    declared = set(re.findall(r"\b(tpconv_\w+)\s*\(", hdr))
    assert declared == set(T.exported_names())
    L = ctypes.CDLL(T._lib.LIB_PATH)
    for name in declared:
        assert hasattr(L, name), name


@pytest.mark.parametrize("name", ["tiny", "mace", "sweep", "wide"])
def test_plan_matches_oracle_path_table(T, name):
    c = W.CONFIGS[name]
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"])
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"], c["radial_params"])
    assert plan.n_paths == len(prob.paths)
    assert (plan.dim_in, plan.dim_out, plan.n_sh, plan.theta_numel) == (prob.dim_in, prob.dim_out, prob.n_sh,
                                                                          prob.theta_numel)
    for a, p in zip(plan.paths, prob.paths):
        assert (a["l1"], a["l2"], a["l3"], a["c_in"], a["c_out"], a["theta_offset"]) == (
            p.l1, p.l2, p.l3, p.c_in, p.c_out, p.theta_off)


@pytest.mark.parametrize("name", ["tiny", "mace", "wide"])
def test_channelwise_plan_matches_oracle_path_table(T, name):
    c = W.CONFIGS[name]
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"], family="channelwise")
    prob = conv.Problem(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], c["radial"], c["radial_params"],
                        family="channelwise")
    assert (plan.n_paths, plan.theta_numel) == (len(prob.paths), prob.theta_numel)
    assert [a["theta_offset"] for a in plan.paths] == [p.theta_off for p in prob.paths]
    # the node-side state does not depend on the family
    full = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], radial=c["radial"],
                  radial_params=c["radial_params"])
    L = T._lib
    for op in (L.OP_FORWARD, L.OP_BACKWARD, L.OP_DOUBLE_BACKWARD):
        a = L.tpconv_workspace_size(plan, op, 1000, 20000)
        b = L.tpconv_workspace_size(full, op, 1000, 20000)
        assert a <= b


def test_channelwise_needs_equal_multiplicities(T):
    with pytest.raises(T._lib.TPConvError) as e:
        T.Plan("4x0e+2x1o", 1, "3x0e+2x1o", 2, family="channelwise")
    assert e.value.status == 1


def test_cg_table_matches_null_space_construction(T):
    worst = 0.0
    for l1 in range(4):
        for l2 in range(4):
            for l3 in range(abs(l1 - l2), min(l1 + l2, 3) + 1):
                got = T.tpconv_cg_coefficients(l1, l2, l3)
                want = so3.real_cg(l1, l2, l3)
                worst = max(worst, np.abs(got - want).max())
    assert worst < 1e-12


def test_errors_are_reported(T):
    with pytest.raises(T.TPConvError) as e:
        T.Plan("8x0e+8xe", 1, "8x0e", 4)
    assert e.value.status == 2
    with pytest.raises(T.TPConvError) as e:
        T.Plan("8x4e", 1, "8x0e", 4)
    assert e.value.status == 3
    with pytest.raises(T.TPConvError) as e:
        T.Plan("8x0e", 4, "8x0e", 4)
    assert e.value.status == 3
    with pytest.raises(T.TPConvError) as e:
        T.Plan("8x0e", 1, "8x0e", 17)
    assert e.value.status == 3
    with pytest.raises(T.TPConvError) as e:
        T.tpconv_cg_coefficients(1, 1, 3)
    assert e.value.status == 3


def test_workspace_independent_of_edges_and_capped(T):
    c = W.CONFIGS["mace"]
    plan = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"])
    sizes = {T.tpconv_workspace_size(plan, op, 4096, E) for op in (0,) for E in (10, 10 ** 6, 10 ** 8)}
    assert len(sizes) == 1
    cap = 64 << 20
    capped = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], workspace_cap=cap)
    theta_ops = 12 * 4 * capped.theta_numel  # tensor-core Theta operands: independent of N and E
    # the tensor-core Theta gradient adds x of one chunk (4 x dim_in floats per
    # node, against the node state's 22016) and a fixed buffer of partial tiles
    partials = 2 * 160 * 64 * 128 * 4
    for op in (0, 1, 2):
        big = T.tpconv_workspace_size(capped, op, 1_222_309, 64_000_000)
        assert big == T.tpconv_workspace_size(capped, op, 500_000, 1_000)
        assert big <= cap * (1 + 4 * 576 / 22016) + theta_ops + partials + (4 << 20)


def test_half_precision_mixing_is_rejected(T):
    """The value between the TF32 and SIMT modes names no mode: plan creation
    reports it unsupported (the Theta contractions are bound by the fp32 state
    read, so a half-precision operand mode is not provided)."""
    import ctypes
    L = T._lib
    o = L.default_options()
    o.gemm = 2
    h = ctypes.c_void_p()
    st = L.lib().tpconv_plan_create(ctypes.byref(h), b"8x0e+8x1o", 2, b"8x0e+8x1o", 4, ctypes.byref(o))
    assert st == 3  # TPCONV_ERR_UNSUPPORTED
    assert "bf16" not in L.GEMM


@pytest.mark.parametrize("gemm,per_op", [("fp32", (2, 4, 12)), ("tf32", (1, 2, 6)), ("simt", (0, 0, 0))])
def test_theta_region_sized_per_operation(T, gemm, per_op):
    """The repacked Theta operands of the tensor-core contractions take what each
    operation uses: forward Theta^T (hi, lo), backward the elementwise split and
    the dx packing, double backward all three for Theta and gg_Theta; none
    without tensor cores.  The wide plan's forward fits the fixed 64 MiB scratch
    of the allocation-free forward only with a node cap."""
    c = W.CONFIGS["wide"]
    L = T._lib

    def size(cap):
        p = T.Plan(c["irreps_in"], c["l_sh_max"], c["irreps_out"], c["R"], gemm=gemm, workspace_cap=cap)
        return p, [L.tpconv_workspace_size(p, op, 8192, 262_144) for op in (0, 1, 2)]

    plan, a = size(1)           # one node per chunk: the Theta region dominates
    tn = (plan.theta_numel + 63) // 64 * 64 * 4
    # backward and double backward on tensor cores also hold the Theta
    # gradient's partial tiles: one 128 x 128 tile per row tile of both operand
    # pairs (23 paths x 8 row tiles x 2), at least two waves of 160
    part = max(2 * 160, 2 * 23 * 8) * 128 * 128 * 4 if gemm != "simt" else 0
    for op, (got, k) in enumerate(zip(a, per_op)):
        extra = part if op > 0 else 0
        assert k * tn + extra <= got <= k * tn + extra + (1 << 20), (op, got, k * tn + extra)
    _, b = size(0)
    state = 4 * 8192 * 101_376  # A floats per node of the wide layer
    assert b[0] >= state + per_op[0] * tn
    if gemm == "fp32":
        assert a[0] <= L.STATIC_SCRATCH_BYTES < b[0]
