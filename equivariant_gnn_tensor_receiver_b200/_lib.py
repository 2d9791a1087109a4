"""ctypes binding of ``libtpconv.so`` (the C ABI declared in include/tpconv.h).

Argument marshalling only: every step of the operator runs in the library's
CUDA kernels.  Functions keep the C names; tensors are torch CUDA tensors
(fp32 / int32, contiguous) whose device pointers are passed through, and the
stream defaults to torch's current stream.  A missing library raises.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtpconv.so")

TPCONV_OK = 0
TPCONV_ERR_WORKSPACE_TOO_SMALL = 4
STATUS = {0: "ok", 1: "invalid argument", 2: "bad irreps", 3: "unsupported", 4: "workspace too small",
          5: "CUDA error", 6: "graph invalid", 7: "timeout", 8: "internal"}
RADIAL = {"gaussian": 0, "bessel": 1}
GEMM = {"fp32": 0, "tf32": 1, "simt": 3}
FAMILY = {"full": 0, "channelwise": 1}
OP_FORWARD, OP_BACKWARD, OP_DOUBLE_BACKWARD, OP_TRANSPOSE = 0, 1, 2, 3


class TPConvError(RuntimeError):
    def __init__(self, fn, status):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status})")
        self.status = status


class Options(ctypes.Structure):
    _fields_ = [("radial", ctypes.c_int), ("radial_p0", ctypes.c_double), ("radial_p1", ctypes.c_double),
                ("gemm", ctypes.c_int), ("workspace_cap", ctypes.c_size_t), ("validate", ctypes.c_int),
                ("family", ctypes.c_int)]


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_EXPORTS = {
    "tpconv_default_options": (None, [ctypes.POINTER(Options)]),
    "tpconv_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "tpconv_plan_create": (ctypes.c_int, [ctypes.POINTER(_P), ctypes.c_char_p, ctypes.c_int, ctypes.c_char_p,
                                          ctypes.c_int, ctypes.POINTER(Options)]),
    "tpconv_plan_destroy": (ctypes.c_int, [_P]),
    "tpconv_plan_info": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int),
                                        ctypes.POINTER(ctypes.c_size_t)]),
    "tpconv_plan_path": (ctypes.c_int, [_P, ctypes.c_int] + [ctypes.POINTER(ctypes.c_int)] * 5
                         + [ctypes.POINTER(ctypes.c_size_t)]),
    "tpconv_cg_coefficients": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.POINTER(ctypes.c_double)]),
    "tpconv_workspace_size": (ctypes.c_int, [_P, ctypes.c_int, _I64, _I64, ctypes.POINTER(ctypes.c_size_t)]),
    "tpconv_graph_transpose": (ctypes.c_int, [_P, _I64, _I64] + [_P] * 5 + [_P, ctypes.c_size_t, _P]),
    "tpconv_forward": (ctypes.c_int, [_P, _I64, _I64] + [_P] * 6 + [_P, ctypes.c_size_t, _P]),
    "tpconv_forward_static": (ctypes.c_int, [_P, _I64, _I64] + [_P] * 6 + [_P]),
    "tpconv_backward": (ctypes.c_int, [_P, _I64, _I64] + [_P] * 14 + [_P, ctypes.c_size_t, _P]),
    "tpconv_double_backward": (ctypes.c_int, [_P, _I64, _I64] + [_P] * 16 + [_P, ctypes.c_size_t, _P]),
    "tpconv_get_device_status": (ctypes.c_int, [_P, _P, ctypes.POINTER(ctypes.c_int)]),
    "tpconv_set_wait_limit": (ctypes.c_int, [ctypes.c_uint64]),
    "tpconv_profile_enable": (ctypes.c_int, [ctypes.c_int]),
    "tpconv_profile_reset": (ctypes.c_int, []),
    "tpconv_profile_read": (ctypes.c_int, [ctypes.c_int, ctypes.POINTER(ctypes.c_double),
                                           ctypes.POINTER(ctypes.c_int64)]),
}
PHASES = ["transpose", "fwd_edge", "fwd_node", "bwd_node_g", "bwd_edge_r", "bwd_edge_s", "bwd_node_x",
          "dbl_edge_a", "dbl_node_a", "dbl_edge_r", "dbl_edge_s", "dbl_node_x", "other"]


def exported_names():
    return list(_EXPORTS)


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m equivariant_gnn_tensor_receiver_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _EXPORTS.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(fn, st):
    if st != TPCONV_OK:
        raise TPConvError(fn, st)


def default_options() -> Options:
    o = Options()
    lib().tpconv_default_options(ctypes.byref(o))
    return o


class Plan:
    """Owner of a ``tpconv_plan*``."""

    def __init__(self, irreps_in, l_sh_max, irreps_out, R, radial="bessel", radial_params=(5.0,), gemm="fp32",
                 workspace_cap=0, validate=False, family="full"):
        o = default_options()
        o.radial = RADIAL[radial]
        o.radial_p0 = float(radial_params[0])
        o.radial_p1 = float(radial_params[1]) if len(radial_params) > 1 else 0.0
        o.gemm = GEMM[gemm]
        o.workspace_cap = int(workspace_cap)
        o.validate = int(bool(validate))
        o.family = FAMILY[family]
        h = _P()
        _check("tpconv_plan_create",
               lib().tpconv_plan_create(ctypes.byref(h), irreps_in.encode(), int(l_sh_max), irreps_out.encode(),
                                        int(R), ctypes.byref(o)))
        self.handle = h
        self.irreps_in, self.irreps_out, self.l_sh_max, self.R = irreps_in, irreps_out, l_sh_max, R
        self.family = family
        self.options = o
        a = [ctypes.c_int() for _ in range(4)]
        t = ctypes.c_size_t()
        _check("tpconv_plan_info", lib().tpconv_plan_info(h, *[ctypes.byref(v) for v in a], ctypes.byref(t)))
        self.n_paths, self.dim_in, self.dim_out, self.n_sh = (v.value for v in a)
        self.theta_numel = t.value
        self.paths = []
        for i in range(self.n_paths):
            v = [ctypes.c_int() for _ in range(5)]
            off = ctypes.c_size_t()
            _check("tpconv_plan_path", lib().tpconv_plan_path(h, i, *[ctypes.byref(x) for x in v],
                                                              ctypes.byref(off)))
            l1, l2, l3, ci, co = (x.value for x in v)
            self.paths.append(dict(l1=l1, l2=l2, l3=l3, c_in=ci, c_out=co, theta_offset=off.value))

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _lib is not None:
            _lib.tpconv_plan_destroy(h)
            self.handle = None


def tpconv_plan_create(irreps_in, l_sh_max, irreps_out, R, **opts) -> Plan:
    return Plan(irreps_in, l_sh_max, irreps_out, R, **opts)


def tpconv_cg_coefficients(l1, l2, l3) -> np.ndarray:
    out = np.zeros((2 * l1 + 1) * (2 * l2 + 1) * (2 * l3 + 1), dtype=np.float64)
    _check("tpconv_cg_coefficients",
           lib().tpconv_cg_coefficients(l1, l2, l3, out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))))
    return out.reshape(2 * l1 + 1, 2 * l2 + 1, 2 * l3 + 1)


def tpconv_workspace_size(plan: Plan, op: int, N: int, E: int) -> int:
    b = ctypes.c_size_t()
    _check("tpconv_workspace_size", lib().tpconv_workspace_size(plan.handle, op, N, E, ctypes.byref(b)))
    return b.value


# --------------------------------------------------------------------------
# device entry points (torch tensors)
# --------------------------------------------------------------------------


def _ptr(t, dtype=None):
    if t is None:
        return None
    import torch
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"expected {dtype}, got {t.dtype}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _ws(workspace):
    if workspace is None:
        return None, 0
    return _ptr(workspace), workspace.numel() * workspace.element_size()


def tpconv_graph_transpose(plan, N, E, rowptr, col, perm, s_rowptr, s_recv, workspace, stream=None):
    import torch
    i32 = torch.int32
    w, wb = _ws(workspace)
    _check("tpconv_graph_transpose",
           lib().tpconv_graph_transpose(plan.handle, N, E, _ptr(rowptr, i32), _ptr(col, i32), _ptr(perm, i32),
                                        _ptr(s_rowptr, i32), _ptr(s_recv, i32), w, wb, _stream(stream)))


def tpconv_forward(plan, N, E, rowptr, col, edge_vec, x, theta, out, workspace, stream=None):
    import torch
    f32, i32 = torch.float32, torch.int32
    w, wb = _ws(workspace)
    _check("tpconv_forward",
           lib().tpconv_forward(plan.handle, N, E, _ptr(rowptr, i32), _ptr(col, i32), _ptr(edge_vec, f32),
                                _ptr(x, f32), _ptr(theta, f32), _ptr(out, f32), w, wb, _stream(stream)))


def tpconv_forward_static(plan, N, E, rowptr, col, edge_vec, x, theta, out, stream=None):
    import torch
    f32, i32 = torch.float32, torch.int32
    _check("tpconv_forward_static",
           lib().tpconv_forward_static(plan.handle, N, E, _ptr(rowptr, i32), _ptr(col, i32), _ptr(edge_vec, f32),
                                       _ptr(x, f32), _ptr(theta, f32), _ptr(out, f32), _stream(stream)))


def tpconv_backward(plan, N, E, rowptr, col, perm, s_rowptr, s_recv, edge_vec, x, theta, g, dx, dtheta, dvec,
                    dY, db, workspace, stream=None):
    import torch
    f32, i32 = torch.float32, torch.int32
    w, wb = _ws(workspace)
    _check("tpconv_backward",
           lib().tpconv_backward(plan.handle, N, E, _ptr(rowptr, i32), _ptr(col, i32), _ptr(perm, i32),
                                 _ptr(s_rowptr, i32), _ptr(s_recv, i32), _ptr(edge_vec, f32), _ptr(x, f32),
                                 _ptr(theta, f32), _ptr(g, f32), _ptr(dx, f32), _ptr(dtheta, f32),
                                 _ptr(dvec, f32), _ptr(dY, f32), _ptr(db, f32), w, wb, _stream(stream)))


def tpconv_double_backward(plan, N, E, rowptr, col, perm, s_rowptr, s_recv, edge_vec, x, theta, g, gg_x, gg_vec,
                           gg_theta, d_g, d_x, d_vec, d_theta, workspace, stream=None):
    import torch
    f32, i32 = torch.float32, torch.int32
    w, wb = _ws(workspace)
    _check("tpconv_double_backward",
           lib().tpconv_double_backward(plan.handle, N, E, _ptr(rowptr, i32), _ptr(col, i32), _ptr(perm, i32),
                                        _ptr(s_rowptr, i32), _ptr(s_recv, i32), _ptr(edge_vec, f32),
                                        _ptr(x, f32), _ptr(theta, f32), _ptr(g, f32), _ptr(gg_x, f32),
                                        _ptr(gg_vec, f32), _ptr(gg_theta, f32), _ptr(d_g, f32),
                                        _ptr(d_x, f32), _ptr(d_vec, f32), _ptr(d_theta, f32), w, wb,
                                        _stream(stream)))


TPCONV_ERR_TIMEOUT = 7


def tpconv_get_device_status(plan, stream=None) -> int:
    """Synchronises the stream; TPCONV_ERR_TIMEOUT if a bounded device wait of
    the tensor-core kernels expired since the last query (the record is
    cleared), else TPCONV_OK."""
    st = ctypes.c_int()
    _check("tpconv_get_device_status", lib().tpconv_get_device_status(plan.handle, _stream(stream), ctypes.byref(st)))
    return st.value


def tpconv_set_wait_limit(ns: int):
    """Limit (ns) of the tensor-core kernels' device waits for later calls; 0 = default (2 s)."""
    _check("tpconv_set_wait_limit", lib().tpconv_set_wait_limit(int(ns)))


def tpconv_profile_enable(on: bool = True):
    _check("tpconv_profile_enable", lib().tpconv_profile_enable(int(bool(on))))


def tpconv_profile_reset():
    _check("tpconv_profile_reset", lib().tpconv_profile_reset())


def tpconv_profile_read(phase: int):
    """(device milliseconds, kernel launches) of one phase since the last reset."""
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    _check("tpconv_profile_read", lib().tpconv_profile_read(int(phase), ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value


STATIC_SCRATCH_BYTES = 64 << 20  # TPCONV_STATIC_SCRATCH_BYTES


def static_device_bytes() -> int:
    """Device memory the loaded library holds on every device by itself: the
    fixed scratch array of ``tpconv_forward_static`` (resident whether or not
    that entry point is called; not visible to torch's allocator statistics)."""
    return STATIC_SCRATCH_BYTES


def profile_all():
    return {name: tpconv_profile_read(i) for i, name in enumerate(PHASES)}
