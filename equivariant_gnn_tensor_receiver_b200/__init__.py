"""Streaming Clebsch-Gordan tensor-product convolution for B200 (sm_100a).

The operator and its schedule follow "Sobek" (arXiv 2607.18074, abstract):
edge-conditioned tensor-product convolution whose edge-local products are
consumed directly into bounded receiver-side state, with forward, backward and
double backward.  All arithmetic runs in the CUDA library ``libtpconv.so``
(C ABI in include/tpconv.h); this package is its thin Python binding.
"""

from ._lib import (GEMM, OP_BACKWARD, OP_DOUBLE_BACKWARD, OP_FORWARD, OP_TRANSPOSE, Plan, TPConvError,
                   exported_names, lib, tpconv_backward, tpconv_cg_coefficients, tpconv_double_backward,
                   tpconv_forward, tpconv_graph_transpose, tpconv_plan_create, tpconv_workspace_size)
from .api import Graph, TPConv, backward, double_backward, forward, workspace

__all__ = ["Plan", "Graph", "TPConv", "TPConvError", "forward", "backward", "double_backward", "workspace", "lib",
           "exported_names", "tpconv_plan_create", "tpconv_forward", "tpconv_backward", "tpconv_double_backward",
           "tpconv_graph_transpose", "tpconv_workspace_size", "tpconv_cg_coefficients", "GEMM", "OP_FORWARD",
           "OP_BACKWARD", "OP_DOUBLE_BACKWARD", "OP_TRANSPOSE"]
