"""Grouped Query Experts (GQE) attention forward pass for NVIDIA B200 (sm_100a).

The computation lives in libgqe.so (hand-written CUDA: routing, tcgen05
projections, tcgen05 flash attention, combine); ``lib`` is its ctypes binding
with the C ABI's entry-point names.
"""
from . import lib  # noqa: F401
from .lib import (  # noqa: F401
    gqe_route, gqe_qproj, gqe_attn, gqe_combine, gqe_forward, gqe_forward_variant, gqe_forward_host, gqe_decode,
    gqa_dense_forward, COMBINE_SLOT, COMBINE_HARD, COMBINE_WEIGHTED, COMBINE_GLOBAL_SLOT, COMBINE_NO_SHARED,
    QPROJ_AUTO, QPROJ_GATHER, QPROJ_DENSE,
    OP_FORWARD_VARIANT,
    gqe_check_error, gqe_status_string, gqe_version, gqe_selftest_wait_timeout, workspace, workspace_bytes, validate_dims,
    forward_views, GqeError, OP_ROUTE, OP_QPROJ, OP_ATTN, OP_COMBINE, OP_FORWARD, OP_DENSE, OP_FORWARD_HOST, OP_DECODE,
)
