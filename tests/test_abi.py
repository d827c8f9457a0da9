"""The C-ABI library: it loads, exports every entry point include/gqe.h
declares, and validates arguments on the host before touching a device (so
these checks run without a GPU)."""
import ctypes
import os
import re

import pytest
import torch

import moe_gqa_query_gqe_b200 as gqe
from moe_gqa_query_gqe_b200 import lib
import oracle.gqe_ref as ref
from gqe_inputs import CONFIGS, Dims

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if not fn.endswith(".h"):
            continue
        src = open(os.path.join(ROOT, "include", fn)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\([^;{]*\)\s*;", src, flags=re.M):
            names.add(m.group(1))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    declared = _declared_functions()
    assert "gqe_route" in declared and "gqa_dense_forward" in declared
    so = lib.load()
    for name in declared:
        assert hasattr(so, name), f"{name} declared in include/ but not exported"
    assert set(declared) == set(lib.EXPORTS)


def test_version_and_status_strings():
    assert gqe.gqe_version() == 100
    for code in range(-7, 1):
        assert gqe.gqe_status_string(code) != "unknown status"


def test_all_workloads_are_supported_and_sized():
    for name, d in CONFIGS.items():
        assert gqe.validate_dims(d) == 0, name
        assert gqe.workspace_bytes(d, gqe.OP_FORWARD) > 0
        assert gqe.workspace_bytes(d, gqe.OP_FORWARD_HOST) > gqe.workspace_bytes(d, gqe.OP_FORWARD)
        assert gqe.workspace_bytes(d, gqe.OP_DENSE) > 0
        assert gqe.workspace_bytes(d, gqe.OP_QPROJ) == 0
        assert gqe.workspace_bytes(d, gqe.OP_DECODE) > 0
        assert gqe.workspace_bytes(d, gqe.OP_FORWARD_VARIANT) > gqe.workspace_bytes(d, gqe.OP_FORWARD)


def test_variant_workspace_holds_the_widest_variant():
    """Beyond gqe_forward's workspace, the variants need the selected
    experts' probabilities (fp32) and their own A (bf16, the widest of the
    non-slot constructions)."""
    for d in (CONFIGS["main_b8_t2048"], Dims(B=2, T=136, D=256, G=8, M=8, k=4), Dims(B=1, T=5, D=128, G=1, M=8, k=2)):
        N = d.B * d.T
        widest = max(ref.combine_width(d, m) for m in ref.VARIANTS)
        extra = gqe.workspace_bytes(d, gqe.OP_FORWARD_VARIANT) - gqe.workspace_bytes(d, gqe.OP_FORWARD)
        assert extra >= N * d.G * d.k * 4 + N * widest * 2
        assert extra <= N * d.G * d.k * 4 + N * widest * 2 + 512  # two 256-byte alignments


def test_decode_workspace_does_not_grow_with_the_cache_capacity():
    # the attention's partial results are per CTA and sequence (one key range
    # each), not per key chunk: the workspace depends on B, G and k only
    d = Dims(B=4, T=1024, D=256, G=4, M=2, k=1)
    small = gqe.workspace_bytes(d, gqe.OP_DECODE)
    assert gqe.workspace_bytes(d.with_(T=32 * 1024), gqe.OP_DECODE) == small
    assert gqe.workspace_bytes(d.with_(T=1 << 20), gqe.OP_DECODE) == small
    assert gqe.workspace_bytes(d.with_(k=2), gqe.OP_DECODE) > small
    assert gqe.workspace_bytes(d.with_(B=8), gqe.OP_DECODE) > small


@pytest.mark.parametrize("bad,code", [
    (dict(dh=32), -2), (dict(D=1000), -2), (dict(k=3, M=2), -1), (dict(M=3, k=1), -2),
    (dict(G=3, M=2), -2), (dict(T=0), -1), (dict(G=1, M=1), -2), (dict(G=2, M=2), -2), (dict(k=0), -1),
])
def test_unsupported_and_invalid_dims(bad, code):
    d = Dims(B=1, T=64, D=256, G=4, M=2, k=1).with_(**bad)
    assert gqe.validate_dims(d) == code
    assert gqe.workspace_bytes(d, gqe.OP_FORWARD) == 0


def _raw(name, *args):
    so = lib.load()
    return getattr(so, name)(*args)


def test_null_and_misaligned_pointers_are_rejected_before_any_launch():
    d = lib.dims_struct(Dims(B=1, T=64, D=256, G=4, M=2, k=1))
    P = 1 << 20  # aligned fake address: never dereferenced, validation fails first
    dp = ctypes.byref(d)
    assert _raw("gqe_attn", dp, None, P, P, P, None, 0, None) == -1
    assert _raw("gqe_attn", dp, P + 2, P, P, P, None, 0, None) == -1
    assert _raw("gqe_route", dp, P, P, None, P, P, None, P, P, None, None, 0, None) == -3  # no workspace
    small = 256
    assert _raw("gqe_route", dp, P, P, None, P, P, None, P, P, None, P, small, None) == -3
    assert _raw("gqe_route", dp, P, P, None, P, P, None, P, P, None, P + 16, 1 << 30, None) == -3  # ws misaligned
    assert _raw("gqa_dense_forward", dp, P, P, P, P, P, None, P, 1 << 30, None) == -1
    # gqe_forward_variant: unknown combine mode, then a valid mode without workspace
    vargs = [P, P, P, P, P, None, P, P]
    # (or an unknown selected-query path: both, or a bit outside the enum)
    for bad_mode in (-1, 5, 7, 0x300, 0x400, 0x105):
        assert _raw("gqe_forward_variant", dp, bad_mode, *vargs, P, 1 << 30, None) == -1
    for mode in range(5):
        for qpath in (gqe.QPROJ_AUTO, gqe.QPROJ_GATHER, gqe.QPROJ_DENSE):
            assert _raw("gqe_forward_variant", dp, mode | qpath, *vargs, None, 0, None) == -3
    # gqe_decode: null cache_len, misaligned x_new, missing workspace
    args = [P, P, P, P, P, P, None, P, P, P, P, P, P]
    assert _raw("gqe_decode", dp, None, *args[1:], P, 1 << 30, None) == -1
    assert _raw("gqe_decode", dp, P, P + 2, *args[2:], P, 1 << 30, None) == -1
    assert _raw("gqe_decode", dp, *args, None, 0, None) == -3


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_valid_call_without_a_device_reports_no_device():
    d = lib.dims_struct(Dims(B=1, T=64, D=256, G=4, M=2, k=1))
    P = 1 << 20
    assert _raw("gqe_attn", ctypes.byref(d), P, P, P, P, None, 0, None) == -6


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device answer")
def test_wait_self_test_without_a_device_reports_no_device():
    assert _raw("gqe_selftest_wait_timeout", None) == -6
