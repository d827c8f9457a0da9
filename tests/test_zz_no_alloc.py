"""gqe_route_noalloc: the router entry point for callers that cannot allocate
device memory (its scratch is a fixed array inside the library).

Checked through the C ABI against gqe_route, which uses a caller workspace:
the outputs must agree (same kernels, so bit for bit, well inside the parity
tolerances) on two calls in a row with different shapes, the second call
reusing the array the first one left behind. Collected last on purpose.
"""
import ctypes

import pytest
import torch

from gqe_inputs import Dims, make_inputs

pytestmark = pytest.mark.gpu


def _outputs(d):
    N = d.B * d.T
    return {
        "sel": torch.full((N, d.G, d.k), -7, dtype=torch.int32, device="cuda"),
        "w": torch.full((N, d.G, d.k), -1.0, dtype=torch.float32, device="cuda"),
        "margin": torch.full((N, d.G), -1.0, dtype=torch.float32, device="cuda"),
        "seg_off": torch.full((d.B * d.G * d.M + 1,), -7, dtype=torch.int32, device="cuda"),
        "seg_tok": torch.full((N * d.G * d.k,), -7, dtype=torch.int32, device="cuda"),
        "row_map": torch.full((N, d.G, d.k), -7, dtype=torch.int32, device="cuda"),
    }


def _route_with_workspace(d, inp):
    import moe_gqa_query_gqe_b200 as gqe
    o = _outputs(d)
    ws = gqe.workspace(d, gqe.OP_ROUTE)
    gqe.gqe_route(d, inp["x"], inp["Wr"], inp["br"], o["sel"], o["w"], o["margin"], o["seg_off"], o["seg_tok"],
                  o["row_map"], ws)
    return o


def _route_noalloc_raw(d, inp):
    """Direct ctypes call of the exported symbol."""
    from moe_gqa_query_gqe_b200 import lib
    so = lib.load()
    o = _outputs(d)
    dims = lib.dims_struct(d)
    rc = so.gqe_route_noalloc(ctypes.byref(dims), inp["x"].data_ptr(), inp["Wr"].data_ptr(), inp["br"].data_ptr(),
                              o["sel"].data_ptr(), o["w"].data_ptr(), o["margin"].data_ptr(),
                              o["seg_off"].data_ptr(), o["seg_tok"].data_ptr(), o["row_map"].data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    assert rc == 0, lib.STATUS.get(rc, rc)
    return o


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a GPU")
def test_noalloc_route_matches_workspace_route_twice_in_a_row():
    from moe_gqa_query_gqe_b200 import lib
    shapes = [Dims(B=3, T=700, D=256, G=4, M=2, k=1),
              Dims(B=2, T=300, D=512, G=8, M=4, k=2, bias0=2.0)]
    for d in shapes:
        inp = {k: v.cuda() for k, v in make_inputs(d, seed=1).items()}
        want = _route_with_workspace(d, inp)
        got = _route_noalloc_raw(d, inp)
        assert lib.load().gqe_check_error(torch.cuda.current_stream().cuda_stream) == 0
        for key in want:
            assert torch.equal(got[key], want[key]), key


@pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a GPU")
def test_noalloc_route_rejects_shapes_beyond_its_scratch():
    from moe_gqa_query_gqe_b200 import lib
    # 2 * 64 * ceil(32768/128) * 16 * 4 bytes = 2 MiB > 1 MiB
    d = Dims(B=64, T=32768, D=1024, G=8, M=2, k=1)
    P = 1 << 20  # never dereferenced: the size check comes first
    rc = lib.load().gqe_route_noalloc(ctypes.byref(lib.dims_struct(d)), P, P, None, P, P, None, P, P, None, None)
    assert rc == -3
