"""Failure detection on the GPU without a fault: a pipeline wait that nothing
completes gives up after its bound, the host reads GQE_ERR_TIMEOUT from the
device error word, and the context stays usable (a forward pass afterwards
still matches its earlier bits)."""
import time

import pytest
import torch

from gqe_inputs import make_inputs

from _cases import SMALL

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import moe_gqa_query_gqe_b200 as gqe
    from _gpu import run_forward, to_dev


def test_bounded_wait_times_out_and_the_context_stays_usable():
    d = SMALL["ragged_b3_t300"]
    dev = to_dev(make_inputs(d, seed=0))
    y0, _, status = run_forward(d, dev)
    assert status == 0
    t0 = time.time()
    gqe.gqe_selftest_wait_timeout()
    status = gqe.gqe_check_error()
    waited = time.time() - t0
    assert status == -5, gqe.gqe_status_string(status)  # GQE_ERR_TIMEOUT
    assert 1.5 < waited < 60.0
    assert gqe.gqe_check_error() == 0  # the word was cleared by the read
    y1, _, status = run_forward(d, dev)
    assert status == 0
    assert torch.equal(y0.cpu(), y1.cpu())
