"""gqe_forward_host: the layer with x and y in pinned host memory gives the
same bits as gqe_forward on device buffers (the same kernels on the same
rows), including when calls follow each other without a synchronisation."""
import pytest
import torch

from gqe_inputs import CONFIGS, make_inputs

from _cases import SMALL

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import moe_gqa_query_gqe_b200 as gqe
    from _gpu import run_forward, to_dev


def _host_forward(d, dev, x_host, ws):
    y_host = torch.full((d.B * d.T, d.D), float("nan"), dtype=torch.bfloat16).pin_memory()
    gqe.gqe_forward_host(d, x_host, dev["Wq"], dev["Wk"], dev["Wv"], dev["Wr"], dev["br"], dev["Wo"], y_host, ws)
    return y_host


@pytest.mark.parametrize("name", ["tiny_b2_t256", "ragged_b3_t300", "pool4_k2_skewed_t384", "pool8_k4_t136",
                                  "single_token_b4", "one_token_b1_t1"])
def test_host_entry_matches_device_entry(name):
    d = SMALL[name]
    inp = make_inputs(d, seed=0)
    dev = to_dev(inp)
    y_dev, _, status = run_forward(d, dev)
    assert status == 0
    ws = gqe.workspace(d, gqe.OP_FORWARD_HOST)
    # the copies are asynchronous: x_host must stay allocated and unchanged
    # until the stream has passed the call
    x_host = inp["x"].pin_memory()
    y_host = _host_forward(d, dev, x_host, ws)
    torch.cuda.synchronize()
    assert gqe.gqe_check_error() == 0
    assert torch.equal(y_host, y_dev.cpu())


def test_host_entry_back_to_back_calls_at_the_main_shape():
    """Two calls with different activations, enqueued one after the other on
    one workspace: each result is that of its own input."""
    d = CONFIGS["main_b8_t2048"]
    inp = make_inputs(d, seed=0)
    dev = to_dev(inp)
    x2 = make_inputs(d, seed=1)["x"]
    ws = gqe.workspace(d, gqe.OP_FORWARD_HOST)
    # Both pinned inputs are held until the stream has passed both calls: the
    # library's copies are asynchronous, and a pinned buffer freed earlier can
    # be handed out again (and overwritten) before its copy has read it.
    x1_host = inp["x"].pin_memory()
    x2_host = x2.pin_memory()
    y1 = _host_forward(d, dev, x1_host, ws)
    y2 = _host_forward(d, dev, x2_host, ws)
    torch.cuda.synchronize()
    assert gqe.gqe_check_error() == 0
    want1, _, s1 = run_forward(d, dev)
    dev2 = dict(dev, x=x2.cuda())
    want2, _, s2 = run_forward(d, dev2)
    assert s1 == 0 and s2 == 0
    assert torch.equal(y1, want1.cpu())
    assert torch.equal(y2, want2.cpu())
