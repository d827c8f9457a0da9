"""GPU parity at the widest head layout the library accepts: 65 query heads
(G*k = 64 routed heads plus the shared head).

* G = 64, M = k = 1: one expert per group. Routing is trivial, and the layer
  is GQA with H = G plus a duplicated slot.
* G = 32, M = 2, k = 2: the widest combine row, (G*k + G + 1) * 64 columns.

Every stage is compared with the oracle through the C ABI. So are the dense
baseline and one decode step.
"""
import numpy as np
import pytest
import torch

import oracle.gqe_ref as ref
from gqe_inputs import Dims, make_decode_inputs, make_inputs

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import moe_gqa_query_gqe_b200 as gqe
    from _gpu import (assert_close_bf16, check_selection, f64, reference_attention, run_dense, run_forward,
                      run_stages, to_dev)

WIDE = {
    "g64_m1_k1": Dims(B=2, T=136, D=128, G=64, M=1, k=1),
    "g32_m2_k2": Dims(B=2, T=72, D=128, G=32, M=2, k=2),
}


@pytest.fixture(scope="module")
def cases():
    out = {}
    for name, d in WIDE.items():
        inp = make_inputs(d, seed=0)
        dev = to_dev(inp)
        out[name] = (d, inp, dev, run_stages(d, dev))
    return out


@pytest.mark.parametrize("name", list(WIDE))
def test_stages_match_oracle(cases, name):
    d, inp, dev, st = cases[name]
    assert st["status"] == 0
    check_selection(d, inp["x"], inp["Wr"], inp["br"], st["sel"])
    seg_off, seg_tok, row_map = ref.compact(st["sel"].numpy(), d.B, d.T, d.G, d.M)
    np.testing.assert_array_equal(st["seg_off"].numpy(), seg_off)
    np.testing.assert_array_equal(st["seg_tok"].numpy(), seg_tok)
    np.testing.assert_array_equal(st["row_map"].numpy(), row_map)
    full = ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], d,
                           forced_sel=st["sel"].numpy())
    N = d.B * d.T
    assert_close_bf16(st["K"], full["K"].reshape(N, d.G, 64), "K")
    assert_close_bf16(st["V"], full["V"].reshape(N, d.G, 64), "V")
    assert_close_bf16(st["Q"], full["Q"], "Q")
    assert_close_bf16(st["O"], reference_attention(d, st["Q"], st["K"], st["V"], np.arange(N)), "O")
    assert_close_bf16(st["y"], full["y"], "y")


@pytest.mark.parametrize("name", list(WIDE))
def test_forward_and_dense_baseline(cases, name):
    d, inp, dev, st = cases[name]
    y, _, status = run_forward(d, dev)
    assert status == 0
    assert torch.equal(y.cpu(), st["y"])
    yd, _, status = run_dense(d, dev)
    assert status == 0
    want = ref.gqa_dense_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wo_dense"], d)
    assert_close_bf16(yd, want["y"], "dense GQA y")


def test_one_expert_per_group_selects_it_with_weight_one(cases):
    d, inp, dev, st = cases["g64_m1_k1"]
    assert torch.all(st["sel"] == 0)
    assert torch.all(st["w"] == 1.0)
    assert torch.all(torch.isinf(st["margin"]))


@pytest.mark.parametrize("name", list(WIDE))
def test_decode_step(name):
    d = WIDE[name]
    lens = [0, d.T - 1]
    inp = make_decode_inputs(d, lens, seed=3)
    dev = to_dev(inp)
    y = torch.empty((d.B, d.D), dtype=torch.bfloat16, device="cuda")
    sel = torch.empty((d.B, d.G, d.k), dtype=torch.int32, device="cuda")
    w = torch.empty((d.B, d.G, d.k), dtype=torch.float32, device="cuda")
    Kc, Vc = dev["K_cache"].clone(), dev["V_cache"].clone()
    ws = gqe.workspace(d, gqe.OP_DECODE)
    gqe.gqe_decode(d, dev["cache_len"], dev["x_new"], dev["Wq"], dev["Wk"], dev["Wv"], dev["Wr"], dev["br"],
                   dev["Wo"], Kc, Vc, y, sel, w, ws)
    assert gqe.gqe_check_error() == 0
    check_selection(d, inp["x_new"], inp["Wr"], inp["br"], sel.cpu())
    want = ref.gqe_decode(inp["x_new"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"],
                          inp["K_cache"], inp["V_cache"], lens, d, forced_sel=sel.cpu().numpy())
    np.testing.assert_allclose(f64(w.cpu()), want["w"], rtol=0, atol=2e-6)
    assert_close_bf16(y, want["y"], "decode y")
