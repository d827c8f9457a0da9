"""GPU parity of the output-construction variants (gqe_forward_variant)
against the fp64 oracle, through the C ABI.

The variants are the ablation of the animattoys.com article, section 6
(hard concatenation; concatenation weighted by the router's scores without
the renormalised slot), the gist.science summary's wording of it,
"Experimental results" (no shared head), and the single-slot reading of the
article's section 4 (one slot averaging all selected experts). The oracle
reruns with the GPU's expert choices (near ties may go either way), and y
must be within the bf16 bars of the parity tests.
"""
import pytest
import torch

import oracle.gqe_ref as ref
from gqe_inputs import make_inputs

from _cases import SMALL

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import moe_gqa_query_gqe_b200 as gqe
    from _gpu import assert_close_bf16, f64, run_dense, run_forward, run_stages, to_dev

    MODE = {"slot": gqe.COMBINE_SLOT, "hard": gqe.COMBINE_HARD, "weighted": gqe.COMBINE_WEIGHTED,
            "global_slot": gqe.COMBINE_GLOBAL_SLOT, "no_shared": gqe.COMBINE_NO_SHARED}

NAMES = ["tiny_b2_t256", "ragged_b3_t300", "pool4_k2_skewed_t384", "pool8_k4_t136", "one_group_g1_m8_k2"]


@pytest.fixture(scope="module")
def cases():
    out = {}
    for name in NAMES:
        d = SMALL[name]
        inp = make_inputs(d, seed=0)
        dev = to_dev(inp)
        out[name] = (d, inp, dev, run_stages(d, dev))
    return out


def _variant_wo(d, mode, seed=6):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((ref.combine_width(d, mode), d.D), generator=g) * 0.02).to(torch.bfloat16)


def _run(d, dev, mode, Wo, Wq=None):
    ws = gqe.workspace(d, gqe.OP_FORWARD_VARIANT)
    y = torch.full((d.B * d.T, d.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    gqe.gqe_forward_variant(d, MODE[mode], dev["x"], dev["Wq"] if Wq is None else Wq, dev["Wk"], dev["Wv"],
                            dev["Wr"], dev["br"], Wo.cuda(), y, ws)
    assert gqe.gqe_check_error() == 0
    return y


@pytest.mark.parametrize("name", NAMES)
@pytest.mark.parametrize("mode", list(ref.VARIANTS))
def test_variant_matches_oracle(cases, name, mode):
    d, inp, dev, st = cases[name]
    assert st["status"] == 0
    Wo = _variant_wo(d, mode)
    y = _run(d, dev, mode, Wo)
    want = ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], Wo, d,
                           forced_sel=st["sel"].numpy(), combine_mode=mode)
    assert_close_bf16(y, want["y"], f"{mode} variant y vs oracle")


def test_slot_mode_of_the_variant_entry_is_gqe_forward(cases):
    d, inp, dev, st = cases["pool4_k2_skewed_t384"]
    y = _run(d, dev, "slot", inp["Wo"])
    assert torch.equal(y.cpu(), st["y"])


@pytest.mark.parametrize("name", ["ragged_b3_t300", "pool4_k2_skewed_t384"])
def test_no_shared_variant_never_reads_the_shared_head(cases, name):
    """Without the shared head, its query weights do not reach y: NaN in
    them leaves y bitwise unchanged."""
    d, inp, dev, st = cases[name]
    Wo = _variant_wo(d, "no_shared")
    y0 = _run(d, dev, "no_shared", Wo)
    Wq = dev["Wq"].clone()
    Wq[:, d.G * d.M * 64:] = float("nan")
    y1 = _run(d, dev, "no_shared", Wo, Wq=Wq)
    assert torch.equal(y0.cpu(), y1.cpu())


def test_k_equals_m_with_zero_slot_and_shared_rows_is_dense_gqa():
    """With k = M every expert is selected and the concatenation is in head
    order (h = g*M + e). With Wo's concatenation rows set to Wo_dense and its
    slot and shared rows set to zero, the layer is the dense GQA layer up to
    rounding (the GQE invariant, checked here on the GPU's two paths)."""
    d = SMALL["k_equals_m_t260"]
    inp = make_inputs(d, seed=0)
    dev = to_dev(inp)
    Wo = torch.zeros((d.wo_rows, d.D), dtype=torch.bfloat16)
    Wo[:d.G * d.k * 64] = inp["Wo_dense"]
    y, _, status = run_forward(d, dict(dev, Wo=Wo.cuda()))
    assert status == 0
    yd, _, status = run_dense(d, dev)
    assert status == 0
    assert_close_bf16(y, f64(yd), "GQE with k = M and zero slot/shared rows vs dense GQA")
