"""bench.py's CPU-baseline leg also scores the timed run: the GPU's expert
selections against the oracle's (near ties counted and accepted, any other
difference counted as a mismatch) and the GPU's y against the oracle's. Here
the "GPU" outputs are stand-ins made on the CPU (the oracle's own selections
and y rounded to bf16, then one planted wrong selection), so the host logic
is checked without a GPU."""
import os
import sys

import numpy as np
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402
import oracle.gqe_ref as ref  # noqa: E402
from gqe_inputs import Dims, make_inputs  # noqa: E402


def _stand_in(d, inp):
    r = ref.route(inp["x"], inp["Wr"], inp["br"], d.G, d.M, d.k)
    y = ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], d)["y"]
    return r, torch.as_tensor(r["sel"], dtype=torch.int32), torch.as_tensor(y).to(torch.bfloat16)


def test_oracle_leg_scores_matching_outputs_as_clean():
    d = Dims(B=2, T=64, D=128, G=2, M=2, k=1)
    inp = make_inputs(d, seed=3)
    r, sel, y = _stand_in(d, inp)
    cpu, par = bench.oracle_leg(d, inp, sel, y, budget_s=0.0)
    assert cpu["kind"] == "oracle" and cpu["value"] > 0 and cpu["cores"] >= 1
    assert par["sequences_checked"] == 1 and par["rows"] == d.T
    assert par["decisions"] == d.T * d.G
    assert par["mismatches_beyond_tie"] == 0 and par["flipped_near_ties"] == 0
    # y rounded to bf16: within the bars, but not exactly zero
    assert 0 < par["worst_rel_l2"] <= 5e-3 and par["worst_max_abs"] <= 1e-2


def test_oracle_leg_counts_a_wrong_selection_and_the_extra_routes():
    d = Dims(B=1, T=48, D=128, G=2, M=4, k=2)
    inp = make_inputs(d, seed=4)
    r, sel, y = _stand_in(d, inp)
    # plant a wrong choice on the decision with the widest margin
    n, g = np.unravel_index(np.argmax(r["margin"]), r["margin"].shape)
    chosen = set(r["sel"][n, g].tolist())
    other = next(e for e in range(d.M) if e not in chosen)
    bad = sel.clone()
    bad[n, g] = torch.as_tensor(sorted([r["sel"][n, g, 0], other]), dtype=torch.int32)
    cpu, par = bench.oracle_leg(d, inp, bad, y, budget_s=0.0,
                                extra_routes=[("again", d, inp["x"], inp["Wr"], inp["br"], bad)])
    assert par["mismatches_beyond_tie"] == 1
    assert par["again"]["mismatches_beyond_tie"] == 1 and par["again"]["decisions"] == d.T * d.G
