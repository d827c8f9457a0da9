"""GPU parity of the decode step (gqe_decode) against the fp64 oracle.

One new token per sequence attends its cache (rows < cache_len[b]) plus
itself; its K/V row is written at cache_len[b]. Checked through the C ABI on
seeded inputs (gqe_inputs.make_decode_inputs): the selections (bit-exact
except near ties), the weights, the appended cache rows, the untouched cache
rows (bit-exact) and y against the oracle's step.
"""
import numpy as np
import pytest
import torch

import moe_gqa_query_gqe_b200 as gqe
import oracle.gqe_ref as ref
from gqe_inputs import Dims, make_decode_inputs

from _gpu import assert_close_bf16, check_selection, f64, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    # ragged lengths: empty cache, one row, chunk boundaries of the split-K attention (1024), capacity - 1
    ("b4_d256_g4m2k1", Dims(B=4, T=2100, D=256, G=4, M=2, k=1), [0, 1, 1023, 2099]),
    ("b3_d512_g8m4k2_skewed", Dims(B=3, T=1500, D=512, G=8, M=4, k=2, bias0=2.0), [1024, 1, 700]),
    ("b2_d256_g2m8k4", Dims(B=2, T=300, D=256, G=2, M=8, k=4), [5, 299]),
    ("b5_d256_g1m8k2_mqa", Dims(B=5, T=130, D=256, G=1, M=8, k=2), [0, 63, 64, 128, 129]),
    # 13, 16, 37 and 64 new tokens on the cluster kernels (ranks with partial
    # and empty token blocks, partial 16-token tiles), 65 on the prefill kernels
    ("b13_d256_g4m2k1", Dims(B=13, T=260, D=256, G=4, M=2, k=1), [(i * 53) % 260 for i in range(13)]),
    ("b16_d512_g8m4k2", Dims(B=16, T=200, D=512, G=8, M=4, k=2), [(i * 37) % 200 for i in range(16)]),
    ("b37_d256_g4m2k1", Dims(B=37, T=260, D=256, G=4, M=2, k=1), [(i * 53) % 260 for i in range(37)]),
    ("b64_d256_g8m4k2", Dims(B=64, T=200, D=256, G=8, M=4, k=2), [(i * 37) % 200 for i in range(64)]),
    ("b65_d256_g4m2k1", Dims(B=65, T=150, D=256, G=4, M=2, k=1), [(i * 29) % 150 for i in range(65)]),
]


def run_decode(d, dev):
    B, G, k = d.B, d.G, d.k
    y = torch.full((B, d.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    sel = torch.full((B, G, k), -7, dtype=torch.int32, device="cuda")
    w = torch.full((B, G, k), float("nan"), dtype=torch.float32, device="cuda")
    Kc, Vc = dev["K_cache"].clone(), dev["V_cache"].clone()
    ws = gqe.workspace(d, gqe.OP_DECODE)
    gqe.gqe_decode(d, dev["cache_len"], dev["x_new"], dev["Wq"], dev["Wk"], dev["Wv"], dev["Wr"], dev["br"],
                   dev["Wo"], Kc, Vc, y, sel, w, ws)
    status = gqe.gqe_check_error()
    return {"y": y.cpu(), "sel": sel.cpu(), "w": w.cpu(), "K": Kc.cpu(), "V": Vc.cpu(), "status": status}


def check_decode(d, lens, seed=0):
    inp = make_decode_inputs(d, lens, seed=seed)
    got = run_decode(d, to_dev(inp))
    assert got["status"] == 0, gqe.gqe_status_string(got["status"])
    chk = check_selection(d, inp["x_new"], inp["Wr"], inp["br"], got["sel"])
    # the oracle follows the GPU's choice on near ties (either is accepted)
    want = ref.gqe_decode(inp["x_new"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"],
                          inp["K_cache"], inp["V_cache"], lens, d, forced_sel=got["sel"].numpy())
    np.testing.assert_allclose(f64(got["w"]), want["w"], rtol=0, atol=2e-6)
    assert_close_bf16(got["y"], want["y"], "decode y")
    Kc0, Vc0 = inp["K_cache"], inp["V_cache"]
    for b, L in enumerate(lens):
        assert_close_bf16(got["K"][b, L], want["K_new"][b], f"appended K row of sequence {b}")
        assert_close_bf16(got["V"][b, L], want["V_new"][b], f"appended V row of sequence {b}")
        keep = torch.ones(d.T, dtype=torch.bool)
        keep[L] = False
        assert torch.equal(got["K"][b][keep], Kc0[b][keep]), f"K cache rows other than {L} changed"
        assert torch.equal(got["V"][b][keep], Vc0[b][keep]), f"V cache rows other than {L} changed"
    return chk


@pytest.mark.parametrize("name,d,lens", CASES, ids=[c[0] for c in CASES])
def test_decode_matches_oracle(name, d, lens):
    check_decode(d, lens)


def test_decode_main_shape_long_caches():
    """The main layer's shape (D 1024, G 8, M 2, k 1), eight sequences with
    cache lengths up to 32K (split-K over up to 32 chunks)."""
    d = Dims(B=8, T=32768, D=1024, G=8, M=2, k=1)
    rng = np.random.default_rng(11)
    lens = [0, 1, 4095, 4096, 12345, 20000, 32000, 32767]
    rng.shuffle(lens)
    check_decode(d, lens, seed=4)


def test_decode_steps_chain_like_a_generation_loop():
    """Three steps in a row: each step's appended row is read by the next."""
    d = Dims(B=2, T=64, D=256, G=4, M=2, k=1)
    inp = make_decode_inputs(d, [10, 20], seed=2)
    dev = to_dev(inp)
    Kc, Vc = dev["K_cache"].clone(), dev["V_cache"].clone()
    Kr, Vr = f64(inp["K_cache"]).copy(), f64(inp["V_cache"]).copy()
    lens = [10, 20]
    ws = gqe.workspace(d, gqe.OP_DECODE)
    gen = torch.Generator().manual_seed(9)
    for step in range(3):
        x_new = torch.randn((d.B, d.D), generator=gen).to(torch.bfloat16)
        y = torch.empty((d.B, d.D), dtype=torch.bfloat16, device="cuda")
        sel = torch.empty((d.B, d.G, d.k), dtype=torch.int32, device="cuda")
        w = torch.empty((d.B, d.G, d.k), dtype=torch.float32, device="cuda")
        cl = torch.tensor(lens, dtype=torch.int32, device="cuda")
        gqe.gqe_decode(d, cl, x_new.cuda(), dev["Wq"], dev["Wk"], dev["Wv"], dev["Wr"], dev["br"], dev["Wo"],
                       Kc, Vc, y, sel, w, ws)
        assert gqe.gqe_check_error() == 0
        want = ref.gqe_decode(x_new, inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], Kr, Vr, lens, d,
                              forced_sel=sel.cpu().numpy())
        assert_close_bf16(y.cpu(), want["y"], f"step {step} y")
        # the reference cache takes the GPU's appended rows (bf16), as the GPU's next step does
        for b in range(d.B):
            Kr[b, lens[b]] = f64(Kc[b, lens[b]].cpu())
            Vr[b, lens[b]] = f64(Vc[b, lens[b]].cpu())
        lens = [L + 1 for L in lens]


def test_decode_cache_length_out_of_range_is_reported():
    d = Dims(B=2, T=32, D=256, G=4, M=2, k=1)
    inp = make_decode_inputs(d, [3, 5], seed=1)
    dev = to_dev(inp)
    dev["cache_len"] = torch.tensor([3, 32], dtype=torch.int32, device="cuda")  # 32 == capacity: invalid
    got = run_decode(d, dev)
    assert got["status"] == -7  # GQE_ERR_DEVICE_CHECK; the bad sequence's cache is not touched
    assert torch.equal(got["K"][1], inp["K_cache"][1]) and torch.equal(got["V"][1], inp["V_cache"][1])
    assert gqe.gqe_check_error() == 0  # the check word was cleared by the first read
