"""Pins of the fp64 oracle against things other than itself (CPU only).

* hand-worked examples (tests/golden/*.txt, closed forms in e);
* brute force: pure-Python attention loops, subset enumeration for top-k;
* library special case: torch's scaled_dot_product_attention in fp64;
* closed-form invariants: rows of the attention matrix sum to 1, causality,
  k = M reduces to dense GQA plus the slot and shared terms, G = 1 is MQA,
  M = k = 1, T = 1;
* planted mistakes: perturbing the oracle in plausible ways makes a pin fail.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle.gqe_ref as ref
from gqe_inputs import Dims, make_inputs

from _golden import load


def _as_inputs(gold):
    return {k: gold[k] for k in ("x", "Wq", "Wk", "Wv", "Wr", "br", "Wo")}


def _run_golden(gold):
    d = gold["dims"]
    inp = _as_inputs(gold)
    return ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], d)


def _check_golden(gold, out):
    d = gold["dims"]
    np.testing.assert_array_equal(out["sel"], gold["expect.sel"].astype(np.int64))
    np.testing.assert_allclose(out["margin"], gold["expect.margin"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["w"], gold["expect.w"], rtol=0, atol=1e-12)
    O = out["O"].reshape(d.B * d.T, -1)
    np.testing.assert_allclose(O, gold["expect.O"], rtol=0, atol=1e-12)
    if "expect.A" in gold:
        np.testing.assert_allclose(out["A"], gold["expect.A"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out["y"], gold["expect.y"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("name", ["worked_example_k1.txt", "worked_example_k2.txt"])
def test_worked_example(name):
    gold = load(name)
    d = gold["dims"]
    out = _run_golden(gold)
    _check_golden(gold, out)
    if "expect.p_t0" in gold:
        np.testing.assert_allclose(out["p"][0], gold["expect.p_t0"], rtol=0, atol=1e-12)
    seg_off, seg_tok, row_map = ref.compact(out["sel"], d.B, d.T, d.G, d.M)
    np.testing.assert_array_equal(seg_off, gold["expect.seg_off"].astype(np.int64))
    np.testing.assert_array_equal(seg_tok, gold["expect.seg_tok"].astype(np.int64))
    np.testing.assert_array_equal(row_map, gold["expect.row_map"].astype(np.int64))


def test_tie_breaks_to_lower_expert():
    # two equal logits: the lower expert index is chosen, margin is exactly 0
    x = np.array([[1.0, 1.0]])
    Wr = np.array([[1.0, 0.0], [0.0, 1.0]])
    r = ref.route(x, Wr, None, G=1, M=2, k=1)
    assert r["sel"][0, 0, 0] == 0
    assert r["margin"][0, 0] == 0.0
    # three-way tie with k = 2 picks {0, 1}
    Wr3 = np.zeros((2, 3))
    r3 = ref.route(x, Wr3, None, G=1, M=3, k=2)
    np.testing.assert_array_equal(r3["sel"][0, 0], [0, 1])


@pytest.mark.parametrize("M,k", [(2, 1), (3, 2), (4, 2), (5, 3), (4, 4)])
def test_topk_matches_subset_enumeration(M, k):
    rng = np.random.default_rng(M * 10 + k)
    N, D, G = 64, 8, 3
    x = rng.standard_normal((N, D))
    Wr = rng.standard_normal((D, G * M))
    br = rng.standard_normal(G * M)
    r = ref.route(x, Wr, br, G, M, k)
    logits = x @ Wr + br
    for n in range(N):
        for g in range(G):
            lg = [float(v) for v in logits[n, g * M:(g + 1) * M]]
            z = sum(math.exp(v) for v in lg)
            p = [math.exp(v) / z for v in lg]
            best = max(itertools.combinations(range(M), k), key=lambda c: sum(p[i] for i in c))
            assert tuple(r["sel"][n, g]) == best
            tot = sum(p[i] for i in best)
            np.testing.assert_allclose(r["w"][n, g], [p[i] / tot for i in best], rtol=1e-12)
            np.testing.assert_allclose(r["p"][n, g], p, rtol=1e-12)
            srt = sorted(lg, reverse=True)
            exp_margin = srt[k - 1] - srt[k] if k < M else math.inf
            assert r["margin"][n, g] == pytest.approx(exp_margin, abs=1e-12)


def _attn_pure_python(q, K, V, t, scale):
    """Brute force: loops over s <= t with math.exp, no numpy arithmetic."""
    sc = [scale * sum(q[d] * K[s][d] for d in range(len(q))) for s in range(t + 1)]
    m = max(sc)
    ws = [math.exp(v - m) for v in sc]
    z = sum(ws)
    return [sum(ws[s] * V[s][d] for s in range(t + 1)) / z for d in range(len(V[0]))]


@pytest.mark.parametrize("T,dh", [(1, 4), (7, 3), (16, 8)])
def test_attention_matches_pure_python_bruteforce(T, dh):
    rng = np.random.default_rng(T * 100 + dh)
    Q = rng.standard_normal((T, dh))
    K = rng.standard_normal((T, dh))
    V = rng.standard_normal((T, dh))
    scale = 1.0 / math.sqrt(dh)
    O = ref.causal_attention(Q, np.arange(T), K, V, scale)
    for t in range(T):
        bf = _attn_pure_python(Q[t].tolist(), K.tolist(), V.tolist(), t, scale)
        np.testing.assert_allclose(O[t], bf, rtol=0, atol=1e-12)


def test_attention_rows_sum_to_one_and_are_causal():
    rng = np.random.default_rng(7)
    T, dh = 40, 16
    Q = rng.standard_normal((T, dh)) * 3
    K = rng.standard_normal((T, dh))
    P = ref.attention_weights(Q, np.arange(T), K, 0.25)
    np.testing.assert_allclose(P.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert np.all(P[np.triu_indices(T, 1)] == 0.0)
    assert np.all(P[np.tril_indices(T)] > 0.0)


def test_attention_matches_torch_sdpa_fp64():
    rng = np.random.default_rng(11)
    T, dh = 96, 64
    Q = rng.standard_normal((T, dh))
    K = rng.standard_normal((T, dh))
    V = rng.standard_normal((T, dh))
    O = ref.causal_attention(Q, np.arange(T), K, V, 1.0 / math.sqrt(dh))
    tq, tk, tv = (torch.from_numpy(a)[None, None] for a in (Q, K, V))
    Ot = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(O, Ot, rtol=0, atol=1e-12)


def _small(B=2, T=24, D=32, G=2, M=2, k=1, dh=8, bias0=0.0, seed=3):
    d = Dims(B=B, T=T, D=D, G=G, M=M, k=k, dh=dh, bias0=bias0)
    inp = make_inputs(d, seed=seed)
    # small D: raise the weight scale so routing and attention are not flat
    for key in ("Wq", "Wk", "Wv", "Wr", "Wo", "Wo_dense"):
        inp[key] = (inp[key].float() * 20).to(torch.bfloat16)
    return d, inp


def _fwd(d, inp, **kw):
    return ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], d, **kw)


def _sdpa_heads(Qh, Kg, Vg, dh):
    """torch SDPA in fp64: Qh [T, H, dh], Kg/Vg [T, H, dh] (already expanded)."""
    q = torch.from_numpy(np.ascontiguousarray(Qh.transpose(1, 0, 2)))[None]
    kk = torch.from_numpy(np.ascontiguousarray(Kg.transpose(1, 0, 2)))[None]
    vv = torch.from_numpy(np.ascontiguousarray(Vg.transpose(1, 0, 2)))[None]
    o = torch.nn.functional.scaled_dot_product_attention(q, kk, vv, is_causal=True, scale=1.0 / math.sqrt(dh))
    return o[0].numpy().transpose(1, 0, 2)


def test_dense_gqa_matches_sdpa_with_expanded_kv():
    d, inp = _small(B=2, T=20, G=2, M=3)
    out = ref.gqa_dense_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wo_dense"], d)
    X = inp["x"].double().numpy()
    H = d.G * d.M
    for b in range(d.B):
        xb = X[b * d.T:(b + 1) * d.T]
        Q = (xb @ inp["Wq"].double().numpy()[:, :H * d.dh]).reshape(d.T, H, d.dh)
        K = (xb @ inp["Wk"].double().numpy()).reshape(d.T, d.G, d.dh)
        V = (xb @ inp["Wv"].double().numpy()).reshape(d.T, d.G, d.dh)
        kv_of_head = np.arange(H) // d.M
        O = _sdpa_heads(Q, K[:, kv_of_head], V[:, kv_of_head], d.dh)
        np.testing.assert_allclose(out["O"][b * d.T:(b + 1) * d.T], O, rtol=0, atol=1e-12)
        y = O.reshape(d.T, H * d.dh) @ inp["Wo_dense"].double().numpy()
        np.testing.assert_allclose(out["y"][b * d.T:(b + 1) * d.T], y, rtol=0, atol=1e-11)


def test_gqe_attention_matches_sdpa_per_selected_head():
    d, inp = _small(B=2, T=20, G=2, M=4, k=2)
    out = _fwd(d, inp)
    X = inp["x"].double().numpy()
    Wq = inp["Wq"].double().numpy()
    for b in range(d.B):
        xb = X[b * d.T:(b + 1) * d.T]
        K = (xb @ inp["Wk"].double().numpy()).reshape(d.T, d.G, d.dh)
        V = (xb @ inp["Wv"].double().numpy()).reshape(d.T, d.G, d.dh)
        Qall = (xb @ Wq).reshape(d.T, d.G * d.M + 1, d.dh)
        Oall = _sdpa_heads(Qall, K[:, list(np.arange(d.G * d.M) // d.M) + [0]],
                           V[:, list(np.arange(d.G * d.M) // d.M) + [0]], d.dh)
        for t in range(d.T):
            n = b * d.T + t
            for g in range(d.G):
                for j in range(d.k):
                    h = g * d.M + out["sel"][n, g, j]
                    np.testing.assert_allclose(out["O"][n, g * d.k + j], Oall[t, h], rtol=0, atol=1e-12)
            np.testing.assert_allclose(out["O"][n, d.G * d.k], Oall[t, d.G * d.M], rtol=0, atol=1e-12)


def test_causality_future_tokens_do_not_change_outputs():
    d, inp = _small(B=1, T=32)
    base = _fwd(d, inp)
    t0 = 17
    pert = dict(inp)
    x = inp["x"].clone()
    x[t0 + 1:] = torch.randn(x[t0 + 1:].shape, generator=torch.Generator().manual_seed(5)).to(torch.bfloat16)
    pert["x"] = x
    out = _fwd(d, pert)
    # bitwise: routing is per token and masked scores contribute exact zeros
    assert np.array_equal(out["y"][:t0 + 1], base["y"][:t0 + 1])
    assert not np.array_equal(out["y"][t0 + 1:], base["y"][t0 + 1:])


def test_k_equals_m_is_dense_gqa_plus_slot_and_shared():
    d, inp = _small(B=2, T=16, G=2, M=3, k=3)
    out = _fwd(d, inp)
    cdim = d.G * d.k * d.dh
    Wo = inp["Wo"].double().numpy()
    dense = ref.gqa_dense_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], torch.from_numpy(Wo[:cdim]), d)
    # slot = sum_e p_e O_e over all experts (renormalisation over the full pool is p itself)
    O = dense["O"].reshape(-1, d.G, d.M, d.dh)
    slot = np.einsum("nge,nged->ngd", out["p"], O).reshape(-1, d.G * d.dh)
    shared = out["O"][:, d.G * d.k]
    expect = dense["y"] + slot @ Wo[cdim:cdim + d.G * d.dh] + shared @ Wo[cdim + d.G * d.dh:]
    np.testing.assert_allclose(out["y"], expect, rtol=0, atol=1e-11)
    # zero slot and shared rows: exactly the dense layer with Wo_dense = concat rows
    Wo0 = Wo.copy()
    Wo0[cdim:] = 0
    out0 = ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], Wo0, d)
    np.testing.assert_allclose(out0["y"], dense["y"], rtol=0, atol=1e-12)


def test_g1_is_multi_query_attention():
    d, inp = _small(B=1, T=20, G=1, M=3, k=3)
    out = _fwd(d, inp)
    X = inp["x"].double().numpy()
    K = (X @ inp["Wk"].double().numpy()).reshape(d.T, 1, d.dh)
    V = (X @ inp["Wv"].double().numpy()).reshape(d.T, 1, d.dh)
    Q = (X @ inp["Wq"].double().numpy()).reshape(d.T, d.M + 1, d.dh)
    O = _sdpa_heads(Q, np.repeat(K, d.M + 1, axis=1), np.repeat(V, d.M + 1, axis=1), d.dh)
    np.testing.assert_allclose(out["O"], O, rtol=0, atol=1e-12)


def test_m1_k1_every_token_routes_to_its_only_expert():
    d, inp = _small(B=1, T=16, G=3, M=1, k=1)
    out = _fwd(d, inp)
    assert np.all(out["sel"] == 0)
    assert np.all(out["w"] == 1.0)
    cdim = d.G * d.dh
    # slot equals the concat part exactly
    np.testing.assert_array_equal(out["A"][:, cdim:2 * cdim], out["A"][:, :cdim])


def test_t1_every_head_returns_v0_of_its_kv_group():
    d, inp = _small(B=3, T=1, G=2, M=2, k=1)
    out = _fwd(d, inp)
    X = inp["x"].double().numpy()
    V = (X @ inp["Wv"].double().numpy()).reshape(d.B, d.G, d.dh)
    for n in range(d.B):
        for g in range(d.G):
            np.testing.assert_allclose(out["O"][n, g], V[n, g], rtol=0, atol=1e-14)
        np.testing.assert_allclose(out["O"][n, d.G], V[n, 0], rtol=0, atol=1e-14)
    A = np.concatenate([V.reshape(d.B, -1), V.reshape(d.B, -1), V[:, 0]], axis=1)
    np.testing.assert_allclose(out["y"], A @ inp["Wo"].double().numpy(), rtol=0, atol=1e-13)


def test_rows_subset_equals_full_run():
    d, inp = _small(B=2, T=24, G=2, M=2, k=1)
    full = _fwd(d, inp)
    rows = np.array([0, 5, 23, 24, 31, 47])
    sub = _fwd(d, inp, rows=rows)
    np.testing.assert_allclose(sub["y"], full["y"][rows], rtol=0, atol=1e-13)
    np.testing.assert_array_equal(sub["sel"], full["sel"][rows])


def test_forced_selection_follows_the_given_experts():
    d, inp = _small(B=1, T=12, G=2, M=3, k=2)
    full = _fwd(d, inp)
    same = _fwd(d, inp, forced_sel=full["sel"])
    np.testing.assert_array_equal(same["y"], full["y"])
    flipped = full["sel"].copy()
    flipped[3, 1] = [0, 1] if tuple(flipped[3, 1]) != (0, 1) else [1, 2]
    out = _fwd(d, inp, forced_sel=flipped)
    p = full["p"][3, 1, flipped[3, 1]]
    np.testing.assert_allclose(out["w"][3, 1], p / p.sum(), rtol=1e-13)
    assert not np.allclose(out["y"][3], full["y"][3])


def test_compaction_is_a_permutation_in_ascending_token_order():
    rng = np.random.default_rng(2)
    B, T, G, M, k = 3, 50, 4, 4, 2
    sel = np.sort(np.stack([np.stack([rng.choice(M, k, replace=False) for _ in range(G)]) for _ in range(B * T)]), axis=2)
    seg_off, seg_tok, row_map = ref.compact(sel, B, T, G, M)
    assert seg_off[-1] == B * T * G * k
    seen = np.zeros(B * T * G * k, dtype=int)
    for n in range(B * T):
        for g in range(G):
            for j in range(k):
                r = row_map[n, g, j]
                s = (n // T * G + g) * M + sel[n, g, j]
                assert seg_off[s] <= r < seg_off[s + 1]
                assert seg_tok[r] == n
                seen[r] += 1
    assert np.all(seen == 1)
    for s in range(B * G * M):
        assert np.all(np.diff(seg_tok[seg_off[s]:seg_off[s + 1]]) > 0)


def test_sample_rows_cover_ends_of_every_sequence():
    rows = ref.sample_rows(B=2, T=1000, n_uniform=50, seed=0)
    for b in range(2):
        assert b * 1000 in rows and b * 1000 + 999 in rows
    assert np.all(np.diff(rows) > 0)


# --- planted mistakes: each plausible slip in the oracle trips a pin ---------

def _golden_fails(monkeypatch, name, attr, fake):
    monkeypatch.setattr(ref, attr, fake)
    gold = load(name)
    with pytest.raises(AssertionError):
        _check_golden(gold, _run_golden(gold))


def test_planted_no_causal_mask_is_caught(monkeypatch):
    orig = ref.attention_weights

    def no_mask(q, pos, Kb, scale):
        return orig(q, np.full_like(np.asarray(pos), Kb.shape[0] - 1), Kb, scale)
    _golden_fails(monkeypatch, "worked_example_k1.txt", "attention_weights", no_mask)


def test_planted_k_v_swap_is_caught(monkeypatch):
    orig = ref._project_kv

    def swapped(X, Wk, Wv, B, T, G, dh):
        K, V = orig(X, Wk, Wv, B, T, G, dh)
        return V, K
    _golden_fails(monkeypatch, "worked_example_k1.txt", "_project_kv", swapped)


def test_planted_missing_renormalisation_is_caught(monkeypatch):
    orig = ref.route

    def raw_p(*a, **kw):
        r = orig(*a, **kw)
        r["w"] = np.take_along_axis(r["p"], r["sel"], axis=2)
        return r
    _golden_fails(monkeypatch, "worked_example_k2.txt", "route", raw_p)


def test_planted_descending_concat_order_is_caught(monkeypatch):
    orig = ref.route

    def desc(*a, **kw):
        r = orig(*a, **kw)
        r["sel"] = r["sel"][:, :, ::-1].copy()
        r["w"] = r["w"][:, :, ::-1].copy()
        return r
    _golden_fails(monkeypatch, "worked_example_k2.txt", "route", desc)


def test_planted_wrong_softmax_scale_is_caught():
    rng = np.random.default_rng(1)
    Q, K, V = (rng.standard_normal((12, 16)) for _ in range(3))
    good = ref.causal_attention(Q, np.arange(12), K, V, 0.25)
    bad = ref.causal_attention(Q, np.arange(12), K, V, 1.0 / 16)
    Ot = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a)[None, None] for a in (Q, K, V)), is_causal=True)[0, 0].numpy()
    np.testing.assert_allclose(good, Ot, atol=1e-12)
    assert not np.allclose(bad, Ot, atol=1e-6)


# ---------------------------------------------------------------------------
# Decode step with a key/value cache
# ---------------------------------------------------------------------------
def _decode_from_forward(d, inp, lens, garbage_seed=None):
    """Inputs of one decode step built from a full forward run: the cache of
    sequence b holds the forward's K/V at positions < lens[b] (garbage past
    them when garbage_seed is given) and the new token is x at lens[b]."""
    full = _fwd(d, inp)
    X = inp["x"].reshape(d.B, d.T, d.D)
    x_new = torch.stack([X[b, lens[b]] for b in range(d.B)])
    K = full["K"].copy()
    V = full["V"].copy()
    if garbage_seed is not None:
        rng = np.random.default_rng(garbage_seed)
        for b in range(d.B):
            K[b, lens[b]:] = rng.normal(size=K[b, lens[b]:].shape) * 5
            V[b, lens[b]:] = rng.normal(size=V[b, lens[b]:].shape) * 5
    return full, x_new, K, V


def _dec(d, inp, x_new, K, V, lens, **kw):
    return ref.gqe_decode(x_new, inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], K, V, lens, d, **kw)


@pytest.mark.parametrize("G,M,k", [(2, 2, 1), (2, 3, 2), (1, 4, 4)])
def test_decode_equals_forward_at_the_last_position(G, M, k):
    d, inp = _small(B=3, T=40, G=G, M=M, k=k)
    lens = [39, 17, 0]
    full, x_new, K, V = _decode_from_forward(d, inp, lens, garbage_seed=5)
    out = _dec(d, inp, x_new, K, V, lens)
    rows = np.array([b * d.T + lens[b] for b in range(d.B)])
    np.testing.assert_allclose(out["y"], full["y"][rows], rtol=0, atol=1e-12)
    np.testing.assert_array_equal(out["sel"], full["sel"][rows])
    np.testing.assert_allclose(out["w"], full["w"][rows], rtol=0, atol=1e-14)
    for b in range(d.B):
        np.testing.assert_allclose(out["K_new"][b], full["K"][b, lens[b]], rtol=0, atol=1e-13)
        np.testing.assert_allclose(out["V_new"][b], full["V"][b, lens[b]], rtol=0, atol=1e-13)


def test_decode_with_an_empty_cache_returns_the_new_value():
    d, inp = _small(B=2, T=4, G=2, M=2, k=1)
    X = inp["x"].double().numpy()[:d.B]
    K = np.zeros((d.B, d.T, d.G, d.dh))
    out = _dec(d, inp, inp["x"][:d.B], K, K, [0, 0])
    Vn = (X @ inp["Wv"].double().numpy()).reshape(d.B, d.G, d.dh)
    for b in range(d.B):
        for g in range(d.G):
            np.testing.assert_allclose(out["O"][b, g], Vn[b, g], rtol=0, atol=1e-14)
        np.testing.assert_allclose(out["O"][b, d.G], Vn[b, 0], rtol=0, atol=1e-14)
    A = np.concatenate([Vn.reshape(d.B, -1), Vn.reshape(d.B, -1), Vn[:, 0]], axis=1)
    np.testing.assert_allclose(out["y"], A @ inp["Wo"].double().numpy(), rtol=0, atol=1e-13)


def test_decode_reads_exactly_the_first_cache_len_rows():
    d, inp = _small(B=2, T=30, G=2, M=3, k=2)
    lens = [12, 29]
    _, x_new, K, V = _decode_from_forward(d, inp, lens)
    base = _dec(d, inp, x_new, K, V, lens)["y"]
    K2, V2 = K.copy(), V.copy()
    K2[0, 12:] += 3.0
    V2[0, 12:] -= 3.0
    np.testing.assert_array_equal(_dec(d, inp, x_new, K2, V2, lens)["y"], base)
    K3 = K.copy()
    K3[0, 11, 0] += 1.0
    assert not np.allclose(_dec(d, inp, x_new, K3, V, lens)["y"][0], base[0])
    np.testing.assert_array_equal(_dec(d, inp, x_new, K3, V, lens)["y"][1], base[1])


# ---------------------------------------------------------------------------
# Ablation variants of the output construction
# ---------------------------------------------------------------------------
def _variant(d, inp, mode, Wo, **kw):
    return ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], Wo, d,
                           combine_mode=mode, **kw)


def _wo_variant(d, mode="hard", seed=4):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn((ref.combine_width(d, mode), d.D), generator=g) * 0.4).to(torch.bfloat16)


def test_variant_widths_follow_the_construction():
    d = Dims(B=1, T=1, D=64, G=8, M=2, k=1)
    assert [ref.combine_width(d, m) // 64 for m in ("slot",) + ref.VARIANTS] == [17, 9, 9, 10, 16]


@pytest.mark.parametrize("G,M,k", [(2, 2, 1), (2, 3, 2)])
def test_variant_hard_is_the_slot_construction_without_its_slot(G, M, k):
    d, inp = _small(B=2, T=20, G=G, M=M, k=k)
    full = _fwd(d, inp)
    hard = _variant(d, inp, "hard", _wo_variant(d))
    gk = d.G * d.k * d.dh
    np.testing.assert_array_equal(hard["A"], np.concatenate([full["A"][:, :gk], full["A"][:, -d.dh:]], axis=1))
    np.testing.assert_allclose(hard["y"], hard["A"] @ _wo_variant(d).double().numpy(), rtol=0, atol=1e-12)


def test_variant_weighted_with_a_single_expert_equals_hard():
    d, inp = _small(B=2, T=16, G=3, M=1, k=1)
    Wo = _wo_variant(d)
    np.testing.assert_allclose(_variant(d, inp, "weighted", Wo)["y"], _variant(d, inp, "hard", Wo)["y"],
                               rtol=0, atol=1e-14)


def test_variant_weighted_scales_by_the_hand_worked_probabilities():
    """Token 0 of the hand-worked example: group 0 selects expert 0 with
    in-group probability e/(1+e), group 1 expert 1 with e^2/(1+e^2) (not the
    renormalised weight 1)."""
    gold = load("worked_example_k1.txt")
    d = gold["dims"]
    inp = _as_inputs(gold)
    Wo = torch.ones(((d.G * d.k + 1) * d.dh, d.D), dtype=torch.float64)
    out = _variant(d, inp, "weighted", Wo)
    p0 = gold["expect.p_t0"]
    O0 = gold["expect.O"][0]
    np.testing.assert_allclose(out["A"][0], [p0[0, 0] * O0[0], p0[1, 1] * O0[1], O0[2]], rtol=0, atol=1e-14)
    assert abs(out["A"][0][0] - O0[0]) > 0.1  # the renormalised weight (1) would give O0[0]


def test_planted_renormalised_weights_in_the_weighted_variant_are_caught(monkeypatch):
    real = ref.combine_variant
    monkeypatch.setattr(ref, "combine_variant",
                        lambda O, w, p_sel, dims, mode: real(O, w, np.ones_like(p_sel), dims, mode))
    with pytest.raises(AssertionError):
        test_variant_weighted_scales_by_the_hand_worked_probabilities()


def test_variant_global_slot_of_the_hand_worked_example():
    """The single global slot of the hand-worked example (G = 2, k = 1, dh = 1).
    Token 0: group 0 keeps expert 0 (logits 1, 0: p = e/(1+e)), group 1 keeps
    expert 1 of its pair (logits 0, 2: p = e^2/(1+e^2)); outputs 1 and 2.
    Token 1: group 0 keeps expert 1 (logits 0, 1: p = e/(1+e)) with output
    (e+3)/(e+1), group 1 keeps expert 0 (logits 3, 0: p = e^3/(1+e^3)) with
    output 1. The slot is the probability-weighted average of the two."""
    gold = load("worked_example_k1.txt")
    d = gold["dims"]
    inp = _as_inputs(gold)
    Wo = torch.ones((ref.combine_width(d, "global_slot"), d.D), dtype=torch.float64)
    out = _variant(d, inp, "global_slot", Wo)
    e = math.e
    pa, pb = e / (1 + e), e * e / (1 + e * e)
    want0 = (pa * 1 + pb * 2) / (pa + pb)
    pa, pb = e / (1 + e), e ** 3 / (1 + e ** 3)
    want1 = (pa * (e + 3) / (e + 1) + pb * 1) / (pa + pb)
    O = gold["expect.O"]
    np.testing.assert_allclose(out["A"][0], [O[0][0], O[0][1], want0, O[0][2]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["A"][1], [O[1][0], O[1][1], want1, O[1][2]], rtol=0, atol=1e-14)
    np.testing.assert_allclose(out["y"][:, 0], out["A"].sum(axis=1), rtol=0, atol=1e-13)


def test_variant_global_slot_averages_equal_outputs_to_themselves():
    """Whatever the probabilities, a weighted average of G*k copies of one
    vector is that vector: pins the division by the summed probabilities."""
    d = Dims(B=1, T=5, D=8, G=3, M=4, k=2, dh=4)
    rng = np.random.default_rng(0)
    u = rng.standard_normal((5, 1, 4))
    O = np.concatenate([np.repeat(u, d.G * d.k, axis=1), rng.standard_normal((5, 1, 4))], axis=1)
    p_sel = rng.uniform(0.05, 0.9, size=(5, d.G, d.k))
    A = ref.combine_variant(O, None, p_sel, d, "global_slot")
    gk = d.G * d.k * d.dh
    np.testing.assert_allclose(A[:, gk:gk + d.dh], u[:, 0], rtol=0, atol=1e-14)
    np.testing.assert_array_equal(A[:, -d.dh:], O[:, -1])


def test_variant_global_slot_with_one_group_is_the_per_group_slot():
    """With G = 1 the selected set of the only group is the set of all
    selected experts, so the global slot is the GQE slot (same A)."""
    d, inp = _small(B=2, T=18, G=1, M=3, k=2)
    full = _fwd(d, inp)
    glob = _variant(d, inp, "global_slot", _wo_variant(d, "global_slot"))
    np.testing.assert_allclose(glob["A"], full["A"], rtol=0, atol=1e-13)


@pytest.mark.parametrize("G,M,k", [(2, 2, 1), (3, 3, 2)])
def test_variant_no_shared_is_the_slot_construction_without_the_shared_head(G, M, k):
    d, inp = _small(B=2, T=20, G=G, M=M, k=k)
    full = _fwd(d, inp)
    Wo = _wo_variant(d, "no_shared")
    out = _variant(d, inp, "no_shared", Wo)
    np.testing.assert_array_equal(out["A"], full["A"][:, :-d.dh])
    # the shared head's query weights no longer reach y
    inp2 = dict(inp)
    Wq = inp["Wq"].clone()
    Wq[:, d.G * d.M * d.dh:] = 0
    inp2["Wq"] = Wq
    np.testing.assert_array_equal(_variant(d, inp2, "no_shared", Wo)["y"], out["y"])
    assert not np.allclose(_fwd(d, inp2)["y"], full["y"])


def test_planted_per_group_average_in_the_global_slot_is_caught(monkeypatch):
    """A slot that averages the groups' renormalised slots (each group's
    weights summing to 1, then divided by G) is a different construction."""
    real = ref.combine_variant

    def per_group_average(O, w, p_sel, dims, mode):
        if mode != "global_slot":
            return real(O, w, p_sel, dims, mode)
        p = np.asarray(p_sel, np.float64)
        return real(O, w, p / p.sum(axis=2, keepdims=True) / dims.G, dims, mode)

    monkeypatch.setattr(ref, "combine_variant", per_group_average)
    with pytest.raises(AssertionError):
        test_variant_global_slot_of_the_hand_worked_example()


def test_planted_unnormalised_global_slot_is_caught(monkeypatch):
    real = ref.combine_variant

    def unnormalised(O, w, p_sel, dims, mode):
        A = real(O, w, p_sel, dims, mode)
        if mode == "global_slot":
            gk = dims.G * dims.k * dims.dh
            A[:, gk:gk + dims.dh] *= np.asarray(p_sel, np.float64).reshape(A.shape[0], -1).sum(axis=1)[:, None]
        return A

    monkeypatch.setattr(ref, "combine_variant", unnormalised)
    with pytest.raises(AssertionError):
        test_variant_global_slot_averages_equal_outputs_to_themselves()


# ---------------------------------------------------------------------------
# The skewed-routing input recipe against its closed form
# ---------------------------------------------------------------------------
def test_skewed_recipe_expert0_shares_match_the_closed_form():
    """x ~ N(0, 1) and Wr ~ N(0, 0.02^2) make the logits of a group nearly
    independent N(0, s^2), s = 0.02 sqrt(D). With the +2 bias on expert 0 of
    M = 4, expert 0 ranks first with probability E[Phi(Z + 2/s)^3] and lands
    in the top 2 with probability E[Phi^3 + 3 Phi^2 (1 - Phi)], Z ~ N(0, 1)
    (numerical integration). The oracle's routing of 4096 tokens x 8 groups
    must match both to 0.015."""
    d = Dims(B=1, T=4096, D=2048, G=8, M=4, k=2, bias0=2.0)
    inp = make_inputs(d, seed=0)
    r = ref.route(inp["x"], inp["Wr"], inp["br"], d.G, d.M, d.k)
    rank1 = float(np.mean(np.argmax(r["p"], axis=2) == 0))
    top2 = float(np.mean(np.any(r["sel"] == 0, axis=2)))
    a0 = 2.0 / (0.02 * math.sqrt(d.D))
    z = np.linspace(-10.0, 10.0, 40001)
    phi = np.exp(-0.5 * z * z) / math.sqrt(2.0 * math.pi)
    Phi = np.array([0.5 * (1.0 + math.erf((v + a0) / math.sqrt(2.0))) for v in z])
    want1 = float(np.trapezoid(phi * Phi ** 3, z))
    want2 = float(np.trapezoid(phi * (Phi ** 3 + 3.0 * Phi ** 2 * (1.0 - Phi)), z))
    assert abs(rank1 - want1) < 0.015, (rank1, want1)
    assert abs(top2 - want2) < 0.015, (top2, want2)
    assert 0.85 < want1 < 0.88 and 0.96 < want2 < 0.975
