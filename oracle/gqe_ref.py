"""fp64 CPU oracle of the Grouped Query Experts (GQE) attention forward pass.

TEST INFRASTRUCTURE. Only the tests, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use this module. The CUDA library never imports,
links or calls it, and it imports nothing from the CUDA library. It is a plain,
slow, obviously correct restatement of what the layer computes, in float64,
taking the bf16 input values (exact in float64).

Sources (the method is described in prose only; no formula or code is printed):
  [GS]  "Grouped Query Experts: Mixture-of-Experts on GQA Self-Attention",
        gist.science technical summary (zh / it / es editions), section
        "Architecture and routing" (grouped expert pool, conditional activation,
        dense KV path, output construction: hard concatenation, renormalised
        weighted sum, always-on shared head).
  [AT]  animattoys.com article on the same paper ("讓AI的注意力學會偷懶…"),
        section 4 "How GQE works": per-group router scores, top-k activation,
        each selected expert attends independently, concat + weighted-average
        slot + shared head merged and passed through the output projection.
  [WK]  aiboss88.com wiki "Grouped-Query Attention": query heads of one group
        share one KV head; G = 1 is MQA, G = H is MHA.

Readings where the pages are silent (each one is listed with its reason in the
design notes of this repository):
  * router = linear map of the layer input, logits = x Wr + br, no noise;
  * probabilities = softmax over the M experts of each group;
  * top-k by probability, exact ties broken toward the lower expert index; the
    selected set is concatenated in ascending expert order;
  * renormalised weights w = p_sel / sum(p_sel) over the selected set;
  * one weighted slot per group;
  * shared head attends KV head 0;
  * scale 1/sqrt(dh), causal mask s <= t, no positional encoding or biases;
  * Wo rows: [concat (g-major, slot j) | slot g | shared];
  * variants of the output construction ([AT] sections 4 and 6, [GS]
    "Experimental results"): the hard and the weighted concatenation keep
    the shared head; the weights of the weighted one are the in-group
    probabilities of the selected experts (not renormalised); the single
    global slot averages all selected outputs with those probabilities
    renormalised over all groups; the no-shared-head variant keeps the
    per-group slots;
  * decode step: the new token of sequence b sits at position cache_len[b],
    its K/V row is appended there and its queries attend positions
    0..cache_len[b] (the pages describe no decode procedure).

Layout conventions (match the ones ``gqe_inputs`` draws): x [B*T, D],
Wq [D, (G*M+1)*dh] with routed head h = g*M + e and the shared head last,
Wk/Wv [D, G*dh], Wr [D, G*M], br [G*M], Wo [(G*k+G+1)*dh, D],
Wo_dense [G*M*dh, D]. Token n = b*T + t.

Every function here is pinned by tests/test_oracle.py against hand-worked
examples, brute force and closed-form invariants.
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


def _f64(a) -> np.ndarray:
    """bf16/fp32 torch tensor or array -> float64 numpy (exact)."""
    if hasattr(a, "detach"):
        a = a.detach().to("cpu").float().numpy()
    return np.asarray(a, dtype=F64)


# ---------------------------------------------------------------------------
# Router: [GS] "Conditional activation"; [AT] section 4, routing decision.
# ---------------------------------------------------------------------------
def route(x, Wr, br, G: int, M: int, k: int, forced_sel=None) -> dict:
    """Per-token, per-group expert choice.

    logits[n, g, e] = x[n] . Wr[:, g*M + e] + br[g*M + e]
    p[n, g, :]      = softmax over the M experts of group g
    sel[n, g, :]    = the k experts with the largest p (ties: lower index),
                      listed in ascending expert index
    w[n, g, j]      = p[sel_j] / sum_j' p[sel_j']     (renormalised)
    margin[n, g]    = logit of the k-th ranked expert minus that of the
                      (k+1)-th (+inf when k == M): how far the choice is from
                      flipping.
    ``forced_sel`` replaces the choice (the weights follow it).
    """
    X = _f64(x)
    logits = X @ _f64(Wr)
    if br is not None:
        logits = logits + _f64(br)[None, :]
    n = X.shape[0]
    logits = logits.reshape(n, G, M)
    mx = logits.max(axis=2, keepdims=True)
    ex = np.exp(logits - mx)
    p = ex / ex.sum(axis=2, keepdims=True)

    # rank experts: larger logit first (same order as p), exact ties -> lower e
    idx = np.broadcast_to(np.arange(M), logits.shape)
    order = np.lexsort((idx, -logits), axis=-1)          # [n, G, M]
    ranked = np.take_along_axis(logits, order, axis=2)
    if k < M:
        margin = ranked[:, :, k - 1] - ranked[:, :, k]
    else:
        margin = np.full((n, G), np.inf)

    if forced_sel is None:
        sel = np.sort(order[:, :, :k], axis=2)
    else:
        sel = np.sort(np.asarray(forced_sel, dtype=np.int64).reshape(n, G, k), axis=2)
    psel = np.take_along_axis(p, sel, axis=2)
    w = psel / psel.sum(axis=2, keepdims=True)
    return {"logits": logits, "p": p, "sel": sel.astype(np.int64), "w": w, "margin": margin}


def compact(sel, B: int, T: int, G: int, M: int):
    """Token lists per segment s = (b*G + g)*M + e, tokens ascending.

    seg_off [B*G*M + 1]: exclusive prefix of the segment lengths.
    seg_tok [B*T*G*k]  : flat token index n = b*T + t of each compacted row.
    row_map [B*T, G, k]: compacted row of (n, g, slot j).
    This is the bookkeeping that lets the query projection run only for the
    selected experts ([GS] "Conditional activation"; [AT] section 4).
    """
    sel = np.asarray(sel).reshape(B * T, G, -1)
    k = sel.shape[2]
    seg_off = np.zeros(B * G * M + 1, dtype=np.int64)
    seg_tok = np.zeros(B * T * G * k, dtype=np.int64)
    row_map = np.zeros((B * T, G, k), dtype=np.int64)
    pos = 0
    for b in range(B):
        for g in range(G):
            for e in range(M):
                s = (b * G + g) * M + e
                seg_off[s] = pos
                toks_local, slots = np.nonzero(sel[b * T:(b + 1) * T, g, :] == e)
                toks = toks_local + b * T                      # ascending
                seg_tok[pos:pos + len(toks)] = toks
                row_map[toks, g, slots] = pos + np.arange(len(toks))
                pos += len(toks)
    seg_off[B * G * M] = pos
    return seg_off, seg_tok, row_map


# ---------------------------------------------------------------------------
# Causal scaled dot-product attention of one head against one KV head.
# [AT] section 4: each selected expert computes attention independently
# against its group's (shared, dense) K/V; [GS] "Dense KV path".
# ---------------------------------------------------------------------------
def attention_weights(q, pos, Kb, scale: float) -> np.ndarray:
    """softmax_s(q_r . K_s * scale) over s <= pos_r; zeros for s > pos_r."""
    q = np.asarray(q, F64)
    pos = np.asarray(pos, dtype=np.int64)
    tmax = int(pos.max()) + 1
    S = (q @ Kb[:tmax].T) * scale
    S[np.arange(tmax)[None, :] > pos[:, None]] = -np.inf
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    return P / P.sum(axis=1, keepdims=True)


def causal_attention(q, pos, Kb, Vb, scale: float, chunk_elems: int = 1 << 24) -> np.ndarray:
    """o_r = sum_{s <= pos_r} softmax(q_r . K_s * scale) V_s, row by row."""
    q = np.asarray(q, F64)
    pos = np.asarray(pos, dtype=np.int64)
    out = np.zeros((q.shape[0], Vb.shape[1]), dtype=F64)
    if q.shape[0] == 0:
        return out
    tmax = int(pos.max()) + 1
    step = max(1, chunk_elems // tmax)
    for r0 in range(0, q.shape[0], step):
        sl = slice(r0, r0 + step)
        P = attention_weights(q[sl], pos[sl], Kb, scale)
        out[sl] = P @ Vb[:P.shape[1]]
    return out


def _rows_of(rows, B, T):
    if rows is None:
        return np.arange(B * T, dtype=np.int64)
    return np.asarray(rows, dtype=np.int64)


def _project_kv(X, Wk, Wv, B, T, G, dh):
    K = (X @ _f64(Wk)).reshape(B, T, G, dh)
    V = (X @ _f64(Wv)).reshape(B, T, G, dh)
    return K, V


def _project_q_selected(Xr, Wq, sel, dims) -> np.ndarray:
    """Query rows of the selected experts only ([GS] "query-side sparsity";
    [AT] section 4: every expert has its own query projection), plus the
    shared head: Q[r, g*k + j] = x_r Wq[:, head g*M + sel[r, g, j]],
    Q[r, G*k] = x_r Wq[:, shared]."""
    G, M, k, dh = dims.G, dims.M, dims.k, dims.dh
    WQ = _f64(Wq)
    nr = Xr.shape[0]
    Q = np.zeros((nr, G * k + 1, dh))
    for g in range(G):
        for j in range(k):
            e_col = sel[:, g, j]
            for e in range(M):
                m = e_col == e
                if not m.any():
                    continue
                h = g * M + e
                Q[m, g * k + j] = Xr[m] @ WQ[:, h * dh:(h + 1) * dh]
    Q[:, G * k] = Xr @ WQ[:, G * M * dh:(G * M + 1) * dh]
    return Q


def attend_selected(Q, rows, K, V, dims) -> np.ndarray:
    """Attention step of the GQE layer for query rows ``rows`` (flat n).

    Q [len(rows), G*k+1, dh]: slot g*k+j is the j-th selected expert of group
    g, slot G*k the shared head. Each routed slot attends its group's K/V; the
    shared head attends KV head 0 ([AT] section 4; KV head 0 is this
    library's reading). K, V: [B, T, G, dh]."""
    B, T, G, k, dh = dims.B, dims.T, dims.G, dims.k, dims.dh
    rows = np.asarray(rows, dtype=np.int64)
    Q = np.asarray(Q, F64)
    K = np.asarray(K, F64).reshape(B, T, G, dh)
    V = np.asarray(V, F64).reshape(B, T, G, dh)
    scale = 1.0 / math.sqrt(dh)
    bidx, tpos = rows // T, rows % T
    O = np.zeros(Q.shape)
    for b in range(B):
        mb = bidx == b
        if not mb.any():
            continue
        for g in range(G):
            for j in range(k):
                O[mb, g * k + j] = causal_attention(Q[mb, g * k + j], tpos[mb], K[b, :, g], V[b, :, g], scale)
        O[mb, G * k] = causal_attention(Q[mb, G * k], tpos[mb], K[b, :, 0], V[b, :, 0], scale)
    return O


def combine(O, w, dims) -> np.ndarray:
    """Output construction ([GS] "Architecture and routing", output
    construction; [AT] section 4, merge of the three parts):
    A = [hard concat of the selected outputs (g-major, ascending expert)
         | per-group slot sum_j w[g,j] O[g,j] | shared head]."""
    G, k, dh = dims.G, dims.k, dims.dh
    O = np.asarray(O, F64)
    w = np.asarray(w, F64)
    nr = O.shape[0]
    concat = O[:, :G * k].reshape(nr, G * k * dh)
    slot = np.einsum("ngj,ngjd->ngd", w, O[:, :G * k].reshape(nr, G, k, dh)).reshape(nr, G * dh)
    return np.concatenate([concat, slot, O[:, G * k]], axis=1)


VARIANTS = ("hard", "weighted", "global_slot", "no_shared")


def combine_width(dims, mode: str = "slot") -> int:
    """Columns of A (= rows of Wo) for an output construction."""
    G, k, dh = dims.G, dims.k, dims.dh
    blocks = {"slot": G * k + G + 1, "hard": G * k + 1, "weighted": G * k + 1,
              "global_slot": G * k + 2, "no_shared": G * k + G}
    if mode not in blocks:
        raise ValueError(mode)
    return blocks[mode] * dh


def combine_variant(O, w, p_sel, dims, mode: str) -> np.ndarray:
    """Output construction of the variants of step 5.

    [AT] section 6 (ablation): a pure hard concatenation, and a concatenation
    weighted directly by the router's scores without the renormalised slot.
    [GS] "Experimental results" words the ablation as removing the renormalised slot or
    the shared head. [AT] section 4 can be read as ONE extra output, the
    weighted average of all selected experts' outputs by their router scores.
    Readings: the scores are the in-group softmax probabilities of the
    selected experts (p_sel); the variants keep every part that they do not
    name as removed.
      "hard":        A = [concat | shared]
      "weighted":    A = [p_sel[g, j] * O[g, j] (concat) | shared]
      "global_slot": A = [concat | sum_{g,j} p_sel[g,j] O[g,j] / sum_{g,j} p_sel[g,j] | shared]
      "no_shared":   A = [concat | per-group slot sum_j w[g,j] O[g,j]]"""
    G, k, dh = dims.G, dims.k, dims.dh
    O = np.asarray(O, F64)
    nr = O.shape[0]
    routed = O[:, :G * k]                       # [nr, G*k, dh], g-major, ascending expert
    shared = O[:, G * k]
    concat = routed.reshape(nr, G * k * dh)
    if mode == "hard":
        return np.concatenate([concat, shared], axis=1)
    if mode == "weighted":
        p = np.asarray(p_sel, F64).reshape(nr, G * k)
        return np.concatenate([(routed * p[:, :, None]).reshape(nr, G * k * dh), shared], axis=1)
    if mode == "global_slot":
        p = np.asarray(p_sel, F64).reshape(nr, G * k)
        avg = np.einsum("nh,nhd->nd", p, routed) / p.sum(axis=1, keepdims=True)
        return np.concatenate([concat, avg, shared], axis=1)
    if mode == "no_shared":
        slot = np.einsum("ngj,ngjd->ngd", np.asarray(w, F64), routed.reshape(nr, G, k, dh)).reshape(nr, G * dh)
        return np.concatenate([concat, slot], axis=1)
    raise ValueError(mode)


# ---------------------------------------------------------------------------
# GQE layer forward: [GS] "Architecture and routing", [AT] section 4.
# ---------------------------------------------------------------------------
def gqe_forward(x, Wq, Wk, Wv, Wr, br, Wo, dims, rows=None, forced_sel=None, combine_mode: str = "slot") -> dict:
    """The whole layer for the query tokens ``rows`` (flat n = b*T + t).

    Steps, in the pages' order:
      1. router: logits, in-group softmax, top-k, renormalised weights;
      2. dense K/V projection of every token (K/V stay dense);
      3. query projection for the selected experts (+ the shared head);
      4. each selected expert attends causally to its group's K/V; the
         shared head attends KV head 0;
      5. A = [hard concat of selected outputs | per-group weighted slot |
         shared head];  6. y = A Wo.
    Returns the intermediate values too (all float64, rows in ``rows`` order).
    ``forced_sel`` ([len(rows), G, k]) overrides the router's choice.
    ``combine_mode`` (one of ``VARIANTS``) selects a variant of step 5
    (``combine_variant``; Wo then has ``combine_width(dims, mode)`` rows).
    """
    B, T, D, G, M, k, dh = dims.B, dims.T, dims.D, dims.G, dims.M, dims.k, dims.dh
    X = _f64(x).reshape(B * T, D)
    rows = _rows_of(rows, B, T)
    R = route(X[rows], Wr, br, G, M, k, forced_sel=forced_sel)
    sel, w = R["sel"], R["w"]

    K, V = _project_kv(X, Wk, Wv, B, T, G, dh)
    Q = _project_q_selected(X[rows], Wq, sel, dims)

    O = attend_selected(Q, rows, K, V, dims)
    p_sel = np.take_along_axis(R["p"], sel, axis=2)
    A = combine(O, w, dims) if combine_mode == "slot" else combine_variant(O, w, p_sel, dims, combine_mode)
    y = A @ _f64(Wo)
    return {"rows": rows, "sel": sel, "w": w, "p_sel": p_sel, "margin": R["margin"], "logits": R["logits"],
            "p": R["p"], "K": K, "V": V, "Q": Q, "O": O, "A": A, "y": y}


# ---------------------------------------------------------------------------
# One generation step with a key/value cache. [WK], "from the inference
# angle": a decoder caches the key/value heads and reads them back at every
# step, which is where sharing K/V heads pays. Reading (the pages describe no
# decode procedure): the new token of sequence b sits at position L_b =
# cache_len[b]; its K/V row is appended there and each of its query rows
# attends positions 0..L_b; routing, projections and the output construction
# are those of the layer above applied to that one token.
# ---------------------------------------------------------------------------
def gqe_decode(x_new, Wq, Wk, Wv, Wr, br, Wo, K_cache, V_cache, cache_len, dims, forced_sel=None) -> dict:
    """x_new [B, D]: the token at position cache_len[b] of sequence b.
    K_cache, V_cache [B, Tmax, G, dh]: rows < cache_len[b] of sequence b are
    its keys/values; the rest is ignored. Returns y [B, D], the new token's
    K/V rows K_new, V_new [B, G, dh] (the rows the step appends), and the
    routing and intermediate values (float64)."""
    B, D, G, M, k, dh = dims.B, dims.D, dims.G, dims.M, dims.k, dims.dh
    X = _f64(x_new).reshape(B, D)
    lens = np.asarray(cache_len, dtype=np.int64).reshape(B)
    R = route(X, Wr, br, G, M, k, forced_sel=forced_sel)
    sel, w = R["sel"], R["w"]
    K_new = (X @ _f64(Wk)).reshape(B, G, dh)
    V_new = (X @ _f64(Wv)).reshape(B, G, dh)
    Q = _project_q_selected(X, Wq, sel, dims)
    Kc = _f64(K_cache).reshape(B, -1, G, dh)
    Vc = _f64(V_cache).reshape(B, -1, G, dh)
    scale = 1.0 / math.sqrt(dh)
    O = np.zeros(Q.shape)
    for b in range(B):
        L = int(lens[b])
        for g in range(G):
            Kb = np.concatenate([Kc[b, :L, g], K_new[b, g][None]], axis=0)
            Vb = np.concatenate([Vc[b, :L, g], V_new[b, g][None]], axis=0)
            pos = np.full(k, L)
            O[b, g * k:(g + 1) * k] = causal_attention(Q[b, g * k:(g + 1) * k], pos, Kb, Vb, scale)
        Kb = np.concatenate([Kc[b, :L, 0], K_new[b, 0][None]], axis=0)
        Vb = np.concatenate([Vc[b, :L, 0], V_new[b, 0][None]], axis=0)
        O[b, G * k] = causal_attention(Q[b, G * k][None], np.array([L]), Kb, Vb, scale)[0]
    A = combine(O, w, dims)
    y = A @ _f64(Wo)
    return {"sel": sel, "w": w, "margin": R["margin"], "K_new": K_new, "V_new": V_new, "Q": Q, "O": O, "A": A, "y": y}


def gqa_dense_forward(x, Wq, Wk, Wv, Wo_dense, dims, rows=None) -> dict:
    """All G*M query heads active (the GQA baseline of [GS] "Experimental
    results", 16 query heads over 8 KV groups); head h attends KV group h // M
    ([WK]); y = concat_h O_h Wo_dense."""
    B, T, D, G, M, dh = dims.B, dims.T, dims.D, dims.G, dims.M, dims.dh
    X = _f64(x).reshape(B * T, D)
    rows = _rows_of(rows, B, T)
    scale = 1.0 / math.sqrt(dh)
    K, V = _project_kv(X, Wk, Wv, B, T, G, dh)
    WQ = _f64(Wq)[:, :G * M * dh]
    Xr = X[rows]
    bidx, tpos = rows // T, rows % T
    nr = len(rows)
    H = G * M
    Q = (Xr @ WQ).reshape(nr, H, dh)
    O = np.zeros((nr, H, dh))
    for b in range(B):
        mb = bidx == b
        if not mb.any():
            continue
        for h in range(H):
            g = h // M
            O[mb, h] = causal_attention(Q[mb, h], tpos[mb], K[b, :, g], V[b, :, g], scale)
    y = O.reshape(nr, H * dh) @ _f64(Wo_dense)
    return {"rows": rows, "K": K, "V": V, "Q": Q, "O": O, "y": y}


def sample_rows(B: int, T: int, n_uniform: int, seed: int, n_last: int = 64, n_first: int = 16) -> np.ndarray:
    """Query positions for sampled parity at sizes the full oracle cannot
    finish: the first and last positions of every sequence plus uniform
    draws (flat n = b*T + t, sorted, unique)."""
    rng = np.random.default_rng(seed)
    picks = []
    for b in range(B):
        picks.append(b * T + np.arange(min(n_first, T)))
        picks.append(b * T + np.arange(max(0, T - n_last), T))
    picks.append(rng.integers(0, B * T, size=n_uniform))
    return np.unique(np.concatenate(picks))
