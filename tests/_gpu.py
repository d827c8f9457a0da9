"""Helpers of the GPU parity tests: run the CUDA path stage by stage through the
C ABI, and compare with the fp64 oracle on the same seeded inputs."""
import numpy as np
import torch

import moe_gqa_query_gqe_b200 as gqe
import oracle.gqe_ref as ref

NEAR_TIE = 1e-4          # top-k margin (logit units) under which either choice is accepted
REL_L2_MAX = 5e-3        # bf16 output tolerances against the oracle
MAX_ABS_MAX = 1e-2

# Per parity case: decisions checked, near ties, near ties decided the other
# way, and the worst rel-L2 / max-abs of any bf16 tensor compared. Printed at
# the end of the run (tests/conftest.py) so the counts reach the run's log.
REPORT: dict = {}


def _report(case, **kw):
    if case is None:
        return
    r = REPORT.setdefault(case, {"decisions": 0, "near_ties": 0, "flipped": 0, "rel_l2": 0.0, "max_abs": 0.0,
                                 "worst": ""})
    for key in ("decisions", "near_ties", "flipped"):
        r[key] += kw.get(key, 0)
    if "rel_l2" in kw and kw["rel_l2"] >= r["rel_l2"]:
        r["rel_l2"], r["worst"] = kw["rel_l2"], kw.get("what", "")
    r["max_abs"] = max(r["max_abs"], kw.get("max_abs", 0.0))


def to_dev(inp: dict) -> dict:
    return {k: v.cuda() for k, v in inp.items()}


def run_stages(d, dev: dict) -> dict:
    """route -> qproj -> attn -> combine, each through its own C-ABI entry."""
    N, G, M, k = d.B * d.T, d.G, d.M, d.k
    Ha = G * k + 1
    i32, f32, bf = torch.int32, torch.float32, torch.bfloat16
    o = {
        "sel": torch.full((N, G, k), -1, dtype=i32, device="cuda"),
        "w": torch.full((N, G, k), float("nan"), dtype=f32, device="cuda"),
        "margin": torch.full((N, G), float("nan"), dtype=f32, device="cuda"),
        "seg_off": torch.full((d.B * G * M + 1,), -1, dtype=i32, device="cuda"),
        "seg_tok": torch.full((N * G * k,), -1, dtype=i32, device="cuda"),
        "row_map": torch.full((N, G, k), -1, dtype=i32, device="cuda"),
        "Q": torch.full((N, Ha, 64), float("nan"), dtype=bf, device="cuda"),
        "K": torch.full((N, G, 64), float("nan"), dtype=bf, device="cuda"),
        "V": torch.full((N, G, 64), float("nan"), dtype=bf, device="cuda"),
        "O": torch.full((N, Ha, 64), float("nan"), dtype=bf, device="cuda"),
        "y": torch.full((N, d.D), float("nan"), dtype=bf, device="cuda"),
    }
    ws_r = gqe.workspace(d, gqe.OP_ROUTE)
    gqe.gqe_route(d, dev["x"], dev["Wr"], dev["br"], o["sel"], o["w"], o["margin"], o["seg_off"],
                  o["seg_tok"], o["row_map"], ws_r)
    gqe.gqe_qproj(d, dev["x"], dev["Wq"], dev["Wk"], dev["Wv"], o["sel"], o["seg_off"], o["seg_tok"],
                  o["Q"], o["K"], o["V"])
    gqe.gqe_attn(d, o["Q"], o["K"], o["V"], o["O"])
    ws_c = gqe.workspace(d, gqe.OP_COMBINE)
    gqe.gqe_combine(d, o["O"], o["w"], dev["Wo"], o["y"], ws_c)
    o["status"] = gqe.gqe_check_error()
    return {k: (v.cpu() if torch.is_tensor(v) else v) for k, v in o.items()}


def run_forward(d, dev: dict):
    ws = gqe.workspace(d, gqe.OP_FORWARD)
    y = torch.full((d.B * d.T, d.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    gqe.gqe_forward(d, dev["x"], dev["Wq"], dev["Wk"], dev["Wv"], dev["Wr"], dev["br"], dev["Wo"], y, ws)
    status = gqe.gqe_check_error()
    return y, ws, status


def run_dense(d, dev: dict):
    ws = gqe.workspace(d, gqe.OP_DENSE)
    y = torch.full((d.B * d.T, d.D), float("nan"), dtype=torch.bfloat16, device="cuda")
    gqe.gqa_dense_forward(d, dev["x"], dev["Wq"], dev["Wk"], dev["Wv"], dev["Wo_dense"], y, ws)
    status = gqe.gqe_check_error()
    return y, ws, status


def f64(t) -> np.ndarray:
    return t.detach().cpu().double().numpy() if torch.is_tensor(t) else np.asarray(t, dtype=np.float64)


def errors(got, want) -> dict:
    got, want = f64(got), np.asarray(want, dtype=np.float64)
    diff = got - want
    nrm = np.linalg.norm(want)
    return {"rel_l2": float(np.linalg.norm(diff) / nrm) if nrm > 0 else float(np.linalg.norm(diff)),
            "max_abs": float(np.abs(diff).max()) if diff.size else 0.0,
            "finite": bool(np.isfinite(got).all())}


def assert_close_bf16(got, want, what: str, rel_l2=REL_L2_MAX, max_abs=MAX_ABS_MAX, case=None) -> dict:
    e = errors(got, want)
    _report(case, rel_l2=e["rel_l2"], max_abs=e["max_abs"], what=what)
    assert e["finite"], f"{what}: non-finite values"
    assert e["rel_l2"] <= rel_l2, f"{what}: rel-L2 {e['rel_l2']:.3e} > {rel_l2:.1e}"
    assert e["max_abs"] <= max_abs, f"{what}: max-abs {e['max_abs']:.3e} > {max_abs:.1e}"
    return e


def check_selection(d, x, Wr, br, gpu_sel, rows=None, case=None) -> dict:
    """Selections must equal the oracle's except on near-tie decisions
    (oracle margin < NEAR_TIE), which are accepted either way and reported."""
    x = x.cpu()
    xr = x if rows is None else x[torch.as_tensor(rows)]
    r = ref.route(xr, Wr.cpu(), br.cpu(), d.G, d.M, d.k)
    g = gpu_sel.numpy().astype(np.int64)
    if rows is not None:
        g = g[rows]
    differ = np.any(g != r["sel"], axis=2)
    near = r["margin"] < NEAR_TIE
    bad = differ & ~near
    _report(case, decisions=int(differ.size), near_ties=int(near.sum()), flipped=int((differ & near).sum()))
    assert not bad.any(), f"{int(bad.sum())} selections differ with margin >= {NEAR_TIE}"
    return {"near_ties": int(near.sum()), "flipped_near_ties": int((differ & near).sum()), "oracle": r}


def reference_attention(d, Q, K, V, rows) -> np.ndarray:
    """The oracle's attention step applied to the GPU's own bf16 Q/K/V."""
    rows = np.asarray(rows)
    return ref.attend_selected(f64(Q)[rows], rows, f64(K).reshape(d.B, d.T, d.G, 64),
                               f64(V).reshape(d.B, d.T, d.G, 64), d)
