"""Throughput of the GQE attention-layer forward pass on B200.

One step = one full forward pass of the layer (route -> selected-expert and
K/V projections -> routed causal attention -> combine + output projection)
over one batch of the main workload (8 sequences x 2048 tokens, d_model 1024,
8 KV groups x 2 experts, k = 1, shared head, head dim 64), inputs resident in
HBM. Prints one JSON line.

  python bench.py [--gpus N --steps K --warmup W] [--workload NAME] [--impl reference]

Timing: CUDA events on the launching stream around every step, an L2 flush
(256 MiB write) between steps outside the events, max over ranks. With N > 1
every rank runs its own batch (weak scaling, no data-path collective).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GQE fwd tokens/s, TFLOP/s % BF16 peak, speedup vs dense GQA at 2K–1M tokens"
DEFAULT_WORKLOAD = "main_b8_t2048"


def flops_model(d) -> dict:
    """Algorithmic flops of one forward pass (what the method must compute;
    masked halves of diagonal tiles are not counted)."""
    N = d.B * d.T
    Ha = d.G * d.k + 1
    causal_pairs = d.B * d.T * (d.T + 1) // 2           # sum over rows of (t + 1), per row set
    f = {
        "router": 2 * N * d.D * d.G * d.M,
        "q_proj": 2 * N * d.D * d.dh * Ha,
        "kv_proj": 2 * N * d.D * 2 * d.G * d.dh,
        "attention": 4 * d.dh * Ha * causal_pairs,
        "wo": 2 * N * (d.G * d.k + d.G + 1) * d.dh * d.D,
    }
    dense = {
        "qkv_proj": 2 * N * d.D * (d.G * d.M + 2 * d.G) * d.dh,
        "attention": 4 * d.dh * d.G * d.M * causal_pairs,
        "wo": 2 * N * d.G * d.M * d.dh * d.D,
    }
    return {"gqe": f, "gqe_total": sum(f.values()), "dense": dense, "dense_total": sum(dense.values())}


def stage_rooflines(d, stage_ms: dict, peaks: dict) -> dict:
    """Roofline of each of the four stage calls. Routing is bound by HBM: it
    reads x and writes the decisions, their weights, margins, token lists and
    row map (algorithmic bytes). The other three stages are tensor-bound:
    their algorithmic flops over the stage time, against the bf16 peak."""
    N = d.B * d.T
    fl = flops_model(d)["gqe"]
    route_bytes = 2 * N * d.D + 2 * d.D * d.G * d.M + 4 * N * d.G * d.k * 4 + 4 * N * d.G + 4 * (d.B * d.G * d.M + 1)
    out = {"route": {"bound": "hbm", "unit": "GB/s", "algorithmic": route_bytes,
                     "achieved": route_bytes / (stage_ms["route"] / 1e3) / 1e9, "peak": peaks["hbm_gbs"]}}
    for name, flops in (("qproj", fl["q_proj"] + fl["kv_proj"]), ("attention", fl["attention"]), ("combine", fl["wo"])):
        out[name] = {"bound": "tensor", "unit": "TFLOP/s", "algorithmic": flops,
                     "achieved": flops / (stage_ms[name] / 1e3) / 1e12, "peak": peaks["bf16_tflops"]}
    for v in out.values():
        v["frac"] = v["achieved"] / v["peak"]
    return out


def load_peaks() -> dict:
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def kernel_source_hash(name: str) -> str:
    with open(os.path.join(ROOT, "moe_gqa_query_gqe_b200", "csrc", name), "rb") as fh:
        return hashlib.sha256(fh.read()).hexdigest()[:16]


def recorded_traffic(workload: str, src: str) -> float | None:
    """DRAM bytes per launch of the kernel in csrc/<src>, from the committed
    ncu summary profiles/traffic_<kernel source>_<workload>.md, but only if
    that capture was taken on the current kernel source (its
    `source_sha256_16:` line matches)."""
    path = os.path.join(ROOT, "profiles", f"traffic_{src.split('.')[0]}_{workload}.md")
    try:
        fields = {}
        with open(path) as fh:
            for line in fh:
                if ":" in line and not line.startswith("#"):
                    key, val = line.split(":", 1)
                    fields[key.strip("-* `")] = val.strip().strip("`")
        if fields.get("source_sha256_16") == kernel_source_hash(src):
            return float(fields["bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(gpu_index)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def wait_first(self, timeout=3.0):
        t0 = time.time()
        while self.proc and not self.samples and time.time() - t0 < timeout:
            time.sleep(0.05)

    def stop(self, t_begin, t_end) -> dict:
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=2)
            except Exception:
                self.proc.kill()
        window = [s for (t, s) in self.samples if t_begin - 0.2 <= t <= t_end + 0.2]
        scope = "timed"
        if not window:
            window = [s for (_, s) in self.samples]
            scope = "run"
        if not window:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no-samples"], "samples": 0}
        sm = [float(s[1]) for s in window if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in window for i in range(4) if s[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": float(window[0][2]) if window[0][2].replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(window), "scope": scope}


def reduce_max(values, world: int, device) -> list:
    """Element-wise max over ranks (timings: the slowest rank sets the job's
    time). Works on any process group backend; identity for one rank."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Whole-job tokens/s: every rank processes its own batch (weak scaling)."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(d, budget_s: float, max_steps: int | None = None):
    """Time the fp64 oracle on whole sequences of the workload (one sequence
    per sample, all its rows), until ``budget_s`` of CPU work or ``max_steps``."""
    import oracle.gqe_ref as ref
    from gqe_inputs import make_inputs
    d1 = d.with_(B=1)
    inp = make_inputs(d1, seed=0)
    times = []
    t_all = time.time()
    while True:
        t0 = time.perf_counter()
        ref.gqe_forward(inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], d1)
        times.append(time.perf_counter() - t0)
        if max_steps is not None and len(times) >= max_steps:
            break
        if max_steps is None and time.time() - t_all >= budget_s:
            break
    return d1.T, times


NEAR_TIE = 1e-4  # top-k margin (logit units) under which either choice is accepted


def oracle_leg(d, inp: dict, sel_gpu, y_gpu, budget_s: float, extra_routes=()) -> tuple[dict, dict]:
    """The CPU-baseline leg: the fp64 oracle, as it stands, timed on whole
    sequences of the timed run's own batch (sequence i of the batch at sample
    i, cycling), on the host cores, for about ``budget_s`` seconds.

    The same oracle outputs also score the timed run: per sequence, the GPU's
    expert selections against the oracle's (bit-exact, except near-tie
    decisions whose margin is below 1e-4, which are counted and accepted) and
    the GPU's y against the oracle's y (rel-L2 and max-abs; the oracle is
    rerun, untimed, with the GPU's selections where a near tie flipped).
    ``extra_routes`` are (name, dims, x, Wr, br, sel_gpu) of other workloads
    whose selections are scored the same way (routing only)."""
    import numpy as np
    import oracle.gqe_ref as ref
    d1 = d.with_(B=1)
    w = {kk: v.cpu() for kk, v in inp.items() if kk != "x"}
    x_all = inp["x"]
    sel_all = sel_gpu.cpu().numpy().astype(np.int64)
    y_all = y_gpu.cpu().double().numpy()
    times, checked = [], {}
    worst = {"rel_l2": 0.0, "max_abs": 0.0}
    ties = {"decisions": 0, "near_ties": 0, "flipped_near_ties": 0, "mismatches_beyond_tie": 0}
    t_all = time.time()
    i = 0
    while True:
        b = i % d.B
        xs = x_all[b * d.T:(b + 1) * d.T].cpu()
        t0 = time.perf_counter()
        out = ref.gqe_forward(xs, w["Wq"], w["Wk"], w["Wv"], w["Wr"], w["br"], w["Wo"], d1)
        times.append(time.perf_counter() - t0)
        if b not in checked:
            sg = sel_all[b * d.T:(b + 1) * d.T]
            r = ref.route(xs, w["Wr"], w["br"], d.G, d.M, d.k)
            differ = np.any(sg != r["sel"], axis=2)
            near = r["margin"] < NEAR_TIE
            ties["decisions"] += differ.size
            ties["near_ties"] += int(near.sum())
            ties["flipped_near_ties"] += int((differ & near).sum())
            ties["mismatches_beyond_tie"] += int((differ & ~near).sum())
            want = out["y"]
            if differ.any():
                want = ref.gqe_forward(xs, w["Wq"], w["Wk"], w["Wv"], w["Wr"], w["br"], w["Wo"], d1,
                                       forced_sel=sg)["y"]
            diff = y_all[b * d.T:(b + 1) * d.T] - want
            worst["rel_l2"] = max(worst["rel_l2"], float(np.linalg.norm(diff) / np.linalg.norm(want)))
            worst["max_abs"] = max(worst["max_abs"], float(np.abs(diff).max()))
            checked[b] = True
        i += 1
        if time.time() - t_all >= budget_s and i >= 1:
            break
    sec = sum(times) / len(times)
    cpu = {"value": d.T / sec, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
           "sample": f"{len(times)} x one full sequence ({d.T} tokens, all rows) of the timed batch, fp64"}
    parity = {"sequences_checked": len(checked), "of_sequences": d.B, "rows": len(checked) * d.T,
              "worst_rel_l2": worst["rel_l2"], "worst_max_abs": worst["max_abs"],
              "bars": {"rel_l2": 5e-3, "max_abs": 1e-2, "near_tie_margin": NEAR_TIE}, **ties}
    for name, dx, x, Wr, br, sg in extra_routes:
        r = ref.route(x.cpu(), Wr.cpu(), br.cpu(), dx.G, dx.M, dx.k)
        sg = sg.cpu().numpy().astype(np.int64)
        differ = np.any(sg != r["sel"], axis=2)
        near = r["margin"] < NEAR_TIE
        parity[name] = {"decisions": int(differ.size), "near_ties": int(near.sum()),
                        "flipped_near_ties": int((differ & near).sum()),
                        "mismatches_beyond_tie": int((differ & ~near).sum())}
    return cpu, parity


def run_reference(args, d, rank, world):
    """The oracle arm: the fp64 CPU oracle as it stands, on host cores."""
    if rank != 0:
        return
    tokens, times = oracle_sample(d, 0, max_steps=args.warmup + args.steps)
    timed = times[args.warmup:] or times
    sec = sum(timed) / len(timed)
    value = tokens / sec
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, **{k: getattr(d, k) for k in ("B", "T", "D", "G", "M", "k", "dh")},
                       "l2": "n/a (host)"},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": host_cores(), "kind": "oracle",
                             "sample": f"one sequence ({tokens} tokens, all rows) of the workload per step"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def pool_study(steps: int, warmup: int) -> None:
    """Expert-pool study: the layer at 32K tokens (D 1024, G 8) for pools of
    M = 2, 4 and 8 experts per group with k selected, under near-balanced
    routing and under the +2 bias on expert 0. Per configuration: one JSON
    line with the GQE and dense step times (CUDA-graph replays, L2 flushed),
    the speedup, the algorithmic flop ratio, and how unevenly the tokens
    spread over the experts (largest and smallest segment over the mean)."""
    import torch
    import moe_gqa_query_gqe_b200 as gqe
    from gqe_inputs import Dims, make_inputs

    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")

    def graph(fn):
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                fn()
        torch.cuda.synchronize()
        return g

    def timed(g):
        for _ in range(warmup):
            flush.fill_(1)
            g.replay()
        evs = []
        for _ in range(steps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in evs) / steps

    for (M, k) in [(2, 1), (4, 1), (4, 2), (8, 1), (8, 2), (8, 4)]:
        for bias0 in (0.0, 2.0):
            d = Dims(B=1, T=32768, D=1024, G=8, M=M, k=k, bias0=bias0)
            inp = make_inputs(d, seed=0, device="cuda")
            N = d.B * d.T
            ws, wd = gqe.workspace(d, gqe.OP_FORWARD), gqe.workspace(d, gqe.OP_DENSE)
            y = torch.empty(N, d.D, dtype=torch.bfloat16, device="cuda")
            y2 = torch.empty_like(y)
            g1 = graph(lambda: gqe.gqe_forward(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"],
                                               inp["Wo"], y, ws))
            g2 = graph(lambda: gqe.gqa_dense_forward(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wo_dense"],
                                                     y2, wd))
            t_gqe, t_dense = timed(g1), timed(g2)
            status = gqe.gqe_check_error()
            # tokens per (sequence, group, expert) from the decisions (the
            # forward builds segment lists only on its gather path)
            sel = gqe.forward_views(d, ws)["sel"].long() & 0xFF                   # [N, G, k]
            gidx = torch.arange(d.G, device=sel.device).view(1, d.G, 1) * M
            bidx = (torch.arange(N, device=sel.device) // d.T).view(N, 1, 1) * (d.G * M)
            seg = torch.bincount((sel + gidx + bidx).flatten(), minlength=d.B * d.G * M).double()
            mean = N * k / M
            fl = flops_model(d)
            print(json.dumps({"study": "expert_pool", "M": M, "k": k, "bias0": bias0, "T": d.T, "G": d.G,
                              "gqe_ms": t_gqe, "dense_ms": t_dense, "speedup": t_dense / t_gqe,
                              "flop_ratio": fl["dense_total"] / fl["gqe_total"],
                              "segment_max_over_mean": float(seg.max() / mean),
                              "segment_min_over_mean": float(seg.min() / mean), "status": status}), flush=True)
            del g1, g2


def decode_study(steps: int, warmup: int, cases: str = "") -> None:
    """Decode step (gqe_decode): one new token per sequence against caches of
    L positions, for the main layer's shape (D 1024, G 8, M 2, k 1). Per
    configuration: one JSON line with the step time (CUDA-graph replays, L2
    flushed between them), tokens/s, the bytes the step must read (the K/V
    cache rows up to each new token, plus the weights) and that rate as a
    fraction of the measured HBM bandwidth. `cases` ("8x32767,1x131071")
    picks configurations by B x L; empty: all three."""
    import torch
    import moe_gqa_query_gqe_b200 as gqe
    from gqe_inputs import Dims, make_decode_inputs

    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    peaks = load_peaks()
    todo = [(8, 32767), (64, 4095), (1, 131071)]
    if cases:
        todo = [tuple(int(v) for v in c.split("x")) for c in cases.split(",")]
    for (B, L) in todo:
        d = Dims(B=B, T=L + 1, D=1024, G=8, M=2, k=1)
        inp = {kk: v.cuda() for kk, v in make_decode_inputs(d, [L] * B, seed=0, device="cpu").items()}
        y = torch.empty(B, d.D, dtype=torch.bfloat16, device="cuda")
        sel = torch.empty(B, d.G, d.k, dtype=torch.int32, device="cuda")
        w = torch.empty(B, d.G, d.k, dtype=torch.float32, device="cuda")
        ws = gqe.workspace(d, gqe.OP_DECODE)

        def step():
            gqe.gqe_decode(d, inp["cache_len"], inp["x_new"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"],
                           inp["Wo"], inp["K_cache"], inp["V_cache"], y, sel, w, ws)

        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            step()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                step()
        torch.cuda.synchronize()
        evs = []
        for i in range(warmup + steps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            if i >= warmup:
                evs.append((a, b))
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / steps
        cache_bytes = B * (L + 1) * d.G * 64 * 2 * 2
        weight_bytes = sum(inp[kk].numel() * inp[kk].element_size() for kk in ("Wq", "Wk", "Wv", "Wr", "Wo"))
        gbs = (cache_bytes + weight_bytes) / (ms / 1e3) / 1e9
        print(json.dumps({"study": "decode", "B": B, "L": L, "D": d.D, "G": d.G, "M": d.M, "k": d.k,
                          "us_per_step": ms * 1e3, "tokens_per_s": B / (ms / 1e3),
                          "bytes_per_step": cache_bytes + weight_bytes, "achieved_gbs": gbs,
                          "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
                          "status": gqe.gqe_check_error()}), flush=True)
        del g


def long_context(names, steps: int, warmup: int, seed: int, peaks: dict, flush) -> tuple[dict, list]:
    """The layer at long context: per workload, the GQE forward and the same
    library's dense GQA forward as CUDA-graph replays (L2 flushed before each,
    CUDA events on the launching stream), the routed attention alone (its
    C-ABI call on the forward's own Q/K/V), and the GPU's routing decisions
    for scoring against the oracle. The million-token workload takes one
    warm-up and two timed steps per arm (about 2 and 3 s a step)."""
    import torch
    import moe_gqa_query_gqe_b200 as gqe
    from gqe_inputs import CONFIGS, make_inputs
    out, routes = {}, []
    stream = torch.cuda.current_stream()
    for name in names:
        d = CONFIGS[name]
        big = d.B * d.T > (1 << 18)
        n_steps, n_warm = (2, 1) if big else (max(3, min(steps, 10)), max(3, warmup))
        inp = make_inputs(d, seed=seed, device="cuda")
        N = d.B * d.T
        ws, wd = gqe.workspace(d, gqe.OP_FORWARD), gqe.workspace(d, gqe.OP_DENSE)
        y = torch.empty(N, d.D, dtype=torch.bfloat16, device="cuda")
        yd = torch.empty_like(y)

        def graph(fn):
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            with torch.cuda.stream(side):
                fn()
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                fn()
            torch.cuda.synchronize()
            return g

        def timed(fn, n, w):
            evs = []
            for i in range(w + n):
                flush.fill_(1)
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                fn()
                b.record(stream)
                if i >= w:
                    evs.append((a, b))
            torch.cuda.synchronize()
            return sum(a.elapsed_time(b) for a, b in evs) / n

        g1 = graph(lambda: gqe.gqe_forward(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"],
                                           inp["Wo"], y, ws))
        t_gqe = timed(g1.replay, n_steps, n_warm)
        st1 = gqe.gqe_check_error()
        del g1
        v = gqe.forward_views(d, ws)
        t_attn = timed(lambda: gqe.gqe_attn(d, v["Q"], v["K"], v["V"], v["O"]), n_steps, 1)
        st2 = gqe.gqe_check_error()
        g2 = graph(lambda: gqe.gqa_dense_forward(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wo_dense"],
                                                 yd, wd))
        t_dense = timed(g2.replay, n_steps, n_warm)
        st3 = gqe.gqe_check_error()
        del g2
        fl = flops_model(d)
        attn_tf = fl["gqe"]["attention"] / (t_attn / 1e3) / 1e12
        margin = v["margin"]
        out[name] = {"T": d.T, "B": d.B, "steps": n_steps, "warmup": n_warm, "ms_per_step": t_gqe,
                     "tokens_per_s": N / (t_gqe / 1e3), "dense_ms": t_dense, "speedup_vs_dense": t_dense / t_gqe,
                     "flop_ratio": fl["dense_total"] / fl["gqe_total"],
                     "tflops": fl["gqe_total"] / (t_gqe / 1e3) / 1e12,
                     "attention_ms": t_attn, "attention_tflops": attn_tf,
                     "attention_frac": attn_tf / peaks["bf16_tflops"],
                     "attention_frac_sustained": attn_tf / peaks["bf16_tflops_sustained"],
                     "gpu_margin_below_1e-4": int((margin < NEAR_TIE).sum().item()),
                     "status": [st1, st2, st3]}
        routes.append((name, d, inp["x"].cpu(), inp["Wr"].cpu(), inp["br"].cpu(), v["sel"].cpu()))
        del inp, ws, wd, y, yd, v, margin
        torch.cuda.empty_cache()
    return out, routes


def stage_study(workload: str, steps: int, warmup: int) -> None:
    """Each stage entry point of the layer (route, qproj, attn, combine) on one
    workload, called alone: one JSON line per stage with its CUDA-event time
    (L2 flushed before each call) and its roofline (routing and the k > 1
    combine against HBM bandwidth with their algorithmic bytes; the
    projections, attention and Wo against the bf16 peak)."""
    import torch
    import moe_gqa_query_gqe_b200 as gqe
    from gqe_inputs import CONFIGS, make_inputs

    d = CONFIGS[workload]
    inp = make_inputs(d, seed=0, device="cuda")
    N, G, M, k = d.B * d.T, d.G, d.M, d.k
    Ha = G * k + 1
    sel = torch.empty(N, G, k, dtype=torch.int32, device="cuda")
    wts = torch.empty(N, G, k, dtype=torch.float32, device="cuda")
    margin = torch.empty(N, G, dtype=torch.float32, device="cuda")
    seg_off = torch.empty(d.B * G * M + 1, dtype=torch.int32, device="cuda")
    seg_tok = torch.empty(N * G * k, dtype=torch.int32, device="cuda")
    row_map = torch.empty(N, G, k, dtype=torch.int32, device="cuda")
    Q = torch.empty(N, Ha, 64, dtype=torch.bfloat16, device="cuda")
    K = torch.empty(N, G, 64, dtype=torch.bfloat16, device="cuda")
    V = torch.empty(N, G, 64, dtype=torch.bfloat16, device="cuda")
    O = torch.empty(N, Ha, 64, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(N, d.D, dtype=torch.bfloat16, device="cuda")
    ws_route = gqe.workspace(d, gqe.OP_ROUTE)
    ws_comb = gqe.workspace(d, gqe.OP_COMBINE)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    calls = {
        "route": lambda: gqe.gqe_route(d, inp["x"], inp["Wr"], inp["br"], sel, wts, margin, seg_off, seg_tok, row_map,
                                       ws_route),
        "qproj": lambda: gqe.gqe_qproj(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], sel, seg_off, seg_tok, Q, K, V),
        "attention": lambda: gqe.gqe_attn(d, Q, K, V, O),
        "combine": lambda: gqe.gqe_combine(d, O, wts, inp["Wo"], y, ws_comb),
    }
    peaks = load_peaks()
    fl = flops_model(d)["gqe"]
    Ka = (G * k + G + 1) * 64
    for name, fn in calls.items():
        evs = []
        for i in range(warmup + steps):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            if i >= warmup:
                evs.append((a, b))
        torch.cuda.synchronize()
        ms = sorted(a.elapsed_time(b) for a, b in evs)[len(evs) // 2]
        line = {"study": "stages", "workload": workload, "stage": name, "us": ms * 1e3, "status": gqe.gqe_check_error()}
        if name == "route":
            by = 2 * N * d.D + 2 * d.D * G * M + 4 * N * G * k * 4 + 4 * N * G + 4 * (d.B * G * M + 1)
            line.update(bound="hbm", algorithmic_bytes=by, achieved_gbs=by / (ms / 1e3) / 1e9, peak=peaks["hbm_gbs"])
        elif name == "combine" and k > 1:
            by = N * (Ha * 128 + G * k * 4) + N * Ka * 2 * 2 + Ka * d.D * 2 + N * d.D * 2  # O, w, A out+in, Wo, y
            line.update(bound="hbm+tensor", algorithmic_bytes=by, achieved_gbs=by / (ms / 1e3) / 1e9,
                        peak=peaks["hbm_gbs"], tflops=fl["wo"] / (ms / 1e3) / 1e12)
        else:
            flops = {"qproj": fl["q_proj"] + fl["kv_proj"], "attention": fl["attention"], "combine": fl["wo"]}[name]
            line.update(bound="tensor", algorithmic_flops=flops, tflops=flops / (ms / 1e3) / 1e12,
                        peak=peaks["bf16_tflops"])
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="gqe", choices=["gqe", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle timing (rank 0, N=1)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--long", default="long_b1_t32768,million_b1_t1048576",
                    help="comma-separated long-context workloads timed after the headline (empty: none)")
    ap.add_argument("--study", choices=["pools", "decode", "stages"],
                    help="print the expert-pool, decode-step or per-stage study lines instead of the bench line")
    ap.add_argument("--cases", default="",
                    help="decode study: configurations as BxL, comma-separated (default: all three)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from gqe_inputs import CONFIGS
    d = CONFIGS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.study == "pools":
        pool_study(steps=min(args.steps, 20), warmup=args.warmup)
        return
    if args.study == "decode":
        decode_study(steps=min(args.steps, 20), warmup=args.warmup, cases=args.cases)
        return
    if args.study == "stages":
        stage_study(args.workload, steps=min(args.steps, 20), warmup=args.warmup)
        return
    if args.impl == "reference":
        run_reference(args, d, rank, world)
        return

    import torch
    import torch.distributed as dist
    import moe_gqa_query_gqe_b200 as gqe
    from gqe_inputs import make_inputs

    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))

    inp = make_inputs(d, seed=rank, device="cuda")
    N, G, M, k = d.B * d.T, d.G, d.M, d.k
    Ha = G * k + 1
    dev = "cuda"
    sel = torch.empty(N, G, k, dtype=torch.int32, device=dev)
    wts = torch.empty(N, G, k, dtype=torch.float32, device=dev)
    margin = torch.empty(N, G, dtype=torch.float32, device=dev)
    seg_off = torch.empty(d.B * G * M + 1, dtype=torch.int32, device=dev)
    seg_tok = torch.empty(N * G * k, dtype=torch.int32, device=dev)
    row_map = torch.empty(N, G, k, dtype=torch.int32, device=dev)
    Q = torch.empty(N, Ha, 64, dtype=torch.bfloat16, device=dev)
    K = torch.empty(N, G, 64, dtype=torch.bfloat16, device=dev)
    V = torch.empty(N, G, 64, dtype=torch.bfloat16, device=dev)
    O = torch.empty(N, Ha, 64, dtype=torch.bfloat16, device=dev)
    y = torch.empty(N, d.D, dtype=torch.bfloat16, device=dev)
    ws_route = gqe.workspace(d, gqe.OP_ROUTE)
    ws_comb = gqe.workspace(d, gqe.OP_COMBINE)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def stage_step(ev):
        # the forward pass as four C-ABI calls, events between them (per-stage times)
        ev[0].record(stream)
        gqe.gqe_route(d, inp["x"], inp["Wr"], inp["br"], sel, wts, margin, seg_off, seg_tok, row_map, ws_route)
        ev[1].record(stream)
        gqe.gqe_qproj(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], sel, seg_off, seg_tok, Q, K, V)
        ev[2].record(stream)
        gqe.gqe_attn(d, Q, K, V, O)
        ev[3].record(stream)
        gqe.gqe_combine(d, O, wts, inp["Wo"], y, ws_comb)
        ev[4].record(stream)

    ws_fwd = gqe.workspace(d, gqe.OP_FORWARD)
    ws_dense = gqe.workspace(d, gqe.OP_DENSE)
    y_dense = torch.empty_like(y)

    def gqe_step():
        gqe.gqe_forward(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], y, ws_fwd)

    def dense_step():
        gqe.gqa_dense_forward(d, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"], inp["Wo_dense"], y_dense, ws_dense)

    def as_graph(fn):
        # one step captured as a CUDA graph: the same kernels, no host enqueue
        # inside the timed region
        side = torch.cuda.Stream()
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            fn()
        torch.cuda.synchronize()
        return g

    # kernels launched per forward step: K/V + shared-query + router pair GEMM,
    # the selected queries, attention (which also builds the output operand
    # when k > 1), Wo. The selected queries are one dense pair GEMM over the
    # routed heads when M <= 2k; otherwise the routing scan and compaction
    # (one launch when the per-chunk counts fit a block's shared memory, else
    # two) and the gather.
    n_counts = d.B * d.G * d.M * ((d.T + 127) // 128)
    launches_per_step = 4 if d.M <= 2 * d.k else 4 + (1 if n_counts <= 4096 else 2)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def timed(fn, n):
        """n calls, L2 flushed before each outside the events; per-call ms."""
        evs = []
        for _ in range(n):
            flush.fill_(1)
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            evs.append((a, b))
        return evs

    g_gqe = as_graph(gqe_step)
    g_dense = as_graph(dense_step)

    # ---- warm-up, then K timed steps (L2 flushed between steps) -----------
    sampler = ClockSampler(local_rank)
    sampler.wait_first()
    timed(g_gqe.replay, args.warmup)
    assert gqe.gqe_check_error() == 0
    barrier()
    t_begin = time.time()
    evs = timed(g_gqe.replay, args.steps)
    barrier()
    t_end = time.time()
    clocks = sampler.stop(t_begin, t_end)
    status = gqe.gqe_check_error()
    assert status == 0, gqe.gqe_status_string(status)
    total_ms = sum(a.elapsed_time(b) for a, b in evs)
    total_ms = reduce_max([total_ms], world, dev)[0]
    ms_per_step = total_ms / args.steps
    value = job_throughput(world, N, ms_per_step)

    # ---- per-stage times (the same kernels through the four stage calls) -----
    sevs = []
    for i in range(args.warmup + args.steps):
        flush.fill_(1)
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        stage_step(ev)
        if i >= args.warmup:
            sevs.append(ev)
    torch.cuda.synchronize()
    stage_ms = [[ev[j].elapsed_time(ev[j + 1]) for j in range(4)] for ev in sevs]
    attn_ms = sum(s[2] for s in stage_ms) / len(stage_ms)
    stage_avg = {n: sum(s[j] for s in stage_ms) / len(stage_ms) for j, n in
                 enumerate(("route", "qproj", "attention", "combine"))}

    # ---- dense GQA baseline of the same library (speedup denominator) -------
    timed(g_dense.replay, args.warmup)
    devs = timed(g_dense.replay, args.steps)
    torch.cuda.synchronize()
    dense_ms = sum(a.elapsed_time(b) for a, b in devs) / args.steps

    # ---- the same layer with the selected heads' queries only (per-expert
    # gather; gqe_forward takes the dense product when M <= 2k): same y, bit
    # for bit, reported beside the headline --------------------------------
    ws_var = gqe.workspace(d, gqe.OP_FORWARD_VARIANT)
    y_sel = torch.empty_like(y)

    def gather_step():
        gqe.gqe_forward_variant(d, gqe.COMBINE_SLOT | gqe.QPROJ_GATHER, inp["x"], inp["Wq"], inp["Wk"], inp["Wv"],
                                inp["Wr"], inp["br"], inp["Wo"], y_sel, ws_var)

    g_gather = as_graph(gather_step)
    timed(g_gather.replay, args.warmup)
    gevs = timed(g_gather.replay, args.steps)
    torch.cuda.synchronize()
    gather_ms = sum(a.elapsed_time(b) for a, b in gevs) / args.steps
    gather_ms = reduce_max([gather_ms], world, dev)[0]
    gather_same = bool(torch.equal(y_sel, y))
    del g_gather

    # ---- end to end through the host-buffer entry point ---------------------
    x_host = inp["x"].cpu().pin_memory()
    y_host = torch.empty(N, d.D, dtype=torch.bfloat16).pin_memory()
    ws_host = gqe.workspace(d, gqe.OP_FORWARD_HOST)
    e2e = []
    for i in range(args.warmup + args.steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gqe.gqe_forward_host(d, x_host, inp["Wq"], inp["Wk"], inp["Wv"], inp["Wr"], inp["br"], inp["Wo"], y_host,
                             ws_host)
        e1.record(stream)
        if i >= args.warmup:
            e2e.append((e0, e1))
    torch.cuda.synchronize()
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e) / args.steps
    e2e_ms, dense_ms = reduce_max([e2e_ms, dense_ms], world, dev)
    status = gqe.gqe_check_error()
    assert status == 0, gqe.gqe_status_string(status)

    fl = flops_model(d)
    peaks = load_peaks()
    attn_flops = fl["gqe"]["attention"]
    attn_tflops = attn_flops / (attn_ms / 1e3) / 1e12
    roofline = {"bound": "tensor", "kernel": "attn2_fwd_kernel", "achieved": attn_tflops,
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": attn_tflops / peaks["bf16_tflops"],
                "peak_source": f"{peaks['source']} bf16 burst",
                "traffic": recorded_traffic(args.workload, "attn2.cuh"),
                "algorithmic_flops_per_launch": attn_flops}

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) activations, N(0,0.02^2) weights)",
            "config": {"workload": args.workload, **{kk: getattr(d, kk) for kk in ("B", "T", "D", "G", "M", "k", "dh")},
                       "tokens_per_step_per_gpu": N, "l2": "flushed between steps (256 MiB write)",
                       "parallelism": f"replicas x{world}"},
            "tflops": fl["gqe_total"] / (ms_per_step / 1e3) / 1e12 * world,
            "frac_bf16_peak": fl["gqe_total"] / (ms_per_step / 1e3) / 1e12 / peaks["bf16_tflops"],
            "dense_gqa_ms_per_step": dense_ms, "speedup_vs_dense": dense_ms / ms_per_step,
            "stage_ms": stage_avg, "stage_roofline": stage_rooflines(d, stage_avg, peaks), "roofline": roofline,
            "clocks": clocks,
            "e2e": {"value": job_throughput(world, N, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": N * d.D * 2, "d2h_bytes_per_step": N * d.D * 2,
                    "entry": "gqe_forward_host"},
            "gpu_launches": launches_per_step * args.steps,
            "qproj_path": "dense product over all routed heads, selected rows kept" if d.M <= 2 * d.k
                          else "selected heads only (per-expert gather)",
            "selected_heads_only": {"ms_per_step": gather_ms, "tokens_per_s": job_throughput(world, N, gather_ms),
                                    "speedup_vs_dense": dense_ms / gather_ms, "same_y_bits": gather_same,
                                    "entry": "gqe_forward_variant(COMBINE_SLOT | QPROJ_GATHER)"},
            "timing": "each step one CUDA-graph replay of gqe_forward; stage_ms from the four stage calls"}

    # long-context keys: one GPU, headline workload only (a scaling run keeps its timed work short)
    long_names = [n for n in args.long.split(",") if n] if (args.workload == DEFAULT_WORKLOAD and world == 1) else []
    routes = []
    if long_names:
        line["long_ctx"], routes = long_context(long_names, args.steps, args.warmup, rank, peaks, flush)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sel_fwd = gqe.forward_views(d, ws_fwd)["sel"]
        line["cpu_baseline"], line["parity"] = oracle_leg(d, inp, sel_fwd, y, args.cpu_budget, routes)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
