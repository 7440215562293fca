#!/usr/bin/env python
"""Committed tokens/s of Streaming Parallel Decoding on B200.

Default workload: the Qwen3-8B-shaped bf16 model (36 layers, d 4096, 32/8
heads, head_dim 128, FFN 12288, vocab 151936) at batch 16, prompts of
U[128, 1024] uniform-random tokens, 1024 tokens to generate, window 16,
lambda 0.1, tau 0.3, LM-head logit scale x4 (the medium-entropy regime).
Batch 1 (prompt 256) and the x16 / x1 regimes are reported under "extra".

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One process per GPU (torchrun for N > 1).  Sequences are independent, so
ranks are replicas with their own prompts and no data-path collective
("scaling": "weak"); rank 0 prints one JSON line.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "committed tokens/s"
UNIT = "tok/s"
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_8b_b16")
    ap.add_argument("--no-extra", action="store_true", help="skip the batch-1 and regime sweeps")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true", help="headline measurement only (for profiler runs)")
    ap.add_argument("--tile-n", type=int, default=0, help="kernel case: pin the GEMM tile width (0 = automatic)")
    ap.add_argument("--cta-pair", action="store_true", help="kernel case: CTA-pair GEMM tiles (tile width 128 or 256)")
    ap.add_argument("--micro-cell", default=None,
                    help="attn_micro: run one cell 'S,B' (attention, then the entropy pass at s=4) and exit "
                         "(single-kernel captures)")
    ap.add_argument("--k-splits", type=int, default=0, help="kernel case: pin the GEMM K slices (0 = automatic)")
    ap.add_argument("--rows", type=int, default=0,
                    help="kernel case: activation rows of the projection (0 = the batch-16 step's 256; 16 = batch 1)")
    ap.add_argument("--kernel-case", default=None,
                    help="run one projection of the batch-16 step (gemm_qkv|gemm_o|gemm_gate_up|gemm_down|"
                         "gemm_lm_head) three times through wedlm_linear_bf16, or 'attention' (3 decode steps of "
                         "a 2-layer model with the batch-16 shapes), and exit (single-kernel captures)")
    return ap.parse_args()


def workload_desc(cfg: dict, name: str) -> str:
    m = cfg["model"]
    P = cfg["P"]
    ps = f"U[{P[0]}, {P[1]}]" if isinstance(P, (tuple, list)) else str(P)
    return (f"{name}: random-init bf16 model L{m['L']} d{m['d']} heads {m['hq']}/{m['hkv']} hd{m['hd']} "
            f"ffn {m['F']} vocab {m['V']}; batch {cfg['B']}, prompts {ps} uniform ids, {cfg['N']} new tokens, "
            f"W {cfg['W']}, lambda {cfg['lam']}, tau {cfg['tau']}, logit scale x{cfg['logit_scale']:g}")


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm=p["hbm_gbs"], tc=p["bf16_tflops"], tc_sus=p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                    src="measured")
    return dict(hbm=6650.0, tc=1590.0, tc_sus=1400.0, src="fallback")


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ["index", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + ",".join(self.FIELDS), "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *a):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.t.join(timeout=2)

    def summary(self):
        rows = []
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], cap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        load = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"), ("swt", "sw_thermal_slowdown"),
                              ("cap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(load),
                "power_w_median": statistics.median(r["power"] for r in load)}


# ------------------------------------------------------------- our arm ---
class Replica:
    """One engine holding the Qwen3-8B-shaped model with max batch 16."""

    def __init__(self, cfg: dict, device: int, seed: int):
        import torch
        from streaming_decoding_b200 import Engine
        self.torch = torch
        self.cfg = cfg
        self.dims = cfg["model"]
        torch.cuda.set_device(device)
        self.stream = torch.cuda.Stream()
        Pmax = max(cfg["P"]) if isinstance(cfg["P"], (tuple, list)) else cfg["P"]
        self.max_ctx = max(Pmax, 256) + cfg["N"]
        t0 = time.perf_counter()
        self.eng = Engine(self.dims, max_batch=cfg["B"], max_window=cfg["W"], max_ctx=self.max_ctx,
                          stream=self.stream)
        for kind, layer, arr in synth.iter_weights(self.dims, seed=0, dtype="bf16"):
            self.eng.load_weights(kind, layer, arr)
        self.load_s = time.perf_counter() - t0
        self.seed = seed

    def admit(self, prompts, N, W):
        self.eng.kv_reset(-1)
        t0 = time.perf_counter()
        for b, p in enumerate(prompts):
            self.eng.prefill(b, p, N, W)
        self.prefill_s = time.perf_counter() - t0
        self.prefill_tokens = int(sum(len(p) for p in prompts))

    def committed(self, B):
        return sum(self.eng.stats(b)["committed"] for b in range(B))

    def timed_async(self, params, steps, B):
        """Device time of `steps` back-to-back steps (no host sync inside)."""
        torch = self.torch
        c0 = self.committed(B)
        l0 = self.eng.kernel_launches()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(self.stream)
        torch.cuda.nvtx.range_push("timed")  # lets a profiler select the timed launches
        self.eng.stream_step_async(params, steps)
        torch.cuda.nvtx.range_pop()
        end.record(self.stream)
        end.synchronize()
        ms = start.elapsed_time(end)
        return ms, self.committed(B) - c0, self.eng.kernel_launches() - l0

    def timed_e2e(self, params, steps):
        """Same metric through the synchronous public call (wedlm_stream_step,
        one call per step, each returning that step's committed tokens in pinned
        host buffers), timed on the host wall clock."""
        torch = self.torch
        B, W = self.cfg["B"], self.cfg["W"]
        committed = torch.zeros((B, W), dtype=torch.int32).pin_memory().numpy()
        counts = torch.zeros(B, dtype=torch.int32).pin_memory().numpy()
        active = torch.zeros(1, dtype=torch.int32).pin_memory().numpy()
        total = 0
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(steps):
            self.eng.stream_step_into(params, committed, counts, active)
            total += int(counts.sum())
        wall = time.perf_counter() - t0
        d2h = (2 * B + B * W + 1) * 4
        return wall, total, d2h

    def profile(self, params, steps):
        self.eng.profile_enable(True)
        self.eng.stream_step_async(params, steps)
        prof = self.eng.profile_read()
        self.eng.profile_enable(False)
        return prof


def gemm_shapes(dims, M):
    d, hq, hkv, hd, F, V = dims["d"], dims["hq"], dims["hkv"], dims["hd"], dims["F"], dims["V"]
    L = dims["L"]
    return {"gemm_qkv": (L, M, (hq + 2 * hkv) * hd, d), "gemm_o": (L, M, d, hq * hd),
            "gemm_gate_up": (L, M, 2 * F, d), "gemm_down": (L, M, d, F), "gemm_lm_head": (1, M, V, d)}


def src_hash(*names):
    """Hash of the named CUDA sources' code: comments and trailing blanks are
    dropped, so an edit that only touches comments keeps a profile valid."""
    import re
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "streaming_decoding_b200", "csrc", n), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln).encode())
    return h.hexdigest()[:16]


def measured_traffic(kernel_file: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    path = os.path.join(PROFILES, f"{kernel_file}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        p = json.load(f)
    if p.get("source_hash") != src_hash(*p.get("sources", [])) or p.get("workload") != workload:
        return None
    return p.get("dram_bytes_per_launch")


def roofline(prof, dims, M, pk, workload):
    """Dominant kernel: the tcgen05 GEMM over all projections of the step."""
    shapes = gemm_shapes(dims, M)
    bytes_tot = flops_tot = ms_tot = 0.0
    launches = 0
    for kind, (count, m, n, k) in shapes.items():
        ms, nl = prof.get(kind, (0.0, 0))
        if nl == 0:
            continue
        per = nl / count  # profiled steps
        bytes_tot += per * count * (2.0 * n * k + 2.0 * m * k + 4.0 * m * n)
        flops_tot += per * count * 2.0 * m * n * k
        ms_tot += ms
        launches += nl
    t_hbm = bytes_tot / (pk["hbm"] * 1e9)
    t_tc = flops_tot / (pk["tc_sus"] * 1e12)
    sec = ms_tot / 1e3
    traffic = measured_traffic("gemm_tc", workload)
    if t_hbm >= t_tc:
        ach = bytes_tot / sec / 1e9
        out = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
               "frac": round(ach / pk["hbm"], 4)}
    else:
        ach = flops_tot / sec / 1e12
        out = {"bound": "tensor", "achieved": round(ach, 1), "peak": pk["tc_sus"], "unit": "TFLOP/s",
               "frac": round(ach / pk["tc_sus"], 4)}
    out.update({"traffic": traffic, "kernel": "gemm_tc_kernel (all projections and LM head)",
                "launches_profiled": launches, "avg_launch_us": round(ms_tot * 1e3 / max(1, launches), 2),
                "algorithmic_bytes_per_launch": round(bytes_tot / max(1, launches)),
                "peak_source": f"{pk['src']} ({'hbm_gbs' if out['bound'] == 'hbm' else 'bf16_tflops_sustained'})"})
    return out, bytes_tot, flops_tot


def attention_roofline(prof, dims, B, W, S_mean, pk, steps):
    """The decode attention's own fraction of HBM: K and V of every committed
    position read once per sequence and layer (plus q and the output), over the
    attention kernel's event-timed duration."""
    ms, nl = prof.get("attention", (0.0, 0))
    if nl == 0:
        return None
    hq, hkv, hd, L = dims["hq"], dims["hkv"], dims["hd"], dims["L"]
    per_layer = B * (S_mean + W) * 2 * hkv * hd * 2 + 2 * B * W * hq * hd * 2
    sec = ms / 1e3 / steps / L
    ach = per_layer / sec / 1e9
    return {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm"], "unit": "GB/s",
            "frac": round(ach / pk["hbm"], 4), "kernel": "attn_tc_kernel", "us_per_layer": round(sec * 1e6, 2),
            "algorithmic_bytes_per_launch": round(per_layer),
            "peak_source": f"{pk['src']} (hbm_gbs)"}


def step_bytes_flops(dims, B, W, S_mean):
    """Algorithmic bytes and flops of one decode step (weights once, committed KV
    once per sequence and layer, logits once)."""
    d, hq, hkv, hd, F, V, L = (dims[k] for k in ("d", "hq", "hkv", "hd", "F", "V", "L"))
    params = L * ((hq + 2 * hkv) * hd * d + d * hq * hd + 3 * F * d) + V * d
    M = B * W
    byt = 2.0 * params + B * S_mean * L * 2 * hkv * hd * 2 + M * V * 4
    fl = 2.0 * M * (params - V * d) + 2.0 * M * V * d + 4.0 * M * hq * hd * (S_mean + W / 2) * L
    return byt, fl


def combine_ranks(dist, ms: float, tokens: float, device) -> tuple:
    """Whole-job aggregation across ranks: the slowest rank's device time (max)
    and the committed tokens of all ranks (sum); throughput = sum / max."""
    import torch
    t = torch.tensor([ms, tokens], dtype=torch.float64, device=device)
    mx = t.clone()
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(mx[0]), float(t[1])


def rank_prompts(cfg: dict, rank: int):
    """Each replica decodes its own prompts (weak scaling: fixed work per GPU)."""
    return synth.prompts(cfg, seed=cfg["prompt_seed"] + 100 * rank)


def run_ours(a):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        from datetime import timedelta
        dist = dist_mod
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    cfg = dict(synth.CONFIGS[a.workload])
    dims = cfg["model"]
    pk = peaks()
    rep = Replica(cfg, local, seed=rank)
    prompts = rank_prompts(cfg, rank)
    B, W, N = cfg["B"], cfg["W"], cfg["N"]
    from streaming_decoding_b200 import step_params
    prm = step_params(cfg["lam"], cfg["tau"], False, cfg["logit_scale"])

    # headline: device-resident steps, CUDA events on the library's stream
    rep.admit(prompts, N, W)
    rep.eng.stream_step_async(prm, a.warmup)
    torch.cuda.synchronize()
    S0 = np.mean([rep.eng.stats(b)["committed_len"] for b in range(B)])
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms, committed, launches = rep.timed_async(prm, a.steps, B)
    ms_all = ms
    tok_all = committed
    if dist:
        ms_all, tok_all = combine_ranks(dist, ms, committed, "cuda")
    value = tok_all / (ms_all / 1e3)
    S1 = np.mean([rep.eng.stats(b)["committed_len"] for b in range(B)])

    # per-kernel profile (separate pass; event gaps do not touch the headline)
    prof = rep.profile(prm, 10)
    M = B * W
    roof, gb, gf = roofline(prof, dims, M, pk, a.workload)
    sb, sf = step_bytes_flops(dims, B, W, (S0 + S1) / 2)
    step_floor_ms = max(sb / (pk["hbm"] * 1e9), sf / (pk["tc_sus"] * 1e12)) * 1e3

    # end to end through the public synchronous call: the same decode segment
    # (prompts admitted again, the same warm-up steps, the same step count),
    # host wall clock around the step calls
    rep.admit(prompts, N, W)
    rep.eng.stream_step_async(prm, a.warmup)
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    e_wall, e_tok, d2h = rep.timed_e2e(prm, a.steps)
    e2e_val = e_tok / e_wall
    if dist:
        e_max, e_sum = combine_ranks(dist, e_wall * 1e3, e_tok, "cuda")
        e2e_val = e_sum / (e_max / 1e3)

    extra = {"prefill": {"tokens": rep.prefill_tokens, "seconds": round(rep.prefill_s, 3),
                         "tok_per_s": round(rep.prefill_tokens / rep.prefill_s, 1)},
             "weights_load_s": round(rep.load_s, 2),
             "committed_per_step": round(committed / a.steps, 3),
             "mean_committed_len": [round(S0, 1), round(S1, 1)],
             "step_ms_floor_algorithmic": round(step_floor_ms, 3),
             "step_roofline_frac": round(step_floor_ms / (ms / a.steps), 4),
             "profile_ms_per_step": {k: round(v[0] / 10, 4) for k, v in prof.items() if v[1]},
             "attention_roofline": attention_roofline(prof, dims, B, W, (S0 + S1) / 2, pk, 10),
             "e2e_wall_s": round(e_wall, 3),
             "e2e_committed_per_step": round(e_tok / a.steps, 3),
             "gemm_plans_rows%d" % (B * W): {k: rep.eng.gemm_plan(k, B * W) for k in gemm_shapes(dims, M)},
             "gemm_schedules_rows%d" % (B * W): {k: rep.eng.gemm_schedule(k, B * W) for k in gemm_shapes(dims, M)}}
    if not a.quick and not a.no_extra and world == 1:
        if a.workload == "qwen3_8b_b16":
            extra.update(sweeps(rep, cfg, a))
        elif "lams" in cfg:
            extra.update(knob_sweep(rep, cfg, a, prompts))
    cpu = None
    if rank == 0 and world == 1 and not a.no_cpu_baseline and not a.quick:
        cpu = cpu_baseline(cfg, budget_s=25.0)
        cpu.pop("steps_timed", None)

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": a.steps,
            "warmup": a.warmup, "ms_per_step": round(ms_all / a.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded random-init weights, uniform-random prompt ids)",
            "config": {"workload": workload_desc(cfg, a.workload), "batch_per_gpu": B, "window": W,
                       "global_batch": B * world, "l2": "inputs larger than L2 (15.1 GB of weights read per step)",
                       "parallelism": f"replicas x{world} (independent sequences, no collective)"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 2), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": d2h,
                    "api": "wedlm_stream_step (synchronous, one call per step), pinned host outputs, host wall clock",
                    "segment": "the same prompts, warm-up and step count as value",
                    "note": "h2d_bytes_per_step is 0 because a decode step takes no host input: the window, "
                            "the KV cache and every per-step size stay on the device; each step copies its "
                            "committed tokens, counts and committed lengths back (d2h_bytes_per_step)"},
            "gpu_launches": int(launches),
            "clocks": clk.summary(),
            "extra": extra}
    print(json.dumps(line))


def sweeps(rep, cfg, a):
    """Batch 1 (prompt 256) and the logit-scale regimes at batch 16."""
    from streaming_decoding_b200 import step_params
    out = {}
    steps = min(a.steps, 150)
    b1 = synth.CONFIGS["qwen3_8b_b1"]
    rep.admit(synth.prompts(b1), b1["N"], b1["W"])
    prm = step_params(b1["lam"], b1["tau"], False, b1["logit_scale"])
    rep.eng.stream_step_async(prm, a.warmup)
    ms, com, _ = rep.timed_async(prm, steps, 1)
    out["batch1"] = {"workload": workload_desc(b1, "qwen3_8b_b1"), "tok_per_s": round(com / (ms / 1e3), 2),
                     "ms_per_step": round(ms / steps, 4), "committed_per_step": round(com / steps, 3),
                     "gemm_plans_rows16": {k: rep.eng.gemm_plan(k, b1["W"]) for k in gemm_shapes(rep.dims, 16)}}
    reg = {}
    prompts = synth.prompts(cfg)
    for scale in cfg["logit_scales"]:
        rep.admit(prompts, cfg["N"], cfg["W"])
        prm = step_params(cfg["lam"], cfg["tau"], False, scale)
        rep.eng.stream_step_async(prm, a.warmup)
        n = min(steps, 40 if scale >= 16 else steps)
        ms, com, _ = rep.timed_async(prm, n, cfg["B"])
        reg[f"x{scale:g}"] = {"tok_per_s": round(com / (ms / 1e3), 2), "ms_per_step": round(ms / n, 4),
                              "committed_per_step": round(com / n, 3)}
    out["regimes_batch16"] = reg
    # the pages' comparison decoders on the same kernels: block-wise
    # (stop-and-wait) commits and sampled fills at T = 0.1, batch 16, x4
    cmp_ = {}
    scale = cfg["logit_scale"]
    for name, kw in (("streaming_greedy", {}), ("blockwise_greedy", {"blockwise": True}),
                     ("streaming_sampled_t0.1", {"temperature": 0.1, "seed": 1234})):
        rep.admit(prompts, cfg["N"], cfg["W"])
        prm = step_params(cfg["lam"], cfg["tau"], False, scale, **kw)
        rep.eng.stream_step_async(prm, a.warmup)
        n = min(steps, 60)
        ms, com, _ = rep.timed_async(prm, n, cfg["B"])
        cmp_[name] = {"tok_per_s": round(com / (ms / 1e3), 2), "ms_per_step": round(ms / n, 4),
                      "committed_per_step": round(com / n, 3)}
    out["decoders_batch16_x%g" % scale] = cmp_
    return out


def knob_sweep(rep, cfg, a, prompts):
    """lambda x tau sweep of a workload that lists them: the batch is admitted
    once and each setting then decodes a stretch of steps in turn (the context
    grows by the tokens committed in between)."""
    from streaming_decoding_b200 import step_params
    rep.admit(prompts, cfg["N"], cfg["W"])
    out = {}
    n = max(5, min(a.steps, 20))
    for lam in cfg["lams"]:
        for tau in cfg["taus"]:
            prm = step_params(lam, tau, False, cfg["logit_scale"])
            rep.eng.stream_step_async(prm, 2)
            ms, com, _ = rep.timed_async(prm, n, cfg["B"])
            out[f"lambda{lam:g}_tau{tau:g}"] = {"tok_per_s": round(com / (ms / 1e3), 2),
                                               "ms_per_step": round(ms / n, 4),
                                               "committed_per_step": round(com / n, 3)}
    return {"lambda_tau_sweep": out, "lambda_tau_sweep_steps": n}


# ------------------------------------------------------- C2 microbench --
def run_micro(a):
    """Single-layer decode-step microbench: the decode attention over random
    page tables at committed lengths S x batch sizes B (W = 16 window rows, 32 /
    8 heads, head_dim 128), and the vocabulary-151936 entropy + selection pass
    over N(0, s^2) logits of the masked half of each window.  Each cell is
    timed with CUDA events around single launches, after an L2 flush (a 256
    MB write) before every launch; achieved GB/s counts the algorithmic bytes
    (K and V of every position once, q and the output; the masked rows'
    logits once)."""
    import torch
    from streaming_decoding_b200 import (attention_bf16, attention_error, attention_workspace, entropy_select_async,
                                         step_params)
    cfg = synth.CONFIGS["attn_micro"]
    m = cfg["model"]
    hq, hkv, V, W = m["hq"], m["hkv"], m["V"], cfg["W"]
    pk = peaks()
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(cfg["prompt_seed"])
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    iters = max(5, min(a.steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def timed(fn):
        for _ in range(3):
            fn()
        ts = []
        for _ in range(iters):
            flush.zero_()
            e0.record()
            fn()
            e1.record()
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    cells_S, cells_B, stds = cfg["S"], cfg["B"], cfg["logit_std"]
    if a.micro_cell:
        S1, B1 = (int(v) for v in a.micro_cell.split(","))
        cells_S, cells_B, stds = (S1,), (B1,), (4.0,)
    att = []
    for S in cells_S:
        for B in cells_B:
            pps = (S + W + 15) // 16
            pool = torch.randn(B * pps, 2, hkv, 16, 128, device="cuda", generator=g, dtype=torch.bfloat16)
            table = torch.randperm(B * pps, device="cuda", generator=g).to(torch.int32).view(B, pps)
            q = torch.randn(B * W, hq, 128, device="cuda", generator=g, dtype=torch.bfloat16)
            Sd = torch.full((B,), S, dtype=torch.int32, device="cuda")
            nd = torch.full((B,), W, dtype=torch.int32, device="cuda")
            ws = attention_workspace(B, W, hq, hkv, S + W)
            out = torch.empty_like(q)
            ms = timed(lambda: attention_bf16(q, pool, table, Sd, nd, W, hq, hkv, S + W, ws, out=out))
            torch.cuda.synchronize()
            assert attention_error(ws) == 0
            byt = B * (S + W) * hkv * 128 * 2 * 2 + 2 * B * W * hq * 128 * 2
            att.append({"S": S, "B": B, "us": round(ms * 1e3, 2), "GB_s": round(byt / (ms / 1e3) / 1e9, 1),
                        "frac": round(byt / (ms / 1e3) / 1e9 / pk["hbm"], 4)})
            del pool, table, q, ws, out
    ent = []
    nf = cfg["n_filled"]
    prm = step_params(0.1, 0.3, False, 1.0)
    for s_ in stds:
        for B in cells_B:
            filled, _ = synth.window_state(2002, int(s_), B, W, nf, V, V - 1)
            fd = torch.from_numpy(filled).cuda()
            nd = torch.full((B,), W, dtype=torch.int32, device="cuda")
            z = torch.randn(B * W, V, device="cuda", generator=g) * s_
            outs = entropy_select_async(z, V, V - 1, fd, nd, W, prm)
            ws = outs[3]
            ms = timed(lambda: entropy_select_async(z, V, V - 1, fd, nd, W, prm, workspace=ws, out=outs[:3]))
            byt = B * (W - nf) * V * 4
            ent.append({"s": s_, "B": B, "us": round(ms * 1e3, 2), "GB_s": round(byt / (ms / 1e3) / 1e9, 1),
                        "frac": round(byt / (ms / 1e3) / 1e9 / pk["hbm"], 4)})
            del z
    big = max(att, key=lambda c: (c["S"], c["B"]))
    line = {"metric": "decode attention GB/s (largest cell)", "value": big["GB_s"], "unit": "GB/s", "n_gpus": 1,
            "steps": iters, "warmup": 3, "higher_is_better": True, "dtype": "bf16",
            "data": "synthetic (torch.randn K/V, q and logits; random page tables)",
            "config": {"workload": "attn_micro: one layer, 32/8 heads, head_dim 128, W 16 (8 slots filled), "
                                   "16-token pages; S x B grid; entropy over vocab 151936",
                       "l2": "flushed before every launch (256 MB write)"},
            "peak": {"hbm_gbs": pk["hbm"], "source": pk["src"]},
            "attention": att, "entropy": ent}
    print(json.dumps(line))


# ------------------------------------------------------------ CPU oracle --
def cpu_baseline(cfg, budget_s: float, steps_max: int = 50, warmup: int = 1):
    """The oracle as it stands on the host cores: one sequence of the workload
    (its first 16 prompt tokens), decoded step by step until the time budget
    or `steps_max` is used; weight widening and prefill are untimed."""
    from oracle import wedlm_oracle as O
    dims = cfg["model"]
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 0) for i in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count()
    w = synth.model_weights(dims, seed=0, dtype="bf16")
    # widened fp64 copies of every matrix (8 bytes a parameter) only when the
    # host has the room; otherwise each matrix is widened where it is used
    n_par = sum(int(np.prod(x.shape)) for x in [w["embed"], w["lm_head"]] +
                [a for layer in w["layers"] for a in layer.values()])
    try:
        import psutil
        avail = psutil.virtual_memory().available
    except Exception:
        avail = 0
    cache = avail > 1.3 * 8 * n_par + 16e9
    m = O.Model(dims, w, cache_fp64=cache)
    prompt = synth.prompts(cfg)[0][:16]
    st = O.prefill(m, prompt, cfg["N"], cfg["W"])
    for _ in range(warmup):
        O.stream_step(m, st, cfg["lam"], cfg["tau"], False, cfg["logit_scale"], keep_trace=False)
    c0 = len(st.out)
    t0 = time.perf_counter()
    n = 0
    while n < steps_max and time.perf_counter() - t0 < budget_s and not st.done:
        O.stream_step(m, st, cfg["lam"], cfg["tau"], False, cfg["logit_scale"], keep_trace=False)
        n += 1
    dt = time.perf_counter() - t0
    com = len(st.out) - c0
    return {"value": round(com / dt, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"1 sequence (first 16 prompt tokens), {n} decode steps after {warmup} untimed, "
                      f"{com} tokens committed in {dt:.1f} s; fp64 numpy, weights "
                      f"{'widened once' if cache else 'widened per use (host memory)'}",
            "s_per_step": round(dt / max(1, n), 3), "steps_timed": n}


def run_reference(a):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cfg = dict(synth.CONFIGS[a.workload])
    # at least 8 timed steps: the first steps of a fresh window commit nothing yet
    res = cpu_baseline(cfg, budget_s=120.0, steps_max=max(8, a.steps), warmup=max(1, min(a.warmup, 2)))
    steps = res.pop("steps_timed")
    line = {"impl": "reference", "metric": METRIC, "value": res["value"], "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": a.warmup, "ms_per_step": round(res["s_per_step"] * 1e3, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded random-init weights, uniform-random prompt ids)",
            "config": {"workload": workload_desc(cfg, a.workload), "batch_per_gpu": cfg["B"], "window": cfg["W"]},
            "cpu_baseline": res,
            "e2e": {"value": res["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def attention_case(steps: int = 3):
    """Decode steps of a 2-layer model with the Qwen3-8B head layout on the
    batch-16 prompts (same attention shapes per layer as the full model, a few
    GB on the device): the case for single-kernel captures of the attention."""
    import torch
    from streaming_decoding_b200 import Engine, step_params
    cfg = dict(synth.CONFIGS["qwen3_8b_b16"])
    dims = dict(cfg["model"], L=2)
    eng = Engine(dims, max_batch=cfg["B"], max_window=cfg["W"], max_ctx=1024 + cfg["N"])
    eng.load_model(synth.iter_weights(dims, seed=0, dtype="bf16"))
    for b, p in enumerate(synth.prompts(cfg)):
        eng.prefill(b, p, cfg["N"], cfg["W"])
    eng.stream_step_async(step_params(cfg["lam"], cfg["tau"], False, cfg["logit_scale"]), steps)
    torch.cuda.synchronize()
    print(json.dumps({"kernel_case": "attention", "layers": 2, "batch": cfg["B"], "steps": steps,
                      "prefill_attention_launches": cfg["B"] * 2}))


def kernel_case(name: str, tile_n: int = 0, cta_pair: bool = False, rows: int = 0, k_splits: int = 0):
    import torch
    from streaming_decoding_b200 import linear_bf16
    if name == "attention":
        return attention_case()
    cfg = synth.CONFIGS["qwen3_8b_b16"]
    dims = cfg["model"]
    L, M, N, K = gemm_shapes(dims, rows if rows > 0 else cfg["B"] * cfg["W"])[name]
    g = torch.Generator(device="cuda").manual_seed(0)
    X = torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16)
    W = (torch.randn(N, K, device="cuda", generator=g) * 0.02).to(torch.bfloat16)
    for _ in range(3):
        linear_bf16(X, W, tile_n=tile_n, k_splits=k_splits, cta_pair=cta_pair)
    torch.cuda.synchronize()
    print(json.dumps({"kernel_case": name, "M": M, "N": N, "K": K, "weight_bytes": 2 * N * K, "tile_n": tile_n,
                      "k_splits": k_splits, "cta_pair": cta_pair}))


if __name__ == "__main__":
    args = parse()
    if args.kernel_case:
        kernel_case(args.kernel_case, args.tile_n, args.cta_pair, args.rows, args.k_splits)
    elif args.workload == "attn_micro" and args.impl == "ours":
        run_micro(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)
