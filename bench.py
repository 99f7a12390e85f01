#!/usr/bin/env python
"""Routed FP4 MoE layer benchmark on B200.

One step = one pass of the whole layer (route -> sort -> INT8 quant -> W1 ->
SwiGLU + requant -> W2 -> combine) over one batch of seeded synthetic input,
through the library's one-call entry point moe_layer_forward.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl moe|reference]

Prints one JSON line on rank 0.  `value` is tokens/s of the whole job with
inputs resident in HBM; `e2e` is the same through host buffers (pinned H2D of
x and logits, D2H of y, inside the timed region).  Multi-GPU runs are
independent replicas (weak scaling), timed as the max over ranks.
The reference arm (--impl reference) times the CPU oracle on the same
workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

# Algorithmic HBM bytes of one expert's weights (codes + scales, W1 and W2).
def expert_bytes(H: int, I: int) -> int:
    return (2 * I * H + H * I) * 17 // 32


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["moe", "reference"], default="moe")
    ap.add_argument("--workload", default="decode_T8")
    ap.add_argument("--prefill-workload", default="prefill_T4604")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-skew", action="store_true", help="skip the skewed prefill lines")
    ap.add_argument("--no-decode-t64", action="store_true", help="skip the decode_T64 line")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 dense projection lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tc-pair", type=int, choices=[0, 1], default=None,
                    help="MOE_OPT_TC_PAIR for the run (default: the library's default)")
    ap.add_argument("--tc-min", type=int, default=None,
                    help="MOE_OPT_TC_MIN_ROWS for the run (1: every expert on the tensor cores)")
    ap.add_argument("--tc-a-tmem", type=int, choices=[0, 1], default=None,
                    help="MOE_OPT_TC_A_TMEM for the run (default: the library's default)")
    ap.add_argument("--tc-form", type=int, choices=[0, 1, 2], default=None,
                    help="MOE_OPT_TC_FORM for the run (default: the library's default)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile-run", action="store_true",
                    help="no timing, no JSON: pack the workload and run --steps layer calls "
                         "(the command profiled under ncu)")
    ap.add_argument("--experts", type=int, default=None,
                    help="with --profile-run: override E (a smaller capture of the same kernels)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="with --profile-run: override T (with --experts: keep the rows per expert)")
    ap.add_argument("--fp8-workload", default=None,
                    help="with --profile-run: run the FP8 dense projection of this workload instead")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------
# distributed plumbing (replicas: barrier + max-over-ranks only, no data-path collective)

class Dist:
    """One process per GPU (torchrun env vars): barrier and max over ranks.
    backend/device default to NCCL on the rank's GPU; the CPU tests use gloo."""

    def __init__(self, n_expected: int, backend: str | None = None, device: str | None = None):
        import torch
        import torch.distributed as dist
        self.torch, self.dist = torch, dist
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.backend = backend or "nccl"
        self.device = device or "cuda"
        if self.device == "cuda":
            torch.cuda.set_device(self.local if self.world > 1 else 0)
        if self.world > 1:
            import datetime
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120))
        if n_expected != self.world:
            print(f"warning: --gpus {n_expected} but WORLD_SIZE {self.world}", file=sys.stderr)

    def barrier(self):
        if self.world > 1:
            self.dist.barrier()

    def max(self, v: float) -> float:
        if self.world == 1:
            return v
        t = self.torch.tensor([v], dtype=self.torch.float64, device=self.device)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def whole_job_value(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Tokens/s of the whole job: every replica processes tokens_per_step tokens per
    step (weak scaling); the slowest rank's time bounds the job."""
    return world * tokens_per_step * steps / (max_ms * 1e-3)


# ---------------------------------------------------------------------------------------
# clocks sampled during the timed region

class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", str(gpu_index), "--query-gpu=" + self.Q,
                                       "--format=csv,noheader,nounits", "-lms", "100"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None
        time.sleep(0.3)

    def stop(self) -> dict:
        if self.p is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.p.terminate()
        try:
            self.p.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.p.kill()
        self.f.flush()
        rows = [r.split(",") for r in open(self.f.name).read().strip().splitlines() if r.strip()]
        os.unlink(self.f.name)
        sm, mx, reasons, pw = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = float(r[2])
                pw.append(float(r[3]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w": statistics.median(pw) if pw else None}


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def profiled_traffic(summary: str):
    """DRAM bytes per launch (read + write) of a GEMM kernel, from a committed ncu
    summary under profiles/; None unless every kernel source is unchanged since
    the capture (the summary records each source file and its SHA-256)."""
    p = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(p):
        return None
    text = open(p).read()
    srcs = re.findall(r"^\s*kernel_source:\s*(\S+)", text, re.M)
    shas = re.findall(r"^\s*kernel_source_sha256:\s*([0-9a-f]{64})", text, re.M)
    val = re.search(r"^\s*dram_bytes_per_launch:\s*(\d+)", text, re.M)
    if not (srcs and len(srcs) == len(shas) and val):
        return None
    for src, sha in zip(srcs, shas):   # every source the captured kernels were built from
        path = os.path.join(ROOT, src)
        if not os.path.exists(path) or hashlib.sha256(open(path, "rb").read()).hexdigest() != sha:
            return None
    return int(val.group(1))


# ---------------------------------------------------------------------------------------

def run_gpu_workload(name: str, steps: int, warmup: int, dist: Dist, want_e2e: bool,
                     want_clocks: bool):
    import torch

    import fp4_routed_mixture_b200 as moe

    w = synth.WORKLOADS[name]
    T, H, I, E, k = w.T, w.H, w.I, w.E, w.k
    d = synth.make(w)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    canon = [cu(d[n]) for n in ("w1_codes", "w1_scales", "w2_codes", "w2_scales")]
    packed = moe.moe_pack_weights(*canon)
    del canon
    logits = cu(d["logits"])
    x = cu(d["x"]).view(torch.bfloat16)
    ws = torch.empty(moe.moe_layer_workspace_bytes(T, H, I, E, k), dtype=torch.uint8, device="cuda")
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()

    # touched experts of this batch (outside the timed region)
    idx, _ = moe.moe_route(logits, k)
    touched = int(torch.unique(idx).numel())
    alg_bytes_step = touched * expert_bytes(H, I)
    alg_flop_step = 6.0 * T * k * I * H

    def step(dbg=None):
        moe.moe_layer_forward(logits, x, packed, H, I, E, k, ws=ws, y=y, dbg=dbg, stream=stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()

    # Timed region 1, the metric: the layer exactly as a caller runs it (its
    # kernels chained by programmatic dependent launch).
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = Clocks(torch.cuda.current_device()) if want_clocks else None
    launches0 = moe.moe_launch_count()
    dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for s in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    launches = moe.moe_launch_count() - launches0
    clk = clocks.stop() if clocks else None
    ms = dist.max(t0.elapsed_time(t1))
    # Timed region 2, the GEMM roofline: the same steps with CUDA events around
    # each GEMM phase (W1 start/end, W2 start/end).  An event recorded between
    # two launches ends their programmatic overlap, so this region runs slower
    # than region 1; the phase times it gives include each GEMM launch's
    # start-up and drain (conservative for the roofline).
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    dbgs = [moe.make_debug(None, e) for e in ev]
    dist.barrier()
    torch.cuda.synchronize()
    t2, t3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t2.record(stream)
    for s in range(steps):
        step(dbgs[s])
    t3.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    ms_events = dist.max(t2.elapsed_time(t3))
    gemm_ms = sum(e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev)
    w1_ms = sum(e[0].elapsed_time(e[1]) for e in ev)
    w2_ms = sum(e[2].elapsed_time(e[3]) for e in ev)
    flag = moe.moe_check_device_flag(ws)
    assert flag == 0, f"device error word {flag:#x}"

    res = dict(workload=w, T=T, ms=ms, steps=steps, launches=launches, clocks=clk, touched=touched,
               alg_bytes_step=alg_bytes_step, alg_flop_step=alg_flop_step, gemm_ms=gemm_ms,
               w1_ms=w1_ms, w2_ms=w2_ms, ms_events=ms_events)

    # the router projection in front of the path (not part of the metric's
    # A1-A7 step): its own time per step, same tokens
    wr = torch.from_numpy(synth.router_weight(w.seed, E, H)).cuda()
    rb = synth.router_bias(E, w.bias_coef)
    rb = None if rb is None else torch.from_numpy(rb.astype(np.float32)).cuda()
    lg = torch.empty((T, E), dtype=torch.float32, device="cuda")
    for _ in range(3):
        moe.moe_router_logits(x, wr, rb, out=lg, stream=stream)
    r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    rsteps = max(3, min(steps, 200))
    r0.record(stream)
    for _ in range(rsteps):
        moe.moe_router_logits(x, wr, rb, out=lg, stream=stream)
    r1.record(stream)
    torch.cuda.synchronize()
    res["router_ms"] = r0.elapsed_time(r1) / rsteps
    res["router_flop"] = 2.0 * T * H * E
    del wr, lg

    if want_e2e:
        xh = torch.from_numpy(d["x"]).view(torch.bfloat16).pin_memory()
        lh = torch.from_numpy(d["logits"]).pin_memory()
        yh = torch.empty((T, H), dtype=torch.bfloat16).pin_memory()
        xd = torch.empty_like(x)
        ld = torch.empty_like(logits)

        def e2e_step():
            xd.copy_(xh, non_blocking=True)
            ld.copy_(lh, non_blocking=True)
            moe.moe_layer_forward(ld, xd, packed, H, I, E, k, ws=ws, y=y, stream=stream)
            yh.copy_(y, non_blocking=True)

        for _ in range(max(3, warmup)):
            e2e_step()
        torch.cuda.synchronize()
        dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        res["e2e_ms"] = dist.max(e0.elapsed_time(e1))
        res["h2d"] = xh.numel() * 2 + lh.numel() * 4
        res["d2h"] = yh.numel() * 2
    del packed, ws
    torch.cuda.empty_cache()
    return res


def run_fp8_dense(name: str, steps: int, warmup: int, dist: Dist, peaks: dict, want_clocks: bool) -> dict:
    """The FP8 block-quantised dense projection (moe_fp8_linear: activation
    quantisation + tcgen05 kind::mxf8f6f4 GEMM), timed as whole calls."""
    import torch

    import fp4_routed_mixture_b200 as moe
    w = synth.DENSE_WORKLOADS[name]
    d = synth.make_dense(w)
    cu = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    packed = moe.moe_fp8_pack_weights(cu(d["w_codes"]), cu(d["w_scales"]))
    x = cu(d["x"]).view(torch.bfloat16)
    ws = torch.empty(moe.lib.moe_fp8_workspace_bytes(w.T, w.N, w.K), dtype=torch.uint8, device="cuda")
    y = torch.empty((w.T, w.N), dtype=torch.bfloat16, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        moe.moe_fp8_linear(x, packed, w.N, ws=ws, y=y, stream=stream)
    torch.cuda.synchronize()
    clocks = Clocks(torch.cuda.current_device()) if want_clocks else None
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(steps):
        moe.moe_fp8_linear(x, packed, w.N, ws=ws, y=y, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop() if clocks else None
    ms = dist.max(e0.elapsed_time(e1)) / steps
    assert moe.moe_check_device_flag(ws) == 0
    flop = 2.0 * w.T * w.N * w.K
    wbytes = w.N * w.K + (w.N // 128) * (w.K // 128)
    line = {"workload": name, "T": w.T, "N": w.N, "K": w.K, "steps": steps,
            "value": round(whole_job_value(dist.world, w.T, steps, ms * steps), 1), "unit": "tokens/s",
            "ms_per_step": round(ms, 5), "clocks": clk,
            "kernels": "k_fp8_quant_act + k_fp8_gemm (tcgen05 kind::mxf8f6f4 block-scaled) + k_fp8_reduce "
                       "(calls of at most 64 tokens: the split K ranges' partial sums); the step times them all"}
    traffic = profiled_traffic(f"k_fp8_gemm_{name}.md")
    if w.T >= 1024:
        tf = flop / (ms * 1e-3) / 1e12
        fp8_peak = 2.0 * peaks["bf16_tflops"]
        line["roofline"] = {"bound": "tensor", "achieved": round(tf, 2), "unit": "TFLOP/s", "peak": fp8_peak,
                            "frac": round(tf / fp8_peak, 5),
                            "peak_source": peaks["source"] + " bf16 x 2 (fp8/bf16 nominal ratio)", "traffic": traffic}
    else:
        gbs = wbytes / (ms * 1e-3) / 1e9
        line["roofline"] = {"bound": "hbm", "achieved": round(gbs, 1), "unit": "GB/s", "peak": peaks["hbm_gbs"],
                            "frac": round(gbs / peaks["hbm_gbs"], 4), "alg_bytes_per_launch": wbytes,
                            "peak_source": peaks["source"] + " (hbm_gbs: stream copy)", "traffic": traffic}
    del packed, ws
    torch.cuda.empty_cache()
    return line


def cpu_baseline(name: str, seconds: float) -> dict:
    import oracle
    w = synth.WORKLOADS[name]
    d = synth.make(w)
    t0 = time.time()
    reps = 0
    if w.T <= 64:
        # the whole step (all T tokens) per repetition
        while True:
            oracle.forward(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                           d["w2_scales"], w.k)
            reps += 1
            if time.time() - t0 >= seconds:
                break
        toks = reps * w.T
        sample = f"{reps} full steps of {name} ({w.T} tokens each)"
    else:
        tok = 0
        while time.time() - t0 < seconds:
            oracle.forward_tokens(d["x"], d["logits"], d["w1_codes"], d["w1_scales"],
                                  d["w2_codes"], d["w2_scales"], w.k, [tok % w.T])
            tok += 1
        toks = tok
        sample = f"{tok} single-token layer evaluations of {name}"
    dt = time.time() - t0
    return {"value": toks / dt, "unit": "tokens/s", "cores": oracle.nthreads(), "kind": "oracle",
            "sample": sample, "seconds": round(dt, 2)}


def router_line(r: dict) -> dict:
    """The router projection (logits = x W_r^T, moe_router_logits) timed on its own:
    the step in front of the layer, outside the A1-A7 metric."""
    return {"ms_per_step": round(r["router_ms"], 5),
            "tflops": round(r["router_flop"] / (r["router_ms"] * 1e-3) / 1e12, 3),
            "kernel": "k_router_logits (fp32 CUDA-core contraction)", "in_metric": False}


def roofline_hbm(r: dict, peaks: dict, traffic, kernel="k_gemv (W1 and W2 launches)", per_phase=1):
    """HBM roofline of the W1 + W2 GEMM phases (events around each phase, one or
    more launches each).  The step's weight bytes are split over the two
    phases; with one launch per phase they are the bytes per launch, and the
    traffic (DRAM bytes, from a committed ncu summary) is per phase."""
    n_launch = 2 * per_phase * r["steps"]
    bytes_per_phase = r["alg_bytes_step"] / 2.0
    achieved = (r["alg_bytes_step"] * r["steps"]) / (r["gemm_ms"] * 1e-3) / 1e9
    per = {"alg_bytes_per_launch": bytes_per_phase} if per_phase == 1 else \
          {"alg_bytes_per_phase": bytes_per_phase, "traffic_is": "DRAM bytes per phase"}
    return {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1),
            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
            "traffic": traffic, "launches": n_launch, **per,
            "peak_source": peaks["source"] + " (hbm_gbs: stream copy)"}


def profile_run(a):
    import dataclasses

    import torch

    import fp4_routed_mixture_b200 as moe
    if a.fp8_workload:
        fw = synth.DENSE_WORKLOADS[a.fp8_workload]
        fd = synth.make_dense(fw)
        cu = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
        packed = moe.moe_fp8_pack_weights(cu(fd["w_codes"]), cu(fd["w_scales"]))
        x = cu(fd["x"]).view(torch.bfloat16)
        ws = torch.empty(moe.lib.moe_fp8_workspace_bytes(fw.T, fw.N, fw.K), dtype=torch.uint8, device="cuda")
        for _ in range(a.steps or 3):
            y = moe.moe_fp8_linear(x, packed, fw.N, ws=ws)
        torch.cuda.synchronize()
        assert moe.moe_check_device_flag(ws) == 0
        print(f"profile run ok: {fw.name}, {a.steps or 3} steps, max|y| = {float(y.float().abs().max())}")
        return
    w = synth.WORKLOADS[a.workload]
    if a.experts:
        w = dataclasses.replace(w, name=f"{w.name}_E{a.experts}", E=a.experts)
    if a.tokens:
        w = dataclasses.replace(w, name=f"{w.name}_T{a.tokens}", T=a.tokens)
    d = synth.make(w)
    cu = lambda x: torch.from_numpy(np.ascontiguousarray(x)).cuda()
    packed = moe.moe_pack_weights(*[cu(d[n]) for n in ("w1_codes", "w1_scales", "w2_codes", "w2_scales")])
    torch.cuda.empty_cache()
    logits, x = cu(d["logits"]), cu(d["x"]).view(torch.bfloat16)
    ws = torch.empty(moe.moe_layer_workspace_bytes(w.T, w.H, w.I, w.E, w.k), dtype=torch.uint8, device="cuda")
    for _ in range(a.steps or 3):
        y = moe.moe_layer_forward(logits, x, packed, w.H, w.I, w.E, w.k, ws=ws)
    torch.cuda.synchronize()
    assert moe.moe_check_device_flag(ws) == 0
    print(f"profile run ok: {w.name}, {a.steps or 3} steps, max|y| = {float(y.float().abs().max())}")


def apply_options(a):
    import fp4_routed_mixture_b200 as moe
    for value, opt in ((a.tc_pair, moe.MOE_OPT_TC_PAIR), (a.tc_a_tmem, moe.MOE_OPT_TC_A_TMEM),
                       (a.tc_form, moe.MOE_OPT_TC_FORM), (a.tc_min, moe.MOE_OPT_TC_MIN_ROWS)):
        if value is not None:
            moe.moe_set_option(opt, value)


def main():
    a = parse()
    if a.profile_run:
        apply_options(a)
        return profile_run(a)
    if a.impl == "reference":
        return main_reference(a)
    steps = a.steps if a.steps is not None else 2000
    warmup = a.warmup if a.warmup is not None else 20
    assert warmup >= 3 or a.warmup is not None
    dist = Dist(a.gpus)
    import torch

    import fp4_routed_mixture_b200 as moe
    apply_options(a)
    rank0 = dist.rank == 0
    peaks = measured_peaks()
    r = run_gpu_workload(a.workload, steps, warmup, dist, want_e2e=True, want_clocks=rank0)
    w = r["workload"]
    N = dist.world
    value = whole_job_value(N, w.T, steps, r["ms"])
    out = {
        "metric": "routed-MoE layer tokens/s (T=8 decode, T=4604 prefill); % HBM / TC roofline",
        "value": round(value, 1), "unit": "tokens/s", "n_gpus": N, "steps": steps,
        "warmup": warmup, "ms_per_step": round(r["ms"] / steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8 x e2m1 -> int32 block sums, fp64 acc",
        "data": "synthetic (seeded SplitMix64; random MXFP4 weights, N(0,1) activations)",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "I": w.I, "E": w.E, "k": w.k,
                   "seed": w.seed, "parallelism": f"replicas x{N}",
                   "touched_experts": r["touched"],
                   "l2": "inputs larger than L2: %.2f GB of expert weights streamed per step "
                         "vs 126 MB L2" % (r["alg_bytes_step"] / 1e9)},
        "roofline": roofline_hbm(r, peaks, profiled_traffic(f"k_gemv_{w.name}.md")),
        "e2e": {"value": round(whole_job_value(N, w.T, steps, r["e2e_ms"]), 1), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
        # the GEMM phases, timed in the second region (with events between the
        # launches, which also end their overlap: step_ms there is the layer
        # time with that overlap lost)
        "kernel_ms_per_step": {"w1": round(r["w1_ms"] / steps, 5), "w2": round(r["w2_ms"] / steps, 5),
                               "step_ms_with_phase_events": round(r["ms_events"] / steps, 5)},
        "router_projection": router_line(r),
    }
    if not a.no_decode_t64:
        # the larger decode batch (most experts get 1-3 rows): same HBM roofline
        dw = synth.WORKLOADS["decode_T64"]
        dsteps = max(3, min(500, steps // 4))
        rd = run_gpu_workload(dw.name, dsteps, max(3, warmup), dist, want_e2e=False, want_clocks=False)
        out["decode_T64"] = {
            "workload": dw.name, "T": dw.T, "steps": dsteps,
            "value": round(whole_job_value(N, dw.T, dsteps, rd["ms"]), 1), "unit": "tokens/s",
            "ms_per_step": round(rd["ms"] / dsteps, 5), "touched_experts": rd["touched"],
            "ms_per_step_with_phase_events": round(rd["ms_events"] / dsteps, 5),
            # (at 64 tokens experts with two or more rows take the tensor cores)
            "roofline": roofline_hbm(rd, peaks, profiled_traffic(f"k_tc_gemm_{dw.name}.md"),
                                     kernel="W1 and W2 phases, two launches each: k_gemv for one-row experts, "
                                            "then the tensor cores for experts with two or more rows "
                                            "(W1 k_tc_gemm_tn, W2 k_tc_gemm decode configuration)",
                                     per_phase=2),
        }
    if not a.no_prefill:
        # prefill lines (tensor-core path): the prefill chunk, the skewed
        # prefill as specified (one expert takes almost every row) and its
        # labelled milder variant (c = 1.25: empty experts, thousands of rows on
        # the top experts, many small experts on the streaming GEMM)
        fp8_peak = 2.0 * peaks["bf16_tflops"]
        # ~0.2 s of timed steps per line, so that the clocks sampled under load
        # say whether the tensor-core GEMM ran at the burst or the power-capped
        # sustained clock
        # two regimes per line: a short run (20 / 5 / 5 steps) against the burst
        # peak, and ~0.2 s of steps with clocks sampled against the sustained
        # (power-capped) peak
        for key, pname, cap, long_cap in (("prefill", a.prefill_workload, 20, 150),
                                          ("prefill_skew", "prefill_skew_T16384", 5, 50),
                                          ("prefill_skew1.25", "prefill_skew1.25_T16384", 5, 40)):
            if key.startswith("prefill_skew") and a.no_skew:
                continue
            pw = synth.WORKLOADS[pname]
            psteps = max(3, min(cap, steps // 100))
            rp = run_gpu_workload(pw.name, psteps, 3, dist, want_e2e=False, want_clocks=False)
            lsteps = max(3, min(long_cap, steps // 10))
            rl = run_gpu_workload(pw.name, lsteps, 3, dist, want_e2e=False, want_clocks=rank0)
            ptf = rp["alg_flop_step"] * psteps / (rp["gemm_ms"] * 1e-3) / 1e12
            ltf = rl["alg_flop_step"] * lsteps / (rl["gemm_ms"] * 1e-3) / 1e12
            sus = 2.0 * peaks["bf16_tflops_sustained"] if peaks.get("bf16_tflops_sustained") else None
            out[key] = {
                "workload": pw.name, "T": pw.T, "steps": psteps,
                "value": round(whole_job_value(N, pw.T, psteps, rp["ms"]), 1), "unit": "tokens/s",
                "ms_per_step": round(rp["ms"] / psteps, 4),
                "gemm_ms_per_step": round(rp["gemm_ms"] / psteps, 4),
                "touched_experts": rp["touched"],
                "roofline": {"bound": "tensor",
                             "kernel": "W1 and W2 grouped GEMM launches (tcgen05 kind::mxf4 block-scaled: "
                                       "k_tc_gemm_tn token-major for W1, k_tc_gemm weight-major for W2; "
                                       "k_gemv for one-row experts)",
                             "achieved": round(ptf, 2), "unit": "TFLOP/s", "peak": fp8_peak,
                             "frac": round(ptf / fp8_peak, 5),
                             "peak_source": peaks["source"] + " bf16 burst x 2 (fp8/bf16 nominal ratio); "
                                            "a short run of steps",
                             # the INT8 operand enters the FP4 MMA as three exact digit planes,
                             # so the tensor pipe issues 3x the algorithmic work at the FP4 rate
                             "mma_issued_tflops": round(3 * ptf, 2),
                             "mma_peak_fp4": 4.0 * peaks["bf16_tflops"],
                             "mma_frac_fp4": round(3 * ptf / (4.0 * peaks["bf16_tflops"]), 5),
                             "hbm_achieved_gbs": round(rp["alg_bytes_step"] * psteps / (rp["gemm_ms"] * 1e-3) / 1e9, 1),
                             "traffic": profiled_traffic(f"k_tc_gemm_{pw.name}.md")},
                # (both from the region with events around the GEMM phases)
                "non_gemm_frac": round(1.0 - rp["gemm_ms"] / rp["ms_events"], 4),
                "ms_per_step_with_phase_events": round(rp["ms_events"] / psteps, 4),
                "sustained": {"steps": lsteps, "ms_per_step": round(rl["ms"] / lsteps, 4),
                              "value": round(whole_job_value(N, pw.T, lsteps, rl["ms"]), 1),
                              "gemm_tflops": round(ltf, 2), "peak": sus,
                              "frac": round(ltf / sus, 5) if sus else None,
                              "peak_source": peaks["source"] + " bf16 sustained x 2", "clocks": rl["clocks"]},
                "router_projection": router_line(rp),
                "tc_pair": moe.moe_get_option(moe.MOE_OPT_TC_PAIR),
                "tc_a_tmem": moe.moe_get_option(moe.MOE_OPT_TC_A_TMEM),
                "tc_form": moe.moe_get_option(moe.MOE_OPT_TC_FORM),
            }
    if not a.no_fp8:
        out["fp8_dense"] = [run_fp8_dense(n, max(3, min(cap, steps // 2)), 5, dist, peaks, want_clocks=rank0)
                            for n, cap in (("dense_T4604", 400), ("dense_T8", 2000))]
    if rank0 and N == 1 and not a.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(a.workload, a.cpu_seconds)
    if rank0:
        print(json.dumps(out), flush=True)
    dist.close()


def main_reference(a):
    """The oracle, timed on this host's cores, on the same workload and metric."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    steps = a.steps if a.steps is not None else 5
    warmup = a.warmup if a.warmup is not None else 1
    w = synth.WORKLOADS[a.workload]
    d = synth.make(w)
    # each step is a bounded sample: the layer for one token of the batch
    def step(i):
        oracle.forward_tokens(d["x"], d["logits"], d["w1_codes"], d["w1_scales"], d["w2_codes"],
                              d["w2_scales"], w.k, [i % w.T])
    for i in range(warmup):
        step(i)
    t0 = time.time()
    for i in range(steps):
        step(i)
    dt = time.time() - t0
    value = steps / dt
    out = {"metric": "routed-MoE layer tokens/s (T=8 decode, T=4604 prefill); % HBM / TC roofline",
           "value": round(value, 4), "unit": "tokens/s", "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
           "steps": steps, "warmup": warmup, "ms_per_step": round(dt * 1e3 / steps, 2),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic (seeded SplitMix64)", "impl": "reference",
           "config": {"workload": w.name, "T": w.T, "H": w.H, "I": w.I, "E": w.E, "k": w.k},
           "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": oracle.nthreads(),
                            "kind": "oracle",
                            "sample": f"each step: the whole layer for one token of {w.name}"},
           "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
