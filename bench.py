#!/usr/bin/env python
"""Benchmark of the paged-KV GQA attention engine on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one ``pa_run`` (device scheduler + attention kernel + split merge
when used) over one batch of the headline workload: Llama-3.1-8B-shaped paged
decode, B=256, 32 query / 8 KV heads, head_dim 128, page size 16, seq_lens
uniform in [1024, 2048], one query token per request, shuffled pool 25% larger
than needed, N(0,1) bf16 inputs drawn on the GPU from a seeded generator.
Inputs are resident in HBM when the timed region starts; the 1.6 GB of KV is
far larger than the 126 MB L2, so no flush is needed between steps.

Rank 0 prints one JSON line.  ``value`` is the decode KV-read rate (K and V
bytes the step must read, divided by the device time of the step, summed over
ranks).  ``roofline`` relates the attention kernel's algorithmic bytes per
launch to its measured duration and to the measured HBM copy bandwidth;
``per_config`` adds the other workloads (causal prefill TFLOP/s, the unified
mixed batch, the long-context GQA-32 split-KV decode, the tiny decode).
``cpu_baseline`` times the CPU oracle on the host cores.  ``--impl reference``
times only the CPU oracle (the reference arm of this build).

With N > 1 (torchrun) every rank runs an independent replica of the workload
on its own GPU (the attention path has no exchange step): scaling is weak.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_gqa_fmha_b200 import workloads as W  # noqa: E402

METRIC = "decode KV-read GB/s and prefill TFLOP/s on 1 B200, as % of roofline"
HEADLINE = "llama8b_decode"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ----------------------------------------------------------------------------- accounting
def work_counts(w) -> dict:
    """Algorithmic traffic and FLOPs of one pass (what the method must touch):
    K and V of every visible key once per KV head (GQA packing shares them
    across the G query heads), Q, O and LSE once, the live page-table entries,
    seq_lens and cu_q_lens; FLOPs count only visible (query, key) pairs."""
    q = np.array(w["q_lens"], dtype=np.int64)
    kv = np.array(w["kv_lens"], dtype=np.int64)
    Hq, Hkv, D, ps = w["Hq"], w["Hkv"], w["D"], w["ps"]
    T = int(q.sum())
    kv_bytes = int(kv.sum()) * Hkv * D * 2 * 2
    q_bytes = T * Hq * D * 2
    o_bytes = T * Hq * D * 2
    lse_bytes = T * Hq * 4
    meta = int(np.sum(-(-kv // ps))) * 4 + len(kv) * 4 + (len(kv) + 1) * 4
    pairs = q * (kv - q) + q * (q + 1) // 2
    flops = 4 * D * Hq * int(pairs.sum())
    return dict(kv_bytes=kv_bytes, bytes=kv_bytes + q_bytes + o_bytes + lse_bytes + meta,
                flops=flops, T=T)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "paged_kv_gqa_fmha_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str):
    """DRAM bytes per attention-kernel launch from the committed ncu summary,
    or None when it is missing or was taken on other kernel sources."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(workload)
    if not e or e.get("kernel_sources") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = os.path.join("/tmp", "pa_clocks_%d_%d.csv" % (os.getpid(), device_index))
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            ident = str(device_index)
        self.ident = ident

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", self.ident], stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- runs
def make_plan(w, num_splits=0):
    from paged_kv_gqa_fmha_b200 import Plan
    return Plan(w["B"], w["Hq"], w["Hkv"], w["D"], w["ps"], w["C"], scale=w["scale"],
                num_pages=w["P"], num_splits=num_splits)


def run_args(w):
    decode_only = w["spec"].decode_only
    return (w["q"], w["k_pool"], w["v_pool"], w["page_table"], w["seq_lens"],
            None if decode_only else w["cu_q_lens"])


def time_headline(w, plan, steps, warmup, dist_on):
    """K steps bracketed by barrier + synchronize, one event pair around them.
    The attention kernel's own duration is measured in a second pass with the
    plan's per-launch event pairs (kept out of the timed steps: an event between
    the scheduler and the attention kernel would stop their launch overlap)."""
    args = run_args(w)
    out = torch.empty_like(w["q"])
    lse = torch.empty(w["T"], w["Hq"], device=w["q"].device)
    for _ in range(warmup):
        plan.run(*args, out=out, lse=lse)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        plan.run(*args, out=out, lse=lse)
    e1.record(stream)
    torch.cuda.synchronize()
    if dist_on:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    n_prof = min(steps, 500)
    plan.profile_start(n_prof)
    for _ in range(n_prof):
        plan.run(*args, out=out, lse=lse)
    attn_ms, n_rec, per_run = plan.profile_read()
    status = plan.status()
    return ms, attn_ms / max(1, n_rec), per_run, status


def time_config(w, steps, warmup, flush):
    """Per-step event pairs (L2 flushed between steps for small working sets)."""
    plan = make_plan(w)
    args = run_args(w)
    out = torch.empty_like(w["q"])
    lse = torch.empty(w["T"], w["Hq"], device=w["q"].device)
    scratch = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=w["q"].device) \
        if flush else None
    for _ in range(warmup):
        plan.run(*args, out=out, lse=lse)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    tot = 0.0
    for _ in range(steps):
        if scratch is not None:
            scratch.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        plan.run(*args, out=out, lse=lse)
        e1.record(stream)
        e1.synchronize()
        tot += e0.elapsed_time(e1)
    plan.profile_start(steps)
    for _ in range(steps):
        if scratch is not None:
            scratch.fill_(1.0)
        plan.run(*args, out=out, lse=lse)
    attn_ms, n_rec, per_run = plan.profile_read()
    st = plan.status()
    plan.close()
    return tot / steps, attn_ms / max(1, n_rec), st


def time_e2e(w, steps, warmup):
    """Same metric through the public API with host buffers: every step copies
    the inputs from pinned host memory to the device, runs, and copies O and
    LSE back; one event pair around all steps."""
    plan = make_plan(w)
    names = ["q", "k_pool", "v_pool", "page_table", "seq_lens"]
    if not w["spec"].decode_only:
        names.append("cu_q_lens")
    host = {k: w[k].cpu().pin_memory() for k in names}
    dev = {k: torch.empty_like(w[k]) for k in names}
    out = torch.empty_like(w["q"])
    lse = torch.empty(w["T"], w["Hq"], device=w["q"].device)
    out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    lse_h = torch.empty(lse.shape, dtype=lse.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size() + lse_h.numel() * lse_h.element_size()

    def step():
        for k in names:
            dev[k].copy_(host[k], non_blocking=True)
        plan.run(dev["q"], dev["k_pool"], dev["v_pool"], dev["page_table"], dev["seq_lens"],
                 dev.get("cu_q_lens"), out=out, lse=lse)
        out_h.copy_(out, non_blocking=True)
        lse_h.copy_(lse, non_blocking=True)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    plan.close()
    del host, dev
    return ms, h2d, d2h


def cpu_oracle_rate(w, target_s=10.0, max_reps=50, request_subset=None):
    """The CPU oracle, as it stands, on the host cores: the whole workload (or
    a subset of its requests) repeated until about ``target_s`` seconds."""
    from oracle import oracle as O
    q = W.bf16_bits(w["q"])
    k = W.bf16_bits(w["k_pool"])
    v = W.bf16_bits(w["v_pool"])
    table = w["page_table_cpu"].numpy()
    seq = w["seq_lens_cpu"].numpy()
    cu = w["cu_q_lens_cpu"].numpy()
    B = w["B"]
    nb = B if request_subset is None else min(B, request_subset)
    cu_s = cu[: nb + 1]
    q_s = q[: int(cu_s[-1])]
    threads = O.default_threads()
    kv_bytes = int(seq[:nb].sum()) * w["Hkv"] * w["D"] * 4
    O.paged_attention(q_s[:1], k, v, table[:1], seq[:1], cu[:2] * 0 + np.array([0, 1]),
                      w["scale"], nthreads=threads)   # load + build outside the timing
    reps, t0 = 0, time.time()
    while reps < max_reps:
        O.paged_attention(q_s, k, v, table[:nb], seq[:nb], cu_s, w["scale"], nthreads=threads)
        reps += 1
        if time.time() - t0 >= target_s:
            break
    dt = time.time() - t0
    return dict(value=kv_bytes * reps / dt / 1e9, unit="GB/s", cores=threads, kind="oracle",
                sample="%d of %d requests of %s (all %d query heads, full KV), %d repetitions "
                       "in %.1f s" % (nb, B, w["spec"].name, w["Hq"], reps, dt),
                seconds=dt)


# Requests each workload's CPU-oracle sample takes: whole workloads where one
# pass takes seconds, otherwise a subset with the workload's own mix (the
# causal prefill's requests are all alike; the mixed batch keeps its ratio of
# one prefill request to 31 decode requests).
CPU_SAMPLE = {
    "tiny_decode": None,
    "llama8b_decode": None,
    "llama8b_causal_prefill": [0],
    "unified_mixed": [0] + list(range(8, 39)),
    "long_gqa32_decode": None,
}


def cpu_oracle_config(w, reqs=None, target_s=4.0, max_reps=200):
    """The CPU oracle, as it stands, on all host cores over the requests
    ``reqs`` of the workload (all of them when None), repeated until about
    ``target_s`` seconds.  Rates use the same algorithmic counts as the GPU
    rows; ``est_seconds_full`` scales the per-pass time to the whole workload
    by FLOPs (the oracle's cost is one dot product over D per visible
    (query, key) pair and one weighted V row)."""
    from oracle import oracle as O
    B = w["B"]
    idx = list(range(B)) if reqs is None else [b for b in reqs if b < B]
    cu = w["cu_q_lens_cpu"].numpy()
    q_all = W.bf16_bits(w["q"])
    q = np.concatenate([q_all[cu[b]:cu[b + 1]] for b in idx], 0)
    q_lens = [int(cu[b + 1] - cu[b]) for b in idx]
    cu_s = np.zeros(len(idx) + 1, dtype=np.int32)
    cu_s[1:] = np.cumsum(q_lens)
    table = w["page_table_cpu"].numpy()[idx]
    seq = w["seq_lens_cpu"].numpy()[idx]
    k = W.bf16_bits(w["k_pool"])
    v = W.bf16_bits(w["v_pool"])
    threads = O.default_threads()
    sub = dict(q_lens=q_lens, kv_lens=[int(x) for x in seq], Hq=w["Hq"], Hkv=w["Hkv"],
               D=w["D"], ps=w["ps"])
    c_sub, c_all = work_counts(sub), work_counts(w)
    O.paged_attention(q[:1], k, v, table[:1], seq[:1], np.array([0, 1], np.int32),
                      w["scale"], nthreads=threads)   # load + build outside the timing
    reps, t0 = 0, time.time()
    while reps < max_reps:
        O.paged_attention(q, k, v, table, seq, cu_s, w["scale"], nthreads=threads)
        reps += 1
        if time.time() - t0 >= target_s:
            break
    dt = (time.time() - t0) / reps
    return {"kind": "oracle", "cores": threads, "seconds_per_pass": dt,
            "GBps": c_sub["bytes"] / dt / 1e9, "TFLOPs": c_sub["flops"] / dt / 1e12,
            "est_seconds_full": dt * c_all["flops"] / max(1, c_sub["flops"]),
            "sample": "%d of %d requests (all %d query heads, full KV), %d passes"
                      % (len(idx), B, w["Hq"], reps)}


# ----------------------------------------------------------------------------- main
def config_desc(w) -> str:
    q, kv = w["q_lens"], w["kv_lens"]
    return ("%s: B=%d, Hq=%d, Hkv=%d, D=%d, page_size=%d, capacity=%d, pool=%d pages, "
            "q_len %d..%d, kv_len %d..%d, bf16 N(0,1), seed %d"
            % (w["spec"].name, w["B"], w["Hq"], w["Hkv"], w["D"], w["ps"], w["C"], w["P"],
               min(q), max(q), min(kv), max(kv), w["seed"]))


def max_over_ranks(ms: float, device) -> float:
    """Device time of the slowest rank (the whole job ends when it does); the
    local time when no process group is running."""
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def replica_value(kv_bytes_per_step: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job K+V GB/s: every rank runs `steps` steps of its own replica of
    the workload, and the job takes the slowest rank's time."""
    return kv_bytes_per_step * world * steps / (ms_max * 1e-3) / 1e9


def attention_kernel_name(w, decode_only: bool) -> str:
    """The kernel a default plan runs for this workload: decode-only head_dim
    128 runs (no cu_q_lens) go to the keys-as-M decode kernel, whose rows
    template is G rounded up to a power of two (at least 4)."""
    G = w["Hq"] // w["Hkv"]
    if decode_only and w["D"] == 128 and G <= 32:
        rr = 4
        while rr < G:
            rr *= 2
        return "pa_decode_kernel<128, %d, false>" % rr
    return "pa_attention_kernel<%d, false>" % w["D"]


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="skip per-config, e2e and CPU legs")
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(W.CONFIGS),
                    help="workload of the timed steps (default: the headline decode)")
    ap.add_argument("--kv-fp8", action="store_true",
                    help="E4M3 pools (implies --no-extra): the metric then counts one byte "
                         "per K/V element")
    args = ap.parse_args()
    if args.kv_fp8:
        args.no_extra = True
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    spec = W.CONFIGS[args.workload]
    peaks, peak_kind = load_peaks()

    if args.impl == "reference":
        if rank != 0:
            return
        w = W.generate(spec, W.default_seed(args.workload),
                       device="cuda" if torch.cuda.is_available() else "cpu")
        wv = w
        calib = cpu_oracle_rate(wv, target_s=0.5, max_reps=1, request_subset=16)
        per_req_s = calib["seconds"] / 16
        budget = 120.0 / max(1, args.steps + args.warmup)       # seconds per step
        n_req = max(1, min(w["B"], int(budget / max(per_req_s, 1e-6))))
        from oracle import oracle as O
        q = W.bf16_bits(wv["q"]); k = W.bf16_bits(wv["k_pool"]); v = W.bf16_bits(wv["v_pool"])
        table = w["page_table_cpu"].numpy(); seq = w["seq_lens_cpu"].numpy()
        cu = w["cu_q_lens_cpu"].numpy()[: n_req + 1]
        for _ in range(args.warmup):
            O.paged_attention(q[:n_req], k, v, table[:n_req], seq[:n_req], cu, w["scale"])
        t0 = time.time()
        for _ in range(args.steps):
            O.paged_attention(q[:n_req], k, v, table[:n_req], seq[:n_req], cu, w["scale"])
        dt = time.time() - t0
        kv_bytes = int(seq[:n_req].sum()) * w["Hkv"] * w["D"] * 4
        value = kv_bytes * args.steps / dt / 1e9
        line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "config": {"workload": config_desc(w), "sample": "first %d requests" % n_req},
                "cpu_baseline": {"value": value, "unit": "GB/s", "cores": O.default_threads(),
                                 "kind": "oracle",
                                 "sample": "first %d of %d requests per step" % (n_req, w["B"])},
                "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dist_on = world > 1
    torch.cuda.set_device(local)
    if dist_on:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    w = W.generate(spec, W.default_seed(args.workload), device="cuda")
    counts = work_counts(w)
    plan = make_plan(w)
    kernel = attention_kernel_name(w, spec.decode_only)
    if args.kv_fp8:
        to_fp8_pools(w)
        plan.set_kv_fp8(True, FP8_DESCALE, FP8_DESCALE)
        counts["bytes"] -= counts["kv_bytes"] // 2
        counts["kv_bytes"] //= 2
        kernel = ("pa_decode_kernel<%d, %d, true>" % (
            w["D"], max(4, 1 << (w["Hq"] // w["Hkv"] - 1).bit_length()))
            if spec.decode_only else "pa_attention_kernel<%d, true>" % w["D"])
    clocks = ClockSampler(local)
    clocks.start()
    ms, attn_ms, per_run, status = time_headline(w, plan, args.steps, args.warmup, dist_on)
    clk = clocks.stop()
    plan.close()
    ms_max = max_over_ranks(ms, "cuda")
    ms_step = ms_max / args.steps
    value = replica_value(counts["kv_bytes"], world, args.steps, ms_max)

    achieved = counts["bytes"] / (attn_ms * 1e-3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    traffic = ncu_traffic(args.workload + ("_fp8" if args.kv_fp8 else ""))
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 KV, bf16 q/out, fp16 MMAs" if args.kv_fp8 else "bf16",
        "data": "synthetic",
        "config": {"workload": config_desc(w) + (", E4M3 pools" if args.kv_fp8 else ""),
                   "l2": "inputs larger than L2 (%.2f GB of KV), no flush" % (counts["kv_bytes"] / 1e9),
                   "value_counts": "K+V bytes of every visible key per KV head",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": kernel,
                     "algorithmic_bytes_per_launch": counts["bytes"],
                     "kernel_ms": attn_ms, "peak_source": "%s hbm_gbs" % peak_kind},
        "gpu_launches": per_run * args.steps,
        "status_word": status,
        "clocks": clk,
    }

    if rank == 0 and world == 1 and not args.no_extra:
        line["per_config"] = per_config(peaks)
    if not args.no_extra:
        # every rank copies, runs and reads back its own replica through the
        # public API; the job takes the slowest rank, and the byte counts are
        # the whole job's (every rank's copies)
        e_ms, h2d, d2h = time_e2e(w, steps=5, warmup=2)
        e_max = max_over_ranks(e_ms, "cuda")
        line["e2e"] = {"value": replica_value(counts["kv_bytes"], world, 1, e_max),
                       "unit": "GB/s", "h2d_bytes_per_step": h2d * world,
                       "d2h_bytes_per_step": d2h * world, "ms_per_step": e_max}
    if rank == 0 and world == 1 and not args.no_extra:
        line["cpu_baseline"] = {k: v for k, v in cpu_oracle_rate(w).items() if k != "seconds"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist_on:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def per_config(peaks, cpu=True):
    res = {}
    bw = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    for name in W.CONFIGS:
        w = W.generate(W.CONFIGS[name], W.default_seed(name), device="cuda")
        c = work_counts(w)
        flush = c["bytes"] < 2 * L2_BYTES
        steps = 20 if name != "tiny_decode" else 50
        ms, attn_ms, st = time_config(w, steps=steps, warmup=5, flush=flush)
        r = {"ms_per_step": ms, "attn_kernel_ms": attn_ms, "status_word": st,
             "algorithmic_bytes": c["bytes"], "kv_bytes": c["kv_bytes"], "flops": c["flops"],
             "l2": "flushed between steps" if flush else "inputs larger than L2"}
        gbs = c["bytes"] / (attn_ms * 1e-3) / 1e9
        tfs = c["flops"] / (attn_ms * 1e-3) / 1e12
        r["kernel_GBps"] = gbs
        r["kernel_TFLOPs"] = tfs
        r["hbm_frac"] = gbs / bw
        r["tensor_frac"] = tfs / tf
        r["step_KV_GBps"] = c["kv_bytes"] / (ms * 1e-3) / 1e9
        r["step_TFLOPs"] = c["flops"] / (ms * 1e-3) / 1e12
        t_bw = c["bytes"] / (bw * 1e9)
        t_fl = c["flops"] / (tf * 1e12)
        r["roofline_ms_max_form"] = max(t_bw, t_fl) * 1e3
        r["roofline_frac_max_form"] = max(t_bw, t_fl) / (attn_ms * 1e-3)
        if cpu:
            r["cpu_baseline"] = cpu_oracle_config(w, CPU_SAMPLE.get(name))
        res[name] = r
        del w
        torch.cuda.empty_cache()
    res["kv_append"] = kv_append_rates(bw)
    res["kv_fp8"] = kv_fp8_rates(bw, tf)
    return res


FP8_DESCALE = 0.25


def to_fp8_pools(w):
    """Replace the workload's bf16 pools by E4M3 codes of 4x their values
    (round to nearest on the device, in chunks that bound the fp32 temporaries);
    read back with descales FP8_DESCALE the values are the bf16 ones rounded to
    E4M3."""
    for key in ("k_pool", "v_pool"):
        src = w[key]
        dst = torch.empty(src.shape, dtype=torch.uint8, device=src.device)
        for a in range(0, src.shape[0], 4096):
            dst[a:a + 4096] = (src[a:a + 4096].float() * 4).to(torch.float8_e4m3fn).view(
                torch.uint8)
        w[key] = dst
        del src
    torch.cuda.empty_cache()


def kv_fp8_rates(bw, tf):
    """Every non-tiny workload over E4M3 pools (pa_set_kv_fp8): the bf16 pools
    are quantised on the device (x4, round to nearest E4M3) and read back with
    descales 0.25.  Decode-only workloads run on the kernel a default plan
    picks (the E4M3 decode kernel at head_dim 128, the one-stage kernel's E4M3
    variant at 256); in prefill and mixed batches the requests of two or more
    query blocks are widened once into bf16 scratch pages (pa_widen_kernel)
    and run on the bf16 one-stage kernel, rows of one query token on the E4M3
    decode kernel (head_dim 128) and the rest on the one-stage kernel's E4M3
    variant; the time covers all of these launches.  Bytes
    per launch = the bf16 formula with K and V at one byte per element;
    per-launch CUDA events (the plan's profile pairs) over 20 launches, each
    synchronised, after 5 warm-up launches (pools larger than L2)."""
    out = {}
    for name in ("llama8b_decode", "llama8b_causal_prefill", "unified_mixed",
                 "long_gqa32_decode"):
        spec = W.CONFIGS[name]
        w = W.generate(spec, W.default_seed(name), device="cuda")
        c = work_counts(w)
        to_fp8_pools(w)
        plan = make_plan(w)
        plan.set_kv_fp8(True, FP8_DESCALE, FP8_DESCALE)
        args = (w["q"], w["k_pool"], w["v_pool"], w["page_table"], w["seq_lens"],
                None if spec.decode_only else w["cu_q_lens"])
        for _ in range(5):
            plan.run(*args)
        torch.cuda.synchronize()
        plan.profile_start(20)
        for _ in range(20):
            plan.run(*args)
            torch.cuda.synchronize()
        attn_ms, n_rec, _ = plan.profile_read()
        ms = attn_ms / max(1, n_rec)
        nbytes = c["bytes"] - c["kv_bytes"] // 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        tfs = c["flops"] / (ms * 1e-3) / 1e12
        G = w["Hq"] // w["Hkv"]
        if spec.decode_only:
            kernel = ("pa_decode_kernel<%d, %d, true>" % (w["D"], max(4, 1 << (G - 1).bit_length()))
                      if w["D"] == 128 else "pa_attention_kernel<%d, true>" % w["D"])
        else:
            kernel = ("pa_widen_kernel + pa_attention_kernel<{0}, false> (widened requests) + "
                      "pa_attention_kernel<{0}, true>".format(w["D"]))
            if w["D"] == 128 and G <= 32:
                kernel += " + pa_decode_kernel<128, %d, true> (one-token rows)" % max(
                    4, 1 << (G - 1).bit_length())
        out[name] = {"attn_kernel_ms": ms, "algorithmic_bytes": nbytes, "flops": c["flops"],
                     "kernel_GBps": gbs, "kernel_TFLOPs": tfs, "hbm_frac": gbs / bw,
                     "tensor_frac": tfs / tf, "status_word": plan.status(), "kernel": kernel}
        plan.close()
        del w
        torch.cuda.empty_cache()
    return out


def kv_append_rates(bw):
    """pa_append_kv on the K/V shapes of the prefill and decode workloads: new
    rows drawn on the device, written into a shuffled pool.  Bytes per launch =
    read + write of K and V rows (4 * T * Hkv * D * 2); CUDA events around 20
    launches after 5 warm-up launches (rows and pools larger than L2 for the
    prefill shape; the decode shape is latency-bound)."""
    out = {}
    for name in ("llama8b_causal_prefill", "llama8b_decode"):
        w = W.generate(W.CONFIGS[name], W.default_seed(name), device="cuda")
        T = w["q"].shape[0]
        g = torch.Generator(device="cuda")
        g.manual_seed(7)
        k_new = torch.randn((T, w["Hkv"], w["D"]), generator=g, device="cuda").to(torch.bfloat16)
        v_new = torch.randn((T, w["Hkv"], w["D"]), generator=g, device="cuda").to(torch.bfloat16)
        plan = make_plan(w)
        cu = None if W.CONFIGS[name].decode_only else w["cu_q_lens"]
        args = (k_new, v_new, w["k_pool"], w["v_pool"], w["page_table"], w["seq_lens"], cu)
        for _ in range(5):
            plan.append_kv(*args)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(20):
            plan.append_kv(*args)
        e1.record()
        torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / 20
        nbytes = 4 * T * w["Hkv"] * w["D"] * 2
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"tokens": T, "kernel_ms": ms, "bytes": nbytes, "kernel_GBps": gbs,
                     "hbm_frac": gbs / bw, "status_word": plan.status()}
        plan.close()
        del w, k_new, v_new
        torch.cuda.empty_cache()
    return out


if __name__ == "__main__":
    main()
