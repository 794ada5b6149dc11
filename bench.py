#!/usr/bin/env python
"""Benchmark of the batched speculative-sampling verification step.

One step = one verification call over one batch (statistics, acceptance scan,
residual / bonus draw for every sequence).  Default workload: the multi-branch
batch, 32 sequences x 8 candidate branches = 256 rows, gamma = 5, V = 152064,
bf16 logits, T = 1 (the largest of the benchmark configurations with
V >= 32000; its 856 MB of logits exceed the 126 MB L2, so no flush is needed).

Metric: verified positions per second (B * gamma per step, summed over all
ranks) and the achieved HBM bandwidth of the fused kernel, algorithmic bytes =
logits read once = B (2 gamma + 1) V * sizeof(logit).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload multibranch|b64_g8_v128256|b8_g3_v32000|char_level]

For the multi-branch batch the same positions are also timed through the
shared-row entry point (each distinct target/draft row once, plus row maps),
reported under "shared_rows".  The fold gate (relative hidden-state difference
per branch and position, provenance, packing of the rows to recompute) is
timed on 128 sequences x 8 branches x 32 positions x 4096 bf16 hidden states,
reported under "specfold_gate".  The sampling-variant entry point (greedy;
top-k 50 with top-p 0.9; top-p 0.9 alone; top-k 2000 alone) is timed on the
same batch under "sampling_variants", and the step fused with a 128256 x 4096
LM head on tensor cores (64 sequences, gamma 8) under "lmhead_fused".

N > 1 runs under torch.distributed.run, one rank per GPU: every rank verifies
its own batch (weak scaling, no data-path collective); the extra measurements
(shared rows, sampling variants, fold gate, LM-head-fused step) run at N = 1
only.  ``--impl reference``
times the CPU oracle on the host cores on a bounded sample of the workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from speculative_decoding_verification_90_b200 import dist as svdist  # noqa: E402
from speculative_decoding_verification_90_b200 import workloads  # noqa: E402

METRIC = "verified positions/s and achieved HBM GB/s vs B200 peak (spec-verify, 1 GPU)"
UNIT = "positions/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0
# the source of the kernel whose DRAM traffic the committed ncu summary records
KERNEL_SOURCES = [
    "speculative_decoding_verification_90_b200/csrc/verify_kernel.cuh",
]


# sampling-variant settings timed by the bench: name -> (temperature, top_k, top_p);
# None = the workload's temperature
SAMPLING_SETTINGS = {"greedy": (0.0, 0, 1.0), "top_k50_top_p0.9": (None, 50, 0.9),
                     "top_p0.9": (None, 0, 0.9), "top_k2000": (None, 2000, 1.0)}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="multibranch", choices=sorted(workloads.REGISTRY))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--slices", type=int, default=0, help="override blocks per position")
    ap.add_argument("--threads", type=int, default=0, help="override threads per CTA")
    ap.add_argument("--draw-slices", type=int, default=0, help="override draw blocks per sequence")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-shared-rows", action="store_true",
                    help="skip the timing of the shared-row entry point (multibranch)")
    ap.add_argument("--fused", action="store_true",
                    help="time the headline step in the single-launch form (specverify_set_fused)")
    ap.add_argument("--no-single-launch", action="store_true",
                    help="skip the extra timing of the single-launch form on the bench batch")
    ap.add_argument("--no-sampling", action="store_true",
                    help="skip the timing of the sampling variants")
    ap.add_argument("--sampling", default=None,
                    help="comma-separated sampling settings to time (" + ", ".join(SAMPLING_SETTINGS)
                         + "; default: all)")
    ap.add_argument("--no-lmhead", action="store_true",
                    help="skip the timing of the LM-head-fused step (64 x 8, V 128256, d 4096)")
    ap.add_argument("--no-gate", action="store_true",
                    help="skip the timing of the fold gate (128 x 8 branches, 32 x 4096 bf16)")
    ap.add_argument("--oracle-table", action="store_true",
                    help="with --impl reference: time the CPU oracle on every benchmark "
                         "configuration at one thread and at all host threads (bounded samples)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other benchmark configurations (64 x 8 at V 128256, 8 x 3 at "
                         "V 32000, the char-level calls, the 60000-row exactness batch)")
    args = ap.parse_args()
    if args.sampling:
        unknown = [n for n in args.sampling.split(",") if n not in SAMPLING_SETTINGS]
        if unknown:
            ap.error(f"--sampling: unknown setting(s) {unknown}; known: {list(SAMPLING_SETTINGS)}")
    return args


# the parts of the kernel source that make up the statistics kernel
STATS_SOURCE_RANGES = [
    ("// phase 1: streaming softmax statistics", "// phase 4 helpers"),
    ("// block-level helpers", "// block-wide scan of one double"),
    ("// kernel 1: streaming statistics", "// kernel 2:"),
]


def kernel_hash() -> str:
    """Hash of the statistics kernel's code: the streaming-statistics helpers,
    the block reduction and the kernel itself."""
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel)) as f:
            text = f.read()
        for start, end in STATS_SOURCE_RANGES:
            a, b = text.find(start), text.find(end)
            h.update(text[a:b].encode() if 0 <= a < b else text.encode())
    return h.hexdigest()[:16]


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, copy burst)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier measurement on this pool)"


def profiled_traffic(workload_name: str):
    """DRAM bytes per launch from a committed ncu summary, if it matches this kernel source."""
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return None
    want = kernel_hash()
    for fn in sorted(os.listdir(d)):
        if not fn.endswith(".md"):
            continue
        text = open(os.path.join(d, fn)).read()
        w = re.search(r"^workload:\s*(\S+)", text, re.M)
        hsh = re.search(r"^kernel_source_sha256_16:\s*(\S+)", text, re.M)
        tr = re.search(r"^dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text, re.M)
        if w and hsh and tr and w.group(1) == workload_name and hsh.group(1) == want:
            return float(tr.group(1))
    return None


def make_workload(name: str, seed: int):
    return workloads.REGISTRY[name](seed=seed)


def positions_per_step(wl) -> int:
    return wl.batch * wl.gamma


# ----------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-i", str(gpu_index)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                frac = float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                rows.append({"t": ts + frac, "sm": float(parts[2]), "sm_max": float(parts[3]),
                             "power": float(parts[4]) if parts[4] not in ("[N/A]", "") else None,
                             "hw_slowdown": parts[6], "hw_thermal": parts[7],
                             "sw_thermal": parts[8], "sw_power_cap": parts[9]})
            except Exception:
                continue
        return rows


def summarize_clocks(rows, t0, t1):
    if not rows:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
    inside = [r for r in rows if t0 - 0.06 <= r["t"] <= t1 + 0.06]
    if not inside:  # timed region shorter than the sampling period: nearest sample
        inside = [min(rows, key=lambda r: abs(r["t"] - 0.5 * (t0 + t1)))]
    reasons = set()
    for r in inside:
        for key, name in (("hw_slowdown", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                          ("sw_thermal", "sw_thermal_slowdown"), ("sw_power_cap", "sw_power_cap")):
            if r[key].lower() == "active":
                reasons.add(name)
    return {"sm_mhz": float(np.median([r["sm"] for r in inside])),
            "sm_max_mhz": float(max(r["sm_max"] for r in inside)),
            "reasons": sorted(reasons), "samples": len(inside)}


# ----------------------------------------------------------------------------
# the CPU oracle (reference arm and cpu_baseline)
# ----------------------------------------------------------------------------

def time_oracle(wl, budget_s: float):
    """Oracle over the whole batch on all host cores, repeated until `budget_s`
    of CPU time is reached with at least one pass; bounded to a sample of
    sequences when one pass would take longer than the budget."""
    import oracle
    threads = os.cpu_count() or 1
    # calibrate on one sequence per thread
    n_cal = min(wl.batch, threads)
    t = time.perf_counter()
    oracle.verify(wl.target[:n_cal], wl.draft[:n_cal], wl.tokens[:n_cal], wl.u_accept[:n_cal],
                  wl.u_resample[:n_cal], wl.temperature, threads=threads)
    per_seq_wall = (time.perf_counter() - t) / max(1, math.ceil(n_cal / threads))
    seqs = wl.batch
    if per_seq_wall * math.ceil(seqs / threads) > budget_s:
        seqs = max(threads, int(budget_s / per_seq_wall) * threads)
        seqs = min(seqs, wl.batch)
    passes, elapsed = 0, 0.0
    while passes == 0 or elapsed < budget_s:
        t = time.perf_counter()
        oracle.verify(wl.target[:seqs], wl.draft[:seqs], wl.tokens[:seqs], wl.u_accept[:seqs],
                      wl.u_resample[:seqs], wl.temperature, threads=threads)
        elapsed += time.perf_counter() - t
        passes += 1
    value = passes * seqs * wl.gamma / elapsed
    sample = (f"{seqs} of {wl.batch} sequences of the workload ({seqs * wl.gamma} positions), "
              f"{passes} pass(es), {elapsed:.1f} s wall on {threads} threads")
    return value, threads, sample, elapsed / passes


def oracle_table(args):
    """Oracle positions/s on every configuration, one thread and all host
    threads, each a bounded sample (about 2 s of wall time per entry)."""
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    with open(os.path.join(ROOT, "tests", "golden", "exactness_beta.json")) as f:
        beta = json.load(f)["beta"]
    wls = {"char_level": workloads.char_level(seed=args.seed),
           "exactness": workloads.exactness(beta, seed=args.seed, batch=4096),
           "b8_g3_v32000": workloads.b8_g3_v32000(seed=args.seed),
           "b64_g8_v128256": workloads.b64_g8_v128256(seed=args.seed),
           "multibranch": workloads.multibranch(seed=args.seed)}
    out = {}
    for name, wl in wls.items():
        row = {"workload": wl.name}
        for th in (1, threads):
            n = min(wl.batch, th)
            t = time.perf_counter()
            oracle.verify(wl.target[:n], wl.draft[:n], wl.tokens[:n], wl.u_accept[:n],
                          wl.u_resample[:n], wl.temperature, threads=th)
            one = max(1e-6, time.perf_counter() - t)
            n = int(min(wl.batch, max(1, 2.0 / one) * n))
            t = time.perf_counter()
            oracle.verify(wl.target[:n], wl.draft[:n], wl.tokens[:n], wl.u_accept[:n],
                          wl.u_resample[:n], wl.temperature, threads=th)
            el = time.perf_counter() - t
            row[f"threads_{th}"] = {"positions_per_s": n * wl.gamma / el, "sequences": n,
                                    "seconds": el}
        out[name] = row
    print(json.dumps({"impl": "reference", "oracle_table": out, "cores": threads}), flush=True)
    return 0


def run_reference(args):
    rank = svdist.env_rank()[0]
    if rank != 0:
        return 0  # the CPU reference runs once, on rank 0
    if args.oracle_table:
        return oracle_table(args)
    wl = make_workload(args.workload, args.seed)
    import oracle
    oracle.build()
    threads = os.cpu_count() or 1
    # each step: a bounded sample of the workload's sequences
    per_step_budget = max(0.5, 120.0 / max(1, args.steps + args.warmup))
    n_seq = min(wl.batch, threads)
    t = time.perf_counter()
    oracle.verify(wl.target[:n_seq], wl.draft[:n_seq], wl.tokens[:n_seq], wl.u_accept[:n_seq],
                  wl.u_resample[:n_seq], wl.temperature, threads=threads)
    one = time.perf_counter() - t
    n_seq = int(min(wl.batch, max(1, per_step_budget / one) * n_seq))
    for _ in range(args.warmup):
        oracle.verify(wl.target[:n_seq], wl.draft[:n_seq], wl.tokens[:n_seq],
                      wl.u_accept[:n_seq], wl.u_resample[:n_seq], wl.temperature, threads=threads)
    t = time.perf_counter()
    for _ in range(args.steps):
        oracle.verify(wl.target[:n_seq], wl.draft[:n_seq], wl.tokens[:n_seq],
                      wl.u_accept[:n_seq], wl.u_resample[:n_seq], wl.temperature, threads=threads)
    el = time.perf_counter() - t
    value = args.steps * n_seq * wl.gamma / el
    sample = f"{n_seq} of {wl.batch} sequences per step ({n_seq * wl.gamma} positions)"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * el / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "gamma": wl.gamma, "vocab": wl.vocab,
                   "logits": wl.dtype, "temperature": wl.temperature},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, local, world = svdist.env_rank()
    if args.gpus != world and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE {world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        svdist.init("nccl", device=dev)

    from speculative_decoding_verification_90_b200.specverify import SpecVerify

    # every rank verifies its own batch (weak scaling, no data-path collective)
    wl = make_workload(args.workload, svdist.rank_seed(args.seed, rank))
    B, G, V = wl.batch, wl.gamma, wl.vocab
    step_bytes = wl.logit_bytes

    def put(a, logits):
        if logits and wl.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    # inputs larger than L2 in total: rotate copies when one batch is smaller
    n_sets = max(1, math.ceil(2 * L2_BYTES / step_bytes)) if step_bytes < 2 * L2_BYTES else 1
    n_sets = min(n_sets, 256)
    base = {"target": put(wl.target, True), "draft": put(wl.draft, True),
            "tokens": put(wl.tokens, False), "u_accept": put(wl.u_accept, False),
            "u_resample": put(wl.u_resample, False)}
    sets = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(n_sets - 1)]
    out_t = torch.empty((B, G + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((B,), dtype=torch.int32, device=dev)

    sv = SpecVerify(B, G, V, wl.dtype, local)
    if args.fused:
        sv.set_fused(True)
    if args.slices or args.threads or args.draw_slices:
        c0, t0 = sv.launch()
        sv.set_launch(args.slices or c0, args.threads or t0, args.draw_slices)
    slices, threads = sv.launch()
    sv_draw = sv.draw_slices
    kernels_per_step = sv.kernels_per_run()

    def step(i):
        s = sets[i % n_sets]
        sv.run(s["target"], s["draft"], s["tokens"], s["u_accept"], s["u_resample"],
               wl.temperature, out_t, out_n)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    st, bits = sv.status()
    if st != 0:
        raise SystemExit(f"device status {st} (bits {bits}) during warm-up")

    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local) if rank == 0 else None
    time.sleep(0.15)
    # the headline: K steps back to back as a caller runs them (nothing
    # between the launches, so each step's kernels overlap through
    # programmatic dependent launch)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ev0.record(stream)
    for i in range(args.steps):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    # the same K steps again with CUDA events on the launch stream around
    # each kernel: the per-kernel device times of the roofline (an event
    # between two kernels ends their overlap, so this pass is not the
    # headline)
    sv.profile_begin(args.steps)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    ev2, ev3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev2.record(stream)
    for i in range(args.steps):
        step(i)
    ev3.record(stream)
    torch.cuda.synchronize()
    kern = sv.profile_end()
    if world > 1:
        dist.barrier(device_ids=[local])
    time.sleep(0.12)
    rows = sampler.stop() if sampler else []
    ms = ev0.elapsed_time(ev1)
    ms_profiled = ev2.elapsed_time(ev3)
    ms_max = svdist.max_over_ranks(ms, device=dev)  # the job takes as long as its slowest rank
    stats_launch_s = kern["stats_ms"] / 1e3  # the kernel that streams every logit once

    # end to end through the host-buffer entry point (pinned host memory)
    def pinned(a, logits):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if logits and wl.dtype == "bf16"
                             else np.ascontiguousarray(a))
        if logits and wl.dtype == "bf16":
            t = t.view(torch.bfloat16)
        return t.pin_memory()

    h_in = [pinned(wl.target, True), pinned(wl.draft, True), pinned(wl.tokens, False),
            pinned(wl.u_accept, False), pinned(wl.u_resample, False)]
    h_ot = torch.empty((B, G + 1), dtype=torch.int32).pin_memory()
    h_on = torch.empty((B,), dtype=torch.int32).pin_memory()
    e2e_steps = max(1, min(args.e2e_steps, args.steps))
    sv.run_host(*h_in[:5], wl.temperature, h_ot, h_on)  # staging allocation outside the timing
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        sv.run_host(*h_in[:5], wl.temperature, h_ot, h_on)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = svdist.max_over_ranks(e0.elapsed_time(e1), device=dev)
    h2d = sum(t.numel() * t.element_size() for t in h_in)
    d2h = h_ot.numel() * 4 + h_on.numel() * 4
    st, bits = sv.status()

    # the extra measurements run at one GPU only: a scaling run times the
    # headline step (each rank would otherwise build every extra workload)
    extras = world == 1
    # the same batch under sampling variants (separate kernels)
    sampling = None
    if extras and not args.no_sampling:
        sampling = time_sampling(args, wl, sv, sets, n_sets, out_t, out_n, dev, world, local)

    # the same batch in the single-launch form (one persistent kernel)
    single = None
    if extras and not args.fused and not args.no_single_launch:
        single = time_single_launch(args, sv, step, dev, world, local)

    # the same batch through the shared-row entry point: each distinct row once
    shared = None
    if extras and wl.mapped and not args.no_shared_rows:
        shared = time_shared_rows(args, wl, sv, put, out_t, out_n, dev, world, local)
    sv.close()
    others = None if (args.no_configs or not extras) else time_other_configs(args, dev)
    gate = None if (args.no_gate or not extras) else time_gate(args, dev, world, local)
    lmh = None if (args.no_lmhead or not extras) else time_lmhead(args, dev, world, local)
    # tokens settled per step on this rank = accepted + 1 per sequence (last device step)
    emitted = int((out_n.cpu().numpy().astype(np.int64) + 1).sum())

    line = None
    if rank == 0:
        peak, peak_src = measured_peak()
        achieved = step_bytes / stats_launch_s / 1e9
        default_shape = not (args.slices or args.threads or args.draw_slices)
        traffic = profiled_traffic(wl.name) if default_shape else None
        positions = positions_per_step(wl) * world
        value = positions * args.steps / (ms_max / 1e3)
        e2e_value = positions * e2e_steps / (e2e_ms / 1e3)
        clocks = summarize_clocks(rows, t_wall0, t_wall1)
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            v, cores, sample, _ = time_oracle(wl, budget_s=12.0)
            cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl.name, "batch": B, "gamma": G, "vocab": V,
                       "logits": wl.dtype, "temperature": wl.temperature,
                       "parallelism": f"dp{world} (independent batches per GPU)",
                       "l2": ("inputs larger than L2 (%.0f MB per step, %d rotating set(s))"
                              % (step_bytes / 1e6, n_sets)),
                       "launch": {"blocks_per_row": slices, "threads": threads,
                                  "draw_blocks_per_sequence_max": sv_draw}},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                         "algorithmic_bytes_per_launch": step_bytes,
                         "kernel": ("fused_kernel (the whole step in one launch)" if args.fused
                                    else "stats_kernel (streams every logit once)")},
            "kernels_us_per_step": {"stats": 1e3 * kern["stats_ms"],
                                    "decide_and_draw": 1e3 * kern["draw_ms"],
                                    "runs": kern["runs"],
                                    "step_us_with_kernel_events": 1e3 * ms_profiled / args.steps},
            "step_hbm_gbs": step_bytes / (ms / 1e3 / args.steps) / 1e9,
            "step_frac": step_bytes / (ms / 1e3 / args.steps) / 1e9 / peak,
            "emitted_tokens_per_step": emitted,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps},
            "gpu_launches": kernels_per_step * args.steps,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "status_after": st,
        }
        if others is not None:
            line["other_configs"] = others_summary(others, peak)
        if gate is not None:
            line["specfold_gate"] = gate_summary(gate, peak)
        if lmh is not None:
            line["lmhead_fused"] = lmhead_summary(lmh)
        if sampling is not None:
            line["sampling_variants"] = {
                name: {"entry": "specverify_run_sampling", "settings": v["settings"],
                       "value": positions * args.steps / (v["ms_max"] / 1e3), "unit": UNIT,
                       "ms_per_step": v["ms_max"] / args.steps,
                       "logit_gbs": step_bytes / (v["ms_max"] / 1e3 / args.steps) / 1e9,
                       "select_us": v["select_us"],
                       "decide_and_draw_us": v["decide_and_draw_us"],
                       "status_after": v["status"]}
                for name, v in sampling.items()}
        if single is not None:
            line["single_launch"] = {
                "entry": "specverify_run with specverify_set_fused(h, 1, 0, 0, -1)",
                "value": positions * args.steps / (single["ms_max"] / 1e3), "unit": UNIT,
                "ms_per_step": single["ms_max"] / args.steps,
                "kernel_us": 1e3 * single["stats_ms"], "kernels_per_step": single["kernels"],
                "step_hbm_gbs": step_bytes / (single["ms_max"] / 1e3 / args.steps) / 1e9,
                "status_after": single["status"]}
        if shared is not None:
            sh_bytes = shared["bytes"]
            sh_ach = sh_bytes / (shared["stats_ms"] / 1e3) / 1e9
            line["shared_rows"] = {
                "entry": "specverify_run_mapped", "value": positions * args.steps
                / (shared["ms_max"] / 1e3), "unit": UNIT,
                "ms_per_step": shared["ms_max"] / args.steps,
                "distinct_row_bytes_per_step": sh_bytes,
                "stats_us": 1e3 * shared["stats_ms"], "decide_and_draw_us": 1e3 * shared["draw_ms"],
                "stats_hbm_gbs": sh_ach, "stats_frac": sh_ach / peak,
                "l2": "inputs larger than L2 (%.0f MB per step, %d rotating set(s))"
                      % (sh_bytes / 1e6, shared["sets"]),
                "status_after": shared["status"]}
    if world > 1:
        dist.barrier(device_ids=[local])
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


def _device_inputs(wl, dev):
    import torch

    def put(a, logits):
        if logits and wl.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    return {"target": put(wl.target, True), "draft": put(wl.draft, True),
            "tokens": put(wl.tokens, False), "u_accept": put(wl.u_accept, False),
            "u_resample": put(wl.u_resample, False)}


def timed_then_profiled(step, n, profile_begin, profile_end, world, local):
    """Device time of n calls of step() back to back (CUDA events on the launch
    stream around the loop only), then the same n calls again with the
    handle's per-kernel events armed: returns (ms of the first pass, the
    per-kernel means of the second).  Events between kernels end their
    overlap, so only the first pass is a timed figure."""
    import torch
    import torch.distributed as dist
    stream = torch.cuda.current_stream()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier(device_ids=[local])
    torch.cuda.synchronize()
    ev0.record(stream)
    for i in range(n):
        step(i)
    ev1.record(stream)
    torch.cuda.synchronize()
    profile_begin(n)
    for i in range(n):
        step(i)
    torch.cuda.synchronize()
    kern = profile_end()
    return ev0.elapsed_time(ev1), kern


def _time_calls(sv, sets, wl, calls, warmup, out_t, out_n, slices=None):
    """Device time of `calls` verification calls (CUDA events on the launch
    stream), cycling through the input sets; returns (ms, per-kernel means)."""
    import torch
    n = len(sets)

    def call(i):
        d = sets[i % n]
        if slices is None:
            sv.run(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                   wl.temperature, out_t, out_n)
        else:
            b0, b1 = slices[i % len(slices)]
            sv.run(d["target"][b0:b1], d["draft"][b0:b1], d["tokens"][b0:b1],
                   d["u_accept"][b0:b1], d["u_resample"][b0:b1], wl.temperature, out_t, out_n)

    for i in range(max(3, warmup)):
        call(i)
    torch.cuda.synchronize()
    return timed_then_profiled(call, calls, sv.profile_begin, sv.profile_end, 1, 0)


def _time_graph(sv, sets, wl, calls, out_t, out_n, slices=None):
    """Device time of `calls` calls captured once in a CUDA graph and replayed
    (launch-bound configurations: the host's per-call overhead is left out).
    Returns milliseconds per replay of all calls, or None if capture fails."""
    import torch
    n = len(sets)
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    try:
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for i in range(calls):
                    d = sets[i % n]
                    if slices is None:
                        sv.run(d["target"], d["draft"], d["tokens"], d["u_accept"],
                               d["u_resample"], wl.temperature, out_t, out_n)
                    else:
                        b0, b1 = slices[i % len(slices)]
                        sv.run(d["target"][b0:b1], d["draft"][b0:b1], d["tokens"][b0:b1],
                               d["u_accept"][b0:b1], d["u_resample"][b0:b1], wl.temperature,
                               out_t, out_n)
    except Exception as exc:  # capture not possible here: report eager timing only
        torch.cuda.synchronize()
        return None, f"{type(exc).__name__}: {exc}"[:200]
    torch.cuda.synchronize()
    g.replay()
    torch.cuda.synchronize()
    reps = 5
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record()
    for _ in range(reps):
        g.replay()
    ev1.record()
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1) / reps
    del g
    return ms, None


def time_other_configs(args, dev):
    """The other benchmark configurations, one GPU: the 64-sequence gamma-8
    batch at V = 128256 (a plain step like the headline's); the 8-sequence
    batch at V = 32000 and the char-level calls (B = 1, V = 256), both
    launch-bound, as calls per second over rotating input copies larger than
    L2 in total; the 60000-row exactness batch (one call) with the total
    variation distance of its emitted tokens to q."""
    import torch
    from speculative_decoding_verification_90_b200.specverify import SpecVerify
    res = {}
    steps = max(1, args.steps)
    # configuration 4: a bandwidth-bound step (279 MB of logits > 2 x L2)
    wl = workloads.b64_g8_v128256(seed=args.seed)
    d = _device_inputs(wl, dev)
    n_sets = max(1, math.ceil(2 * L2_BYTES / wl.logit_bytes)) if wl.logit_bytes < 2 * L2_BYTES else 1
    sets = [d] + [{k: v.clone() for k, v in d.items()} for _ in range(n_sets - 1)]
    out_t = torch.empty((wl.batch, wl.gamma + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((wl.batch,), dtype=torch.int32, device=dev)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype, dev.index) as sv:
        ms, kern = _time_calls(sv, sets, wl, steps, args.warmup, out_t, out_n)
        st, _ = sv.status()
    res["b64_g8_v128256"] = {"wl": wl, "ms": ms, "calls": steps, "kern": kern, "sets": n_sets,
                             "status": st}
    del sets, d
    # configuration 3: 3.6 MB per call, launch-bound; copies rotate past L2
    wl = workloads.b8_g3_v32000(seed=args.seed)
    d = _device_inputs(wl, dev)
    n_sets = min(256, max(1, math.ceil(2 * L2_BYTES / wl.logit_bytes)))
    sets = [d] + [{k: v.clone() for k, v in d.items()} for _ in range(n_sets - 1)]
    out_t = torch.empty((wl.batch, wl.gamma + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((wl.batch,), dtype=torch.int32, device=dev)
    calls = max(200, 4 * steps)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype, dev.index) as sv:
        ms, kern = _time_calls(sv, sets, wl, calls, args.warmup, out_t, out_n)
        gms, gerr = _time_graph(sv, sets, wl, calls, out_t, out_n)
        st, _ = sv.status()
    res["b8_g3_v32000"] = {"wl": wl, "ms": ms, "calls": calls, "kern": kern, "sets": n_sets,
                           "status": st, "graph_ms": gms, "graph_err": gerr}
    del sets, d
    # configuration 1: 1000 independent calls of one sequence each
    wl = workloads.char_level(calls=1000, seed=args.seed)
    d = _device_inputs(wl, dev)
    out_t = torch.empty((1, wl.gamma + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((1,), dtype=torch.int32, device=dev)
    one_by_one = [(b, b + 1) for b in range(wl.batch)]
    with SpecVerify(1, wl.gamma, wl.vocab, wl.dtype, dev.index) as sv:
        ms, kern = _time_calls(sv, [d], wl, wl.batch, args.warmup, out_t, out_n,
                               slices=one_by_one)
        gms, gerr = _time_graph(sv, [d], wl, wl.batch, out_t, out_n, slices=one_by_one)
        st, _ = sv.status()
    res["char_level"] = {"wl": wl, "ms": ms, "calls": wl.batch, "kern": kern, "sets": 1,
                         "status": st, "graph_ms": gms, "graph_err": gerr}
    del d
    # configuration 2: the exactness batch, one call; the law of its outputs
    with open(os.path.join(ROOT, "tests", "golden", "exactness_beta.json")) as f:
        beta = json.load(f)["beta"]
    wl = workloads.exactness(beta, seed=args.seed)
    d = _device_inputs(wl, dev)
    out_t = torch.empty((wl.batch, wl.gamma + 1), dtype=torch.int32, device=dev)
    out_n = torch.empty((wl.batch,), dtype=torch.int32, device=dev)
    with SpecVerify(wl.batch, wl.gamma, wl.vocab, wl.dtype, dev.index) as sv:
        ms, kern = _time_calls(sv, [d], wl, max(3, steps // 10), args.warmup, out_t, out_n)
        st, _ = sv.status()
    sv_out = out_t[:, 0].cpu().numpy()
    x = wl.target[0, 0].astype(np.float64) / wl.temperature
    q = np.exp(x - x.max())
    q /= q.sum()
    N, V = wl.batch, wl.vocab
    tv = 0.5 * float(np.abs(np.bincount(sv_out, minlength=V)[:V] / N - q).sum())
    rng = np.random.default_rng(1234)
    direct = [0.5 * float(np.abs(np.bincount(rng.choice(V, N, p=q), minlength=V) / N - q).sum())
              for _ in range(20)]
    res["exactness"] = {"wl": wl, "ms": ms, "calls": max(3, steps // 10), "kern": kern, "sets": 1,
                        "status": st, "tv": tv, "tv_direct_mean": float(np.mean(direct)),
                        "tv_direct_sd": float(np.std(direct))}
    del d
    return res


def others_summary(res, peak):
    out = {}
    for name, r in res.items():
        wl = r["wl"]
        per_call_s = r["ms"] / 1e3 / r["calls"]
        positions = wl.batch * wl.gamma
        e = {"workload": wl.name, "batch": wl.batch, "gamma": wl.gamma, "vocab": wl.vocab,
             "logits": wl.dtype, "temperature": wl.temperature,
             "calls": r["calls"], "us_per_call": per_call_s * 1e6,
             "kernels_us_per_call": {"stats": 1e3 * r["kern"]["stats_ms"],
                                     "decide_and_draw": 1e3 * r["kern"]["draw_ms"]},
             "status_after": r["status"]}
        if r.get("graph_ms") is not None or r.get("graph_err"):
            # launch-bound: the same calls captured once in a CUDA graph and
            # replayed, so the host's per-call overhead is left out
            if r.get("graph_ms") is not None:
                gcall = r["graph_ms"] / 1e3 / r["calls"]
                e["graph"] = {"us_per_call": gcall * 1e6, "calls_per_s": 1.0 / gcall,
                              "value": (wl.gamma if name == "char_level" else positions) / gcall,
                              "unit": "positions/s"}
            else:
                e["graph"] = {"unavailable": r["graph_err"]}
        if name == "char_level":
            # one sequence per call
            e["calls_per_s"] = 1.0 / per_call_s
            e["value"] = wl.gamma / per_call_s
            e["unit"] = "positions/s"
            e["l2"] = "one sequence per call (9 KB); launch-bound"
        else:
            step_bytes = wl.logit_bytes
            e["value"] = positions / per_call_s
            e["unit"] = "positions/s"
            e["calls_per_s"] = 1.0 / per_call_s
            e["step_hbm_gbs"] = step_bytes / per_call_s / 1e9
            e["step_frac"] = e["step_hbm_gbs"] / peak
            e["stats_hbm_gbs"] = step_bytes / (r["kern"]["stats_ms"] / 1e3) / 1e9
            e["l2"] = ("inputs larger than L2 (%.1f MB per call, %d rotating set(s))"
                       % (step_bytes / 1e6, r["sets"]))
        if name == "exactness":
            e["tv_emitted_vs_q"] = r["tv"]
            e["tv_direct_sampling"] = {"mean": r["tv_direct_mean"], "sd": r["tv_direct_sd"],
                                       "reps": 20}
        out[name] = e
    return out


def time_single_launch(args, sv, step, dev, world, local):
    """Time the bench's steps with the handle in the single-launch form, then
    restore the three-kernel form."""
    import torch
    sv.set_fused(True)
    try:
        for i in range(max(3, args.warmup)):
            step(i)
        torch.cuda.synchronize()
        ms, kern = timed_then_profiled(step, args.steps, sv.profile_begin, sv.profile_end, world,
                                       local)
        st, _ = sv.status()
        kernels = sv.kernels_per_run()
    finally:
        sv.set_fused(False)
    return {"ms_max": svdist.max_over_ranks(ms, device=dev), "stats_ms": kern["stats_ms"],
            "status": st, "kernels": kernels}


def time_shared_rows(args, wl, sv, put, out_t, out_n, dev, world, local):
    """Time specverify_run_mapped on the workload's distinct rows and row maps."""
    import torch
    import torch.distributed as dist
    m = wl.meta
    nbytes = wl.unique_logit_bytes
    n_sets = max(1, math.ceil(2 * L2_BYTES / nbytes)) if nbytes < 2 * L2_BYTES else 1
    base = {"target_rows": put(m["target_rows"], True), "target_map": put(m["target_map"], False),
            "draft_rows": put(m["draft_rows"], True), "draft_map": put(m["draft_map"], False),
            "tokens": put(wl.tokens, False), "u_accept": put(wl.u_accept, False),
            "u_resample": put(wl.u_resample, False)}
    sets = [base] + [{k: v.clone() for k, v in base.items()} for _ in range(n_sets - 1)]

    def step(i):
        d = sets[i % n_sets]
        sv.run_mapped(d["target_rows"], d["target_map"], d["draft_rows"], d["draft_map"],
                      d["tokens"], d["u_accept"], d["u_resample"], wl.temperature, out_t, out_n)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    ms, kern = timed_then_profiled(step, args.steps, sv.profile_begin, sv.profile_end, world, local)
    ms_max = svdist.max_over_ranks(ms, device=dev)
    st, _ = sv.status()
    del sets, base
    return {"ms_max": ms_max, "stats_ms": kern["stats_ms"], "draw_ms": kern["draw_ms"],
            "bytes": nbytes, "sets": n_sets, "status": st}


def time_sampling(args, wl, sv, sets, n_sets, out_t, out_n, dev, world, local):
    """Time the sampling-variant entry point on the bench batch: greedy; top-k
    50 with top-p 0.9; top-p 0.9 alone; top-k 2000 alone (the last three at the
    workload's temperature)."""
    import torch
    import torch.distributed as dist
    res = {}
    configs = {name: (wl.temperature if T is None else T, k, p)
               for name, (T, k, p) in SAMPLING_SETTINGS.items()}
    if args.sampling:
        configs = {name: configs[name] for name in args.sampling.split(",")}
    for name, (T, k, p) in configs.items():
        temps = torch.full((wl.batch,), T, dtype=torch.float32, device=dev)
        # greedy: the draft "samples" its argmax, which is the method's
        # precondition (t drawn from the adjusted p); tokens drawn at T = 1
        # would hand the rule tokens that p gives no mass
        use = sets
        if T == 0.0:
            use = [dict(d, tokens=d["draft"].argmax(dim=-1).to(torch.int32).contiguous())
                   for d in sets]

        def step(i, use=use):
            d = use[i % n_sets]
            sv.run_sampling(d["target"], d["draft"], d["tokens"], d["u_accept"], d["u_resample"],
                            temps, out_t, out_n, top_k=k, top_p=p)

        for i in range(max(3, args.warmup)):
            step(i)
        torch.cuda.synchronize()
        ms, kern = timed_then_profiled(step, args.steps, sv.profile_begin, sv.profile_end, world,
                                       local)
        ms_max = svdist.max_over_ranks(ms, device=dev)
        st, _ = sv.status()
        res[name] = {"settings": {"temperature": T, "top_k": k, "top_p": p}, "ms_max": ms_max,
                     "select_us": 1e3 * kern["stats_ms"], "decide_and_draw_us": 1e3 * kern["draw_ms"],
                     "status": st}
    return res


def bf16_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]), "measured"
    except Exception:
        return 1590.0, 1400.0, "fallback (1.59 PFLOP/s burst, 1.4 sustained)"


def time_lmhead(args, dev, world, local):
    """Time the verification step fused with the LM head (every rank its own copy)."""
    import torch
    import torch.distributed as dist
    from speculative_decoding_verification_90_b200.specverify import LmHeadVerify
    w = workloads.lmhead(seed=svdist.rank_seed(args.seed, svdist.env_rank()[0]))

    def bf(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)

    ht, wt, hd = bf(w.target_hidden), bf(w.target_weight), bf(w.draft_hidden)
    wd = wt if w.draft_weight is w.target_weight else bf(w.draft_weight)
    tok = torch.from_numpy(w.tokens).to(dev)
    ua = torch.from_numpy(w.u_accept).to(dev)
    ur = torch.from_numpy(w.u_resample).to(dev)
    B, G = w.batch, w.gamma
    ot = torch.empty((B, G + 1), dtype=torch.int32, device=dev)
    on = torch.empty((B,), dtype=torch.int32, device=dev)
    lm = LmHeadVerify(B, G, w.vocab, w.hidden, local)

    def step():
        lm.run(ht, wt, hd, wd, tok, ua, ur, w.temperature, ot, on)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(5, min(args.steps, 50))
    ms, kern = timed_then_profiled(lambda i: step(), steps, lm.profile_begin, lm.profile_end,
                                   world, local)
    ms_max = svdist.max_over_ranks(ms, device=dev)
    st, _ = lm.status()
    keep = lm.keep_logits
    lm.close()
    rows = B * (2 * G + 1)
    return {"workload": w.name, "steps": steps, "ms_max": ms_max, "stats_ms": kern["stats_ms"],
            "rest_ms": kern["rest_ms"], "positions": B * G * world, "keep_logits": keep,
            "stats_flops": 2.0 * rows * w.vocab * w.hidden,
            # the drawn rows' logits come from the kept logits, or from a second GEMM
            "draw_flops": 0.0 if keep else 2.0 * 2 * B * w.vocab * w.hidden,
            "weight_bytes": w.vocab * w.hidden * 2 * (1 if w.draft_weight is w.target_weight else 2),
            "status": st}


def lmhead_summary(g):
    peak, peak_sus, src = bf16_peak()
    ms = g["ms_max"] / g["steps"]
    stats_tf = g["stats_flops"] / (g["stats_ms"] / 1e3) / 1e12
    step_tf = (g["stats_flops"] + g["draw_flops"]) / (ms / 1e3) / 1e12
    return {
        "workload": g["workload"], "entry": "specverify_lmhead_run",
        "value": g["positions"] / (ms / 1e3), "unit": UNIT, "ms_per_step": ms,
        "roofline": {"bound": "tensor", "kernel": "LM-head statistics GEMMs (tcgen05)",
                     "achieved": stats_tf, "peak": peak, "unit": "TFLOP/s",
                     "frac": stats_tf / peak, "peak_source": f"{src} bf16 (burst)",
                     "algorithmic_flops_per_step": g["stats_flops"]},
        "step_tflops": step_tf,
        "stats_gemm_us": 1e3 * g["stats_ms"], "rest_us": 1e3 * g["rest_ms"],
        "logits_kept": g.get("keep_logits"),
        "logits_written_per_step": ("every row's fp32 logits (kept by the statistics GEMMs; "
                                    "the draw reads its 2 rows per sequence there)"
                                    if g.get("keep_logits") else
                                    "only the 2 drawn rows per sequence (fp32, a second GEMM)"),
        "status_after": g["status"],
    }


def time_gate(args, dev, world, local):
    """Time the fold gate on its benchmark tree (every rank its own copy)."""
    import torch
    import torch.distributed as dist
    from speculative_decoding_verification_90_b200.specverify import FoldGate
    w = workloads.gate_tree(seed=svdist.rank_seed(args.seed, svdist.env_rank()[0]))
    H = torch.from_numpy(w.hidden.view(np.int16)).view(torch.bfloat16).to(dev)
    par = torch.from_numpy(w.parent).to(dev)
    rows = w.rows
    packed = torch.empty(rows, dtype=torch.int32, device=dev)
    n = torch.empty(1, dtype=torch.int32, device=dev)
    rel = torch.empty((w.branches, w.positions), dtype=torch.float32, device=dev)
    prov = torch.empty((w.branches, w.positions), dtype=torch.int32, device=dev)
    src = torch.empty((w.branches, w.positions), dtype=torch.int32, device=dev)
    ph = torch.empty((rows, w.dim), dtype=torch.bfloat16, device=dev)
    gate = FoldGate(w.branches, w.positions, w.dim, w.dtype, local)

    def step():
        gate.run(H, par, w.tau, packed, n, rel_diff=rel, provenance=prov, source=src,
                 packed_hidden=ph)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    steps = max(10, min(args.steps, 200))
    ms, kern = timed_then_profiled(lambda i: step(), steps, gate.profile_begin, gate.profile_end,
                                   world, local)
    ms_max = svdist.max_over_ranks(ms, device=dev)
    k = int(n.item())
    # diagnostic: the same passes without the packed batch (the packing kernel
    # then writes no rows), so the difference kernel does not run while the
    # previous pass's 105 MB of packed rows are written back from L2
    def step_unpacked():
        gate.run(H, par, w.tau, packed, n, rel_diff=rel, provenance=prov, source=src)

    for _ in range(3):
        step_unpacked()
    torch.cuda.synchronize()
    _, kern_u = timed_then_profiled(lambda i: step_unpacked(), steps, gate.profile_begin,
                                    gate.profile_end, world, local)
    st, _ = gate.status()
    gate.close()
    return {"workload": w.name, "steps": steps, "ms_max": ms_max, "rows_ms": kern["rows_ms"],
            "rows_ms_unpacked": kern_u["rows_ms"],
            "pack_ms": kern["pack_ms"], "rows": rows, "packed": k,
            "read_bytes": w.rows_read() * w.dim * w.elem_size,
            "packed_bytes": k * w.dim * w.elem_size, "hidden_bytes": w.hidden.nbytes,
            "status": st, "world": world}


def gate_summary(g, peak):
    rows_gbs = g["read_bytes"] / (g["rows_ms"] / 1e3) / 1e9
    # the packing kernel writes the packed batch (its algorithmic bytes); it
    # re-reads those rows, which is not counted
    pack_gbs = g["packed_bytes"] / (g["pack_ms"] / 1e3) / 1e9 if g["pack_ms"] > 0 else None
    ms = g["ms_max"] / g["steps"]
    return {
        "workload": g["workload"], "entry": "specfold_gate_run",
        "rows_per_s": g["rows"] * g["world"] / (ms / 1e3), "ms_per_pass": ms,
        "rows": g["rows"], "packed_rows": g["packed"],
        "difference_kernel": {"us": 1e3 * g["rows_ms"], "algorithmic_bytes": g["read_bytes"],
                              "achieved_gbs": rows_gbs, "peak_gbs": peak,
                              "frac": rows_gbs / peak},
        # the same kernel in passes that write no packed rows (a diagnostic:
        # the figure above includes the write-back of the previous pass's
        # packed batch from L2)
        "difference_kernel_without_packed_rows": {
            "us": 1e3 * g["rows_ms_unpacked"],
            "frac": g["read_bytes"] / (g["rows_ms_unpacked"] / 1e3) / 1e9 / peak},
        "pack_kernel": {"us": 1e3 * g["pack_ms"], "algorithmic_bytes": g["packed_bytes"],
                        "achieved_gbs": pack_gbs},
        "l2": "inputs larger than L2 (%.0f MB of hidden states per pass)" % (g["hidden_bytes"] / 1e6),
        "status_after": g["status"],
    }


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
