#!/usr/bin/env python
"""Decode-step benchmark of hash-scored top-k sparse attention on B200.

One step = append the current token to the cache (hash its key: one key per
(batch, KV-head) pair) + the fused decode (soft bucket tables, soft collision
scores of all N cached keys, exact top-k, attention over the k selected keys)
for the whole batch. Inputs are seeded synthetic caches of the Llama-3.1-8B-like
100K-token decode layer; steps rotate over several independent caches whose
bucket IDs and norms together exceed L2, so every step streams from HBM.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Under torchrun each rank runs the full workload on its own GPU (independent
decode batches: weak scaling, no data-path collective); rank 0 prints one
JSON line. ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attention steps/sec and keys scored/sec at N=100K; HBM GB/s vs peak"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["attend.cuh", "common.cuh", "score.cuh", "select.cuh", "socket_kernels.cuh", "table.cuh",
                 "hash_kernels.cuh"]
NOMINAL_HBM_GBS = 8000.0


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--workload", default="llama3.1-8b_n100k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--caches", type=int, default=4, help="independent caches rotated over (L2 defeat)")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--no-extras", action="store_true", help="skip the dense-decode and CPU baselines")
    ap.add_argument("--no-others", action="store_true", help="skip the records of the other workloads")
    ap.add_argument("--prefill-only", action="store_true",
                    help="build one cache and time only the prefill hashing (a small command for profilers)")
    ap.add_argument("--adaptive-only", action="store_true",
                    help="build the caches and time only the adaptive-k decode (a small command for profilers)")
    ap.add_argument("--estimator-only", action="store_true",
                    help="build one cache and time only the soft-count estimator over its selection "
                         "(a small command for profilers)")
    ap.add_argument("--clock-window", type=float, default=0.5,
                    help="seconds of untimed replays under the clock sampler right before the timed region")
    return ap.parse_args()


# ---------------------------------------------------------------- helpers
def required_bytes(w) -> dict:
    """Algorithmic bytes of one fused decode launch and of one whole step."""
    if w.hata:
        lp, nb, r_bytes = 16, 0, 128 * w.d * 2                                  # 128-bit codes, no norms
    else:
        lp = 16 if w.L <= 16 else 32 if w.L <= 32 else 48 if w.L <= 48 else 64    # ID bytes per key
        nb, r_bytes = 2, w.L * w.P * w.d * 2
    q_bytes = w.B * w.Hq * w.d * 2
    o_bytes = w.B * w.Hq * w.d * 4
    select = w.pairs * (w.N * (lp + nb) + w.k * 4) + q_bytes + r_bytes        # ids (+ f16 norms) in, index list out
    attend = w.pairs * w.k * (2 * w.d * 2 + 4) + q_bytes + o_bytes           # index list + K/V rows in, O out
    decode = select + attend - w.pairs * w.k * 4 - q_bytes                   # the index list stays in L2
    append = w.pairs * (2 * w.d * 2 + lp + nb) + r_bytes                     # new K/V row read, ids + norm written
    estimate = w.pairs * w.k * (w.d * 2 + lp + 4) + q_bytes + r_bytes + o_bytes  # index list, V rows, their IDs
    return {"select": select, "attend": attend, "decode": decode, "step": decode + append,
            "dense": w.pairs * w.N * 2 * w.d * 2 + q_bytes + o_bytes, "estimate": estimate}


def load_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def sources_digest() -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "hash_scored_top_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per selection-kernel launch from the committed ncu summary, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"socket_select_kernel_{workload}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.]+)\s+sources_sha:\s*([0-9a-f]+)", text)
    if not m or m.group(2) != sources_digest():
        return None
    return float(m.group(1))


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_uuid: str | None):
        self.proc = None
        self.uuid = device_uuid

    def __enter__(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "20"]
        if self.uuid:
            cmd += ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        self.t0 = time.perf_counter()
        return self

    def __exit__(self, *exc):
        self.window_s = time.perf_counter() - self.t0
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self) -> dict:
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in (self.out or "").splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for name, val in zip(names, parts[3:7]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        window = round(getattr(self, "window_s", 0.0), 3)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window_s": window}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm), "window_s": window}


# ---------------------------------------------------------------- distributed plumbing
def dist_setup(gpus: int):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    torch.cuda.set_device(local)
    return world, rank, local


def dist_barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_max(world, x: float) -> float:
    """Max of x over ranks (device timings: the slowest rank sets the job's time)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(world: int, steps: int, elapsed_ms_max: float) -> float:
    """Whole-job steps/s: every rank decodes its own batch for `steps` steps."""
    return world * steps / (elapsed_ms_max * 1e-3)


def cache_seed(w, cache: int, rank: int) -> int:
    """Seed of one rank's cache: ranks decode different batches (data parallel)."""
    return w.seed + 101 * cache + 7919 * rank


# ---------------------------------------------------------------- our arm
def build_caches(w, api, wl, n_caches, device, rank=0):
    """Independent seeded caches (different seeds), each hashed by the library."""
    import dataclasses
    import torch
    caches = []
    for c in range(n_caches):
        wc = dataclasses.replace(w, seed=cache_seed(w, c, rank))
        inp = wl.make_inputs(wc, device)
        Ncap = inp["K"].shape[2]
        if w.hata:
            codes = api.empty_codes(w.B, w.Hkv, Ncap, device)
            api.hata_hash_keys(inp["K"], inp["R128"], codes, 0, w.N - 1)
            caches.append({"Q": inp["Q"], "K": inp["K"], "V": inp["V"], "R": inp["R128"], "ids": codes})
        else:
            ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, device)
            norms = api.empty_norms(w.B, w.Hkv, Ncap, device)
            api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms, 0, w.N - 1)
            caches.append({"Q": inp["Q"], "K": inp["K"], "V": inp["V"], "R": inp["R"], "ids": ids, "norms": norms})
        torch.cuda.synchronize()
    return caches


def run_ours(args, world, rank, local):
    import torch
    from hash_scored_top_b200 import api, build
    from hash_scored_top_b200 import workloads as wl

    if rank == 0:
        build.build()
    dist_barrier(world)
    w = wl.WORKLOADS[args.workload]
    device = torch.device("cuda", local)
    # one cache already streams more than L2 per step for the hard-hash workload (17 GB of K/V each)
    n_caches = 1 if (w.hata or args.prefill_only or args.estimator_only) else args.caches
    caches = build_caches(w, api, wl, n_caches, device, rank)
    if args.adaptive_only:
        peak, _ = load_peaks()
        rec = run_adaptive(w, api, caches, device, peak)
        rec.update({"workload": w.name})
        return rec
    if args.estimator_only:
        peak, _ = load_peaks()
        rec = run_estimator(w, api, caches, device, required_bytes(w), peak)
        rec.update({"workload": w.name, "launches": "1 selection, then the factor and attend kernels of "
                                                     "4 warm-up calls, then CUDA graph replays"})
        return rec
    if args.prefill_only:
        peak, _ = load_peaks()
        rec = run_prefill_hash(w, api, caches, device, peak)
        rec.update({"workload": w.name, "launches": "1 while building the cache, 2 warm-up, 5 timed"})
        return rec
    Ncap = caches[0]["K"].shape[2]
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    op = api.OP_HATA_DECODE if w.hata else api.OP_DECODE
    ws = torch.empty(api.workspace_bytes(op, w.B, w.Hq, w.Hkv, Ncap, w.N, w.d, w.L, w.P, w.k),
                     dtype=torch.uint8, device=device)

    def append(c):
        if w.hata:
            api.hata_hash_keys(c["K"], c["R"], c["ids"], w.N - 1, 1)
        else:
            api.socket_hash_keys(c["K"], c["V"], c["R"], w.L, w.P, c["ids"], c["norms"], w.N - 1, 1)

    idx_sel = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=device)

    def select(c):
        if not w.hata:
            api.socket_select(c["Q"], c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau, w.k, idx_sel)

    def decode(c):
        if w.hata:
            api.hata_decode(c["Q"], c["K"], c["V"], c["R"], c["ids"], w.N, w.k, w.scale, O, None, ws)
        else:
            api.socket_decode(c["Q"], c["K"], c["V"], c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau, w.k,
                              w.scale, O, None, ws)

    def step(c):
        # one decoder step: hash the current token (key N - 1), then decode over N keys
        if w.hata:
            append(c)
            decode(c)
        else:
            api.socket_decode_append(c["Q"], c["K"], c["V"], c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau,
                                     w.k, w.scale, O, None, ws)

    # warm-up through the plain API (also sets the kernels' attributes)
    for i in range(args.warmup):
        c = caches[i % len(caches)]
        append(c)
        decode(c)
        select(c)
    api.check_status()

    # CUDA graphs: one step per cache (append + decode), and the decode alone
    per_graph = len(caches)
    side = torch.cuda.Stream(device=device)
    g_step, g_dec, g_sel = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g_step, stream=side):
            for c in caches:
                step(c)
        with torch.cuda.graph(g_dec, stream=side):
            for c in caches:
                decode(c)
        if not w.hata:
            with torch.cuda.graph(g_sel, stream=side):
                for c in caches:
                    select(c)
    torch.cuda.synchronize()
    reps = max(1, args.steps // per_graph)
    steps = reps * per_graph
    for _ in range(3):
        g_step.replay()
        g_dec.replay()
        if not w.hata:
            g_sel.replay()
    torch.cuda.synchronize()

    # ---- timed region: `steps` steps back to back
    stream = torch.cuda.current_stream()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
    except Exception:
        pass
    dist_barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(uuid) as clk:
        # the clock record needs a window of a few hundred ms: untimed replays of
        # the same step fill it up to the timed region, which follows at once
        t_end = time.perf_counter() + args.clock_window
        while time.perf_counter() < t_end:
            g_step.replay()
            torch.cuda.synchronize()
        start.record(stream)
        torch.cuda.nvtx.range_push("timed")
        for _ in range(reps):
            g_step.replay()
        torch.cuda.nvtx.range_pop()
        end.record(stream)
        torch.cuda.synchronize()
    dist_barrier(world)
    api.check_status()
    elapsed_ms = dist_max(world, start.elapsed_time(end))
    ms_per_step = elapsed_ms / steps
    clocks = clk.summary()

    # the decode kernels alone (same caches, same back-to-back replay)
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(reps):
        g_dec.replay()
    d1.record(stream)
    torch.cuda.synchronize()
    decode_us = dist_max(world, d0.elapsed_time(d1) * 1e3 / steps)
    # the selection kernel alone (the dominant kernel of the step)
    select_us = None
    if not w.hata:
        d0.record(stream)
        for _ in range(reps):
            g_sel.replay()
        d1.record(stream)
        torch.cuda.synchronize()
        select_us = dist_max(world, d0.elapsed_time(d1) * 1e3 / steps)

    rb = required_bytes(w)
    peak, peak_kind = load_peaks()
    # the hard-hash workload has no selection-only entry point: its roofline
    # unit is the decode launch pair
    roof_us, roof_bytes = (decode_us, rb["decode"]) if w.hata else (select_us, rb["select"])
    achieved = roof_bytes / (roof_us * 1e-6) / 1e9
    result = {
        "metric": METRIC,
        "value": weak_value(world, steps, elapsed_ms),
        "unit": "decode steps/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic: seeded Gaussian K/V caches with outlier channels and planted needles",
        "config": {
            "workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N, "L": w.L, "P": w.P,
            "tau": w.tau, "k": w.k, "kv_dtype": w.kv_dtype, "global_batch": w.B * world,
            "step": ("hata_hash_keys of 1 new token per pair, then hata_decode (codes, Hamming scores, exact "
                     "top-k, sparse attention)") if w.hata else
                    ("socket_decode_append: hash 1 new token per pair, then decode (tables, scores, exact top-k, "
                     "sparse attention)"),
            "launch": f"CUDA graph of {per_graph} steps replayed {reps} times",
            "l2": f"inputs larger than L2: {n_caches} rotating caches x "
                  f"{rb['select'] / 1e6:.0f} MB of hashed keys per step",
            "parallelism": f"replicas x{world}",
        },
        "keys_scored_per_s": world * steps * w.pairs * w.N / (elapsed_ms * 1e-3),
        "required_bytes_per_step": rb["step"],
        "hbm_gbs_required": world * rb["step"] * steps / (elapsed_ms * 1e-3) / 1e9,
        "roofline": {
            "kernel": "socket_select_kernel + socket_attend_kernel (hard hash)" if w.hata else "socket_select_kernel",
            "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "peak_kind": peak_kind, "traffic": None if w.hata else profiled_traffic(w.name),
            "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS,
            "bytes_per_launch": roof_bytes, "avg_launch_us": roof_us,
        },
        "decode_kernels": {
            "kernels": "socket_select_kernel -> socket_attend_kernel (programmatic dependent launch)",
            "avg_us": decode_us, "bytes": rb["decode"], "gbs": rb["decode"] / (decode_us * 1e-6) / 1e9,
            "frac": rb["decode"] / (decode_us * 1e-6) / 1e9 / peak,
            "frac_of_nominal_8tbs": rb["decode"] / (decode_us * 1e-6) / 1e9 / NOMINAL_HBM_GBS,
        },
        "gpu_launches": 3 * steps,
        "clocks": clocks,
    }
    # the records beyond the headline run at N = 1 only: the scaling runs hold
    # every GPU of the node, and these records add minutes and per-rank host
    # memory (pinned pools) without measuring scaling
    if not args.no_others and world == 1:
        result["workloads"] = {}
        for name in wl.WORKLOADS:
            if name != w.name:
                result["workloads"][name] = run_workload_record(name, api, wl, device, peak)
    if not args.no_extras and not w.hata:
        result["e2e"] = run_e2e(args, w, api, caches, device, world, ws)
    if not args.no_extras and not w.hata and world == 1:
        result["dense_decode"] = run_dense(w, api, caches, device, rb, peak)
        result["prefill_hash"] = run_prefill_hash(w, api, caches, device, peak)
        result["soft_count_estimator"] = run_estimator(w, api, caches, device, rb, peak)
        result["per_head_decode"] = run_heads(w, api, caches, device, peak)
        result["adaptive_decode"] = run_adaptive(w, api, caches, device, peak)
        result["paged_decode"] = run_paged(w, api, caches, device, rb, peak)
        if rank == 0:
            result["cpu_baseline"] = cpu_baseline(w, caches[0], sample_pairs=8)
    del g_step, g_dec, g_sel
    return result


OTHER_STEPS = {"tiny_f32": 200, "llama3.2-1b_n32k": 200, "llama3.1-8b_n100k": 100, "qwen3-30b_n140k": 50,
               "hata_n256k": 20}


def run_workload_record(name, api, wl, device, peak):
    """One decode step of another workload, timed step by step with CUDA events
    (an L2 flush of 256 MB between steps, outside the events): one cache drawn
    and hashed by the library, then socket_decode_append (or the hard-hash
    append + decode) over all N keys."""
    import torch
    w = wl.WORKLOADS[name]
    inp = wl.make_inputs(w, device)
    Ncap = inp["K"].shape[2]
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    if w.hata:
        codes = api.empty_codes(w.B, w.Hkv, Ncap, device)
        api.hata_hash_keys(inp["K"], inp["R128"], codes, 0, w.N - 1)
        ws = torch.empty(api.workspace_bytes(api.OP_HATA_DECODE, w.B, w.Hq, w.Hkv, Ncap, w.N, w.d, 16, 8, w.k),
                         dtype=torch.uint8, device=device)

        def step():
            api.hata_hash_keys(inp["K"], inp["R128"], codes, w.N - 1, 1)
            api.hata_decode(inp["Q"], inp["K"], inp["V"], inp["R128"], codes, w.N, w.k, w.scale, O, None, ws)
    else:
        ids = api.empty_ids(w.B, w.Hkv, Ncap, w.L, device)
        norms = api.empty_norms(w.B, w.Hkv, Ncap, device)
        api.socket_hash_keys(inp["K"], inp["V"], inp["R"], w.L, w.P, ids, norms, 0, w.N - 1)
        ws = torch.empty(api.workspace_bytes(api.OP_DECODE, w.B, w.Hq, w.Hkv, Ncap, w.N, w.d, w.L, w.P, w.k),
                         dtype=torch.uint8, device=device)

        def step():
            api.socket_decode_append(inp["Q"], inp["K"], inp["V"], inp["R"], ids, norms, w.N, w.L, w.P, w.tau, w.k,
                                     w.scale, O, None, ws)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    n = OTHER_STEPS.get(name, 50)
    for _ in range(3):
        step()
    api.check_status()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    for e0, e1 in ev:
        flush.zero_()
        e0.record()
        step()
        e1.record()
    torch.cuda.synchronize()
    api.check_status()
    times = [e0.elapsed_time(e1) * 1e3 for e0, e1 in ev]
    us = sum(times) / n
    rb = required_bytes(w)
    gbs = rb["step"] / (us * 1e-6) / 1e9
    rec = {"us_per_step": us, "us_median": statistics.median(times), "steps_per_s": 1e6 / us,
           "required_bytes_per_step": rb["step"], "hbm_gbs": gbs, "frac_of_peak": gbs / peak,
           "keys_scored_per_s": w.pairs * w.N / (us * 1e-6), "steps": n,
           "shape": {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N, "L": w.L, "P": w.P, "k": w.k,
                     "kv_dtype": w.kv_dtype, "hard_hash": w.hata},
           "timing": "CUDA events around each step, 256 MB L2 flush between steps outside the events"}
    del inp, O, ws, flush
    torch.cuda.empty_cache()
    return rec


def run_e2e(args, w, api, caches, device, world, ws):
    """Same step through the public API with host buffers: per step
    socket_decode_step_host copies the new token's query and K/V rows in from
    pinned host memory, runs the step and copies the output back to it."""
    import torch
    c = caches[0]
    n = max(args.e2e_steps, 3)
    q_host = c["Q"].cpu().pin_memory()
    k_host = c["K"][:, :, w.N - 1].contiguous().cpu().pin_memory()
    v_host = c["V"][:, :, w.N - 1].contiguous().cpu().pin_memory()
    o_host = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(c["Q"])
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    stream = torch.cuda.current_stream()

    def e2e_step():
        api.socket_decode_step_host(q_host, k_host, v_host, q_dev, c["K"], c["V"], c["R"], c["ids"], c["norms"], w.N,
                                    w.L, w.P, w.tau, w.k, w.scale, O, o_host, ws)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(n):
        e2e_step()
    e.record(stream)
    torch.cuda.synchronize()
    ms = dist_max(world, s.elapsed_time(e))
    h2d = sum(t.numel() * t.element_size() for t in (q_host, k_host, v_host))
    return {"value": world * n / (ms * 1e-3), "unit": "decode steps/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": o_host.numel() * o_host.element_size(), "steps": n,
            "note": "one socket_decode_step_host call per step (no graph): the query and the new token's K/V rows "
                    "copied in from pinned host memory, O copied back to pinned host memory; KV cache resident in HBM"}


def run_prefill_hash(w, api, caches, device, peak):
    """Prefill hashing (SOCKET step 1) of all N cached keys of one cache: reads K and V once."""
    import torch
    c = caches[0]
    n, warm = 5, 2
    for _ in range(warm):
        api.socket_hash_keys(c["K"], c["V"], c["R"], w.L, w.P, c["ids"], c["norms"], 0, w.N)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(n):
        api.socket_hash_keys(c["K"], c["V"], c["R"], w.L, w.P, c["ids"], c["norms"], 0, w.N)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / n
    lp = 16 if w.L <= 16 else 32 if w.L <= 32 else 48 if w.L <= 48 else 64
    nbytes = w.pairs * w.N * (2 * w.d * 2 + lp + 2) + w.L * w.P * w.d * 2   # K, V in; ids, norms out
    gbs = nbytes / (ms * 1e-3) / 1e9
    kernel = "hash_keys_tcgen05_kernel" if (w.kv_dtype == "bf16" and w.P == 8) else "hash_keys_simt_kernel"
    return {"kernel": kernel, "us": ms * 1e3, "bytes": nbytes, "hbm_gbs": gbs, "frac_of_peak": gbs / peak,
            "keys_per_s": w.pairs * w.N / (ms * 1e-3)}


def run_estimator(w, api, caches, device, rb, peak):
    """The soft-count attention estimator over each cache's selected keys
    (selection done once per cache, untimed), the caches taken in turn."""
    import torch
    Ncap = caches[0]["K"].shape[2]
    idxs = []
    for c in caches:
        idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=device)
        api.socket_select(c["Q"], c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau, w.k, idx)
        idxs.append(idx)
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    ws = torch.empty(api.workspace_bytes(api.OP_SOFT_COUNT, w.B, w.Hq, w.Hkv, Ncap, w.k, w.d, w.L, w.P, w.k),
                     dtype=torch.uint8, device=device)
    def est(i):
        c = caches[i]
        api.socket_soft_count_attend(c["Q"], c["V"], c["R"], c["ids"], idxs[i], w.L, w.P, w.tau, O, ws)

    us = _time_calls(est, len(caches))
    api.check_status()
    gbs = rb["estimate"] / (us * 1e-6) / 1e9
    return {"kernel": "soft_count_attend_kernel", "us": us, "bytes": rb["estimate"], "hbm_gbs": gbs,
            "frac_of_peak": gbs / peak, "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "launch": f"CUDA graph of {len(caches)} calls (one per cache, each with its own selected index list)"}


def _time_calls(fn, n_caches, reps=50, warm=3):
    """Average device microseconds of one fn(i) call: the calls over all caches
    (i = 0 .. n_caches - 1) are captured in one CUDA graph, which is replayed
    `reps` times back to back between two CUDA events (the host's per-call
    overhead stays out of the measurement, as in the timed step)."""
    import torch
    for i in range(n_caches):
        fn(i)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for i in range(n_caches):
                fn(i)
    torch.cuda.synchronize()
    for _ in range(warm):
        g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    stream = torch.cuda.current_stream()
    s.record(stream)
    for _ in range(reps):
        g.replay()
    e.record(stream)
    torch.cuda.synchronize()
    us = s.elapsed_time(e) * 1e3 / (reps * n_caches)
    del g
    return us


def run_heads(w, api, caches, device, peak):
    """Decode with one index set per query head (socket_decode_heads): B * Hq
    units, each scoring its KV head's N keys with its own table and gathering
    its own k rows. Required bytes: the cached IDs and norms once per KV head,
    k K/V rows per query head."""
    import torch
    Ncap = caches[0]["K"].shape[2]
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    ws = torch.empty(api.workspace_bytes(api.OP_DECODE_HEADS, w.B, w.Hq, w.Hkv, Ncap, w.N, w.d, w.L, w.P, w.k),
                     dtype=torch.uint8, device=device)

    def call(i):
        c = caches[i]
        api.socket_decode_heads(c["Q"], c["K"], c["V"], c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau, w.k,
                                w.scale, O, None, ws)

    us = _time_calls(call, len(caches))
    api.check_status()
    lp = 16 if w.L <= 16 else 32 if w.L <= 32 else 48 if w.L <= 48 else 64
    nbytes = w.pairs * w.N * (lp + 2) + w.B * w.Hq * w.k * (2 * w.d * 2 + 4) + w.B * w.Hq * w.d * (2 + 4)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"kernels": "socket_select_kernel (B*Hq units) -> socket_attend_kernel", "us": us,
            "required_bytes": nbytes, "hbm_gbs": gbs, "frac_of_peak": gbs / peak,
            "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS, "units": w.B * w.Hq,
            "launch": f"CUDA graph of {len(caches)} calls (one per cache)"}


ADAPTIVE_MASS = 0.25


def run_adaptive(w, api, caches, device, peak):
    """Decode with the adaptive k (socket_decode_adaptive, one unit per KV head):
    k from the cumulative soft-score mass ADAPTIVE_MASS, clamped to
    [k / 4, 4 k]. Four kernels: tables, scores (to HBM), adaptive top-k,
    attention. Required bytes: IDs and norms, the scores written and read
    once, the chosen K/V rows."""
    import torch
    Ncap = caches[0]["K"].shape[2]
    k_min, k_max = max(1, w.k // 4), min(w.N, 4 * w.k)
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    idx = torch.empty(w.B, w.Hkv, k_max, dtype=torch.int32, device=device)
    kc = torch.empty(w.B, w.Hkv, dtype=torch.int32, device=device)
    ws = torch.empty(api.workspace_bytes(api.OP_DECODE_ADAPTIVE, w.B, w.Hq, w.Hkv, Ncap, w.N, w.d, w.L, w.P, k_max),
                     dtype=torch.uint8, device=device)

    def call(i):
        c = caches[i]
        api.socket_decode_adaptive(c["Q"], c["K"], c["V"], c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau,
                                   ADAPTIVE_MASS, k_min, k_max, w.scale, O, idx, kc, ws=ws)

    us = _time_calls(call, len(caches))
    api.check_status()
    ks = []
    for i in range(len(caches)):
        call(i)
        torch.cuda.synchronize()
        ks.extend(kc.flatten().tolist())
    mean_k = sum(ks) / len(ks)
    lp = 16 if w.L <= 16 else 32 if w.L <= 32 else 48 if w.L <= 48 else 64
    nbytes = int(w.pairs * w.N * (lp + 2 + 8) + w.pairs * mean_k * (2 * w.d * 2 + 8) + w.B * w.Hq * w.d * (2 + 4))
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"kernels": "bucket_table_kernel -> socket_score_kernel -> socket_adaptive_topk_kernel -> "
                       "socket_attend_kernel", "us": us, "mass": ADAPTIVE_MASS, "k_min": k_min, "k_max": k_max,
            "k_mean": mean_k, "k_range": [min(ks), max(ks)], "required_bytes": nbytes, "hbm_gbs": gbs,
            "frac_of_peak": gbs / peak, "frac_of_nominal_8tbs": gbs / NOMINAL_HBM_GBS,
            "launch": f"CUDA graph of {len(caches)} calls (one per cache)"}


PAGE_SIZE = 64


def _to_pages(K, V, page_size, seed):
    """The cache [B, Hkv, Ncap, d] scattered over a shuffled pool of pages, and its page table."""
    import torch
    B, Hkv, Ncap, d = K.shape
    per = Ncap // page_size
    g = torch.Generator().manual_seed(seed)
    phys = torch.randperm(B * Hkv * per, generator=g).to(K.device)
    Kp = torch.empty(B * Hkv * per, page_size, d, dtype=K.dtype, device=K.device)
    Vp = torch.empty_like(Kp)
    Kp[phys] = K.reshape(-1, page_size, d)
    Vp[phys] = V.reshape(-1, page_size, d)
    return Kp, Vp, phys.view(B, Hkv, per).int().contiguous()


def run_paged(w, api, caches, device, rb, peak):
    """The decode step with the K/V cache in a pool of 64-key pages
    (socket_decode_paged): device-resident pools (one per cache, pages
    shuffled), and one pinned host pool, whose selected rows cross the host
    link. The host-link peak is the measured pinned host-to-device copy rate."""
    import torch
    Ncap = caches[0]["K"].shape[2]
    if Ncap % PAGE_SIZE:
        return {"skipped": f"Ncap {Ncap} is not a multiple of the page size {PAGE_SIZE}"}
    pools = [_to_pages(c["K"], c["V"], PAGE_SIZE, 17 + i) for i, c in enumerate(caches)]
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    ws = torch.empty(api.workspace_bytes(api.OP_DECODE_PAGED, w.B, w.Hq, w.Hkv, Ncap, w.N, w.d, w.L, w.P, w.k),
                     dtype=torch.uint8, device=device)

    def dev_call(i):
        c = caches[i]
        Kp, Vp, tab = pools[i]
        api.socket_decode_paged(c["Q"], Kp, Vp, tab, c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau, w.k,
                                w.scale, O, None, ws)

    us_dev = _time_calls(dev_call, len(caches))
    api.check_status()
    rec = {"page_size": PAGE_SIZE, "device_pool": {
        "us": us_dev, "steps_per_s": 1e6 / us_dev, "required_bytes": rb["decode"],
        "hbm_gbs": rb["decode"] / (us_dev * 1e-6) / 1e9, "frac_of_peak": rb["decode"] / (us_dev * 1e-6) / 1e9 / peak,
        "kernels": "socket_select_kernel -> socket_attend_kernel (rows through the page table)",
        "launch": f"CUDA graph of {len(caches)} calls (one per cache)"}}
    # the host link: pinned -> device copy rate of 256 MB
    src = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dst = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    for _ in range(2):
        dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for _ in range(5):
        dst.copy_(src, non_blocking=True)
    e.record()
    torch.cuda.synchronize()
    link_gbs = 5 * (256 << 20) / (s.elapsed_time(e) * 1e-3) / 1e9
    del src, dst
    Kp, Vp, tab = pools[0]
    Kh, Vh = Kp.cpu().pin_memory(), Vp.cpu().pin_memory()

    def host_call(i):
        c = caches[0]
        api.socket_decode_paged(c["Q"], Kh, Vh, tab, c["R"], c["ids"], c["norms"], w.N, w.L, w.P, w.tau, w.k,
                                w.scale, O, None, ws)

    us_host = _time_calls(host_call, 1, reps=10, warm=2)
    api.check_status()
    link_bytes = w.pairs * w.k * 2 * w.d * 2
    rec["host_pool"] = {
        "us": us_host, "steps_per_s": 1e6 / us_host, "host_link_bytes": link_bytes,
        "host_link_gbs": link_bytes / (us_host * 1e-6) / 1e9, "host_link_peak_gbs": link_gbs,
        "frac_of_link_peak": link_bytes / (us_host * 1e-6) / 1e9 / link_gbs,
        "kernels": "socket_select_kernel -> paged_gather_kernel (plain loads of pinned host rows) -> "
                   "socket_attend_kernel (dense over the gathered rows)",
        "launch": "CUDA graph of 1 call, 10 replays (the one host pool)"}
    del pools, Kh, Vh, ws
    torch.cuda.empty_cache()
    return rec


def run_dense(w, api, caches, device, rb, peak):
    """Dense decode attention over all N keys (the FlashAttention-style baseline), same caches."""
    import torch
    O = torch.empty(w.B, w.Hq, w.d, device=device)
    ws = torch.empty(api.workspace_bytes(api.OP_DENSE_DECODE, w.B, w.Hq, w.Hkv, caches[0]["K"].shape[2], w.N, w.d),
                     dtype=torch.uint8, device=device)
    n, warm = 200, 10
    for i in range(warm):
        c = caches[i % len(caches)]
        api.dense_decode(c["Q"], c["K"], c["V"], w.N, w.scale, O, ws)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record()
    for i in range(n):
        c = caches[i % len(caches)]
        api.dense_decode(c["Q"], c["K"], c["V"], w.N, w.scale, O, ws)
    e.record()
    torch.cuda.synchronize()
    ms = s.elapsed_time(e) / n
    gbs = rb["dense"] / (ms * 1e-3) / 1e9
    return {"steps_per_s": 1e3 / ms, "ms_per_step": ms, "hbm_gbs": gbs, "frac_of_peak": gbs / peak,
            "bytes_per_step": rb["dense"]}


# ---------------------------------------------------------------- CPU oracle timing
def _oracle_pair_inputs(w, cache, pairs):
    """Per-pair float64 inputs and the oracle's own cache (hashing is prefill, not timed)."""
    from oracle import socket_ref as so
    R = cache["R"].double().cpu().numpy()
    out = []
    for b, h in pairs:
        K = cache["K"][b, h, : w.N].double().cpu().numpy()
        V = cache["V"][b, h, : w.N].double().cpu().numpy()
        Qg = cache["Q"][b, h * w.G:(h + 1) * w.G].double().cpu().numpy()
        ids, _ = so.hash_key_ids(K, R, w.L, w.P)
        norms = so.value_norms_f16(V)
        out.append((Qg, K, V, R, ids, norms))
    return out


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _limit_blas_env(env):
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        env[var] = "1"


def _cpu_worker(i, wname, barrier, queue, reps=1):
    """One host core: draws one seeded (batch, kv-head) pair of the workload on
    the CPU, hashes it with the oracle (prefill, untimed), then times the
    oracle's decode of that pair between two barriers."""
    _limit_blas_env(os.environ)
    from threadpoolctl import threadpool_limits
    from hash_scored_top_b200 import workloads as wl
    from oracle import hata_ref as ho
    from oracle import socket_ref as so
    w = wl.WORKLOADS[wname]
    wp = wl.shrink(w, B=1, Hkv=1, Hq=w.G, seed=w.seed + 7919 * (i + 1))
    inp = wl.make_inputs(wp, "cpu")
    Qg = inp["Q"][0].double().numpy()
    K = inp["K"][0, 0, : w.N].float().numpy()
    V = inp["V"][0, 0, : w.N].float().numpy()
    with threadpool_limits(1):
        if w.hata:
            R = inp["R128"].double().numpy()
            codes, _ = ho.binary_codes(K, R)

            def decode():
                ho.hata_decode_pair(Qg, K, V, R, codes, w.k, w.scale)
        else:
            R = inp["R"].double().numpy()
            ids, _ = so.hash_key_ids(K, R, w.L, w.P)
            norms = so.value_norms_f16(V)

            def decode():
                so.socket_decode_pair(Qg, K, V, R, ids, norms, w.L, w.P, w.tau, w.k, w.scale)
        decode()                                   # untimed: first-touch of the arrays
        barrier.wait(timeout=600)
        t0 = time.monotonic()
        for _ in range(reps):
            decode()
        t1 = time.monotonic()
    queue.put((i, t0, t1))


CPU_REPS = 25      # decodes per core: about 1 s of oracle work per core at the 8B shape


def cpu_baseline_all_cores(w, max_workers=32, reps=CPU_REPS):
    """The oracle on every host core at once: one process per core (spawned),
    each decoding its own seeded pair of the workload `reps` times; the wall
    time from the first start to the last finish covers n * reps pair decodes."""
    import multiprocessing as mp
    n = max(1, min(host_cores(), max_workers, w.pairs))
    ctx = mp.get_context("spawn")
    barrier = ctx.Barrier(n)
    queue = ctx.Queue()
    env_backup = {v: os.environ.get(v) for v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    _limit_blas_env(os.environ)
    try:
        procs = [ctx.Process(target=_cpu_worker, args=(i, w.name, barrier, queue, reps)) for i in range(n)]
        for p in procs:
            p.start()
        res = [queue.get(timeout=900) for _ in range(n)]
        for p in procs:
            p.join(60)
    finally:
        for var, val in env_backup.items():
            if val is None:
                os.environ.pop(var, None)
            else:
                os.environ[var] = val
    wall = max(r[2] for r in res) - min(r[1] for r in res)
    return {"value": n * reps / (wall * w.pairs), "unit": "decode steps/s", "cores": n, "kind": "oracle",
            "wall_s": wall, "cpu_s": sum(r[2] - r[1] for r in res),
            "sample": f"{n} seeded (batch, kv-head) pairs of the workload drawn on the host, one per core "
                      f"(spawned processes, BLAS 1 thread each), each decoded {reps} times at once; "
                      f"{n * reps} pair decodes = {n * reps / w.pairs:.1f} steps of {w.pairs} pairs"}


def cpu_baseline(w, cache, sample_pairs=8):
    from threadpoolctl import threadpool_limits
    from oracle import socket_ref as so
    pairs = [(p // w.Hkv, p % w.Hkv) for p in range(min(sample_pairs, w.pairs))]
    data = _oracle_pair_inputs(w, cache, pairs)
    times = []
    with threadpool_limits(1):
        for _ in range(3):
            t0 = time.perf_counter()
            for Qg, K, V, R, ids, norms in data:
                so.socket_decode_pair(Qg, K, V, R, ids, norms, w.L, w.P, w.tau, w.k, w.scale)
            times.append(time.perf_counter() - t0)
    t = statistics.median(times)
    single = {"value": len(pairs) / (t * w.pairs), "cores": 1,
              "sample": f"{len(pairs)} of {w.pairs} (batch, kv-head) pairs of the bench's first cache, "
                        f"median of 3, float64 numpy, BLAS limited to 1 thread; scaled to a whole step"}
    out = cpu_baseline_all_cores(w)
    out["single_core"] = single
    out["cpu_model"] = cpu_model()
    out["host_cores"] = host_cores()
    return out


def run_reference(args):
    """The CPU oracle as the reference arm: each step decodes a bounded sample of one pair."""
    import numpy as np
    import torch
    from threadpoolctl import threadpool_limits
    from hash_scored_top_b200 import workloads as wl
    from oracle import hata_ref as ho
    from oracle import socket_ref as so

    w = wl.WORKLOADS[args.workload]
    inp = wl.make_inputs(wl.shrink(w, B=1, Hkv=1, Hq=w.G), "cpu")
    Qg = inp["Q"][0].double().numpy()
    K = inp["K"][0, 0, : w.N].double().numpy()
    V = inp["V"][0, 0, : w.N].double().numpy()
    R = inp["R128" if w.hata else "R"].double().numpy()
    if w.hata:
        codes, _ = ho.binary_codes(K, R)

        def decode(n, kk):
            ho.hata_decode_pair(Qg, K[:n], V[:n], R, codes[:n], kk, w.scale)
    else:
        ids, _ = so.hash_key_ids(K, R, w.L, w.P)
        norms = so.value_norms_f16(V)

        def decode(n, kk):
            so.socket_decode_pair(Qg, K[:n], V[:n], R, ids[:n], norms[:n], w.L, w.P, w.tau, kk, w.scale)
    # size the per-step sample so that warmup + steps fit in about two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    with threadpool_limits(1):
        n_try = min(w.N, 8192)
        t0 = time.perf_counter()
        decode(n_try, max(1, w.k * n_try // w.N))
        per_key = (time.perf_counter() - t0) / n_try
        n = int(min(w.N, max(256, budget / per_key)))
        kk = max(1, w.k * n // w.N)
        for _ in range(args.warmup):
            decode(n, kk)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            decode(n, kk)
        dt = time.perf_counter() - t0
    scale = (w.pairs * w.N) / n                      # sample keys -> one whole step
    value = args.steps / (dt * scale)
    sample = (f"each step: the first {n} of {w.N} keys of one of {w.pairs} (batch, kv-head) pairs, k={kk}; "
              f"time scaled by {scale:.1f} to a whole step (linear in keys scored)")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "decode steps/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / value, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, same workload)",
        "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "N": w.N, "L": w.L,
                   "P": w.P, "tau": w.tau, "k": w.k},
        "ms_per_step_extrapolated": True,
        "extrapolation": f"each timed step decodes {n} keys of one pair; ms_per_step and value scale that time "
                         f"by {scale:.1f} to a whole step of {w.pairs} pairs x {w.N} keys",
        "cpu_baseline": {"value": value, "unit": "decode steps/s", "cores": 1, "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "decode steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args)))
        return 0
    world, rank, local = dist_setup(args.gpus)
    try:
        result = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(result))
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
