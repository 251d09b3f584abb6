#!/usr/bin/env python3
"""Benchmark of the Rodimus+ token-mixing hot path on B200.

One step = one prefill pass of the long-context Rodimus+ mixer stack (B=1, T=131072,
hidden 2048 = 16 heads x 128, 24 layers alternating the gated linear recurrence and SW-SKA
with window 4096), every layer through the library's C ABI. value = prefill tokens/s over all
ranks (each rank runs its own replica on its own seeded inputs: weak scaling, no collective
in the data path). The same line carries the batched decode step (256 sequences x 1 token:
recurrence update + readout over 16 heads of 128x128 fp32 state, and SW-SKA over a
4096-slot ring buffer) as "decode", the roofline of the dominant kernel, the oracle's CPU
baseline, an end-to-end number through host buffers, clocks and the launch count.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "Rodimus+ mixer prefill tokens/s & decode tok/s on 1 B200; % of HBM/TC roofline"
WORKLOAD = "stack_t131072"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------------------------------
# helpers
# ------------------------------------------------------------------------------------------


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def swska_pairs(T, W):
    """Number of (query, key) pairs inside the causal window, per (batch, head)."""
    if W >= T:
        return T * (T + 1) // 2
    return W * T - W * (W - 1) // 2


class ClockSampler:
    """nvidia-smi sampled every 100 ms. Started before the warm-up steps, so that the tool is
    already sampling when the timed region begins; mark() brackets the timed region, and the
    summary keeps the samples whose timestamps fall inside it (all samples if the timestamps
    cannot be read)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, interval_ms=100):
        self.gpu = gpu_index
        self.interval_ms = interval_ms
        self.proc = None
        self.file = None
        self.window = None  # (start, end) of the timed region, host epoch seconds

    def __enter__(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.interval_ms)],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def wait_started(self, timeout_s=5.0):
        """Return once the first sample is written (or after timeout_s)."""
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < timeout_s:
            try:
                if os.path.getsize(self.file.name) > 0:
                    return
            except OSError:
                return
            time.sleep(0.05)

    def mark(self, start, end):
        self.window = (start, end)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    @staticmethod
    def _epoch(stamp):
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(stamp.strip(), fmt).timestamp()
            except ValueError:
                continue
        return None

    def summary(self):
        if self.proc is None or self.file is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.file.flush()
        with open(self.file.name) as f:
            lines = [line for line in f if line.strip()]
        os.unlink(self.file.name)
        return self.summarise(lines, self.window)

    @classmethod
    def summarise(cls, lines, window=None):
        """Median SM clock under load, the maximum clock and the throttle reasons seen, from
        nvidia-smi rows (the FIELDS above), restricted to the timed window when it can be."""
        rows = []
        for line in lines:
            r = [x.strip() for x in line.strip().split(",")]
            if len(r) < 10:
                continue
            try:
                rows.append((cls._epoch(r[0]), float(r[2]), float(r[3]), float(r[4]), r[6:10]))
            except ValueError:
                continue
        in_window = rows
        if window is not None and rows and all(t is not None for t, *_ in rows):
            lo, hi = window[0] - 0.05, window[1] + 0.15
            inside = [x for x in rows if lo <= x[0] <= hi]
            if inside:
                in_window = inside
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = [x[1] for x in in_window]
        power = [x[3] for x in in_window]
        mx = in_window[-1][2] if in_window else None
        reasons = set()
        for x in in_window:
            for n, val in zip(names, x[4]):
                if val.lower() == "active":
                    reasons.add(n)
        loaded = [c for c, p in zip(sm, power) if p > 300] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def kernel_source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sliding_window_attention_chunked_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_key, sources):
    """DRAM bytes per launch from a committed ncu capture, if the kernel is unchanged since."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel_key)
    if not rec or rec.get("source_hash") != kernel_source_hash(*sources):
        return None
    return rec.get("dram_bytes_per_launch")


def replica_seed_base(rank):
    """Each rank runs its own replica of the workload on its own seeded inputs."""
    return 1000 * rank


def max_over_ranks(x, device="cpu"):
    """Max of a per-rank scalar over the default process group (identity on one rank)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, steps, world, ms_max):
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank_step * world * steps / (ms_max / 1e3)


# ------------------------------------------------------------------------------------------
# CPU baseline: the oracle, timed on a bounded sample of the same workload
# ------------------------------------------------------------------------------------------


def oracle_stack_sample(dims):
    """Time the fp64 oracle on a sample of the stack and scale to stack tokens/s.

    Recurrence layer: all 16 heads over the first n tokens (sequential in t, one thread per
    (b,h) unit). SW-SKA layer: full-window rows (t >= W) of random (head, t) pairs. The stack
    time per token is 12 x (recurrence per token + SW-SKA per token)."""
    import numpy as np

    import oracle
    from sliding_window_attention_chunked_b200 import workloads as wl

    H, dk, dv, W, T = dims["H"], dims["dk"], dims["dv"], dims["window"], dims["T"]
    n_gla = 32768
    q, k, v, g = wl.gla_inputs(1, H, n_gla, dk, dv, dist="l2", seed=0)
    t0 = time.perf_counter()
    oracle.gla_prefill(q, k, v, g)
    t_gla = time.perf_counter() - t0
    gla_per_tok = t_gla / n_gla                   # all H heads for one token
    # SW-SKA: rows with a full window
    Ts = W + 64
    qs, ks, vs = wl.swska_inputs(1, H, Ts, dk, dv, dist="l2", seed=1)
    n_rows = 32768
    rng = np.random.default_rng(0)
    hs = rng.integers(0, H, n_rows)
    ts = rng.integers(W - 1, Ts, n_rows)
    rows = hs * Ts + ts
    t0 = time.perf_counter()
    oracle.swska_prefill(qs, ks, vs, W, rows=rows)
    t_ska = time.perf_counter() - t0
    ska_per_tok = t_ska / n_rows * H               # all H heads for one token
    layers = dims["layers"]
    per_tok = (layers // 2) * (gla_per_tok + ska_per_tok)
    cores = oracle.default_threads()
    sample = (f"oracle fp64 on {cores} threads: recurrence {H} heads x {n_gla} tokens "
              f"({t_gla:.2f} s) + SW-SKA {n_rows} full-window rows ({t_ska:.2f} s), scaled to "
              f"the {layers}-layer stack per token")
    return {"value": 1.0 / per_tok, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": sample, "seconds": t_gla + t_ska}


# ------------------------------------------------------------------------------------------
# the GPU arm
# ------------------------------------------------------------------------------------------


def run_gpu(args):
    import torch
    import torch.distributed as dist

    import sliding_window_attention_chunked_b200 as rod
    from sliding_window_attention_chunked_b200 import build as rbuild
    from sliding_window_attention_chunked_b200 import workloads as wl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    if rank == 0:
        rbuild.build()
    if world > 1:
        dist.barrier()
    rod.load_library()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def ranks_max(x):
        return max_over_ranks(x, device=dev)

    d = wl.WORKLOADS[WORKLOAD].dims
    B, H, T, dk, dv, L, W, C = d["B"], d["H"], d["T"], d["dk"], d["dv"], d["layers"], d["window"], d["chunk"]
    seed_base = replica_seed_base(rank)
    layers = []
    for l in range(L):
        ins = wl.stack_layer_inputs(l, B, H, T, dk, dv, seed_base=seed_base, device=dev)
        out = torch.empty(B, H, T, dv, dtype=torch.bfloat16, device=dev)
        st = torch.zeros(B, H, dk, dv, device=dev) if wl.stack_layer_kind(l) == "gla" else None
        layers.append((wl.stack_layer_kind(l), ins, out, st))
    ws_bytes = rod.gla_prefill_workspace_size(B, H, T, dk, dv, C)
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    ska_events = []

    def step(record=False):
        for kind, ins, out, st in layers:
            if kind == "gla":
                q, k, v, g = ins
                st.zero_()
                rod.gla_prefill(q, k, v, g, st, o=out, chunk=C, workspace=ws)
            else:
                q, k, v = ins
                if record:
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                rod.swska_prefill(q, k, v, W, o=out)
                if record:
                    e1.record(stream)
                    ska_events.append((e0, e1))

    with ClockSampler(dev.index) as clk:
        clk.wait_started()
        for _ in range(args.warmup):
            step()
        rod.check()
        barrier()
        n0 = rod.launch_count()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        t_start = time.time()
        ev0.record(stream)
        for _ in range(args.steps):
            step(record=True)
        ev1.record(stream)
        barrier()
        clk.mark(t_start, time.time())
        launches = rod.launch_count() - n0
    rod.check()
    ms_local = ev0.elapsed_time(ev1)
    ms = ranks_max(ms_local)
    ms_per_step = ms / args.steps
    value = job_throughput(B * T, args.steps, world, ms)
    ska_ms = [a.elapsed_time(b) for a, b in ska_events]
    ska_avg_ms = ranks_max(sum(ska_ms) / len(ska_ms))
    clocks = clk.summary()

    peaks, peaks_src = load_peaks()
    ska_flop = 4.0 * (dk + dv) / 2 * swska_pairs(T, W) * B * H  # 2*dk (QK^T) + 2*dv (PV) per pair
    achieved_tflops = ska_flop / (ska_avg_ms / 1e3) / 1e12
    peak_tf = peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops")
    roofline = {"bound": "tensor", "kernel": "rod_swska_prefill", "achieved": round(achieved_tflops, 2),
                "peak": peak_tf, "unit": "TFLOP/s", "frac": round(achieved_tflops / peak_tf, 4),
                "peak_source": f"{peaks_src} (bf16_tflops_sustained: kernel timed inside a long step)",
                "flop_per_launch": ska_flop, "avg_launch_ms": round(ska_avg_ms, 4),
                "traffic": recorded_traffic("swska_prefill_stack", ["swska_prefill_tc.cu", "tc.cuh", "common.cuh"])}

    # ---- batched decode step (recurrence + SW-SKA), 256 sequences ----
    # Timed over rotating input sets so that no iteration finds its state or cache in L2 from
    # the one before: 4 recurrence sets (state 537 MB each, 2.1 GB in all) and 2 SW-SKA sets
    # (4.6 GB of cache each), each set visited once per rotation.
    dd_dims = wl.WORKLOADS["decode_n256"].dims
    N, Wd = dd_dims["N"], dd_dims["window"]
    n_gla_sets, n_ska_sets = 4, 2
    gsets = [wl.decode_inputs(N, H, dk, dv, Wd, seed=seed_base + 77 + i, device=dev)
             for i in range(max(n_gla_sets, n_ska_sets))]
    for i, sset in enumerate(gsets):  # keep the recurrence part of every set, caches of the first two
        if i >= n_ska_sets:
            del sset["k_cache"], sset["v_cache"]
    torch.cuda.empty_cache()
    dd = gsets[0]
    o1 = torch.empty(N, H, dv, dtype=torch.bfloat16, device=dev)
    o2 = torch.empty_like(o1)

    def dec_step(i):
        a, b = gsets[i % n_gla_sets], gsets[i % n_ska_sets]
        rod.gla_decode_step(a["q"], a["k"], a["v"], a["g"], a["state"], o=o1)
        rod.swska_decode(b["sq"], b["k_new"], b["v_new"], b["k_cache"], b["v_cache"],
                         b["pos"], Wd, o=o2)

    for i in range(max(4, args.warmup)):
        dec_step(i)
    rod.check()
    dsteps = max(20, args.steps * 4)
    ge = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(dsteps)]
    se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(dsteps)]
    barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(dsteps):
        a, b = gsets[i % n_gla_sets], gsets[i % n_ska_sets]
        ge[i][0].record(stream)
        rod.gla_decode_step(a["q"], a["k"], a["v"], a["g"], a["state"], o=o1)
        ge[i][1].record(stream)
        se[i][0].record(stream)
        rod.swska_decode(b["sq"], b["k_new"], b["v_new"], b["k_cache"], b["v_cache"],
                         b["pos"], Wd, o=o2)
        se[i][1].record(stream)
    e1.record(stream)
    barrier()
    rod.check()
    dec_ms = ranks_max(e0.elapsed_time(e1) / dsteps)
    gla_dec_ms = ranks_max(sum(a.elapsed_time(b) for a, b in ge) / dsteps)
    ska_dec_ms = ranks_max(sum(a.elapsed_time(b) for a, b in se) / dsteps)
    gla_dec_bytes = 2.0 * N * H * dk * dv * 4 + N * H * (2 * dk * 2 + dk * 4 + dv * 2 + dv * 2)
    ska_dec_bytes = 1.0 * N * Wd * dk * 2 + N * H * Wd * dv * 2 + N * H * (dk + dv + dv) * 2 + N * dk * 2
    hbm = peaks.get("hbm_gbs")

    # the same SW-SKA decode over a paged window cache: pages of 64 slots, shuffled table
    page = 64
    pps = Wd // page
    k_pool = dd["k_cache"].reshape(N * pps, page, dk)
    v_pool = (dd["v_cache"].reshape(N, H, pps, page, dv).permute(0, 2, 1, 3, 4)
              .reshape(N * pps, H, page, dv).contiguous())
    tgen = torch.Generator(device=dev)
    tgen.manual_seed(seed_base + 78)
    table = torch.randperm(N * pps, generator=tgen, device=dev).to(torch.int32).reshape(N, pps)
    for _ in range(3):
        rod.swska_decode_paged(dd["sq"], dd["k_new"], dd["v_new"], k_pool, v_pool, table, page,
                               dd["pos"], Wd, o=o2)
    rod.check()
    pe0, pe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    pe0.record(stream)
    for _ in range(dsteps):
        rod.swska_decode_paged(dd["sq"], dd["k_new"], dd["v_new"], k_pool, v_pool, table, page,
                               dd["pos"], Wd, o=o2)
    pe1.record(stream)
    barrier()
    rod.check()
    paged_ms = ranks_max(pe0.elapsed_time(pe1) / dsteps)
    del v_pool, k_pool, table

    # the same SW-SKA decode over FP8 (E4M3) rings (SALA blog §4.3): one byte per cached element
    kc8 = wl.fp8_codes((N, Wd, dk), seed=seed_base + 81, device=dev)
    vc8 = wl.fp8_codes((N, H, Wd, dv), seed=seed_base + 82, device=dev)
    for _ in range(3):
        rod.swska_decode_fp8(dd["sq"], dd["k_new"], dd["v_new"], kc8, vc8, dd["pos"], Wd, o=o2)
    rod.check()
    fe0, fe1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    fe0.record(stream)
    for _ in range(dsteps):
        rod.swska_decode_fp8(dd["sq"], dd["k_new"], dd["v_new"], kc8, vc8, dd["pos"], Wd, o=o2)
    fe1.record(stream)
    barrier()
    rod.check()
    fp8_ms = ranks_max(fe0.elapsed_time(fe1) / dsteps)
    ska_fp8_bytes = 1.0 * N * Wd * dk + N * H * Wd * dv + N * H * (dk + dv + dv) * 2 + N * dk * 2
    del kc8, vc8
    decode = {
        "workload": "decode_n256 (N=256 sequences x 1 token, H=16, 128x128 fp32 state, "
                    "SW-SKA ring window 4096)",
        "l2": f"rotating input sets: {n_gla_sets} recurrence sets (537 MB of state each), "
              f"{n_ska_sets} SW-SKA sets (4.6 GB of cache each)",
        "value": round(N * world / (dec_ms / 1e3), 1), "unit": "tokens/s",
        "ms_per_step": round(dec_ms, 4),
        # the step as a whole: a kernel's dirty lines can still sit in L2 when it ends and be
        # written back under the next kernel, so the pair's bytes over the pair's time is the
        # fraction free of that shift
        "step_frac_hbm": round((gla_dec_bytes + ska_dec_bytes) / (dec_ms / 1e3) / 1e9 / hbm, 4),
        "kernels": {
            "rod_gla_decode_step": {"bound": "hbm", "avg_launch_ms": round(gla_dec_ms, 4),
                                    "algorithmic_bytes": gla_dec_bytes,
                                    "achieved": round(gla_dec_bytes / (gla_dec_ms / 1e3) / 1e9, 1),
                                    "peak": hbm, "unit": "GB/s",
                                    "frac": round(gla_dec_bytes / (gla_dec_ms / 1e3) / 1e9 / hbm, 4),
                                    "traffic": recorded_traffic("gla_decode_n256",
                                                                ["gla_decode.cu", "common.cuh"])},
            "rod_swska_decode": {"bound": "hbm", "avg_launch_ms": round(ska_dec_ms, 4),
                                 "algorithmic_bytes": ska_dec_bytes,
                                 "achieved": round(ska_dec_bytes / (ska_dec_ms / 1e3) / 1e9, 1),
                                 "peak": hbm, "unit": "GB/s",
                                 "frac": round(ska_dec_bytes / (ska_dec_ms / 1e3) / 1e9 / hbm, 4),
                                 "traffic": recorded_traffic("swska_decode_n256",
                                                             ["swska_decode_warp.cu", "common.cuh", "fp8.cuh"])},
            "rod_swska_decode_paged": {"bound": "hbm", "page_slots": page,
                                       "avg_launch_ms": round(paged_ms, 4),
                                       "algorithmic_bytes": ska_dec_bytes,
                                       "achieved": round(ska_dec_bytes / (paged_ms / 1e3) / 1e9, 1),
                                       "peak": hbm, "unit": "GB/s",
                                       "frac": round(ska_dec_bytes / (paged_ms / 1e3) / 1e9 / hbm, 4),
                                       "note": "not in the step: the same decode over 64-slot pages "
                                               "through a shuffled block table"},
            "rod_swska_decode_fp8": {"bound": "hbm", "avg_launch_ms": round(fp8_ms, 4),
                                     "algorithmic_bytes": ska_fp8_bytes,
                                     "achieved": round(ska_fp8_bytes / (fp8_ms / 1e3) / 1e9, 1),
                                     "peak": hbm, "unit": "GB/s",
                                     "frac": round(ska_fp8_bytes / (fp8_ms / 1e3) / 1e9 / hbm, 4),
                                     "speedup_vs_bf16_cache": round(ska_dec_ms / fp8_ms, 3),
                                     "note": "not in the step: the same decode over E4M3 rings (one "
                                             "byte per cached element, fp32 scales)"},
        },
    }

    # ---- per-layer-type breakdown of the prefill step (GLA layers by difference) ----
    gla_ms_per_layer = (ms_per_step - (L // 2) * ska_avg_ms) / (L // 2)
    gla_bytes = B * H * T * (3 * dk * 2 + dk * 4 + dv * 2) + B * H * dk * dv * 4 * 2
    kernels = {
        "rod_swska_prefill": {"bound": "tensor", "avg_launch_ms": round(ska_avg_ms, 4),
                              "achieved_tflops": round(achieved_tflops, 2)},
        "rod_gla_prefill": {"bound": "hbm", "avg_layer_ms": round(gla_ms_per_layer, 4),
                            "algorithmic_bytes": gla_bytes,
                            "achieved_gbs": round(gla_bytes / (gla_ms_per_layer / 1e3) / 1e9, 1),
                            "frac_hbm": round(gla_bytes / (gla_ms_per_layer / 1e3) / 1e9 / hbm, 4),
                            "traffic": recorded_traffic("gla_prefill_stack",
                                                        ["gla_prefill_tc.cu", "tc.cuh", "common.cuh"])},
    }

    # ---- end to end through the public API with host buffers ----
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, rod, torch, layers, d, ws, stream, barrier, ranks_max, world)

    del layers, dd, gsets
    torch.cuda.empty_cache()

    # ---- generation loop: one token through all 24 layers' decode kernels, eager vs graph ----
    generate = None
    if not args.no_generate:
        generate = run_generate(rod, torch, wl, dev, L, H, dk, W, seed_base, barrier, ranks_max,
                                world)
    backward = None
    if not args.no_backward:
        backward = run_backward(rod, torch, wl, dev, H, dk, W, seed_base, barrier, ranks_max, world)
    configs = None
    if not args.no_configs:
        configs = run_configs(rod, torch, wl, dev, seed_base, barrier, ranks_max, world, rank,
                              with_oracle=(rank == 0 and world == 1 and not args.no_cpu_baseline))
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_stack_sample(d)
        cpu.pop("seconds", None)

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; per-layer inputs drawn on the device, seed = 1000*rank + layer)",
        "config": {"workload": f"{WORKLOAD}: Rodimus+ mixer stack prefill, B=1, T=131072, "
                               "H=16, d=128, 24 layers alternating recurrence (chunk 64) / "
                               "SW-SKA (window 4096)",
                   "global_batch": B * world, "seq_len": T, "layers": L,
                   "parallelism": f"replicas x{world} (independent sequences, no collective)",
                   "l2": "inputs > L2 (55 GB per step), no flush needed"},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
        "clocks": clocks, "decode": decode, "generate": generate, "backward": backward,
        "kernels": kernels, "configs": configs,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_backward(rod, torch, wl, dev, H, d, W, seed_base, barrier, reduce_max, world):
    """Training path: the backward of each mixer on its own configuration, timed with CUDA
    events after a warm-up call. Both run on the tensor cores. The recurrence's backward moves
    about 84 FLOP per algorithmic byte, below the ridge, so its roofline is the measured HBM
    copy bandwidth; the SW-SKA backward is tensor-bound (roofline: the measured dense bf16 peak,
    burst figure: timed alone)."""
    peaks, peaks_src = load_peaks()
    tc_peak = peaks.get("bf16_tflops")
    out = {}

    def timed(fn, iters):
        fn()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        barrier()
        rod.check()
        return reduce_max(e0.elapsed_time(e1) / iters)

    # recurrence: B4 H16 T4096, d 128 (the chunked-prefill workload); 13 dk dv FLOP per
    # head-token (S_t, dq, dS, dk, dv, dg)
    B, T = 4, 4096
    q, k, v, g = wl.gla_inputs(B, H, T, d, d, dist="l2", seed=seed_base + 300, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed_base + 301)
    dO = (torch.randn(B, H, T, d, generator=gen, device=dev) * 0.2).to(q.dtype)
    S0 = torch.zeros(B, H, d, d, device=dev)
    dSf = torch.randn(B, H, d, d, generator=gen, device=dev) * 0.1
    ws = torch.empty(rod.load_library().rod_gla_backward_workspace_size(B, H, T, d, d), dtype=torch.uint8,
                     device=dev)
    ms = timed(lambda: rod.gla_backward(q, k, v, g, dO, S0, dSf, workspace=ws), 10)
    # chunkwise on the tensor cores: algorithmic bytes are the inputs (q, k, v, dO bf16, g fp32)
    # and outputs (dq, dk, dv bf16, dg fp32) per head-token plus the three states per (b, h);
    # algorithmic FLOP per head-token at chunk 64: the ten products of the chunk form
    hbm = peaks.get("hbm_gbs")
    nbytes = B * H * T * (4 * d * 2 + d * 4 + 3 * d * 2 + d * 4) + 3 * B * H * d * d * 4
    flop = B * H * T * (2 * d * (64 + 1) * 3 + 2 * d * d * 5)
    out["gla_backward"] = {"workload": f"B{B} H{H} T{T} d{d} bf16", "ms": round(ms, 3),
                           "tokens_per_s": round(B * T * world / (ms / 1e3), 1),
                           "bound": "hbm", "algorithmic_bytes": nbytes,
                           "achieved": round(nbytes / (ms / 1e3) / 1e9, 1), "peak": hbm, "unit": "GB/s",
                           "frac": round(nbytes / (ms / 1e3) / 1e9 / hbm, 4),
                           "tflops_algorithmic": round(flop / (ms / 1e3) / 1e12, 2),
                           "peak_source": f"{peaks_src} hbm_gbs",
                           "traffic": recorded_traffic("gla_backward_b4_t4096",
                                                       ["gla_backward_tc.cu", "tc.cuh", "common.cuh"]),
                           "note": "chunkwise tensor-core backward (contributions, scans, gradients); "
                                   "its workspace traffic (per-chunk states and contributions) is "
                                   "about 3.5x the algorithmic bytes"}
    del q, k, v, g, dO, S0, dSf, ws
    # SW-SKA: B1 H16 T8192, window W, d 128; algorithmic work 10 d FLOP per (query, key, head)
    # pair inside the window: the five products S = Q K^T, dP = dO V^T, dV = P^T dO,
    # dK = dS^T Q, dQ = dS K (the kernels recompute S and dP, 18 d FLOP per pair in all)
    B, T = 1, 8192
    q, k, v = wl.swska_inputs(B, H, T, d, d, seed=seed_base + 302, device=dev)
    dO = (torch.randn(B, H, T, d, generator=gen, device=dev) * 0.5).to(q.dtype)
    ws = torch.empty(rod.load_library().rod_swska_backward_workspace_size(B, H, T), dtype=torch.uint8,
                     device=dev)
    ms = timed(lambda: rod.swska_backward(q, k, v, dO, W, workspace=ws), 10)
    flop = 10.0 * d * swska_pairs(T, W) * B * H
    out["swska_backward"] = {"workload": f"B{B} H{H} T{T} d{d} window {W} bf16", "ms": round(ms, 3),
                             "tokens_per_s": round(B * T * world / (ms / 1e3), 1),
                             "bound": "tensor", "achieved": round(flop / (ms / 1e3) / 1e12, 1),
                             "peak": tc_peak, "unit": "TFLOP/s",
                             "frac": round(flop / (ms / 1e3) / 1e12 / tc_peak, 4),
                             "peak_source": f"{peaks_src} bf16_tflops (burst: timed alone)",
                             "executed_flop_per_pair": 18 * d}
    # the same gradients from the forward's saved output and log-sum-exp (what a training step
    # keeps from its forward): the statistics pass becomes one read of o, dO and lse, and the
    # kernels execute 14 d FLOP per pair
    o, lse = rod.swska_prefill_lse(q, k, v, W)
    ms_s = timed(lambda: rod.swska_backward_lse(q, k, v, o, lse, dO, W, workspace=ws), 10)
    out["swska_backward_saved_statistics"] = {
        "workload": f"B{B} H{H} T{T} d{d} window {W} bf16, from swska_prefill_lse's o and lse",
        "ms": round(ms_s, 3), "tokens_per_s": round(B * T * world / (ms_s / 1e3), 1),
        "bound": "tensor", "achieved": round(flop / (ms_s / 1e3) / 1e12, 1), "peak": tc_peak,
        "unit": "TFLOP/s", "frac": round(flop / (ms_s / 1e3) / 1e12 / tc_peak, 4),
        "peak_source": f"{peaks_src} bf16_tflops (burst: timed alone)", "executed_flop_per_pair": 14 * d}
    del q, k, v, dO, o, lse
    torch.cuda.empty_cache()
    return out


def run_configs(rod, torch, wl, dev, seed_base, barrier, reduce_max, world, rank, with_oracle):
    """The three single-mixer workloads beside the stack, each with its own throughput, its
    roofline fraction and the oracle timed on the host cores (rank 0, one GPU only):
      tiny_fp32                 both mixers, B1 T256 H2 dk16 dv32 (latency-bound: no fraction)
      gla_prefill_b4_t4096      recurrence prefill, HBM-bound
      swska_prefill_b2_t32768   SW-SKA prefill, tensor-bound (burst bf16 peak: timed alone)
    Launches of the two large ones are timed one by one with CUDA events, with a read of a
    512 MB buffer between them (outside the events) so that every launch starts with its
    inputs out of L2 and with no dirty lines of the previous launch left to write back."""
    import numpy as np

    import oracle

    peaks, peaks_src = load_peaks()
    hbm, tc_peak = peaks.get("hbm_gbs"), peaks.get("bf16_tflops")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    out = {}

    def timed_flushed(fn, iters):
        fn()
        barrier()
        ts = []
        for _ in range(iters):
            flush.sum(dtype=torch.int64)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1))
        rod.check()
        return reduce_max(statistics.median(ts))

    def timed_loop(fn, iters):
        fn()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(iters):
            fn()
        e1.record()
        barrier()
        rod.check()
        return reduce_max(e0.elapsed_time(e1) / iters)

    def oracle_timed(fn):
        t0 = time.perf_counter()
        fn()
        return time.perf_counter() - t0

    cores = oracle.default_threads()
    # ---- tiny fp32: both mixers, every product an fp32 FMA (CUDA cores) ----
    d = wl.WORKLOADS["tiny_fp32"].dims
    B, T, H, dk, dv, C, W = d["B"], d["T"], d["H"], d["dk"], d["dv"], d["chunk"], d["window"]
    q, k, v, g = wl.gla_inputs(B, H, T, dk, dv, dist="tiny", seed=seed_base, dtype="fp32")
    sq, sk, sv = wl.swska_inputs(B, H, T, dk, dv, dist="tiny", seed=seed_base + 1, dtype="fp32")
    gq, gk, gv, gg = [t.to(dev) for t in (q, k, v, g)]
    dq_, dk_, dv_ = [t.to(dev) for t in (sq, sk, sv)]
    st = torch.zeros(B, H, dk, dv, device=dev)
    o1 = torch.empty(B, H, T, dv, device=dev)
    o2 = torch.empty(B, H, T, dv, device=dev)
    gla_ms = timed_loop(lambda: rod.gla_prefill(gq, gk, gv, gg, st.zero_(), o=o1, chunk=C), 200)
    ska_ms = timed_loop(lambda: rod.swska_prefill(dq_, dk_, dv_, W, o=o2), 200)
    ent = {"workload": "tiny_fp32: recurrence + SW-SKA, B1 T256 H2 dk16 dv32 chunk 32 window 64, fp32",
           "bound": "latency", "frac": None,
           "gla_prefill_us": round(gla_ms * 1e3, 2), "swska_prefill_us": round(ska_ms * 1e3, 2),
           "value": round(B * T * world / ((gla_ms + ska_ms) / 1e3), 1),
           "unit": "tokens/s (both mixers)"}
    if with_oracle:
        reps = 20
        sec = oracle_timed(lambda: [(oracle.gla_prefill(q, k, v, g), oracle.swska_prefill(sq, sk, sv, W))
                                    for _ in range(reps)]) / reps
        ent["cpu_baseline"] = {"value": round(B * T / sec, 1), "unit": "tokens/s (both mixers)",
                               "cores": cores, "kind": "oracle", "sample": "the whole workload"}
    out["tiny_fp32"] = ent
    del gq, gk, gv, gg, dq_, dk_, dv_, st, o1, o2

    # ---- recurrence prefill B4 T4096 H16 d128 chunk 64 (HBM-bound) ----
    d = wl.WORKLOADS["gla_prefill_b4_t4096"].dims
    B, T, H, dk, dv, C = d["B"], d["T"], d["H"], d["dk"], d["dv"], d["chunk"]
    q, k, v, g = wl.gla_inputs(B, H, T, dk, dv, dist="l2", seed=seed_base + 2, device=dev)
    st = torch.zeros(B, H, dk, dv, device=dev)
    o = torch.empty(B, H, T, dv, dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(rod.gla_prefill_workspace_size(B, H, T, dk, dv, C), 16), dtype=torch.uint8, device=dev)
    ms = timed_flushed(lambda: rod.gla_prefill(q, k, v, g, st.zero_(), o=o, chunk=C, workspace=ws), 20)
    nbytes = B * H * T * (3 * dk * 2 + dk * 4 + dv * 2) + B * H * dk * dv * 4 * 2
    flop = B * H * T * (2 * dk * (C + 1) / 2 * 2 + 4 * dk * dv)  # intra QK + AV, readout, state
    ent = {"workload": "gla_prefill_b4_t4096: recurrence prefill, B4 T4096 H16 d128 chunk 64, bf16 in, "
                       "fp32 gates and state",
           "ms": round(ms, 4), "value": round(B * T * world / (ms / 1e3), 1), "unit": "tokens/s",
           "bound": "hbm", "algorithmic_bytes": nbytes,
           "achieved": round(nbytes / (ms / 1e3) / 1e9, 1), "peak": hbm, "peak_unit": "GB/s",
           "frac": round(nbytes / (ms / 1e3) / 1e9 / hbm, 4),
           "tflops_algorithmic": round(flop / (ms / 1e3) / 1e12, 2),
           "traffic": recorded_traffic("gla_prefill_b4_t4096", ["gla_prefill_tc.cu", "tc.cuh", "common.cuh"])}
    del q, k, v, g, st, o, ws
    if with_oracle:
        qh, kh, vh, gh = wl.gla_inputs(B, H, T, dk, dv, dist="l2", seed=seed_base + 2)
        sec = oracle_timed(lambda: oracle.gla_prefill(qh, kh, vh, gh))
        ent["cpu_baseline"] = {"value": round(B * T / sec, 1), "unit": "tokens/s", "cores": cores,
                               "kind": "oracle", "sample": f"the whole workload ({sec:.2f} s)"}
        del qh, kh, vh, gh
    out["gla_prefill_b4_t4096"] = ent

    # ---- SW-SKA prefill B2 T32768 H16 d128 window 4096 (tensor-bound) ----
    d = wl.WORKLOADS["swska_prefill_b2_t32768"].dims
    B, T, H, dk, dv, W = d["B"], d["T"], d["H"], d["dk"], d["dv"], d["window"]
    q, k, v = wl.swska_inputs(B, H, T, dk, dv, seed=seed_base + 3, device=dev)
    o = torch.empty(B, H, T, dv, dtype=torch.bfloat16, device=dev)
    ms = timed_flushed(lambda: rod.swska_prefill(q, k, v, W, o=o), 10)
    flop = 2.0 * (dk + dv) * swska_pairs(T, W) * B * H
    nbytes = B * H * T * (dk + 2 * dv) * 2 + B * T * dk * 2
    ent = {"workload": "swska_prefill_b2_t32768: SW-SKA prefill, B2 T32768 H16 d128 window 4096, bf16",
           "ms": round(ms, 4), "value": round(B * T * world / (ms / 1e3), 1), "unit": "tokens/s",
           "bound": "tensor", "flop": flop, "achieved": round(flop / (ms / 1e3) / 1e12, 1),
           "peak": tc_peak, "peak_unit": "TFLOP/s",
           "peak_source": f"{peaks_src} bf16_tflops (burst: timed alone)",
           "frac": round(flop / (ms / 1e3) / 1e12 / tc_peak, 4),
           "achieved_gbs": round(nbytes / (ms / 1e3) / 1e9, 1)}
    del q, k, v, o
    if with_oracle:
        qh, kh, vh = wl.swska_inputs(B, H, T, dk, dv, seed=seed_base + 3)
        n_rows = 8192
        rng = np.random.default_rng(3)
        rows = rng.integers(0, B * H * T, n_rows)
        # the cost of a row is its window length: scale by the workload's mean window length
        tt = rows % T
        mean_w_sample = float(np.mean(np.minimum(tt + 1, W)))
        mean_w_all = swska_pairs(T, W) / T
        sec = oracle_timed(lambda: oracle.swska_prefill(qh, kh, vh, W, rows=rows))
        sec_all = sec / n_rows * (B * H * T) * mean_w_all / mean_w_sample
        ent["cpu_baseline"] = {"value": round(B * T / sec_all, 2), "unit": "tokens/s", "cores": cores,
                               "kind": "oracle",
                               "sample": f"{n_rows} random output rows ({sec:.2f} s), scaled to the whole "
                                         "workload by window length"}
        del qh, kh, vh
    out["swska_prefill_b2_t32768"] = ent
    del flush
    torch.cuda.empty_cache()
    return out


def run_generate(rod, torch, wl, dev, L, H, d, W, seed_base, barrier, reduce_max, world):
    """Per-token decode step of the whole L-layer stack (every layer's decode kernel, then the
    position advance) for N sequences with full windows: eager launches against one CUDA-graph
    replay per token. Caches, states and per-step inputs are seeded random, resident in HBM."""
    from sliding_window_attention_chunked_b200.generate import MixerStack

    out = {"workload": f"{L}-layer Rodimus+ decode step (alternating recurrence / SW-SKA, H={H}, "
                       f"d={d}, window {W}, full windows), one token per sequence",
           "unit": "ms per token step", "runs": []}
    for N in (1, 256):
        stack = MixerStack(L, N, H, d, W, device=dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(seed_base + 9000 + N)
        for lay in stack.layers:
            for key, t in lay.items():
                if key == "g":
                    t.uniform_(0.9, 1.0, generator=gen)
                else:
                    t.normal_(generator=gen)
        pos = wl.decode_positions(N, W, full=True, device=dev)
        stack.pos.copy_(pos)
        for _ in range(3):
            stack.step_eager()
        rod.check()
        steps = 50 if N == 1 else 20

        def timed(fn):
            barrier()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(steps):
                fn()
            e1.record()
            barrier()
            return reduce_max(e0.elapsed_time(e1) / steps)

        eager_ms = timed(stack.step_eager)
        stack.capture()
        for _ in range(3):
            stack.step()
        graph_ms = timed(stack.step)
        rod.check()
        out["runs"].append({"N": N, "eager_ms": round(eager_ms, 4), "graph_ms": round(graph_ms, 4),
                            "graph_tokens_per_s": round(N * world / (graph_ms / 1e3), 1),
                            "kernels_per_step": stack.kernels_per_step()})
        del stack
        torch.cuda.empty_cache()
    return out


def run_e2e(args, rod, torch, layers, d, ws, stream, barrier, reduce_max, world):
    """Same stack, but every step copies each layer's inputs from pinned host memory into the
    device buffers and reads each layer's output back to pinned host memory. The copies run as a
    pipeline on their own streams: layer l+1's inputs go up and layer l-1's output comes down
    (the link is full duplex) while layer l computes. Events order each layer's copy-in, kernel
    and copy-out, and across steps a layer's buffers are rewritten only after their last use."""
    B, T, C, W = d["B"], d["T"], d["chunk"], d["window"]
    host = {}
    for kind, ins, out, st in layers:
        if kind not in host:
            host[kind] = ([t.to("cpu").pin_memory() for t in ins],
                          torch.empty(out.shape, dtype=out.dtype).pin_memory())
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()
    n_l = len(layers)
    in_done = [ev() for _ in range(n_l)]
    comp_done = [ev() for _ in range(n_l)]
    out_done = [ev() for _ in range(n_l)]
    first = [True]
    h2d = d2h = 0

    def step():
        nonlocal h2d, d2h
        h2d = d2h = 0
        for i, (kind, ins, out, st) in enumerate(layers):
            hin, hout = host[kind]
            with torch.cuda.stream(s_in):
                if not first[0]:
                    s_in.wait_event(comp_done[i])  # the previous step's kernel has read these inputs
                for dst, src in zip(ins, hin):
                    dst.copy_(src, non_blocking=True)
                    h2d += src.numel() * src.element_size()
                in_done[i].record(s_in)
            stream.wait_event(in_done[i])
            if not first[0]:
                stream.wait_event(out_done[i])  # the previous step's output has been read back
            if kind == "gla":
                st.zero_()
                rod.gla_prefill(ins[0], ins[1], ins[2], ins[3], st, o=out, chunk=C, workspace=ws)
            else:
                rod.swska_prefill(ins[0], ins[1], ins[2], W, o=out)
            comp_done[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[i])
                hout.copy_(out, non_blocking=True)
                d2h += out.numel() * out.element_size()
                out_done[i].record(s_out)
        first[0] = False

    def join():  # the timing stream waits for both copy streams
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    step()
    join()
    torch.cuda.synchronize()
    barrier()
    n = args.e2e_steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for _ in range(n):
        step()
    join()
    e1.record(stream)
    barrier()
    ms = reduce_max(e0.elapsed_time(e1))
    return {"value": round(job_throughput(B * T, n, world, ms), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n,
            "note": "pinned host buffers per layer kind reused for every layer; copy-in, kernels "
                    "and copy-out pipelined on three streams"}


# ------------------------------------------------------------------------------------------
# the reference arm: the oracle, timed on the host cores
# ------------------------------------------------------------------------------------------


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    from sliding_window_attention_chunked_b200 import workloads as wl
    d = wl.WORKLOADS[WORKLOAD].dims
    for _ in range(args.warmup):
        oracle_stack_sample(d)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        r = oracle_stack_sample(d)
        vals.append(r["value"])
        secs += r.pop("seconds")
    value = statistics.mean(vals)
    r["value"] = value
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * secs / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": f"{WORKLOAD}: Rodimus+ mixer stack prefill (bounded sample, "
                               "scaled per token)", "seq_len": d["T"], "layers": d["layers"]},
        "cpu_baseline": r,
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """One kernel family on one layer of the stack workload (or one decode batch), for ncu:
    warm-up + steps launches, each timed with CUDA events; no stack, no e2e, no oracle. The
    device holds one layer's inputs (about 1.6 GB for SW-SKA, 3 GB for the recurrence) or the
    decode caches of --profile-n sequences (17 MiB each)."""
    import torch

    import sliding_window_attention_chunked_b200 as rod
    from sliding_window_attention_chunked_b200 import build as rbuild
    from sliding_window_attention_chunked_b200 import workloads as wl

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    rbuild.build()
    rod.load_library()
    d = wl.WORKLOADS[WORKLOAD].dims
    B, H, T, dk, dv, W, C = d["B"], d["H"], d["T"], d["dk"], d["dv"], d["window"], d["chunk"]
    case = args.profile_case
    if args.profile_t:
        T = args.profile_t
    if args.profile_b:
        B = args.profile_b
    if case in ("ska_prefill", "gla_prefill"):
        layer = 1 if case == "ska_prefill" else 0
        ins = wl.stack_layer_inputs(layer, B, H, T, dk, dv, device=dev)
        out = torch.empty(B, H, T, dv, dtype=torch.bfloat16, device=dev)
        if case == "ska_prefill":
            q, k, v = ins
            fn = lambda: rod.swska_prefill(q, k, v, W, o=out)
        else:
            q, k, v, g = ins
            st = torch.zeros(B, H, dk, dv, device=dev)
            ws = torch.empty(max(rod.gla_prefill_workspace_size(B, H, T, dk, dv, C), 16),
                             dtype=torch.uint8, device=dev)
            fn = lambda: rod.gla_prefill(q, k, v, g, st.zero_(), o=out, chunk=C, workspace=ws)
    elif case == "gla_backward":  # B4 H16 T4096 (the backward line of the bench)
        q, k, v, g = wl.gla_inputs(4, H, 4096, dk, dv, dist="l2", seed=300, device=dev)
        dO = (torch.randn(4, H, 4096, dv, device=dev) * 0.2).to(q.dtype)
        S0 = torch.zeros(4, H, dk, dv, device=dev)
        fn = lambda: rod.gla_backward(q, k, v, g, dO, S0, None)
    elif case == "ska_backward":  # B1 H16 T8192, window W
        q, k, v = wl.swska_inputs(1, H, 8192, dk, dv, seed=302, device=dev)
        dO = (torch.randn(1, H, 8192, dv, device=dev) * 0.5).to(q.dtype)
        fn = lambda: rod.swska_backward(q, k, v, dO, W)
    else:
        N, Wd = args.profile_n, wl.WORKLOADS["decode_n256"].dims["window"]
        dd = wl.decode_inputs(N, H, dk, dv, Wd, seed=77, device=dev)
        o = torch.empty(N, H, dv, dtype=torch.bfloat16, device=dev)
        if case == "ska_decode":
            fn = lambda: rod.swska_decode(dd["sq"], dd["k_new"], dd["v_new"], dd["k_cache"],
                                          dd["v_cache"], dd["pos"], Wd, o=o)
        elif case == "ska_decode_fp8":  # E4M3 rings
            kc8 = wl.fp8_codes((N, Wd, dk), seed=81, device=dev)
            vc8 = wl.fp8_codes((N, H, Wd, dv), seed=82, device=dev)
            fn = lambda: rod.swska_decode_fp8(dd["sq"], dd["k_new"], dd["v_new"], kc8, vc8, dd["pos"], Wd, o=o)
        elif case == "ska_decode_paged":  # pages of 64 slots, shuffled table
            page, pps = 64, Wd // 64
            k_pool = dd["k_cache"].reshape(N * pps, page, dk)
            v_pool = (dd["v_cache"].reshape(N, H, pps, page, dv).permute(0, 2, 1, 3, 4)
                      .reshape(N * pps, H, page, dv).contiguous())
            table = torch.randperm(N * pps, device=dev).to(torch.int32).reshape(N, pps)
            fn = lambda: rod.swska_decode_paged(dd["sq"], dd["k_new"], dd["v_new"], k_pool, v_pool,
                                                table, page, dd["pos"], Wd, o=o)
        else:
            fn = lambda: rod.gla_decode_step(dd["q"], dd["k"], dd["v"], dd["g"], dd["state"], o=o)
    for _ in range(args.warmup):
        fn()
    rod.check()
    times = []
    for _ in range(args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    rod.check()
    print(json.dumps({"profile_case": case, "launch_ms": [round(t, 4) for t in times],
                      "n": args.profile_n if "decode" in case else None}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="rod", choices=["rod", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-generate", action="store_true")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--no-configs", action="store_true")
    ap.add_argument("--profile-case", choices=["ska_prefill", "gla_prefill", "ska_decode", "gla_decode",
                                               "ska_decode_paged", "ska_decode_fp8", "gla_backward",
                                               "ska_backward"],
                    help="run one kernel family alone (for ncu captures) and exit")
    ap.add_argument("--profile-n", type=int, default=128, help="sequences for the decode cases")
    ap.add_argument("--profile-t", type=int, default=0,
                    help="tokens per sequence for the prefill cases (default: the stack's 131072)")
    ap.add_argument("--profile-b", type=int, default=0,
                    help="sequences for the prefill cases (default: the stack's 1)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # timing rule: at least 3 untimed warm-up steps
    if args.profile_case:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
