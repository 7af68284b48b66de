#!/usr/bin/env python
"""Benchmark of the NOSA decode step on B200 (one JSON line on rank 0).

Workload (default): offloaded batch decode at B=64 -- 32 query / 8 KV heads,
head_dim 128, 4096-token context (64 blocks of 64), budget 16 blocks (12
query-aware + 4 agnostic, overlap >= 13), full KV in pinned host memory, GPU
block cache of 32 blocks per (sequence, KV head), AR(1) queries rho = 0.95.

A step is one pass of the whole path: score -> select -> fetch (plan + PCIe
gather of the misses) -> sparse attention, captured once in a CUDA graph and
replayed.  Step 0 (cold cache) and the other warm-up steps run eagerly and are
not timed.  The per-step traffic (256 MiB of selected K/V + 32 MiB of pooled
keys) exceeds the 126 MB L2, so no flush is needed between steps.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--workload NAME]

Under torchrun every rank runs its own copy of the workload on its own GPU
(weak scaling, no collective on the data path); rank 0 prints the line with
the max-over-ranks time.
"""

from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NOSA decode tokens/s at B=64 (1 GPU); HBM & PCIe GB/s vs roofline"
UNIT = "tokens/s"
HBM_NOMINAL_GBS = 8000.0


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=4000)
    p.add_argument("--warmup", type=int, default=8)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--workload", default="offload_b64")
    p.add_argument("--policy", default="nosa", choices=["nosa", "paper", "infllmv2", "full"],
                   help="selection policy on the same kernels (see configs.POLICIES)")
    p.add_argument("--k-query", type=int, default=None,
                   help="query-aware blocks of the 64-block budget (paper policy; default 16)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--e2e-steps", type=int, default=500)
    return p.parse_args()


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms; only the
    samples whose timestamps fall inside the timed window are summarised."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        # the raw samples (NOSA_CLOCKS_DIR, default the temp directory); the
        # bench line carries their summary
        import tempfile
        d = os.environ.get("NOSA_CLOCKS_DIR") or tempfile.gettempdir()
        self.path = os.path.join(d, "nosa_clocks_%s.csv" % gpu_id.replace(":", "_").replace(".", "_"))
        self.t0 = self.t1 = None

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=self.f, stderr=subprocess.STDOUT)
        except Exception:
            self.proc = None

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        import datetime
        sm, smax, pw, reasons, n_all = [], [], [], set(), 0
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                clk, cmax = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            n_all += 1
            if self.t0 is not None and not (self.t0 <= ts <= self.t1):
                continue
            sm.append(clk)
            smax.append(cmax)
            try:
                pw.append(float(parts[4]))
            except ValueError:
                pass
            for n, v in zip(names, parts[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "samples_total": n_all}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(pw) if pw else None}


# ------------------------------------------------------------------ helpers
def max_over_ranks(torch, dist, ms_local, device, world):
    """The slowest rank's timed-region length (every rank takes part)."""
    t = torch.tensor([float(ms_local)], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gpu_pci_bus_id(torch, local):
    """PCI bus id of CUDA device `local` (NVML and nvidia-smi number devices
    differently once CUDA_VISIBLE_DEVICES is set)."""
    pr = torch.cuda.get_device_properties(local)
    return f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"


def bind_to_gpu_numa_node(bus_id):
    """Restrict this process to the CPUs nearest the GPU before any pinned
    allocation, so that pinned host memory (the offloaded KV the gather reads
    over PCIe) is allocated on the GPU's NUMA node.  Reads the affinity from
    NVML; changes no GPU setting.  Returns the CPU count, or None."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByPciBusId(bus_id)
            ncpu = os.cpu_count() or 1
            words = pynvml.nvmlDeviceGetCpuAffinity(h, (ncpu + 63) // 64)
        finally:
            pynvml.nvmlShutdown()
        cpus = {64 * i + b for i, wd in enumerate(words) for b in range(64) if (int(wd) >> b) & 1}
        cpus &= os.sched_getaffinity(0)
        if not cpus:
            return None
        os.sched_setaffinity(0, cpus)
        return len(cpus)
    except Exception:
        return None


def job_tokens_per_s(world, batch, steps, ms_max):
    """Whole-job throughput: every rank decodes `batch` tokens per step."""
    return world * batch * steps / (ms_max * 1e-3)


def measured_peaks():
    try:
        return json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
    except Exception:
        return {}


def hbm_bytes_per_step(w, fetched_blocks_per_step):
    """Algorithmic HBM bytes of one step: pooled keys, scores (fp64 write +
    read), agnostic scores, selected K+V, cache writes of fetched blocks, q and
    out."""
    U, n, R, d = w.units, w.n_blocks0, w.block // w.sub_block, w.head_dim
    pooled = U * n * R * d * 2
    scores = U * n * 8 * 2
    agn = U * n * 4
    selected = U * w.k * w.block * d * 2 * 2
    writes = fetched_blocks_per_step * w.block * d * 2 * 2
    qo = w.batch * w.n_q_heads * d * 2 * 2
    return pooled + scores + agn + selected + writes + qo


def measure_h2d_peak(torch, dev, mib=256, reps=3):
    """Copy-engine host->device bandwidth from pinned memory (GB/s)."""
    n = mib * (1 << 20)
    src = torch.empty(n, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(n, dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(dev)
    best = 0.0
    with torch.cuda.stream(s):
        for _ in range(reps + 1):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(s)
            dst.copy_(src, non_blocking=True)
            e1.record(s)
            s.synchronize()
            best = max(best, n / (e0.elapsed_time(e1) * 1e-3) / 1e9)
    del src, dst
    return best


def cpu_baseline(w, target_s=12.0):
    """The oracle, as it stands, on a bounded sample of the workload on the
    host cores (OpenMP over units).  Returns (tokens/s, cores, sample text)."""
    import numpy as np
    import oracle
    from kv_cache_decode_step_b200 import inputs

    def run(n_units, steps):
        units = list(range(n_units))
        d = inputs.generate(w.with_(steps=steps), units=units)
        cfg = oracle.cfg_from_workload(w, steps=steps)
        t0 = time.perf_counter()
        _, _, _, th = oracle.run_units(cfg, d["k"], d["v"], d["a"], d["q"], attend_steps=None)
        return time.perf_counter() - t0, th

    t_probe, th = run(min(w.units, 32), 4)
    per_unit_step = t_probe / (min(w.units, 32) * 4)  # wall time per unit-step, all cores
    n_units = w.units
    steps = max(2, min(256, int(target_s / max(per_unit_step * n_units, 1e-6))))
    t, th = run(n_units, steps)
    step_time = t / steps * (w.units / n_units)
    return (w.batch / step_time, th,
            f"oracle on {n_units} of {w.units} units x {steps} steps (all phases, attention every "
            f"step), scaled to the full batch; {t:.1f} s of CPU work")


def workload_config(w, policy, world):
    """The bench line's `config`: the workload alone, identical for both arms."""
    hbm_lo = hbm_bytes_per_step(w, 0)
    return {"workload": w.name, "policy": policy, "batch": w.batch, "context": w.context,
            "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "block": w.block, "sub_block": w.sub_block, "k": w.k, "k_query": w.k_query,
            "k_agnostic": w.k_agnostic, "min_overlap": w.min_overlap, "sink_blocks": w.sink_blocks,
            "window_blocks": w.window_blocks, "cache_slots": w.cache_slots,
            "kv": "pinned host" if w.offloaded else "HBM", "parallelism": f"replicas x{world}",
            "l2": (f"per-step HBM traffic >= {hbm_lo / 2**20:.0f} MiB "
                   + ("> 126 MB L2, no flush" if hbm_lo > 126e6 else "< 126 MB L2, not flushed"))}


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank, world, local = dist_env()
    if rank != 0:
        return
    from kv_cache_decode_step_b200 import configs
    import oracle
    from kv_cache_decode_step_b200 import inputs
    base_w = configs.with_policy(configs.get(args.workload), args.policy, args.k_query)
    w = base_w
    # bounded sample per step: a few units of the workload, scaled to the batch
    n_units = min(w.units, 16)
    steps = args.warmup + args.steps
    d = inputs.generate(w.with_(steps=max(steps, 2)), units=list(range(n_units)))
    cfg = oracle.cfg_from_workload(w, steps=max(steps, 2))
    t0 = time.perf_counter()
    _, _, _, th = oracle.run_units(cfg, d["k"], d["v"], d["a"], d["q"], attend_steps=None)
    t = time.perf_counter() - t0
    step_time = t / max(steps, 2) * (w.units / n_units)
    value = w.batch / step_time
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_time * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 K/V, U(0,1) agnostic scores, AR(1) queries)",
        "config": workload_config(base_w, args.policy, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": th, "kind": "oracle",
                         "sample": f"fp64 CPU oracle on {n_units} of {w.units} units x {max(steps, 2)} "
                                   f"steps, scaled to the full batch"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    from kv_cache_decode_step_b200 import build, configs, inputs, nosa, runner

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    bus_id = gpu_pci_bus_id(torch, local)
    numa_cpus = bind_to_gpu_numa_node(bus_id)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    build.build()

    base = configs.with_policy(configs.get(args.workload), args.policy, args.k_query)
    # With KV in host memory every step of the run gets a fresh query of the
    # seeded AR(1) stream: revisiting queries would find their blocks still in
    # the cache and understate the misses.  The timed steps are capped so the
    # queries fit a memory budget (growing sequences: their KV capacity).
    # With KV in HBM there is no cache state, and queries are reused past the
    # workload's last step.
    untimed = (1 + args.warmup + 1 + 32 + WARM_STEPS + 2 * min(args.steps, 50) + 2 * (args.e2e_steps + 4)
               + LATENCY_STEPS + 8)
    q_step_bytes = base.batch * base.n_q_heads * base.head_dim * 2
    if base.append:
        timed_cap = max(args.steps, APPEND_TIMED_STEPS)
    elif base.offloaded:
        timed_cap = max(args.steps, min(MAX_QUERY_STEPS, int(QUERY_BUDGET_BYTES // q_step_bytes)) - untimed)
    else:
        timed_cap = None
    w = base.with_(steps=max(base.steps, untimed + timed_cap)) if timed_cap is not None else base
    data = inputs.generate(w)
    dec = runner.Decoder(w, data, device=local)

    h2d_peak = measure_h2d_peak(torch, dev)

    # warm-up: step 0 (cold cache) plus W eager steps
    for _ in range(1 + args.warmup):
        dec.step()
    dec.stream.synchronize()
    dec.capture()
    dec.replay()  # one untimed replay
    dec.stream.synchronize()
    nosa.nosa_reset_stats(dec.ctx, dec.stream)

    # ---- timed region: the K-replay block, repeated until at least
    # MIN_TIMED_MS of GPU time has passed (so the clock sampler sees the run and
    # start-up cost drops out); every rank repeats it the same number of times
    est = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(8):
        dec.replay()
    est[0].record(dec.stream)
    for _ in range(24):
        dec.replay()
    est[1].record(dec.stream)
    torch.cuda.synchronize()
    est_ms = est[0].elapsed_time(est[1]) / 24
    repeats = max(1, math.ceil(1.2 * MIN_TIMED_MS / max(est_ms * args.steps, 1e-3)))
    if timed_cap is not None:
        repeats = max(1, min(repeats, timed_cap // args.steps))
    repeats = int(max_over_ranks(torch, dist, repeats, dev, world))
    nosa.nosa_reset_stats(dec.ctx, dec.stream)
    clocks = ClockSampler(bus_id)
    clocks.start()
    time.sleep(1.0)  # let the sampler start before the timed window
    # the GPU idled during the sleep: untimed steps bring it back to speed
    for _ in range(WARM_STEPS):
        dec.replay()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark_start()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(repeats + 1)]
    ev[0].record(dec.stream)
    for r in range(repeats):
        for _ in range(args.steps):
            dec.replay()
        ev[r + 1].record(dec.stream)
    torch.cuda.synchronize()
    clocks.mark_end()
    if world > 1:
        dist.barrier()
    clk = clocks.stop()
    ms = ev[0].elapsed_time(ev[repeats])
    block_ms = [ev[r].elapsed_time(ev[r + 1]) for r in range(repeats)]
    st = dec.stats()
    dec.check()
    steps_timed = repeats * args.steps
    ms_max = max_over_ranks(torch, dist, ms, dev, world)
    ms_step = ms_max / steps_timed
    value = job_tokens_per_s(world, w.batch, steps_timed, ms_max)

    fetched_blocks = st["misses"] / steps_timed
    pcie_bytes = st["fetched_bytes"] / steps_timed
    hbm_bytes = hbm_bytes_per_step(w, fetched_blocks)
    peaks = measured_peaks()
    hbm_meas = float(peaks.get("hbm_gbs", 6650.0))
    hbm_src = "of measured" if "hbm_gbs" in peaks else "of fallback"
    t_hbm = hbm_bytes / (HBM_NOMINAL_GBS * 1e9)
    t_hbm_meas = hbm_bytes / (hbm_meas * 1e9)
    t_pcie = pcie_bytes / (h2d_peak * 1e9)
    step_s = ms_step * 1e-3

    # ---- instrumented passes: per-phase events between the ABI calls.  With
    # the side copy stream the gather's own duration is visible; with a single
    # stream the attention launches no longer wait on it.
    phase = instrumented_pass(torch, dec, w, nosa, n=min(args.steps, 50), single_stream=False)
    phase1 = instrumented_pass(torch, dec, w, nosa, n=min(args.steps, 50), single_stream=True)
    phase["attention_ms"] = phase1["decode_ms"]
    phase["single_stream_step_ms"] = phase1["step_ms"]
    phase["note"] = ("graph-captured step with timing events between the ABI calls; gather_ms (the fused "
                     "gather + miss attention, from the end of the plan to the end of the step, the hits pass "
                     "running beside it and ending first: hits_side_ms) from the side-stream pass; "
                     "attention_ms = the decode call of a single-stream pass (KV in HBM: the hits pass; KV in "
                     "host memory: the gather + miss attention, then the hits pass)")

    latency = step_latency_pass(torch, dec, w, LATENCY_STEPS)

    # ---- end to end through host buffers: q from pinned host, out to pinned host
    e2e = e2e_pass(torch, dec, w, nosa, args.e2e_steps, dist=dist, world=world, dev=dev)
    e2e["host_wait_value"] = e2e_pass(torch, dec, w, nosa, args.e2e_steps, host_wait=True, dist=dist,
                                      world=world, dev=dev)["value"]

    # kernels per step: score, select, [plan, gather + miss attention], hits
    # pass -- the fused entry point makes score, select and plan one kernel up
    # to 512 blocks per unit and two (the scoring grid, then select + plan) up
    # to 1024; with appends also append, close and advance (otherwise the last
    # unit merged ends the step), and with KV in host memory the write-through
    # of a block the previous step closed
    if dec.fused and w.max_blocks <= 512:
        first_half, calls = 1, "nosa_score_select_fetch (one kernel) + nosa_sparse_decode"
    elif dec.fused and w.max_blocks <= 1024:
        first_half = 2
        calls = "nosa_score_select_fetch (scoring grid + select/plan kernel) + nosa_sparse_decode"
    else:
        # beyond 1024 blocks nosa_score_select_fetch makes these three calls itself
        first_half = 3 if w.offloaded else 2
        calls = "nosa_score_blocks + nosa_select + nosa_fetch_missing + nosa_sparse_decode"
    launches_per_step = first_half + (2 if w.offloaded else 1) \
        + (3 if w.append else 0) + (1 if w.append and w.offloaded else 0)
    gather_ms = phase["gather_ms"]
    attn_ms = phase["attention_ms"]
    gather_gbs = (phase["fetched_bytes_per_step"] / (gather_ms * 1e-3) / 1e9) if gather_ms > 0 else 0.0
    attn_bytes = w.units * w.k * w.block * w.head_dim * 2 * 2 + w.batch * w.n_q_heads * w.head_dim * 2 * 2
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9 if attn_ms > 0 else 0.0
    rl_gather = {"kernel": "gather_attend_kernel", "bound": "pcie", "achieved": gather_gbs, "peak": h2d_peak,
                 "unit": "GB/s", "frac": gather_gbs / h2d_peak if h2d_peak else None, "traffic": None,
                 "peak_source": "pinned cudaMemcpyAsync H2D measured in this run (256 MiB)",
                 "bytes_per_launch": phase["fetched_bytes_per_step"], "ms_per_launch": gather_ms}
    rl_attn = {"kernel": "attend_hits_ws_kernel", "bound": "hbm", "achieved": attn_gbs,
               "peak": hbm_meas, "unit": "GB/s", "frac": attn_gbs / hbm_meas, "traffic": None,
               "peak_source": f"hbm_gbs {hbm_src}", "bytes_per_launch": attn_bytes, "ms_per_launch": attn_ms}
    if w.offloaded:
        # the hits pass runs beside the gather (and, on one stream, after it):
        # its own duration is not separable from the step's events
        dominant, other = rl_gather, None
    else:
        dominant, other = rl_attn, None
    tr = NCU_TRAFFIC.get((dominant["kernel"], w.name))
    if tr:
        dominant["traffic"] = tr["dram"]
        if "pcie_read" in tr:
            dominant["traffic_pcie_read"] = tr["pcie_read"]
        if "payload" in tr:
            # the host-memory bytes the captured launch read (its own misses), beside its link bytes
            dominant["traffic_payload"] = tr["payload"]
            dominant["traffic_link_per_payload"] = tr["pcie_read"] / tr["payload"]
        dominant["traffic_source"] = "ncu capture of this kernel on this workload (bytes per launch)"

    result = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            v, cores, sample = cpu_baseline(w)
            cpu = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        result = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step,
            "timed_region": {"repeats_of_k_steps": repeats, "steps_timed": steps_timed, "ms": ms_max,
                             "min_ms": MIN_TIMED_MS, "ms_per_step_block_median": statistics.median(block_ms) / args.steps,
                             "ms_per_step_block_min": min(block_ms) / args.steps,
                             "ms_per_step_block_max": max(block_ms) / args.steps,
                             "slowest_blocks": sorted(((round(b / args.steps, 4), i) for i, b in enumerate(block_ms)),
                                                      reverse=True)[:5]}, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 K/V, U(0,1) agnostic scores, AR(1) queries)",
            "config": workload_config(base, args.policy, world),
            "run": {"graph": "cuda graph replay",
                    "cpu_affinity": (f"{numa_cpus} CPUs local to the GPU" if numa_cpus else "unchanged"),
                    "calls": calls,
                    "hbm_bytes_per_step": hbm_bytes},
            "roofline": dominant,
            "roofline_other": other,
            "roofline_step": {
                "hbm_bytes_per_step": hbm_bytes, "pcie_bytes_per_step": pcie_bytes,
                "h2d_peak_gbs": h2d_peak, "t_hbm_nominal_us": t_hbm * 1e6, "t_hbm_measured_us": t_hbm_meas * 1e6,
                "t_pcie_us": t_pcie * 1e6,
                "frac_nominal": max(t_hbm, t_pcie) / step_s,
                "frac_measured": max(t_hbm_meas, t_pcie) / step_s,
                "hbm_gbs_achieved": hbm_bytes / step_s / 1e9, "h2d_gbs_achieved": pcie_bytes / step_s / 1e9,
            },
            "decode_stats": {
                "hit_rate": st["hits"] / max(1, st["hits"] + st["misses"]),
                "fetched_blocks_per_step": fetched_blocks,
                "fetched_mib_per_step": pcie_bytes / 2**20,
                "locality_mean": st["overlap_sum"] / max(1, st["overlap_terms"] * w.k),
                "locality_min": st["min_overlap"] / w.k,
            },
            "phases_ms": phase,
            "e2e": e2e,
            "step_latency_us": latency,
            "gpu_launches": launches_per_step * steps_timed,
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(result), flush=True)
    dec.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return result


def instrumented_pass(torch, dec, w, nosa, n, single_stream):
    """Per-phase GPU durations: the step is captured once more as a CUDA graph
    with timing events between the ABI calls (external event-record nodes), so
    the events fire on the GPU timeline with no host gaps; the graph is replayed
    n times and the events are read after each replay."""
    s = dec.stream
    cs = s if single_stream else dec.copy_stream
    ev = {k: torch.cuda.Event(enable_timing=True, external=True) for k in ("a", "b", "c", "d", "g", "e")}
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        if w.append:
            nosa.nosa_append_token(dec.ctx, dec.k_in, dec.v_in, dec.a_in, s)
        ev["a"].record(s)
        if dec.fused:
            # score, select and plan in one launch (b and c mark nothing)
            nosa.nosa_score_select_fetch(dec.ctx, dec.q, dec.scores, dec.sel, dec.fetch, dec.n_fetch, s, cs)
            ev["b"].record(s)
            ev["c"].record(s)
        else:
            nosa.nosa_score_blocks(dec.ctx, dec.q, dec.scores, s)
            ev["b"].record(s)
            nosa.nosa_select(dec.ctx, dec.scores, dec.sel, s)
            ev["c"].record(s)
            nosa.nosa_fetch_missing(dec.ctx, dec.sel, dec.fetch, dec.n_fetch, s, cs)
        ev["d"].record(s)
        # the decode call launches the fused gather + miss attention on s and,
        # with a second stream, the hits pass beside it on cs: g marks the hits
        # pass's end, e the gather's (the library joins cs back into s)
        nosa.nosa_sparse_decode(dec.ctx, dec.q, dec.sel, dec.out, s)
        ev["g"].record(cs)
        if cs is not s:
            s.wait_stream(cs)  # join the timing node recorded on the copy stream
        ev["e"].record(s)
    acc = {"score_ms": 0.0, "select_ms": 0.0, "plan_ms": 0.0, "prepare_ms": 0.0, "gather_ms": 0.0,
           "hits_side_ms": 0.0, "decode_ms": 0.0, "step_ms": 0.0}
    fb0 = dec.stats()["fetched_bytes"]
    for _ in range(n):
        t = dec.t
        with torch.cuda.stream(s):
            dec._load_inputs(t)
            g.replay()
        dec.t += 1
        torch.cuda.synchronize()
        acc["score_ms"] += ev["a"].elapsed_time(ev["b"])
        acc["select_ms"] += ev["b"].elapsed_time(ev["c"])
        acc["plan_ms"] += ev["c"].elapsed_time(ev["d"])
        acc["prepare_ms"] += ev["a"].elapsed_time(ev["d"])
        if cs is not s and w.offloaded:
            acc["gather_ms"] += ev["d"].elapsed_time(ev["e"])
            acc["hits_side_ms"] += ev["d"].elapsed_time(ev["g"])
        acc["decode_ms"] += ev["d"].elapsed_time(ev["e"])
        acc["step_ms"] += ev["a"].elapsed_time(ev["e"])
    del g
    out = {k: v / n for k, v in acc.items()}
    out["fetched_bytes_per_step"] = (dec.stats()["fetched_bytes"] - fb0) / n
    out["steps"] = n
    out["single_stream"] = bool(single_stream)
    out["fused_prepare"] = bool(dec.fused and w.max_blocks <= 512)
    if out["fused_prepare"]:
        for k in ("score_ms", "select_ms", "plan_ms"):
            out.pop(k)
    return out


LATENCY_STEPS = 256
MIN_TIMED_MS = 1000.0      # the timed region repeats its K steps until this much GPU time has passed
WARM_STEPS = 64            # untimed replays right before the timed region
APPEND_TIMED_STEPS = 2400  # most timed steps of a growing workload (its KV capacity is sized for them)
QUERY_BUDGET_BYTES = 3.5e9  # queries of an offloaded run (on the device, and pinned for the end-to-end pass)
MAX_QUERY_STEPS = 16000

# dram__bytes_read.sum + dram__bytes_write.sum per launch from one single-pass
# ncu capture of the dominant kernel on its workload (pcie: link-level read
# bytes, the traffic that bounds the gather; payload: the host-memory sectors
# the same launch read).  The hits pass was captured with the caches left as the
# step leaves them (--cache-control none), so its DRAM bytes are those read
# inside its own launch.  Retake after changing the kernel.
NCU_TRAFFIC = {
    ("gather_attend_kernel", "offload_b64"): {"dram": 591616 + 31744, "pcie_read": 20726784,
                                              "payload": 593076 * 32},
    ("attend_hits_ws_kernel", "layer8b"): {"dram": 261179904 + 0},
}


def step_latency_pass(torch, dec, w, n):
    """Per-step device time of n graph replays queued back to back (an event
    between consecutive steps).  With growing sequences, the steps whose
    appended token fills the tail block (and so close it) are reported apart."""
    s = dec.stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n + 1)]
    steps = []
    torch.cuda.synchronize()
    for i in range(n):
        steps.append(dec.t)
        ev[i].record(s)
        dec.replay()
    ev[n].record(s)
    torch.cuda.synchronize()
    us = np.array([ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(n)])
    out = {"n": n, "mean": float(us.mean()), "p50": float(np.percentile(us, 50)),
           "p90": float(np.percentile(us, 90)), "p99": float(np.percentile(us, 99)), "max": float(us.max())}
    if w.append:
        close = np.array([(w.context + t + 1) % w.block == 0 for t in steps])
        out["close_steps"] = int(close.sum())
        out["close_mean"] = float(us[close].mean()) if close.any() else None
        out["other_mean"] = float(us[~close].mean())
        out["other_max"] = float(us[~close].max())
    return out


def e2e_pass(torch, dec, w, nosa, n, host_wait=False, dist=None, world=1, dev=None):
    """End to end through the library's one-call step, as a decode loop whose
    queries and outputs live in pinned host memory runs it: every step calls
    nosa_decode_step with that step's queries (a slice of a pinned host
    array) and a pinned host output buffer; the library's kernels read the
    queries over PCIe and write the outputs back themselves.  Growing
    sequences first copy the new token's K/V in and append it.  host_wait:
    also wait on the host for each step's output (a sampling loop)."""
    q_host = dec.q_all.cpu().pin_memory()
    out_host = [torch.empty(dec.out.shape, dtype=dec.out.dtype, pin_memory=True) for _ in range(2)]
    s = dec.stream
    for i in range(4):  # untimed
        dec.step_through(q_host[dec.q_index(dec.t)], out_host[i % 2])
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0.record(s)
    t0 = time.perf_counter()
    for i in range(n):
        dec.step_through(q_host[dec.q_index(dec.t)], out_host[i % 2])
        if host_wait:
            s.synchronize()
    e1.record(s)
    torch.cuda.synchronize()
    wall = time.perf_counter() - t0
    # whole job: every rank decodes its own batch; the slowest rank's time
    ms = max_over_ranks(torch, dist, e0.elapsed_time(e1), dev, world)
    wall = max_over_ranks(torch, dist, wall * 1e3, dev, world) * 1e-3
    qb = dec.q.numel() * 2
    if w.append:
        qb += (dec.k_in.numel() + dec.v_in.numel()) * 2 + dec.a_in.numel() * 4
    ob = dec.out.numel() * 2
    return {"value": world * w.batch * n / (ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": qb,
            "d2h_bytes_per_step": ob, "steps": n, "wall_tokens_per_s": world * w.batch * n / wall,
            "note": ("nosa_decode_step per step, eager: queries read from pinned host memory and outputs written "
                     "to pinned host memory by the library's kernels, inside the timed region"
                     + ("; the host waits for each step's output" if host_wait else ""))}


def main():
    args = parse()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
