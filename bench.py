#!/usr/bin/env python
"""Benchmark: SSM-layer decode tokens/s at batch 256, ReplaySSM replay decode
against the conventional full-state decode, and the achieved HBM bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload m2_serving: Mamba-2 layer, batch 256, 128 heads, headdim 64,
d_state 128, 16 groups (8 heads share B/C), bf16 inputs, fp32 checkpoint,
16-record window.  One benchmark step is one 16-token window of decode for the
whole batch: 15 non-flush steps and one flush step (16 launches of the replay
decode kernel), i.e. 4096 tokens.  Inputs are seeded and synthetic and are
resident in HBM before timing; the 1 GiB checkpoint is far larger than L2, so
every step streams it from HBM.

Rank 0 prints one JSON line.  Under torchrun every rank runs an independent
replica (the path has no exchange step): value = tokens of all ranks / the
slowest rank's time.

--impl reference times the CPU oracle (fp64, the machine's host cores) on a
bounded sample of the same workload and prints the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSM-layer decode tokens/s @B=256 (replay vs full-state); achieved HBM GB/s"
WORKLOAD = "m2_serving"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300, help="timed 16-token windows")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=60, help="windows timed end to end")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only-main", action="store_true",
                    help="skip the Gated DeltaNet and speculative-verify measurements")
    ap.add_argument("--batch", type=int, default=256,
                    help="sequences of m2_serving (profiling captures use a smaller batch)")
    ap.add_argument("--sub-steps", type=int, default=60,
                    help="timed windows / rounds of the secondary measurements")
    ap.add_argument("--drift", action="store_true",
                    help="instead of timing: output-error drift of the low-precision read copy "
                         "and of a quantised checkpoint over m2_readcopy (batch 64, 8192 steps)")
    ap.add_argument("--drift-steps", type=int, default=8192)
    return ap.parse_args()


# Per-kernel DRAM traffic recorded under profiles/ by ncu (one capture at batch 64,
# scaled to the bench's batch by the number of work items): a figure applies only
# while the content hash of the kernel's sources equals the one recorded with it.
KERNEL_SOURCES = {
    "m2_decode_kernel_m2_serving": ("m2.cu", "m2_device.cuh", "common.cuh", "pipeline.cuh",
                                    "codec.cuh", "internal.h", "umma.cuh"),
    "gdn_decode2_kernel_gdn_serving": ("gdn.cu", "common.cuh", "pipeline.cuh", "internal.h",
                                      "umma.cuh"),
    "kda_decode2_kernel_kda_serving": ("kda.cu", "common.cuh", "internal.h", "pipeline.cuh"),
    "m2_verify_kernel_m2_verify": ("m2_verify.cu", "m2_device.cuh", "common.cuh", "pipeline.cuh",
                                   "codec.cuh", "internal.h"),
    "gdn_verify2_kernel_gdn_verify": ("gdn.cu", "common.cuh", "pipeline.cuh", "internal.h",
                                     "umma.cuh"),
}


def sources_sha256(files):
    import hashlib
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "ssm_state_storage_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(record, batch, bench_batch):
    """DRAM bytes (read + write) per launch at the bench's batch from the
    committed ncu summary profiles/<record>_traffic.txt, or None when absent,
    for another batch, or taken on different kernel sources."""
    path = os.path.join(ROOT, "profiles", record + "_traffic.txt")
    if batch != bench_batch or not os.path.exists(path):
        return None
    kv = {}
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) == 2 and not line.startswith("#"):
                kv[parts[0]] = parts[1]
    if kv.get("source_sha256") != sources_sha256(KERNEL_SOURCES[record]):
        return None
    return float(kv["traffic_bytes_per_launch"])


def max_over_ranks(ms, world, device=None):
    """The slowest rank's time: every rank takes part in one MAX all-reduce
    (a no-op with one rank).  Times are device times from CUDA events."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_rank, ms_max):
    """Whole-job throughput of independent replicas: all ranks' tokens over the
    slowest rank's time (weak scaling: per-rank work is fixed)."""
    return world * tokens_per_rank / (ms_max * 1e-3)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs, STREAM-style copy)"
    return FALLBACK_HBM_GBS, "fallback (6.65 TB/s, earlier copy measurement on this pool)"


# ------------------------------------------------------------------ clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.dev), "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9 and parts[1].replace(".", "").isdigit():
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({n for r in rows for n, v in zip(names, r[5:9]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max(float(r[3]) for r in rows if r[3].replace(".", "").isdigit())}


# ------------------------------------------------------------- CPU oracle

def oracle_inputs(n_seq, n_steps):
    from ssm_state_storage_b200 import workloads as wl
    w = wl.make(WORKLOAD)
    g = wl.Generator(w, seqs=range(n_seq))
    A, D = g.params()
    S0 = g.initial_state()
    return w, A, D, S0, g.steps(n_steps)


def oracle_time(inputs):
    """Seconds the fp64 CPU oracle (replay decode, as it stands) takes on them."""
    import oracle
    w, A, D, S0, st = inputs
    oracle.lib()
    rp = oracle.M2Replay(S0, G=w.G, L=w.L)
    t0 = time.perf_counter()
    rp.decode(st["x"], st["dt"], st["Bm"], st["Cm"], A, D)
    return time.perf_counter() - t0


def oracle_sample(n_seq=64, n_steps=256):
    """The oracle on a bounded sample: n_seq sequences of m2_serving, all 128
    heads, n_steps decode steps (16 windows, 16 flushes)."""
    secs = oracle_time(oracle_inputs(n_seq, n_steps))
    return {"value": n_seq * n_steps / secs, "unit": "tokens/s",
            "cores": len(os.sched_getaffinity(0)), "kind": "oracle", "seconds": secs,
            "sample": f"{n_seq} sequences x {n_steps} decode steps x all 128 heads of "
                      f"{WORKLOAD} (replay oracle, fp64, OpenMP over (sequence, head))"}


def run_reference(args, rank):
    if rank != 0:
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(len(os.sched_getaffinity(0))))
    n_seq, n_steps = 16, 16
    inputs = oracle_inputs(n_seq, n_steps)
    per_step = []
    for i in range(args.warmup + args.steps):
        secs = oracle_time(inputs)
        if i >= args.warmup:
            per_step.append(secs)
    tok = n_seq * n_steps
    total = sum(per_step)
    value = tok * len(per_step) / total
    cb = {"value": value, "unit": "tokens/s", "cores": len(os.sched_getaffinity(0)),
          "kind": "oracle",
          "sample": f"each step: {n_seq} sequences x {n_steps} decode steps (one window) x all "
                    f"128 heads of {WORKLOAD}, replay oracle in fp64"}
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * total / len(per_step), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch": 256, "sample_batch": n_seq},
            "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm

def run_ours(args, rank, world):
    import torch
    import torch.distributed as dist

    from ssm_state_storage_b200 import bytes_model as bm
    from ssm_state_storage_b200 import replayssm as rs
    from ssm_state_storage_b200 import workloads as wl

    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = wl.make(WORKLOAD, B=args.batch)
    L = w.L
    pool = 4 * L  # distinct input steps, cycled (each step's inputs are 6 MiB)
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    st = g.steps(pool)
    Ad, Dd = A.to(dev), D.to(dev)
    inputs = {k: v.to(dev) for k, v in st.items()}
    layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=L, in_dtype=w.in_dtype)
    state = rs.ReplayState(layer, device=dev)
    rs.replayssm_init(layer, state, S0.to(dev))
    S_full = S0.to(dev)
    y = torch.empty(w.B, w.H, w.P, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step_inp(t):
        i = t % pool
        return dict(x=inputs["x"][i], dt=inputs["dt"][i], Bm=inputs["Bm"][i],
                    Cm=inputs["Cm"][i], A=Ad, D=Dd)

    step_in = [step_inp(t) for t in range(pool)]

    def replay_window(wi):
        for j in range(L):
            rs.replayssm_decode_step(layer, state, step_in[(wi * L + j) % pool], y, stream)

    def full_window(wi):
        for j in range(L):
            rs.replayssm_full_decode_step(layer, S_full, step_in[(wi * L + j) % pool], y,
                                          stream=stream)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    def timed(fn, n, offset):
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            fn(offset + i)
        e1.record(stream)
        barrier()
        return max_over_ranks(e0.elapsed_time(e1), world, dev)

    for i in range(args.warmup):
        replay_window(i)
    dev_index = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]
    with ClockSampler(dev_index) as clk:
        ms_replay = timed(replay_window, args.steps, args.warmup)
    clocks = clk.summary()
    if state.status() != 0:
        raise RuntimeError(f"device status {state.status()} after the replay run")

    steps_us = per_launch_us(lambda i: rs.replayssm_decode_step(layer, state, step_in[i % pool], y,
                                                                stream), L, 10, stream, torch, dev)

    for i in range(args.warmup):
        full_window(i)
    ms_full = timed(full_window, args.steps, args.warmup)

    # ---- end to end: pinned host inputs in, y out, through the C ABI
    e2e = run_e2e(args, w, layer, state, st, Ad, Dd, dev, world, rs, torch, dist)

    tok_per_step = w.B * L
    hpg = w.H // w.G
    inb = 2 if w.in_dtype == torch.bfloat16 else 4
    win_bytes = bm.m2_replay_window_bytes(L, w.P, w.N, hpg, inb) * w.B * w.H
    full_bytes = bm.m2_conventional_bytes(w.P, w.N, hpg, inb) * w.B * w.H * L
    ms_per_window = ms_replay / args.steps
    ms_per_window_full = ms_full / args.steps
    achieved = win_bytes / (ms_per_window * 1e-3) / 1e9
    achieved_full = full_bytes / (ms_per_window_full * 1e-3) / 1e9
    peak, peak_src = peaks()
    value = job_tokens_per_s(world, tok_per_step * args.steps, ms_replay)
    value_full = job_tokens_per_s(world, tok_per_step * args.steps, ms_full)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_window,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "model": "Mamba-2 SSM layer (decode step only)",
                   "global_batch": w.B * world, "batch_per_gpu": w.B, "heads": w.H,
                   "headdim": w.P, "d_state": w.N, "groups": w.G, "window": L,
                   "inputs": "bf16", "checkpoint": "fp32", "parallelism": f"replicas x{world}",
                   "step": "one 16-token window = 15 non-flush + 1 flush decode steps",
                   "l2": "inputs larger than L2 (1 GiB checkpoint streamed every step)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak,
                     "traffic": recorded_traffic("m2_decode_kernel_m2_serving", w.B, 256),
                     "kernel": "m2_decode_kernel",
                     "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": win_bytes / L},
        "full_state": {"value": value_full, "unit": "tokens/s", "ms_per_step": ms_per_window_full,
                       "achieved_gbs": achieved_full, "frac": achieved_full / peak,
                       "kernel": "m2_full_kernel"},
        "replay_over_full": value / value_full,
        "step_times": steps_us,
        "bytes_per_head_token": {"replay": win_bytes / (w.B * w.H * L),
                                 "full_state": full_bytes / (w.B * w.H * L)},
        "clocks": clocks,
        "gpu_launches": args.steps * L,
        "e2e": e2e,
    }
    if not args.only_main:
        # free the m2_serving buffers before the other workloads
        del state, S_full, inputs, step_in, y
        torch.cuda.empty_cache()
        line["gdn"] = bench_gdn(args, dev, peak, rs, bm, wl, torch)
        torch.cuda.empty_cache()
        line["kda"] = bench_kda(args, dev, peak, rs, bm, wl, torch)
        torch.cuda.empty_cache()
        line["verify"] = bench_verify(args, dev, peak, rs, bm, wl, torch)
        torch.cuda.empty_cache()
        line["verify_gdn"] = bench_verify_gdn(args, dev, peak, rs, bm, wl, torch)
        torch.cuda.empty_cache()
        line["read_copy"] = bench_readcopy(args, dev, peak, rs, bm, wl, torch, ms_per_window)
        torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = oracle_sample()
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_e2e(args, w, layer, state, st, Ad, Dd, dev, world, rs, torch, dist):
    """Per decode step: H2D copy of the step's inputs from pinned host memory,
    the decode call, D2H copy of y to pinned host memory -- pipelined over three
    streams with double-buffered device inputs/outputs."""
    L = w.L
    pool = st["x"].shape[0]
    host = {k: v.pin_memory() for k, v in st.items()}
    keys = ("x", "dt", "Bm", "Cm")
    dbuf = [{k: torch.empty_like(host[k][0], device=dev) for k in keys} for _ in range(2)]
    ydev = [torch.empty(w.B, w.H, w.P, device=dev) for _ in range(2)]
    yhost = [torch.empty(w.B, w.H, w.P).pin_memory() for _ in range(2)]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_yfree = [torch.cuda.Event() for _ in range(2)]
    ev_infree = [torch.cuda.Event() for _ in range(2)]
    for e in ev_yfree + ev_infree:
        e.record(s_cmp)
    n_steps = args.e2e_steps * L
    h2d = sum(host[k][0].numel() * host[k][0].element_size() for k in keys)
    d2h = yhost[0].numel() * 4

    def run(n, t0):
        for t in range(t0, t0 + n):
            i = t % 2
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev_infree[i])
                for k in keys:
                    dbuf[i][k].copy_(host[k][t % pool], non_blocking=True)
                ev_in[i].record(s_in)
            s_cmp.wait_event(ev_in[i])
            s_cmp.wait_event(ev_yfree[i])
            inp = dict(dbuf[i], A=Ad, D=Dd)
            rs.replayssm_decode_step(layer, state, inp, ydev[i], s_cmp)
            ev_done[i].record(s_cmp)
            ev_infree[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[i])
                yhost[i].copy_(ydev[i], non_blocking=True)
                ev_yfree[i].record(s_out)

    run(2 * L, 0)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    run(n_steps, 0)
    s_in.wait_stream(s_out)
    e1.record(s_in)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    if state.status() != 0:
        raise RuntimeError(f"device status {state.status()} after the e2e run")
    return {"value": job_tokens_per_s(world, w.B * n_steps, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d * L, "d2h_bytes_per_step": d2h * L,
            "steps": args.e2e_steps, "pipelined": "H2D / decode / D2H on three streams"}


def per_launch_us(step, L, windows, stream, torch, dev):
    """CUDA-event time of every launch of `windows` windows of L decode steps
    (an event between consecutive launches on the launching stream), averaged
    per position in the window: the last position is the flush step."""
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(L * windows + 1)]
    ev[0].record(stream)
    for i in range(L * windows):
        step(i)
        ev[i + 1].record(stream)
    torch.cuda.synchronize(dev)
    per = [0.0] * L
    for i in range(L * windows):
        per[i % L] += ev[i].elapsed_time(ev[i + 1]) * 1e3 / windows
    return {"nonflush_avg_us": sum(per[:-1]) / max(L - 1, 1), "flush_us": per[-1],
            "per_position_us": [round(v, 1) for v in per], "windows": windows}


def _events_ms(fn, n, stream, torch, dev):
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(n):
        fn(i)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1)


def bench_gdn(args, dev, peak, rs, bm, wl, torch):
    """gdn_serving: Gated DeltaNet, batch 256, 32 heads, 128 x 128 state."""
    w = wl.make("gdn_serving")
    L, pool = w.L, 4 * w.L
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = {k: v.to(dev) for k, v in g.steps(pool).items()}
    layer = rs.Layer("gdn", w.B, w.H, w.P, w.N, window=L, in_dtype=w.in_dtype)
    state = rs.ReplayState(layer, device=dev)
    rs.replayssm_init(layer, state, S0.to(dev))
    S = S0.to(dev)
    o = torch.empty(w.B, w.H, w.P, device=dev)
    stream = torch.cuda.current_stream(dev)
    step_in = [{k: st[k][t] for k in st} for t in range(pool)]

    def replay_window(wi):
        for j in range(L):
            rs.replayssm_decode_step(layer, state, step_in[(wi * L + j) % pool], o, stream)

    def full_window(wi):
        for j in range(L):
            rs.replayssm_full_decode_step(layer, S, step_in[(wi * L + j) % pool], o, stream=stream)

    n = args.sub_steps
    for i in range(3):
        replay_window(i)
        full_window(i)
    ms_r = _events_ms(replay_window, n, stream, torch, dev)
    ms_f = _events_ms(full_window, n, stream, torch, dev)
    steps_us = per_launch_us(lambda i: rs.replayssm_decode_step(layer, state, step_in[i % pool], o,
                                                                stream), L, 10, stream, torch, dev)
    if state.status() != 0:
        raise RuntimeError(f"device status {state.status()} after the GDN run")
    inb = 2
    wb = bm.gdn_replay_window_bytes(L, w.N, w.P, inb) * w.B * w.H
    wb_rec = bm.gdn_replay_window_bytes_records(L, w.N, w.P, inb) * w.B * w.H
    fb = bm.gdn_conventional_bytes(w.N, w.P, inb) * w.B * w.H * L
    ach_r = wb / (ms_r / n * 1e-3) / 1e9
    ach_rec = wb_rec / (ms_r / n * 1e-3) / 1e9
    ach_f = fb / (ms_f / n * 1e-3) / 1e9
    tok = w.B * L * n
    return {"workload": "gdn_serving", "value": tok / (ms_r * 1e-3), "unit": "tokens/s",
            "ms_per_window": ms_r / n,
            "roofline": {"bound": "hbm", "achieved": ach_r, "peak": peak, "unit": "GB/s",
                         "frac": ach_r / peak, "kernel": "gdn_decode2_kernel",
                         "traffic": recorded_traffic("gdn_decode2_kernel_gdn_serving", w.B, 256),
                         "algorithmic_bytes_per_launch": wb / L,
                         "bytes": "records with their cached corrections u (as stored)",
                         "frac_input_records_only": ach_rec / peak,
                         "achieved_input_records_only": ach_rec},
            "full_state": {"value": tok / (ms_f * 1e-3), "unit": "tokens/s",
                           "achieved_gbs": ach_f, "frac": ach_f / peak,
                           "kernel": "kda_kernel<full> (scalar decay)"},
            "replay_over_full": ms_f / ms_r,
            "step_times": steps_us,
            "bytes_per_head_token": {"replay": wb / (w.B * w.H * L),
                                     "replay_input_records_only": wb_rec / (w.B * w.H * L),
                                     "full_state": fb / (w.B * w.H * L)},
            "gpu_launches": n * L}


def bench_kda(args, dev, peak, rs, bm, wl, torch):
    """kda_serving: Kimi Delta Attention, batch 256, 32 heads, 128 x 128
    state, one decay per key channel; replay against the conventional step."""
    w = wl.make("kda_serving")
    L, pool = w.L, 4 * w.L
    g = wl.Generator(w)
    S0 = g.initial_state()
    st = {k: v.to(dev) for k, v in g.steps(pool).items()}
    layer = rs.Layer("kda", w.B, w.H, w.P, w.N, window=L, in_dtype=w.in_dtype)
    state = rs.ReplayState(layer, device=dev)
    rs.replayssm_init(layer, state, S0.to(dev))
    S = S0.to(dev)
    o = torch.empty(w.B, w.H, w.P, device=dev)
    stream = torch.cuda.current_stream(dev)
    step_in = [{k: st[k][t] for k in st} for t in range(pool)]

    def replay_window(wi):
        for j in range(L):
            rs.replayssm_decode_step(layer, state, step_in[(wi * L + j) % pool], o, stream)

    def full_window(wi):
        for j in range(L):
            rs.replayssm_full_decode_step(layer, S, step_in[(wi * L + j) % pool], o, stream=stream)

    n = args.sub_steps
    for i in range(3):
        replay_window(i)
        full_window(i)
    ms_r = _events_ms(replay_window, n, stream, torch, dev)
    ms_f = _events_ms(full_window, n, stream, torch, dev)
    steps_us = per_launch_us(lambda i: rs.replayssm_decode_step(layer, state, step_in[i % pool], o,
                                                                stream), L, 10, stream, torch, dev)
    if state.status() != 0:
        raise RuntimeError(f"device status {state.status()} after the KDA run")
    wb = bm.kda_replay_window_bytes(L, w.N, w.P, 2) * w.B * w.H
    fb = bm.kda_conventional_bytes(w.N, w.P, 2) * w.B * w.H * L
    ach_r = wb / (ms_r / n * 1e-3) / 1e9
    ach_f = fb / (ms_f / n * 1e-3) / 1e9
    tok = w.B * L * n
    return {"workload": "kda_serving", "value": tok / (ms_r * 1e-3), "unit": "tokens/s",
            "ms_per_window": ms_r / n,
            "roofline": {"bound": "hbm", "achieved": ach_r, "peak": peak, "unit": "GB/s",
                         "frac": ach_r / peak, "kernel": "kda_decode2_kernel",
                         "traffic": recorded_traffic("kda_decode2_kernel_kda_serving", w.B, 256),
                         "algorithmic_bytes_per_launch": wb / L},
            "full_state": {"value": tok / (ms_f * 1e-3), "unit": "tokens/s",
                           "achieved_gbs": ach_f, "frac": ach_f / peak,
                           "kernel": "kda_kernel<full>"},
            "replay_over_full": ms_f / ms_r,
            "step_times": steps_us,
            "bytes_per_head_token": {"replay": wb / (w.B * w.H * L),
                                     "full_state": fb / (w.B * w.H * L)},
            "gpu_launches": n * L}


def bench_readcopy(args, dev, peak, rs, bm, wl, torch, ms_fp32):
    """m2_serving (batch 256) decoded with a low-precision read copy of the
    checkpoint: every output reads the FP8 / NVFP4 copy instead of the fp32
    checkpoint (which the flush fold still reads and writes)."""
    w = wl.make(WORKLOAD)
    L, pool = w.L, 4 * w.L
    g = wl.Generator(w)
    A, D = (t.to(dev) for t in g.params())
    S0 = g.initial_state().to(dev)
    st = {k: v.to(dev) for k, v in g.steps(pool).items()}
    step_in = [dict(x=st["x"][t], dt=st["dt"][t], Bm=st["Bm"][t], Cm=st["Cm"][t], A=A, D=D)
               for t in range(pool)]
    y = torch.empty(w.B, w.H, w.P, device=dev)
    stream = torch.cuda.current_stream(dev)
    n = args.sub_steps
    out = {"workload": WORKLOAD, "note": "outputs read the copy; the fold keeps the fp32 checkpoint"}
    for fmt in ("fp8", "nvfp4"):
        layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=L, in_dtype=w.in_dtype,
                         read_fmt=fmt)
        state = rs.ReplayState(layer, device=dev)
        rs.replayssm_init(layer, state, S0)

        def window(wi):
            for j in range(L):
                rs.replayssm_decode_step(layer, state, step_in[(wi * L + j) % pool], y, stream)

        for i in range(3):
            window(i)
        ms = _events_ms(window, n, stream, torch, dev)
        steps_us = per_launch_us(lambda i: rs.replayssm_decode_step(layer, state,
                                                                    step_in[i % pool], y, stream),
                                 L, 10, stream, torch, dev)
        if state.status() != 0:
            raise RuntimeError(f"device status {state.status()} after the {fmt} read-copy run")
        wb = bm.m2_replay_window_bytes_rc(L, w.P, w.N, w.H // w.G, 2, fmt) * w.B * w.H
        ach = wb / (ms / n * 1e-3) / 1e9
        out[fmt] = {"value": w.B * L * n / (ms * 1e-3), "unit": "tokens/s", "ms_per_window": ms / n,
                    "roofline": {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s",
                                 "frac": ach / peak, "kernel": "m2_decode_kernel (read copy)"},
                    "bytes_per_head_token": wb / (w.B * w.H * L),
                    "over_fp32_replay": ms_fp32 / (ms / n), "step_times": steps_us,
                    "gpu_launches": n * L}
        del state
        torch.cuda.empty_cache()
    return out


def bench_verify(args, dev, peak, rs, bm, wl, torch):
    """m2_verify: Mamba-2 m2_serving heads at batch 512, 4 drafts per round,
    acceptance ~ U{0..4}; replay verify/commit against snapshot-and-restore
    decoding of the full state."""
    w = wl.make("m2_verify")
    pool = 16
    g = wl.Generator(w)
    A, D = g.params()
    S0 = g.initial_state()
    rd = g.rounds(pool)
    acc_host = rd["acc"].clone()
    rd = {k: v.to(dev) for k, v in rd.items()}
    Ad, Dd = A.to(dev), D.to(dev)
    layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L, draft_max=w.n_draft,
                     in_dtype=w.in_dtype)
    state = rs.ReplayState(layer, device=dev)
    rs.replayssm_init(layer, state, S0.to(dev))
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device=dev)
    stream = torch.cuda.current_stream(dev)
    drafts = [dict(x=rd["x"][r], dt=rd["dt"][r], Bm=rd["Bm"][r], Cm=rd["Cm"][r], A=Ad, D=Dd)
              for r in range(pool)]
    n = args.sub_steps

    def replay_round(r):
        rs.replayssm_verify_commit(layer, state, rd["acc"][(r - 1) % pool] if r else None,
                                   drafts[r % pool], y, stream)

    for r in range(3):
        replay_round(r)
    rs.replayssm_commit(layer, state, rd["acc"][2 % pool], Ad, stream)
    torch.cuda.synchronize(dev)
    lens0 = state.len[:, 0].cpu().long()
    def timed_round(r):
        # timed round r evaluates draft set r+3; its predecessor's acceptance
        # (set r+2) is committed first, except for r = 0 (already committed)
        rs.replayssm_verify_commit(layer, state, rd["acc"][(r + 2) % pool] if r else None,
                                   drafts[(r + 3) % pool], y, stream)

    ms_r = _events_ms(timed_round, n, stream, torch, dev)
    if state.status() != 0:
        raise RuntimeError(f"device status {state.status()} after the verify run")
    # algorithmic bytes: replay the length bookkeeping on the host
    hpg = w.H // w.G
    st_b, x_b, dt_b, bc_b, b_b, y_b = bm.m2_sizes(w.P, w.N, hpg, 2)
    lens = lens0.clone()
    total = 0.0
    for r in range(n):
        a = acc_host[(r + 2) % pool].long() if r else torch.zeros_like(lens)
        n1 = lens + a
        fold = n1 >= w.L
        nb = torch.where(fold, torch.zeros_like(n1), n1)
        per = (st_b + n1 * (x_b + 4 + b_b) + w.n_draft * ((x_b + dt_b + bc_b) + (x_b + 4 + bc_b))
               + w.n_draft * y_b + fold.double() * st_b)
        total += float(per.double().sum()) * w.H
        lens = nb
    ach_r = total / (ms_r * 1e-3) / 1e9
    committed = float(sum(acc_host[(r + 2) % pool].sum() for r in range(1, n)))

    # snapshot-and-restore conventional decoding of the full state
    fl = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L, in_dtype=w.in_dtype)
    S = S0.to(dev)
    snap = torch.empty_like(S)
    ysn = torch.empty(w.B, w.n_draft, w.H, w.P, device=dev)
    junk = torch.empty(w.B, w.H, w.P, device=dev)

    def snap_round(r):
        i = r % pool
        snap.copy_(S)
        for d in range(w.n_draft):
            inp = dict(x=rd["x"][i][:, d], dt=rd["dt"][i][:, d], Bm=rd["Bm"][i][:, d],
                       Cm=rd["Cm"][i][:, d], A=Ad, D=Dd)
            rs.replayssm_full_decode_step(fl, S, inp, ysn[:, d], stream=stream)
        S.copy_(snap)
        for d in range(w.n_draft):
            inp = dict(x=rd["x"][i][:, d], dt=rd["dt"][i][:, d], Bm=rd["Bm"][i][:, d],
                       Cm=rd["Cm"][i][:, d], A=Ad, D=Dd)
            rs.replayssm_full_decode_step(fl, S, inp, junk, limit=rd["acc"][i], step_index=d,
                                          stream=stream)

    for r in range(2):
        snap_round(r)
    ms_s = _events_ms(snap_round, n, stream, torch, dev)
    conv = bm.m2_conventional_bytes(w.P, w.N, hpg, 2)
    snap_bytes = 0.0
    for r in range(n):
        a = acc_host[r % pool].double()
        snap_bytes += float((4 * st_b + (w.n_draft + a) * conv).sum()) * w.H
    ach_s = snap_bytes / (ms_s * 1e-3) / 1e9
    rounds = n
    return {"workload": "m2_verify", "rounds_per_s": rounds / (ms_r * 1e-3),
            "ms_per_round": ms_r / rounds,
            "drafts_evaluated_per_s": w.B * w.n_draft * rounds / (ms_r * 1e-3),
            "committed_tokens_per_s": committed / (ms_r * 1e-3),
            "roofline": {"bound": "hbm", "achieved": ach_r, "peak": peak, "unit": "GB/s",
                         "frac": ach_r / peak, "kernel": "m2_verify_kernel",
                         "traffic": recorded_traffic("m2_verify_kernel_m2_verify", w.B, 512),
                         "algorithmic_bytes_per_launch": total / n},
            "snapshot_restore": {"rounds_per_s": rounds / (ms_s * 1e-3), "ms_per_round": ms_s / rounds,
                                 "achieved_gbs": ach_s, "frac": ach_s / peak,
                                 "kernels": "cudaMemcpyAsync x2 + m2_full_kernel x8"},
            "replay_over_snapshot": ms_s / ms_r,
            "gpu_launches": rounds}


def bench_verify_gdn(args, dev, peak, rs, bm, wl, torch):
    """gdn_verify: Gated DeltaNet gdn_serving heads at batch 256, 4 drafts per
    round, acceptance ~ U{0..4}; replay verify/commit against snapshot-and-
    restore decoding of the full state."""
    w = wl.make("gdn_verify")
    pool = 16
    g = wl.Generator(w)
    S0 = g.initial_state()
    rd = g.rounds(pool)
    acc_host = rd["acc"].clone()
    rd = {k: v.to(dev) for k, v in rd.items()}
    names = ("q", "k", "v", "alpha", "beta")
    layer = rs.Layer("gdn", w.B, w.H, w.P, w.N, window=w.L, draft_max=w.n_draft,
                     in_dtype=w.in_dtype)
    state = rs.ReplayState(layer, device=dev)
    rs.replayssm_init(layer, state, S0.to(dev))
    y = torch.empty(w.B, w.n_draft, w.H, w.P, device=dev)
    stream = torch.cuda.current_stream(dev)
    drafts = [{k: rd[k][r] for k in names} for r in range(pool)]
    n = args.sub_steps
    for r in range(3):
        rs.replayssm_verify_commit(layer, state, rd["acc"][(r - 1) % pool] if r else None,
                                   drafts[r % pool], y, stream)
    rs.replayssm_commit(layer, state, rd["acc"][2 % pool], stream=stream)
    torch.cuda.synchronize(dev)
    lens0 = state.len[:, 0].cpu().long()

    def timed_round(r):
        rs.replayssm_verify_commit(layer, state, rd["acc"][(r + 2) % pool] if r else None,
                                   drafts[(r + 3) % pool], y, stream)

    ms_r = _events_ms(timed_round, n, stream, torch, dev)
    if state.status() != 0:
        raise RuntimeError(f"device status {state.status()} after the GDN verify run")
    lens = lens0.clone()
    total = 0.0
    for r in range(n):
        a = acc_host[(r + 2) % pool].long() if r else torch.zeros_like(lens)
        n1 = lens + a
        fold = n1 >= w.L
        per = [bm.gdn_verify_round_bytes(int(n1[b]), bool(fold[b]), w.n_draft, w.N, w.P, 2)
               for b in range(w.B)]
        total += sum(per) * w.H
        lens = torch.where(fold, torch.zeros_like(n1), n1)
    ach_r = total / (ms_r * 1e-3) / 1e9

    fl = rs.Layer("gdn", w.B, w.H, w.P, w.N, window=w.L, in_dtype=w.in_dtype)
    S = S0.to(dev)
    snap = torch.empty_like(S)
    ysn = torch.empty(w.B, w.n_draft, w.H, w.P, device=dev)
    junk = torch.empty(w.B, w.H, w.P, device=dev)

    def snap_round(r):
        i = r % pool
        snap.copy_(S)
        for d in range(w.n_draft):
            rs.replayssm_full_decode_step(fl, S, {k: rd[k][i][:, d] for k in names}, ysn[:, d],
                                          stream=stream)
        S.copy_(snap)
        for d in range(w.n_draft):
            rs.replayssm_full_decode_step(fl, S, {k: rd[k][i][:, d] for k in names}, junk,
                                          limit=rd["acc"][i], step_index=d, stream=stream)

    for r in range(2):
        snap_round(r)
    ms_s = _events_ms(snap_round, n, stream, torch, dev)
    st_b = w.N * w.P * 4
    conv = bm.gdn_conventional_bytes(w.N, w.P, 2)
    snap_bytes = 0.0
    for r in range(n):
        a = acc_host[r % pool].double()
        snap_bytes += float((4 * st_b + (w.n_draft + a) * conv).sum()) * w.H
    ach_s = snap_bytes / (ms_s * 1e-3) / 1e9
    return {"workload": "gdn_verify", "rounds_per_s": n / (ms_r * 1e-3),
            "ms_per_round": ms_r / n,
            "drafts_evaluated_per_s": w.B * w.n_draft * n / (ms_r * 1e-3),
            "roofline": {"bound": "hbm", "achieved": ach_r, "peak": peak, "unit": "GB/s",
                         "frac": ach_r / peak, "kernel": "gdn_verify2_kernel",
                         "traffic": recorded_traffic("gdn_verify2_kernel_gdn_verify", w.B, 256),
                         "algorithmic_bytes_per_launch": total / n},
            "snapshot_restore": {"rounds_per_s": n / (ms_s * 1e-3), "ms_per_round": ms_s / n,
                                 "achieved_gbs": ach_s, "frac": ach_s / peak,
                                 "kernels": "cudaMemcpyAsync x2 + kda_kernel<full> x8"},
            "replay_over_snapshot": ms_s / ms_r,
            "gpu_launches": n}


def run_drift(args, rank):
    """m2_readcopy: batch 64 of the m2_serving heads decoded for 8192 steps by
    five replay variants on the same inputs -- fp32 checkpoint (the
    reference), FP8 / NVFP4 read copy over an fp32 checkpoint, and FP8 / NVFP4
    quantised checkpoint -- plus the conventional fp32 full-state decode, for
    two decay settings: the workload's A_h = -exp(U(0, ln 16)) (the state
    forgets a window in ~e^-8) and a long-memory A_h / 100.  Per step, each
    variant's output error against the fp32 replay output of its setting:
    max_i |y - y_ref| / max(|y_ref|, 1e-2 rms(y_ref)) and the normwise
    ||y - y_ref|| / ||y_ref||.  Prints one JSON line (errors at t = 16, 128,
    1024, 8192 as the max over the preceding half-decade, and the fitted
    growth exponent of the normwise error in t)."""
    if rank != 0:
        return
    import math

    import torch

    from ssm_state_storage_b200 import replayssm as rs
    from ssm_state_storage_b200 import workloads as wl
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w = wl.make("m2_readcopy")
    T = args.drift_steps
    g = wl.Generator(w)
    A0, D = (t.to(dev) for t in g.params())
    S0 = g.initial_state().to(dev)
    settings = {"workload_A": A0, "long_memory_A/100": A0 / 100.0}
    fmts = [("fp32", {}), ("read_fp8", {"read_fmt": "fp8"}), ("read_nvfp4", {"read_fmt": "nvfp4"}),
            ("ckpt_fp8", {"ckpt_fmt": "fp8"}), ("ckpt_nvfp4", {"ckpt_fmt": "nvfp4"})]
    runs = {}
    for sname in settings:
        for name, kw in fmts:
            layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L,
                             in_dtype=w.in_dtype, **kw)
            st = rs.ReplayState(layer, device=dev)
            rs.replayssm_init(layer, st, S0)
            runs[(sname, name)] = (layer, st, torch.empty(w.B, w.H, w.P, device=dev))
    full_layer = rs.Layer("m2", w.B, w.H, w.P, w.N, ngroups=w.G, window=w.L, in_dtype=w.in_dtype)
    S_full = {sname: S0.clone() for sname in settings}
    y_full = {sname: torch.empty(w.B, w.H, w.P, device=dev) for sname in settings}
    names = [n for n, _ in fmts[1:]] + ["full_state_fp32"]
    keys = [(sn, n) for sn in settings for n in names]
    maxrel = {k: torch.zeros(T, dtype=torch.float64) for k in keys}
    normw = {k: torch.zeros(T, dtype=torch.float64) for k in keys}
    chunk = 256
    t0 = time.time()
    for c0 in range(0, T, chunk):
        n = min(chunk, T - c0)
        stp = {k: v.to(dev) for k, v in g.steps(n).items()}
        mr = {k: torch.empty(n, device=dev) for k in keys}
        nw = {k: torch.empty(n, device=dev) for k in keys}
        for t in range(n):
            for sname, A in settings.items():
                inp = dict(x=stp["x"][t], dt=stp["dt"][t], Bm=stp["Bm"][t], Cm=stp["Cm"][t], A=A, D=D)
                for name, _ in fmts:
                    layer, st, yv = runs[(sname, name)]
                    rs.replayssm_decode_step(layer, st, inp, yv)
                rs.replayssm_full_decode_step(full_layer, S_full[sname], inp, y_full[sname])
                ref = runs[(sname, "fp32")][2]
                rms = ref.square().mean().sqrt()
                den = torch.maximum(ref.abs(), 1e-2 * rms)
                for name in names:
                    yv = y_full[sname] if name == "full_state_fp32" else runs[(sname, name)][2]
                    diff = yv - ref
                    mr[(sname, name)][t] = (diff.abs() / den).max()
                    nw[(sname, name)][t] = diff.norm() / ref.norm()
        for k in keys:
            maxrel[k][c0:c0 + n] = mr[k].double().cpu()
            normw[k][c0:c0 + n] = nw[k].double().cpu()
    for (sname, name), (_, st, _) in runs.items():
        if st.status() != 0:
            raise RuntimeError(f"device status {st.status()} in variant {sname}/{name}")
    marks = [m for m in (16, 128, 1024, 8192) if m <= T]

    def at(series, m):  # max over (m / sqrt(8), m]
        lo = max(int(m / math.sqrt(8)), 1)
        return float(series[lo - 1:m].max())

    def growth(series):  # least-squares slope of log(err) in log(t), t >= 16
        ts = torch.arange(16, T + 1, dtype=torch.float64)
        e = series[15:T].clamp_min(1e-30)
        lx, ly = ts.log(), e.log()
        lx, ly = lx - lx.mean(), ly - ly.mean()
        return float((lx * ly).sum() / (lx * lx).sum())

    out = {"metric": "output error vs the fp32 replay output over a long decode", "workload":
           "m2_readcopy", "config": {"batch": w.B, "heads": w.H, "headdim": w.P, "d_state": w.N,
                                      "groups": w.G, "window": w.L, "steps": T, "inputs": "bf16"},
           "data": "synthetic", "seconds": time.time() - t0, "settings": {}}
    for sname in settings:
        out["settings"][sname] = {
            name: {"max_rel": {str(m): at(maxrel[(sname, name)], m) for m in marks},
                   "normwise": {str(m): at(normw[(sname, name)], m) for m in marks},
                   "normwise_growth_exponent": growth(normw[(sname, name)])}
            for name in names}
    print(json.dumps(out), flush=True)


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    if args.drift:
        run_drift(args, rank)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
