#!/usr/bin/env python
"""Benchmark of suffix-replay state reconstruction on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One *step* is one pass of the replay hot path over one batch of synthetic,
seeded input (``workloads.py``); inputs are resident in HBM before timing.
Prints ONE JSON line on rank 0 with the replayed-token throughput, the
dominant kernel's roofline fraction (measured live with CUDA events on the
launching stream), an end-to-end figure through the C ABI with host buffers,
the clocks seen during the timed region, and the fp64 oracle timed on the
host cores as a CPU baseline.

Multi-GPU: one process per GPU (torchrun); each rank replays its own,
independent batch (weak scaling, no collective on the data path); the time is
the max over ranks.

``--impl reference`` times the fp64 oracle (the method's plain definition) on
the host cores instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_BYTES = 126 * 1024 * 1024


def load_peaks():
    try:
        with open(PEAKS_PATH) as f:
            p = json.load(f)
        return p, "measured"
    except Exception:
        return FALLBACK_PEAKS, "fallback"


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Samples nvidia-smi clocks and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ workloads


class RawGdn:
    """One GDN layer's recurrence over packed suffixes (sr_gdn_replay)."""

    def __init__(self, name, rank):
        self.name = name
        if name == "raw_qwen":
            self.x = W.raw_qwen(seed=0x5EED0001 + rank)
            self.desc = "one GDN layer, 8 suffixes ~U{512..2048} tok, H_k=16 H_v=32 d=128"
        elif name == "raw_small":
            self.x = W.raw_small(seed=0x5EED0000 + rank)
            self.desc = "one GDN layer, 1 suffix of 256 tok, H_k=2 H_v=4 d=64"
        else:
            raise ValueError(name)
        x = self.x
        self.tokens = sum(x.lengths)
        T, hk, d = x.q.shape
        hv = x.v.shape[1]
        self.hv, self.d, self.hk = hv, d, hk
        # algorithmic work (chunk-64 convention) and bytes per replayed token
        C = 64
        self.flop_per_tok = hv * 2 * (C * (3 * d + 2 * d) + 3 * d * d)
        self.bytes_per_tok = hk * 2 * d * 2 + hv * (2 * d * 2 + 8)
        self.state_bytes = x.n_seqs * hv * d * d * 4
        self.input_bytes = sum(t.numel() * t.element_size() for t in (x.q, x.k, x.v, x.g, x.beta))

    def setup(self, sr, dev):
        x = self.x
        self.sr = sr
        d = lambda t: t.to(dev).contiguous()
        self.q, self.k, self.v, self.g, self.b, self.cu = map(d, (x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens))
        self.o = torch.empty_like(self.v)
        self.s = torch.empty(x.n_seqs, self.hv, self.d, self.d, dtype=torch.float32, device=dev)
        self.ws = sr.workspace(1 << 20, dev)
        self.max_len = x.max_seqlen
        # pinned host copies for the end-to-end leg
        pin = lambda t: t.contiguous().pin_memory()
        self.h_in = [pin(t) for t in (x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens)]
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h_s = torch.empty(self.s.shape, dtype=torch.float32).pin_memory()
        self.d_in = [self.q, self.k, self.v, self.g, self.b, self.cu]

    def step(self):
        self.sr.gdn_replay(self.q, self.k, self.v, self.g, self.b, self.cu, max_seqlen=self.max_len,
                           o=self.o, s_out=self.s, ws=self.ws)

    launches_per_step = 1

    def step_e2e(self):
        for h, d in zip(self.h_in, self.d_in):
            d.copy_(h, non_blocking=True)
        self.step()
        self.h_o.copy_(self.o, non_blocking=True)
        self.h_s.copy_(self.s, non_blocking=True)

    @property
    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.h_in)

    @property
    def d2h_bytes(self):
        return self.h_o.numel() * self.h_o.element_size() + self.h_s.numel() * 4

    def dominant(self):
        return {"name": "gdn_chunk_kernel", "bound": "tensor",
                "flop": self.flop_per_tok * self.tokens,
                "bytes": self.bytes_per_tok * self.tokens + self.state_bytes}

    def oracle_sample(self, stride=1, min_s=0.0):
        """Bounded oracle run over every stride-th (sequence, head) unit,
        repeated until min_s seconds have passed; returns (tokens/s of a full
        layer, description, threads used)."""
        import oracle
        x = self.x
        n_units = x.n_seqs * self.hv
        lens = x.lengths
        units = list(range(0, n_units, stride))
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle.gdn_replay(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, units=units)
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= min_s:
                break
        head_tokens = sum(lens[u // self.hv] for u in units) * reps
        tok_per_s = head_tokens / self.hv / dt
        return tok_per_s, (f"{len(units)} of {n_units} (sequence, head) units x {reps} reps, "
                           f"{head_tokens} head-tokens, {dt:.1f} s; tokens/s = head-tokens / H_v / s"), \
            oracle.num_threads()


WORKLOADS = {"raw_qwen": RawGdn, "raw_small": RawGdn}


# ------------------------------------------------------------------ arms


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def run_ours(args):
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    import gated_deltanet_state_sr_b200 as sr
    wl = WORKLOADS[args.workload](args.workload, rank)
    wl.setup(sr, dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        wl.step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        e0.record(stream)
        for _ in range(args.steps):
            wl.step()
        e1.record(stream)
        barrier()
        # keep the GPU busy long enough for the clock sampler to see load
        extra = 0
        t_end = time.perf_counter() + 0.6
        while time.perf_counter() < t_end:
            wl.step()
            extra += 1
        torch.cuda.synchronize(dev)
    ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([ms], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    ms_per_step = ms / args.steps
    tokens_all = wl.tokens * world * args.steps
    value = tokens_all / (ms / 1e3)

    # end-to-end through the C ABI with host buffers (copies inside the timed region)
    for _ in range(2):
        wl.step_e2e()
    barrier()
    k_e2e = max(3, min(args.steps, 10))
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(k_e2e):
        wl.step_e2e()
    f1.record(stream)
    barrier()
    ms_e2e = f0.elapsed_time(f1)
    if world > 1:
        t = torch.tensor([ms_e2e], device=dev)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms_e2e = float(t.item())
    e2e_value = wl.tokens * world * k_e2e / (ms_e2e / 1e3)

    peaks, src = load_peaks()
    dom = wl.dominant()
    kern_ms = ms_per_step  # the dominant kernel is the whole step for the raw workloads
    if dom["bound"] == "tensor":
        achieved = dom["flop"] / (kern_ms / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        unit = "TFLOP/s"
    else:
        achieved = dom["bytes"] / (kern_ms / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        unit = "GB/s"
    hbm_gbs = dom["bytes"] / (kern_ms / 1e3) / 1e9
    roofline = {"kernel": dom["name"], "bound": dom["bound"], "achieved": round(achieved, 2),
                "peak": peak, "unit": unit, "frac": round(achieved / peak, 4), "traffic": None,
                "peak_source": src, "hbm_gbs": round(hbm_gbs, 1),
                "hbm_frac": round(hbm_gbs / peaks["hbm_gbs"], 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, sample, cores = wl.oracle_sample(stride=1, min_s=10.0)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample}

    line = {
        "metric": "replayed tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded, workloads.py)",
        "config": {"workload": args.workload, "desc": wl.desc, "tokens_per_step_per_gpu": wl.tokens,
                   "l2": f"inputs {wl.input_bytes / 2**20:.0f} MiB > L2, no flush",
                   "parallelism": f"dp{world} (independent replays per GPU)"},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": wl.h2d_bytes,
                "d2h_bytes_per_step": wl.d2h_bytes},
        "gpu_launches": wl.launches_per_step * args.steps,
        "roofline": roofline,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


def run_reference(args):
    world, rank, local = dist_setup()
    if rank != 0:
        return
    wl = WORKLOADS[args.workload](args.workload, 0)
    for _ in range(args.warmup):
        wl.oracle_sample(stride=8)
    vals = []
    for _ in range(args.steps):
        v, sample, cores = wl.oracle_sample(stride=8)
        vals.append(v)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": "replayed tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": wl.tokens / value * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, workloads.py)",
            "config": {"workload": args.workload, "desc": wl.desc, "tokens_per_step_per_gpu": wl.tokens},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="raw_qwen")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
