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
import hashlib
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


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu
# capture of the one-group workload scaled by groups, keyed by workload.  Each entry records
# the kernel source it was taken on; once that file changes the figure no
# longer describes the kernel and the bench reports null.
MEASURED_TRAFFIC = {
    # gate/up (single-CTA tiles) of the 1-group workload with the fp8 low pass: 155.8 MB read +
    # 30.0 MB written, x 8 groups
    "model_32k_5": ("gemm_tc.cu", "47f52f1e08eba982", 8 * 185.8e6, "gemm_gateup"),
    # the raw workload's call, both kernels of the two-phase form: prep 76.3 MB read +
    # 208.0 MB written, sequential 379.1 MB read + 64.2 MB written
    "raw_qwen": ("gdn_tc.cu", "caa0762384027f6e", 727.6e6, None),
    # the Mamba2 workload's launch: 1271.3 MB read + 1217.4 MB written
    "mamba2": ("mamba2_tc.cu", "5ed6885dc4fb76fe", 2488.6e6, None),
}


def measured_traffic(workload, kind=None):
    """The recorded DRAM traffic per launch of the workload's dominant kernel, or
    None when there is none for this kernel kind or its source has changed."""
    ent = MEASURED_TRAFFIC.get(workload)
    if ent is None:
        return None
    fn, digest, nbytes, ent_kind = ent
    if ent_kind is not None and ent_kind != kind:
        return None
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "gated_deltanet_state_sr_b200", "csrc", fn)
    try:
        with open(path, "rb") as f:
            now = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return nbytes if now == digest else None


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
        self.f32 = name == "raw_qwen_f32"
        if name in ("raw_qwen", "raw_qwen_f32"):
            self.x = W.raw_qwen(seed=0x5EED0001 + rank)
            self.desc = "one GDN layer, 8 suffixes ~U{512..2048} tok, H_k=16 H_v=32 d=128"
            if self.f32:
                # the fp32-input mode: the same values carried as fp32 q, k, v (and o)
                x = self.x
                x.q, x.k, x.v = x.q.float(), x.k.float(), x.v.float()
                self.desc += ", fp32 q/k/v/o (the fp32-input mode)"
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
        if self.f32:
            # the token recurrence's multiply-adds per token and V head: S k, the
            # rank-one update and S q, 3 d_k d_v FMAs = 6 d_k d_v flops
            self.flop_per_tok = hv * 6 * d * d
        else:
            self.flop_per_tok = hv * 2 * (C * (3 * d + 2 * d) + 3 * d * d)
        esz = 4 if self.f32 else 2
        self.bytes_per_tok = hk * 2 * d * esz + hv * (2 * d * esz + 8)
        self.state_bytes = x.n_seqs * hv * d * d * 4
        self.input_bytes = sum(t.numel() * t.element_size() for t in (x.q, x.k, x.v, x.g, x.beta))

    def setup(self, sr, dev):
        x = self.x
        self.sr = sr
        d = lambda t: t.to(dev).contiguous()
        self.q, self.k, self.v, self.g, self.b, self.cu = map(d, (x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens))
        self.o = torch.empty_like(self.v)
        self.s = torch.empty(x.n_seqs, self.hv, self.d, self.d, dtype=torch.float32, device=dev)
        self.max_len = x.max_seqlen
        # the call's own scratch (the two-phase form's chunk images), sized once
        args = sr.gdn_args(self.q, self.k, self.v, self.g, self.b, self.cu, n_seqs=x.n_seqs, max_seqlen=self.max_len,
                           o=self.o, s_out=self.s)
        self.ws = sr.workspace(max(sr.gdn_workspace_bytes(args), 1 << 20), dev)
        # pinned host copies for the end-to-end leg
        pin = lambda t: t.contiguous().pin_memory()
        self.h_in = [pin(t) for t in (x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens)]
        self.h_o = torch.empty(self.o.shape, dtype=self.o.dtype).pin_memory()
        self.h_s = torch.empty(self.s.shape, dtype=torch.float32).pin_memory()
        self.d_in = [self.q, self.k, self.v, self.g, self.b, self.cu]
        # second device buffer set for the pipelined end-to-end leg
        self.alt_in = [t.clone() for t in self.d_in]
        self.alt_o, self.alt_s = torch.empty_like(self.o), torch.empty_like(self.s)

    def e2e_inputs(self, b):
        return list(zip(self.h_in, self.d_in if b == 0 else self.alt_in))

    def e2e_outputs(self, b):
        o, s = (self.o, self.s) if b == 0 else (self.alt_o, self.alt_s)
        return [(o, self.h_o), (s, self.h_s)]

    def step_on(self, b):
        if b == 0:
            self.step()
            return
        q, k, v, g, be, cu = self.alt_in
        self.sr.gdn_replay(q, k, v, g, be, cu, max_seqlen=self.max_len, o=self.alt_o, s_out=self.alt_s, ws=self.ws)

    def step(self):
        self.sr.gdn_replay(self.q, self.k, self.v, self.g, self.b, self.cu, max_seqlen=self.max_len,
                           o=self.o, s_out=self.s, ws=self.ws)

    @property
    def launches_per_step(self):
        # the two-phase tcgen05 pair: the chunk-parallel prep, then the state chain;
        # the fp32-input mode: one token-by-token launch
        return 1 if self.f32 else 2

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
        if self.f32:
            # fp32 inputs run the token-by-token recurrence on the fp32 FMA units
            return {"name": "gdn_token_kernel", "bound": "alu", "flop": self.flop_per_tok * self.tokens,
                    "bytes": self.bytes_per_tok * self.tokens + self.state_bytes}
        # the default algorithm: the two tcgen05 kernels of one replay (the chunk-parallel
        # prep, then the per-sequence state chain), timed as the pair; at d = 64 they run
        # on 128-wide tiles whose upper halves stay zero
        return {"name": "gdn_prep_kernel + gdn_seq_kernel", "bound": "tensor",
                "flop": self.flop_per_tok * self.tokens,
                "bytes": self.bytes_per_tok * self.tokens + self.state_bytes}

    def oracle_piece(self, i):
        """One bounded piece of the oracle's work on this workload: every
        (sequence, V head) unit u with u % stride == i % stride (the whole
        replay when it is small, every 8th unit of the 8-suffix one).  Returns
        the replayed tokens the piece stands for (its head-tokens / H_v) and a
        description."""
        import oracle
        x = self.x
        n_units = x.n_seqs * self.hv
        stride = 1 if self.tokens * self.hv * self.d * self.d < 2**26 else 8
        units = list(range(i % stride, n_units, stride))
        oracle.gdn_replay(x.q, x.k, x.v, x.g, x.beta, x.cu_seqlens, units=units)
        head_tokens = sum(x.lengths[u // self.hv] for u in units)
        return head_tokens / self.hv, (f"{len(units)} of the {n_units} (sequence, V head) units per piece, "
                                       f"fp64 token-by-token recurrence; tokens = head-tokens / H_v")


class GroupReplay:
    """Whole replay groups from anchors (sr_group_replay): one group of 3 GDN
    layers + SwiGLU MLPs over a 1638-token suffix, or the 8-group whole-model
    replay of a [GDN, GDN, GDN, FA] x 8 hybrid with suffix k = ceil(r m)."""

    FULL_LAYER_MFLOP = None  # filled from shapes

    def __init__(self, name, rank, precision="split_fp8"):
        self.name = name
        if name == "group":
            self.gis = [W.group(seed=0x5EED0002 + 1000 * rank)]
            self.desc = "one group: 3 GDN layers + SwiGLU MLP, hidden 2560, inter 9216, 1638-token suffix"
        elif name.startswith("model_"):
            _, m, r = name.split("_")
            prefix = {"8k": 8192, "16k": 16384, "32k": 32768}[m]
            ratio = {"5": 0.05, "10": 0.10}[r]
            self.gis = [W.model_group(prefix, ratio, g, seed=0x5EED0003 + 1000 * rank) for g in range(8)]
            self.desc = (f"whole model: [GDN,GDN,GDN,FA]x8, 8 groups replayed group-parallel, FA skipped, "
                         f"suffix k = ceil({ratio} * {prefix}) = {W.model_suffix(prefix, ratio)}")
        elif name == "sparse_32k":
            # token-sparse anchors: each group's pool holds the 2048 anchors of a 32K
            # prefix (4 per 64-token page); the replay gathers the last
            # k = min(ceil(0.05 * 32768), 512) = 512 through the planner's pool rows
            n_pages = W.SPARSE_PREFIX // W.SPARSE_PAGE
            k = min(W.model_suffix(W.SPARSE_PREFIX, 0.05), W.SPARSE_K_MAX)
            self.gis = [W.anchor_pool_group(n_pages * W.SPARSE_PER_PAGE, k, seed=0x5EED0005 + 1000 * rank + g)
                        for g in range(8)]
            self.block_table = W.block_table(n_pages, 0x5EED0005 + 1000 * rank)
            # pool rows of the last k anchors (page-tail layout: anchor a sits in page
            # a // 4, slot a % 4), for the oracle's pieces, which run without the library
            n_anchors = n_pages * W.SPARSE_PER_PAGE
            self.h_rows = [self.block_table[a // W.SPARSE_PER_PAGE] * W.SPARSE_PER_PAGE + a % W.SPARSE_PER_PAGE
                           for a in range(n_anchors - k, n_anchors)]
            self.desc = (f"whole model, token-sparse anchors: 8 groups replay k = {k} anchors gathered from "
                         f"pools of {n_pages * W.SPARSE_PER_PAGE} (32K prefix, 4 per 64-token page, "
                         f"shuffled block table)")
        else:
            raise ValueError(name)
        self.sparse = name == "sparse_32k"
        self.precision = precision
        s = self.gis[0].shape
        self.s = s
        self.G = len(self.gis)
        self.L = len(self.gis[0].layers)
        self.tokens = sum(self.gis[0].lengths)
        T, H, I = self.tokens, s.hidden, s.inter
        C = 64
        # chunk-64 convention per token and V head: with the output o,
        # 2 (C (3 d_k + 2 d_v) + 3 d_k d_v); without it (the last layer in skip
        # mode) 2 (C 3 d_k + 2 d_k d_v)
        gdn_o = float(T) * s.h_v * 2 * (C * (3 * s.d_k + 2 * s.d_v) + 3 * s.d_k * s.d_v) * self.G
        gdn_no_o = float(T) * s.h_v * 2 * (C * 3 * s.d_k + 2 * s.d_k * s.d_v) * self.G
        in_full = 2.0 * T * H * s.proj_dim * self.G
        in_last = 2.0 * T * H * (s.proj_dim - s.v_dim) * self.G  # skip mode: the last layer needs no z
        self.flop = {  # algorithmic flops of one launch (all groups)
            # the mean over the step's in_proj launches: L - 1 full, the last without z
            "gemm_in": ((self.L - 1) * in_full + in_last) / self.L,
            "gemm_out": 2.0 * T * s.v_dim * H * self.G,
            "gemm_gateup": 2.0 * T * H * 2 * I * self.G,
            "gemm_down": 2.0 * T * I * H * self.G,
            # the mean over the step's GDN launches: L - 1 with o, the last without
            "gdn": ((self.L - 1) * gdn_o + gdn_no_o) / self.L,
        }
        full = in_full + self.flop["gemm_out"] + self.flop["gemm_gateup"] + self.flop["gemm_down"] + gdn_o
        last = in_last + gdn_no_o
        self.step_flop = (self.L - 1) * full + last  # skip mode
        # algorithmic bytes of one launch (all groups) for the HBM-bound layer kernels
        split = 1 if precision == "bf16" else 2  # k, v: bf16, or hi + lo bf16
        act_out = {"split": 4, "split_fp8": 3, "bf16": 2}[precision]  # projection operand bytes per element
        qd, vd = s.qk_dim, s.v_dim
        # algorithmic bytes per launch of the HBM-bound layer kernels: the
        # operation's own inputs and outputs in bf16 (gates fp32), whatever the
        # arithmetic carries
        self.bytes = {
            # [q|k|v] pre-conv channels and the b, a columns in; q, k, v out; g, beta (fp32) out
            "conv": float(T) * self.G * ((s.conv_dim + 2 * s.h_v) * 2 + (2 * qd + vd) * 2 + 2 * s.h_v * 4),
            # x in, RMSNorm(x) w out
            "row_prep": float(T) * self.G * (H * 2 + H * 2),
            # o and z in, y out
            "gated_norm": float(T) * self.G * (vd * 2 * 3),
        }
        # the bytes the kernels move in this precision mode: the in_proj output p is
        # fp32, the residual stream fp32, projection operands hi + lo (or hi + fp8 lo),
        # k and v hi + lo in the split modes
        self.bytes_impl = {
            "conv": float(T) * self.G * ((s.conv_dim + 2 * s.h_v) * 4 + qd * 2 + (qd + vd) * 2 * split
                                         + 2 * s.h_v * 4),
            # layer 0 only (later layers get the operand from the residual GEMMs' epilogues):
            # bf16 anchors in, the fp32 residual stream, the operand and r out
            "row_prep": float(T) * self.G * (H * 2 + H * 4 + H * act_out + 4),
            "gated_norm": float(T) * self.G * (vd * 2 + vd * 4 + vd * act_out),
        }
        self.input_bytes = self.G * T * H * 2 + sum(
            sum(getattr(lw, f).numel() * getattr(lw, f).element_size() for f in ("w_in", "w_out", "w_gate", "w_up",
                                                                              "w_down"))
            for gi in self.gis for lw in gi.layers)

    launches_per_step = None  # counted from the profiler

    def setup(self, sr, dev):
        self.sr = sr
        s = self.s
        self.anchors = [gi.anchors.to(dev).contiguous() for gi in self.gis]
        keys = ("w_in_norm", "w_in", "conv_w", "a_log", "dt_bias", "w_gnorm", "w_out", "w_post_norm", "w_gate",
                "w_up", "w_down")

        class L:
            pass

        self.weights = []
        for gi in self.gis:
            row = []
            for lw in gi.layers:
                o = L()
                for k in keys:
                    setattr(o, k, getattr(lw, k).to(dev).contiguous())
                row.append(o)
            self.weights.append(row)
        self.cu = self.gis[0].cu_seqlens.to(dev)
        self.max_len = max(self.gis[0].lengths)
        prec = {"split": sr.SR_PREC_SPLIT, "split_fp8": sr.SR_PREC_SPLIT_FP8, "bf16": sr.SR_PREC_BF16}
        self.kw = dict(max_seqlen=self.max_len, hidden=s.hidden, inter=s.inter, h_k=s.h_k, h_v=s.h_v, d=s.d_k,
                       eps=s.eps, mode=sr.SR_MODE_SKIP, precision=prec[self.precision])
        if self.precision == "split_fp8":
            # the low-pass weight copies are made once, as at model load
            for row in self.weights:
                for o in row:
                    sr.attach_lo8(o)
            torch.cuda.synchronize(dev)
        if self.sparse:
            _, rows = sr.sparse_anchor_plan(W.SPARSE_PREFIX, page_size=W.SPARSE_PAGE,
                                            anchors_per_page=W.SPARSE_PER_PAGE, k_max=W.SPARSE_K_MAX, ratio=0.05,
                                            block_table=self.block_table)
            assert len(rows) == self.tokens and list(rows) == self.h_rows
            self.h_index = torch.tensor(rows, dtype=torch.int32).pin_memory()
            self.index = self.h_index.to(dev)
            self.kw["anchor_index"] = self.index
        self.outputs = sr.group_replay(self.anchors, self.cu, self.weights, **self.kw)
        args = sr.group_args(self.anchors, self.cu, self.weights, self.outputs, **self.kw)
        self.ws = sr.workspace(sr.group_workspace_bytes(args), dev)
        self.prof = None
        # pinned host buffers for the end-to-end leg
        self.h_anchors = [gi.anchors.contiguous().pin_memory() for gi in self.gis]
        self.h_cu = self.gis[0].cu_seqlens.contiguous().pin_memory()
        self.h_out = [[(torch.empty(o[0].shape, dtype=o[0].dtype).pin_memory(),
                        torch.empty(o[1].shape, dtype=o[1].dtype).pin_memory()) for o in row]
                      for row in self.outputs]
        # second device buffer set for the pipelined end-to-end leg
        self.alt_anchors = [a.clone() for a in self.anchors]
        self.alt_cu = self.cu.clone()
        self.alt_index = self.index.clone() if self.sparse else None
        self.alt_outputs = [[(o[0].clone(), o[1].clone(), None) for o in row] for row in self.outputs]

    # ---- pipelined end-to-end leg: buffer set b of inputs / outputs
    def e2e_inputs(self, b):
        anchors, cu, index = (self.anchors, self.cu, self.index if self.sparse else None) if b == 0 else \
            (self.alt_anchors, self.alt_cu, self.alt_index)
        pairs = list(zip(self.h_anchors, anchors)) + [(self.h_cu, cu)]
        if self.sparse:
            pairs.append((self.h_index, index))
        return pairs

    def e2e_outputs(self, b):
        outs = self.outputs if b == 0 else self.alt_outputs
        return [(d, h) for hrow, drow in zip(self.h_out, outs) for (hs, hc), (ds, dc, _) in zip(hrow, drow)
                for d, h in ((ds, hs), (dc, hc))]

    def step_on(self, b):
        if b == 0:
            self.step()
            return
        kw = dict(self.kw)
        if self.sparse:
            kw["anchor_index"] = self.alt_index
        self.sr.group_replay(self.alt_anchors, self.alt_cu, self.weights, outputs=self.alt_outputs, ws=self.ws, **kw)

    def step(self, profile=None):
        self.sr.group_replay(self.anchors, self.cu, self.weights, outputs=self.outputs, ws=self.ws,
                             profile=profile, **self.kw)

    def step_e2e(self):
        for h, d in zip(self.h_anchors, self.anchors):
            d.copy_(h, non_blocking=True)
        self.cu.copy_(self.h_cu, non_blocking=True)
        if self.sparse:
            self.index.copy_(self.h_index, non_blocking=True)
        self.step()
        for hrow, drow in zip(self.h_out, self.outputs):
            for (hs, hc), (ds, dc, _) in zip(hrow, drow):
                hs.copy_(ds, non_blocking=True)
                hc.copy_(dc, non_blocking=True)

    @property
    def h2d_bytes(self):
        return (sum(t.numel() * t.element_size() for t in self.h_anchors) + self.h_cu.numel() * 4
                + (self.h_index.numel() * 4 if self.sparse else 0))

    @property
    def d2h_bytes(self):
        return sum(hs.numel() * 4 + hc.numel() * 2 for row in self.h_out for hs, hc in row)

    def oracle_piece(self, i):
        """One bounded piece of the oracle's work on this workload: the whole
        replay of group i % G (every layer in skip mode, as the step computes
        it, over the whole suffix).  Returns the replayed tokens the piece
        stands for (the suffix over G: a step replays every token through all
        G groups, which have the same shapes) and a description."""
        from oracle import layers as OL
        g = i % self.G
        gi = self.gis[g]
        if self.sparse:
            OL.group_replay(gi, "skip", anchor_index=self.h_rows)
        else:
            OL.group_replay(gi, "skip")
        return self.tokens / self.G, (f"one whole group per piece (group i mod {self.G}: {self.L} layers, skip "
                                      f"mode, {self.tokens} tokens), fp64 numpy layer math + C recurrence; "
                                      f"tokens = suffix / {self.G} groups per piece")


class Mamba2Replay:
    """Mamba2 replay (sr_mamba2_replay): 64 varlen suffixes of U{256..4096}
    tokens, 64 heads, P = 64, N = 128, one B/C group."""

    launches_per_step = 1
    precision = "bf16 inputs, hi/lo state write"

    def __init__(self, name, rank):
        self.m = W.mamba2(seed=0x5EED0004 + rank)
        self.desc = "Mamba2: 64 suffixes ~U{256..4096} tok, 64 heads, head dim 64, d_state 128"
        m = self.m
        self.tokens = sum(m.lengths)
        T, H, P = m.x.shape
        Ns = m.B.shape[2]
        self.H, self.P, self.Ns = H, P, Ns
        # algorithmic bytes per token: x, y (bf16), B, C (bf16, shared by heads), dt (fp32)
        self.bytes_per_tok = H * P * 2 * 2 + 2 * Ns * 2 + H * 4
        self.state_bytes = len(m.lengths) * H * P * Ns * 4
        self.flop_per_tok = H * (4 * P * Ns + 2 * 64 * P) + 2 * 64 * Ns
        self.input_bytes = sum(t.numel() * t.element_size() for t in (m.x, m.B, m.C, m.dt))

    def setup(self, sr, dev):
        self.sr = sr
        m = self.m
        d = lambda t: t.to(dev).contiguous()
        self.x, self.B, self.C, self.dt, self.A, self.cu = map(d, (m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens))
        self.y = torch.empty_like(self.x)
        self.s = torch.empty(len(m.lengths), self.H, self.P, self.Ns, dtype=torch.float32, device=dev)
        self.ws = sr.workspace(1 << 20, dev)
        self.max_len = m.max_seqlen
        pin = lambda t: t.contiguous().pin_memory()
        self.h_in = [pin(t) for t in (m.x, m.B, m.C, m.dt, m.cu_seqlens)]
        self.d_in = [self.x, self.B, self.C, self.dt, self.cu]
        self.h_y = torch.empty(self.y.shape, dtype=self.y.dtype).pin_memory()
        self.h_s = torch.empty(self.s.shape, dtype=torch.float32).pin_memory()
        # second device buffer set for the pipelined end-to-end leg
        self.alt_in = [t.clone() for t in self.d_in]
        self.alt_y, self.alt_s = torch.empty_like(self.y), torch.empty_like(self.s)

    def e2e_inputs(self, b):
        return list(zip(self.h_in, self.d_in if b == 0 else self.alt_in))

    def e2e_outputs(self, b):
        y, s = (self.y, self.s) if b == 0 else (self.alt_y, self.alt_s)
        return [(y, self.h_y), (s, self.h_s)]

    def step_on(self, b):
        if b == 0:
            self.step()
            return
        x, B, C, dt, cu = self.alt_in
        self.sr.mamba2_replay(x, B, C, dt, self.A, cu, max_seqlen=self.max_len, y=self.alt_y, s_out=self.alt_s,
                              ws=self.ws)

    def step(self):
        self.sr.mamba2_replay(self.x, self.B, self.C, self.dt, self.A, self.cu, max_seqlen=self.max_len,
                              y=self.y, s_out=self.s, ws=self.ws)

    def step_e2e(self):
        for h, d in zip(self.h_in, self.d_in):
            d.copy_(h, non_blocking=True)
        self.step()
        self.h_y.copy_(self.y, non_blocking=True)
        self.h_s.copy_(self.s, non_blocking=True)

    @property
    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.h_in)

    @property
    def d2h_bytes(self):
        return self.h_y.numel() * 2 + self.h_s.numel() * 4

    def dominant(self):
        return {"name": "mamba2_tc_kernel", "bound": "hbm", "flop": self.flop_per_tok * self.tokens,
                "bytes": self.bytes_per_tok * self.tokens + self.state_bytes}

    def oracle_piece(self, i, units=16):
        """One bounded piece of the oracle's work on this workload: `units`
        (sequence, head) pairs spread over the batch (offset by i).  Returns
        the replayed tokens the piece stands for (head-tokens / H) and a
        description."""
        import oracle
        m = self.m
        n_units = len(m.lengths) * self.H
        step = max(1, n_units // units)
        us = list(range(i % step, n_units, step))[:units]
        oracle.mamba2_replay(m.x, m.B, m.C, m.dt, m.A, m.cu_seqlens, units=us)
        head_tokens = sum(m.lengths[u // self.H] for u in us)
        return head_tokens / self.H, (f"{len(us)} of the {n_units} (sequence, head) units per piece, fp64 "
                                      f"token-by-token recurrence; tokens = head-tokens / H")


WORKLOADS = {"raw_qwen": RawGdn, "raw_small": RawGdn, "raw_qwen_f32": RawGdn, "group": GroupReplay,
             "mamba2": Mamba2Replay,
             "sparse_32k": GroupReplay,
             **{f"model_{m}_{r}": GroupReplay for m in ("8k", "16k", "32k") for r in ("5", "10")}}
DEFAULT_WORKLOAD = "model_32k_5"
L2_BYTES = 126 * 10**6  # B200 L2
FP32_FMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # 74.4


# ------------------------------------------------------------------ arms


def make_workload(args, rank):
    cls = WORKLOADS[args.workload]
    if cls is GroupReplay:
        return cls(args.workload, rank, precision=args.precision)
    return cls(args.workload, rank)


def run_e2e_pipelined(wl, k, stream):
    """k end-to-end steps with copies overlapped: buffer set b = i % 2 takes step
    i's inputs (copy stream) while step i-1 replays, and is read back (second
    copy stream) while step i+1 replays.  Ends with `stream` waiting for the
    last read-back, so an event recorded on it afterwards covers every copy."""
    if not hasattr(wl, "_pipe"):
        wl._pipe = dict(h2d=torch.cuda.Stream(), d2h=torch.cuda.Stream(),
                        ev={n: [torch.cuda.Event(), torch.cuda.Event()] for n in ("in", "done", "out")})
    h2d, d2h, ev = wl._pipe["h2d"], wl._pipe["d2h"], wl._pipe["ev"]
    for n in ev:
        for e in ev[n]:
            e.record(stream)
    for i in range(k):
        b = i % 2
        h2d.wait_event(ev["done"][b])  # the replay that last read set b has finished
        with torch.cuda.stream(h2d):
            for h, d in wl.e2e_inputs(b):
                d.copy_(h, non_blocking=True)
        ev["in"][b].record(h2d)
        stream.wait_event(ev["in"][b])
        stream.wait_event(ev["out"][b])  # set b's previous outputs have been read back
        wl.step_on(b)
        ev["done"][b].record(stream)
        d2h.wait_event(ev["done"][b])
        with torch.cuda.stream(d2h):
            for d, h in wl.e2e_outputs(b):
                h.copy_(d, non_blocking=True)
        ev["out"][b].record(d2h)
    for e in ev["out"]:
        stream.wait_event(e)


def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(ms, world, device):
    """Device-timed milliseconds of this rank -> the slowest rank's (the job's time)."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_step_per_rank, world, steps, ms):
    """Whole-job throughput: the units every rank processed over the slowest rank's time."""
    return units_per_step_per_rank * world * steps / (ms / 1e3)


def workload_config(args, wl, world):
    """The `config` object of the JSON line, the same for both arms."""
    mib = wl.input_bytes / 2**20
    l2 = (f"inputs {mib:.0f} MiB > L2, no flush" if wl.input_bytes > L2_BYTES else
          f"inputs {mib:.1f} MiB < L2: flushed by a 256 MiB write before every step, each step timed alone")
    return {"workload": args.workload, "desc": wl.desc, "tokens_per_step_per_gpu": wl.tokens, "l2": l2,
            "parallelism": f"dp{world} (independent replays per GPU)"}


def oracle_rate(wl, min_s):
    """The oracle on the host cores: pieces i = 0, 1, ... of the workload until
    min_s seconds have passed; returns (replayed tokens/s, pieces, seconds,
    description, threads)."""
    import oracle
    tok, i, t0 = 0.0, 0, time.perf_counter()
    while True:
        n, desc = wl.oracle_piece(i)
        tok += n
        i += 1
        secs = time.perf_counter() - t0
        if secs >= min_s:
            break
    return tok / secs, i, secs, desc, oracle.num_threads()


def run_ours(args):
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=dev)
    import gated_deltanet_state_sr_b200 as sr
    wl = make_workload(args, rank)
    wl.setup(sr, dev)
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(dev)

    for _ in range(args.warmup):
        wl.step()
    barrier()
    profiled = isinstance(wl, GroupReplay)
    profs = [sr.LaunchProfiler(64) for _ in range(args.steps)] if profiled else None
    # The single-call workloads (one replay call of a few tens of microseconds of GPU
    # work) are launch-bound from the host; as a serving engine would, they run as a
    # CUDA graph of the call, replayed per step.  The group workloads (28 launches,
    # milliseconds of GPU work per call) run eagerly, with per-launch events.
    graph = None
    if not profiled and not args.no_graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            wl.step()
        torch.cuda.synchronize(dev)
        for _ in range(args.warmup):
            graph.replay()
        barrier()
    step = graph.replay if graph is not None else wl.step
    # inputs that fit in L2: a 256 MiB write flushes it before every step, and each
    # step is timed by its own events (the flushes stay outside the timed sum)
    flush = None
    if wl.input_bytes <= L2_BYTES and not profiled:
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        e0.record(stream)
        for i in range(args.steps):
            if profiled:
                wl.step(profs[i])
            elif flush is not None:
                flush.fill_(i & 0xFF)
                ev[i][0].record(stream)
                step()
                ev[i][1].record(stream)
            else:
                step()
        e1.record(stream)
        barrier()
        # keep the GPU busy long enough for the clock sampler to see load
        t_end = time.perf_counter() + 0.6
        while time.perf_counter() < t_end:
            step()
        torch.cuda.synchronize(dev)
    ms_dev = sum(a.elapsed_time(b) for a, b in ev) if flush is not None else e0.elapsed_time(e1)
    ms = max_over_ranks(ms_dev, world, dev)
    ms_per_step = ms / args.steps
    value = job_throughput(wl.tokens, world, args.steps, ms)

    # per-kernel device time inside the timed region (events on the launching stream)
    kernels = None
    launches = None
    if profiled:
        tot, cnt = {}, {}
        launches = 0
        for pr in profs:
            for kind, t in pr.times():
                # two kernels per event pair: conv (conv_gates + conv_state) and gdn (the
                # two-phase prep + state chain)
                launches += 2 if kind in ("conv", "gdn") else 1
                tot[kind] = tot.get(kind, 0.0) + t
                cnt[kind] = cnt.get(kind, 0) + 1
        busy = sum(tot.values())
        peaks_, _ = load_peaks()
        kernels = {}
        for k in sorted(tot, key=lambda k: -tot[k]):
            per_launch = tot[k] / cnt[k]
            ent = {"ms_per_step": round(tot[k] / args.steps, 4), "launches_per_step": cnt[k] // args.steps,
                   "share": round(tot[k] / busy, 4)}
            if k in wl.flop:
                tf = wl.flop[k] / (per_launch / 1e3) / 1e12
                ent.update(bound="tensor", achieved_tflops=round(tf, 1),
                           frac=round(tf / peaks_.get("bf16_tflops_sustained", peaks_["bf16_tflops"]), 4))
            elif k in wl.bytes:
                gbs = wl.bytes[k] / (per_launch / 1e3) / 1e9
                gbs_impl = wl.bytes_impl[k] / (per_launch / 1e3) / 1e9
                ent.update(bound="hbm", achieved_gbs=round(gbs, 1), frac=round(gbs / peaks_["hbm_gbs"], 4),
                           achieved_gbs_impl=round(gbs_impl, 1), frac_impl=round(gbs_impl / peaks_["hbm_gbs"], 4))
            kernels[k] = ent
    else:
        launches = wl.launches_per_step * args.steps

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
    ms_e2e = max_over_ranks(f0.elapsed_time(f1), world, dev)
    e2e_value = job_throughput(wl.tokens, world, k_e2e, ms_e2e)
    e2e_serial = e2e_value
    if hasattr(wl, "e2e_inputs"):
        # pipelined: step i+1's host->device copy and step i-1's device->host copy run
        # on their own streams while step i replays (two buffer sets)
        run_e2e_pipelined(wl, 2, stream)
        barrier()
        f0.record(stream)
        run_e2e_pipelined(wl, k_e2e, stream)
        f1.record(stream)
        barrier()
        ms_e2e = max_over_ranks(f0.elapsed_time(f1), world, dev)
        e2e_value = job_throughput(wl.tokens, world, k_e2e, ms_e2e)

    peaks, src = load_peaks()
    if profiled:
        # dominant kernel: the kind with the most device time; algorithmic flops per
        # launch over its average launch duration; timed inside a long step -> sustained peak
        dom_kind = max((k for k in kernels if k in wl.flop), key=lambda k: kernels[k]["ms_per_step"])
        per_launch_ms = kernels[dom_kind]["ms_per_step"] / kernels[dom_kind]["launches_per_step"]
        achieved = wl.flop[dom_kind] / (per_launch_ms / 1e3) / 1e12
        peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
        names = {"gemm_in": "gemm_pair_kernel (in_proj)", "gemm_out": "gemm_pair_kernel (out_proj)",
                 "gemm_down": "gemm_pair_kernel (down)", "gemm_gateup": "gemm_tc_kernel (gate/up)",
                 "gdn": "gdn_prep_kernel + gdn_seq_kernel"}
        roofline = {"kernel": names.get(dom_kind, dom_kind),
                    "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                    "frac": round(achieved / peak, 4),
                    "traffic": measured_traffic(args.workload, dom_kind),
                    "peak_source": f"{src} (sustained bf16: kernel timed inside a long step)",
                    "flop_per_launch": wl.flop[dom_kind], "ms_per_launch": round(per_launch_ms, 4),
                    "mma_passes": {"split": "2 bf16", "split_fp8": "1 bf16 + 1 fp8 (e4m3 x e5m2)",
                                   "bf16": "1 bf16"}[wl.precision],
                    "step_tflops": round(wl.step_flop / (ms_per_step / 1e3) / 1e12, 2)}
    else:
        dom = wl.dominant()
        kern_ms = ms_per_step  # the dominant kernel is the whole step for the raw workloads
        tflops = dom["flop"] / (kern_ms / 1e3) / 1e12
        hbm_gbs = dom["bytes"] / (kern_ms / 1e3) / 1e9
        if dom["bound"] == "alu":
            # fp32 FMA peak from the unit counts: 148 SMs x 128 fp32 lanes x 2 flop x the
            # maximum SM clock (1965 MHz) = 74.4 TFLOP/s
            peak = FP32_FMA_TFLOPS
            roofline = {"kernel": dom["name"], "bound": "alu", "achieved": round(tflops, 2), "peak": peak,
                        "unit": "TFLOP/s", "frac": round(tflops / peak, 4), "traffic": measured_traffic(args.workload),
                        "peak_source": "derived: 148 SMs x 128 fp32 FMA lanes x 2 flop x 1965 MHz",
                        "hbm_gbs": round(hbm_gbs, 1), "hbm_frac": round(hbm_gbs / peaks["hbm_gbs"], 4)}
        elif dom["bound"] == "hbm":
            roofline = {"kernel": dom["name"], "bound": "hbm", "achieved": round(hbm_gbs, 1),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(hbm_gbs / peaks["hbm_gbs"], 4),
                        "traffic": measured_traffic(args.workload), "peak_source": f"{src} (HBM copy)",
                        "bytes_per_launch": dom["bytes"], "tflops": round(tflops, 2)}
        else:
            peak = peaks["bf16_tflops"]
            roofline = {"kernel": dom["name"], "bound": dom["bound"], "achieved": round(tflops, 2),
                        "peak": peak, "unit": "TFLOP/s", "frac": round(tflops / peak, 4),
                        "traffic": measured_traffic(args.workload),
                        "peak_source": f"{src} (burst bf16)", "hbm_gbs": round(hbm_gbs, 1),
                        "hbm_frac": round(hbm_gbs / peaks["hbm_gbs"], 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, pieces, secs, desc, cores = oracle_rate(wl, min_s=10.0)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"{pieces} pieces in {secs:.1f} s, timed (no extrapolation): {desc}"}

    line = {
        "metric": "replayed tokens/s", "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32" if getattr(wl, "f32", False) else "bf16",
        "data": "synthetic (seeded, workloads.py)",
        "config": workload_config(args, wl, world),
        "precision": getattr(wl, "precision", "fp32 inputs" if getattr(wl, "f32", False) else "bf16 inputs"),
        "e2e": {"value": e2e_value, "unit": "tokens/s", "serial_value": e2e_serial,
                "copies": "overlapped with the replay (two buffer sets, copy streams)" if hasattr(wl, "e2e_inputs")
                else "serialised with the replay", "h2d_bytes_per_step": wl.h2d_bytes,
                "d2h_bytes_per_step": wl.d2h_bytes},
        "gpu_launches": launches,
        "launch": "cuda graph of the call" if graph is not None else "eager",
        "roofline": roofline,
        "kernels": kernels,
        "clocks": clk.summary(),
        "cpu_baseline": cpu,
    }
    if isinstance(wl, GroupReplay):
        line["per_group_ms"] = ms_per_step / wl.G
        line["group_tokens_per_s"] = value * wl.G
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


def run_reference(args):
    """The fp64 oracle as the reference arm: each step is one bounded piece of
    the oracle's work on the workload (a whole group for the group workloads),
    timed as it runs; the value is the replayed tokens the pieces stand for
    over the time they took."""
    world, rank, local = dist_setup()
    if rank != 0:
        return
    wl = make_workload(args, 0)
    for i in range(args.warmup):
        wl.oracle_piece(i)
    tok, secs = 0.0, []
    for i in range(args.steps):
        t0 = time.perf_counter()
        n, desc = wl.oracle_piece(i)
        secs.append(time.perf_counter() - t0)
        tok += n
    value = tok / sum(secs)
    import oracle
    cores = oracle.num_threads()
    line = {"impl": "reference", "metric": "replayed tokens/s", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(secs) / len(secs), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded, workloads.py)",
            "config": workload_config(args, wl, world),
            "precision": "fp64 (the oracle)",
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"one piece per step, {args.steps} pieces in {sum(secs):.1f} s, timed "
                                       f"(no extrapolation): {desc}"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-graph", action="store_true",
                    help="run the single-call workloads eagerly instead of as a CUDA graph")
    ap.add_argument("--precision", choices=["split", "split_fp8", "bf16"], default="split_fp8",
                    help="group workloads: split_fp8 (hi/lo activations, low pass on the fp8 tensor cores; "
                         "parity-checked, the default), split (both passes bf16; parity-checked) or bf16 "
                         "(single pass)")
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
