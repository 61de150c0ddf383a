#!/usr/bin/env python
"""Decode-attention benchmark of the ODA hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl oda|reference]

A step is one ODA decode step of the whole attention stack: Local attention with commit at
every layer, the FP32 recall head and its gate, and the gated Full recompute with commit,
as one CUDA-graph launch (liboda's step graph). The default workload is the long-context
efficiency point: 28 layers (Qwen3-1.7B attention shapes: 16 query / 8 KV heads, head dim
128), batch 1, 131072 prefilled tokens, s = 4, w = 2048, theta calibrated so that about
12.5 % of steps recompute with Full. Inputs are seeded synthetic tensors (bf16 K/V/Q ~
N(0, 1)) resident in HBM; the 15 GB KV cache is far larger than L2, so no flush is needed.

Printed on rank 0: one JSON line with tokens/s (value), the KV bytes/s the step streams,
the dominant kernel's roofline fraction, an end-to-end figure through the same API with
host buffers, the clocks seen during the timed region and the fp64 oracle's CPU baseline.
Under torchrun each rank runs its own sequences (no data-path collective: weak scaling).
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import math
import os
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import oda_synth  # noqa: E402

METRIC = "decode-attn tokens/s & achieved HBM GB/s (% of roofline) at 128K ctx, ρ≈12.5%"
UNIT = "tokens/s"
DEFAULT_WORKLOAD = "qwen3-1.7b-128k-b1"
ROW_BYTES = 2 * 128 * 2          # K row + V row of one (position, KV head): 512 B
PAGE_BYTES = 2 * 16 * 128 * 2    # K page + V page of one (page, KV head): 8 KB
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0         # B200 HBM3e nominal (~8 TB/s), reported beside the measured peak
# Machine-readable ncu figures (written by `bench.py --ncu-summary` from a capture's raw CSV),
# beside the prose summaries of the same captures in profiles/*.md.
# Committed ncu summaries (JSON written by --ncu-summary) of the step's kernels on the
# long-context workload, by kernel, and the device sources each was taken on.
PROFILES = {
    "full_chain": os.path.join(ROOT, "profiles", "full_chain_128k.json"),
    "full_layer": os.path.join(ROOT, "profiles", "decode_full_128k.json"),
    "local_cluster": os.path.join(ROOT, "profiles", "local_cluster_128k.json"),
    "local_chain": os.path.join(ROOT, "profiles", "local_chain_128k.json"),
    "recall": os.path.join(ROOT, "profiles", "recall_h2048.json"),
}
PROFILE = PROFILES["full_chain"]
KERNEL_SOURCES = ["oda_decode.cuh", "oda_decode.cu", "oda_chain.cu", "oda_plan.cuh",
                  "oda_common.cuh", "oda_recall.cuh"]
RECALL_SOURCES = ["oda_recall.cu", "oda_recall.cuh", "oda_common.cuh"]


def profile_sources(key_or_kernel: str):
    """Device sources an ncu summary of this kernel depends on."""
    return RECALL_SOURCES if "recall" in key_or_kernel else KERNEL_SOURCES


STEP_KERNELS = {"full-persistent": 0, "per-layer": 1, "persistent": 2}  # ODA_STEP_*


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["oda", "reference"], default="oda")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(oda_synth.WORKLOADS))
    ap.add_argument("--calib-steps", type=int, default=512)
    ap.add_argument("--phase-steps", type=int, default=256)
    ap.add_argument("--kernel-reps", type=int, default=28)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-gate-point", action="store_true",
                    help="skip the 4K-history gate-overhead point")
    ap.add_argument("--no-da", action="store_true",
                    help="skip the block-mask (Declarative Attention) sub-measurement")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the short runs of the other workloads")
    ap.add_argument("--quick", action="store_true",
                    help="main timed region only (used for profiler launch lists)")
    ap.add_argument("--conditional", action="store_true",
                    help="put the Full phase behind a graph IF node set by the gate, instead of "
                         "the default device-side early exit of the persistent Full kernel (ncu "
                         "lists kernel nodes only of graphs without conditional nodes)")
    ap.add_argument("--step-kernels", choices=sorted(STEP_KERNELS), default="full-persistent",
                    help="full-persistent: Local one launch per layer, the gate kernel, Full "
                         "at every layer as one launch; persistent: Local at every layer with "
                         "the fused gate as one launch too; per-layer: one launch per layer "
                         "and phase")
    ap.add_argument("--profile-kernel",
                    choices=["full", "local", "recall", "train", "step"],
                    help="a small case for ncu captures, launched --steps times; prints "
                         "nothing. full / local / recall / train: one layer of the workload "
                         "and the named per-layer kernel; step: the step graph over "
                         "--profile-layers layers with every step gated (theta = -inf), so "
                         "that both persistent kernels run")
    ap.add_argument("--profile-layers", type=int, default=4)
    ap.add_argument("--ncu-summary", nargs=4, metavar=("CSV", "KERNEL", "OUT", "EXTRA"),
                    help="write OUT (JSON): the per-launch DRAM bytes of KERNEL's launches in "
                         "CSV (an `ncu --page raw --csv` export), with the JSON object EXTRA "
                         "describing one launch (tokens_per_layer, layers_per_launch, ...); "
                         "needs no GPU")
    return ap.parse_args()


# ---------------------------------------------------------------------------------------
# Distributed plumbing: one process per GPU, each rank its own replica of the workload.
# ---------------------------------------------------------------------------------------
class Dist:
    def __init__(self, gpus: int):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            backend = "nccl" if torch.cuda.is_available() else "gloo"
            if backend == "nccl":
                torch.cuda.set_device(self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            self.pg.barrier()

    def max(self, x: float) -> float:
        if self.pg is None:
            return x
        t = torch.tensor([x], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def sum(self, x: float) -> float:
        if self.pg is None:
            return x
        t = torch.tensor([x], dtype=torch.float64,
                         device="cuda" if torch.cuda.is_available() else "cpu")
        self.pg.all_reduce(t, op=self.pg.ReduceOp.SUM)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------------------------------
# Clocks sampled during the timed region.
# ---------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", "oda_clocks_%d_%d.csv" % (os.getpid(), index))

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), parts[4:8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        seen = sorted({names[i] for _, _, r in rows for i, v in enumerate(r) if v == "Active"})
        return {"sm_mhz": float(np.median([r[0] for r in rows])),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": seen, "samples": len(rows)}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            return float(json.load(open(p))["hbm_gbs"]), "measured"
        except (ValueError, KeyError):
            pass
    return FALLBACK_HBM_GBS, "fallback"


HOST_MARK = "// Host side."


def kernel_source_hash(sources=None) -> str:
    """Hash of a kernel's device code (default: the decode kernels'): each source file up to
    its "// Host side." section (host argument checks and launch wrappers cannot change what
    a kernel reads), with comments and blank lines removed, so that a change of wording does
    not void the stored ncu counters but any change of device code does."""
    h = hashlib.sha256()
    for name in (KERNEL_SOURCES if sources is None else sources):
        text = open(os.path.join(ROOT, "sparse_kv_recall_b200", "csrc", name)).read()
        if HOST_MARK in text:
            text = text[:text.index(HOST_MARK)]
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        lines = [ln.rstrip() for ln in text.splitlines() if ln.strip()]
        h.update("\n".join(lines).encode())
    return h.hexdigest()[:16]


def _profile_fields(path: str, sources=None) -> dict:
    """The figures of a committed ncu capture (a JSON file written by --ncu-summary); empty when
    the file is missing or was taken on other kernel sources."""
    if not os.path.exists(path):
        return {}
    try:
        info = json.load(open(path))
    except ValueError:
        return {}
    return info if info.get("source_sha") == kernel_source_hash(sources) else {}


def profiled_traffic(n_ctx_tokens_per_layer: float, layers: int = 1, key: str = "full_chain"):
    """DRAM bytes of a Full launch covering `layers` layers at this many context tokens per
    layer, from the committed ncu capture of that Full kernel (the persistent one, or one
    layer of the split kernel), scaled by tokens and layers, as its traffic grows in
    proportion; None when missing or stale."""
    info = _profile_fields(PROFILES[key], profile_sources(key))
    try:
        per_token = float(info["dram_bytes_per_launch"]) / (
            float(info["tokens_per_layer"]) * float(info["layers_per_launch"]))
        return per_token * n_ctx_tokens_per_layer * layers
    except (KeyError, ValueError, ZeroDivisionError):
        return None


def profiled_step_bytes(mode: str, layers: int, full_phases_per_step: float,
                        n_ctx_tokens: float):
    """DRAM bytes one step of the long-context workload reads and writes, from the committed
    ncu captures of the kernels the step mode runs (Local: the per-layer cluster kernel and
    the recall kernel, or the persistent Local kernel with the fused recall head; Full: the
    persistent Full kernel, or one split launch per layer, on the steps that run it): the
    "bytes actually moved" figure beside the attended (algorithmic) bytes. None when a capture
    is missing or stale."""
    def per_launch(key):
        info = _profile_fields(PROFILES[key], profile_sources(key))
        return float(info["dram_bytes_per_launch"]) / float(info.get("layers_per_launch", 1))
    try:
        if mode == "persistent":
            local = per_launch("local_chain") * layers
        else:
            local = per_launch("local_cluster") * layers + per_launch("recall")
    except (KeyError, ValueError, ZeroDivisionError):
        return None
    full = profiled_traffic(n_ctx_tokens, layers,
                            "full_layer" if mode == "per-layer" else "full_chain")
    if full is None:
        return None
    return local + full_phases_per_step * full


def ncu_summary(csv_path: str, kernel: str, out_path: str, extra: dict) -> dict:
    """Average per-launch DRAM bytes of the launches of `kernel` (a substring of the kernel
    name) in an `ncu --page raw --csv` export, written as JSON with the hash of the device
    sources they were taken on and the caller's description of the launch (`extra`)."""
    import csv
    rows = list(csv.reader(open(csv_path)))
    head = None
    for i, r in enumerate(rows):
        if "Kernel Name" in r:
            head, rows = r, rows[i + 1:]
            break
    if head is None:
        raise ValueError("no header row in %s" % csv_path)
    ki = head.index("Kernel Name")
    cols = {m: head.index(m) for m in ("dram__bytes_read.sum", "dram__bytes_write.sum",
                                       "gpu__time_duration.sum") if m in head}
    units = rows[0] if rows and not rows[0][ki] else None
    scale = {}
    for m, j in cols.items():
        u = (units[j] if units else "").strip().lower()
        scale[m] = {"byte": 1, "kbyte": 1e3, "mbyte": 1e6, "gbyte": 1e9, "ns": 1e-9, "us": 1e-6,
                    "usecond": 1e-6, "msecond": 1e-3, "nsecond": 1e-9}.get(u, 1)
    picked = [r for r in rows if len(r) > ki and kernel in r[ki]]
    if not picked:
        raise ValueError("no launch of %s in %s" % (kernel, csv_path))

    def mean(m):
        vals = [float(r[cols[m]].replace(",", "")) * scale[m] for r in picked]
        return sum(vals) / len(vals)

    info = dict(extra)
    info.update({"kernel": picked[0][ki][:120], "launches_captured": len(picked),
                 "source_sha": kernel_source_hash(profile_sources(kernel)),
                 "dram_bytes_read_per_launch": mean("dram__bytes_read.sum"),
                 "dram_bytes_write_per_launch": mean("dram__bytes_write.sum")})
    info["dram_bytes_per_launch"] = (info["dram_bytes_read_per_launch"]
                                     + info["dram_bytes_write_per_launch"])
    if "gpu__time_duration.sum" in cols:
        info["gpu_time_s_per_launch_under_ncu"] = mean("gpu__time_duration.sum")
    json.dump(info, open(out_path, "w"), indent=1)
    return info


# ---------------------------------------------------------------------------------------
# The product arm.
# ---------------------------------------------------------------------------------------
class Setup:
    """Caches, recall head, engine and the resident pool of per-step inputs."""

    def __init__(self, w, seed_offset: int, n_steps_total: int, theta: float, dev: str,
                 use_conditional: bool = False, step_kernels: int = 0):
        from sparse_kv_recall_b200.engine import OdaEngine, StagingLayout, fill_staging
        self.w = oda_synth.scaled(w, seed=w.seed + 1000 * seed_offset)
        w = self.w
        self.lengths = oda_synth.prefill_lengths(w)
        # a fixed capacity keeps the page layout, hence the synthetic cache, the same whatever
        # number of steps a run takes
        self.layout = oda_synth.make_layout(w, extra_tokens=max(n_steps_total + 4, 8192),
                                            device=dev)
        self.caches = [oda_synth.make_kv_cache(w, self.layout, l, device=dev) for l in range(w.layers)]
        rw = oda_synth.make_recall_weights(w, device=dev)
        self.recall = (rw.w1, rw.b1, rw.w2, rw.b2)
        self.eng = OdaEngine([c[0] for c in self.caches], [c[1] for c in self.caches],
                             self.layout.block_table, w.num_q_heads, self.recall, theta,
                             sink=w.sink, window=w.window, use_conditional=use_conditional,
                             step_kernels=step_kernels, staging_slots=2)
        self.eng.set_h_prev(oda_synth.make_h0(w, device=dev), 0)
        lay = StagingLayout(w.layers, w.batch, w.num_q_heads, w.num_kv_heads, w.hidden)
        self.slot = lay.nbytes
        self.pool = torch.empty((n_steps_total, lay.nbytes), dtype=torch.uint8, device=dev)
        for i in range(n_steps_total):
            si = oda_synth.make_step_inputs(w, i, device=dev)
            fill_staging(lay.views(self.pool[i]), si, [n + i + 1 for n in self.lengths])
        torch.cuda.synchronize()

    def feed(self, i: int):
        """Step i's inputs from the resident pool into the staging slot its graph reads."""
        self.eng.staging_for(i).copy_(self.pool[i], non_blocking=True)


def launches_per_step(kernels, phases: int, steps: int, conditional: bool = True) -> int:
    """Kernels of this library launched by `steps` steps of which `phases` ran Full, for a
    step graph launching kernels = (Local, gate, Full) kernels per step."""
    local, gate, full = kernels
    return steps * (local + gate) + (phases if conditional else steps) * full


def calibrate_theta(s, w, C: int, step: int):
    """theta for the target Full-call rate, in two passes: the (1 - target rho) quantile of q
    over C/2 Local-only steps (graphs captured with theta = +inf), then the same quantile
    over C/2 steps gated at that first theta (q then sees the h_{t-1} trajectory that gating
    produces); returns (theta, next step index)."""
    def collect(n):
        nonlocal step
        qs = []
        for _ in range(n):
            s.feed(step)
            s.eng.launch(step)
            qs.append(s.eng.q_out.clone())
            step += 1
        return torch.cat(qs).double().cpu().numpy()
    theta = float(np.quantile(collect(C // 2), 1.0 - w.target_rho))
    s.eng.set_theta(theta)
    theta = float(np.quantile(collect(C - C // 2), 1.0 - w.target_rho))
    return theta, step


def phase_breakdown(s, w, theta: float, PH: int, step: int, stream):
    """PH steps of the same graphs with event nodes at the step's start and where the Full phase
    starts and ends (timing mode 2: no node between the last Local layer and the recall head,
    which would break the programmatic dependency the recall head's weight prefetch rides on);
    returns (phase dict, next step index)."""
    eng = s.eng
    eng.timing = 2
    eng.set_theta(theta)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(PH)]
    for row in evs:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    gated = []
    gates = torch.zeros((PH, w.batch), dtype=torch.int32, device=eng.gate.device)
    first = step
    for i in range(PH):
        before = eng.full_count[1].clone()
        eng.set_events(step, evs[i])
        s.feed(step)
        eng.launch(step)
        gates[i].copy_(eng.gate, non_blocking=True)
        gated.append(before)
        step += 1
    torch.cuda.synchronize()
    # Full-phase bytes of each step: its gated sequences' whole histories at every layer
    lens = np.array(s.lengths, dtype=np.float64)
    g_h = gates.cpu().numpy().astype(np.float64)
    full_bytes = [float((g_h[i] * (lens + first + i + 1)).sum()) * w.num_kv_heads * ROW_BYTES
                  * w.layers for i in range(PH)]
    counts = torch.stack(gated).cpu().tolist() + [int(eng.full_count[1].item())]
    ran_full = [counts[i + 1] > counts[i] for i in range(PH)]
    t_local = [evs[i][0].elapsed_time(evs[i][1]) for i in range(PH)]
    t_full = [evs[i][2].elapsed_time(evs[i][3]) for i in range(PH)]
    t_step = [evs[i][0].elapsed_time(evs[i][3]) for i in range(PH)]
    full_steps = [i for i in range(PH) if ran_full[i]]
    local_steps = [i for i in range(PH) if not ran_full[i]]
    mean = lambda xs: float(np.mean(xs)) if xs else None
    T_step, T_loc = mean(t_step), mean(t_local)
    T_full_exec = sum(t_full[i] for i in full_steps) / PH if PH else 0.0
    # The Local kernels alone (the same graphs captured with the Local phase only, event nodes
    # around it): with the persistent kernels the gate runs inside the Local launch, so the
    # step's Local phase above includes it and only this measurement separates them.
    from sparse_kv_recall_b200 import oda
    lo = eng.capture(math.inf, oda.ODA_PHASE_LOCAL)
    t_lo = []
    for i in range(min(PH, 64)):
        lo[step % 2].set_events(*evs[i])
        s.feed(step)
        lo[step % 2].launch()
        step += 1
        if i % 16 == 15:
            torch.cuda.synchronize()
            t_lo += [evs[k][0].elapsed_time(evs[k][1]) for k in range(i - 15, i + 1)]
    torch.cuda.synchronize()
    for x in lo:
        x.close()
    T_lo = mean(t_lo)
    gate_over = (T_step - T_lo - T_full_exec) / T_step if T_step and T_lo else None
    local_rows = sum(min(n + step - PH / 2 + 1, w.sink + w.window) for n in s.lengths)
    eng.timing = False
    eng.set_theta(theta)
    return {
        "steps": PH, "steps_with_full": len(full_steps), "ms_step": T_step,
        "ms_local_and_recall_phase": T_loc, "ms_local_kernels_alone": T_lo,
        "ms_recall_exposed": (T_loc - T_lo) if T_loc and T_lo else None,
        "ms_full_phase_when_run": mean([t_full[i] for i in full_steps]),
        "ms_full_phase_when_skipped": mean([t_full[i] for i in local_steps]),
        "gate_overhead": gate_over,
        "gate_overhead_def": "(T_step - T_local - T_full_executed) / T_step with event nodes at the "
                             "step's start and where the Full phase starts and ends: T_step and the "
                             "executed Full phase (summed over the steps that ran it, divided by all "
                             "steps) from the step graphs, T_local from the Local-only graph (the "
                             "gate excluded)",
        "local_phase_kv_gbs": (w.layers * w.num_kv_heads * local_rows * ROW_BYTES
                               / (T_lo / 1e3) / 1e9) if T_lo else None,
        "full_phase_kv_gbs": (sum(full_bytes[i] for i in full_steps)
                              / (sum(t_full[i] for i in full_steps) / 1e3) / 1e9)
                             if full_steps else None,
        "full_bytes_per_phase": mean([full_bytes[i] for i in full_steps]),
    }, step


def timed_steps(s, n: int, step: int, stream):
    """ms per step over n steps of the engine's current graphs (inputs fed from the pool)."""
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(n):
        s.feed(step)
        s.eng.launch(step)
        step += 1
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / n, step


def gate_cost(s, w, theta: float, n: int, step: int, stream, rounds: int = 4):
    """Step time of the same PDL-chained graphs (no event nodes inside) at the calibrated
    theta, at theta = +inf (Local + recall + skipped IF node), at theta = -inf (every step
    runs Full), as a Local-only graph and as a Local + recall graph (no IF node); the recall
    head and the IF machinery cost T(+inf) - T(Local only), split into the recall head
    T(Local + recall) - T(Local only) and the skipped IF node T(+inf) - T(Local + recall);
    the Full phase costs T(-inf) - T(+inf). The variants are captured once and timed in
    `rounds` interleaved rounds of n steps each; each figure is the median over rounds."""
    from sparse_kv_recall_b200 import oda
    eng = s.eng
    variants = [("oda", theta, 0), ("theta_plus_inf", math.inf, 0),
                ("theta_minus_inf", -math.inf, 0), ("local_only", math.inf, oda.ODA_PHASE_LOCAL),
                ("local_recall", math.inf, oda.ODA_PHASE_LOCAL | oda.ODA_PHASE_RECALL)]
    graphs = {name: eng.capture(th, ph) for name, th, ph in variants}
    times = {name: [] for name, _, _ in variants}
    gated = 0
    for _ in range(rounds):
        for name, _, _ in variants:
            g = graphs[name]
            for _ in range(4):                                # settle on this graph
                s.feed(step)
                g[step % 2].launch()
                step += 1
            fc0 = eng.full_count.clone()
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(n):
                s.feed(step)
                g[step % 2].launch()
                step += 1
            b.record(stream)
            torch.cuda.synchronize()
            times[name].append(a.elapsed_time(b) / n)
            if name == "oda":
                gated += int((eng.full_count - fc0)[0].item())
    for g in graphs.values():
        for x in g:
            x.close()
    T = {name: float(np.median(v)) for name, v in times.items()}
    overhead = T["theta_plus_inf"] - T["local_only"]
    rho = gated / float(w.batch * n * rounds)
    full = T["theta_minus_inf"] - T["theta_plus_inf"]
    return {"ms_per_step": T, "rounds": rounds, "steps_per_round": n,
            "rho_realised": rho,
            "ms_gate_and_full_skip": overhead,
            "ms_gate": T["local_recall"] - T["local_only"],
            "ms_full_phase_skipped": T["theta_plus_inf"] - T["local_recall"],
            "ms_full_phase": full,
            "gate_overhead": overhead / T["oda"],
            "gate_overhead_def": "(T(theta=+inf) - T(Local-only graph)) / T(calibrated theta): "
                                 "the gate and the skipped Full phase per step over the whole "
                                 "step, graphs without event nodes, medians of interleaved rounds",
            "gate_overhead_survey": (T["oda"] - T["local_only"] - rho * full) / T["oda"],
            "gate_overhead_survey_def": "(T_step - T_local - T_full_executed) / T_step from the same "
                                        "graphs without event nodes: T_full_executed = realised rho "
                                        "x (T(theta=-inf) - T(theta=+inf))"}, step


def step_variants(s, w, theta: float, rho: float, n: int, step: int, stream):
    """Two variants of the same step graphs, timed like the main region:
    * the random-timing ablation at the realised Full-call rate rho (gate = u < rho on the
      step's uniform draws, no recall head);
    * a hybrid access range: every 4th layer outside the Local restriction (it attends its
      whole history in the Local pass too), the rest Local-first as usual."""
    eng = s.eng
    res = {}
    for name, kw in [("random_schedule_matched_rho", {"random_rho": rho}),
                     ("hybrid_every_4th_layer_full", {"local_layers": [0 if l % 4 == 3 else 1
                                                                       for l in range(w.layers)]})]:
        eng.random_rho = kw.get("random_rho")
        eng.local_layers = kw.get("local_layers")
        eng.set_theta(theta)
        _, step = timed_steps(s, 8, step, stream)
        fc0 = eng.full_count.clone()
        ms, step = timed_steps(s, n, step, stream)
        res[name] = {"steps": n, "ms_per_step": ms, "tokens_per_s": w.batch / (ms / 1e3),
                     "rho_realised": float((eng.full_count - fc0)[0].item()) / (w.batch * n)}
    res["hybrid_every_4th_layer_full"]["layers_outside_restriction"] = w.layers // 4
    eng.random_rho, eng.local_layers = None, None
    eng.set_theta(theta)
    return res, step


def cp_emulation(s, w, stream, reps: int = 10):
    """Context-parallel Full on one GPU: the history split into R page-aligned shards
    (cp.shard_bounds), each shard's SHARD decode timed alone -- the Full work one GPU of an
    R-GPU group would do -- plus the LSE merge of R partials. The all-gather between GPUs is
    not part of it (one GPU here)."""
    from sparse_kv_recall_b200 import cp, oda
    eng = s.eng
    kv, q = eng.kvs[min(1, w.layers - 1)], eng.v["q_full_%d" % min(1, w.layers - 1)]
    B, Hq = w.batch, w.num_q_heads
    dev = q.device
    cap = int(eng.seq_lens.max().item())

    def time_it(fn):
        # reps launches captured in one CUDA graph, so that host launch cost (ctypes and the
        # launch call, ~10 us) cannot hide a short kernel's device time
        fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / reps

    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=dev)
    full_ms = time_it(lambda: oda.oda_decode_full(kv, q, eng.scale, out, eng.decode_ws))
    res = {"context_tokens": cap, "full_ms": full_ms, "note": "per-GPU shard decode and merge "
           "timed on one GPU (%d launches per CUDA graph, no PDL); the NCCL all-gather (%d B "
           "per sequence per rank) is not timed" % (reps, Hq * 129 * 4)}
    for R in (2, 4, 8):
        o_all = torch.empty(R, B, Hq, 128, dtype=torch.float32, device=dev)
        l_all = torch.empty(R, B, Hq, dtype=torch.float32, device=dev)
        shard_ms = []
        for r, (lo, hi) in enumerate(cp.shard_bounds(cap, R)):
            vis = oda.shard_visibility(lo, hi)
            shard_ms.append(time_it(lambda: oda.oda_decode(kv, vis, q, eng.scale, o_all[r],
                                                           eng.decode_ws, lse=l_all[r])))
        merge_ms = time_it(lambda: oda.oda_merge_partials(o_all, l_all, out))
        res["cp%d" % R] = {"shard_ms_max": max(shard_ms), "shard_ms_min": min(shard_ms),
                           "merge_ms": merge_ms,
                           "full_speedup_excl_allgather": full_ms / (max(shard_ms) + merge_ms)}
    return res


def run_train_grad(w, dev, stream, batch: int = 8, reps: int = 50):
    """Recall-head training objective: loss and gradient (oda_recall_loss_grad, two
    launches) for a batch of `batch` rows at the workload's hidden size, timed over `reps`
    calls captured in one CUDA graph. Bytes: W1 read once, dW1 written once."""
    from sparse_kv_recall_b200 import oda
    wl = oda_synth.scaled(w, batch=batch, name=w.name + "-train")
    rw = oda_synth.make_recall_weights(wl, device=dev)
    g = torch.Generator(device=dev).manual_seed(wl.seed)
    hp, em, hl = (torch.randn(batch, wl.hidden, generator=g, device=dev) for _ in range(3))
    gain = oda_synth.make_gains(wl, 0, device=dev)
    ws = torch.zeros(oda.oda_recall_train_workspace_size(batch, wl.hidden, wl.mlp),
                     dtype=torch.uint8, device=dev)
    loss, db2 = torch.empty(1, device=dev), torch.empty(1, device=dev)
    dw1, db1, dw2 = torch.empty_like(rw.w1), torch.empty_like(rw.b1), torch.empty_like(rw.w2)
    call = lambda: oda.oda_recall_loss_grad(hp, em, hl, rw.w1, rw.b1, rw.w2, rw.b2, gain, 0.5, ws,
                                            loss, dw1, db1, dw2, db2)
    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(reps):
            call()
    graph.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    graph.replay()
    b.record(stream)
    torch.cuda.synchronize()
    us = a.elapsed_time(b) / reps * 1e3
    nbytes = 2 * rw.w1.numel() * 4
    del graph
    return {"batch": batch, "hidden": wl.hidden, "mlp": wl.mlp, "us_per_call": us,
            "launches_per_call": 2, "w1_read_plus_dw1_write_bytes": nbytes,
            "gbs": nbytes / (us / 1e6) / 1e9, "loss": float(loss.item())}


def run_brief(name: str, dev: str, stream, steps: int = 64, with_gate_cost: bool = False):
    """A short run of another workload through the same step graphs: theta calibrated to its
    target Full-call rate (or its fixed theta), `steps` timed steps; tokens/s, the realised
    rate and the KV bytes it attended per second."""
    w = oda_synth.WORKLOADS[name]
    C = 0 if w.theta is not None else 256
    GC = 16 if with_gate_cost else 0
    total = C + 8 + steps + (5 * 4 * (GC + 4) if GC else 0) + 8
    s = Setup(w, 0, total, float("inf") if w.theta is None else w.theta, dev)
    theta, step = w.theta, 0
    if theta is None:
        theta, step = calibrate_theta(s, w, C, step)
        s.eng.set_theta(theta)
    for _ in range(8):
        s.feed(step)
        s.eng.launch(step)
        step += 1
    torch.cuda.synchronize()
    fc0, st0 = s.eng.full_count.clone(), s.eng.stats.clone()
    ms, step = timed_steps(s, steps, step, stream)
    fc = (s.eng.full_count - fc0).cpu().tolist()
    st = (s.eng.stats - st0).cpu().tolist()
    peak, peak_kind = measured_peak()
    kv = st[0] * ROW_BYTES / (ms * steps / 1e3) / 1e9
    res = {"workload": w.name, "layers": w.layers, "batch": w.batch, "q_heads": w.num_q_heads,
           "kv_heads": w.num_kv_heads, "prefill": w.prefill if w.ragged is None else
           "U%s" % (list(w.ragged),), "steps": steps, "ms_per_step": ms,
           "tokens_per_s": w.batch / (ms / 1e3), "rho_target": w.target_rho, "theta": theta,
           "rho_realised": fc[0] / float(w.batch * steps), "kv_gbs": kv,
           "frac_of_peak": kv / peak, "peak_kind": peak_kind,
           "kernels_per_step": s.eng.graphs[0].kernels()}
    if GC:
        res["gate_cost"], step = gate_cost(s, w, theta, GC, step, stream)
    assert int(s.eng.status.item()) == 0
    s.eng.close()
    del s
    torch.cuda.empty_cache()
    return res


def run_gate_point(args, dev, stream, prefill: int = 4096, steps: int = 256):
    """The gate-overhead point: the default workload's shapes with a short history."""
    w = oda_synth.scaled(oda_synth.WORKLOADS[args.workload], prefill=prefill,
                         name=args.workload + "@%d" % prefill)
    C, W = 256, 8
    s = Setup(w, 0, C + W + 5 * 4 * (steps // 4 + 4) + steps + 128, float("inf"), dev)
    theta, step = calibrate_theta(s, w, C, 0)
    s.eng.set_theta(theta)
    for _ in range(W):
        s.feed(step)
        s.eng.launch(step)
        step += 1
    res, step = gate_cost(s, w, theta, steps // 4, step, stream)
    ph, step = phase_breakdown(s, w, theta, steps, step, stream)
    assert int(s.eng.status.item()) == 0
    s.eng.close()
    res.update({"workload": w.name, "tokens_per_s": w.batch / (res["ms_per_step"]["oda"] / 1e3),
                "theta": theta, "phases_with_event_nodes": ph})
    return res


def run_da(w, dist: Dist, steps: int, warmup: int, dev: str, stream, e2e: bool = True,
           device_modes: bool = False):
    """Declarative-Attention block-mask decode: per step and sequence a mode is drawn
    (global / focus / local), its keep-page list built on the host (da.keep_pages), and the
    step runs the commit of the step's K/V (oda_kv_append) and the keep-list decode
    (oda_decode_blockmask). Keep lists, counts, lengths and q/k/v for every step sit in a
    resident pool (one copy per step); with e2e the same steps run from pinned host memory.
    device_modes: the step carries only each sequence's declared mode and focus offset, and
    oda_decode compiles them into page runs on the device (no keep list exists)."""
    from sparse_kv_recall_b200 import da, oda
    lengths = oda_synth.prefill_lengths(w)
    total = warmup + steps + (steps if e2e else 0)
    lay = oda_synth.make_layout(w, extra_tokens=total + 4, device=dev)
    kc, vc = oda_synth.make_kv_cache(w, lay, 0, device=dev)
    maxkeep = lay.block_table.shape[1]
    B, Hq, Hkv = w.batch, w.num_q_heads, w.num_kv_heads
    # pool row: seq_lens [B] | counts [B] | keep [B][maxkeep] (int32) | q | k | v (bf16), or
    # with device_modes seq_lens [B] | modes [B] | offsets [B]; the int32 block is padded to
    # 256 bytes so the bf16 tensors start 16-byte aligned
    n_used = 3 * B if device_modes else 2 * B + B * maxkeep
    n_int = n_used
    n_int = (n_int * 4 + 255) // 256 * 256 // 4
    n_bf = B * Hq * 128 + 2 * B * Hkv * 128
    row = n_int * 4 + n_bf * 2
    pool = torch.empty((total, row), dtype=torch.uint8, device=dev)
    for i in range(total):
        pos = [n + i for n in lengths]
        draws = oda_synth.draw_da_modes(w, i, pos)
        ints = np.zeros(n_int, np.int32)
        lens = np.array([p + 1 for p in pos], np.int32)
        if device_modes:
            ints[:n_used] = np.concatenate([lens, [d.mode for d in draws],
                                            [d.focus_offset for d in draws]])
        else:
            keep, counts = da.keep_lists(draws, pos, maxkeep)
            ints[:n_used] = np.concatenate([lens, counts, keep.reshape(-1)])
        ints = torch.from_numpy(ints)
        si = oda_synth.make_step_inputs(w, i, device=dev)
        pool[i, :n_int * 4].copy_(ints.view(torch.uint8))
        bf = torch.cat([si.q_local[0].reshape(-1), si.k_local[0].reshape(-1), si.v_local[0].reshape(-1)])
        pool[i, n_int * 4:].copy_(bf.view(torch.uint8))
    stage = torch.empty(row, dtype=torch.uint8, device=dev)
    ints = stage[:n_int * 4].view(torch.int32)
    seq = ints[:B]
    if device_modes:
        vis = oda.da_visibility(ints[B:2 * B], ints[2 * B:3 * B], focus_len=w.da_focus_len,
                                recent=w.da_recent, local_len=w.da_local_len)
    else:
        counts, keep = ints[B:2 * B], ints[2 * B:2 * B + B * maxkeep].view(B, maxkeep)
    bfv = stage[n_int * 4:].view(torch.bfloat16)
    q = bfv[:B * Hq * 128].view(B, Hq, 128)
    k_new = bfv[B * Hq * 128:B * Hq * 128 + B * Hkv * 128].view(B, Hkv, 128)
    v_new = bfv[B * Hq * 128 + B * Hkv * 128:].view(B, Hkv, 128)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stats = torch.zeros(2, dtype=torch.int64, device=dev)
    kv = oda.make_kv(kc, vc, lay.block_table, seq, status, stats)
    ws = torch.zeros(oda.oda_decode_workspace_size(B, Hkv, Hq), dtype=torch.uint8, device=dev)
    out = torch.empty(B, Hq, 128, dtype=torch.float32, device=dev)
    scale = 1.0 / math.sqrt(128)

    def step(src):
        stage.copy_(src, non_blocking=True)
        oda.oda_kv_append(kv, k_new, v_new)
        if device_modes:
            oda.oda_decode(kv, vis, q, scale, out, ws)
        else:
            oda.oda_decode_blockmask(kv, q, scale, keep, counts, out, ws)

    for i in range(warmup):
        step(pool[i])
    torch.cuda.synchronize()
    st0 = stats.clone()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(warmup, warmup + steps):
        step(pool[i])
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    st = (stats - st0).cpu().tolist()
    res = {"workload": w.name, "keep_spec": "device-compiled modes (%d B per step)" % (3 * 4 * B)
           if device_modes else "host keep lists (%d B per step)" % (4 * (2 * B + B * maxkeep)),
           "steps": steps, "tokens_per_s": B * steps / (ms / 1e3),
           "ms_per_step": ms / steps, "attended_rows_per_step": st[0] / steps,
           "kv_gbs": st[0] * ROW_BYTES / (ms / 1e3) / 1e9,
           "page_gbs": st[1] * PAGE_BYTES / (ms / 1e3) / 1e9,
           "gpu_launches": 2 * steps}
    if e2e:
        host = torch.empty((steps, row), dtype=torch.uint8, pin_memory=True)
        host.copy_(pool[warmup + steps:])
        out_h = torch.empty((B, Hq, 128), dtype=torch.float32, pin_memory=True)
        torch.cuda.synchronize()
        a.record(stream)
        for i in range(steps):
            step(host[i])
            out_h.copy_(out, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        res["e2e"] = {"tokens_per_s": B * steps / (a.elapsed_time(b) / 1e3),
                      "h2d_bytes_per_step": row, "d2h_bytes_per_step": B * Hq * 128 * 4}
    assert int(status.item()) == 0, "device status %d" % int(status.item())
    del kc, vc, pool
    torch.cuda.empty_cache()
    return res


def run_da_main(args, dist: Dist, w, dev: str):
    """The block-mask workload as the bench's main line."""
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    dist.barrier()
    r = run_da(oda_synth.scaled(w, seed=w.seed + 1000 * dist.rank), dist, args.steps,
               max(args.warmup, 3), dev, stream, e2e=not args.no_e2e)
    dist.barrier()
    ms = dist.max(r["ms_per_step"] * args.steps)
    peak, peak_kind = measured_peak()
    res = {"metric": METRIC, "value": dist.sum(w.batch * args.steps) / (ms / 1e3), "unit": UNIT,
           "n_gpus": dist.world, "steps": args.steps, "warmup": max(args.warmup, 3),
           "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": {"workload": w.name, "layers": 1, "batch_per_gpu": w.batch,
                      "q_heads": w.num_q_heads, "kv_heads": w.num_kv_heads, "prefill": w.prefill,
                      "modes": "global/focus/local p=%s" % (w.da_probs,), "kv_dtype": "bf16",
                      "l2": "no flush: ~1.9 GB of kept pages per step >> L2"},
           "kv_stream": {"gbs": r["kv_gbs"], "frac_of_peak": r["kv_gbs"] / peak, "peak_gbs": peak,
                         "peak_kind": peak_kind, "frac_of_nominal": r["kv_gbs"] / NOMINAL_HBM_GBS,
                         "nominal_gbs": NOMINAL_HBM_GBS,
                         "attended_rows_per_step": r["attended_rows_per_step"]},
           "gpu_launches": r["gpu_launches"], "clocks": clocks.stop()}
    if "e2e" in r:
        res["e2e"] = {"value": r["e2e"]["tokens_per_s"], "unit": UNIT,
                      "h2d_bytes_per_step": r["e2e"]["h2d_bytes_per_step"],
                      "d2h_bytes_per_step": r["e2e"]["d2h_bytes_per_step"]}
    return res


def run_oda(args, dist: Dist):
    from sparse_kv_recall_b200 import build as B
    from sparse_kv_recall_b200 import oda
    B.build()
    oda.load()
    dev = "cuda:%d" % dist.local
    torch.cuda.set_device(dist.local)
    w = oda_synth.WORKLOADS[args.workload]
    if w.mode == "da":
        return run_da_main(args, dist, w, dev), None
    K, W, C = args.steps, max(args.warmup, 3), args.calib_steps
    if w.theta is not None:
        C = 0
    PH = 0 if args.quick else args.phase_steps
    GC = 0 if args.quick else 64
    E2E = 0 if (args.quick or args.no_e2e) else min(K, 256)
    VAR = 0 if args.quick else 128
    total = (C + W + K + PH + min(PH, 64) + (5 * 4 * (GC + 4) if GC else 0) + E2E
             + (2 * VAR + 16 if VAR else 0))
    s = Setup(w, dist.rank, total, float("inf") if w.theta is None else w.theta, dev,
              use_conditional=args.conditional,
              step_kernels=STEP_KERNELS[args.step_kernels])
    eng = s.eng
    stream = torch.cuda.current_stream()
    step = 0

    # theta for the target Full-call rate: quantile of q over Local-only calibration steps
    theta = w.theta
    if theta is None:
        theta, step = calibrate_theta(s, w, C, step)
        eng.set_theta(theta)

    for _ in range(W):
        s.feed(step)
        eng.launch(step)
        step += 1
    torch.cuda.synchronize()

    # ---- main timed region: K steps, inputs resident in HBM ----
    fc0 = eng.full_count.clone()
    st0 = eng.stats.clone()
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    step0 = step
    e0.record(stream)
    for _ in range(K):
        s.feed(step)
        eng.launch(step)
        step += 1
    e1.record(stream)
    torch.cuda.synchronize()
    dist.barrier()
    clk = clocks.stop()
    ms_local = e0.elapsed_time(e1)
    ms = dist.max(ms_local)
    fc = (eng.full_count - fc0).cpu().tolist()
    st = (eng.stats - st0).cpu().tolist()
    tokens_local = w.batch * K
    tokens = dist.sum(tokens_local)
    rho = fc[0] / float(w.batch * K)
    kv_bytes = st[0] * ROW_BYTES
    page_bytes = st[1] * PAGE_BYTES
    kernels = eng.graphs[0].kernels()
    launches = launches_per_step(kernels, fc[1], K, args.conditional)
    peak, peak_kind = measured_peak()
    result = {
        "metric": METRIC, "value": tokens / (ms / 1e3), "unit": UNIT, "n_gpus": dist.world,
        "steps": K, "warmup": W, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "layers": w.layers, "batch_per_gpu": w.batch,
                   "global_batch": w.batch * dist.world, "q_heads": w.num_q_heads,
                   "kv_heads": w.num_kv_heads, "head_dim": 128, "prefill": w.prefill,
                   "sink": w.sink, "window": w.window, "kv_dtype": "bf16",
                   "rho_target": w.target_rho, "rho_realised": rho, "theta": theta,
                   "calibration_steps": C, "full_phase": "graph IF node" if args.conditional
                   else "device early exit (no IF node)", "l2": "no flush: 15 GB KV stream per Full step >> 126 MB L2"
                   if w.name == DEFAULT_WORKLOAD else "no flush: KV working set > L2",
                   "parallelism": "replicas (dp%d, no collective)" % dist.world},
        "kv_stream": {"attended_bytes": kv_bytes, "gbs": kv_bytes / (ms_local / 1e3) / 1e9,
                      "frac_of_peak": kv_bytes / (ms_local / 1e3) / 1e9 / peak,
                      "page_bytes": page_bytes, "peak_gbs": peak, "peak_kind": peak_kind,
                      "frac_of_nominal": kv_bytes / (ms_local / 1e3) / 1e9 / NOMINAL_HBM_GBS,
                      "nominal_gbs": NOMINAL_HBM_GBS},
        "rho_realised": rho,
        "hbm_frac_whole_step": kv_bytes / (ms_local / 1e3) / 1e9 / peak,
        "gpu_launches": launches,
        "kernels_per_step": {"local": kernels[0], "gate": kernels[1], "full": kernels[2],
                             "step_kernels": args.step_kernels},
        "clocks": clk,
    }
    if w.name == DEFAULT_WORKLOAD:
        # DRAM bytes of the step's kernels as ncu counted them (committed summaries), with the
        # Full launches at the timed region's mean context
        ctx_mid = float(np.mean(s.lengths)) + step0 + K / 2.0 + 1.0
        sb = profiled_step_bytes(args.step_kernels, w.layers, fc[1] / float(K), ctx_mid * w.batch)
        result["kv_stream"]["ncu_bytes_per_step"] = sb
        result["kv_stream"]["ncu_gbs"] = (sb * K / (ms_local / 1e3) / 1e9) if sb else None
        result["kv_stream"]["ncu_frac_of_peak"] = (sb * K / (ms_local / 1e3) / 1e9 / peak
                                                   if sb else None)
    if args.quick:
        return result, s

    # ---- phase breakdown: same graphs with event nodes at the phase boundaries ----
    result["phases"], step = phase_breakdown(s, w, theta, PH, step, stream)
    result["gate_cost"], step = gate_cost(s, w, theta, GC, step, stream)
    # the two ends of the Full-call rate: every step Local only (rho = 0) and every step
    # recomputed with Full (rho = 1), from the same interleaved timings
    ctx = float(np.mean(s.lengths)) + step
    T = result["gate_cost"]["ms_per_step"]
    for name, key, rows in [("rho_0", "theta_plus_inf", min(ctx, w.sink + w.window)),
                            ("rho_1", "theta_minus_inf", min(ctx, w.sink + w.window) + ctx)]:
        kv = w.batch * w.layers * w.num_kv_heads * rows * ROW_BYTES
        result[name] = {"tokens_per_s": w.batch / (T[key] / 1e3), "ms_per_step": T[key],
                        "kv_gbs": kv / (T[key] / 1e3) / 1e9,
                        "frac_of_peak": kv / (T[key] / 1e3) / 1e9 / peak}
    # the same step at the target Full-call rate, from the interleaved timings: the step without
    # Full plus the target share of the Full phase (a step's time is linear in its Full calls)
    gc = result["gate_cost"]
    if w.target_rho is not None:
        ms_t = T["theta_plus_inf"] + w.target_rho * gc["ms_full_phase"]
        kv_t = w.batch * w.layers * w.num_kv_heads * ROW_BYTES * (
            min(ctx, w.sink + w.window) + w.target_rho * ctx)
        result["at_target_rho"] = {
            "rho": w.target_rho, "ms_per_step": ms_t, "tokens_per_s": w.batch / (ms_t / 1e3),
            "kv_gbs": kv_t / (ms_t / 1e3) / 1e9, "frac_of_peak": kv_t / (ms_t / 1e3) / 1e9 / peak,
            "how": "T(theta=+inf) + rho x (T(theta=-inf) - T(theta=+inf)) from gate_cost's "
                   "interleaved medians; KV bytes at the same context"}
    result["variants"], step = step_variants(s, w, theta, rho, VAR, step, stream)

    # ---- one Full layer alone: the split decode kernel at this context, CUDA events per launch
    from sparse_kv_recall_b200 import oda as O
    ones = torch.ones(w.batch, dtype=torch.int32, device=dev)
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float32, device=dev)
    q = eng.v["q_full_1" if w.layers > 1 else "q_full_0"]
    kevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.kernel_reps)]
    for r in range(3):
        O.oda_decode_full(eng.kvs[r % w.layers], q, eng.scale, out, eng.decode_ws, gate=ones)
    torch.cuda.synchronize()
    for r, (a, b) in enumerate(kevs):
        a.record(stream)
        O.oda_decode_full(eng.kvs[r % w.layers], q, eng.scale, out, eng.decode_ws, gate=ones)
        b.record(stream)
    torch.cuda.synchronize()
    dur = float(np.mean([a.elapsed_time(b) for a, b in kevs]))
    ctx_tokens = int(eng.seq_lens.sum().item())
    alg_layer = ctx_tokens * w.num_kv_heads * ROW_BYTES
    achieved_alone = alg_layer / (dur / 1e3) / 1e9
    # The dominant kernel as the step runs it: the Full phase -- one persistent launch over
    # every layer (or one launch per layer, chained by programmatic dependent launch) -- timed
    # by event nodes at its boundaries on the graph's stream; its bytes are the gated
    # sequences' histories at every layer at the phase's context.
    ph = result["phases"]
    full_launches = kernels[2]
    if ph.get("full_phase_kv_gbs"):
        achieved = ph["full_phase_kv_gbs"]
        alg = ph["full_bytes_per_phase"] / full_launches
        ms_launch = ph["ms_full_phase_when_run"] / full_launches
        how = ("the Full phase inside the step graph between event nodes: %d launch%s per step"
               % (full_launches, "" if full_launches == 1 else "es, PDL-chained"))
    else:
        achieved, alg, ms_launch, how = achieved_alone, alg_layer, dur, "one layer alone"
    traffic = profiled_traffic(alg / (w.num_kv_heads * ROW_BYTES * w.layers), w.layers) \
        if full_launches == 1 else profiled_traffic(alg / (w.num_kv_heads * ROW_BYTES), 1,
                                                    "full_layer")
    name = ("full_chain_kernel<%d> (Full at every layer, one launch)" % w.group
            if full_launches == 1 else "decode_kernel<%d> (Full, one layer)" % w.group)
    result["roofline"] = {"kernel": name,
                          "bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                          "frac": achieved / peak, "traffic": traffic,
                          "algorithmic_bytes": alg, "ms_per_launch": ms_launch, "timed": how,
                          "one_layer_alone": {"kernel": "decode_kernel<%d>" % w.group,
                                              "achieved": achieved_alone,
                                              "frac": achieved_alone / peak, "ms": dur,
                                              "algorithmic_bytes": alg_layer},
                          "peak_kind": peak_kind + " (copy)",
                          "frac_of_nominal": achieved / NOMINAL_HBM_GBS}

    if w.name == DEFAULT_WORKLOAD:
        result["context_parallel_1gpu"] = cp_emulation(s, w, stream)
        result["recall_train_grad"] = run_train_grad(w, dev, stream)

    # ---- end to end through the same API: host inputs in, selected output out ----
    if E2E:
        host_pool = torch.empty((E2E, s.slot), dtype=torch.uint8, pin_memory=True)
        host_pool.copy_(s.pool[step:step + E2E])
        out_h = torch.empty((2, w.batch, w.hidden), dtype=torch.float32, pin_memory=True)
        torch.cuda.synchronize()
        dist.barrier()
        fc_e = eng.full_count.clone()
        # through the engine's host path: inputs copied in and each step's result read out on
        # their own streams, overlapping the steps (OdaEngine.run_from_host)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step = eng.run_from_host(host_pool, out_h, step, stream)
        b.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        ms_e2e = dist.max(a.elapsed_time(b))
        rho_e = float((eng.full_count - fc_e)[0].item()) / (w.batch * E2E)
        gc = result.get("gate_cost", {}).get("ms_per_step", {})
        dev_model = (gc["theta_plus_inf"] + rho_e * (gc["theta_minus_inf"] - gc["theta_plus_inf"])
                     if gc else None)
        result["e2e"] = {"value": dist.sum(w.batch * E2E) / (ms_e2e / 1e3), "unit": UNIT,
                         "h2d_bytes_per_step": s.slot,
                         "d2h_bytes_per_step": w.batch * w.hidden * 4, "steps": E2E,
                         "ms_per_step": ms_e2e / E2E,
                         "device_ms_per_step_at_its_rho": dev_model,
                         "rho_realised": rho_e,
                         "note": "its own steps (later in the same decode), so its Full-call "
                                 "rate differs from the main region's"}
    assert int(eng.status.item()) == 0, "device status %d" % int(eng.status.item())
    if not args.no_gate_point and w.name == DEFAULT_WORKLOAD:
        result["gate_point_4k"] = run_gate_point(args, dev, stream)
    if not args.no_da and w.name == DEFAULT_WORKLOAD:
        result["da_blockmask_1m"] = run_da(oda_synth.WORKLOADS["da-1m-b2"], dist, 128, 4, dev,
                                           stream, e2e=False)
        result["da_device_modes_1m"] = run_da(oda_synth.WORKLOADS["da-1m-b2"], dist, 128, 4, dev,
                                              stream, e2e=False, device_modes=True)
    if not args.no_workloads and w.name == DEFAULT_WORKLOAD:
        # every other workload, briefly, through the same step graphs (this one's buffers freed
        # first: the ragged batch alone holds 87 GB of KV)
        s.eng.close()
        del s, eng
        torch.cuda.empty_cache()
        s = None
        wl = {}
        wl["pr1-ref-4k"] = run_brief("pr1-ref-4k", dev, stream, steps=64, with_gate_cost=True)
        for name in ("qwen3-1.7b-16k-b8", "qwen3-8b-ragged-b16"):
            wl[name] = run_brief(name, dev, stream, steps=64)
        wl[w.name] = {"workload": w.name, "see": "the main line", "tokens_per_s": result["value"],
                      "rho_realised": rho, "kv_gbs": result["kv_stream"]["gbs"],
                      "frac_of_peak": result["kv_stream"]["frac_of_peak"]}
        if "da_device_modes_1m" in result:
            d = result["da_device_modes_1m"]
            wl["da-1m-b2"] = {"workload": "da-1m-b2", "tokens_per_s": d["tokens_per_s"],
                              "rho_realised": None, "kv_gbs": d["kv_gbs"],
                              "frac_of_peak": d["kv_gbs"] / peak,
                              "note": "block-mask mode: no gate (device-compiled DA modes)"}
        result["workloads"] = wl
    return result, s


# ---------------------------------------------------------------------------------------
# The fp64 oracle on the host: the CPU baseline leg and the reference arm.
# ---------------------------------------------------------------------------------------
def _blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    except Exception:
        return 1


class OracleSampler:
    """Times the oracle on bounded pieces of one decode step of the workload and
    extrapolates to a whole step: Local at one layer (all heads), the recall head, and Full
    at one layer for one KV head (its G query heads) over one of `chunks` equal slices of the
    history (sample i takes slice i mod chunks; the oracle's cost is linear in positions);
    a step costs L * local + recall + rho * L * Hkv * chunks * full_slice."""

    def __init__(self, w, rho: float, dev: str, chunks: int = 1):
        self.chunks = chunks
        from oracle import oda_oracle as O
        self.O, self.w, self.rho = O, w, rho
        lay = oda_synth.make_layout(w, extra_tokens=8, device=dev)
        kc, vc = oda_synth.make_kv_cache(w, lay, 0, device=dev)
        self.kbits, self.vbits = oda_synth.bf16_bits(kc), oda_synth.bf16_bits(vc)
        del kc, vc
        self.bt = lay.block_table.cpu().numpy()
        self.t = oda_synth.prefill_lengths(w)[0]
        g = torch.Generator().manual_seed(w.seed)
        self.q = torch.randn((w.num_q_heads, 128), generator=g).to(torch.bfloat16)
        self.qbits = oda_synth.bf16_bits(self.q)
        rw = oda_synth.make_recall_weights(w)
        self.rec = [x.double().numpy() for x in (rw.w1, rw.b1, rw.w2)] + [rw.b2]
        self.h = np.random.default_rng(0).standard_normal((3, w.batch, w.hidden))

    def sample(self, i: int):
        """One bounded sample: (seconds it took, seconds a whole decode step of the batch
        would take at the same rates, i.e. the sample's time scaled by the share of the step's
        attended rows and recall work it covers)."""
        O, w = self.O, self.w
        G = w.num_q_heads // w.num_kv_heads
        qf = O.widen_bf16(self.qbits)
        t0 = time.perf_counter()
        pos = O.local_positions(self.t, w.sink, w.window)
        ks = [O.paged_rows(self.kbits, self.bt[0], pos, g) for g in range(w.num_kv_heads)]
        vs = [O.paged_rows(self.vbits, self.bt[0], pos, g) for g in range(w.num_kv_heads)]
        O.decode_attention(qf, ks, vs, 1 / math.sqrt(128))
        t1 = time.perf_counter()
        O.recall_score(self.h[0], self.h[1], self.h[2], *self.rec)
        t2 = time.perf_counter()
        g = i % w.num_kv_heads
        pos = np.array_split(O.full_positions(self.t), self.chunks)[i % self.chunks]
        kr = O.paged_rows(self.kbits, self.bt[0], pos, g)
        vr = O.paged_rows(self.vbits, self.bt[0], pos, g)
        O.decode_attention(qf[g * G:(g + 1) * G], [kr], [vr], 1 / math.sqrt(128))
        t3 = time.perf_counter()
        per_seq = (w.layers * (t1 - t0)
                   + self.rho * w.layers * w.num_kv_heads * self.chunks * (t3 - t2))
        return t3 - t0, w.batch * per_seq + (t2 - t1)


def host_cores() -> dict:
    return {"host_cores": os.cpu_count(), "blas_threads": _blas_threads()}


def cpu_baseline(w, rho: float, dev: str, budget_s: float = 20.0) -> dict:
    """The oracle on the host at the bench's workload: bounded samples, extrapolated."""
    s = OracleSampler(w, rho, dev)
    spent, n, total = 0.0, 0, 0.0
    while spent < budget_s and n < 64:
        wall, whole = s.sample(n)
        total += whole
        spent += wall
        n += 1
    res = {"value": w.batch * n / total, "unit": UNIT, "cores": _blas_threads(),
           "kind": "oracle", "extrapolated": True,
           "sample": ("%d oracle samples of one %s decode step (Local at one layer, recall, Full "
                      "at one layer for one KV head), EXTRAPOLATED by their share of the step's "
                      "work to all %d layers, %d KV heads and rho=%.3f; %.1f s of CPU time"
                      % (n, w.name, w.layers, w.num_kv_heads, rho, spent))}
    res.update(host_cores())
    return res


def cpu_baseline_full(name: str = "pr1-ref-4k") -> dict:
    """The oracle on the host over a whole small workload, every step, no extrapolation: the
    1-layer 4K workload (batch 1, 16 q / 8 KV heads, s = 4, w = 256, theta = 0, 64 steps), its
    inputs drawn on the host by the same seeded generators."""
    from oracle import oda_oracle as O
    w = oda_synth.WORKLOADS[name]
    lengths = oda_synth.prefill_lengths(w)
    lay = oda_synth.make_layout(w, extra_tokens=w.steps + 2, device="cpu")
    bt = lay.block_table.numpy()
    hist = []
    for l in range(w.layers):
        pair = []
        for t in oda_synth.make_kv_cache(w, lay, l, device="cpu"):
            bits = oda_synth.bf16_bits(t)
            arr = np.zeros((w.batch, w.num_kv_heads, max(lay.capacity), 128), dtype=np.uint16)
            for b, cap in enumerate(lay.capacity):
                p = np.arange(cap)
                arr[b, :, :cap] = bits[bt[b, p // 16], :, p % 16, :].transpose(1, 0, 2)
            pair.append(arr)
        hist.append(pair)
    rw = oda_synth.make_recall_weights(w)
    rec = (rw.w1.double().numpy(), rw.b1.double().numpy(), rw.w2.double().numpy(), rw.b2)
    dec = O.OdaDecoder([h[0] for h in hist], [h[1] for h in hist], lengths,
                       oda_synth.make_h0(w).double().numpy(), rec, sink=w.sink,
                       window=w.window, theta=w.theta)
    inputs = []
    for i in range(w.steps):
        si = oda_synth.make_step_inputs(w, i)
        inp = {k: [oda_synth.bf16_bits(x) for x in getattr(si, k)]
               for k in ("q_local", "k_local", "v_local", "q_full", "k_full", "v_full")}
        inp["emb"] = si.emb.double().numpy()
        inputs.append(inp)
    gated = 0
    t0 = time.perf_counter()
    for inp in inputs:
        _, _, _, g = dec.step(inp)
        gated += int(np.sum(g))
    wall = time.perf_counter() - t0
    res = {"workload": w.name, "value": w.batch * w.steps / wall, "unit": UNIT, "kind": "oracle",
           "extrapolated": False, "steps": w.steps, "seconds": wall,
           "rho_realised": gated / float(w.batch * w.steps),
           "sample": "every step of the workload through the oracle's ODA step (Local, recall "
                     "head, gate, Full when gated, commit), timed as one region"}
    res.update(host_cores())
    res["cores"] = res["blas_threads"]
    return res


def run_reference(args, dist: Dist):
    """The oracle, as it stands, timed on the host cores on this workload. Each step is one
    bounded sample of a decode step; the line's ms_per_step is the real wall time of a sample
    and its tokens/s counts each sample as the share of a decode step it covers."""
    if dist.rank != 0:
        return None
    w = oda_synth.WORKLOADS[args.workload]
    rho = w.target_rho if w.target_rho is not None else 0.5
    dev = "cuda:%d" % dist.local if torch.cuda.is_available() else "cpu"
    s = OracleSampler(w, rho, dev, chunks=16)
    for i in range(max(args.warmup, 3)):
        s.sample(i)
    t0 = time.perf_counter()
    samples = [s.sample(i) for i in range(args.steps)]
    wall = time.perf_counter() - t0
    tokens = sum(w.batch * sw / whole for sw, whole in samples)   # share of a step each covers
    value = tokens / wall
    cores = _blas_threads()
    sample = ("each step: one oracle sample of a %s decode step (Local at one layer, recall, "
              "Full at one layer for one KV head over 1/16 of the history), counted as the "
              "share of a whole step (%d layers, %d KV heads, the whole history, rho=%.3f) that "
              "its work covers; %.1f s wall" % (w.name, w.layers, w.num_kv_heads, rho, wall))
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": dist.world,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": 1e3 * wall / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": w.name, "rho": rho},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "host_cores": os.cpu_count(), "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_profile_case(args):
    """One layer of the workload (its KV pages still far larger than L2, a few GB at most),
    one decode step's inputs, and the named kernel launched args.steps times."""
    from sparse_kv_recall_b200 import build as B
    from sparse_kv_recall_b200 import oda
    B.build()
    oda.load()
    dev = "cuda"
    if args.profile_kernel == "step":
        run_profile_step(args, dev)
        return
    w = oda_synth.scaled(oda_synth.WORKLOADS[args.workload], layers=1)
    lengths = oda_synth.prefill_lengths(w)
    lay = oda_synth.make_layout(w, extra_tokens=8, device=dev)
    kc, vc = oda_synth.make_kv_cache(w, lay, 0, device=dev)
    si = oda_synth.make_step_inputs(w, 0, device=dev)
    seq = torch.tensor([n + 1 for n in lengths], dtype=torch.int32, device=dev)
    kv = oda.make_kv(kc, vc, lay.block_table, seq)
    ws = torch.zeros(oda.oda_decode_workspace_size(w.batch, w.num_kv_heads, w.num_q_heads),
                     dtype=torch.uint8, device=dev)
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float32, device=dev)
    rw = oda_synth.make_recall_weights(w, device=dev)
    rws = torch.zeros(oda.oda_recall_workspace_size(w.batch, w.hidden, w.mlp), dtype=torch.uint8,
                      device=dev)
    h = oda_synth.make_h0(w, device=dev)
    qo = torch.empty(w.batch, dtype=torch.float32, device=dev)
    go = torch.empty(w.batch, dtype=torch.int32, device=dev)
    scale = 1.0 / math.sqrt(128)
    if args.profile_kernel == "train":          # the recall head's loss and gradient, batch 8
        wt = oda_synth.scaled(w, batch=8)
        g = torch.Generator(device=dev).manual_seed(wt.seed)
        x = [torch.randn(8, wt.hidden, generator=g, device=dev) for _ in range(3)]
        gain = oda_synth.make_gains(wt, 0, device=dev)
        tws = torch.zeros(oda.oda_recall_train_workspace_size(8, wt.hidden, wt.mlp),
                          dtype=torch.uint8, device=dev)
        loss, db2 = torch.empty(1, device=dev), torch.empty(1, device=dev)
        dw1, db1, dw2 = torch.empty_like(rw.w1), torch.empty_like(rw.b1), torch.empty_like(rw.w2)
        train = lambda: oda.oda_recall_loss_grad(*x, rw.w1, rw.b1, rw.w2, rw.b2, gain, 0.5, tws,
                                                 loss, dw1, db1, dw2, db2)
    for _ in range(args.steps):
        if args.profile_kernel == "full":
            oda.oda_decode_full(kv, si.q_full[0], scale, out, ws)
        elif args.profile_kernel == "local":
            oda.oda_decode_local(kv, si.q_local[0], w.sink, w.window, scale, out, ws)
        elif args.profile_kernel == "recall":
            oda.oda_recall_score(h, si.emb, out.view(w.batch, -1), rw.w1, rw.b1, rw.w2, rw.b2,
                                 0.0, qo, go, rws)
        else:
            train()
    torch.cuda.synchronize()


def run_profile_step(args, dev: str):
    """The step graph of the workload over --profile-layers layers (KV pages far larger than
    L2, a few GB), every step gated, launched --steps times on fresh staged inputs."""
    from sparse_kv_recall_b200.engine import OdaEngine, fill_staging
    w = oda_synth.scaled(oda_synth.WORKLOADS[args.workload], layers=args.profile_layers)
    lengths = oda_synth.prefill_lengths(w)
    lay = oda_synth.make_layout(w, extra_tokens=args.steps + 8, device=dev)
    caches = [oda_synth.make_kv_cache(w, lay, l, device=dev) for l in range(w.layers)]
    rw = oda_synth.make_recall_weights(w, device=dev)
    eng = OdaEngine([c[0] for c in caches], [c[1] for c in caches], lay.block_table,
                    w.num_q_heads, (rw.w1, rw.b1, rw.w2, rw.b2), -float("inf"), sink=w.sink,
                    window=w.window, use_conditional=False)
    eng.set_h_prev(oda_synth.make_h0(w, device=dev), 0)
    for i in range(args.steps):
        si = oda_synth.make_step_inputs(w, i, device=dev)
        fill_staging(eng.v, si, [n + i + 1 for n in lengths])
        eng.launch(i)
    torch.cuda.synchronize()
    assert int(eng.status.item()) == 0, "device status %d" % int(eng.status.item())
    eng.close()


def main():
    args = parse_args()
    if args.ncu_summary:
        csv_path, kernel, out, extra = args.ncu_summary
        print(json.dumps(ncu_summary(csv_path, kernel, out, json.loads(extra))))
        return
    if args.profile_kernel:
        run_profile_case(args)
        return
    dist = Dist(args.gpus)
    try:
        if args.impl == "reference":
            res = run_reference(args, dist)
        else:
            res, setup = run_oda(args, dist)
            if (dist.rank == 0 and dist.world == 1 and "config" in res
                    and not (args.no_cpu_baseline or args.quick)):
                rho = res["config"].get("rho_realised") or 0.5
                del setup
                torch.cuda.empty_cache()
                res["cpu_baseline"] = cpu_baseline(oda_synth.WORKLOADS[args.workload], rho,
                                                   "cuda:%d" % dist.local)
                res["cpu_baseline_full_run"] = cpu_baseline_full()
        if res is not None and dist.rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        dist.close()


if __name__ == "__main__":
    main()
