#!/usr/bin/env python
"""Throughput of the gated delta rule on B200: one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: one chunked forward
(``gdr_chunk_fwd``) of the workload, or for the decode workload its 1000
consecutive single-token steps.  Default workload: the KDA forward at head
dim 128 (B=2, H=32, T=8192, d_k=d_v=128, C=64, bf16) -- the size the method's
throughput target is quoted at.

Multi-GPU (launched with torch.distributed.run, one process per GPU): every
(b, h) sequence is an independent recurrence, so each rank runs its own batch
of the same shape (different seed) with no collective on the data path
(weak scaling).  Timing: W untimed warm-up steps, then K steps bracketed by a
barrier and a device synchronize on both sides, timed with CUDA events on the
launching stream; the job time is the max over ranks; ``value`` is the
tokens all ranks processed divided by that time.

``--impl reference`` times the fp64 CPU oracle (the only reference this
method has) on the host cores, rank 0 only, each step a bounded sample of
the same workload.
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

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gdr_workloads as W  # noqa: E402

METRIC = "tokens/s (device-timed) of gated-delta-rule chunk fwd; % of roofline"
METRIC_DECODE = "tokens/s (device-timed) of gated-delta-rule recurrent decode step; % of HBM roofline"
METRIC_BWD = "tokens/s (device-timed) of gated-delta-rule chunk backward; % of roofline"
DEFAULT_WORKLOAD = "kda_d128_t8192"

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) per call of the
# path, from one ncu capture of every kernel the call launches, keyed by
# workload with the hash of the sources those kernels are built from; an
# entry is ignored (traffic = null) as soon as any of the sources changes.
TRAFFIC = {
    # B=1 capture doubled (4096 chunks; inputs and hand-off above L2 at both sizes):
    # ut_prep 276.4 MB read + 223.2 MB written, chunk_scan 339.8 + 52.6 MB (the sources
    # changed since only in comments)
    "kda_d128_t8192": {"src_sha": "19b440d103a63729", "bytes_per_launch": 1784198656},
    # recurrent_step, one decode step: 547.4 MB read + 477.8 MB written (recurrent_step.cu
    # unchanged since the capture; the shared header changed only in the tensor-core
    # workspace layout, which this kernel does not use)
    "kda_decode_b256": {"src_sha": "83851ff3a738fcf9", "bytes_per_launch": 1025204480},
}

CHUNK_SOURCES = ("chunk_tc.cu", "ut_prep.cu", "sm100_ptx.cuh", "gdr_internal.cuh")
DECODE_SOURCES = ("recurrent_step.cu", "gdr_internal.cuh")
BWD_SOURCES = ("chunk_bwd.cu", "gdr_internal.cuh")


# ----------------------------------------------------------------- helpers

def algorithmic_bytes(w: W.Workload) -> int:
    """Bytes one step must move at least: every input read once, every output
    written once (no intermediates)."""
    e = 2 if w.dtype == torch.bfloat16 else 4
    gate = w.dk * 4 if w.gate == "per_channel" else 4
    if w.g_recipe == "prologue":    # gate pre-activation in the input dtype, beta logits fp32
        gate = w.dk * e if w.gate == "per_channel" else e
    strength = 4                                                    # beta
    if w.rule == "gdr2":            # erase gate [dk] and write gate [dv] in the input dtype
        strength = (w.dk + w.dv) * e
    per_token = 2 * w.dk * e + w.dv * e + gate + strength + w.dv * e   # q, k, v, g, beta, O
    if w.out == "gated":            # the output gate pre-activation is read too
        per_token += w.dv * e
    heads = w.B * w.H
    state = 2 * w.dv * w.dk * 4                                     # S0 read + S_T write
    if w.direction == "bwd":
        # reads q, k, v, g, beta, dO; writes dq, dk, dv, dg, dbeta; S0 and dS_T read, dS0 written
        per_token = 2 * w.dk * e + w.dv * e + gate + 4 + w.dv * e + (2 * w.dk * e + w.dv * e + gate + 4)
        state = 3 * w.dv * w.dk * 4
    if w.kind == "decode":
        return w.T * heads * (per_token + state)                    # the state moves every step
    return heads * w.T * per_token + heads * state


def dense_flops(w: W.Workload) -> int:
    """Tensor-core flops of one step of the chunk form (C x C tiles counted full)."""
    if w.kind == "decode":
        return w.T * w.B * w.H * 8 * w.dk * w.dv
    C, dk, dv = w.C, w.dk, w.dv
    per_chunk = 2 * C * C * (3 * dk + 2 * dv) + 6 * C * dk * dv
    return w.B * w.H * (w.T // C) * per_chunk


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# B200 datasheet peaks (HBM3e bandwidth, dense bf16 tensor throughput): the
# contract's `frac` is taken against the measured peaks above; `frac_vs_spec`
# states the same achievement against these.
SPEC_HBM_GBS = 8000.0
SPEC_BF16_TFLOPS = 2250.0


def roofline(w: W.Workload, seconds_per_launch: float, peaks, kernel_src: str = None):
    byts = algorithmic_bytes(w)
    flops = dense_flops(w)
    t_hbm = byts / (peaks["hbm_gbs"] * 1e9)
    t_tc = flops / (peaks["bf16_tflops"] * 1e12)
    traffic = None
    ent = TRAFFIC.get(w.name)
    if ent and kernel_src and ent.get("src_sha") == file_sha(kernel_src):
        traffic = ent["bytes_per_launch"]
    if t_hbm >= t_tc:
        ach = byts / seconds_per_launch / 1e9
        return {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": traffic,
                "peak_source": peaks["source"] + " (copy bandwidth)", "algorithmic_bytes": byts,
                "frac_vs_spec": round(ach / SPEC_HBM_GBS, 4), "spec_peak": SPEC_HBM_GBS}
    ach = flops / seconds_per_launch / 1e12
    return {"bound": "tensor", "achieved": round(ach, 2), "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(ach / peaks["bf16_tflops"], 4), "traffic": traffic,
            "peak_source": peaks["source"], "algorithmic_flops": flops,
            "frac_vs_spec": round(ach / SPEC_BF16_TFLOPS, 4), "spec_peak": SPEC_BF16_TFLOPS}


def file_sha(paths) -> str:
    """Hash of the concatenated sources (one path or several)."""
    if isinstance(paths, str):
        paths = [paths]
    h = hashlib.sha256()
    try:
        for p in paths:
            h.update(open(p, "rb").read())
    except OSError:
        return ""
    return h.hexdigest()[:16]


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """Weak scaling: rank r runs the same shapes with its own seed."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + 1000 * rank)


def job_throughput(units_per_rank_step: int, world: int, total_ms_max: float, steps: int) -> float:
    """Weak scaling: units all ranks processed per second of the slowest rank."""
    return units_per_rank_step * world / (total_ms_max / steps / 1e3)


def reduce_max(x: float, world: int, device) -> float:
    if world <= 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------ clock sampler

_REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]


class NvmlClockSampler:
    """SM clock, max SM clock and active clock-event reasons read through NVML
    (the library nvidia-smi reports from) every ~1 ms in a background thread,
    so that even a timed region of a few milliseconds holds several samples.
    Only reads settings."""

    _BITS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40, "sw_power_cap": 0x4}

    def __init__(self, device_index: int, period_s: float = 0.001):
        import pynvml
        pynvml.nvmlInit()
        self.nv = pynvml
        self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
        self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM))
        self.samples = []
        self.period = period_s
        self.running = True
        self.proc = True
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def _run(self):
        nv = self.nv
        while self.running:
            try:
                mhz = float(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.time(), mhz, self.max_mhz, [r for r, b in self._BITS.items() if bits & b]))
            except Exception:
                pass
            time.sleep(self.period)

    def wait_first(self, timeout_s: float = 5.0):
        t0 = time.time()
        while not self.samples and time.time() - t0 < timeout_s:
            time.sleep(0.001)

    def stop(self):
        self.running = False
        self.thread.join(timeout=2)

    def summary(self, t0: float, t1: float):
        return ClockSampler.summary(self, t0, t1)

    def window(self, t0: float, t1: float):
        return self.summary(t0, t1)


def make_sampler(device):
    try:
        return NvmlClockSampler(device.index if device.index is not None else 0)
    except Exception:
        return ClockSampler(gpu_id_for(device))


class ClockSampler:
    """nvidia-smi samples (SM clock, max clock, throttle reasons) in the background."""

    def __init__(self, gpu_id: str, period_ms: int = 20):
        self.samples = []
        self.proc = None
        fields = "timestamp,clocks.sm,clocks.max.sm,power.draw," + ",".join(
            "clocks_event_reasons." + r for r in _REASONS)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={fields}", "--format=csv,noheader,nounits",
                 f"-lms={period_ms}"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4 + len(_REASONS):
                continue
            try:
                self.samples.append((time.time(), float(parts[1]), float(parts[2]),
                                     [r for r, v in zip(_REASONS, parts[4:]) if v.lower() == "active"]))
            except ValueError:
                pass

    def wait_first(self, timeout_s: float = 5.0):
        """Block until the sampler has produced a sample (so the timed region is covered)."""
        t0 = time.time()
        while self.proc is not None and not self.samples and time.time() - t0 < timeout_s:
            time.sleep(0.01)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "note": "nvidia-smi unavailable"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        note = "samples inside the timed region"
        if not inside:
            inside = sorted(self.samples, key=lambda s: min(abs(s[0] - t0), abs(s[0] - t1)))[:3]
            note = "timed region shorter than the sampling period; nearest samples"
        reasons = sorted({r for s in inside for r in s[3]})
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": max(s[2] for s in inside),
                "reasons": reasons, "samples": len(inside), "note": note}


def gpu_id_for(device) -> str:
    try:
        u = torch.cuda.get_device_properties(device).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return str(device.index if device.index is not None else 0)


# ------------------------------------------------------------ CPU oracle leg

def api_call(gdr, w: W.Workload, x, **kw):
    """One forward of workload ``w`` through the public Python API."""
    if w.g_recipe == "prologue":
        return gdr.chunk_fwd_prologue(x["q_raw"], x["k_raw"], x["v"], x["a"], x["A_log"], x["dt_bias"],
                                      x["b_logit"], x["S0"], C=w.C, gate=w.gate, **kw)
    if w.direction == "bwd":
        return gdr.chunk_bwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["dO"], S0=x["S0"], dS_T=x["dS_T"],
                             C=w.C, gate=w.gate, **kw)
    if w.out == "gated":
        return gdr.chunk_fwd_gated(x["q"], x["k"], x["v"], x["g"], x["beta"], x["ogate"], x["norm_w"], 1e-6,
                                   x["S0"], C=w.C, gate_mode=w.gate, **{("Y" if k == "O" else k): v for k, v in kw.items()})
    if w.rule == "gdr2":
        return gdr.chunk_fwd_gdr2(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"], C=w.C, gate=w.gate, **kw)
    return gdr.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], C=w.C, gate=w.gate, **kw)


def oracle_sample(w: W.Workload, budget_s: float, seed_rank: int = 0):
    """Time the fp64 oracle on a bounded sample of workload ``w``.

    The sample is whole heads (spread over the batch) over the first
    ``tokens`` tokens (or decode steps), sized from a short calibration run to
    take about ``budget_s`` seconds; when the whole workload takes less than
    that, the whole workload is run, repeatedly, until the budget is used.
    Returns (tokens/s in the workload's unit, description dict).
    """
    import oracle
    cores = oracle.online_cores()
    heads_total = w.B * w.H

    def pick(nh):
        step = max(1, heads_total // nh)
        return list(range(0, heads_total, step))[:nh]

    def run(hl, ntok):
        if w.kind == "decode":
            x = W.generate(w, heads=hl, steps=ntok)
            t = time.perf_counter()
            if w.rule == "gdr2":
                oracle.decode_gdr2(x["q"], x["k"], x["v"], x["g"], x["b"], x["w"], x["S0"], gate=w.gate,
                                   threads=cores)
            else:
                oracle.decode(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], gate=w.gate, threads=cores)
            return time.perf_counter() - t
        if w.g_recipe == "prologue":
            # the sampled heads laid out as B = 1, H = len(hl), with their own A_log, dt_bias
            x = W.generate_prologue(w, heads=hl)
            sl = lambda a: a.transpose(0, 1)[:, :, :ntok].contiguous()
            args = [sl(x[k]) for k in ("q_raw", "k_raw", "v", "a")]
            t = time.perf_counter()
            oracle.forward_prologue(*args, x["A_log"], x["dt_bias"], sl(x["b_logit"]), x["S0"].transpose(0, 1),
                                    gate=w.gate, threads=cores)
            return time.perf_counter() - t
        x = W.generate(w, heads=hl)
        sl = lambda a: a[:, :, :ntok].contiguous()
        if w.direction == "bwd":
            gr = W.generate_grads(w, heads=hl)
            args = [sl(x[k]) for k in ("q", "k", "v", "g", "beta")]
            t = time.perf_counter()
            oracle.backward(*args, x["S0"], sl(gr["dO"]), gr["dS_T"], gate=w.gate, threads=cores)
            return time.perf_counter() - t
        if w.rule == "gdr2":
            args = [sl(x[k]) for k in ("q", "k", "v", "g", "b", "w")]
            t = time.perf_counter()
            oracle.forward_gdr2(*args, x["S0"], gate=w.gate, threads=cores)
            return time.perf_counter() - t
        args = [sl(x[k]) for k in ("q", "k", "v", "g", "beta")]
        t = time.perf_counter()
        if w.out == "gated":
            oracle.forward_gated(*args, sl(x["ogate"]), x["norm_w"], 1e-6, x["S0"], gate_mode=w.gate, threads=cores)
        else:
            oracle.forward(*args, x["S0"], gate=w.gate, threads=cores)
        return time.perf_counter() - t

    # calibrate on one head per core
    hl = pick(min(heads_total, cores))
    cal_tok = min(w.T, 256)
    per_head_tok = run(hl, cal_tok) / (len(hl) * cal_tok) * min(len(hl), cores)
    full_est = per_head_tok * heads_total * w.T / min(heads_total, cores)
    if full_est <= budget_s:
        hl, ntok = pick(heads_total), w.T
    else:
        ntok = w.T
        nh = int(budget_s / (per_head_tok * ntok) * min(heads_total, cores))
        if nh < min(heads_total, cores):
            nh = min(heads_total, cores)
            ntok = max(cal_tok, int(budget_s / (per_head_tok * ntok) * ntok))
        hl = pick(max(1, min(heads_total, nh)))
    times = []
    t_all = time.perf_counter()
    while True:
        times.append(run(hl, ntok))
        if time.perf_counter() - t_all >= budget_s or len(times) >= 50:
            break
    dt = statistics.median(times)
    head_tokens_per_s = len(hl) * ntok / dt
    # a workload token (one position of one sequence) spans all H heads
    tokens_per_s = head_tokens_per_s / w.H
    unit_note = "decode steps" if w.kind == "decode" else "tokens"
    return tokens_per_s, {"kind": "oracle", "cores": min(cores, len(hl)),
                          "sample": f"fp64 oracle on {len(hl)} of {heads_total} heads x {ntok} {unit_note} "
                                    f"of {w.name}, median of {len(times)} runs ({sum(times):.1f} s total)",
                          "seconds": round(sum(times), 2)}


# ------------------------------------------------------------------ main

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other configurations timed after the headline (one GPU only)")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch size (smaller profiler captures; not a bench line)")
    return ap.parse_args()


def base_line(w: W.Workload, args, world: int):
    return {
        "metric": METRIC_DECODE if w.kind == "decode" else METRIC_BWD if w.direction == "bwd" else METRIC,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == torch.bfloat16 else "f32",
        "data": "synthetic (seeded counter-based generator, shapes and value recipes of the workload)",
        "config": {
            "workload": w.name, "description": w.description, "B": w.B, "H": w.H, "T": w.T,
            "dk": w.dk, "dv": w.dv, "C": w.C, "gate": w.gate,
            "global_batch": w.B * world, "seq_len": w.T,
            "parallelism": f"dp{world} (independent sequences per GPU, no collective)",
            "l2": "inputs larger than L2 (%.0f MB per step vs 126 MB)" % (algorithmic_bytes(w) / 1e6),
        },
    }


def run_reference(args, w: W.Workload, rank: int, world: int):
    if rank != 0:
        return 0
    budget = max(1.0, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    vals = []
    desc = None
    for i in range(args.warmup + args.steps):
        v, desc = oracle_sample(w, budget)
        if i >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    line = base_line(w, args, world)
    line.update({"impl": "reference", "value": value,
                 "ms_per_step": (w.tokens / value) * 1e3,
                 "cpu_baseline": dict(desc, value=value, unit="tokens/s"),
                 "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
                 "gpu_launches": 0})
    print(json.dumps(line), flush=True)
    return 0


def build_step(gdr, w: W.Workload, device):
    """Inputs of workload ``w`` resident in HBM and the step that runs it:
    returns (step, x, O, S_T) with O, S_T the buffers the step writes."""
    if w.kind == "decode":
        x = W.generate(w, device=device, steps=w.T)
        S = x["S0"].clone()
        o = torch.empty(w.B, w.H, w.dv, dtype=w.dtype, device=device)

        if w.rule == "gdr2":
            def step():
                for s in range(w.T):
                    gdr.recurrent_step_gdr2(x["q"][s], x["k"][s], x["v"][s], x["g"][s], x["b"][s], x["w"][s], S,
                                            o=o)
        else:
            def step():
                for s in range(w.T):
                    gdr.recurrent_step(x["q"][s], x["k"][s], x["v"][s], x["g"][s], x["beta"][s], S, o=o)
        return step, x, o, S
    if w.g_recipe == "prologue":
        x = W.generate_prologue(w, device=device)
        O = torch.empty(w.B, w.H, w.T, w.dv, dtype=w.dtype, device=device)
        S_T = torch.empty(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=device)
        return (lambda: api_call(gdr, w, x, O=O, S_T=S_T)), x, O, S_T
    if w.direction == "bwd":
        x = W.generate(w, device=device)
        x.update(W.generate_grads(w, device=device))
        bws = torch.empty(gdr.chunk_bwd_workspace_size(w.B, w.H, w.T, w.dk, w.dv, w.C, w.gate, w.dtype),
                          dtype=torch.uint8, device=device)
        # the result read back in the end-to-end measurement: dq (shape of q) and dS0
        return (lambda: api_call(gdr, w, x, workspace=bws)), x, x["dO"], x["dS_T"]
    x = W.generate(w, device=device)
    if w.rule == "gdr2":
        del x["beta"]           # the erase and write gates take its place
    O = torch.empty(w.B, w.H, w.T, w.dv, dtype=w.dtype, device=device)
    S_T = torch.empty(w.B, w.H, w.dv, w.dk, dtype=torch.float32, device=device)
    return (lambda: api_call(gdr, w, x, O=O, S_T=S_T)), x, O, S_T


def time_steps(step, steps: int, warmup: int, stream, device, world: int):
    """W untimed steps, then K steps between barriers and synchronizes, each
    bracketed by CUDA events on the launching stream.  Returns the per-step
    device times (ms) and the wall-clock window of the timed region."""
    for _ in range(warmup):
        step()
    torch.cuda.synchronize(device)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    t_wall0 = time.time()
    for i in range(steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
    torch.cuda.synchronize(device)
    t_wall1 = time.time()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    return [a.elapsed_time(b) for a, b in ev], t_wall0, t_wall1


def kernel_sources(w: W.Workload):
    return [os.path.join(ROOT, "gated_delta_rule_89_b200", "csrc", f)
            for f in (DECODE_SOURCES if w.kind == "decode" else BWD_SOURCES if w.direction == "bwd"
                      else CHUNK_SOURCES)]


def roofline_for(w: W.Workload, step_ms, peaks):
    """Roofline of one launch of the dominant path: one chunked call, or one
    decode step (a decode workload step is w.T launches)."""
    import dataclasses
    per_launch_s = statistics.mean(step_ms) / 1e3 / (w.T if w.kind == "decode" else 1)
    wk = dataclasses.replace(w, T=1) if w.kind == "decode" else w
    return roofline(wk, per_launch_s, peaks, kernel_sources(w))


# the other configurations of the method's workload list, timed in the same
# process after the headline (one GPU only)
EXTRA_WORKLOADS = ("gdn_scalar_t4096", "kda_long_t65536", "kda_decode_b256")


def main():
    args = parse()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", str(args.gpus)))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w0 = W.WORKLOADS[args.workload]
    if args.batch is not None:
        import dataclasses
        w0 = dataclasses.replace(w0, B=args.batch, name=f"{w0.name}_b{args.batch}")

    if args.impl == "reference":
        return run_reference(args, w0, rank, world if "WORLD_SIZE" in os.environ else args.gpus)

    import gated_delta_rule_89_b200 as gdr

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=device)
    w = rank_workload(w0, rank)
    stream = torch.cuda.current_stream(device)

    # ---- inputs resident in HBM before timing
    step, x, O, S_T = build_step(gdr, w, device)
    torch.cuda.synchronize(device)

    sampler = make_sampler(device) if rank == 0 else None
    if sampler is not None:
        sampler.wait_first()
    step()
    launches_per_step = gdr.last_launch_count() * (w.T if w.kind == "decode" else 1)
    step_ms, t_wall0, t_wall1 = time_steps(step, args.steps, max(0, args.warmup - 1), stream, device, world)
    total_ms = reduce_max(sum(step_ms), world, device)
    ms_per_step = total_ms / args.steps
    # chunk: B*T tokens per step; decode: B sequences x T consecutive steps
    value = job_throughput(w.B * w.T, world, total_ms, args.steps)
    clocks = sampler.summary(t_wall0, t_wall1) if sampler is not None else None

    # ---- end to end through the public API with host buffers (pinned)
    e2e = None
    if w.kind != "decode" and args.e2e_steps > 0:
        hx = {k: v.to("cpu").pin_memory() for k, v in x.items()}
        h2d = sum(v.numel() * v.element_size() for v in hx.values())
        if w.direction == "bwd":   # every gradient comes back
            d2h = sum(x[n].numel() * x[n].element_size() for n in ("q", "k", "v", "g", "beta", "S0"))
        else:
            d2h = O.numel() * O.element_size() + S_T.numel() * S_T.element_size()
        api_call(gdr, w, hx)  # warm
        torch.cuda.synchronize(device)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            res = api_call(gdr, w, hx)
        e1.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = reduce_max(e0.elapsed_time(e1), world, device) / args.e2e_steps
        e2e = {"value": w.tokens * world / (e2e_ms / 1e3), "unit": "tokens/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 3)}
        del hx
    elif w.kind == "decode":
        e2e = {"value": None, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0,
               "note": "not measured for the decode workload"}

    line = None
    if rank == 0:
        peaks = load_peaks()
        line = base_line(w0, args, world)
        line.update({
            "value": value,
            "ms_per_step": round(ms_per_step, 4),
            "roofline": roofline_for(w0, step_ms, peaks),
            "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e,
            "clocks": clocks,
        })
        if world == 1 and not args.no_cpu_baseline:
            v, desc = oracle_sample(w0, args.cpu_budget)
            line["cpu_baseline"] = dict(desc, value=v, unit="tokens/s")

    # ---- the other configurations, same process, same steps (one GPU only)
    if world == 1 and not args.no_extra:
        del step, x, O, S_T
        torch.cuda.empty_cache()
        extra = {}
        for name in EXTRA_WORKLOADS:
            if name == w0.name:
                continue
            we = W.WORKLOADS[name]
            st, xe, Oe, Se = build_step(gdr, we, device)
            torch.cuda.synchronize(device)
            st()
            lp = gdr.last_launch_count() * (we.T if we.kind == "decode" else 1)
            ms, a0, a1 = time_steps(st, args.steps, max(0, args.warmup - 1), stream, device, 1)
            extra[name] = {
                "metric": METRIC_DECODE if we.kind == "decode" else METRIC,
                "config": {"B": we.B, "H": we.H, "T": we.T, "dk": we.dk, "dv": we.dv, "C": we.C, "gate": we.gate,
                           "description": we.description},
                "ms_per_step": round(statistics.mean(ms), 4),
                "value": we.B * we.T / (statistics.mean(ms) / 1e3),
                "unit": "tokens/s",
                "roofline": roofline_for(we, ms, load_peaks()),
                "gpu_launches": lp * args.steps,
                "clocks": sampler.summary(a0, a1) if sampler is not None else None,
            }
            del st, xe, Oe, Se
            torch.cuda.empty_cache()
        if line is not None:
            line["workloads"] = extra

    if sampler is not None:
        sampler.stop()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
