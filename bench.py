#!/usr/bin/env python
"""Throughput of the NF4-LoRA linear layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-graph] [--no-few]

One step is one pass of the layer over one batch of the workload.  The
default workload is the LLaMA-65B layer's seven linears (q/k/v/o 8192 x 8192,
gate/up 8192 -> 22016, down 22016 -> 8192), NF4 + double quantisation, LoRA
r = 64, 2048 tokens: forward then backward (dX, dA, dB) of every module in
layer order.  That step is dense-bf16 tensor bound, so the headline `value`
is its algorithmic TFLOP/s.  The same line carries, as sub-objects:

* ``quantize`` -- the encoding of the seven fp32 weights (nf4_quantize),
  HBM bound, in GB/s;
* ``few_token`` -- the LLaMA-7B q_proj 4096 x 4096 at M in {1, 4, 16},
  forward plus input gradient (the decode-like, HBM-bound path), in GB/s
  of the weight stream;
* ``optimizer`` (the AdamW step of A and B) and ``merge`` (the adapter folded
  into the base and encoded again), each with its roofline.

Inputs are seeded and synthetic (``workloads.py``).  Between timed steps the
encoded weights rotate over enough copies to exceed 4x the L2 cache, so every
pass streams its weight from HBM.  The timed steps are replayed from CUDA
graphs captured without the library's launch tracing; the per-kernel device
times behind each roofline come from a separate traced pass of the same steps
right after the timed region.  ``--only quantize|merge|optimizer`` times one
phase alone (a short command to profile).

Rank 0 prints ONE JSON line.  With N > 1 (torchrun, one process per GPU)
every rank runs the same per-GPU workload on its own data (weak scaling) and
the time is the max over ranks.  A forward + input-gradient workload has no
exchange step (independent replicas); a full-backward workload is a
data-parallel training step, so the ranks sum their adapter gradients dA, dB
with one all-reduce per module (``nf4_base_lora_b200.dp``) inside the timed
region.  ``--impl reference`` times the CPU oracle (the plain fp64 statement
of the method) on the host on the same bounded sample of the workload that the
``cpu_baseline`` key reports.
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
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "NF4-LoRA linear fwd+bwd TFLOP/s & weight GB/s at 1 B200; % of roofline"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ---------------------------------------------------------------- accounting
def weight_bytes(d_out, d_in):
    """Stored bytes of one NF4 + double-quantised weight (4.127 bits/weight)."""
    n = d_out * d_in
    return n / 2 + n / 64 + 4 * n / (64 * 256)


def pass_bytes(d_out, d_in, m, r, kind):
    """Algorithmic bytes of one pass: weights, adapters, activations in and out."""
    w = weight_bytes(d_out, d_in)
    if kind == "fwd":
        return w + 2 * m * d_in + 2 * m * d_out + 2 * r * (d_in + d_out) + 2 * m * r
    if kind == "dx":
        return w + 2 * m * d_out + 2 * m * d_in + 2 * r * (d_in + d_out) + 2 * m * r
    return w + 2 * m * d_out + 4 * m * d_in + 4 * r * (d_in + d_out) + 2 * m * r


def pass_flops(d_out, d_in, m, r, kind):
    if kind == "fwd" or kind == "dx":
        return 2 * m * d_in * d_out + 2 * m * r * (d_in + d_out)
    return 2 * m * d_in * d_out + 4 * m * r * (d_in + d_out)


def step_plan(wl):
    """[(module index, module, M, kind)] of one step."""
    plan = []
    for i, mod in enumerate(wl.modules):
        for m in wl.tokens:
            plan.append((i, mod, m, "fwd"))
            plan.append((i, mod, m, "dx" if wl.backward == "dx" else "full"))
    return plan


def exchange_points(plan):
    """{pass index: module index} of the pass after which a module's adapter
    gradients are final for the step (its last full backward pass)."""
    last = {}
    for p, (i, _, _, kind) in enumerate(plan):
        if kind == "full":
            last[i] = p
    return {p: i for i, p in last.items()}


def step_totals(wl):
    b = f = 0.0
    for _, mod, m, kind in step_plan(wl):
        b += pass_bytes(mod.d_out, mod.d_in, m, wl.r, kind)
        f += pass_flops(mod.d_out, mod.d_in, m, wl.r, kind)
    return b, f


def load_peaks():
    """Roofline denominators: the measured copy bandwidth and bf16 GEMM
    rates of this machine's B200s (burst: a kernel timed alone; sustained: a
    seconds-long loop under the power cap), else the recorded fallback."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        burst = float(p["bf16_tflops"])
        return {"hbm": float(p["hbm_gbs"]), "bf16": burst,
                "bf16_sustained": float(p.get("bf16_tflops_sustained", burst)), "source": "measured"}
    except Exception:
        return {"hbm": FALLBACK_HBM_GBS, "bf16": FALLBACK_BF16_TFLOPS, "bf16_sustained": 1400.0,
                "source": "fallback"}


def kernel_flops(d_out, d_in, m, r, kernel):
    """Algorithmic flops of one launch of a fused dequant-GEMM: the base
    product plus the rank-r term it accumulates (the LoRA-up T B^T for the
    forward, V A for the input gradient)."""
    if kernel.startswith("nf4_gemm_fwd"):
        return 2 * m * d_in * d_out + 2 * m * r * d_out
    return 2 * m * d_in * d_out + 2 * m * r * d_in


def tensor_bound(wl):
    return max(wl.tokens) > 16


def kernel_source_hash(files=None):
    """Hash of the CUDA sources a kernel is built from (all of the library's
    when `files` is None): a traffic figure is used only while the kernel is
    the one it was measured on."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "nf4_base_lora_b200", "csrc")
    names = sorted(files) if files else sorted(os.listdir(csrc))
    for name in names:
        if name.endswith((".cu", ".cuh", ".h")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode())
                h.update(f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source
    has not changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        e = t.get(workload, {}).get(kernel)
        if e and e.get("source_hash") == kernel_source_hash(e.get("sources")):
            return float(e["bytes_per_launch"])
    except Exception:
        pass
    return None


def load_traffic_per_weight(kernel):
    """DRAM bytes per weight of a kernel whose traffic grows in proportion to
    the weights it processes (the encoder, the merge), from a capture of a
    smaller case, under the same source-hash rule."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            e = json.load(f).get("per_weight", {}).get(kernel)
        if e and e.get("source_hash") == kernel_source_hash(e.get("sources")):
            return float(e["bytes_per_weight"])
    except Exception:
        pass
    return None


# ---------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.device_index = device_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.device_index), "--query-gpu=" + self.QUERY,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append(ln.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- oracle arm
# The CPU oracle is timed on one fixed, bounded sample of the workload: the
# first ORACLE_ROWS weight rows (a whole number of 256-block groups) of the
# first module, i.e. that slice's share of every pass of the step.  The
# cpu_baseline key and the --impl reference arm time the same sample, in the
# headline's unit.
ORACLE_ROWS = 256


def oracle_rows(mod):
    unit = max(4, (256 * 64) // mod.d_in)   # rows of one 256-block group
    return max(unit, ORACLE_ROWS // unit * unit)


def oracle_sample_step(oracle, qt, mod, wl, host, rows):
    """The oracle on `rows` weight rows of one module: its share of every
    pass of the step.  Returns (algorithmic bytes, flops) of that share."""
    d_in = mod.d_in
    n = rows * d_in
    packed = qt["packed"][:n // 2]
    q = qt["q"][:n // 64]
    a2 = qt["a2"]
    bits = oracle.dequantize_bits(packed, q, a2, float(qt["mu"]), n)
    W_hat = oracle.bf16_bits_to_f32(bits).reshape(rows, d_in)
    A, B = host["A"], host["B"][:rows]
    nbytes = nflops = 0.0
    for m in wl.tokens:
        X = host["X"][:m]
        dY = host["dY"][:m, :rows]
        oracle.forward(W_hat, A, B, X, wl.scaling)
        if wl.backward == "dx":
            oracle.input_grad_rows(W_hat, A, B, dY, wl.scaling)
            kinds = ("fwd", "dx")
        else:
            oracle.backward(W_hat, A, B, X, dY, wl.scaling)
            kinds = ("fwd", "full")
        for kind in kinds:
            nbytes += pass_bytes(rows, d_in, m, wl.r, kind)
            nflops += pass_flops(rows, d_in, m, wl.r, kind)
    return nbytes, nflops


def oracle_setup(wl):
    import oracle
    mod = wl.modules[0]
    W = workloads.weight(mod.d_out, mod.d_in, wl.sigma, wl.outliers, 0)
    qt = oracle.quantize(W)
    mmax = max(wl.tokens)
    host = {"A": workloads.lora_a(wl.r, mod.d_in, 0), "B": workloads.lora_b(mod.d_out, wl.r, 0),
            "X": workloads.activations(mmax, mod.d_in), "dY": workloads.grad_output(mmax, mod.d_out, 0)}
    return oracle, qt, mod, host


def oracle_unit(wl):
    return "TFLOP/s" if tensor_bound(wl) else "GB/s"


def oracle_value(wl, nbytes, nflops, seconds):
    return nflops / seconds / 1e12 if tensor_bound(wl) else nbytes / seconds / 1e9


def oracle_sample_text(wl, mod, rows):
    return "%d of %d weight rows of %s (its share of every pass of the step: %s at M = %s)" % (
        rows, mod.d_out, mod.name, "fwd + dX" if wl.backward == "dx" else "fwd + dX + dA + dB",
        "/".join(str(m) for m in wl.tokens))


def host_cores():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def time_oracle(wl, budget_s, min_steps=1):
    """Time oracle sample steps for about budget_s seconds of host work."""
    oracle, qt, mod, host = oracle_setup(wl)
    rows = oracle_rows(mod)
    t0 = time.perf_counter()
    oracle_sample_step(oracle, qt, mod, wl, host, rows)
    one = time.perf_counter() - t0
    steps = max(min_steps, int(budget_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    nb = nf = 0.0
    for _ in range(steps):
        b, f = oracle_sample_step(oracle, qt, mod, wl, host, rows)
        nb += b
        nf += f
    dt = time.perf_counter() - t0
    return {"value": oracle_value(wl, nb, nf, dt), "unit": oracle_unit(wl), "cores": host_cores(),
            "kind": "oracle", "sample": oracle_sample_text(wl, mod, rows) + ", %d steps in %.1f s" % (steps, dt),
            "seconds": dt, "steps": steps}


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    oracle, qt, mod, host = oracle_setup(wl)
    rows = oracle_rows(mod)
    for _ in range(args.warmup):
        oracle_sample_step(oracle, qt, mod, wl, host, rows)
    t0 = time.perf_counter()
    nb = nf = 0.0
    for _ in range(args.steps):
        b, f = oracle_sample_step(oracle, qt, mod, wl, host, rows)
        nb += b
        nf += f
    dt = time.perf_counter() - t0
    value = oracle_value(wl, nb, nf, dt)
    unit = oracle_unit(wl)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": DATA, "config": workload_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": unit, "cores": host_cores(), "kind": "oracle",
                             "sample": oracle_sample_text(wl, mod, rows) + " per step"},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
DATA = ("synthetic: seeded N(0, sigma) fp32 weights (0.1% x10 outliers where the workload has them), "
        "N(0, 1) bf16 activations and output gradients, random-init bf16 adapters")


def parallelism(wl, gpus):
    if gpus <= 1:
        return "dp1"
    if wl.backward == "dx":
        return "dp%d (independent replicas: no exchange step)" % gpus
    return "dp%d (token shards; all-reduce of dA, dB per module)" % gpus


def workload_config(wl, gpus=1):
    """The workload as both arms report it (identical keys and values)."""
    return {"workload": wl.name,
            "modules": [[m.name, m.d_out, m.d_in] for m in wl.modules],
            "tokens": list(wl.tokens), "r": wl.r, "alpha": wl.alpha,
            "passes": "fwd+dX" if wl.backward == "dx" else "fwd+bwd(dX,dA,dB)",
            "weights": "NF4 blocksize 64 + double-quantised scales (8-bit, blocks of 256)",
            "l2_flush": "encoded weights rotate over copies totalling at least 4x L2, so every pass reads "
                        "its weight from HBM",
            "parallelism": parallelism(wl, gpus)}


class GpuWorkload:
    def __init__(self, nf, wl, device, copies, keep_fp32=False):
        self.nf, self.wl, self.device = nf, wl, device
        self.mods = []
        self.fp32 = []  # the fp32 weights, kept where the workload times their encoding
        for i, mod in enumerate(wl.modules):
            W = torch.from_numpy(workloads.weight(mod.d_out, mod.d_in, wl.sigma, wl.outliers, i)).to(device)
            enc = nf.nf4_quantize(W)
            if wl.quantize_timed or keep_fp32:
                self.fp32.append(W)
            del W
            encs = [enc] + [nf.NF4Tensor(mod.d_out, mod.d_in, device, buffer=enc.buffer.clone())
                            for _ in range(copies - 1)]
            x_seed = workloads.x_seed(mod.d_in, wl.modules[0].d_in)
            mmax = max(wl.tokens)
            d = {"encs": encs, "A": workloads.lora_a(wl.r, mod.d_in, i).to(device),
                 "B": workloads.lora_b(mod.d_out, wl.r, i).to(device),
                 "X": workloads.activations(mmax, mod.d_in, x_seed).to(device),
                 "dY": workloads.grad_output(mmax, mod.d_out, i).to(device)}
            d["Y"] = {m: torch.empty((m, mod.d_out), dtype=torch.bfloat16, device=device) for m in wl.tokens}
            d["T"] = {m: torch.empty((m, wl.r), dtype=torch.float32, device=device) for m in wl.tokens}
            d["dX"] = {m: torch.empty((m, mod.d_in), dtype=torch.bfloat16, device=device) for m in wl.tokens}
            d["dA"] = torch.zeros((wl.r, mod.d_in), dtype=torch.bfloat16, device=device)
            d["dB"] = torch.zeros((mod.d_out, wl.r), dtype=torch.bfloat16, device=device)
            self.mods.append(d)
        ws = 0
        for mod in wl.modules:
            for m in wl.tokens:
                ws = max(ws, nf.qlora_fwd_workspace_bytes(m, mod.d_out, mod.d_in, wl.r),
                         nf.qlora_bwd_workspace_bytes(m, mod.d_out, mod.d_in, wl.r))
        self.ws = torch.empty(ws, dtype=torch.uint8, device=device)
        self.plan = step_plan(wl)
        self.sms = torch.cuda.get_device_properties(device).multi_processor_count

    def step(self, copy_base, X=None, dY=None, outs=None, after_pass=None):
        """Enqueue one step; pass p uses encoded copy (copy_base + p);
        after_pass(p), if given, runs after each pass is enqueued."""
        for p in range(len(self.plan)):
            self.step_pass(copy_base, p, X, dY, outs)
            if after_pass is not None:
                after_pass(p)

    def step_pass(self, copy_base, p, X=None, dY=None, outs=None):
        nf, wl = self.nf, self.wl
        i, mod, m, kind = self.plan[p]
        d = self.mods[i]
        enc = d["encs"][(copy_base + p) % len(d["encs"])]
        x = (X[i] if X is not None else d["X"])[:m]
        if kind == "fwd":
            # a full backward follows: the forward keeps T = s X A^T (fp32) for it,
            # as a training step does; a dX-only backward needs no T
            keep = wl.backward != "dx"
            nf.qlora_linear_fwd(enc, d["A"], d["B"], wl.scaling, x, save_t=keep,
                                Y=(outs[i]["Y"][m] if outs else d["Y"][m]), workspace=self.ws,
                                T=d["T"][m])
        else:
            dy = (dY[i] if dY is not None else d["dY"])[:m]
            if kind == "dx":
                nf.qlora_linear_bwd(enc, d["A"], d["B"], wl.scaling, None, None, dy, need_da=False,
                                    need_db=False, dX=(outs[i]["dX"][m] if outs else d["dX"][m]),
                                    workspace=self.ws)
            else:
                nf.qlora_linear_bwd(enc, d["A"], d["B"], wl.scaling, x, d["T"][m], dy, dA=d["dA"], dB=d["dB"],
                                    dX=(outs[i]["dX"][m] if outs else d["dX"][m]), workspace=self.ws)


def dominant_kernel_stats(records, names):
    per = {}
    for name, ms in records:
        per.setdefault(name, []).append(ms)
    stats = {k: (len(v), sum(v)) for k, v in per.items()}
    dom = max((k for k in stats if k in names), key=lambda k: stats[k][1], default=None)
    return dom, stats


def quantize_bytes(d_out, d_in):
    """Algorithmic bytes of one encoding: the fp32 weight read once, the
    packed codes, int8 scale codes, fp32 group scales and mean written once."""
    n = d_out * d_in
    nb = n // 64
    return 4 * n + n // 2 + nb + 4 * ((nb + 255) // 256) + 4


def time_forward(nf, gw, args, stream, device, world):
    """The forward passes of the step plan on their own, eager: W warm-up
    passes, then K passes timed together (a short command whose kernels are
    the step's forwards, to profile)."""
    fwd = [p for p, (_, _, _, kind) in enumerate(gw.plan) if kind == "fwd"]

    def one_pass():
        with torch.cuda.stream(stream):
            for p in fwd:
                gw.step_pass(0, p)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        one_pass()
    stop.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(stop)
    if world > 1:
        from nf4_base_lora_b200 import dp
        ms = dp.max_over_ranks(ms, device)
    flops = sum(pass_flops(mod.d_out, mod.d_in, m, gw.wl.r, "fwd") for _, mod, m, kind in gw.plan if kind == "fwd")
    ms_pass = ms / args.steps
    return {"ms_per_pass": ms_pass, "passes": args.steps, "launches_per_pass": len(fwd),
            "value": world * flops / (ms_pass * 1e-3) / 1e12, "unit": "TFLOP/s"}


def time_quantize(nf, gw, args, stream, device, world, peaks):
    """Encoding of every module's fp32 weight through nf4_quantize, timed on
    its own: K passes over all modules after W warm-up passes (the fp32
    weights total more than 4x L2, so every pass reads them from HBM)."""
    wl = gw.wl
    outs = [nf.NF4Tensor(m.d_out, m.d_in, device) for m in wl.modules]
    ws = torch.empty(max(nf.nf4_quantize_workspace_bytes(m.d_out, m.d_in) for m in wl.modules),
                     dtype=torch.uint8, device=device)
    per_pass = sum(quantize_bytes(m.d_out, m.d_in) for m in wl.modules)
    weights = sum(m.d_out * m.d_in for m in wl.modules)

    def one_pass():
        with torch.cuda.stream(stream):
            for W, enc in zip(gw.fp32, outs):
                nf.nf4_quantize(W, out=enc, workspace=ws)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    passes = max(3, min(args.steps, 50))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(passes):
        one_pass()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / passes
    if world > 1:
        from nf4_base_lora_b200 import dp
        ms = dp.max_over_ranks(ms, device)
    # the encode kernel's own device time (library tracing, one more pass)
    nf.trace_start(16 * len(wl.modules) + 64)
    one_pass()
    torch.cuda.synchronize()
    records = nf.trace_records()
    nf.trace_stop()
    per_kernel = {}
    for name, kms in records:
        per_kernel.setdefault(name, []).append(kms)
    enc_ms = sum(per_kernel.get("nf4_encode", [0.0]))
    enc_bytes = sum(4 * m.d_out * m.d_in + m.d_out * m.d_in // 2 for m in wl.modules)
    value = world * per_pass / (ms * 1e-3) / 1e9
    out = {"ms_per_pass": ms, "passes": passes, "value": value, "unit": "GB/s",
           "weights_per_pass": weights, "bytes_per_pass": per_pass,
           "algorithmic": "per module 4n + n/2 + n/64 + 4*ceil(n/16384) + 4 bytes (n weights)",
           "frac": value / world / peaks["hbm"],
           "kernels": {k: {"launches": len(v), "avg_us": sum(v) / len(v) * 1e3} for k, v in sorted(per_kernel.items())}}
    if enc_ms > 0:
        achieved = enc_bytes / (enc_ms * 1e-3) / 1e9
        bpw = load_traffic_per_weight("nf4_encode")
        out["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                           "frac": achieved / peaks["hbm"], "kernel": "nf4_encode",
                           "traffic": None if bpw is None else bpw * weights / len(wl.modules),
                           "algorithmic": "4n read + n/2 written per launch (fp32 weight in, packed codes out)",
                           "peak_source": peaks["source"] + " (hbm_gbs)"}
    return out


def time_adamw(nf, gw, args, stream, device, world, peaks, l2):
    """The step after the backward: one lora_adamw_step over every module's A
    and B (fp32 master, bf16 copy, bf16 gradient from the backward, fp32
    moments), timed on its own.  The optimizer state rotates over enough
    copies to exceed 4x L2, as it would be cold after the layer's GEMMs."""
    grads = [t for d in gw.mods for t in (d["dA"], d["dB"])]
    n_total = sum(g.numel() for g in grads)
    per_copy = 26 * n_total  # fp32 master, m, v + bf16 copy and gradient
    copies = max(1, int(math.ceil(4 * l2 / per_copy)))
    states = []
    for _ in range(copies):
        st = []
        for g, src in zip(grads, [t for d in gw.mods for t in (d["A"], d["B"])]):
            st.append((src.float().reshape(-1).contiguous(), torch.empty_like(src).reshape(-1),
                       g.reshape(-1), torch.zeros(g.numel(), dtype=torch.float32, device=device),
                       torch.zeros(g.numel(), dtype=torch.float32, device=device)))
        states.append(st)

    def one_pass(k, t):
        with torch.cuda.stream(stream):
            nf.lora_adamw_step(states[k % copies], lr=2e-4, beta1=0.9, beta2=0.999, eps=1e-8,
                               weight_decay=0.0, step=t)

    for k in range(max(args.warmup, copies)):
        one_pass(k, k + 1)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    passes = max(3, min(args.steps, 50))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for k in range(passes):
        one_pass(k, 100 + k)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / passes
    if world > 1:
        from nf4_base_lora_b200 import dp
        ms = dp.max_over_ranks(ms, device)
    nf.trace_start(64)
    one_pass(0, 200)
    torch.cuda.synchronize()
    recs = nf.trace_records()
    nf.trace_stop()
    k_ms = [r[1] for r in recs if r[0] == "lora_adamw"]
    step_bytes = 28 * n_total
    value = world * step_bytes / (ms * 1e-3) / 1e9
    out = {"ms_per_pass": ms, "passes": passes, "params": n_total, "bytes_per_pass": step_bytes,
           "value": value, "unit": "GB/s", "frac": value / world / peaks["hbm"],
           "algorithmic": "28 bytes per parameter: fp32 master, m, v read and written, bf16 gradient read, "
                          "bf16 copy written",
           "l2_flush": "rotating %d optimizer-state copies (%.0f MB)" % (copies, copies * per_copy / 1e6),
           "peak_source": peaks["source"] + " (hbm_gbs)"}
    if k_ms:
        out["kernels"] = {"lora_adamw": {"launches": len(k_ms), "avg_us": sum(k_ms) / len(k_ms) * 1e3}}
    return out


FP64_FMA_PER_CLK_PER_SM = 64  # B200: 148 SMs x 64 x 2 x 1.965 GHz = 37.2 TFLOP/s fp64, the published figure


def time_merge(nf, gw, args, stream, device, world, clocks_mhz=1965.0):
    """Deployment: the adapter folded into each module's base and the result
    encoded again (nf4_merge_requantize), timed on its own over all modules.
    The merge kernel is bound by its fp64 multiply-adds (n r per module);
    its roofline is the fp64 FMA rate of the SMs at the maximum SM clock."""
    wl = gw.wl
    outs = [nf.NF4Tensor(m.d_out, m.d_in, device) for m in wl.modules]
    ws = torch.empty(max(nf.nf4_merge_workspace_bytes(m.d_out, m.d_in) for m in wl.modules),
                     dtype=torch.uint8, device=device)

    def one_pass():
        with torch.cuda.stream(stream):
            for d, out in zip(gw.mods, outs):
                nf.nf4_merge_requantize(d["encs"][0], d["A"], d["B"], wl.scaling, out=out, workspace=ws)

    for _ in range(args.warmup):
        one_pass()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    passes = max(3, min(args.steps, 20))
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(passes):
        one_pass()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / passes
    if world > 1:
        from nf4_base_lora_b200 import dp
        ms = dp.max_over_ranks(ms, device)
    nf.trace_start(16 * len(wl.modules) + 64)
    one_pass()
    torch.cuda.synchronize()
    per_kernel = {}
    for name, kms in nf.trace_records():
        per_kernel.setdefault(name, []).append(kms)
    nf.trace_stop()
    weights = sum(m.d_out * m.d_in for m in wl.modules)
    flops = 2.0 * weights * wl.r
    peak = gw.sms * FP64_FMA_PER_CLK_PER_SM * 2 * clocks_mhz * 1e6 / 1e12
    out = {"ms_per_pass": ms, "passes": passes, "weights_per_pass": weights,
           "kernels": {k: {"launches": len(v), "avg_us": sum(v) / len(v) * 1e3} for k, v in sorted(per_kernel.items())}}
    mk = per_kernel.get("nf4_merge_lora")
    if mk:
        achieved = flops / (sum(mk) * 1e-3) / 1e12
        bpw = load_traffic_per_weight("nf4_merge_lora")
        out["roofline"] = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s (fp64)",
                           "frac": achieved / peak, "kernel": "nf4_merge_lora",
                           "traffic": None if bpw is None else bpw * weights / len(wl.modules),
                           "algorithmic": "2 n r fp64 flops per module (the rank-r sum of each merged weight)",
                           "peak_source": "derived: %d SMs x %d fp64 FMA/clk x 2 x %.0f MHz"
                                          % (gw.sms, FP64_FMA_PER_CLK_PER_SM, clocks_mhz)}
    return out


def time_workload(nf, wl, args, stream, device, world, peaks, l2, with_e2e):
    """Time K steps of one workload (replayed from CUDA graphs captured
    without tracing), then one traced pass of the same steps for the
    per-kernel device times.  Returns the numbers and the GpuWorkload."""
    plan = step_plan(wl)
    wbytes = sum(weight_bytes(mod.d_out, mod.d_in) for mod in wl.modules)
    # enough encoded copies that consecutive passes of one module never share L2
    copies = 1
    if wbytes < 4 * l2:
        copies = int(math.ceil(4 * l2 / wbytes)) + len(plan)
        copies = int(math.ceil(copies / len(plan))) * len(plan)
    gw = GpuWorkload(nf, wl, device, copies)
    cycle = max(1, copies // len(plan)) if copies > 1 else 1
    step_bytes, step_flops = step_totals(wl)

    # data-parallel exchange of the adapter gradients (full backward, N > 1):
    # module i's dA, dB are all-reduced on a side stream as soon as its last
    # backward pass of the step is enqueued, overlapping the later passes
    exchange = None
    if (world > 1 or getattr(args, "force_exchange", False)) and wl.backward != "dx":
        from nf4_base_lora_b200 import dp
        exchange = dp.OverlappedGradExchange([[d["dA"], d["dB"]] for d in gw.mods])
    exchange_after = exchange_points(plan)

    def after_pass(p):
        if exchange is not None and p in exchange_after:
            exchange.launch(exchange_after[p])

    def enqueue(s_index, **kw):
        gw.step((s_index % cycle) * len(plan), after_pass=after_pass, **kw)
        if exchange is not None:
            exchange.finish()

    # eager warm-up step, traced only to count the library's launches per step
    nf.trace_start(len(plan) * 16 + 64)
    with torch.cuda.stream(stream):
        gw.step(0)
    torch.cuda.synchronize()
    launches_per_step = nf.trace_count()
    nf.trace_stop()

    # one graph per step, or with an exchange one per pass (the collectives
    # run eagerly on their side stream between the replays)
    graphs = []
    if not args.no_graph:
        for g in range(cycle):
            if exchange is None:
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    gw.step(g * len(plan))
                graphs.append([graph])
            else:
                per_pass = []
                for p in range(len(plan)):
                    graph = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(graph, stream=stream):
                        gw.step_pass(g * len(plan), p)
                    per_pass.append(graph)
                graphs.append(per_pass)

    def run_steps(k, base):
        with torch.cuda.stream(stream):
            for i in range(k):
                if graphs:
                    for p, graph in enumerate(graphs[(base + i) % cycle]):
                        graph.replay()
                        if exchange is not None:
                            after_pass(p)
                    if exchange is not None:
                        exchange.finish()
                else:
                    enqueue(base + i)

    run_steps(args.warmup, 0)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.3)
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    start.record(stream)
    run_steps(args.steps, args.warmup)
    stop.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    ms = start.elapsed_time(stop)
    if world > 1:
        from nf4_base_lora_b200 import dp
        ms = dp.max_over_ranks(ms, device)
    ms_per_step = ms / args.steps
    gbps = world * step_bytes / (ms_per_step * 1e-3) / 1e9
    tflops = world * step_flops / (ms_per_step * 1e-3) / 1e12

    # per-kernel device times: a separate pass of the same steps with the
    # library's launch tracing on (an event pair around each launch).  With
    # graphs, the traced steps are captured too (the events become
    # event-record nodes) and replayed, so no host launch latency falls
    # between a pair; otherwise the traced steps run eagerly.
    if graphs and exchange is None:
        nf.trace_start(int(launches_per_step) * cycle + 64)
        traced = []
        for g in range(cycle):
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                gw.step(g * len(plan))
            traced.append(graph)
        with torch.cuda.stream(stream):
            for _ in range(2):  # the records hold the second replay's times
                for graph in traced:
                    graph.replay()
        torch.cuda.synchronize()
        records = nf.trace_records()
        nf.trace_stop()
        del traced
        timing_source = ("traced graph replay of %d steps right after the timed region (an event-record node "
                         "before and after each launch)" % cycle)
    else:
        k_eager = max(cycle, min(args.steps, 50))
        nf.trace_start(int(launches_per_step) * k_eager + 64)
        with torch.cuda.stream(stream):
            for i in range(k_eager):
                enqueue(args.warmup + i)
        torch.cuda.synchronize()
        records = nf.trace_records()
        nf.trace_stop()
        timing_source = "traced eager pass of %d steps right after the timed region" % k_eager
    hbm = not tensor_bound(wl)
    names = ("nf4_gemm_fwd_few", "nf4_gemm_dx_few") if hbm else ("nf4_gemm_fwd", "nf4_gemm_dx")
    dom, kstats = dominant_kernel_stats(records, names)
    roofline = None
    if dom is not None:
        n_launch, tot_ms = kstats[dom]
        avg_ms = tot_ms / n_launch
        # the algorithmic work of the dominant kernel's launches in one step
        launches = [(mod, m) for _, mod, m, kind in plan
                    if (kind == "fwd") == dom.startswith("nf4_gemm_fwd")]
        if hbm:
            per_launch = sum(weight_bytes(mod.d_out, mod.d_in) for mod, _ in launches) / len(launches)
            achieved = per_launch / (avg_ms * 1e-3) / 1e9
            roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm"], "unit": "GB/s",
                        "frac": achieved / peaks["hbm"], "traffic": load_traffic(dom, wl.name),
                        "kernel": dom, "launches_timed": n_launch, "avg_us": avg_ms * 1e3,
                        "timing": timing_source,
                        "algorithmic": "NF4 weight stream, K*N*(0.5 + 1/64 + 4/16384) bytes per launch",
                        "peak_source": peaks["source"] + " (hbm_gbs, copy bandwidth)"}
        else:
            per_launch = sum(kernel_flops(mod.d_out, mod.d_in, m, wl.r, dom) for mod, m in launches) / len(launches)
            achieved = per_launch / (avg_ms * 1e-3) / 1e12
            roofline = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"], "unit": "TFLOP/s",
                        "frac": achieved / peaks["bf16"], "traffic": load_traffic(dom, wl.name),
                        "kernel": dom, "launches_timed": n_launch, "avg_us": avg_ms * 1e3,
                        "timing": timing_source,
                        "algorithmic": ("2*M*K*N + 2*M*r*N flops per launch (base product + LoRA up)"
                                        if dom == "nf4_gemm_fwd" else
                                        "2*M*K*N + 2*M*r*K flops per launch (base product + V A)"),
                        "peak_source": peaks["source"] + " (bf16_tflops, burst: a kernel timed alone)",
                        "peak_sustained": peaks["bf16_sustained"],
                        "frac_of_sustained": achieved / peaks["bf16_sustained"]}
    kernel_table = {k: {"launches": v[0], "avg_us": v[1] / v[0] * 1e3} for k, v in sorted(kstats.items())}
    out = {"value": tflops if not hbm else gbps, "unit": "TFLOP/s" if not hbm else "GB/s",
           "ms_per_step": ms_per_step, "tflops": tflops, "gbps": gbps, "roofline": roofline, "kernels": kernel_table,
           "launches_per_step": launches_per_step, "copies": copies, "graphs": bool(graphs), "clocks": clocks,
           "exchange": exchange is not None, "config": workload_config(wl, world)}
    # weight GB/s: each step passes over every module's encoded weight once per pass of the plan
    out["weight_gbps"] = world * sum(weight_bytes(mod.d_out, mod.d_in) for _, mod, _, _ in plan) / (
        ms_per_step * 1e-3) / 1e9

    if with_e2e:
        out["e2e"] = time_e2e(gw, wl, args, stream, device, world, cycle, plan, exchange, after_pass, step_bytes,
                              step_flops)
    graphs.clear()
    return out, gw


def time_e2e(gw, wl, args, stream, device, world, cycle, plan, exchange, after_pass, step_bytes, step_flops):
    """The same step end to end through the public API: pinned host inputs
    copied to the device, the layer calls, the outputs copied back, every
    step inside the timed region."""
    e2e_steps = max(3, min(args.steps, 200))
    hostX = [torch.empty_like(d["X"], device="cpu").pin_memory() for d in gw.mods]
    hostdY = [torch.empty_like(d["dY"], device="cpu").pin_memory() for d in gw.mods]
    for i, d in enumerate(gw.mods):
        hostX[i].copy_(d["X"])
        hostdY[i].copy_(d["dY"])
    devX = [torch.empty_like(d["X"]) for d in gw.mods]
    devdY = [torch.empty_like(d["dY"]) for d in gw.mods]
    outs = [{"Y": {m: torch.empty_like(d["Y"][m]) for m in wl.tokens},
             "dX": {m: torch.empty_like(d["dX"][m]) for m in wl.tokens}} for d in gw.mods]
    hostY = [{m: torch.empty_like(o["Y"][m], device="cpu").pin_memory() for m in wl.tokens} for o in outs]
    hostdX = [{m: torch.empty_like(o["dX"][m], device="cpu").pin_memory() for m in wl.tokens} for o in outs]
    h2d = sum(t.numel() * t.element_size() for t in hostX + hostdY)
    d2h = sum(t.numel() * t.element_size() for hy in hostY + hostdX for t in hy.values())

    def e2e_step(s):
        with torch.cuda.stream(stream):
            for i in range(len(gw.mods)):
                devX[i].copy_(hostX[i], non_blocking=True)
                devdY[i].copy_(hostdY[i], non_blocking=True)
            gw.step((s % cycle) * len(plan), X=devX, dY=devdY, outs=outs, after_pass=after_pass)
            if exchange is not None:
                exchange.finish()
            for i in range(len(gw.mods)):
                for m in wl.tokens:
                    hostY[i][m].copy_(outs[i]["Y"][m], non_blocking=True)
                    hostdX[i][m].copy_(outs[i]["dX"][m], non_blocking=True)

    for s in range(3):
        e2e_step(s)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(e2e_steps):
        e2e_step(s)
    e1.record(stream)
    torch.cuda.synchronize()
    ems = e0.elapsed_time(e1)
    if world > 1:
        from nf4_base_lora_b200 import dp
        ems = dp.max_over_ranks(ems, device)
    sec = ems / e2e_steps * 1e-3
    value = world * (step_flops / sec / 1e12 if tensor_bound(wl) else step_bytes / sec / 1e9)
    return {"value": value, "unit": "TFLOP/s" if tensor_bound(wl) else "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": ems / e2e_steps}


FEW_TOKEN_WORKLOAD = "q_proj4096_r64_m1-4-16"


def run_ours(args, wl):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1 or getattr(args, "force_exchange", False):
        import datetime
        if world == 1:
            # a group of one rank, so that --force-exchange runs the collective path
            import socket
            with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sk:
                sk.bind(("127.0.0.1", 0))
                os.environ.setdefault("MASTER_PORT", str(sk.getsockname()[1]))
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            os.environ.setdefault("RANK", "0")
            os.environ.setdefault("WORLD_SIZE", "1")
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    import nf4_base_lora_b200 as nf
    peaks = load_peaks()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    stream = torch.cuda.Stream(device)
    if args.only:
        # one phase of the workload on its own (a short command to profile):
        # the encoding, the merge + re-encoding or the optimizer step
        gw = GpuWorkload(nf, wl, device, 1, keep_fp32=args.only == "quantize")
        if args.only == "quantize":
            obj = time_quantize(nf, gw, args, stream, device, world, peaks)
        elif args.only == "forward":
            obj = time_forward(nf, gw, args, stream, device, world)
        elif args.only == "merge":
            obj = time_merge(nf, gw, args, stream, device, world)
        else:
            with torch.cuda.stream(stream):
                gw.step(0)  # the backward fills dA, dB
            obj = time_adamw(nf, gw, args, stream, device, world, peaks, l2)
        if dist.is_initialized():
            dist.barrier()
            dist.destroy_process_group()
        if rank == 0:
            print(json.dumps({"metric": METRIC, "phase": args.only, "n_gpus": world,
                              "config": workload_config(wl, world), args.only: obj}), flush=True)
        return

    head, gw = time_workload(nf, wl, args, stream, device, world, peaks, l2, with_e2e=True)
    quantize = time_quantize(nf, gw, args, stream, device, world, peaks) if gw.fp32 else None
    optimizer = time_adamw(nf, gw, args, stream, device, world, peaks, l2) if wl.backward != "dx" else None
    merge = time_merge(nf, gw, args, stream, device, world) if wl.quantize_timed and not args.no_merge else None
    del gw
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    few = None
    if tensor_bound(wl) and not args.no_few:
        fwl = workloads.WORKLOADS[FEW_TOKEN_WORKLOAD]
        fobj, fgw = time_workload(nf, fwl, args, stream, device, world, peaks, l2, with_e2e=False)
        del fgw
        few = {k: fobj[k] for k in ("value", "unit", "ms_per_step", "roofline", "kernels", "launches_per_step",
                                    "clocks", "config")}
        few["steps"] = args.steps

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = time_oracle(wl, budget_s=args.cpu_budget)
        cpu_baseline = {k: cb[k] for k in ("value", "unit", "cores", "kind", "sample")}

    if dist.is_initialized():
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {"metric": METRIC, "value": head["value"], "unit": head["unit"], "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": DATA, "config": head["config"],
            "roofline": head["roofline"], "cpu_baseline": cpu_baseline, "e2e": head["e2e"],
            "gpu_launches": int(head["launches_per_step"] * args.steps),
            "clocks": head["clocks"],
            "tflops": head["tflops"], "weight_gbps": head["weight_gbps"],
            "graphs": head["graphs"], "weight_copies": head["copies"],
            "kernels": head["kernels"]}
    if quantize is not None:
        line["quantize"] = quantize
    if few is not None:
        line["few_token"] = few
    if optimizer is not None:
        line["optimizer"] = optimizer
    if merge is not None:
        line["merge"] = merge
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default="llama65b_layer_r64_m2048", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--force-exchange", action="store_true",
                    help="run the data-parallel gradient exchange even on one rank (a process group of one)")
    ap.add_argument("--no-few", action="store_true", help="skip the few-token sub-object")
    ap.add_argument("--no-merge", action="store_true", help="skip the merge + re-encoding phase")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--only", choices=("quantize", "merge", "optimizer", "forward"),
                    help="time one phase of the workload alone (encoding, merge + re-encoding, optimizer step, "
                         "the forward passes)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    wl = workloads.WORKLOADS[args.workload]
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
