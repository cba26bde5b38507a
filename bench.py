#!/usr/bin/env python
"""Benchmark of the fused linear-recurrence scan: forward + backward tokens/s and the achieved
fraction of the HBM roofline, per scan kind, on B200.

One step = one forward and one backward pass over one batch of the workload (every step of the
hot path: gate formation / discretisation, scan, carries, readout, checkpoints, recompute,
adjoint scan and gradients).  The headline line reports the mamba-370m-like SSD workload (or the
first built workload in BENCH_ORDER if that kind is not built); ``per_kind`` carries the same
measurement for every built workload.  Inputs are seeded synthetic tensors resident in HBM.

Timing: W untimed warm-up steps, then exactly K steps timed with CUDA events on the launching
stream; between timed steps a 256 MiB buffer is written to flush L2 (outside the events).  For
N > 1 processes (one per GPU, torchrun), every rank runs its own batch (weak scaling), the f32
parameter gradients are summed across ranks with NCCL inside the step, and the time is the max
over ranks.

``--impl reference`` times the fp64 CPU oracle (the only other implementation of this path) on
rank 0 over bounded samples of the same workload.
"""
import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd scan tokens/s & achieved HBM GB/s (% of B200 peak) per scan kind"
BENCH_ORDER = ["ssd", "rglru", "gla", "s6_zoh", "s6_bilinear", "rotlru", "ssd_mamba2", "rglru_gated",
               "ssd_bilinear"]
NAMES = {
    "ssd": "Mamba-2 SSD scan (mamba-370m-like), bf16, B=2 H=32 P=64 N=128 L=4096, chunk 128, S=128, ZOH",
    "rglru": "rglru_scan, f32, B=1 D=256 L=1024, S=128",
    "gla": "GLA scan, bf16, B=4 H=16 K=V=128 L=2048, chunk 128, S=128",
    "s6_zoh": "Mamba-1 S6 selective scan, bf16, B=8 D=2048 N=16 L=2048, S=64, ZOH, D skip + silu(z)",
    "s6_bilinear": "Mamba-1 S6 selective scan, bf16, B=8 D=2048 N=16 L=2048, S=64, bilinear, D skip + silu(z)",
    "rotlru": "rotlru_scan, f32, B=16 D=4096 L=16384, S=256",
    "ssd_mamba2": "SSD scan, Mamba-2 step length: dt = softplus(delta + bias) in-kernel, ZOH-Euler (beta = dt), "
                  "bf16, B=2 H=32 P=64 N=128 L=4096, chunk 128, S=128",
    "rglru_gated": "rglru_scan with the RG-LRU gates in-kernel (a = sigmoid(Lambda)^(8 r), b = sqrt(1 - a^2) i x), "
                   "f32, B=1 D=256 L=1024, S=128",
    "ssd_bilinear": "SSD scan, bilinear (Tustin) discretisation with signed decays, bf16, B=2 H=32 P=64 N=128 "
                    "L=4096, chunk 128, S=128",
}
INPUT_NAMES = {
    "rglru": ["a", "b", "x", "A"], "rotlru": ["b", "g", "mag", "theta"],
    "s6": ["x", "delta", "A", "Bm", "Cm", "Dskip", "z", "delta_bias"],
    "ssd": ["x", "delta", "A", "Bm", "Cm", "Dskip", "z", "delta_bias"],
    "gla": ["q", "k", "v", "g"],
}
FALLBACK_HBM = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# Sources each kernel family is built from (its own file and the headers it includes): a committed
# ncu figure stays valid while these are unchanged.
KERNEL_SOURCES = {
    "ssd": ("ssd.cu", "chunk_scan.cuh", "chunk_common.cuh", "common.cuh", "tc.cuh", "host_common.h"),
    "gla": ("gla.cu", "chunk_scan.cuh", "chunk_common.cuh", "common.cuh", "tc.cuh", "host_common.h"),
    "s6": ("s6.cu", "common.cuh", "host_common.h"),
    "rglru": ("diag.cu", "common.cuh", "host_common.h"),
    "rotlru": ("diag.cu", "common.cuh", "host_common.h"),
}


def src_sha(kernel=None):
    """Hash of the kernel family's sources (of every source when `kernel` is None)."""
    h = hashlib.sha1()
    cdir = os.path.join(ROOT, "selective_state_space_09_b200", "csrc")
    fam = kernel.split("_")[0] if kernel else None
    names = KERNEL_SOURCES.get(fam) or sorted(os.listdir(cdir))
    for n in names:
        with open(os.path.join(cdir, n), "rb") as f:
            h.update(n.encode() + f.read())
    return h.hexdigest()[:12]


def ncu_traffic(kernel, pas=None):
    """DRAM bytes per launch of `kernel` (of pass `pas` when the name occurs in both passes) from
    the committed ncu summary, if it was taken on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get("%s@%s" % (kernel, pas)) or d.get(kernel)
    if not e or e.get("src_sha") != src_sha(kernel):
        return None
    return e.get("bytes_per_launch")


# ------------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id, period_ms=20):
        self.gpu_id, self.period_ms = gpu_id, period_ms
        self.samples, self.proc, self.thread = [], None, None
        self.windows = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_id), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for ts, line in self.samples:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((ts, float(parts[1]), float(parts[2]), parts))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        inwin = [r for r in rows if any(a - 0.05 <= r[0] <= b + 0.05 for a, b in self.windows)]
        use = inwin or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in use:
            for i, n in enumerate(names):
                if r[3][5 + i].lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": sorted(reasons), "samples": len(use), "in_window": bool(inwin)}


# ------------------------------------------------------------------------------ workloads
BATCH_OVERRIDE = None  # --batch: a smaller batch of the same workload (profiling captures)


def workload_inputs(name, device, seed):
    from selective_state_space_09_b200 import inputs
    w = dict(inputs.WORKLOADS[name])
    if BATCH_OVERRIDE:
        w["B"] = BATCH_OVERRIDE
        inp = inputs.workload(name, seed=seed, device=device, B=BATCH_OVERRIDE)
    else:
        inp = inputs.workload(name, seed=seed, device=device)
    return w, inp


def api_inputs(kind, inp):
    return {k: inp[k] for k in INPUT_NAMES[kind] if inp.get(k) is not None}


def nbytes(t):
    return t.numel() * t.element_size()


def operand_bytes(kind, inp, y, grads, dy, ckpt_bytes):
    """Bytes of every operand of one step (each tensor once): the inputs, the output, the upstream
    gradient, every gradient, and the f32 checkpoint states at the configured segment length
    (written by the forward pass, read by the backward pass).  Intermediates a kernel creates for
    another kernel (per-chunk state tiles, partial sums) are not operands."""
    ops = {k: nbytes(v) for k, v in api_inputs(kind, inp).items()}
    ops["y"] = nbytes(y)
    ops["dy"] = nbytes(dy)
    ops.update({k: nbytes(v) for k, v in grads.items()})
    ops["ckpt"] = ckpt_bytes
    return ops


def algorithmic_bytes(kind, ops, grad_names):
    """Bytes a pass must move at minimum: every input read once and every output written once,
    plus the checkpoints (forward: written; backward: read)."""
    ins = sum(ops[k] for k in INPUT_NAMES[kind] if k in ops)
    fwd = ins + ops["y"] + ops["ckpt"]
    bwd = ins + ops["dy"] + ops["ckpt"] + sum(ops[k] for k in grad_names)
    return fwd, bwd


# Operands each kernel of the chunked kinds reads or writes (names as in operand_bytes); the
# kernels that are a whole pass (diagonal kinds, S6) carry the pass's bytes.
CHUNK_KERNEL_OPERANDS = {
    ("ssd_state_scan", "fwd"): ("x", "Bm", "delta", "ckpt"),
    ("ssd_chunk_out", "fwd"): ("x", "Bm", "Cm", "delta", "Dskip", "z", "y"),
    ("ssd_state_scan", "bwd"): ("Cm", "dy", "delta", "z"),
    ("ssd_chunk_grad", "bwd"): ("x", "Bm", "Cm", "delta", "Dskip", "z", "dy", "ckpt",
                                "dx", "ddelta", "dBm", "dCm", "dz"),
    ("gla_state_scan", "fwd"): ("k", "v", "g", "ckpt"),
    ("gla_chunk_out", "fwd"): ("q", "k", "v", "g", "y"),
    ("gla_state_scan", "bwd"): ("q", "dy", "g"),
    ("gla_chunk_grad", "bwd"): ("q", "k", "v", "g", "dy", "ckpt", "dq", "dk", "dv", "dg"),
}


def chunk_flops(w, name):
    """FLOPs of the method's products in one launch of a chunked kind's kernel (M = C B^T counted
    once per row, chunk and group for SSD)."""
    Q = w.get("chunk") or 128
    nc = -(-w["L"] // Q)
    if w["kind"] == "ssd":
        B, H, P, N, G = w["B"], w["H"], w["P"], w["N"], w.get("G", 1)
        hc = nc * B * H
        if name == "ssd_state_scan":
            return (nc - 1) * B * H * 2 * N * P * Q
        if name == "ssd_chunk_out":
            return hc * (2 * Q * P * Q + 2 * Q * P * N) + nc * B * G * 2 * Q * Q * N
        if name == "ssd_chunk_grad":
            per = 2 * Q * (Q * P + 2 * Q * N + Q * P + 2 * P * N + 2 * N * P)
            return hc * per + nc * B * G * 2 * Q * Q * N
    if w["kind"] == "gla":
        B, H, K, V = w["B"], w["H"], w["K"], w["V"]
        hc = nc * B * H
        prod = 2 * Q * Q * max(K, V)
        if name == "gla_state_scan":
            return (nc - 1) * B * H * 2 * K * V * Q
        if name == "gla_chunk_out":
            return hc * 3 * prod
        if name == "gla_chunk_grad":
            return hc * 9 * prod
    return 0


def kernel_cost(w, name, pas, ops, pass_bytes):
    """Algorithmic bytes and FLOPs of one launch of kernel `name` of a workload's pass: the
    operands the kernel must read and write at minimum (each once) and the products of the method
    it evaluates.  Kernels that are a whole pass carry the pass's bytes; small fixed-order
    reductions and the workspace zeroing are counted as 0 (they are not candidates for the
    dominant kernel)."""
    if name.endswith("param_reduce") or name.endswith("ws_zero"):
        return 0, 0
    key = (name, pas)
    if key in CHUNK_KERNEL_OPERANDS:
        return sum(ops.get(k, 0) for k in CHUNK_KERNEL_OPERANDS[key]), chunk_flops(w, name)
    return pass_bytes, 0


# S6 is bound by plain arithmetic, not memory.  Per (b, t, d, n) element, the method needs at
# least one exponential (or, bilinear, one reciprocal) per pass -- the forward forms abar, the
# backward re-forms it from the checkpoint -- and the fp32 FMA-pipe operations counted below
# (forward: beta, the state update, the readout term; backward: the state recompute, the adjoint
# update and the six gradient terms).  The peak rate of each pipe is measured on the device by
# lr_probe_pipe at the start of the run.
S6_ALU = {"fwd": {"ffma": 5, "mufu": 1}, "bwd": {"ffma": 15, "mufu": 1}}


def kernel_alu(w, name, pas, rates):
    if w["kind"] != "s6" or name.endswith("param_reduce") or not rates:
        return None
    c = S6_ALU[pas]
    elems = w["B"] * w["L"] * w["D"] * w["N"]
    t_mufu = elems * c["mufu"] / rates["ex2_per_s"]
    t_fma = elems * c["ffma"] / rates["ffma_per_s"]
    return {"elements": elems, "pipe": "mufu" if t_mufu >= t_fma else "ffma",
            "peak_elems_per_s": elems / max(t_mufu, t_fma), "ops_per_element": c}


def kernel_table(w, names, ms, pas, ops, pass_bytes, rates):
    rows = []
    for k, (n, t) in enumerate(zip(names, ms)):
        b, f = kernel_cost(w, n, pas, ops, pass_bytes)
        rows.append({"pass": pas, "index": k, "kernel": n, "ms": t, "bytes": b, "flops": f,
                     "alu": kernel_alu(w, n, pas, rates)})
    return rows


def kernel_roofline(row, pk):
    """Roofline entry of one timed kernel: the bound is whichever of its algorithmic bytes at the
    measured copy bandwidth, its FLOPs at the measured bf16 GEMM rate and (S6) its arithmetic at
    the measured pipe rates takes longer.  Chunked kinds also carry their tensor-pipe figure."""
    t_hbm = row["bytes"] / (pk["hbm_gbs"] * 1e9)
    t_tc = row["flops"] / (pk["bf16_tflops"] * 1e12)
    sec = row["ms"] * 1e-3
    alu = row.get("alu")
    out = None
    if alu and alu["elements"] / alu["peak_elems_per_s"] > max(t_hbm, t_tc):
        ach = alu["elements"] / sec / 1e9
        pk_g = alu["peak_elems_per_s"] / 1e9
        out = {"bound": "alu", "achieved": round(ach, 2), "peak": round(pk_g, 2), "unit": "Gelem/s",
               "frac": round(ach / pk_g, 4), "pipe": alu["pipe"], "ops_per_element": alu["ops_per_element"]}
    elif t_tc > t_hbm:
        ach = row["flops"] / sec / 1e12
        out = {"bound": "tensor", "achieved": round(ach, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
               "frac": round(ach / pk["bf16_tflops"], 4)}
    else:
        ach = row["bytes"] / sec / 1e9
        out = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
               "frac": round(ach / pk["hbm_gbs"], 4)}
    if row["flops"]:
        tf = row["flops"] / sec / 1e12
        out["tensor"] = {"achieved_tflops": round(tf, 1), "frac_of_bf16_burst": round(tf / pk["bf16_tflops"], 4),
                         "hbm_frac": round(row["bytes"] / sec / 1e9 / pk["hbm_gbs"], 4)}
    return out


def measure_pipe_rates(device):
    """Rates of the special-function unit (ex2) and the fp32 FMA pipe on this device, from one
    timed launch each of lr_probe_pipe (CUDA events; best of 3)."""
    import torch
    from selective_state_space_09_b200 import lrscan
    sms = torch.cuda.get_device_properties(device).multi_processor_count
    blocks, threads = sms * 8, 256
    out = torch.empty(blocks * threads, dtype=torch.float32, device=device)
    res = {"sms": sms}
    for which, iters in (("ex2", 2048), ("ffma", 8192)):
        best = None
        for _ in range(4):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            n = lrscan.probe_pipe(which, out, blocks, threads, iters)
            e1.record()
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1)
            best = ms if best is None else min(best, ms)
        res[which + "_per_s"] = n / (best * 1e-3)
        res[which + "_per_clk_per_sm_at_max_clock"] = round(res[which + "_per_s"] / (sms * SM_MAX_HZ), 2)
    del out
    return res


SM_MAX_HZ = 1.965e9


def host_ahead(steps=1):
    """A short spin on the GPU (no memory traffic) before a timed step, so that the host has enqueued
    the step's launches (descriptors, tensor maps, ctypes) before the GPU reaches its first event:
    the events then bracket device work only, not host enqueue time."""
    import torch
    torch.cuda._sleep(int(200000 * steps))  # about 0.1 ms per step at the SM clock


def tokens_of(w):
    return w["B"] * w["L"]


def run_workload(name, steps, warmup, device, rank, world, flush_buf, e2e=False, rates=None):
    import torch
    import torch.distributed as dist
    from selective_state_space_09_b200 import dp, lrscan

    torch.cuda.empty_cache()
    torch.cuda.reset_peak_memory_stats(device)
    mem0 = torch.cuda.memory_allocated(device)
    w, inp = workload_inputs(name, device, seed=1000 + rank)
    kind = w["kind"]
    ai = api_inputs(kind, inp)
    plan = lrscan.plan_for(kind, ai, w["segment"], w.get("disc", "none"), w.get("chunk", 0), w.get("softplus", False),
                           w.get("gates", False))
    y, grads = lrscan.alloc_outputs(kind, ai)
    dy = inp["dy"]

    def step():
        plan.fwd(ai, y)
        plan.bwd(ai, dy, grads)
        if world > 1:
            dp.reduce_param_grads(kind, grads)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    plan.fwd(ai, y)
    fwd_launch, fwd_names = lrscan.last_launch_count(), lrscan.last_dispatch()
    plan.bwd(ai, dy, grads)
    bwd_launch, bwd_names = lrscan.last_launch_count(), lrscan.last_dispatch()
    torch.cuda.synchronize()
    st = plan.device_error()
    if st != (0, 0):
        raise RuntimeError("device error %s in %s" % (st, name))

    flush = flush_buf is not None
    fl = flush_buf
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
            torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    # per-kernel start events (the library's timing hook records kev[k] before its k-th launch)
    fnames, bnames = fwd_names.split("+"), bwd_names.split("+")
    kev_f = [[torch.cuda.Event(enable_timing=True) for _ in fnames] for _ in range(steps)]
    kev_b = [[torch.cuda.Event(enable_timing=True) for _ in bnames] for _ in range(steps)]
    for row in kev_f + kev_b:
        for e in row:
            e.record()  # creates the CUDA event
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    for i in range(steps):
        if fl is not None:
            fl.fill_(float(i))
        host_ahead()
        e0, e1, e2 = evs[i]
        e0.record()
        plan.fwd(ai, y)
        e1.record()
        plan.bwd(ai, dy, grads)
        if world > 1:
            dp.reduce_param_grads(kind, grads)
        e2.record()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    t1 = time.time()
    # Per-kernel times: a second timed loop of the same steps with the library's timing hook on
    # (an event recorded between two kernels makes the second wait for the first to finish, so the
    # headline loop above runs without the hook).
    kevs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        if fl is not None:
            fl.fill_(float(i))
        host_ahead()
        lrscan.set_launch_events(kev_f[i])
        plan.fwd(ai, y)
        kevs[i][0].record()
        lrscan.set_launch_events(kev_b[i])
        plan.bwd(ai, dy, grads)
        lrscan.set_launch_events(None)
        kevs[i][1].record()
        if world > 1:
            dp.reduce_param_grads(kind, grads)
    torch.cuda.synchronize()

    # The same steps back to back without the flush (inputs left in L2 by the previous step):
    # reported beside the flushed figure for workloads small enough to stay in L2.
    warm = None
    if flush:
        wev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        host_ahead(steps)
        for i in range(steps):
            wev[i][0].record()
            plan.fwd(ai, y)
            wev[i][1].record()
            plan.bwd(ai, dy, grads)
            if world > 1:
                dp.reduce_param_grads(kind, grads)
            wev[i][2].record()
        torch.cuda.synchronize()
        wf = statistics.mean(a.elapsed_time(b) for a, b, _ in wev)
        wb = statistics.mean(b.elapsed_time(c) for _, b, c in wev)
        warm = {"ms_fwd": round(wf, 5), "ms_bwd": round(wb, 5),
                "tokens_per_s": round(tokens_of(w) * world / ((wf + wb) * 1e-3), 1)}

    # The same steps replayed from a CUDA graph of the two calls (lrscan.StepGraph), one rank: the
    # kernels and their work are the same, the per-launch overhead is paid once per graph.
    graph = None
    if world == 1:
        sg = lrscan.StepGraph(plan, ai, dy, y, grads)
        gev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            if fl is not None:
                fl.fill_(float(i))
            host_ahead()
            gev[i][0].record()
            sg.replay()
            gev[i][1].record()
        torch.cuda.synchronize()
        gms = statistics.mean(a.elapsed_time(b) for a, b in gev)
        graph = {"ms_per_step": round(gms, 5), "tokens_per_s": round(tokens_of(w) / (gms * 1e-3), 1),
                 "l2": "flushed between steps" if flush else "inputs larger than L2"}
        del sg

    def kernel_ms(kev, ends):
        n = len(kev[0])
        return [statistics.mean(kev[s][k].elapsed_time(kev[s][k + 1] if k + 1 < n else ends[s])
                                for s in range(steps)) for k in range(n)]
    kms_f = kernel_ms(kev_f, [k[0] for k in kevs])
    kms_b = kernel_ms(kev_b, [k[1] for k in kevs])
    fwd_ms = [a.elapsed_time(b) for a, b, _ in evs]
    bwd_ms = [b.elapsed_time(c) for _, b, c in evs]
    step_ms = statistics.mean(f + b for f, b in zip(fwd_ms, bwd_ms))
    fwd_mean, bwd_mean = statistics.mean(fwd_ms), statistics.mean(bwd_ms)
    if world > 1:
        kt = torch.tensor(kms_f + kms_b, dtype=torch.float64, device=device)
        dist.all_reduce(kt, op=dist.ReduceOp.MAX)
        kms_f, kms_b = kt.tolist()[:len(kms_f)], kt.tolist()[len(kms_f):]
        t = torch.tensor([step_ms, fwd_mean, bwd_mean], dtype=torch.float64, device=device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        step_ms, fwd_mean, bwd_mean = (float(v) for v in t.tolist())
    ckpt_b = plan.ckpt_view().numel() * 4  # the f32 states at the configured segment length
    ops = operand_bytes(kind, inp, y, grads, dy, ckpt_b)
    fwd_b, bwd_b = algorithmic_bytes(kind, ops, list(grads))
    res = {
        "workload": name, "kind": kind, "desc": NAMES[name],
        "tokens_per_step": tokens_of(w) * world,
        "ms_per_step": step_ms, "ms_fwd": fwd_mean, "ms_bwd": bwd_mean,
        "tokens_per_s": tokens_of(w) * world / (step_ms * 1e-3),
        "fwd_bytes": fwd_b, "bwd_bytes": bwd_b,
        "fwd_gbs": fwd_b / (fwd_mean * 1e-3) / 1e9, "bwd_gbs": bwd_b / (bwd_mean * 1e-3) / 1e9,
        "step_gbs": (fwd_b + bwd_b) / (step_ms * 1e-3) / 1e9,
        "launches_per_step": fwd_launch + bwd_launch,
        "kernels_timed": kernel_table(w, fnames, kms_f, "fwd", ops, fwd_b, rates)
                         + kernel_table(w, bnames, kms_b, "bwd", ops, bwd_b, rates),
        "ckpt_bytes": ckpt_b, "segment": w["segment"],
        "fwd_kernels": fwd_names, "bwd_kernels": bwd_names,
        "window": (t0, t1), "wall_s": t1 - t0,
        "peak_mem_bytes": torch.cuda.max_memory_allocated(device) - mem0,
        "io_dtype": "bf16" if y.dtype == torch.bfloat16 else "f32",
        "l2": "flushed between steps" if flush else "inputs larger than L2",
        "l2_warm": warm,
        "graph": graph,
    }
    if e2e:
        res["e2e"] = run_e2e(plan, kind, ai, dy, y, grads, steps, warmup, world, w)
    if world == 1:
        res["decode"] = run_decode(kind, ai, w)
        if kind in ("rglru", "rotlru", "s6") and not w.get("gates"):
            res["full_state"] = run_full_state(kind, ai, dy, w, plan, steps, flush_buf)
        if kind in ("ssd", "gla") and not w.get("softplus"):
            res["segments"] = run_segments(kind, ai, dy, w, plan, steps, flush_buf)
    return res


def run_segments(kind, ai, dy, w, plan, steps, flush_buf, segments=(256, 512)):
    """The chunked kinds' checkpoint trade-off: the same step with checkpoint segments of several
    chunks (f32 states at segment starts only; the backward rebuilds every chunk's entering state
    from them) beside the default of one chunk per segment, timed the same way.  Also the bytes a
    per-step full-state design would keep (every step's state, f32), for the memory ratio."""
    import torch
    from selective_state_space_09_b200 import lrscan
    out = {"default": {"segment": w["segment"], "checkpoint_bytes": lrscan.ckpt_bytes(plan.desc)}}
    L = w["L"]
    state = plan.ckpt_view()[0].numel() * 4
    out["per_step_state_bytes"] = L * state
    for S in segments:
        desc = lrscan.desc_for(kind, ai, S, w.get("disc", "none"), w.get("chunk", 0))
        sp = lrscan.Plan(desc, ai[lrscan.TOKEN_INPUTS[kind][0]].device)
        y, grads = lrscan.alloc_outputs(kind, ai)
        for _ in range(2):
            sp.fwd(ai, y)
            sp.bwd(ai, dy, grads)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            if flush_buf is not None:
                flush_buf.fill_(float(i))
            host_ahead()
            ev[i][0].record()
            sp.fwd(ai, y)
            ev[i][1].record()
            sp.bwd(ai, dy, grads)
            ev[i][2].record()
        torch.cuda.synchronize()
        st = sp.device_error()
        if st != (0, 0):
            raise RuntimeError("device error %s in the segment-%d run" % (st, S))
        fwd = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
        bwd = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
        out["S%d" % S] = {"segment": S, "ms_fwd": round(fwd, 5), "ms_bwd": round(bwd, 5),
                          "checkpoint_bytes": lrscan.ckpt_bytes(desc),
                          "tokens_per_s": round(tokens_of(w) / ((fwd + bwd) * 1e-3), 1),
                          "kernels": lrscan.last_dispatch()}
        del sp, y, grads
    torch.cuda.empty_cache()
    return out


def run_full_state(kind, ai, dy, w, plan, steps, flush_buf):
    """The same fwd+bwd step in the library's full-state mode (every step's state stored by the
    forward, read by the backward: the design segment checkpoints replace), timed the same way;
    reported beside the default mode's checkpoint bytes and time."""
    import torch
    from selective_state_space_09_b200 import lrscan
    desc = lrscan.desc_for(kind, ai, w["segment"], w.get("disc", "none"), w.get("chunk", 0))
    desc.flags |= lrscan.FULL_STATE
    fp = lrscan.Plan(desc, ai[lrscan.TOKEN_INPUTS[kind][0]].device)
    y, grads = lrscan.alloc_outputs(kind, ai)
    fl = flush_buf
    for _ in range(2):
        fp.fwd(ai, y)
        fp.bwd(ai, dy, grads)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        if fl is not None:
            fl.fill_(float(i))
        host_ahead()
        ev[i][0].record()
        fp.fwd(ai, y)
        ev[i][1].record()
        fp.bwd(ai, dy, grads)
        ev[i][2].record()
    torch.cuda.synchronize()
    st = fp.device_error()
    if st != (0, 0):
        raise RuntimeError("device error %s in the full-state run" % (st,))
    fwd = statistics.mean(a.elapsed_time(b) for a, b, _ in ev)
    bwd = statistics.mean(b.elapsed_time(c) for _, b, c in ev)
    ck_full, ck_seg = lrscan.ckpt_bytes(desc), lrscan.ckpt_bytes(plan.desc)
    out = {"ms_fwd": round(fwd, 5), "ms_bwd": round(bwd, 5), "state_bytes": ck_full,
           "checkpoint_bytes": ck_seg, "memory_ratio": round(ck_full / max(ck_seg, 1), 1)}
    del fp
    torch.cuda.empty_cache()
    return out


def run_decode(kind, ai, w, T=256, reps=20):
    """Decode: one token per batch row per step through lr_step, T steps captured in a CUDA graph
    (the first T tokens of the workload, state carried in place), timed over `reps` replays with
    CUDA events.  Outside the fwd+bwd timed region; the state stays in L2, so this measures the
    per-token latency of the step path, not HBM bandwidth."""
    import torch
    from selective_state_space_09_b200 import lrscan
    toks = lrscan.TOKEN_INPUTS[kind]
    seq = {n: (v[:, :T].transpose(0, 1).unsqueeze(2).contiguous() if n in toks and v is not None else v)
           for n, v in ai.items()}
    first = {n: (v[0] if n in toks and v is not None else v) for n, v in seq.items()}
    desc = lrscan.desc_for(kind, first, 1, w.get("disc", "none"), delta_softplus=w.get("softplus", False),
                           gates=w.get("gates", False))
    state = torch.zeros(lrscan.state_shape(desc), dtype=torch.float32, device=ai[toks[0]].device)
    out = ai["v"] if kind == "gla" else (ai["b"] if kind in ("rglru", "rotlru") else ai["x"])
    y = torch.empty((T, out.shape[0], 1) + tuple(out.shape[2:]), dtype=out.dtype, device=out.device)
    graph = lrscan.DecodeGraph(kind, seq, state, y, w.get("disc", "none"), w.get("softplus", False),
                               w.get("gates", False))
    for _ in range(3):
        graph.replay()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    us = ms * 1e3 / (T * reps)
    B = out.shape[0]
    tok_bytes = sum(v[0].numel() * v.element_size() for n, v in seq.items() if n in toks and v is not None)
    step_bytes = 2 * state.numel() * 4 + tok_bytes + y[0].numel() * y.element_size()  # state in and out
    return {"tokens_per_s": B / (us * 1e-6), "us_per_step": round(us, 3), "batch": B, "steps_per_graph": T,
            "state_bytes": state.numel() * 4, "bytes_per_step": step_bytes,
            "achieved_gbs": round(step_bytes / (us * 1e-6) / 1e9, 1),
            "note": "state L2-resident between steps: latency / launch bound",
            "kernel": lrscan.last_dispatch() or kind + "_step"}


def run_e2e(plan, kind, ai, dy, y, grads, steps, warmup, world, w):
    """Same step through the public API from pinned host buffers: every step copies its inputs
    host->device, runs forward and backward, and copies y and all gradients back.  Copies run on
    their own streams with two sets of device (and host) buffers, so that the inputs of step i + 1
    land and the results of step i - 1 leave while step i's kernels run (PCIe in both directions
    beside the GPU work, as a training loop feeding the layer would overlap them)."""
    import torch
    import torch.distributed as dist
    from selective_state_space_09_b200 import dp
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    h_in = {k: v.to("cpu").pin_memory() for k, v in ai.items()}
    h_dy = dy.to("cpu").pin_memory()
    sets = []
    for j in range(2):
        sets.append({
            "in": {k: torch.empty_like(v) for k, v in ai.items()}, "dy": torch.empty_like(dy),
            "y": y if j == 0 else torch.empty_like(y),
            "g": grads if j == 0 else {k: torch.empty_like(v) for k, v in grads.items()},
            "hy": torch.empty(y.shape, dtype=y.dtype).pin_memory(),
            "hg": {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in grads.items()},
            "ev_in": torch.cuda.Event(), "ev_comp": torch.cuda.Event(), "ev_out": torch.cuda.Event(),
            "used": False})

    def step(i):
        S = sets[i % 2]
        with torch.cuda.stream(s_in):
            if S["used"]:
                s_in.wait_event(S["ev_comp"])  # the kernels of two steps ago have read these inputs
            for k in S["in"]:
                S["in"][k].copy_(h_in[k], non_blocking=True)
            S["dy"].copy_(h_dy, non_blocking=True)
            S["ev_in"].record(s_in)
        comp.wait_event(S["ev_in"])
        if S["used"]:
            comp.wait_event(S["ev_out"])  # the results of two steps ago have left
        plan.fwd(S["in"], S["y"])
        plan.bwd(S["in"], S["dy"], S["g"])
        if world > 1:
            dp.reduce_param_grads(kind, S["g"])
        S["ev_comp"].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(S["ev_comp"])
            S["hy"].copy_(S["y"], non_blocking=True)
            for k in S["g"]:
                S["hg"][k].copy_(S["g"][k], non_blocking=True)
            S["ev_out"].record(s_out)
        S["used"] = True

    for i in range(max(1, warmup)):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(comp)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        step(i)
    comp.wait_stream(s_out)  # the last results have left
    e1.record(comp)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=y.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    bi = sum(nbytes(v) for v in h_in.values()) + nbytes(h_dy)
    bo = nbytes(sets[0]["hy"]) + sum(nbytes(v) for v in sets[0]["hg"].values())
    return {"value": tokens_of(w) * world / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": bi, "d2h_bytes_per_step": bo,
            "note": "inputs of step i + 1 and results of step i - 1 cross PCIe while step i runs"}


# ------------------------------------------------------------------------ oracle (CPU)
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(name, units):
    """CPU inputs of a bounded sample of the workload with at least `units` independent units
    (as far as the workload has them), a description, and the fraction of one step's tokens the
    sample represents.  Units are the oracle's parallel loop: (row, head) for SSD and GLA, batch
    rows for S6's backward, pairs for rotlru, channels for rglru."""
    from selective_state_space_09_b200 import inputs
    w = inputs.WORKLOADS[name]
    kind = w["kind"]
    units = max(1, int(units))
    if kind == "rglru":
        return kind, inputs.workload(name, seed=0), 1.0, w, "the whole workload (%d channels)" % w["D"]
    if kind in ("ssd", "gla"):
        H = min(w["H"], units)
        B = min(w["B"], -(-units // H))
        if kind == "ssd":
            inp = inputs.workload(name, seed=0, B=B, H=H)
        else:
            inp = inputs.gla(B, w["L"], H, w["K"], w["V"], seed=0)
        return kind, inp, (B / w["B"]) * (H / w["H"]), w, \
            "batch rows 0-%d, heads 0-%d of %d, full L=%d" % (B - 1, H - 1, w["H"], w["L"])
    if kind == "s6":
        B = min(w["B"], units)
        inp = inputs.s6(B, w["L"], 128, w["N"], seed=0)
        return kind, inp, (B / w["B"]) * (128 / w["D"]), w, \
            "batch rows 0-%d, channels 0-127 of %d, full L=%d" % (B - 1, w["D"], w["L"])
    if kind == "rotlru":
        K = max(32, units)
        inp = inputs.rotlru(1, w["L"], 2 * K, seed=0)
        return kind, inp, (1 / w["B"]) * (2 * K / w["D"]), w, \
            "batch row 0, pairs 0-%d of %d, full L=%d" % (K - 1, w["D"] // 2, w["L"])
    raise KeyError(name)


def oracle_step(kind, inp, w):
    import oracle
    if kind == "rglru" and w.get("gates"):
        oracle.rglru_gated_fwd(inp["a"], inp["b"], inp["x"], inp["A"], S=w["segment"])
        oracle.rglru_gated_bwd(inp["a"], inp["b"], inp["x"], inp["A"], inp["dy"])
    elif kind == "rglru":
        oracle.rglru_fwd(inp["a"], inp["b"], S=w["segment"])
        oracle.rglru_bwd(inp["a"], inp["b"], inp["dy"])
    elif kind == "rotlru":
        oracle.rotlru_fwd(inp["b"], inp["g"], inp["mag"], inp["theta"], S=w["segment"])
        oracle.rotlru_bwd(inp["b"], inp["g"], inp["mag"], inp["theta"], inp["dy"])
    elif kind == "s6":
        a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"])
        oracle.s6_fwd(*a, disc=w["disc"], S=w["segment"])
        oracle.s6_bwd(*a, inp["dy"], disc=w["disc"])
    elif kind == "ssd":
        a = (inp["x"], inp["delta"], inp["A"], inp["Bm"], inp["Cm"], inp["Dskip"], inp["z"])
        sp = dict(delta_softplus=True, delta_bias=inp["delta_bias"]) if w.get("softplus") else {}
        oracle.ssd_fwd(*a, disc=w["disc"], S=w["segment"], **sp)
        oracle.ssd_bwd(*a, inp["dy"], disc=w["disc"], **sp)
    elif kind == "gla":
        oracle.gla_fwd(inp["q"], inp["k"], inp["v"], inp["g"], S=w["segment"])
        oracle.gla_bwd(inp["q"], inp["k"], inp["v"], inp["g"], inp["dy"])


def parallel_units(kind, inp):
    if kind == "rglru":
        return inp["a"].shape[0] * inp["a"].shape[2]
    if kind == "rotlru":
        return inp["b"].shape[2] // 2
    if kind == "s6":
        return inp["x"].shape[0]
    if kind in ("ssd", "gla"):
        t = inp["v" if kind == "gla" else "x"]
        return t.shape[0] * t.shape[2]
    return 1


def time_oracle(name, threads, min_seconds=1.0):
    """The fp64 oracle's forward + backward on a bounded sample with at least `threads` units, on
    `threads` host threads; tokens/s scaled to the workload's tokens."""
    import oracle
    kind, inp, frac, w, desc = oracle_sample(name, threads)
    oracle.set_threads(threads)
    oracle_step(kind, inp, w)  # warm (page-in, library load)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_step(kind, inp, w)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    per = el / n
    toks = tokens_of(w) * frac
    return {"value": toks / per, "unit": "tokens/s", "cores": min(threads, parallel_units(kind, inp)),
            "kind": "oracle", "sample": desc + " (fp64 C oracle, forward + backward, %d run(s))" % n,
            "seconds_per_sample": per}


def cpu_baseline(name):
    """The oracle at all host cores (the reported value) and at one thread."""
    cores = host_cores()
    os.environ["OMP_NUM_THREADS"] = str(cores)  # read by the OpenMP runtime when the oracle loads
    allc = time_oracle(name, cores)
    one = time_oracle(name, 1)
    out = {k: allc[k] for k in ("value", "unit", "cores", "kind", "sample")}
    out["host_cores"] = cores
    out["one_thread"] = {"value": one["value"], "unit": "tokens/s", "sample": one["sample"]}
    return out


# ---------------------------------------------------------------------------------- main
def built_workloads():
    """Workloads whose kind the library implements (lr_validate reports UNSUPPORTED otherwise)."""
    import torch
    from selective_state_space_09_b200 import inputs, lrscan
    ok = []
    for name in BENCH_ORDER:
        w = dict(inputs.WORKLOADS[name])
        kind = w.pop("kind")
        io = torch.bfloat16 if w.pop("io") == "bf16" else torch.float32
        if kind == "gla":
            w["N"], w["P"] = w.pop("K"), w.pop("V")
        seg = w.pop("segment")
        softplus = w.pop("softplus", False)
        gates = w.pop("gates", False)
        d = lrscan.make_desc(kind, io, segment=seg, **w)
        if softplus:
            d.flags |= lrscan.DELTA_SOFTPLUS
        if gates:
            d.flags |= lrscan.RGLRU_GATES
        if lrscan.validate(d) == 0:
            ok.append(name)
    return ok


def relaunch_ranks(args):
    """`--gpus N` with N > 1 outside a torchrun launch: start N ranks, one per GPU, through
    torch.distributed.run on this host and return its exit status (rank 0 prints the line)."""
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(args.gpus),
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__)] + sys.argv[1:]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None, help="headline workload (default: ssd)")
    ap.add_argument("--only-headline", action="store_true", help="skip the per-kind lines")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's batch (small profiling cases only)")
    args = ap.parse_args()
    global BATCH_OVERRIDE
    BATCH_OVERRIDE = args.batch
    assert args.warmup >= 3 or args.impl == "reference", "at least 3 warm-up steps"

    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return relaunch_ranks(args)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        print("bench: --gpus %d but WORLD_SIZE %d; timing %d rank(s)" % (args.gpus, world, world), file=sys.stderr)

    if args.impl == "reference":
        if rank != 0:
            return 0
        return reference_arm(args, world)

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    from selective_state_space_09_b200 import build as _b  # noqa: F401
    built = built_workloads()
    if not built:
        raise SystemExit("no workload is built")
    head = args.workload or ("ssd" if "ssd" in built else built[0])
    others = [] if args.only_headline else [n for n in BENCH_ORDER if n in built and n != head]

    pk = peaks()
    rates = measure_pipe_rates(device)
    flush_buf = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=device)  # 256 MiB > L2
    props = torch.cuda.get_device_properties(device)
    sampler = ClockSampler(getattr(props, "uuid", None) and ("GPU-" + str(props.uuid)) or local)
    sampler.start()
    time.sleep(0.3)
    results = {}
    for name in [head] + others:
        big = name == "rotlru"  # 10 GiB of inputs: far larger than L2, no flush needed
        r = run_workload(name, args.steps, args.warmup, device, rank, world, None if big else flush_buf,
                         e2e=(name == head), rates=rates)
        sampler.mark(*r["window"])
        results[name] = r
        torch.cuda.empty_cache()
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary()
    del flush_buf

    h = results[head]
    dom_row = max(h["kernels_timed"], key=lambda r: r["ms"])
    roofline = kernel_roofline(dom_row, pk)
    step_bytes = h["fwd_bytes"] + h["bwd_bytes"]
    roofline.update({
        "traffic": ncu_traffic(dom_row["kernel"], dom_row["pass"]), "kernel": dom_row["kernel"], "pass": dom_row["pass"],
        "algorithmic_bytes_per_launch": dom_row["bytes"], "algorithmic_flops_per_launch": dom_row["flops"],
        "ms_per_launch": round(dom_row["ms"], 5), "segment": h["segment"],
        "step": {"algorithmic_bytes": step_bytes, "ms": round(h["ms_per_step"], 5),
                 "achieved_gbs": round(h["step_gbs"], 1), "frac": round(h["step_gbs"] / pk["hbm_gbs"], 4)},
        "kernels": [dict(kernel_roofline(r, pk), kernel=r["kernel"], **{"pass": r["pass"], "ms": round(r["ms"], 5)})
                    for r in h["kernels_timed"] if r["bytes"] or r["flops"]],
        "note": "of %s peak (burst GEMM / copy); algorithmic bytes = the kernel's operands each once "
                "(inputs, outputs, gradients, f32 checkpoints at the configured segment length; no "
                "intermediates); kernel time from CUDA events the library records before each launch "
                "on the call's stream, in a second timed loop of the same steps (events between kernels "
                "stop the next kernel from starting early, so the headline loop runs without them)" % pk["source"]})
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(head)
    per_kind = {}
    for name, r in results.items():
        dom = max(r["kernels_timed"], key=lambda q: q["ms"])
        per_kind[name] = {
            "desc": r["desc"], "tokens_per_s": round(r["tokens_per_s"], 1),
            "ms_fwd": round(r["ms_fwd"], 5), "ms_bwd": round(r["ms_bwd"], 5),
            "fwd_gbs": round(r["fwd_gbs"], 1), "bwd_gbs": round(r["bwd_gbs"], 1),
            "fwd_frac_hbm": round(r["fwd_gbs"] / pk["hbm_gbs"], 4),
            "bwd_frac_hbm": round(r["bwd_gbs"] / pk["hbm_gbs"], 4),
            "step_frac_hbm": round(r["step_gbs"] / pk["hbm_gbs"], 4),
            "kernels": r["fwd_kernels"] + " | " + r["bwd_kernels"],
            "kernel_ms": {"%s:%d:%s" % (k["pass"], k["index"], k["kernel"]): round(k["ms"], 5)
                          for k in r["kernels_timed"]},
            "kernel_roofline": {"%s:%d:%s" % (k["pass"], k["index"], k["kernel"]): kernel_roofline(k, pk)
                                for k in r["kernels_timed"] if k["bytes"] or k["flops"]},
            "dominant_kernel": dict(kernel_roofline(dom, pk), kernel=dom["kernel"]),
            "peak_mem_gib": round(r["peak_mem_bytes"] / 2 ** 30, 3), "l2": r["l2"],
            "segment": r["segment"], "checkpoint_bytes": r["ckpt_bytes"],
        }
        if r.get("l2_warm"):
            per_kind[name]["l2_warm"] = r["l2_warm"]
        if r.get("graph"):
            per_kind[name]["graph"] = r["graph"]
        if "decode" in r:
            d = dict(r["decode"])
            d["tokens_per_s"] = round(d["tokens_per_s"], 1)
            per_kind[name]["decode"] = d
        if "full_state" in r:
            f = dict(r["full_state"])
            f["time_ratio"] = round((f["ms_fwd"] + f["ms_bwd"]) / (r["ms_fwd"] + r["ms_bwd"]), 3)
            per_kind[name]["full_state"] = f
        if "segments" in r:
            sg = dict(r["segments"])
            sg["default"].update(ms_fwd=round(r["ms_fwd"], 5), ms_bwd=round(r["ms_bwd"], 5))
            sg["note"] = ("one chunk per segment keeps every chunk's entering state (f32 + bf16 copy), the "
                          "chunked form's full-state analog; longer segments keep f32 segment states and "
                          "rebuild the rest; per_step_state_bytes: every step's state, which the chunked "
                          "backward never reads")
            per_kind[name]["segments"] = sg
            # the full-state comparison in the chunked form: every chunk's entering state kept
            # (segment = chunk, the default) against the longest measured segment's checkpoints
            ck = max((k for k in sg if k.startswith("S") and k[1:].isdigit()), key=lambda k: int(k[1:]), default=None)
            if ck:
                lo = sg[ck]
                per_kind[name]["full_state"] = {
                    "analog": "every chunk's entering state kept (segment = chunk) vs f32 checkpoints every "
                              "%d steps" % lo["segment"],
                    "ms_fwd": round(r["ms_fwd"], 5), "ms_bwd": round(r["ms_bwd"], 5),
                    "state_bytes": sg["default"]["checkpoint_bytes"], "checkpoint_bytes": lo["checkpoint_bytes"],
                    "memory_ratio": round(sg["default"]["checkpoint_bytes"] / lo["checkpoint_bytes"], 2),
                    "time_ratio": round((r["ms_fwd"] + r["ms_bwd"]) / (lo["ms_fwd"] + lo["ms_bwd"]), 3),
                    "per_step_state_bytes": sg["per_step_state_bytes"]}
    line = {
        "metric": METRIC, "value": round(h["tokens_per_s"], 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(h["ms_per_step"], 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": h["io_dtype"], "data": "synthetic (seeded; distributions of the workload)",
        "config": {"workload": NAMES[head], "global_batch": h["tokens_per_step"] // inputs_L(head),
                   "seq_len": inputs_L(head), "parallelism": "dp%d" % world if world > 1 else "single",
                   "l2": h["l2"]},
        "e2e": {k: (round(v, 1) if isinstance(v, float) else v) for k, v in h["e2e"].items()},
        "gpu_launches": args.steps * sum(r["launches_per_step"] for r in [h]),
        "graph": h.get("graph"),
        "roofline": roofline,
        "cpu_baseline": cpu,
        "clocks": clocks,
        "pipe_rates": {k: (round(v, 1) if isinstance(v, float) and v > 1e6 else v) for k, v in rates.items()},
        "per_kind": per_kind,
        "src_sha": src_sha(),
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        dist.destroy_process_group()
    return 0


def inputs_L(name):
    from selective_state_space_09_b200 import inputs
    return inputs.WORKLOADS[name]["L"]


def reference_arm(args, world):
    """The fp64 CPU oracle on all host cores: each step is a bounded sample of the workload.  The
    workload is chosen by name; nothing here loads the CUDA library."""
    # torch.distributed.run exports OMP_NUM_THREADS=1, which the OpenMP runtime reads when the
    # oracle library loads
    os.environ["OMP_NUM_THREADS"] = str(host_cores())
    import oracle
    from selective_state_space_09_b200 import inputs
    name = args.workload or "ssd"
    if name not in inputs.WORKLOADS:
        raise SystemExit("unknown workload %s" % name)
    cores = host_cores()
    kind, inp, frac, w, desc = oracle_sample(name, cores)
    oracle.set_threads(cores)
    for _ in range(args.warmup):
        oracle_step(kind, inp, w)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(kind, inp, w)
    el = time.perf_counter() - t0
    per = el / max(args.steps, 1)
    toks = tokens_of(w) * frac
    v = toks / per
    line = {
        "impl": "reference", "metric": METRIC, "value": round(v, 1), "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(per * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; distributions of the workload)",
        "config": {"workload": NAMES[name], "global_batch": w["B"] * world, "seq_len": w["L"],
                   "parallelism": "dp%d" % world if world > 1 else "single",
                   "l2": "inputs larger than L2" if name == "rotlru" else "flushed between steps"},
        "cpu_baseline": {"value": round(v, 1), "unit": "tokens/s",
                         "cores": min(cores, parallel_units(kind, inp)), "kind": "oracle",
                         "sample": desc + " per step (fp64 C oracle, forward + backward)"},
        "e2e": {"value": round(v, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
