#!/usr/bin/env python
"""Benchmark of the q4gsw linear layer on B200.

One step = the adapter-training pass of one 1B-class decoder layer (hidden
2048, 32 query / 8 key-value heads of width 64, MLP 8192) over a frozen q4gsw
base, 512 tokens, group size 32:
    fused Q/K/V forward   x[512,2048] -> y_q[512,2048], y_k[512,512], y_v[512,512]
    MLP up forward        x[512,2048] -> y[512,8192]
    MLP down forward      x[512,8192] -> y[512,2048]
    MLP down input grad   d_out[512,2048] -> d_x[512,8192]
    MLP up input grad     d_out[512,8192] -> d_x[512,2048]
All inputs are seeded synthetic tensors (x ~ N(0,1), codes uniform 0..15,
scales U[0.005, 0.02], d_out ~ N(0, 1e-2)), prepacked once (not timed).
Between steps the weights and activations rotate over R copies whose total
exceeds the 126 MB L2, so every step reads its weights from HBM.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
        python bench.py --sweep        (one JSON line per configuration shape)
Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import glob
import json
import math
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_group_quantized_q4gsw_b200 import workloads as wl  # noqa: E402

METRIC = "q4gsw fwd+bwd_input TFLOP/s and weight GB/s on 1 B200, % of roofline"
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
WORKLOAD = ("adapter-training step of one 1B-class decoder layer on a frozen q4gsw base: "
            "fused QKV fwd (K2048->2048+512+512) + MLP up fwd (2048->8192) + down fwd (8192->2048) "
            "+ down and up input grads; M=512 tokens, group_size 32")

# DRAM bytes per launch from one ncu capture of each op (dram__bytes_read.sum +
# dram__bytes_write.sum), with the hash of the tensor-memory GEMM's sources they
# were taken on: reported only while those sources still match, null otherwise.
NCU_TRAFFIC = {"sources_sha": "84dc57c36ba89256", "bytes_per_launch": {'qkv_fwd': 5713000, 'up_fwd': 11604000, 'down_fwd': 17896000, 'down_bwd': 11604000, 'up_bwd': 17897000}}


# the files the tensor-memory GEMM (every op of the step) is built from
TS_SOURCES = ("q4gsw_gemm_ts.cuh", "q4gsw_sm100.cuh", "q4gsw_common.cuh", "q4gsw_internal.h")


def sources_sha() -> str:
    h = hashlib.sha256()
    for f in TS_SOURCES:
        h.update(open(os.path.join(ROOT, "bit_group_quantized_q4gsw_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def measured_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "tflops": d["bf16_tflops"], "tflops_sustained": d["bf16_tflops_sustained"],
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "tflops": 1590.0, "tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- the step
def step_ops():
    """(name, kind, shape) for the five operations of one step."""
    qkv = wl.by_name("qkv_M512")
    up, down = wl.adapter()
    return [("qkv_fwd", "qkv", qkv), ("up_fwd", "fwd", up), ("down_fwd", "fwd", down),
            ("down_bwd", "bwd", down), ("up_bwd", "bwd", up)]


ADAPTER_RANK = 16   # rank of the low-rank adapter beside the frozen base in the adapter legs


def op_flops(kind, sh, M=None):
    M = sh.M if M is None else M
    if kind == "emb":
        return float(M * sh.K)          # one multiply per gathered element
    if kind in ("ad_fwd", "ad_bwd"):   # base product plus the two low-rank products
        return 2.0 * M * sh.N * sh.K + 2.0 * M * ADAPTER_RANK * (sh.N + sh.K)
    return 2.0 * M * sh.N * sh.K


def op_bytes(kind, sh, M=None):
    """Algorithmic bytes: packed codes + scales once, activations in, fp32 out."""
    M = sh.M if M is None else M
    if kind == "emb":
        # per gathered row: its nibble-pair row (K bytes, the row shares them
        # with its pair), its K/gs fp16 scales, K fp32 outputs; the 4-byte id
        return M * (sh.K + 2 * (sh.K // sh.group_size) + 4 * sh.K + 4)
    w = sh.N * sh.K // 2 + 2 * (sh.K // sh.group_size) * sh.N
    if kind in ("ad_fwd", "ad_bwd"):   # plus both adapter matrices
        w += 2 * ADAPTER_RANK * (sh.N + sh.K)
    if kind in ("bwd", "ad_bwd"):
        return w + 2 * M * sh.N + 4 * M * sh.K
    return w + 2 * M * sh.K + 4 * M * sh.N


def weight_bytes(sh):
    return sh.N * sh.K // 2 + 2 * (sh.K // sh.group_size) * sh.N


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {"gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
               "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100}

    def __init__(self, index: int):
        self.samples = []
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _run(self):
        while not self._stop.is_set():
            try:
                mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= r
        reasons = [k for k, v in self.REASONS.items() if bits & v and k != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.samples)}


# ----------------------------------------------------------------------------- CPU oracle legs
def oracle_sample_step(inputs, frac_cols: int):
    """The five operations through the oracle on a sample: all tokens, and the
    first 1/frac_cols of each operation's output features (whole groups).
    Returns (seconds, flops of the sample)."""
    import oracle as o
    bits = lambda a: np.asarray(a, np.float16).view(np.uint16)
    t0 = time.perf_counter()
    flops = 0.0
    for name, kind, sh in step_ops():
        inp = inputs[name]
        M = inp.x.shape[0]
        if kind in ("fwd", "qkv"):
            n = max(8, (sh.N // frac_cols) // 8 * 8)
            o.linear_fwd(bits(inp.x), inp.codes[:n], bits(inp.scales[:, :n]), sh.group_size)
            flops += 2.0 * M * n * sh.K
        else:
            kk = max(sh.group_size, (sh.K // frac_cols) // sh.group_size * sh.group_size)
            o.linear_bwd_input(bits(inp.d_out), inp.codes[:, :kk], bits(inp.scales[:kk // sh.group_size]),
                               sh.group_size)
            flops += 2.0 * M * sh.N * kk
    return time.perf_counter() - t0, flops


def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        info = [d for d in threadpool_info() if d.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return os.cpu_count() or 1


def host_inputs():
    out = {}
    for name, kind, sh in step_ops():
        out[name] = wl.make_inputs(sh)
    return out


ORACLE_BUDGET_S = 150.0   # bound on the oracle's whole timed run (warm-up included)


def oracle_sample_fraction(inputs, runs: int) -> int:
    """The one sample rule of both oracle legs: the first 1/frac of each op's
    output features, frac the smallest power of two >= 16 for which `runs`
    sample steps fit in ORACLE_BUDGET_S on this host."""
    t, _ = oracle_sample_step(inputs, 64)
    t16 = 4.0 * t                    # cost grows with the sampled features
    frac = 16
    while frac < 4096 and runs * t16 * 16 / frac > ORACLE_BUDGET_S:
        frac *= 2
    return frac


def oracle_sample_text(frac: int, flops: float) -> str:
    return (f"all 5 ops of the step, all 512 tokens, first 1/{frac} of each op's output features "
            f"({flops / 1e9:.3f} GFLOP per sample step)")


def cpu_baseline(inputs, runs: int = 10):
    frac = oracle_sample_fraction(inputs, runs)
    times, flops = [], 0.0
    for _ in range(runs):
        dt, flops = oracle_sample_step(inputs, frac)
        times.append(dt)
    value = flops / statistics.median(times) / 1e12
    return {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
            "sample": oracle_sample_text(frac, flops) + f"; {runs} sample steps, median"}


def step_config(world: int) -> dict:
    """The workload description both arms print (identical keys and values)."""
    ops = step_ops()
    set_bytes = sum(weight_bytes(sh) for sh in {sh.name: sh for _, _, sh in ops}.values())
    act_bytes = sum(2 * sh.M * (sh.N if k == "bwd" else sh.K) for _, k, sh in ops)
    copies = max(2, math.ceil(2.0 * L2_BYTES / (set_bytes + act_bytes)))
    return {"workload": WORKLOAD, "global_batch": 512 * world, "seq_len": 512,
            "parallelism": f"replicas{world}" if world > 1 else "single",
            "l2": f"rotating {copies} copies of weights+activations "
                  f"({copies * (set_bytes + act_bytes) / 1e6:.0f} MB) > 126 MB L2"}, copies


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    inputs = host_inputs()
    frac = oracle_sample_fraction(inputs, args.steps + args.warmup)
    for _ in range(args.warmup):
        oracle_sample_step(inputs, frac)
    times, flops = [], 0.0
    for _ in range(args.steps):
        dt, flops = oracle_sample_step(inputs, frac)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms / 1e3) / 1e12
    config, _ = step_config(world)
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle_threads(), "kind": "oracle",
                             "sample": oracle_sample_text(frac, flops) + f"; {args.steps} timed steps, mean"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm
class GpuStep:
    """Device buffers for R rotating copies of the step's weights and activations."""

    def __init__(self, inputs, copies, device):
        import torch
        import bit_group_quantized_q4gsw_b200 as q
        self.q = q
        self.torch = torch
        self.lib = q.library()
        self.dev = device
        self.stream = torch.cuda.current_stream(device)
        self.sptr = self.stream.cuda_stream
        self.ops = step_ops()
        self.copies = copies
        self.packed, self.acts, self.outs = {}, {}, {}
        for name, kind, sh in self.ops:
            inp = inputs[name]
            key = sh.name
            if key not in self.packed:
                codes = torch.from_numpy(inp.codes).to(device)
                scales = torch.from_numpy(inp.scales).to(device)
                first = q.q4gsw_prepack(codes, scales, sh.group_size)
                self.packed[key] = [first] + [first.clone() for _ in range(copies - 1)]
            src = inp.d_out if kind == "bwd" else inp.x
            self.acts[name] = [torch.from_numpy(src).to(device) for _ in range(copies)]
            if kind == "qkv":
                Nq, Nk, Nv = sh.splits
                self.outs[name] = [torch.empty((sh.M, n), dtype=torch.float32, device=device) for n in (Nq, Nk, Nv)]
            elif kind == "fwd":
                self.outs[name] = [torch.empty((sh.M, sh.N), dtype=torch.float32, device=device)]
            else:
                self.outs[name] = [torch.empty((sh.M, sh.K), dtype=torch.float32, device=device)]
        torch.cuda.synchronize(device)

    def bytes_resident(self):
        tot = 0
        for v in self.packed.values():
            tot += sum(t.numel() for t in v)
        for v in self.acts.values():
            tot += sum(t.numel() * t.element_size() for t in v)
        return tot

    def call(self, name, kind, sh, c):
        """One operation through the C ABI on copy c (raw pointers, current stream)."""
        lib, s = self.lib, self.torch.cuda.current_stream(self.dev).cuda_stream
        pk = self.packed[sh.name][c].data_ptr()
        a = self.acts[name][c].data_ptr()
        o = self.outs[name]
        if kind == "qkv":
            Nq, Nk, Nv = sh.splits
            st = lib.q4gsw_qkv_fwd(pk, Nq, Nk, Nv, sh.K, sh.group_size, a, sh.M, o[0].data_ptr(), o[1].data_ptr(),
                                   o[2].data_ptr(), s)
        elif kind == "fwd":
            st = lib.q4gsw_linear_fwd(pk, sh.N, sh.K, sh.group_size, a, sh.M, o[0].data_ptr(), s)
        else:
            st = lib.q4gsw_linear_bwd_input(pk, sh.N, sh.K, sh.group_size, a, sh.M, o[0].data_ptr(), s)
        if st != 0:
            raise RuntimeError(f"{name}: status {st} ({lib.q4gsw_status_str(st).decode()})")

    def launches_per_call(self):
        out = {}
        for name, kind, sh in self.ops:
            self.call(name, kind, sh, 0)
            route = self.lib.q4gsw_last_route().decode()
            n = 1
            for tok in route.split():
                if tok.startswith("launches="):
                    n = int(tok.split("=")[1])
            out[name] = (n, route)
        self.torch.cuda.synchronize(self.dev)
        return out


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    """Largest value over all ranks (every rank gets it); the job time of a
    multi-GPU run is the slowest rank's.  Works on the nccl and gloo backends."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, units_per_rank: float, ms_per_step_max: float, unit_scale: float = 1e12) -> float:
    """Whole-job rate: the units all ranks processed per step over the slowest
    rank's step time (replicas: every rank does the same step)."""
    return world * units_per_rank / (ms_per_step_max / 1e3) / unit_scale


def run_gpu(args, rank, world, local_rank):
    import torch
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    peaks = measured_peaks()
    inputs = host_inputs()
    ops = step_ops()
    config, copies = step_config(world)
    copies = args.copies or copies
    gs = GpuStep(inputs, copies, device)
    per_call = gs.launches_per_call()
    launches_per_step = sum(n for n, _ in per_call.values())
    flops_step = sum(op_flops(k, sh) for _, k, sh in ops)
    wbytes_step = sum(weight_bytes(sh) for _, _, sh in ops)

    # ---- device-resident timed region
    # Consecutive launches overlap (programmatic dependent launch); an event
    # between two launches removes that overlap.  So per-operation events are
    # recorded on every 25th step only (the sampled steps, 8 of the default
    # 200); the other steps run back to back.  ms_per_step covers all K steps.
    nops = len(ops)
    SAMPLE = 25
    sampled = [i for i in range(args.steps) if i % SAMPLE == SAMPLE - 1] or [args.steps - 1]
    ev = {i: [torch.cuda.Event(enable_timing=True) for _ in range(nops + 1)] for i in sampled}
    for i in range(args.warmup):
        for name, kind, sh in ops:
            gs.call(name, kind, sh, i % copies)
    torch.cuda.synchronize(device)
    barrier(world)
    torch.cuda.synchronize(device)
    sampler = ClockSampler(local_rank)
    with sampler:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record()
        for i in range(args.steps):
            c = (args.warmup + i) % copies
            if i in ev:
                ev[i][0].record()
                for j, (name, kind, sh) in enumerate(ops):
                    gs.call(name, kind, sh, c)
                    ev[i][j + 1].record()
            else:
                for name, kind, sh in ops:
                    gs.call(name, kind, sh, c)
        end.record()
        torch.cuda.synchronize(device)
    barrier(world)
    torch.cuda.synchronize(device)
    # a bounded wait that ran out inside the timed region makes its time meaningless
    gs.q.q4gsw_device_error_check()
    ms_total = start.elapsed_time(end)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    value = job_throughput(world, flops_step, ms_step)
    op_ms = {}
    for j, (name, kind, sh) in enumerate(ops):
        op_ms[name] = statistics.mean(ev[i][j].elapsed_time(ev[i][j + 1]) for i in ev)
    clocks = sampler.summary()

    # dominant op -> roofline
    dom = max(op_ms, key=op_ms.get)
    dkind, dsh = [(k, sh) for n, k, sh in ops if n == dom][0]
    n_launch = per_call[dom][0]
    fl = op_flops(dkind, dsh)
    by = op_bytes(dkind, dsh)
    ridge = peaks["tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if fl / by >= ridge:
        achieved = fl / (op_ms[dom] / n_launch / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["tflops"], "unit": "TFLOP/s",
                "peak_kind": f"bf16 dense burst ({peaks['source']})"}
    else:
        achieved = by / (op_ms[dom] / n_launch / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "peak_kind": f"HBM copy ({peaks['source']})"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    traffic = None
    if NCU_TRAFFIC["sources_sha"] == sources_sha():
        traffic = NCU_TRAFFIC["bytes_per_launch"].get(dom)
    roof["traffic"] = traffic
    roof["kernel"] = per_call[dom][1]
    roof["op"] = dom
    roof["duration_us"] = op_ms[dom] * 1e3 / n_launch
    roof["timing"] = (f"CUDA events around each launch on {len(ev)} sampled steps (every {SAMPLE}th) of the "
                      "timed region; an event between launches removes their overlap, so this is the "
                      "launch's stand-alone duration")

    # ---- end to end through the public Python API with pinned host buffers
    q = gs.q
    host_in = {}
    for name, kind, sh in ops:
        src = inputs[name].d_out if kind == "bwd" else inputs[name].x
        host_in[name] = torch.from_numpy(src).pin_memory()
    host_out = {name: [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in gs.outs[name]] for name, _, _ in ops}
    # Three streams, device inputs and outputs double-buffered: the copy-in of
    # step i+1 and the copy-out of step i-1 overlap the launches of step i.
    # Every step still copies all of its inputs in and all of its outputs out.
    dev_in = [{name: torch.empty(host_in[name].shape, dtype=torch.float16, device=device) for name, _, _ in ops}
              for _ in range(2)]
    dev_out = [gs.outs, {name: [torch.empty_like(t) for t in v] for name, v in gs.outs.items()}]
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for v in host_out.values() for t in v)
    e2e_steps = max(1, min(args.steps, 50))
    s_comp = torch.cuda.current_stream(device)
    s_h2d = torch.cuda.Stream(device)
    s_d2h = torch.cuda.Stream(device)
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_copied = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):
        comp_done[b].record(s_comp)
        out_copied[b].record(s_comp)

    def e2e_step(i, c):
        b = i & 1
        s_h2d.wait_event(comp_done[b])          # step i-2 no longer reads dev_in[b]
        with torch.cuda.stream(s_h2d):
            for name, _, _ in ops:
                dev_in[b][name].copy_(host_in[name], non_blocking=True)
            in_ready[b].record(s_h2d)
        s_comp.wait_event(in_ready[b])
        s_comp.wait_event(out_copied[b])        # step i-2's outputs have reached the host
        with torch.cuda.stream(s_comp):
            for name, kind, sh in ops:
                pk = gs.packed[sh.name][c]
                o = dev_out[b][name]
                xin = dev_in[b][name]
                if kind == "qkv":
                    Nq, Nk, Nv = sh.splits
                    q.q4gsw_qkv_fwd(pk, Nq, Nk, Nv, sh.K, sh.group_size, xin, outs=o)
                elif kind == "fwd":
                    q.q4gsw_linear_fwd(pk, sh.N, sh.K, sh.group_size, xin, y=o[0])
                else:
                    q.q4gsw_linear_bwd_input(pk, sh.N, sh.K, sh.group_size, xin, d_x=o[0])
            comp_done[b].record(s_comp)
        s_d2h.wait_event(comp_done[b])
        with torch.cuda.stream(s_d2h):
            for name, _, _ in ops:
                for hb, db in zip(host_out[name], dev_out[b][name]):
                    hb.copy_(db, non_blocking=True)
            out_copied[b].record(s_d2h)

    for i in range(min(args.warmup, 3)):
        e2e_step(i, i % copies)
    torch.cuda.synchronize(device)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    start = torch.cuda.Event()
    e0.record(s_comp)
    start.record(s_comp)
    s_h2d.wait_event(start)
    s_d2h.wait_event(start)
    for i in range(e2e_steps):
        e2e_step(i, i % copies)
    s_comp.wait_event(out_copied[0])
    s_comp.wait_event(out_copied[1])
    e1.record(s_comp)
    torch.cuda.synchronize(device)
    barrier(world)
    gs.q.q4gsw_device_error_check()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    e2e = {"value": job_throughput(world, flops_step, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
           "overlap": "copy-in of step i+1 and copy-out of step i-1 run on their own streams beside the "
                      "launches of step i (device buffers double-buffered)"}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f16 inputs, f32 accumulate", "data": "synthetic",
            "config": config,
            "weight_gbs": world * wbytes_step / (ms_step / 1e3) / 1e9,
            "roofline": roof, "clocks": clocks, "gpu_launches": launches_per_step * args.steps,
            "e2e": e2e,
            "ops_ms_sampled": {k: round(v, 5) for k, v in op_ms.items()},
            "ops_tflops": {n: op_flops(k, sh) / (op_ms[n] / 1e3) / 1e12 for n, k, sh in ops},
            "routes": {k: v[1] for k, v in per_call.items()}}
    if not args.no_shapes:
        line["shapes"] = shape_legs(device, peaks, world)
        gs.q.q4gsw_device_error_check()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(inputs)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- per-shape timing
def time_shape(q, sh, kind, device, flush, peaks):
    """One operation of one configuration shape: mean time per launch over a
    CUDA graph of back-to-back launches whose packed weights rotate through
    copies totalling > 3x the L2, plus one launch timed alone after an L2 flush.
    Returns the JSON record with both rooflines.  A kind "fwd@ts" / "fwd@ss"
    pins the tensor-core GEMM route (tensor-memory or shared-memory tile)."""
    import torch
    if "@" in kind:
        kind, pin = kind.split("@")
        q.q4gsw_debug_pin_routes(gemm=pin)
        try:
            rec = time_shape(q, sh, kind, device, flush, peaks)
        finally:
            q.q4gsw_debug_pin_routes()
        rec["dir"] = f"{kind}@{pin}"
        return rec
    inp = wl.make_inputs(sh)
    codes = torch.from_numpy(inp.codes).to(device)
    scales = torch.from_numpy(inp.scales).to(device)
    first = q.q4gsw_prepack(codes, scales, sh.group_size)
    del codes, scales
    wb = weight_bytes(sh)
    R = max(2, math.ceil(max(3 * L2_BYTES, 512 * 2**20) / wb))   # at least 512 MB of weight copies
    packs = [first] + [first.clone() for _ in range(R - 1)]
    src = inp.d_out if kind in ("bwd", "ad_bwd") else inp.x
    a = torch.from_numpy(src).to(device)
    if kind in ("ad_fwd", "ad_bwd"):
        rng = np.random.default_rng(sh.seed + 1)
        A = torch.from_numpy((rng.standard_normal((ADAPTER_RANK, sh.K)) * 0.05).astype(np.float16)).to(device)
        B = torch.from_numpy((rng.standard_normal((sh.N, ADAPTER_RANK)) * 0.05).astype(np.float16)).to(device)
        ws = torch.empty(q.library().q4gsw_adapter_workspace_bytes(sh.M, ADAPTER_RANK), dtype=torch.uint8,
                         device=device)
        y = torch.empty((sh.M, sh.N if kind == "ad_fwd" else sh.K), dtype=torch.float32, device=device)
        if kind == "ad_fwd":
            fn = lambda pk: q.q4gsw_adapter_fwd(pk, sh.N, sh.K, sh.group_size, A, B, a, y=y, workspace=ws)
        else:
            fn = lambda pk: q.q4gsw_adapter_bwd_input(pk, sh.N, sh.K, sh.group_size, A, B, a, d_x=y, workspace=ws)
    elif kind == "qkv":
        Nq, Nk, Nv = sh.splits
        outs = tuple(torch.empty((sh.M, n), dtype=torch.float32, device=device) for n in (Nq, Nk, Nv))
        fn = lambda pk: q.q4gsw_qkv_fwd(pk, Nq, Nk, Nv, sh.K, sh.group_size, a, outs=outs)
    elif kind == "fwd":
        y = torch.empty((sh.M, sh.N), dtype=torch.float32, device=device)
        fn = lambda pk: q.q4gsw_linear_fwd(pk, sh.N, sh.K, sh.group_size, a, y=y)
    elif kind == "dq8ca":
        y = torch.empty((sh.M, sh.N), dtype=torch.float32, device=device)
        ws = torch.empty(q.library().q4gsw_dq8ca_workspace_bytes(sh.M, sh.K), dtype=torch.uint8, device=device)
        fn = lambda pk: q.q4gsw_linear_dq8ca_fwd(pk, sh.N, sh.K, sh.group_size, a, y=y, workspace=ws)
    elif kind == "emb":
        ids = torch.from_numpy(wl.embedding_indices(sh)).to(device)
        y = torch.empty((sh.M, sh.K), dtype=torch.float32, device=device)
        fn = lambda pk: q.q4gsw_embedding(pk, sh.N, sh.K, sh.group_size, ids, out=y)
    else:
        y = torch.empty((sh.M, sh.K), dtype=torch.float32, device=device)
        fn = lambda pk: q.q4gsw_linear_bwd_input(pk, sh.N, sh.K, sh.group_size, a, d_x=y)
    for i in range(5):
        fn(packs[i % R])
    torch.cuda.synchronize()
    iters = max(R, 50)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(iters):
            fn(packs[i % R])
    g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 3
    e0.record()
    for _ in range(reps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    t = e0.elapsed_time(e1) / (reps * iters) / 1e3
    # one launch after an L2 flush (a 256 MB write), timed alone: the launch is
    # enqueued while the flush still runs, so host launch latency stays
    # outside the events
    singles = []
    for r in range(3):
        torch.cuda.synchronize()
        flush.fill_(r)
        e0.record()
        fn(packs[r % R])
        e1.record()
        torch.cuda.synchronize()
        singles.append(e0.elapsed_time(e1) * 1e3)
    t1 = sorted(singles)[1]
    route = q.q4gsw_last_route()
    del g, packs, first
    fl = op_flops(kind, sh)
    by = op_bytes(kind, sh)
    rec = {"shape": sh.name, "dir": kind, "M": sh.M, "N": sh.N, "K": sh.K, "gs": sh.group_size,
           "us": t * 1e6, "tflops": fl / t / 1e12, "gbs": by / t / 1e9, "weight_gbs": wb / t / 1e9,
           "frac_tc": fl / t / 1e12 / peaks["tflops"], "frac_hbm_measured": by / t / 1e9 / peaks["hbm_gbs"],
           "frac_hbm_8tbs": by / t / 8e12, "us_single_cold": t1, "route": route, "copies": R,
           "timing": f"CUDA graph of {iters} back-to-back launches over {R} rotating weight copies "
                     f"(>= 512 MB, > 3x L2), {reps} replays; us_single_cold: one launch after a 256 MB L2 flush"}
    ridge = peaks["tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if kind != "emb" and fl / by >= ridge:
        rec["roofline"] = {"bound": "tensor", "achieved": fl / t / 1e12, "peak": peaks["tflops"], "unit": "TFLOP/s",
                           "frac": fl / t / 1e12 / peaks["tflops"], "traffic": None,
                           "peak_kind": f"bf16 dense burst ({peaks['source']})"}
    else:
        rec["roofline"] = {"bound": "hbm", "achieved": by / t / 1e9, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                           "frac": by / t / 1e9 / peaks["hbm_gbs"], "traffic": None,
                           "peak_kind": f"HBM copy ({peaks['source']})"}
    return rec


# The configuration shapes timed beside the step: the memory-bound half of the
# metric (decode M=1; the sweep's M=1 and M=16 on both 8B-class matrices) and
# the largest compute-bound shapes (the sweep's M=4096); the adapter and the
# int8-activation product (dq8ca: algorithmic bytes as the fp16 forward, the
# quantised copy of x in the workspace counts as overhead); and at M=512 the
# two tensor-core GEMM routes side by side (dequantised tile in tensor memory,
# the default up to 512 tokens, or in shared memory).
SHAPE_LEGS = [("decode_N2048_K2048", "fwd"), ("decode_N8192_K2048", "fwd"), ("decode_N2048_K8192", "fwd"),
              ("sweep_M1_N14336_K4096", "fwd"), ("sweep_M1_N14336_K4096", "bwd"),
              ("sweep_M1_N4096_K14336", "fwd"), ("sweep_M1_N4096_K14336", "bwd"),
              ("sweep_M16_N14336_K4096", "fwd"), ("sweep_M16_N14336_K4096", "bwd"),
              ("sweep_M16_N4096_K14336", "fwd"), ("sweep_M16_N4096_K14336", "bwd"),
              ("sweep_M4096_N14336_K4096", "fwd"), ("sweep_M4096_N14336_K4096", "bwd"),
              ("sweep_M4096_N4096_K14336", "fwd"), ("sweep_M4096_N4096_K14336", "bwd"),
              ("adapter_up_M512", "ad_fwd"), ("adapter_up_M512", "ad_bwd"),
              ("adapter_down_M512", "ad_fwd"), ("adapter_down_M512", "ad_bwd"),
              ("decode_N8192_K2048", "dq8ca"), ("sweep_M1_N4096_K14336", "dq8ca"),
              ("sweep_M16_N14336_K4096", "dq8ca"),
              ("adapter_up_M512", "fwd@ts"), ("adapter_up_M512", "fwd@ss")]


def shape_legs(device, peaks, world):
    import torch
    import bit_group_quantized_q4gsw_b200 as q
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    out = []
    for name, kind in SHAPE_LEGS:
        barrier(world)
        rec = time_shape(q, wl.by_name(name), kind, device, flush, peaks)
        # whole-job figures: every rank runs the same shape (replicas)
        t_max = max_over_ranks(rec["us"], world)
        rec["us_max_over_ranks"] = t_max
        out.append(rec)
        torch.cuda.empty_cache()
    del flush
    torch.cuda.empty_cache()
    return out


def run_sweep(args):
    import torch
    import bit_group_quantized_q4gsw_b200 as q
    device = torch.device("cuda", 0)
    peaks = measured_peaks()
    shapes = wl.tiny() + wl.decode() + wl.qkv() + wl.adapter() + wl.sweep() + wl.embedding()
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    if args.only:
        import re
        shapes = [s for s in shapes if re.search(args.only, s.name)]
    for sh in shapes:
        kinds = ["qkv"] if sh.splits else list(sh.directions)
        for kind in kinds:
            print(json.dumps(time_shape(q, sh, kind, device, flush, peaks)), flush=True)
        torch.cuda.empty_cache()
    return 0


# ----------------------------------------------------------------------------- profiling cases
def run_case(args):
    """Launch one operation `--iters` times (for ncu captures); no timing."""
    import torch
    import bit_group_quantized_q4gsw_b200 as q
    device = torch.device("cuda", 0)
    name, kind = args.case.rsplit(":", 1)
    sh = wl.by_name(name)
    M = args.case_m or sh.M
    inp = wl.make_inputs(sh, M=M)
    pk = q.q4gsw_prepack(torch.from_numpy(inp.codes).to(device), torch.from_numpy(inp.scales).to(device),
                         sh.group_size)
    a = torch.from_numpy(inp.d_out if kind in ("bwd", "ad_bwd") else inp.x).to(device)
    for _ in range(args.iters):
        if kind == "qkv":
            Nq, Nk, Nv = sh.splits
            q.q4gsw_qkv_fwd(pk, Nq, Nk, Nv, sh.K, sh.group_size, a)
        elif kind == "fwd":
            q.q4gsw_linear_fwd(pk, sh.N, sh.K, sh.group_size, a)
        elif kind == "emb":
            q.q4gsw_embedding(pk, sh.N, sh.K, sh.group_size, torch.from_numpy(wl.embedding_indices(sh, M)).to(device))
        elif kind == "dq8ca":
            q.q4gsw_linear_dq8ca_fwd(pk, sh.N, sh.K, sh.group_size, a)
        elif kind in ("ad_fwd", "ad_bwd"):
            rng = np.random.default_rng(sh.seed + 1)
            A = torch.from_numpy((rng.standard_normal((ADAPTER_RANK, sh.K)) * 0.05).astype(np.float16)).to(device)
            B = torch.from_numpy((rng.standard_normal((sh.N, ADAPTER_RANK)) * 0.05).astype(np.float16)).to(device)
            if kind == "ad_fwd":
                q.q4gsw_adapter_fwd(pk, sh.N, sh.K, sh.group_size, A, B, a)
            else:
                q.q4gsw_adapter_bwd_input(pk, sh.N, sh.K, sh.group_size, A, B, a)
        else:
            q.q4gsw_linear_bwd_input(pk, sh.N, sh.K, sh.group_size, a)
    torch.cuda.synchronize()
    q.q4gsw_device_error_check()
    print(json.dumps({"case": args.case, "M": M, "iters": args.iters, "route": q.q4gsw_last_route()}), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--copies", type=int, default=0)
    ap.add_argument("--sweep", action="store_true")
    ap.add_argument("--only", default="")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-shapes", action="store_true", help="skip the per-shape legs beside the step")
    ap.add_argument("--case", default="", help="SHAPE:DIR, e.g. adapter_up_M512:fwd (profiling launches)")
    ap.add_argument("--case-m", type=int, default=0)
    ap.add_argument("--iters", type=int, default=3)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.sweep:
        return run_sweep(args)
    if args.case:
        return run_case(args)
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        return run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
