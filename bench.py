#!/usr/bin/env python
"""Benchmark of the differential attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload c2|c3|c4|c5|d1|b1|b3|p4] [--no-secondary]

A step is one pass of the hot path over one batch of synthetic input: the on-device
lambda re-parameterisation followed by the fused prefill (or the split-KV decode for the
decode workload). Default workload (the largest one-GPU workload): c5, the V2 long-context
signal-plus-noise prefill (B=1, N=65536, 64 query heads over 8 KV heads, d=128, causal).
Other workloads: c2 the V1 bf16 layer (B=2, 16 heads, N=4096, d=64), c3 V2 prefill
(N=16384, 64/8 heads, d=128), c4 V2 decode (batch 64, cache 32768), d1 V1 decode, b1 the
backward of the V1 layer and b3 that of a V2 prefill (N=4096, 64/8 heads; step = lambda +
the whole backward), p4 the c4 decode over 16-token pages in a shuffled block table.
Inputs are the seeded synthetic tensors of differential_attention_05_b200.synth. With the
default workload the line also carries "secondary": the other rows timed alone (the V1
layer and its backward, on the tensor cores and exact in fp32, the V2 prefill, its window
and chunk forms, the training
forward and the backward from its saved outputs, and the backward that recomputes them, on
the synth tensors; the decodes on same-shape seeded draws made on the device, each entry
saying which).

Timing: W untimed warm-up steps, then K steps between a barrier + synchronize on both
sides; every step is bracketed by CUDA events on the launching stream and L2 is flushed
(256 MB write) between steps when the inputs fit in L2. The maximum over ranks is taken.
Rank 0 prints one JSON line.

--impl reference times the float64 CPU oracle (the checker the kernels are held to) on
the host cores, on a bounded sample of the same workload, and prints the same line with
"impl": "reference".
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

L2_BYTES = 126 * 1024 * 1024


# ---------------------------------------------------------------------------------------
# workloads and their algorithmic work

def workload_inputs(name: str, batch: int = 0):
    """The named workload; `batch` > 0 shrinks the decode workload's batch (profiling runs)."""
    from differential_attention_05_b200 import synth
    if name == "c4" and batch:
        return synth.v2_decode(B=batch, name=f"v2_bf16_decode_b{batch}_l32768_hq64_hkv8_d128")
    if name == "d1":
        return synth.v1_decode(B=batch) if batch else synth.v1_decode()
    if name == "b1":
        return synth.v1_backward()
    if name == "b3":
        return synth.v2_backward()
    if name == "p4":
        return synth.v2_decode(B=batch or 64, name=f"v2_bf16_decode_paged16_b{batch or 64}_l32768_hq64_hkv8_d128")
    return {"c2": synth.config2, "c3": synth.config3, "c4": synth.config4, "c5": synth.config5}[name]()


def prefill_flops(inp) -> float:
    """Algorithmic FLOPs: per causal (i, j) pair, 12 d per V1 head (two d-wide QK^T dot
    products and two 2d-wide P.V rows, 2 flops per multiply-add) and 4 d per V2 query
    head; masked pairs, exp and the norm are not counted."""
    pairs = inp.N * (inp.N + 1) / 2 if inp.causal else float(inp.N) * inp.N
    per = 12 * inp.d * inp.H if inp.variant == 1 else 4 * inp.d * inp.H
    return float(inp.B) * pairs * per


def visible_pairs(Nq: int, Nk: int, causal: bool = True, window: int = 0) -> float:
    """(query, key) pairs a prefill attends: queries at the last Nq of Nk positions, each
    seeing keys up to its own position (causal), the last `window` of them when window > 0."""
    if not causal:
        return float(Nq) * Nk
    off = Nk - Nq
    seen = np.arange(off + 1, Nk + 1, dtype=np.float64)  # keys 0 .. i + off
    if window > 0:
        seen = np.minimum(seen, window)
    return float(seen.sum())


def workload_decode_bytes(inp) -> float:
    """Cache bytes one decode step reads: V2 K and V of width d per KV head; V1 K rows
    (K_1 | K_2, 2d) and V rows (2d) per head."""
    if inp.variant == 1:
        return decode_bytes(inp.B, inp.N, inp.H, 2 * inp.d)
    return decode_bytes(inp.B, inp.N, inp.Hkv, inp.d)


def decode_bytes(B, L, Hkv, d) -> float:
    """Algorithmic bytes: the K and V caches read once (bf16)."""
    return float(B) * L * Hkv * d * 2 * 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return {"hbm_gbs": float(pk["hbm_gbs"]), "bf16_tflops": float(pk["bf16_tflops"]),
                "bf16_tflops_sustained": float(pk.get("bf16_tflops_sustained", pk["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def measured_traffic(kernel: str, workload: str, batch: int, decode: bool):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu record
    (profiles/traffic.txt), or None when the kernel's sources changed since the capture or
    no capture covers the workload. A decode capture at a smaller batch of the same cache
    shape is scaled by the batch ratio (every batch entry reads its own cache once)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    csrc = os.path.join(ROOT, "differential_attention_05_b200", "csrc")
    try:
        lines = [ln.split() for ln in open(path) if ln.strip() and not ln.startswith("#")]
    except OSError:
        return None
    strip = lambda w: re.sub(r"_b\d+_", "_b*_", w)
    for f in lines:
        if len(f) != 5 or f[0] != kernel:
            continue
        if f[1] == workload:
            scale = 1.0
        elif decode and strip(f[1]) == strip(workload):
            scale = batch / float(re.search(r"_b(\d+)_", f[1]).group(1))
        else:
            continue
        m = hashlib.sha256()
        try:
            for src in f[3].split(","):
                m.update(open(os.path.join(csrc, src), "rb").read())
        except OSError:
            return None
        if m.hexdigest()[:16] != f[2]:
            return None
        return float(f[4]) * scale
    return None


def workload_config(inp, world: int) -> dict:
    """The line's "config": the workload and its sizes, identical in both arms."""
    decode = inp.mode == "decode"
    in_bytes = inp.q.nbytes + inp.k.nbytes + inp.v.nbytes
    return {
        "workload": inp.name,
        "batch": inp.B, "seq_len": inp.N, "heads": inp.H, "kv_heads": inp.Hkv,
        "head_dim": inp.d, "causal": bool(inp.causal), "depth": inp.depth,
        "tokens_per_step": inp.B * (1 if decode else inp.N),
        "l2": ("flushed between steps (256 MB write, outside the timed events)"
               if in_bytes < 2 * L2_BYTES else "inputs larger than L2"),
        "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
    }


# ---------------------------------------------------------------------------------------
# across ranks

def max_over_ranks(ms: float, dist=None, device=None) -> float:
    """The slowest rank's time: every rank times its own device with CUDA events and the
    job's time is the maximum (one rank: `ms` itself)."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, work_per_rank: float, steps: int, max_ms: float, scale: float) -> float:
    """Whole-job throughput: the work all ranks processed (each rank runs its own replica of
    the workload) divided by the slowest rank's time, in units of `scale` per second."""
    return world * work_per_rank * steps / (max_ms * 1e-3) / scale


# ---------------------------------------------------------------------------------------
# clocks during the timed region

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = tempfile.NamedTemporaryFile(mode="w+", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.out, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        self.out.flush()
        try:
            lines = open(self.out.name).read().strip().splitlines()
        except OSError:
            lines = []
        os.unlink(self.out.name)
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for nm, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------------------
# the GPU arm

def run_ours(args, rank, world, device):
    import torch

    import differential_attention_05_b200 as da

    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        dist = dist_mod
    peaks = load_peaks()
    inp = workload_inputs(args.workload, args.batch)

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    q, k, v = dev(inp.q), dev(inp.k), dev(inp.v)
    vecs = [dev(getattr(inp, n)) for n in ("lq1", "lk1", "lq2", "lk2")]
    lam = torch.empty(inp.n_units, dtype=torch.float32, device=device)
    li = torch.empty(1, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    decode = inp.mode == "decode"
    backward = args.workload in ("b1", "b3")
    paged = args.workload == "p4"
    if paged:
        # the cache as a pool of 16-token pages in a seeded shuffled order (block table)
        ps = 16
        kp = k.view(inp.B * inp.N // ps, ps, inp.Hkv, inp.d)
        vp = v.view(inp.B * inp.N // ps, ps, inp.Hkv, inp.d)
        gen = torch.Generator(device=device)
        gen.manual_seed(1008)
        bt = torch.randperm(inp.B * inp.N // ps, generator=gen, device=device).to(torch.int32)
        bt = bt.view(inp.B, inp.N // ps)
    if decode:
        if inp.variant == 1:
            out = torch.empty((inp.B, inp.H, 2 * inp.d), dtype=torch.bfloat16, device=device)
            p = da._binding.decode_params_v1(q, k, v, out)
        else:
            out = torch.empty((inp.B, inp.H // 2, inp.d), dtype=torch.bfloat16, device=device)
            p = da._binding.decode_params(q, k, v, out)
        ws = torch.empty(da._binding.diffattn_decode_workspace_size(p), dtype=torch.uint8,
                         device=device)
        work = workload_decode_bytes(inp)
        unit, metric = "GB/s", "diff-attn decode KV GB/s at 1 B200"
    elif backward:
        dy = dev(inp.extra["dy"])
        grads = (torch.empty(q.shape, dtype=torch.float32, device=device),
                 torch.empty(k.shape, dtype=torch.float32, device=device),
                 torch.empty(v.shape, dtype=torch.float32, device=device),
                 torch.empty(lam.shape, dtype=torch.float32, device=device))
        p = da._binding.prefill_params(q, k, v, dy)
        ws = torch.empty(da._binding.diffattn_bwd_workspace_size(p), dtype=torch.uint8, device=device)
        out = grads[0]
        work = backward_flops(inp)
        unit, metric = "TFLOP/s", "diff-attn backward TFLOP/s (% bf16 peak)"
    else:
        out = (torch.empty((inp.B, inp.N, inp.H, 2 * inp.d), dtype=torch.bfloat16, device=device)
               if inp.variant == 1 else
               torch.empty((inp.B, inp.N, inp.H // 2, inp.d), dtype=torch.bfloat16, device=device))
        work = prefill_flops(inp)
        unit, metric = "TFLOP/s", "diff-attn prefill TFLOP/s (% bf16 peak)"
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    flush = in_bytes < 2 * L2_BYTES
    scratch = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device) if flush else None

    # the device tensors of one step; the end-to-end measurement below runs two such sets
    # so that one step's copies overlap another step's kernels
    S0 = {"q": q, "k": k, "v": v, "vecs": vecs, "lam": lam, "li": li, "out": out}
    if backward:
        S0.update(dy=dy, grads=grads)

    def lambda_step(S=S0):
        da.diffattn_lambda(*S["vecs"], depth=inp.depth, lambda_out=S["lam"], lambda_init_out=S["li"])

    def main_kernel(S=S0):
        q, k, v, lam, li, out = S["q"], S["k"], S["v"], S["lam"], S["li"], S["out"]
        if paged:
            kp = k.view(inp.B * inp.N // ps, ps, inp.Hkv, inp.d)
            vp = v.view(inp.B * inp.N // ps, ps, inp.Hkv, inp.d)
            da.diffattn_fwd_decode_paged(q, kp, vp, bt, lam, out=out, workspace=ws)
        elif backward:
            da.diffattn_bwd_prefill(q, k, v, lam, S["dy"], li, causal=inp.causal,
                                    apply_norm=inp.apply_norm, norm_eps=inp.eps, workspace=ws,
                                    grads=S["grads"])
        elif decode and inp.variant == 1:
            da.diffattn_fwd_decode_v1(q, k, v, lam, li, out=out, apply_norm=inp.apply_norm,
                                      norm_eps=inp.eps, workspace=ws)
        elif decode:
            da.diffattn_fwd_decode(q, k, v, lam, out=out, workspace=ws)
        else:
            da.diffattn_fwd_prefill(q, k, v, lam, li, out=out, causal=inp.causal,
                                    apply_norm=inp.apply_norm, norm_eps=inp.eps)

    launches_per_step = 1 + (2 if decode else (4 if backward else 1))

    for _ in range(args.warmup):
        lambda_step()
        main_kernel()
        if flush:
            scratch.zero_()
    torch.cuda.synchronize(device)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        t_wall = time.perf_counter()
        for i in range(args.steps):
            ev[i][0].record(stream)
            lambda_step()
            ev[i][1].record(stream)
            main_kernel()
            ev[i][2].record(stream)
            if flush:
                scratch.zero_()  # outside the timed events
        torch.cuda.synchronize(device)
        if dist is not None:
            dist.barrier()
        t_wall = time.perf_counter() - t_wall
        time.sleep(0.25)
    clocks = clk.summary()
    step_ms = [e[0].elapsed_time(e[2]) for e in ev]
    kern_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = float(sum(step_ms))
    kern_avg = float(sum(kern_ms) / len(kern_ms))
    total_ms = max_over_ranks(total_ms, dist, device)
    ms_per_step = total_ms / args.steps
    if decode:
        value = job_rate(world, work, args.steps, total_ms, 1e9)
        achieved = work / (kern_avg * 1e-3) / 1e9
        peak, bound, runit = peaks["hbm_gbs"], "hbm", "GB/s"
    else:
        value = job_rate(world, work, args.steps, total_ms, 1e12)
        achieved = work / (kern_avg * 1e-3) / 1e12
        peak, bound, runit = peaks["bf16_tflops"], "tensor", "TFLOP/s"

    # end to end through the public API: pinned host inputs -> device, hot path, result -> host
    host_in = [torch.from_numpy(inp.q.view(np.int16) if inp.q.dtype == np.uint16 else inp.q).pin_memory(),
               torch.from_numpy(inp.k.view(np.int16) if inp.k.dtype == np.uint16 else inp.k).pin_memory(),
               torch.from_numpy(inp.v.view(np.int16) if inp.v.dtype == np.uint16 else inp.v).pin_memory()]
    host_vec = [torch.from_numpy(np.ascontiguousarray(getattr(inp, n))).pin_memory()
                for n in ("lq1", "lk1", "lq2", "lk2")]
    if backward:
        host_in.append(torch.from_numpy(inp.extra["dy"].view(np.int16)).pin_memory())
    dev_in_of = lambda S: (S["q"], S["k"], S["v"], S["dy"]) if backward else (S["q"], S["k"], S["v"])
    dev_out_of = lambda S: S["grads"] if backward else (S["out"],)
    S1 = {name: (torch.empty_like(t) if torch.is_tensor(t) else
                 (tuple(torch.empty_like(x) for x in t) if isinstance(t, tuple) else
                  [torch.empty_like(x) for x in t]))
          for name, t in S0.items()}
    sets = (S0, S1)
    host_outs = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out_of(S0)]
                 for _ in range(2)]
    h2d = sum(t.numel() * t.element_size() for t in host_in + host_vec)
    d2h = sum(t.numel() * t.element_size() for t in host_outs[0])
    e2e_steps = max(3, min(args.steps, 10))
    cs_in, cs_out = torch.cuda.Stream(device), torch.cuda.Stream(device)

    def copy_in(S):
        for src, dst in zip(host_in, dev_in_of(S)):
            dst.view(src.dtype).copy_(src, non_blocking=True)
        for src, dst in zip(host_vec, S["vecs"]):
            dst.copy_(src, non_blocking=True)

    def copy_out(S, ho):
        for dst, src in zip(ho, dev_out_of(S)):
            dst.copy_(src, non_blocking=True)

    def e2e_serial(n):
        # every step: inputs in, lambda + hot path, result out, one after the other
        for _ in range(n):
            copy_in(S0)
            lambda_step()
            main_kernel()
            copy_out(S0, host_outs[0])

    def e2e_pipelined(n):
        # step i runs on buffer set i % 2 while step i + 1's inputs are copied in (cs_in) and
        # step i - 1's result is copied out (cs_out); every step's bytes still cross the bus
        ready = [torch.cuda.Event() for _ in range(n)]
        done = [torch.cuda.Event() for _ in range(n)]
        copied = [torch.cuda.Event() for _ in range(n)]
        start = torch.cuda.Event()
        start.record(stream)
        cs_in.wait_event(start)
        cs_out.wait_event(start)
        with torch.cuda.stream(cs_in):
            copy_in(sets[0])
            ready[0].record(cs_in)
        for i in range(n):
            S = sets[i % 2]
            stream.wait_event(ready[i])
            if i >= 2:
                stream.wait_event(copied[i - 2])  # set i % 2's result of step i - 2 is out
            lambda_step(S)
            main_kernel(S)
            done[i].record(stream)
            if i + 1 < n:
                if i >= 1:
                    cs_in.wait_event(done[i - 1])  # set (i + 1) % 2 is free once step i - 1 ran
                with torch.cuda.stream(cs_in):
                    copy_in(sets[(i + 1) % 2])
                    ready[i + 1].record(cs_in)
            cs_out.wait_event(done[i])
            with torch.cuda.stream(cs_out):
                copy_out(S, host_outs[i % 2])
                copied[i].record(cs_out)
        stream.wait_event(copied[n - 1])

    def timed(fn):
        fn(2)  # untimed: first use of the copy streams and the second buffer set
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist is not None:
            dist.barrier()
        e0.record(stream)
        fn(e2e_steps)
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = max_over_ranks(e0.elapsed_time(e1), dist, device)
        return job_rate(world, work, e2e_steps, ms, 1e9 if decode else 1e12)

    e2e_serial_val = timed(e2e_serial)
    serial_result = [t.clone() for t in host_outs[0]]
    e2e_val = timed(e2e_pipelined)
    # the kernels are deterministic and every step reads the same inputs: the pipelined
    # loop's last result must equal the serial loop's bit for bit
    for x, y in zip(host_outs[(e2e_steps - 1) % 2], serial_result):
        if not torch.equal(x, y):
            raise RuntimeError("pipelined end-to-end result differs from the serial one")
    del S1, sets, serial_result

    kernel_name = (("decode_v1_split_kernel" if inp.variant == 1 else "decode_split_kernel")
                   if decode else f"prefill_v{inp.variant}_kernel")
    traffic = measured_traffic(kernel_name, inp.name, inp.B, decode)
    # the bytes the kernel must move at least: its inputs read once and its output written
    # once (prefill), the caches read once (decode)
    algo_bytes = (work if decode else
                  float(in_bytes + out.numel() * out.element_size()))
    if backward:
        # the timed span is the whole backward call (its four launches)
        kernel_name = (f"prefill_v{inp.variant}_kernel (statistics mode) + bwd_v2_dkdv_kernel + "
                       "bwd_v2_dq_kernel + bwd_dlambda_kernel")
        traffic = None
    line = {
        "metric": metric,
        "value": round(value, 3),
        "unit": unit,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded numpy PCG64, bf16-rounded; shapes and distributions of the workload)",
        "config": workload_config(inp, world),
        "tokens_per_s": round(world * inp.B * (1 if decode else inp.N) * args.steps / (total_ms * 1e-3), 1),
        "roofline": {
            "bound": bound, "achieved": round(achieved, 3), "peak": peak, "unit": runit,
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "traffic_over_algorithmic": (round(traffic / algo_bytes, 3)
                                         if traffic and algo_bytes else None),
            "peak_source": f"{peaks['source']} ({'burst bf16' if bound == 'tensor' else 'HBM copy'})",
            "kernel": (kernel_name + (" + decode_v1_combine_kernel" if inp.variant == 1 else
                                      " + decode_combine_kernel") if decode else kernel_name),
            "avg_kernel_ms": round(kern_avg, 5),
            **({"frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4),
                "sustained_peak": peaks["bf16_tflops_sustained"]} if bound == "tensor" else {}),
        },
        "e2e": {"value": round(e2e_val, 3), "unit": unit, "h2d_bytes_per_step": int(h2d),
                "d2h_bytes_per_step": int(d2h), "steps": e2e_steps,
                "overlap": "step i on one of two device buffer sets while step i+1's inputs are "
                           "copied in and step i-1's result copied out on two copy streams",
                "serial_value": round(e2e_serial_val, 3)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "wall_s_timed": round(t_wall, 4),
    }
    S0.clear()  # the step closures keep the dict; release its tensors before the secondaries
    del q, k, v, out, S0
    if backward:
        del dy, grads
    if paged:
        del kp, vp, bt
    torch.cuda.empty_cache()
    if not args.no_secondary and args.workload == "c5":
        line["secondary"] = secondary(device, peaks, torch, da)
    return line


def _timed(fn, torch, reps=10, warm=3):
    """Median CUDA-event time (ms) of `fn` on the current stream over `reps` calls."""
    for _ in range(warm):
        fn()
    es = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in es:
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in es)


def secondary(device, peaks, torch, da):
    """Other rows of the hot path, each timed alone (median of 10 launches):
      * the V1 bf16 layer (B=2, 16 heads, N=4096, d=64), its backward (tensor cores; and
        widened to fp32 through the exact kernels, median of 3), and the V2 prefill
        (N=16384, 64/8 heads, d=128) on their seeded synth tensors, lambda from the lambda
        kernel; the
        V2 tensors also as a 4096-key sliding-window layer and as a 2048-query chunk, and
        the V2 backward on the seeded N=4096 backward workload;
      * the V2 decode (batch 64, cache 32768; contiguous and over 16/256-token pages) and
        the V1 decode (batch 32, cache 32768, 16 heads, d=64) on same-shape seeded N(0,1)
        draws made on the device (the synth caches take minutes to draw on the host), with
        the synth lambda vectors.
    TFLOP/s against the measured bf16 peak, GB/s against the measured copy bandwidth."""
    from differential_attention_05_b200 import synth
    res = {}
    tflops = lambda fl, ms: {"ms": round(ms, 4), "TFLOP/s": round(fl / ms / 1e9, 2),
                             "frac_of_bf16_peak": round(fl / ms / 1e9 / peaks["bf16_tflops"], 4)}
    gbs = lambda by, ms: {"ms": round(ms, 4), "GB/s": round(by / ms / 1e6, 1),
                          "frac_of_hbm": round(by / ms / 1e6 / peaks["hbm_gbs"], 4)}

    def dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)

    def lam_of(vecs, depth):
        lam = torch.empty(vecs[0].shape[0], dtype=torch.float32, device=device)
        li = torch.empty(1, dtype=torch.float32, device=device)
        da.diffattn_lambda(*[dev(x) for x in vecs], depth=depth, lambda_out=lam, lambda_init_out=li)
        return lam, li

    seeded = "seeded synth tensors"
    # ---- V1 layer
    inp = synth.config2()
    q, k, v = dev(inp.q), dev(inp.k), dev(inp.v)
    lam, li = lam_of((inp.lq1, inp.lk1, inp.lq2, inp.lk2), inp.depth)
    out = torch.empty((inp.B, inp.N, inp.H, 2 * inp.d), dtype=torch.bfloat16, device=device)
    ms = _timed(lambda: da.diffattn_fwd_prefill(q, k, v, lam, li, out=out, apply_norm=True,
                                                norm_eps=inp.eps), torch)
    res["v1_layer"] = {"workload": inp.name, "inputs": seeded, **tflops(prefill_flops(inp), ms)}
    # its backward: bf16 on the tensor cores, and the same values widened to fp32 through the
    # exact-fp32 kernels. Algorithmic FLOPs per attended (query, key) pair and head: scores
    # 2 x 2d, dP = dO V^T 4d (V is 2d wide), dV 4d, dK_1 + dK_2 4d, dQ_1 + dQ_2 4d: 20 d
    bwd_flops = 20.0 * inp.d * inp.H * inp.B * visible_pairs(inp.N, inp.N)
    dy = dev(synth.grad_out((inp.B, inp.N, inp.H, 2 * inp.d), 1001))
    grads = (torch.empty(q.shape, dtype=torch.float32, device=device),
             torch.empty(k.shape, dtype=torch.float32, device=device),
             torch.empty(v.shape, dtype=torch.float32, device=device),
             torch.empty(lam.shape, dtype=torch.float32, device=device))
    ms = _timed(lambda: da.diffattn_bwd_prefill(q, k, v, lam, dy, li, apply_norm=True,
                                                norm_eps=inp.eps, grads=grads), torch)
    res["v1_backward"] = {"workload": inp.name + " backward", "inputs": seeded,
                          "path": "tensor cores", **tflops(bwd_flops, ms)}
    q32, k32, v32, dy32 = q.float(), k.float(), v.float(), dy.float()
    ms = _timed(lambda: da.diffattn_bwd_prefill(q32, k32, v32, lam, dy32, li, apply_norm=True,
                                                norm_eps=inp.eps, grads=grads), torch, reps=3, warm=1)
    res["v1_backward_exact_fp32"] = {
        "workload": inp.name + " backward, inputs widened to fp32", "inputs": seeded,
        "path": "exact-fp32 SIMT kernels", **tflops(bwd_flops, ms)}
    del q, k, v, out, dy, q32, k32, v32, dy32, grads
    # ---- V2 prefill, its window and chunk forms
    inp = synth.config3()
    q, k, v = dev(inp.q), dev(inp.k), dev(inp.v)
    lam, li = lam_of((inp.lq1, inp.lk1, inp.lq2, inp.lk2), inp.depth)
    N, Hq, Hkv, d = inp.N, inp.H, inp.Hkv, inp.d
    out = torch.empty((1, N, Hq // 2, d), dtype=torch.bfloat16, device=device)
    ms = _timed(lambda: da.diffattn_fwd_prefill(q, k, v, lam, out=out), torch)
    res["v2_prefill"] = {"workload": inp.name, "inputs": seeded, **tflops(prefill_flops(inp), ms)}
    # the same tensors as a sliding-window layer (4096 keys) and as a 2048-query chunk at
    # the end of the 16384-key context; FLOPs count the attended pairs only
    for name, Nq, window in (("v2_prefill_window4096", N, 4096), ("v2_prefill_chunk2048", 2048, 0)):
        qq, oo = q[:, N - Nq:], out[:, N - Nq:]
        ms = _timed(lambda: da.diffattn_fwd_prefill(qq, k, v, lam, out=oo, window=window), torch)
        res[name] = {"workload": inp.name, "inputs": seeded, "queries": Nq, "keys": N,
                     "window": window, **tflops(4.0 * d * Hq * visible_pairs(Nq, N, True, window), ms)}
    del q, k, v, out, qq, oo
    # ---- V2 backward; algorithmic FLOPs per attended (query head, key) pair: 8 d (scores
    # 2d, dP d per head, dQ 2d, dK 2d, dV d). The training path: the forward that saves
    # O_2 / l_2 and the log-sum-exps (timed as its own line), then the backward from them
    # (statistics rows, dK/dV, dQ, dlambda sum); and the backward that recomputes the
    # statistics with a forward pass of its own.
    inp = synth.v2_backward()
    q, k, v, dy = dev(inp.q), dev(inp.k), dev(inp.v), dev(inp.extra["dy"])
    lam, li = lam_of((inp.lq1, inp.lk1, inp.lq2, inp.lk2), inp.depth)
    bwd_flops = 8.0 * inp.d * inp.H * visible_pairs(inp.N, inp.N)
    o, o2, lse = da.diffattn_fwd_prefill_train(q, k, v, lam)
    ms = _timed(lambda: da.diffattn_fwd_prefill_train(q, k, v, lam, out=o, o2=o2, lse=lse), torch)
    res["v2_forward_train_n4096"] = {"workload": inp.name, "inputs": seeded,
                                     "writes": "out, O_2 / l_2, log-sum-exps",
                                     **tflops(4.0 * inp.d * inp.H * visible_pairs(inp.N, inp.N), ms)}
    grads = tuple(torch.empty(t.shape, dtype=torch.float32, device=device) for t in (q, k, v)) + (
        torch.empty(lam.shape, dtype=torch.float32, device=device),)
    ms = _timed(lambda: da.diffattn_bwd_prefill_saved(q, k, v, lam, o, o2, lse, dy, grads=grads), torch)
    res["v2_backward_n4096"] = {"workload": inp.name, "inputs": seeded,
                                "path": "from the training forward's saved outputs", **tflops(bwd_flops, ms)}
    ms = _timed(lambda: da.diffattn_bwd_prefill(q, k, v, lam, dy, grads=grads), torch)
    res["v2_backward_recompute_n4096"] = {"workload": inp.name, "inputs": seeded,
                                          "path": "statistics recomputed by a forward pass",
                                          **tflops(bwd_flops, ms)}
    del q, k, v, dy, o, o2, lse, grads
    torch.cuda.empty_cache()
    # ---- V2 decode: same-shape draws on the device
    g = torch.Generator(device=device)
    g.manual_seed(1003)
    drawn = "same-shape seeded N(0,1) draws on the device (torch generator), synth lambda vectors"
    B, L = 64, 32768
    q = torch.randn((B, Hq, d), generator=g, device=device).bfloat16()
    k = torch.randn((B, L, Hkv, d), generator=g, device=device).bfloat16()
    v = torch.randn((B, L, Hkv, d), generator=g, device=device).bfloat16()
    lam, _ = lam_of(synth.lambda_vectors(1003, Hq // 2, d), 24)
    out = torch.empty((B, Hq // 2, d), dtype=torch.bfloat16, device=device)
    p = da._binding.decode_params(q, k, v, out)
    ws = torch.empty(da._binding.diffattn_decode_workspace_size(p), dtype=torch.uint8, device=device)
    by = decode_bytes(B, L, Hkv, d)
    ms = _timed(lambda: da.diffattn_fwd_decode(q, k, v, lam, out=out, workspace=ws), torch)
    res["decode"] = {"workload": "v2_bf16_decode_b64_l32768_hq64_hkv8_d128", "inputs": drawn,
                     **gbs(by, ms)}
    # the same cache as a page pool: 16-token pages in a shuffled order (block table), the
    # same pages in order (the paging arithmetic alone), 256-token pages shuffled
    for ps, shuffled in ((16, True), (16, False), (256, True)):
        kp, vp = k.view(B * L // ps, ps, Hkv, d), v.view(B * L // ps, ps, Hkv, d)
        ids = (torch.randperm(B * L // ps, generator=g, device=device) if shuffled
               else torch.arange(B * L // ps, device=device))
        bt = ids.to(torch.int32).view(B, L // ps)
        ms = _timed(lambda: da.diffattn_fwd_decode_paged(q, kp, vp, bt, lam, out=out, workspace=ws),
                    torch)
        res[f"decode_paged{ps}_{'shuffled' if shuffled else 'in_order'}"] = {
            "workload": f"v2_bf16_decode_b64_l32768_hq64_hkv8_d128, {ps}-token pages, "
                        f"{'shuffled' if shuffled else 'in-order'} block table",
            "inputs": drawn, **gbs(by, ms)}
    del q, k, v, out, ws, kp, vp, bt
    torch.cuda.empty_cache()
    # ---- V1 decode: batch 32, cache 32768, 16 heads, d = 64 (the V2 decode's cache bytes)
    B, L, H, d1 = 32, 32768, 16, 64
    q = (torch.randn((B, H, 2, d1), generator=g, device=device) / 8).bfloat16()
    k = (torch.randn((B, L, H, 2, d1), generator=g, device=device) / 8).bfloat16()
    v = (torch.randn((B, L, H, 2 * d1), generator=g, device=device) / 8).bfloat16()
    lam1, li = lam_of(synth.lambda_vectors(1006, H, d1), 12)
    out = torch.empty((B, H, 2 * d1), dtype=torch.bfloat16, device=device)
    p = da._binding.decode_params_v1(q, k, v, out)
    ws = torch.empty(da._binding.diffattn_decode_workspace_size(p), dtype=torch.uint8, device=device)
    ms = _timed(lambda: da.diffattn_fwd_decode_v1(q, k, v, lam1, li, out=out, workspace=ws), torch)
    res["decode_v1"] = {"workload": "v1_bf16_decode_b32_l32768_h16_d64", "inputs": drawn,
                        **gbs(decode_bytes(B, L, H, 2 * d1), ms)}
    del q, k, v, out, ws
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------------------
# the oracle, timed on the host cores (cpu_baseline and the reference arm)

class OracleRows:
    """The oracle on chosen query rows of a prefill workload; inputs converted to float64
    once, the oracle call itself is what gets timed."""

    def __init__(self, inp):
        import oracle
        from differential_attention_05_b200 import synth
        self.inp = inp
        self.lam = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
        self.li = oracle.lambda_init(inp.depth)
        self.k, self.v = inp.as_f64("k"), inp.as_f64("v")
        self._q = (lambda rows: synth.bf16_to_f32(inp.q[:, rows]).astype(np.float64)) \
            if inp.q.dtype == np.uint16 else (lambda rows: inp.q[:, rows].astype(np.float64))
        self.units = inp.B * (inp.H if inp.variant == 1 else inp.H // 2)
        self.per_pair = 12 * inp.d if inp.variant == 1 else 8 * inp.d  # flops per (i, j) per unit

    def flops(self, rows):
        inp = self.inp
        return float(sum((r + 1) if inp.causal else inp.N for r in rows)) * self.per_pair * self.units

    def run(self, rows):
        import oracle
        inp, qr = self.inp, self._q(rows)
        if inp.variant == 1:
            return oracle.prefill_v1(None, self.k, self.v, self.lam, self.li, causal=inp.causal,
                                     apply_norm=inp.apply_norm, eps=inp.eps, rows=rows, q_rows=qr)
        return oracle.prefill_v2(None, self.k, self.v, self.lam, causal=inp.causal, rows=rows,
                                 q_rows=qr)

    def sample(self, seconds: float, seed: int = 7):
        """Seeded query rows sized so that one oracle call takes about `seconds`."""
        inp = self.inp
        rng = np.random.default_rng(seed)
        n = 8
        for _ in range(3):
            rows = sorted(rng.choice(inp.N, size=min(n, inp.N), replace=False).tolist())
            t0 = time.perf_counter()
            self.run(rows)
            dt = time.perf_counter() - t0
            if dt >= 0.5 * seconds or n >= inp.N:
                break
            n = int(min(inp.N, max(n + 1, n * seconds / max(dt, 1e-3))))
        rows = sorted(np.random.default_rng(seed + 1).choice(inp.N, size=min(n, inp.N),
                                                             replace=False).tolist())
        desc = f"{len(rows)} seeded query rows of every one of the {self.units} units of {inp.name}"
        return rows, desc


def oracle_decode_sample(inp, seconds):
    import oracle
    from differential_attention_05_b200 import synth
    lam = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    t0 = time.perf_counter()
    n = 0
    while True:
        b = n % inp.B
        if inp.variant == 1:
            oracle.decode_v1(synth.bf16_to_f32(inp.q[b:b + 1]), synth.bf16_to_f32(inp.k[b:b + 1]),
                             synth.bf16_to_f32(inp.v[b:b + 1]), lam, oracle.lambda_init(inp.depth),
                             apply_norm=inp.apply_norm, eps=inp.eps)
        else:
            oracle.decode_v2(synth.bf16_to_f32(inp.q[b:b + 1]), synth.bf16_to_f32(inp.k[b:b + 1]),
                             synth.bf16_to_f32(inp.v[b:b + 1]), lam)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    return n, dt


def oracle_backward_sample(inp, seconds):
    """The float64 backward oracle on whole units (a V1 head, a V2 query-head pair; full
    sequence, every key) of a backward workload's first batch entry, unit after unit until
    `seconds` have passed; returns (units, s)."""
    import oracle
    from oracle import backward as OB
    from differential_attention_05_b200 import synth
    lam = oracle.lambda_(inp.lq1, inp.lk1, inp.lq2, inp.lk2, inp.depth)
    f64 = lambda a: synth.bf16_to_f32(a).astype(np.float64)
    group = inp.H // inp.Hkv
    t0 = time.perf_counter()
    n = 0
    while True:
        if inp.variant == 1:
            h = n % inp.H
            OB.prefill_v1_bwd(f64(inp.q[:1, :, h:h + 1]), f64(inp.k[:1, :, h:h + 1]),
                              f64(inp.v[:1, :, h:h + 1]), lam[h:h + 1], oracle.lambda_init(inp.depth),
                              f64(inp.extra["dy"][:1, :, h:h + 1]), causal=inp.causal,
                              apply_norm=inp.apply_norm, eps=inp.eps)
        else:
            p = n % (inp.H // 2)
            g = (2 * p) // group
            OB.prefill_v2_bwd(f64(inp.q[:1, :, 2 * p:2 * p + 2]), f64(inp.k[:1, :, g:g + 1]),
                              f64(inp.v[:1, :, g:g + 1]), lam[p:p + 1],
                              f64(inp.extra["dy"][:1, :, p:p + 1]), causal=inp.causal)
        n += 1
        if time.perf_counter() - t0 >= seconds:
            break
    return n, time.perf_counter() - t0


def backward_flops(inp) -> float:
    """Algorithmic FLOPs of a backward workload: per attended (query, key) pair 20 d per V1
    head (scores 2 x 2d, dP = dO V^T 4d with V 2d wide, dV 4d, dK_1 + dK_2 4d, dQ_1 + dQ_2
    4d) and 8 d per V2 query head (scores 2d, dP d per head, dQ 2d, dK 2d, dV d per head)."""
    per = 20.0 * inp.d if inp.variant == 1 else 8.0 * inp.d
    return per * inp.H * inp.B * visible_pairs(inp.N, inp.N, inp.causal)


def backward_unit_flops(inp) -> float:
    """backward_flops of one unit (V1 head, V2 pair) over one batch entry."""
    return backward_flops(inp) / inp.B / inp.n_units


def cpu_baseline(inp, seconds=12.0):
    import oracle
    cores = oracle.default_threads()
    if "dy" in inp.extra:
        n, dt = oracle_backward_sample(inp, seconds)
        return {"value": round(n * backward_unit_flops(inp) / dt / 1e12, 6), "unit": "TFLOP/s",
                "cores": cores, "kind": "oracle",
                "sample": f"{n} whole {'heads' if inp.variant == 1 else 'query-head pairs'} (every row "
                          f"and key) of {inp.name}, {dt:.1f} s"}
    if inp.mode == "decode":
        n, dt = oracle_decode_sample(inp, seconds)
        val = n * workload_decode_bytes(inp) / inp.B / dt / 1e9
        return {"value": round(val, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                "sample": f"{n} batch entries of {inp.name}, {dt:.1f} s"}
    orc = OracleRows(inp)
    rows, desc = orc.sample(seconds)
    t0 = time.perf_counter()
    orc.run(rows)
    dt = time.perf_counter() - t0
    return {"value": round(orc.flops(rows) / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "sample": f"{desc}, {dt:.1f} s"}


def run_reference(args, rank, world):
    import oracle
    oracle.build()
    inp = workload_inputs(args.workload, args.batch)
    cores = oracle.default_threads()
    decode = inp.mode == "decode"
    per_step_s = max(0.5, min(8.0, 120.0 / max(1, args.steps + args.warmup)))
    if "dy" in inp.extra:
        times = []
        for i in range(args.warmup + args.steps):
            n, dt = oracle_backward_sample(inp, per_step_s)
            if i >= args.warmup:
                times.append((n, dt))
        total_units = sum(n for n, _ in times)
        total_s = sum(dt for _, dt in times)
        value = total_units * backward_unit_flops(inp) / total_s / 1e12
        unit, metric = "TFLOP/s", "diff-attn backward TFLOP/s (% bf16 peak)"
        sample = (f"whole {'heads' if inp.variant == 1 else 'query-head pairs'} of {inp.name} "
                  f"({total_units} in {total_s:.1f} s)")
    elif decode:
        times = []
        for i in range(args.warmup + args.steps):
            n, dt = oracle_decode_sample(inp, per_step_s)
            if i >= args.warmup:
                times.append((n, dt))
        total_units = sum(n for n, _ in times)
        total_s = sum(dt for _, dt in times)
        value = total_units * workload_decode_bytes(inp) / inp.B / total_s / 1e9
        unit, metric = "GB/s", "diff-attn decode KV GB/s at 1 B200"
        sample = f"whole batch entries of {inp.name} ({total_units} in {total_s:.1f} s)"
    else:
        orc = OracleRows(inp)
        rows, desc = orc.sample(per_step_s)
        flops = orc.flops(rows)
        ts = []
        for i in range(args.warmup + args.steps):
            t0 = time.perf_counter()
            orc.run(rows)
            if i >= args.warmup:
                ts.append(time.perf_counter() - t0)
        total_s = sum(ts)
        value = flops * len(ts) / total_s / 1e12
        unit, metric = "TFLOP/s", "diff-attn prefill TFLOP/s (% bf16 peak)"
        sample = desc
    ms_per_step = 1e3 * total_s / args.steps
    return {
        "impl": "reference",
        "metric": metric, "value": round(value, 6), "unit": unit, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded numpy PCG64, bf16-rounded; shapes and distributions of the workload)",
        "config": workload_config(inp, world),
        "cpu_baseline": {"value": round(value, 6), "unit": unit, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": unit, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


# ---------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", choices=("c2", "c3", "c4", "c5", "d1", "b1", "b3", "p4"), default="c5")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--batch", type=int, default=0,
                    help="decode workload only: smaller batch (profiling runs)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the oracle timing (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # the oracle runs on the host of rank 0 only; other ranks have nothing to do
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args, rank, world)), flush=True)
        return 0

    import torch
    from datetime import timedelta

    device = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group("nccl", rank=rank, world_size=world, device_id=device,
                                timeout=timedelta(seconds=300))
    try:
        line = run_ours(args, rank, world, device)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            inp = workload_inputs(args.workload, args.batch)
            line["cpu_baseline"] = cpu_baseline(inp, args.cpu_seconds)
        elif rank == 0:
            line["cpu_baseline"] = None
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
