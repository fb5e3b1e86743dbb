#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer on B200.

One step = forward + backward of the Llama-7B-shaped q_proj workload
(X [4096 tokens, 4096] bf16, W 4096x4096 in NF4 with double quantization,
LoRA r = 16, alpha = 32): qlora_linear_fwd then qlora_linear_bwd through the
C ABI, all inputs resident in HBM.  The metric is algorithmic TFLOP/s
(4MNK + 6Mr(K+N) per step; no gradient for W).  L2 is flushed between timed
steps (a 256 MB write, then a 256 MB read so that no dirty lines are left to
be written back inside the timed region); each step is timed with CUDA events on the launching
stream and the per-step times are summed.

Also reported: the fused dequant-GEMM kernel against the tensor-core roofline
(events around each launch), the decode GEMV weight stream (70B-shaped up
projection, 1/4/16 tokens) and nf4_quantize against HBM bandwidth, an
fwd + bwd of the 7B MLP and 70B decoder-layer projections and the 2048 x 2048
forward at 128 tokens (with a dense torch bf16 matmul of each forward shape as a
library ceiling), an
end-to-end number with host buffers (pinned host -> device copies of X and dY,
device -> host copies of Y, dX, dA, dB of every step inside the timed region,
pipelined across steps on copy streams), SM clocks
sampled through NVML during the timed region, and the CPU oracle timed on the
host cores on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs the same step on its
own tokens (weak scaling) and the adapter gradients dA, dB are all-reduced
over NCCL each step, as data-parallel training of the adapters requires.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 weight-stream GB/s on 1 B200; % roofline"
WORKLOAD = "qproj_7b"


class L2Flush:
    """Evicts L2 (126 MB on B200) between timed steps: writes one 256 MB
    buffer, then reads another, so the timed step starts with a cold L2 that
    holds no dirty lines (a write-only flush leaves ~126 MB of dirty lines,
    whose write-back would land inside the timed region)."""

    def __init__(self, dev):
        import torch
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.w.zero_()
        torch.sum(self.r, 0, out=self.out)


def gemm_traffic():
    """DRAM bytes (read + write) per fused-GEMM launch, from the committed ncu
    summary of this workload -- but only while the kernel source is the one the
    counters were taken on (its sha256 prefix is recorded in the summary)."""
    import hashlib
    import re
    here = os.path.dirname(os.path.abspath(__file__))
    try:
        text = open(os.path.join(here, "profiles", "k_nf4_gemm_qproj_7b.md")).read()
        src = open(os.path.join(here, "bit_nf4_quantized_24_b200", "csrc", "gemm_tc.cu"), "rb").read()
    except OSError:
        return None
    sha = re.search(r"gemm_tc\.cu`, sha256 prefix ([0-9a-f]{16})", text)
    val = re.search(r"traffic_bytes_per_launch: (\d+)", text)
    if not sha or not val or hashlib.sha256(src).hexdigest()[:16] != sha.group(1):
        return None
    return int(val.group(1))


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def step_flops(M, N, K, r):
    return 4 * M * N * K + 6 * M * r * (K + N)


# ------------------------------------------------------------------ clocks


class ClockSampler:
    """Polls SM clock and throttle reasons of one GPU through NVML (read only)."""

    def __init__(self, torch_device_index: int, period_s: float = 0.005):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self.ok = False
        self.period = period_s
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode() if isinstance(uuid, str) else uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        names = {
            "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
            "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
            "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for n, bit in names.items():
                    if mask & bit and n not in ("gpu_idle",):
                        self.reasons.add(n)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self._t.join()
        return False

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# -------------------------------------------------------------- CPU oracle


def oracle_prepare():
    """Inputs of the workload for the CPU oracle: drawn on the host, quantized
    and dequantized by the oracle (done once, outside any timed region)."""
    import oracle
    from bit_nf4_quantized_24_b200 import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    p = wl.draw_linear(w)
    N, K = p["N"], p["K"]
    oc, oa, od, _ = oracle.nf4_quantize(p["W"].numpy())
    _, Wp = oracle.nf4_dequantize(oc, oa, od, N, K)
    bits = wl.bf16_bits
    return {"M": p["M"], "N": N, "K": K, "r": p["r"], "scale": p["scale"], "Wp": Wp,
            "X": bits(p["X"]), "A": bits(p["A"]), "B": bits(p["B"]), "dY": bits(p["dY"])}


def oracle_run(prep, rows_sample: int | None = None):
    """Times the CPU oracle on a bounded sample of the workload: Y and dX for
    `rows_sample` token rows, H, dH, dA, dB in full.  Returns (TFLOP/s, cores,
    sample description, seconds)."""
    import numpy as np

    import oracle
    M, N, K, r = prep["M"], prep["N"], prep["K"], prep["r"]
    X, A, B, dY, Wp = prep["X"], prep["A"], prep["B"], prep["dY"], prep["Wp"]
    rows = np.arange(M, dtype=np.int64) if rows_sample is None else np.linspace(0, M - 1, rows_sample).astype(np.int64)
    t0 = time.perf_counter()
    oracle.linear_fwd(X, Wp, A, B, prep["scale"], rows=rows)
    oracle.linear_bwd(X, dY, Wp, A, B, prep["scale"], rows=rows)
    dt = time.perf_counter() - t0
    S = len(rows)
    flops = S * (2 * K * r + 2 * N * K + 2 * N * r)          # forward rows
    flops += 2 * M * K * r + 2 * M * N * r                    # H, dH
    flops += S * (2 * N * K + 2 * r * K)                      # dX rows
    flops += 2 * r * K * M + 2 * N * r * M                    # dA, dB
    desc = (f"{WORKLOAD} (M={M}, N={N}, K={K}, r={r}): Y and dX for {S} of {M} token rows, "
            f"H, dH, dA, dB in full; one fwd+bwd pass of the fp64 oracle")
    return flops / dt / 1e12, oracle.num_threads(), desc, dt


def oracle_sample(rows_sample: int | None = None):
    return oracle_run(oracle_prepare(), rows_sample)


# -------------------------------------------------------------- our arm


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from bit_nf4_quantized_24_b200 import build as qbuild
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if rank == 0:
        qbuild.build()
    if world > 1:
        dist.barrier()
    from bit_nf4_quantized_24_b200 import binding as qb
    from bit_nf4_quantized_24_b200 import dp
    from bit_nf4_quantized_24_b200 import workloads as wl

    pk = peaks()
    w = wl.WORKLOADS[WORKLOAD]
    p = wl.draw_linear(w)
    M, N, K, r, s = p["M"], p["N"], p["K"], p["r"], p["scale"]
    dev = torch.device("cuda", local_rank)
    q = qb.nf4_quantize(p["W"].to(dev))
    X, A, B, dY = (p[k].to(dev) for k in ("X", "A", "B", "dY"))
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
    dA = torch.empty(r, K, dtype=torch.bfloat16, device=dev)
    dB = torch.empty(N, r, dtype=torch.bfloat16, device=dev)
    H = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
    wsf = torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    wsb = torch.empty(qb.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    L = qb.lib()
    import ctypes
    f32 = ctypes.c_float
    P = qb._ptr

    main = {"X": X, "dY": dY, "Y": Y, "dX": dX, "dA": dA, "dB": dB, "H": H, "wsf": wsf, "wsb": wsb}

    def step(b=main):
        st = qb._stream()
        e = L.qlora_linear_fwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(b["X"]), M, P(A), P(B), r, f32(s),
                               P(b["Y"]), P(b["H"]), P(b["wsf"]), b["wsf"].numel(), st)
        if e:
            raise qb.QloraError(e, "fwd")
        e = L.qlora_linear_bwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(b["X"]), P(b["dY"]), M, P(A), P(B),
                               r, f32(s), P(b["H"]), P(b["dX"]), P(b["dA"]), P(b["dB"]), P(b["wsb"]),
                               b["wsb"].numel(), st)
        if e:
            raise qb.QloraError(e, "bwd")
        if world > 1:
            dp.allreduce_adapter_grads(b["dA"], b["dB"])

    # our kernels per step (the ncu launch list shows the same): forward k_rows (H) and
    # k_nf4_gemm; backward k_rows (dH), two k_cols (dA, dB) and k_nf4_gemm (dX)
    launches_per_step = 2 + 4

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    K_steps = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_steps)]
    sampler = ClockSampler(local_rank)
    trace = qb.GemmTrace(2 * K_steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler, trace:
        for i in range(K_steps):
            flush()
            ev[i][0].record()
            step()
            ev[i][1].record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    total_ms = sum(step_ms)
    gemm_ms = trace.times_ms()
    if world > 1:
        t = torch.tensor([total_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        total_ms = float(t.item())
    flops = step_flops(M, N, K, r)
    value = flops * world * K_steps / (total_ms / 1e3) / 1e12

    # dominant kernel: the fused dequant-GEMM, launched twice per step (forward,
    # dX).  The forward launch has the GPU to itself; the dX launch shares it
    # with the dA / dB kernels, which the backward runs on a side stream in the
    # SMs the GEMM's last wave leaves idle, so its event time is not the
    # kernel's own: the roofline uses the forward launches, dx_ms is reported.
    fwd_ms = gemm_ms[0::2]
    bwd_ms = gemm_ms[1::2]
    gemm_flops_fwd = 2 * M * N * K + 2 * M * N * r
    fwd_mean = statistics.mean(fwd_ms) if fwd_ms else float("nan")
    achieved = gemm_flops_fwd / (fwd_mean / 1e3) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16_tflops"], 4), "traffic": gemm_traffic(),
                "kernel": "k_nf4_gemm (fused NF4 dequant + tcgen05 GEMM), forward launches; the dX launch "
                          "overlaps the adapter-gradient kernels (dx_ms)",
                "peak_source": f"{pk['source']} bf16 burst (MEASURED_PEAKS.json)",
                "fwd_ms": round(fwd_mean, 4) if fwd_ms else None,
                "dx_ms": round(statistics.mean(bwd_ms), 4) if bwd_ms else None}

    # End to end through the C ABI with host buffers: every step copies its
    # inputs X, dY from pinned host memory and reads its results Y, dX, dA, dB
    # back, as a training loop does; the copies are pipelined across steps
    # (two device buffer sets; the input copy of step i + 1 and the read-back
    # of step i - 1 run on their own streams while step i computes).
    Xh = p["X"].pin_memory()
    dYh = p["dY"].pin_memory()
    Yh = torch.empty(M, N, dtype=torch.bfloat16).pin_memory()
    dXh = torch.empty(M, K, dtype=torch.bfloat16).pin_memory()
    dAh = torch.empty(r, K, dtype=torch.bfloat16).pin_memory()
    dBh = torch.empty(N, r, dtype=torch.bfloat16).pin_memory()
    second = {k: torch.empty_like(v) for k, v in main.items()}
    sets = (main, second)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    evs = [{k: torch.cuda.Event() for k in ("in", "done", "out")} for _ in sets]

    def e2e_run(n, start_event=None):
        if start_event is not None:
            s_in.wait_event(start_event)
        for i in range(n):
            b, ev = sets[i % 2], evs[i % 2]
            if i >= 2:
                s_in.wait_event(ev["done"])   # step i - 2 has finished reading this set's inputs
            with torch.cuda.stream(s_in):
                b["X"].copy_(Xh, non_blocking=True)
                b["dY"].copy_(dYh, non_blocking=True)
            ev["in"].record(s_in)
            comp.wait_event(ev["in"])
            if i >= 2:
                comp.wait_event(ev["out"])    # step i - 2's results have been read back
            step(b)
            ev["done"].record(comp)
            s_out.wait_event(ev["done"])
            with torch.cuda.stream(s_out):
                Yh.copy_(b["Y"], non_blocking=True)
                dXh.copy_(b["dX"], non_blocking=True)
                dAh.copy_(b["dA"], non_blocking=True)
                dBh.copy_(b["dB"], non_blocking=True)
            ev["out"].record(s_out)
        comp.wait_stream(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    n_e2e = max(3, min(K_steps, 20))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e0.record(comp)
    e2e_run(n_e2e, start_event=e0)
    e1.record(comp)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e = {"value": round(flops * world * n_e2e / (e2e_ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
           "h2d_bytes_per_step": Xh.numel() * 2 + dYh.numel() * 2,
           "d2h_bytes_per_step": (Yh.numel() + dXh.numel() + dAh.numel() + dBh.numel()) * 2,
           "steps": n_e2e, "copies": "pipelined across steps (two device buffer sets, copy streams)"}
    del second, sets

    extra = {}
    if not args.no_extras:
        extra = run_extras(qb, wl, dev, pk, flush)

    status = qb.device_status()
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": K_steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / K_steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; see workloads.py)",
        "config": {"workload": f"{WORKLOAD}: Llama-7B q_proj fwd+bwd, M=4096 tokens (4x1024), N=K=4096, "
                               f"NF4 block 64 + 8-bit double quant (group 256), LoRA r=16 alpha=32",
                   "M": M, "N": N, "K": K, "r": r, "global_batch_tokens": M * world,
                   "parallelism": f"dp{world} (adapter grads all-reduced)" if world > 1 else "single GPU",
                   "l2": "flushed between timed steps (256 MB write, then 256 MB read: cold and clean)"},
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K_steps,
        "clocks": sampler.summary(),
        "extra": extra,
        "device_status": status,
    }
    if rank == 0 and world == 1 and not args.no_cpu:
        tf, cores, desc, dt = oracle_sample()
        out["cpu_baseline"] = {"value": tf, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc,
                               "seconds": round(dt, 2)}
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def run_extras(qb, wl, dev, pk, flush):
    """Decode GEMV weight stream, quantize and dequantize bandwidth."""
    import torch
    res = {}

    def timed(fn, n=20, flush_between=True):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        ts = []
        for _ in range(n):
            if flush_between:
                flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            ts.append((a, b))
        torch.cuda.synchronize()
        return statistics.median([a.elapsed_time(b) for a, b in ts])

    # decode: 70B-shaped up projection, 1 / 4 / 16 tokens
    w = wl.WORKLOADS["decode_70b_up"]
    p = wl.draw_linear(w, M=16)
    Wd = p["W"].to(dev)
    q = qb.nf4_quantize(Wd)
    N, K, r, s = p["N"], p["K"], p["r"], p["scale"]
    weight_bytes = q.codes.numel() + q.absmax_q.numel() + 4 * q.dq_scale.numel()
    A, B = p["A"].to(dev), p["B"].to(dev)
    def graph_time(call):
        """A decode loop issues the call from a CUDA graph: time the replay."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            call()
        torch.cuda.current_stream().wait_stream(side)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        ms = timed(graph.replay)
        del graph
        return ms

    tiles = qb.nf4_decode_tiles(q)
    ms_pack = timed(lambda: qb.nf4_decode_tiles(q, out=tiles), n=10)
    res["nf4_decode_tiles"] = {"ms": round(ms_pack, 4),
                               "gbs": round(2 * q.codes.numel() / ms_pack / 1e6, 1),
                               "note": "one-time rearrangement of the codes for the decode calls"}
    dec, dec_t = {}, {}
    for M in (1, 4, 16):
        X = p["X"][:M].contiguous().to(dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        ws = torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
        total_bytes = weight_bytes + 2 * r * (K + N) + 2 * M * (K + N)
        call = lambda: qb.qlora_linear_fwd(q, X, A, B, s, save_h=False, out=Y, workspace=ws)
        ms = graph_time(call)
        ms_eager = timed(call)
        dec[f"M{M}"] = {"us": round(ms * 1e3, 2), "us_eager_call": round(ms_eager * 1e3, 2),
                        "weight_stream_gbs": round(weight_bytes / ms / 1e6, 1),
                        "total_gbs": round(total_bytes / ms / 1e6, 1),
                        "frac_hbm": round(total_bytes / ms / 1e6 / pk["hbm_gbs"], 4)}
        call_t = lambda: qb.qlora_linear_fwd_tiles(q, tiles, X, A, B, s, save_h=False, out=Y, workspace=ws)
        ms = graph_time(call_t)
        ms_eager = timed(call_t)
        dec_t[f"M{M}"] = {"us": round(ms * 1e3, 2), "us_eager_call": round(ms_eager * 1e3, 2),
                          "weight_stream_gbs": round(weight_bytes / ms / 1e6, 1),
                          "total_gbs": round(total_bytes / ms / 1e6, 1),
                          "frac_hbm": round(total_bytes / ms / 1e6 / pk["hbm_gbs"], 4)}
    res["decode_70b_up"] = dec
    res["decode_70b_up_tiles"] = dec_t
    # multi-adapter decode: 16 tokens spread over 4 adapters (r = 16), graph replay
    na, Mm = 4, 16
    g = torch.Generator().manual_seed(77)
    A_all = ((torch.rand(na, r, K, generator=g) * 2 - 1) / K ** 0.5).bfloat16().to(dev)
    B_all = (torch.randn(na, N, r, generator=g) * 0.01).bfloat16().to(dev)
    sc_all = torch.full((na,), float(s), dtype=torch.float32, device=dev)
    idx = (torch.arange(Mm, dtype=torch.int32) % na).to(dev)
    Xm = p["X"][:Mm].contiguous().to(dev)
    Ym = torch.empty(Mm, N, dtype=torch.bfloat16, device=dev)
    wsm = torch.empty(qb.fwd_workspace_bytes(Mm, N, K, r), dtype=torch.uint8, device=dev)
    mbytes = weight_bytes + 2 * na * r * (K + N) + 2 * Mm * (K + N)
    ms = graph_time(lambda: qb.qlora_linear_fwd_multi(q, Xm, A_all, B_all, sc_all, idx, out=Ym, workspace=wsm))
    res["decode_70b_up_multi_adapter"] = {"tokens": Mm, "adapters": na, "us": round(ms * 1e3, 2),
                                          "total_gbs": round(mbytes / ms / 1e6, 1),
                                          "frac_hbm": round(mbytes / ms / 1e6 / pk["hbm_gbs"], 4)}
    ms = graph_time(lambda: qb.qlora_linear_fwd_multi_tiles(q, tiles, Xm, A_all, B_all, sc_all, idx, out=Ym,
                                                            workspace=wsm))
    res["decode_70b_up_multi_adapter_tiles"] = {"tokens": Mm, "adapters": na, "us": round(ms * 1e3, 2),
                                                "total_gbs": round(mbytes / ms / 1e6, 1),
                                                "frac_hbm": round(mbytes / ms / 1e6 / pk["hbm_gbs"], 4)}
    # quantize of the same weight (4 B read + 0.516 B written per weight)
    numel = N * K
    qbytes = 4 * numel + numel // 2 + numel // 64 + 4 * ((numel // 64 + 255) // 256)
    ms = timed(lambda: qb.nf4_quantize(Wd), n=5)
    res["nf4_quantize"] = {"ms": round(ms, 4), "gbs": round(qbytes / ms / 1e6, 1),
                           "frac_hbm": round(qbytes / ms / 1e6 / pk["hbm_gbs"], 4),
                           "note": "includes the call's stream synchronization (non-finite check)"}
    out = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
    dbytes = numel // 2 + numel // 64 + 4 * ((numel // 64 + 255) // 256) + 2 * numel
    ms = timed(lambda: qb.nf4_dequantize(q, out=out), n=10)
    res["nf4_dequantize"] = {"ms": round(ms, 4), "gbs": round(dbytes / ms / 1e6, 1),
                             "frac_hbm": round(dbytes / ms / 1e6 / pk["hbm_gbs"], 4)}
    # other NF4 formats (block size, double quantization on/off): the codec on
    # the same weight, and the forward of the q_proj workload through the GEMM
    fmts = {}
    for block, dq in ((32, 256), (128, 0), (256, 256)):
        cb, ab, db = qb.nf4_quantized_sizes(N, K, block, dq)
        qf = qb.nf4_quantize(Wd, block, dq)
        ms_q = timed(lambda: qb.nf4_quantize(Wd, block, dq), n=5)
        ms_d = timed(lambda: qb.nf4_dequantize(qf, out=out), n=10)
        fmts[f"b{block}_dq{dq}"] = {
            "quantize_gbs": round((4 * numel + cb + ab + db) / ms_q / 1e6, 1),
            "dequantize_gbs": round((cb + ab + db + 2 * numel) / ms_d / 1e6, 1)}
        del qf
    w2 = wl.WORKLOADS[WORKLOAD]
    p2 = wl.draw_linear(w2)
    W2, X2, A2, B2 = p2["W"].to(dev), p2["X"].to(dev), p2["A"].to(dev), p2["B"].to(dev)
    M2, N2, K2, r2 = p2["M"], p2["N"], p2["K"], p2["r"]
    Y2 = torch.empty(M2, N2, dtype=torch.bfloat16, device=dev)
    ws2 = torch.empty(qb.fwd_workspace_bytes(M2, N2, K2, r2), dtype=torch.uint8, device=dev)
    flops = 2 * M2 * N2 * K2 + 2 * M2 * r2 * (K2 + N2)
    for block, dq in ((64, 256), (32, 256), (128, 0), (256, 256)):
        qf = qb.nf4_quantize(W2, block, dq)
        ms_f = timed(lambda: qb.qlora_linear_fwd(qf, X2, A2, B2, p2["scale"], save_h=False, out=Y2, workspace=ws2),
                     n=10)
        fmts.setdefault(f"b{block}_dq{dq}", {})["qproj_fwd_tflops"] = round(flops / ms_f / 1e9, 1)
        del qf
    res["formats"] = fmts
    # q_proj fwd + bwd with LoRA dropout (p = 0.1, mask drawn once on the host)
    dY2 = torch.randn(M2, N2, generator=torch.Generator().manual_seed(5)).bfloat16().to(dev)
    q2 = qb.nf4_quantize(W2)
    mk = (torch.rand(M2, K2, generator=torch.Generator().manual_seed(6)) >= 0.1).to(torch.uint8).to(dev)
    keep = 1.0 / 0.9
    wsd = torch.empty(qb.dropout_workspace_bytes(M2, N2, K2, r2), dtype=torch.uint8, device=dev)

    def drop_step():
        _, Hd = qb.qlora_linear_fwd_dropout(q2, X2, A2, B2, p2["scale"], mk, keep, out=Y2, workspace=wsd)
        qb.qlora_linear_bwd_dropout(q2, X2, dY2, A2, B2, p2["scale"], mk, keep, H=Hd, workspace=wsd)

    ms_d = timed(drop_step, n=10)
    res["qproj_fwd_bwd_lora_dropout"] = {"ms": round(ms_d, 4),
                                         "tflops": round((4 * M2 * N2 * K2 + 6 * M2 * r2 * (K2 + N2)) / ms_d / 1e9, 1)}
    del q2, dY2, mk, wsd
    # merge of the decode weight with its r = 16 adapter, quantized again
    # (reads codes + scales + A + B, writes codes + scales)
    mbytes = weight_bytes * 2 + 2 * r * (K + N)
    ms_m = timed(lambda: qb.nf4_merge_lora(q, A, B, s), n=5)
    res["nf4_merge_lora"] = {"ms": round(ms_m, 4), "gbs": round(mbytes / ms_m / 1e6, 1),
                             "frac_hbm": round(mbytes / ms_m / 1e6 / pk["hbm_gbs"], 4),
                             "note": "includes the call's stream synchronization (non-finite check)"}
    del Wd, out, W2, X2, Y2
    torch.cuda.empty_cache()
    res["configs"] = run_configs(qb, wl, dev, pk, timed)
    return res


def run_configs(qb, wl, dev, pk, timed):
    """The other configurations: the 2048 x 2048 forward at 128 tokens
    (latency-bound, in us), and fwd + bwd of every projection of the 7B MLP and
    of the 70B decoder layer against the tensor roofline (and the one-time
    quantize of the layer's seven weights).  Timing inputs of the same shapes
    and distributions are drawn on the device (parity of these shapes is in
    the GPU tests).  Beside each projection: a dense torch bf16 matmul of the
    forward shape on the dequantized weight, as a library ceiling."""
    import ctypes

    import torch
    L = qb.lib()
    P = qb._ptr
    f32 = ctypes.c_float
    out = {}
    g = torch.Generator(device=dev)
    for name in ("fwd_2048", "mlp_7b", "layer_70b"):
        w = wl.WORKLOADS[name]
        g.manual_seed(1000 + w.seed)
        M, r, s = w.M, w.r, w.scale
        per, tot_ms, tot_flops, q_ms = {}, 0.0, 0, 0.0
        for pr in w.projections:
            N, K = pr.N, pr.K
            W = torch.randn(N, K, device=dev, generator=g) * w.w_std
            q_ms += timed(lambda: qb.nf4_quantize(W), n=3)
            q = qb.nf4_quantize(W)
            del W
            X = torch.randn(M, K, device=dev, generator=g).bfloat16()
            A = ((torch.rand(r, K, device=dev, generator=g) * 2 - 1) / K ** 0.5).bfloat16()
            B = (torch.randn(N, r, device=dev, generator=g) * w.b_std).bfloat16()
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            H = torch.empty(M, r, dtype=torch.bfloat16, device=dev)
            wsf = torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
            if w.backward:
                dY = torch.randn(M, N, device=dev, generator=g).bfloat16()
                wsb = torch.empty(qb.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)
                dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
                dA = torch.empty(r, K, dtype=torch.bfloat16, device=dev)
                dB = torch.empty(N, r, dtype=torch.bfloat16, device=dev)

                def step():  # as the headline step: H saved by the forward, read by the backward
                    st = qb._stream()
                    e = L.qlora_linear_fwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(X), M, P(A), P(B), r,
                                           f32(s), P(Y), P(H), P(wsf), wsf.numel(), st)
                    if e == 0:
                        e = L.qlora_linear_bwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(X), P(dY), M, P(A),
                                               P(B), r, f32(s), P(H), P(dX), P(dA), P(dB), P(wsb), wsb.numel(), st)
                    if e:
                        raise qb.QloraError(e, "configs step")
                flops = 4 * M * N * K + 6 * M * r * (K + N)
            else:
                def step():
                    e = L.qlora_linear_fwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(X), M, P(A), P(B), r,
                                           f32(s), P(Y), None, P(wsf), wsf.numel(), qb._stream())
                    if e:
                        raise qb.QloraError(e, "configs fwd")
                flops = 2 * M * N * K + 2 * M * r * (K + N)
            ms = timed(step, n=10)
            Wd = qb.nf4_dequantize(q)
            ms_c = timed(lambda: torch.matmul(X, Wd.t()), n=10)
            per[pr.name] = {"N": N, "K": K, "ms": round(ms, 4), "tflops": round(flops / ms / 1e9, 1),
                            "torch_bf16_matmul_fwd_tflops": round(2 * M * N * K / ms_c / 1e9, 1)}
            tot_ms += ms
            tot_flops += flops
            del q, X, A, B, Y, H, wsf, Wd
            if w.backward:
                del dY, wsb, dX, dA, dB
            torch.cuda.empty_cache()
        entry = {"M": M, "r": r, "pass": "fwd+bwd" if w.backward else "fwd", "ms": round(tot_ms, 4),
                 "tflops": round(tot_flops / tot_ms / 1e9, 1),
                 "frac_tensor": round(tot_flops / tot_ms / 1e9 / pk["bf16_tflops"], 4),
                 "quantize_ms": round(q_ms, 4), "projections": per}
        if name == "fwd_2048":
            entry["us"] = round(tot_ms * 1e3, 1)
        out[name] = entry
    return out


# -------------------------------------------------------- reference arm


def run_reference(args, rank, world):
    """The reference arm is the CPU oracle (this method has no runnable
    reference implementation): it is timed as it stands on the host cores,
    W untimed and K timed steps, each step one bounded sample of the workload
    (the row count of a sample shrinks only if the whole run would otherwise
    take more than about 150 s)."""
    if rank != 0:
        return
    prep = oracle_prepare()
    rows = 512
    n_total = max(1, args.warmup + args.steps)
    budget_s = 150.0
    cores = desc = None
    for i in range(args.warmup):
        _, cores, desc, dt = oracle_run(prep, rows)
        if i == 0 and dt * n_total > budget_s:
            rows = max(32, int(rows * budget_s / (dt * n_total)) // 32 * 32)
    vals = []
    for _ in range(max(1, args.steps)):
        tf, cores, desc, dt = oracle_run(prep, rows)
        vals.append(tf)
    v = statistics.median(vals)
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
           "steps": len(vals), "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; see workloads.py)",
           "config": {"workload": f"{WORKLOAD} (bounded sample, see cpu_baseline.sample)"},
           "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": cores, "kind": "oracle", "sample": desc},
           "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def run_profile(args):
    """A few launches of one kernel on one workload, for ncu captures."""
    import torch

    from bit_nf4_quantized_24_b200 import binding as qb
    from bit_nf4_quantized_24_b200 import build as qbuild
    from bit_nf4_quantized_24_b200 import workloads as wl
    qbuild.build()
    dev = torch.device("cuda", 0)
    w = wl.WORKLOADS[args.workload]
    M = args.tokens if args.tokens else None
    p = wl.draw_linear(w, 0, M=M, with_dy=args.profile in ("bwd", "step"))
    q = qb.nf4_quantize(p["W"].to(dev))
    X, A, B = p["X"].to(dev), p["A"].to(dev), p["B"].to(dev)
    dY = p["dY"].to(dev) if "dY" in p else None
    tiles = qb.nf4_decode_tiles(q) if args.profile == "fwd_tiles" else None
    for _ in range(args.warmup + args.steps):
        if args.profile == "fwd_tiles":
            qb.qlora_linear_fwd_tiles(q, tiles, X, A, B, p["scale"])
        if args.profile in ("fwd", "step"):
            _, H = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
        if args.profile in ("bwd", "step"):
            qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"])
        if args.profile == "quantize":
            qb.nf4_quantize(p["W"].to(dev))
        if args.profile == "dequantize":
            qb.nf4_dequantize(q)
    torch.cuda.synchronize()
    assert qb.device_status() == 0
    print(f"profile {args.profile} {args.workload} M={p['M']} N={p['N']} K={p['K']} done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip decode/quantize measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--profile", choices=["fwd", "fwd_tiles", "bwd", "step", "quantize", "dequantize"],
                    help="run only warmup+steps launches of one entry point (for ncu)")
    ap.add_argument("--workload", default=WORKLOAD, help="workload for --profile")
    ap.add_argument("--tokens", type=int, default=0, help="token count for --profile (default: the workload's)")
    args = ap.parse_args()
    if args.profile:
        run_profile(args)
        return
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
