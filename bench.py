#!/usr/bin/env python
"""Benchmark of the QLoRA NF4 linear layer on B200.

One step = forward + backward of every projection of a 70B-shaped decoder
layer (q, o 8192x8192; k, v 1024x8192; gate, up 28672x8192; down 28672 ->
8192), 4096 tokens, LoRA r = 64, alpha = 16 on all seven, the weights NF4 with
8-bit double quantization (block 64, groups of 256 blocks): the forwards in
layer order, then the backwards in reverse order (each reading the H its
forward saved), through the C ABI, all inputs resident in HBM.  The seven
weights are quantized once, before any step, with nf4_quantize (timed on its
own).  The metric is algorithmic TFLOP/s (4MNK + 6Mr(K+N) per projection; no
gradient for W).  L2 is flushed between timed steps (a 256 MB write, then a
256 MB read, so that no dirty lines are left to be written back inside the
timed region); each step is timed with CUDA events on the launching stream and
the per-step times are summed.

Also reported: the fused dequant-GEMM kernel against the tensor-core roofline
(events around each of its 14 launches per step), the decode GEMV weight stream
(70B-shaped up projection, 1/4/16 tokens) and the NF4 codec against HBM
bandwidth, fwd + bwd of the 7B q_proj and MLP projections and the 2048 x 2048
forward at 128 tokens (with a dense torch bf16 matmul of each forward shape as
a library ceiling), an end-to-end number with host buffers (pinned host ->
device copies of every projection's X and dY, device -> host copies of its Y,
dX, dA, dB, every step, inside the timed region, pipelined across steps on copy
streams), SM clocks sampled through NVML during the timed region, and the CPU
oracle timed on the host cores on a bounded sample (the same layer on fewer
tokens).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one rank per GPU) every rank runs the same step on its
own tokens (weak scaling) and the adapter gradients dA, dB are all-reduced
over NCCL each step, as data-parallel training of the adapters requires.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "QLoRA linear fwd+bwd TFLOP/s and NF4 weight-stream GB/s on 1 B200; % roofline"
WORKLOAD = "layer_70b"

# DRAM bytes (read + write) per traced fused-GEMM launch (the GEMM kernel plus,
# where its tiles are split, the reduction kernel of the partial sums), mean
# over the 14 traced launches of one step of the workload above, from one ncu
# capture of `bench.py --profile layer` (metrics dram__bytes_read.sum,
# dram__bytes_write.sum; the summary and the command are in
# profiles/layer_70b_step_launch_list.md).  Valid only for the kernel source it
# was taken on (sha256 prefix of gemm_tc.cu); reported as null otherwise.
GEMM_TRAFFIC = {"gemm_tc_sha16": "fa327ba0a3245d6e", "bytes_per_launch": 509550610}


def gemm_traffic():
    path = os.path.join(ROOT, "bit_nf4_quantized_24_b200", "csrc", "gemm_tc.cu")
    try:
        sha = hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    if GEMM_TRAFFIC["gemm_tc_sha16"] != sha:
        return None
    return GEMM_TRAFFIC["bytes_per_launch"]


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


def layer_flops(w, M=None):
    M = w.M if M is None else M
    return sum(step_flops(M, pr.N, pr.K, w.r) for pr in w.projections)


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


def draw_layer_host(w):
    """The workload's seeded inputs, one dict per projection, on the host."""
    from bit_nf4_quantized_24_b200 import workloads as wl
    return [wl.draw_linear(w, i) for i in range(len(w.projections))]


def oracle_layer_prepare(w, host=None):
    """Per projection: the oracle's own NF4 quantization and dequantization of
    the fp32 weight, and the bf16 bits of X, A, B, dY (done once, untimed)."""
    import oracle
    from bit_nf4_quantized_24_b200 import workloads as wl
    host = draw_layer_host(w) if host is None else host
    bits = wl.bf16_bits
    prep = []
    for p in host:
        N, K = p["N"], p["K"]
        oc, oa, od, _ = oracle.nf4_quantize(p["W"].numpy())
        _, Wp = oracle.nf4_dequantize(oc, oa, od, N, K)
        prep.append({"N": N, "K": K, "Wp": Wp, "X": bits(p["X"]), "A": bits(p["A"]), "B": bits(p["B"]),
                     "dY": bits(p["dY"]), "scale": p["scale"], "name": p["name"]})
    return prep


def oracle_layer_run(w, prep, tokens: int):
    """Times the CPU oracle on a bounded sample of the workload: the same
    layer (all projections, forward and backward: Y, dX, dA, dB, with H and dH)
    on `tokens` of its token rows, evenly spaced.  Returns (TFLOP/s, cores,
    sample description, seconds)."""
    import numpy as np

    import oracle
    M = w.M
    rows = np.linspace(0, M - 1, tokens).astype(np.int64)
    dt = 0.0
    for pp in prep:
        X, dY = np.ascontiguousarray(pp["X"][rows]), np.ascontiguousarray(pp["dY"][rows])
        t0 = time.perf_counter()
        oracle.linear_fwd(X, pp["Wp"], pp["A"], pp["B"], pp["scale"])
        oracle.linear_bwd(X, dY, pp["Wp"], pp["A"], pp["B"], pp["scale"])
        dt += time.perf_counter() - t0
    flops = layer_flops(w, tokens)
    desc = (f"{w.name}: all {len(prep)} projections, forward and backward (Y, dX, dA, dB) of the fp64 oracle "
            f"on {tokens} of the {M} tokens (evenly spaced rows), r={w.r}; the weights quantized and "
            f"dequantized by the oracle beforehand, untimed")
    return flops / dt / 1e12, oracle.num_threads(), desc, dt


# -------------------------------------------------------------- our arm


class Layer:
    """Device state of the workload: per projection the NF4 weight, the LoRA
    adapter and one buffer set (X, dY, Y, H, dX, dA, dB and workspaces); a step
    runs the forwards in layer order, then the backwards in reverse order,
    through the C ABI on the current stream."""

    def __init__(self, qb, w, host, dev):
        import torch
        self.qb, self.w, self.dev = qb, w, dev
        self.M, self.r, self.s = w.M, w.r, w.scale
        self.projs = []
        for p in host:
            N, K = p["N"], p["K"]
            q = qb.nf4_quantize(p["W"].to(dev))
            self.projs.append({"N": N, "K": K, "q": q, "A": p["A"].to(dev), "B": p["B"].to(dev)})
        torch.cuda.synchronize()

    def new_set(self, host=None):
        import torch
        qb, M, r, dev = self.qb, self.M, self.r, self.dev
        out = []
        for i, pr in enumerate(self.projs):
            N, K = pr["N"], pr["K"]
            b = {"Y": torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                 "H": torch.empty(M, r, dtype=torch.bfloat16, device=dev),
                 "dX": torch.empty(M, K, dtype=torch.bfloat16, device=dev),
                 "dA": torch.empty(r, K, dtype=torch.bfloat16, device=dev),
                 "dB": torch.empty(N, r, dtype=torch.bfloat16, device=dev),
                 "wsf": torch.empty(qb.fwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev),
                 "wsb": torch.empty(qb.bwd_workspace_bytes(M, N, K, r), dtype=torch.uint8, device=dev)}
            if host is not None:
                b["X"] = host[i]["X"].to(dev)
                b["dY"] = host[i]["dY"].to(dev)
            else:
                b["X"] = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
                b["dY"] = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            out.append(b)
        return out

    def step(self, bufs, allreduce=None):
        import ctypes
        qb = self.qb
        L, P, f32 = qb.lib(), qb._ptr, ctypes.c_float
        M, r, s = self.M, self.r, self.s
        st = qb._stream()
        for pr, b in zip(self.projs, bufs):
            q, N, K = pr["q"], pr["N"], pr["K"]
            e = L.qlora_linear_fwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(b["X"]), M, P(pr["A"]),
                                   P(pr["B"]), r, f32(s), P(b["Y"]), P(b["H"]), P(b["wsf"]), b["wsf"].numel(), st)
            if e:
                raise qb.QloraError(e, "fwd")
        for pr, b in reversed(list(zip(self.projs, bufs))):
            q, N, K = pr["q"], pr["N"], pr["K"]
            e = L.qlora_linear_bwd(P(q.codes), P(q.absmax_q), P(q.dq_scale), N, K, P(b["X"]), P(b["dY"]), M,
                                   P(pr["A"]), P(pr["B"]), r, f32(s), P(b["H"]), P(b["dX"]), P(b["dA"]),
                                   P(b["dB"]), P(b["wsb"]), b["wsb"].numel(), st)
            if e:
                raise qb.QloraError(e, "bwd")
            if allreduce is not None:
                allreduce(b["dA"], b["dB"])

    def gemm_launch_flops(self):
        """Algorithmic FLOP of each fused-GEMM launch of a step, in launch
        order: the 7 forwards (2MNK + 2MNr), then the 7 dX GEMMs in reverse
        projection order (2MNK + 2MKr)."""
        M, r = self.M, self.r
        fwd = [2 * M * p["N"] * p["K"] + 2 * M * p["N"] * r for p in self.projs]
        dx = [2 * M * p["N"] * p["K"] + 2 * M * p["K"] * r for p in reversed(self.projs)]
        return fwd + dx


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
    dev = torch.device("cuda", local_rank)
    host = draw_layer_host(w)
    flush = L2Flush(dev)

    # the one-time quantization of the seven weights (4 B read, 0.516 B written per weight)
    Wd = [p["W"].to(dev) for p in host]
    for W in Wd:
        qb.nf4_quantize(W)
    torch.cuda.synchronize()
    flush()
    q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    q0.record()
    for W in Wd:
        qb.nf4_quantize(W)
    q1.record()
    torch.cuda.synchronize()
    quant_ms = q0.elapsed_time(q1)
    numel = sum(W.numel() for W in Wd)
    quant_bytes = sum(4 * W.numel() + W.numel() // 2 + W.numel() // 64 + 4 * ((W.numel() // 64 + 255) // 256)
                      for W in Wd)
    del Wd
    torch.cuda.empty_cache()

    layer = Layer(qb, w, host, dev)
    main = layer.new_set(host)
    allreduce = dp.allreduce_adapter_grads if world > 1 else None
    M, r = w.M, w.r
    flops = layer_flops(w)
    n_proj = len(w.projections)
    # our kernels per step (the ncu launch list shows the same): per projection,
    # forward k_rows (H) and k_nf4_gemm; backward k_rows (dH), two k_cols (dA,
    # dB) and k_nf4_gemm (dX); plus k_split_reduce after each GEMM whose tiles
    # the split plan divides
    launches_per_step = n_proj * (2 + 4) + sum(
        qb.gemm_split_plan(mode, M, pr.N, pr.K)[0] > 1 for pr in w.projections for mode in (0, 1))

    for _ in range(args.warmup):
        layer.step(main, allreduce)
    torch.cuda.synchronize()

    K_steps = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K_steps)]
    sampler = ClockSampler(local_rank)
    trace = qb.GemmTrace(2 * n_proj * K_steps)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler, trace:
        for i in range(K_steps):
            flush()
            ev[i][0].record()
            layer.step(main, allreduce)
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
    value = flops * world * K_steps / (total_ms / 1e3) / 1e12

    # dominant kernel: the fused dequant-GEMM, 14 launches per step (7 forwards,
    # 7 dX).  achieved = algorithmic FLOP of all traced launches / their summed
    # event durations (= mean FLOP per launch / mean launch duration).  The dX
    # launches share the GPU with the adapter-gradient kernels of the side
    # stream, so their event times include that sharing.
    per_launch = layer.gemm_launch_flops()
    nl = len(per_launch)
    cnt = min(len(gemm_ms), nl * K_steps)
    lf = [per_launch[i % nl] for i in range(cnt)]
    gt = gemm_ms[:cnt]
    fwd_idx = [i for i in range(cnt) if i % nl < n_proj]
    dx_idx = [i for i in range(cnt) if i % nl >= n_proj]

    def rate(idx):
        t = sum(gt[i] for i in idx)
        return sum(lf[i] for i in idx) / (t / 1e3) / 1e12 if t > 0 else float("nan")

    achieved = rate(range(cnt))
    names = [p.name for p in w.projections]
    per_proj = {}
    for j, nm in enumerate(names):
        fi = [i for i in fwd_idx if i % nl == j]
        di = [i for i in dx_idx if i % nl == nl - 1 - j]
        per_proj[nm] = {"fwd_ms": round(statistics.mean(gt[i] for i in fi), 4) if fi else None,
                        "fwd_tflops": round(rate(fi), 1) if fi else None,
                        "dx_ms": round(statistics.mean(gt[i] for i in di), 4) if di else None,
                        "dx_tflops": round(rate(di), 1) if di else None}
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / pk["bf16_tflops"], 4),
                "frac_of_sustained": round(achieved / pk["bf16_tflops_sustained"], 4),
                "traffic": gemm_traffic(),
                "kernel": "k_nf4_gemm (fused NF4 dequant + tcgen05 GEMM): all 14 launches of a step, 7 forward and "
                          "7 dX (the dX launches overlap the adapter-gradient kernels on the side stream)",
                "peak_source": f"{pk['source']} bf16 burst (MEASURED_PEAKS.json); sustained "
                               f"{pk['bf16_tflops_sustained']} TFLOP/s quoted beside it",
                "launches_timed": cnt,
                "gemm_ms_per_step": round(sum(gt) / K_steps, 4) if cnt else None,
                "fwd_tflops": round(rate(fwd_idx), 1), "dx_tflops": round(rate(dx_idx), 1),
                "step_tflops": round(value / world, 2),
                "step_frac": round(value / world / pk["bf16_tflops"], 4),
                "step_frac_of_sustained": round(value / world / pk["bf16_tflops_sustained"], 4),
                "per_projection": per_proj}

    # End to end through the C ABI with host buffers: every step copies each
    # projection's X and dY from pinned host memory and reads its Y, dX, dA and
    # dB back, as a training loop does; the copies are pipelined across steps
    # (two device buffer sets; the input copies of step i + 1 and the
    # read-backs of step i - 1 run on their own streams while step i computes).
    hin = [{"X": p["X"].pin_memory(), "dY": p["dY"].pin_memory()} for p in host]
    hout = [{k: torch.empty(tuple(b[k].shape), dtype=torch.bfloat16).pin_memory() for k in ("Y", "dX", "dA", "dB")}
            for b in main]
    second = layer.new_set()
    sets = (main, second)
    comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    evs = [{k: torch.cuda.Event() for k in ("in", "done", "out")} for _ in sets]

    def e2e_run(n, start_event=None):
        if start_event is not None:
            s_in.wait_event(start_event)
        for i in range(n):
            bs, ev_ = sets[i % 2], evs[i % 2]
            if i >= 2:
                s_in.wait_event(ev_["done"])   # step i - 2 has finished reading this set's inputs
            with torch.cuda.stream(s_in):
                for b, h in zip(bs, hin):
                    b["X"].copy_(h["X"], non_blocking=True)
                    b["dY"].copy_(h["dY"], non_blocking=True)
            ev_["in"].record(s_in)
            comp.wait_event(ev_["in"])
            if i >= 2:
                comp.wait_event(ev_["out"])    # step i - 2's results have been read back
            layer.step(bs, allreduce)
            ev_["done"].record(comp)
            s_out.wait_event(ev_["done"])
            with torch.cuda.stream(s_out):
                for b, h in zip(bs, hout):
                    for k in ("Y", "dX", "dA", "dB"):
                        h[k].copy_(b[k], non_blocking=True)
            ev_["out"].record(s_out)
        comp.wait_stream(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    n_e2e = max(3, min(K_steps, 10))
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
    h2d = sum(h["X"].numel() * 2 + h["dY"].numel() * 2 for h in hin)
    d2h = sum(v.numel() * 2 for h in hout for v in h.values())
    e2e = {"value": round(flops * world * n_e2e / (e2e_ms / 1e3) / 1e12, 3), "unit": "TFLOP/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
           "copies": "pipelined across steps (two device buffer sets, copy streams)"}
    del second, sets, hin, hout
    torch.cuda.empty_cache()

    extra = {"nf4_quantize_layer": {"weights": numel, "ms": round(quant_ms, 4),
                                    "gbs": round(quant_bytes / quant_ms / 1e6, 1),
                                    "frac_hbm": round(quant_bytes / quant_ms / 1e6 / pk["hbm_gbs"], 4),
                                    "note": "the seven weights of the layer, once before the steps, through "
                                            "nf4_quantize (each call synchronizes for its non-finite check)"}}
    if not args.no_extras:
        del layer, main
        torch.cuda.empty_cache()
        extra.update(run_extras(qb, wl, dev, pk, flush))

    status = qb.device_status()
    proj_desc = ", ".join(f"{p.name} {p.N}x{p.K}" for p in w.projections)
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": K_steps,
        "warmup": args.warmup, "ms_per_step": round(total_ms / K_steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded; see workloads.py)",
        "config": {"workload": f"{WORKLOAD}: 70B-shaped decoder layer, all 7 projections ({proj_desc}; N x K), "
                               f"forward then backward, M={M} tokens, NF4 block 64 + 8-bit double quant "
                               f"(group 256), LoRA r={r} alpha={w.alpha:g} on every projection",
                   "M": M, "r": r, "global_batch_tokens": M * world, "flop_per_step": flops,
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
        prep = oracle_layer_prepare(w, host)
        tf, cores, desc, dt = oracle_layer_run(w, prep, args.cpu_tokens)
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
    w2 = wl.WORKLOADS["qproj_7b"]
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
    (latency-bound, in us), and fwd + bwd of the 7B q_proj and of every
    projection of the 7B MLP against the tensor roofline (and the one-time
    quantize of their weights).  Timing inputs of the same shapes
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
    for name in ("fwd_2048", "qproj_7b", "mlp_7b"):
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
    reference implementation): it is timed as it stands on the host cores, W
    untimed and K timed steps, each step one bounded sample of the workload
    (the layer's forward and backward on a subset of its tokens; the subset
    shrinks only if the whole run would otherwise take more than about 150 s).
    The weights are drawn, quantized and dequantized by the oracle once,
    untimed."""
    if rank != 0:
        return
    from bit_nf4_quantized_24_b200 import workloads as wl
    w = wl.WORKLOADS[WORKLOAD]
    prep = oracle_layer_prepare(w)
    tokens = args.cpu_tokens
    n_total = max(1, args.warmup + args.steps)
    budget_s = 150.0
    cores = desc = None
    for i in range(args.warmup):
        _, cores, desc, dt = oracle_layer_run(w, prep, tokens)
        if i == 0 and dt * n_total > budget_s:
            tokens = max(4, int(tokens * budget_s / (dt * n_total)))
    vals = []
    for _ in range(max(1, args.steps)):
        tf, cores, desc, dt = oracle_layer_run(w, prep, tokens)
        vals.append(tf)
    v = statistics.median(vals)
    out = {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": world,
           "steps": len(vals), "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded; see workloads.py)",
           "config": {"workload": f"{WORKLOAD} (bounded sample, see cpu_baseline.sample)", "tokens": tokens},
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
    if args.profile == "layer":  # warmup + steps of the benchmark's layer step (14 GEMM launches each)
        w = wl.WORKLOADS[WORKLOAD]
        layer = Layer(qb, w, draw_layer_host(w), dev)
        bufs = layer.new_set(draw_layer_host(w))
        for _ in range(args.warmup + args.steps):
            layer.step(bufs)
        torch.cuda.synchronize()
        assert qb.device_status() == 0
        print(f"profile layer {WORKLOAD} M={w.M} steps={args.warmup + args.steps} done")
        return
    w = wl.WORKLOADS[args.workload]
    M = args.tokens if args.tokens else None
    p = wl.draw_linear(w, args.proj, M=M, with_dy=args.profile in ("bwd", "step"))
    q = qb.nf4_quantize(p["W"].to(dev))
    X, A, B = p["X"].to(dev), p["A"].to(dev), p["B"].to(dev)
    dY = p["dY"].to(dev) if "dY" in p else None
    tiles = qb.nf4_decode_tiles(q) if args.profile == "fwd_tiles" else None
    for _ in range(args.warmup + args.steps):
        if args.profile == "fwd_tiles":
            qb.qlora_linear_fwd_tiles(q, tiles, X, A, B, p["scale"])
        H = None
        if args.profile in ("fwd", "step"):
            _, H = qb.qlora_linear_fwd(q, X, A, B, p["scale"])
        if args.profile in ("bwd", "step"):  # "step" reads the H its forward saved, as the benchmark does
            qb.qlora_linear_bwd(q, X, dY, A, B, p["scale"], H=H)
        if args.profile == "quantize":
            qb.nf4_quantize(p["W"].to(dev))
        if args.profile == "dequantize":
            qb.nf4_dequantize(q)
        if args.profile == "merge":  # the weight merged with its adapter and quantized again
            qb.nf4_merge_lora(q, A, B, p["scale"])
    torch.cuda.synchronize()
    assert qb.device_status() == 0
    print(f"profile {args.profile} {args.workload}[{args.proj}] M={p['M']} N={p['N']} K={p['K']} done")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true", help="skip decode/quantize measurements")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--cpu-tokens", type=int, default=128,
                    help="token rows of the layer in the CPU oracle's bounded sample")
    ap.add_argument("--profile", choices=["layer", "fwd", "fwd_tiles", "bwd", "step", "quantize", "dequantize", "merge"],
                    help="run only warmup+steps launches of one entry point (for ncu)")
    ap.add_argument("--workload", default="qproj_7b", help="workload for --profile (other than layer)")
    ap.add_argument("--tokens", type=int, default=0, help="token count for --profile (default: the workload's)")
    ap.add_argument("--proj", type=int, default=0, help="projection index of the workload for --profile")
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
