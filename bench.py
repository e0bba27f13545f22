#!/usr/bin/env python
"""Benchmark: MoE FFN layer forward throughput on B200, one JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config quartz] [--impl ours|reference]

A step is one whole layer forward (route -> permute -> grouped expert GEMMs -> combine -> loss)
over one batch of seeded synthetic tokens, inputs resident in HBM. With N > 1 (torchrun, one
process per GPU) every rank runs its own batch of T tokens (weak scaling, data-parallel replicas);
the only exchange is an NCCL all-reduce of the 2E per-expert statistics that the global
load-balancing loss needs.

Timing: W untimed warm-up steps; then K steps, each bracketed by CUDA events on the launching
stream, with a 256 MiB write between steps (outside the events) to flush the 126 MB L2; a
barrier and a device synchronise on both sides; the max over ranks. SM clocks are sampled with
NVML during the timed region. A second pass of K steps with the library's per-kernel event
profiler gives the per-kernel durations for the roofline figures; a third pass times the same
steps end to end through the public API with pinned host buffers (x in, y and the loss out).

--impl reference times the CPU oracle (the only other implementation of this path) on a bounded
token sample of the same workload, on rank 0.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MoE layer fwd tokens/s on 1 B200; grouped-GEMM % bf16 peak; permute % HBM BW"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
FLUSH_BYTES = 256 << 20


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return d, "measured"
    except Exception:
        return dict(PEAKS_FALLBACK), "fallback"


def kernel_sources_sha256() -> str:
    """sha256 of the sources the forward kernels are built from: every file of csrc in name
    order except the backward-only ones (backward*.cuh), whose code is not part of the step."""
    import glob
    import hashlib
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "fine_grained_mixture_moe_b200", "csrc", "*"))):
        if os.path.basename(f).startswith("backward"):
            continue
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def captured_traffic(config_name: str, kernel: str):
    """DRAM bytes per launch from a committed ncu capture, or None when the kernels changed."""
    path = os.path.join(ROOT, "profiles", f"traffic_{config_name}.txt")
    try:
        vals = {}
        with open(path) as fh:
            for line in fh:
                if line.strip() and not line.startswith("#"):
                    k, v = line.split()
                    vals[k] = v
    except (OSError, ValueError):
        return None
    if vals.get("sources_sha256") != kernel_sources_sha256():
        return None
    return int(vals[kernel]) if kernel in vals else None


def workload_name(c, fp8: bool = False) -> str:
    parts = [f"{c.name}{'_fp8' if fp8 else ''}: T={c.T} d={c.d} E={c.E} top-{c.top_k} {c.score}"]
    if c.expert == "swiglu":
        parts.append(f"SwiGLU ffn {c.ffn}")
    else:
        parts.append(f"low-rank r={c.rank}" + (", U and V stored as E4M3 rows" if fp8 else ""))
    parts.append(f"{c.n_shared} shared" + (f" (ffn {c.ffn_shared})" if c.n_shared else ""))
    parts.append("dropless" if c.capacity_factor <= 0 else f"capacity factor {c.capacity_factor}")
    parts.append(c.dtype)
    return ", ".join(parts)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, device):
        """`device`: the torch CUDA device index of this rank. NVML numbers devices physically,
        so the handle is found by the device's UUID (CUDA_VISIBLE_DEVICES may reorder or name
        devices), falling back to the index."""
        self.samples = []
        self.reasons = 0
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = None
            try:
                uuid = str(torch.cuda.get_device_properties(device).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(
                    uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def sample(self):
        """One reading of the SM clock and the active clock-event reasons."""
        if not self.ok:
            return
        nv = self.nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
            try:
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
            self.reasons |= int(r)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self.sample()
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
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------------ algorithmic work
def algorithmic(c, n_kept: int, fp8: bool = False, active=None):
    """Per-launch algorithmic flops / bytes of each kernel kind (kept rows only, each input
    read once, each output written once, no tile padding). fp8: the low-rank experts' E4M3
    storage (codes of 1 byte, fp32 z, the quantiser's two launches per step). `active`: the
    experts that receive rows (only their weights are read); all E when not given."""
    T, d, k, S, fs = c.T, c.d, c.top_k, c.n_shared, c.ffn_shared
    E = c.E if active is None else active
    N = n_kept
    es = 2 if c.dtype == "bf16" else 4
    out = {}
    out["router"] = {"flops": 2.0 * T * d * c.E, "bytes": T * d * es + c.E * d * es + 8.0 * T * k}
    # fp8: bf16 token rows in, their E4M3 codes and scales out
    out["perm_scatter"] = {"bytes": T * d * es + N * d * (1 if fp8 else es) + 16.0 * T * k +
                           (4.0 * N if fp8 else 0)}
    sh_flops_gu, sh_flops_dn = 4.0 * d * S * fs * T, 2.0 * d * S * fs * T
    sh_bytes_gu = (T * d + 2.0 * S * fs * d + T * S * fs) * es
    sh_bytes_dn = (T * S * fs + S * fs * d) * es + T * d * 4.0
    if c.expert == "swiglu":
        f = c.ffn
        ys = 2 if c.dtype == "bf16" else 4
        out["gemm_gateup"] = {"flops": 4.0 * d * f * N + sh_flops_gu,
                              "bytes": (N * d + 2.0 * E * f * d + N * f) * es + sh_bytes_gu}
        out["gemm_down"] = {"flops": 2.0 * d * f * N + sh_flops_dn,
                            "bytes": (N * f + E * d * f) * es + N * d * ys + sh_bytes_dn}
    else:
        r = c.rank
        if fp8:  # codes of z and their scales written by the V product itself
            out["gemm_lowrank_v"] = {"flops": 2.0 * d * r * N, "bytes": N * d + E * r * d +
                                     N * r + 4.0 * (2 * N + 2 * E * r)}
            out["gemm_lowrank_u"] = {"flops": 2.0 * d * r * N, "bytes": N * r + E * d * r +
                                     N * d * 4.0 + 4.0 * (N + E * d)}
        else:
            out["gemm_lowrank_v"] = {"flops": 2.0 * d * r * N,
                                     "bytes": (N * d + E * r * d + N * 2 * r) * es}
            out["gemm_lowrank_u"] = {"flops": 2.0 * d * r * N,
                                     "bytes": (N * 2 * r + E * d * r) * es + N * d * 4.0}
        if S:
            out["gemm_gateup"] = {"flops": sh_flops_gu, "bytes": sh_bytes_gu}
            out["gemm_down"] = {"flops": sh_flops_dn, "bytes": sh_bytes_dn}
    # routed expert rows (bf16 for bf16 SwiGLU layers, else fp32), shared output and y in fp32
    ys = 2 if (c.dtype == "bf16" and c.expert == "swiglu") else 4
    out["combine"] = {"bytes": n_kept * d * ys + (T * d * 4.0 if S else 0) + 8.0 * T * k +
                      T * d * 4.0,
                      "bytes_dtype_y": n_kept * d * ys + (T * d * es if S else 0) + 8.0 * T * k +
                      T * d * es}
    return out


def roofline_table(c, n_kept, prof, steps, peaks, src, in_step=None, fp8=False, active=None):
    """Achieved vs peak per kernel kind from the profiler's per-launch averages (CUDA events
    around each launch) and, when given, from the in-step durations (device timestamps, the
    launches overlapped as in the step): `in_step_us` and `frac_in_step`. A GEMM is held to the
    tensor peak when its flops per byte exceed the machine's (peak flops / peak HBM bandwidth),
    else to the HBM bandwidth (the low-rank products: K = rank); fp8 products take the measured
    bf16 peak times the nominal fp8 / bf16 ratio of 2."""
    alg = algorithmic(c, n_kept, fp8, active)
    # fp32 FMA on the CUDA cores: 148 SMs x 128 lanes x 2 flops at the maximum SM clock
    fp32_peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12  # TFLOP/s, nominal
    # datasheet figures beside the measured ones: ~8 TB/s HBM3e, 2.25 PFLOP/s dense bf16 (4.5 fp8)
    spec = {"GB/s": 8000.0, "TFLOP/s": 2250.0}
    rows = {}
    for name, (ms, n) in prof.items():
        if n == 0:
            continue
        avg_ms = ms / n
        a = alg.get(name, {})
        row = {"launches": n, "avg_us": avg_ms * 1e3, "share": None}
        if name.startswith("gemm"):
            tpeak = peaks["bf16_tflops"] * (2.0 if fp8 and "lowrank" in name else 1.0)
            ridge = tpeak * 1e12 / (peaks["hbm_gbs"] * 1e9)
            tflops = a["flops"] / (avg_ms * 1e-3) / 1e12
            gbs = a["bytes"] / (avg_ms * 1e-3) / 1e9
            if a["flops"] / a["bytes"] >= ridge:
                row.update(bound="tensor", achieved=tflops, peak=tpeak, unit="TFLOP/s",
                           frac=tflops / tpeak, hbm_gbs=gbs)
            else:
                row.update(bound="hbm", achieved=gbs, peak=peaks["hbm_gbs"], unit="GB/s",
                           frac=gbs / peaks["hbm_gbs"], tflops=tflops)
        elif name == "router":
            ach = a["flops"] / (avg_ms * 1e-3) / 1e12
            row.update(bound="alu", achieved=ach, peak=fp32_peak, unit="TFLOP/s (fp32 FMA)",
                       frac=ach / fp32_peak,
                       hbm_gbs=a["bytes"] / (avg_ms * 1e-3) / 1e9)
        elif "bytes" in a:
            ach = a["bytes"] / (avg_ms * 1e-3) / 1e9
            row.update(bound="hbm", achieved=ach, peak=peaks["hbm_gbs"], unit="GB/s",
                       frac=ach / peaks["hbm_gbs"])
            if "bytes_dtype_y" in a:
                # the same launch against the byte count with y and the shared output in the
                # layer's dtype (what a bf16 output would move), beside the fp32 figure above
                ach2 = a["bytes_dtype_y"] / (avg_ms * 1e-3) / 1e9
                row.update(achieved_dtype_y=ach2, frac_dtype_y=ach2 / peaks["hbm_gbs"])
        if row.get("unit") in spec:
            row["frac_spec"] = row["achieved"] / (spec[row["unit"]] *
                                                  (2.0 if fp8 and "lowrank" in name and
                                                   row["unit"] == "TFLOP/s" else 1.0))
        if in_step and name in in_step and "frac" in row:
            us = in_step[name]
            row["in_step_us"] = us
            row["frac_in_step"] = row["frac"] * row["avg_us"] / us
        rows[name] = row
    tot = sum(ms for ms, n in prof.values())
    for name, (ms, n) in prof.items():
        if name in rows:
            rows[name]["share"] = ms / tot if tot else None
    return rows


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch
    import torch.distributed as dist

    import fine_grained_mixture_moe_b200 as moe
    from fine_grained_mixture_moe_b200 import binding as B
    from fine_grained_mixture_moe_b200 import dist as D
    from fine_grained_mixture_moe_b200.layer import MoELayer, upload_weights, y_perm_dtype
    from moe_synth import get_config, make_inputs

    from fine_grained_mixture_moe_b200 import build as _b
    if rank == 0:
        _b.build()
    if world > 1:
        dist.barrier()
    moe.load()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    fp8 = args.config.endswith("_fp8")  # low-rank experts stored as E4M3 rows
    c = get_config(args.config[:-4] if fp8 else args.config)
    inp = make_inputs(c)
    cfg = B.make_config(T=c.T, d=c.d, E=c.E, top_k=c.top_k, n_shared=c.n_shared, ffn=c.ffn,
                        ffn_shared=c.ffn_shared, rank=c.rank, score=c.score, expert=c.expert,
                        dtype=c.dtype, norm_topk=c.norm_topk, capacity_factor=c.capacity_factor,
                        aux_alpha=c.aux_alpha, expert_storage="fp8" if fp8 else "dtype")
    weights = upload_weights(cfg, inp, dev)
    layer = MoELayer(cfg, weights, dev)
    dt = layer.dtype
    x = torch.as_tensor(inp["x"]).to(dt).contiguous().to(dev)
    y = torch.empty((c.T, c.d), dtype=torch.float32, device=dev)
    aux = torch.empty((), dtype=torch.float32, device=dev)
    cnt = torch.empty(c.E, dtype=torch.int32, device=dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    # multi-GPU: route -> all-reduce(count, prob_sum) -> rest, loss over all ranks' tokens
    if world > 1:
        T, k, E, d = c.T, c.top_k, c.E, c.d
        idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        wts = torch.empty((T, k), dtype=torch.float32, device=dev)
        packed = torch.empty(2 * E, dtype=torch.float32, device=dev)
        prob = torch.empty(E, dtype=torch.float32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        slot = torch.empty((T, k), dtype=torch.int32, device=dev)
        src = torch.empty(T * k, dtype=torch.int32, device=dev)
        xp = torch.empty((T * k, d), dtype=dt, device=dev)
        yp = torch.empty((T * k, d), dtype=y_perm_dtype(cfg), device=dev)
        ysh = torch.empty((T, d), dtype=torch.float32, device=dev) if c.n_shared else None
        gcfg = D.loss_config(cfg, world)

        def step(xb=x, yb=y, ab=aux):
            B.moe_route(cfg, xb, layer.wstruct, idx, wts, cnt, prob, layer.ws, layer.ws_bytes)
            gcnt, gprob = D.allreduce_route_stats(cnt, prob, T * world * k, packed=packed)
            B.moe_permute(cfg, xb, idx, offsets, slot, src, xp, layer.ws, layer.ws_bytes)
            B.moe_expert_forward(cfg, xp, offsets, xb, layer.wstruct, yp, ysh, layer.ws,
                                 layer.ws_bytes)
            B.moe_combine(cfg, yp, ysh, slot, wts, yb)
            B.moe_aux_loss(gcfg, gcnt, gprob, ab)
    else:
        def step(xb=x, yb=y, ab=aux):
            layer.forward(xb, yb, ab, cnt)

    def timed(K, pre=None, tick=None, warm=False):
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for i in range(K):
            if not warm:
                flush.fill_(i & 0xff)
            if pre:
                pre(i)
            starts[i].record(stream)
            step()
            ends[i].record(stream)
            if tick:
                tick()  # the GPU is still working through the queued steps
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        return [s.elapsed_time(e) for s, e in zip(starts, ends)]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, info = B.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error after warm-up: {B.status_str(st)} info={info}")
    n_kept = int(torch.as_tensor(cnt).sum()) if c.capacity_factor <= 0 else None
    if n_kept is None or world > 1:
        offs = torch.empty(c.E + 1, dtype=torch.int32, device=dev)
        tmp_idx = torch.empty((c.T, c.top_k), dtype=torch.int32, device=dev)
        tmp_w = torch.empty((c.T, c.top_k), dtype=torch.float32, device=dev)
        tmp_c = torch.empty(c.E, dtype=torch.int32, device=dev)
        tmp_p = torch.empty(c.E, dtype=torch.float32, device=dev)
        B.moe_route(cfg, x, layer.wstruct, tmp_idx, tmp_w, tmp_c, tmp_p, layer.ws, layer.ws_bytes)
        sl = torch.empty((c.T, c.top_k), dtype=torch.int32, device=dev)
        sr = torch.empty(c.T * c.top_k, dtype=torch.int32, device=dev)
        B.moe_permute(cfg, x, tmp_idx, offs, sl, sr, None, layer.ws, layer.ws_bytes)
        torch.cuda.synchronize()
        n_kept = int(offs[-1])
        counts = tmp_c.cpu().numpy()
    else:
        counts = cnt.cpu().numpy()

    # pass 1: the number
    with ClockSampler(torch.cuda.current_device()) as clk:
        times = timed(args.steps, tick=clk.sample)
    ms = statistics.fmean(times)
    if world > 1:
        t = torch.tensor([ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t)
    st, info = B.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the timed region: {B.status_str(st)} info={info}")

    # pass 1b: the same steps back to back without the flush (warm L2: x, the weights and the
    # workspace stay in the 126 MB L2 between steps), reported beside the number, labelled
    ms_warm = statistics.fmean(timed(args.steps, warm=True))
    if world > 1:
        t = torch.tensor([ms_warm], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_warm = float(t)

    # pass 2: per-kernel durations (library event profiler, same steps), then the same kernels'
    # durations inside the step from the library's device timestamps
    B.moe_debug_set(B.DEBUG_PROFILE, 1)
    timed(args.steps)
    prof = B.moe_profile_read()
    B.moe_debug_set(B.DEBUG_PROFILE, 0)
    in_step = in_step_durations(step, args.steps, flush) if world == 1 else None

    # pass 3: end to end through the public API with pinned host buffers. Each step copies its
    # tokens in, runs the layer and copies y and the loss out. Steps are double-buffered over
    # three streams (copy in, compute, copy out), so step i+1's upload and step i's download
    # overlap compute, as a serving loop would; the number is the wall time of all steps on the
    # device clock divided by the step count, L2 flush included.
    x_host = torch.empty_like(x, device="cpu").pin_memory()
    x_host.copy_(x.cpu())
    y_host = [torch.empty_like(y, device="cpu").pin_memory() for _ in range(2)]
    aux_host = [torch.empty((), dtype=torch.float32).pin_memory() for _ in range(2)]
    xs_dev = [x, torch.empty_like(x)]
    ys_dev = [y, torch.empty_like(y)]
    auxs_dev = [aux, torch.empty_like(aux)]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    done_in = [torch.cuda.Event() for _ in range(args.steps)]
    done_comp = [torch.cuda.Event() for _ in range(args.steps)]
    done_out = [torch.cuda.Event() for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    s_in.wait_event(t_start)
    for i in range(args.steps):
        b = i & 1
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(done_comp[i - 2])  # the layer of step i-2 has read this x buffer
            xs_dev[b].copy_(x_host, non_blocking=True)
            done_in[i].record(s_in)
        stream.wait_event(done_in[i])
        if i >= 2:
            stream.wait_event(done_out[i - 2])  # y and loss buffers b have been downloaded
        flush.fill_(i & 0xff)
        step(xs_dev[b], ys_dev[b], auxs_dev[b])
        done_comp[i].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(done_comp[i])
            y_host[b].copy_(ys_dev[b], non_blocking=True)
            aux_host[b].copy_(auxs_dev[b], non_blocking=True)
            done_out[i].record(s_out)
    stream.wait_event(done_out[args.steps - 1])
    t_end.record(stream)
    torch.cuda.synchronize()
    e2e_ms = t_start.elapsed_time(t_end) / args.steps
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t)
    h2d = x.numel() * x.element_size()
    d2h = y.numel() * y.element_size() + 4

    peaks, peak_src = load_peaks()
    backward = backward_parts(c, cfg, layer, x, flush, stream, args.steps, peaks) \
        if world == 1 and not fp8 else None  # training stays bf16: no backward of fp8 storage
    table = roofline_table(c, n_kept, prof, args.steps, peaks, peak_src, in_step, fp8,
                           int((counts > 0).sum()))
    dom = max(table, key=lambda n: table[n]["share"] or 0.0)
    dr = table[dom]
    launches_per_step = sum(n for _, n in prof.values()) / max(args.steps, 1)
    tokens = c.T * world
    result = {
        "metric": METRIC,
        "value": tokens / (ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": c.dtype,
        "data": "synthetic: seeded torch CPU generator, bf16-rounded N(0,1) tokens and "
                "random-init weights of the configuration's shapes (no dataset, no checkpoint)",
        "config": {
            "workload": workload_name(c, fp8),
            "tokens_per_gpu": c.T,
            "l2": "flushed between timed steps (256 MiB write outside the events)",
            "parallelism": f"dp{world} replicas" + (" + NCCL all-reduce of 2E expert stats"
                                                     if world > 1 else ""),
            "kept_pairs": n_kept,
            "expert_rows_min_max": [int(counts.min()), int(counts.max())],
            "dead_experts": int((counts == 0).sum()),
            "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv)
                            for kk, vv in v.items()} for k, v in table.items()},
            "peaks": f"{peak_src} (MEASURED_PEAKS.json)" if peak_src == "measured" else
                     "fallback pool figures",
        },
        "roofline": {"kernel": dom, "bound": dr.get("bound"), "achieved": dr.get("achieved"),
                     "peak": dr.get("peak"), "unit": dr.get("unit"), "frac": dr.get("frac"),
                     "traffic": captured_traffic(c.name, dom),
                     "traffic_source": "profiles/traffic_quartz.txt (ncu dram bytes read+write per launch)",
                     "peak_kind": f"{peak_src} burst" if dr.get("bound") == "tensor" else peak_src},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": int(round(launches_per_step * args.steps)),
        "clocks": clk.summary(),
        "warm_l2": {"value": tokens / (ms_warm * 1e-3), "unit": "tokens/s", "ms_per_step": ms_warm,
                    "note": "the same steps without the L2 flush between them (not the number)"},
    }
    if backward is not None:
        result["backward_parts"] = backward
    if world == 1 and args.per_config != "none":
        result["per_config"] = {
            name: measure_config(name, args.steps, args.warmup, dev, flush, stream, peaks,
                                 peak_src)
            for name in args.per_config.split(",") if name and name != args.config}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(c, inp)
    return result


def in_step_durations(step, K, flush):
    """Per-kernel-kind durations inside the step from the library's device timestamps
    (MOE_DEBUG_STAMP), averaged over K steps with the L2 flushed before each."""
    import torch

    from fine_grained_mixture_moe_b200 import binding as B
    B.moe_debug_set(B.DEBUG_STAMP, 1)
    acc = {}
    try:
        for i in range(K):
            flush.fill_(i & 0xff)
            torch.cuda.synchronize()
            B.moe_stamp_read()  # clears the records of the flush's interval
            step()
            for n, us in B.moe_stamp_read().items():
                acc.setdefault(n, []).append(us)
    finally:
        B.moe_debug_set(B.DEBUG_STAMP, 0)
    return {n: statistics.fmean(v) for n, v in acc.items()}


def measure_config(name, K, W, dev, flush, stream, peaks, peak_src):
    """One more configuration on this GPU, timed like the headline one: W warm-up layer calls,
    then K calls each bracketed by CUDA events with the L2 flushed in between, then K calls with
    the library's event profiler for the per-kernel table. Inputs resident, weights random-init
    of the configuration's shapes."""
    import torch

    from fine_grained_mixture_moe_b200 import binding as B
    from fine_grained_mixture_moe_b200.layer import MoELayer, upload_weights
    from moe_synth import get_config, make_inputs

    fp8 = name.endswith("_fp8")  # a configuration's low-rank experts stored as E4M3 rows
    c = get_config(name[:-4] if fp8 else name)
    inp = make_inputs(c)
    cfg = B.make_config(T=c.T, d=c.d, E=c.E, top_k=c.top_k, n_shared=c.n_shared, ffn=c.ffn,
                        ffn_shared=c.ffn_shared, rank=c.rank, score=c.score, expert=c.expert,
                        dtype=c.dtype, norm_topk=c.norm_topk, capacity_factor=c.capacity_factor,
                        aux_alpha=c.aux_alpha, expert_storage="fp8" if fp8 else "dtype")
    layer = MoELayer(cfg, upload_weights(cfg, inp, dev), dev)
    x = torch.as_tensor(inp["x"]).to(layer.dtype).contiguous().to(dev)
    y = torch.empty((c.T, c.d), dtype=torch.float32, device=dev)
    aux = torch.empty((), dtype=torch.float32, device=dev)
    cnt = torch.empty(c.E, dtype=torch.int32, device=dev)
    for _ in range(W):
        layer.forward(x, y, aux, cnt)
    torch.cuda.synchronize()

    def timed():
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        torch.cuda.synchronize()
        for i in range(K):
            flush.fill_(i & 0xff)
            ev[i][0].record(stream)
            layer.forward(x, y, aux, cnt)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    ms = statistics.fmean(timed())
    B.moe_debug_set(B.DEBUG_PROFILE, 1)
    timed()
    prof = B.moe_profile_read()
    B.moe_debug_set(B.DEBUG_PROFILE, 0)
    in_step = in_step_durations(lambda: layer.forward(x, y, aux, cnt), K, flush)
    st, info = B.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error ({name}): {B.status_str(st)} info={info}")
    # kept pairs from the permutation's offsets (capacity drops included)
    idx = torch.empty((c.T, c.top_k), dtype=torch.int32, device=dev)
    wts = torch.empty((c.T, c.top_k), dtype=torch.float32, device=dev)
    prob = torch.empty(c.E, dtype=torch.float32, device=dev)
    offs = torch.empty(c.E + 1, dtype=torch.int32, device=dev)
    sl = torch.empty((c.T, c.top_k), dtype=torch.int32, device=dev)
    sr = torch.empty(c.T * c.top_k, dtype=torch.int32, device=dev)
    B.moe_route(cfg, x, layer.wstruct, idx, wts, cnt, prob, layer.ws, layer.ws_bytes)
    B.moe_permute(cfg, x, idx, offs, sl, sr, None, layer.ws, layer.ws_bytes)
    torch.cuda.synchronize()
    n_kept = int(offs[-1])
    counts = cnt.cpu().numpy()
    table = roofline_table(c, n_kept, prof, K, peaks, peak_src, in_step, fp8,
                           int((counts > 0).sum()))
    out = {
        "workload": workload_name(c, fp8),
        "value": c.T / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms, "steps": K,
        "warmup": W, "dtype": c.dtype,
        "kept_pairs": n_kept, "dropped_pairs": c.T * c.top_k - n_kept,
        "expert_rows_min_max": [int(counts.min()), int(counts.max())],
        "dead_experts": int((counts == 0).sum()),
        "kernels": {k: {kk: (round(vv, 4) if isinstance(vv, float) else vv)
                        for kk, vv in v.items()} for k, v in table.items()},
    }
    del layer, x, y
    torch.cuda.empty_cache()
    return out


def backward_calls(c, cfg, layer, x):
    """The forward's outputs (route, permute, experts) on the device and the three backward
    entry points as callables on them, with a seeded upstream gradient: (combine, route,
    experts, info). Used by backward_parts and by --backward-launches."""
    import torch

    from fine_grained_mixture_moe_b200 import binding as B
    from fine_grained_mixture_moe_b200.layer import y_perm_dtype

    dev = x.device
    T, d, E, k = c.T, c.d, c.E, c.top_k
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    wts = torch.empty((T, k), dtype=torch.float32, device=dev)
    cnt = torch.empty(E, dtype=torch.int32, device=dev)
    prob = torch.empty(E, dtype=torch.float32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    slot = torch.empty((T, k), dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    xp = torch.empty((T * k, d), dtype=x.dtype, device=dev)
    yp = torch.empty((T * k, d), dtype=y_perm_dtype(cfg), device=dev)
    ysh = torch.empty((T, d), dtype=torch.float32, device=dev) if c.n_shared else None
    B.moe_route(cfg, x, layer.wstruct, idx, wts, cnt, prob, layer.ws, layer.ws_bytes)
    B.moe_permute(cfg, x, idx, offsets, slot, src, xp, layer.ws, layer.ws_bytes)
    B.moe_expert_forward(cfg, xp, offsets, x, layer.wstruct, yp, ysh, layer.ws, layer.ws_bytes)
    g = torch.Generator(device="cpu")
    g.manual_seed(5)
    dy = torch.randn((T, d), generator=g, dtype=torch.float32).to(dev)
    dyp = torch.empty_like(yp)
    d_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    d_logits = torch.empty((T, E), dtype=torch.float32, device=dev)
    d_wr = torch.empty((E, d), dtype=torch.float32, device=dev)
    dx = torch.empty((T, d), dtype=torch.float32, device=dev)
    torch.cuda.synchronize()
    N = int(offsets[-1])
    # the experts' backward: data and weight gradients of every routed and shared expert
    E_, f_, r_, S_, fs_ = c.E, c.ffn, c.rank, c.n_shared, c.ffn_shared
    if c.expert == "swiglu":
        gr = {"d_w_gate": torch.empty((E_, f_, d), dtype=torch.float32, device=dev),
              "d_w_up": torch.empty((E_, f_, d), dtype=torch.float32, device=dev),
              "d_w_down": torch.empty((E_, d, f_), dtype=torch.float32, device=dev)}
        flop_e = 16.0 * d * f_ * N
    else:
        gr = {"d_lr_V": torch.empty((E_, r_, d), dtype=torch.float32, device=dev),
              "d_lr_s": torch.empty((E_, r_), dtype=torch.float32, device=dev),
              "d_lr_U": torch.empty((E_, d, r_), dtype=torch.float32, device=dev)}
        flop_e = 10.0 * d * r_ * N
    if S_:
        gr.update(d_ws_gate=torch.empty((S_, fs_, d), dtype=torch.float32, device=dev),
                  d_ws_up=torch.empty((S_, fs_, d), dtype=torch.float32, device=dev),
                  d_ws_down=torch.empty((S_, d, fs_), dtype=torch.float32, device=dev))
        flop_e += 16.0 * d * S_ * fs_ * T
    bws = B.moe_backward_workspace_size(cfg)
    bw_ws = torch.empty(bws, dtype=torch.uint8, device=dev)
    dx_e = torch.empty((T, d), dtype=torch.float32, device=dev)
    gstruct = B.make_grads(gr)

    def combine():
        B.moe_combine_backward(cfg, dy, yp, slot, wts, dyp, d_w)

    def route():
        B.moe_route_backward(cfg, x, layer.wstruct, idx, cnt, d_w, 1.0, d_logits, d_wr, dx)

    def experts():
        B.moe_expert_backward(cfg, xp, offsets, slot, x, layer.wstruct, dyp, dy if S_ else None,
                              dx_e, gstruct, bw_ws, bws)

    info = {"N": N, "flop_e": flop_e, "by": yp.element_size(), "bx": x.element_size(),
            "keep": (gr, bw_ws)}
    return combine, route, experts, info


def backward_parts(c, cfg, layer, x, flush, stream, K, peaks):
    """The backward's entry points (combine, experts, router), each call timed alone with CUDA
    events on the forward's resident outputs and a seeded upstream gradient, L2 flushed between
    calls. Not part of the step above."""
    import torch

    from fine_grained_mixture_moe_b200 import binding as B

    T, d, E, k = c.T, c.d, c.E, c.top_k
    combine, route, experts, info = backward_calls(c, cfg, layer, x)
    N, flop_e = info["N"], info["flop_e"]

    def timed_call(fn):
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(K)]
        torch.cuda.synchronize()
        for i in range(K):
            flush.fill_(i & 0xff)
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return statistics.fmean(a.elapsed_time(b) for a, b in ev) * 1e3

    us_c = timed_call(combine)
    us_r = timed_call(route)
    us_e = timed_call(experts)
    st, info_err = B.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the backward pass: {B.status_str(st)} info={info_err}")
    by, bx = info["by"], info["bx"]
    # algorithmic bytes: every input read once, every output written once
    bytes_c = T * d * 4 + 2 * N * d * by + T * k * 12
    bytes_r = T * d * bx + E * d * bx + T * k * 8 + E * 4 + T * E * 4 + E * d * 4 + T * d * 4
    flop_r = 6.0 * T * d * E  # logits again, then the two router products
    hbm = peaks["hbm_gbs"]
    fp32 = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12  # nominal, TFLOP/s
    return {
        "note": "each call timed alone (CUDA events, L2 flushed between calls); not in the step",
        "combine_backward": {"avg_us": round(us_c, 2), "bound": "hbm", "bytes": bytes_c,
                             "achieved_gbs": round(bytes_c / us_c / 1e3, 1),
                             "frac": round(bytes_c / us_c / 1e3 / hbm, 4)},
        "expert_backward": {"avg_us": round(us_e, 2), "bound": "tensor", "flop": flop_e,
                            "achieved_tflops": round(flop_e / us_e / 1e6, 1),
                            "frac": round(flop_e / us_e / 1e6 / peaks["bf16_tflops"], 4),
                            "note": "algorithmic flops: g and u recomputed, dh, dX, the three "
                                    "weight gradients (routed and shared); the kernels run "
                                    "the non-bf16 operands as two bf16 terms"},
        "route_backward": {"avg_us": round(us_r, 2), "bound": "alu", "flop": flop_r,
                           "achieved_tflops": round(flop_r / us_r / 1e6, 3),
                           "frac": round(flop_r / us_r / 1e6 / fp32, 4), "bytes": bytes_r,
                           "achieved_gbs": round(bytes_r / us_r / 1e3, 1)},
    }


def _cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def _oracle_seconds(c, inp, T, threads):
    """Wall seconds of one oracle layer forward over the first T tokens with `threads` BLAS
    threads (numpy's own loops are single-threaded)."""
    import oracle
    from threadpoolctl import threadpool_limits
    sub = dict(inp)
    sub["x"] = inp["x"][:T]
    cs = c.with_(T=T)
    with threadpool_limits(limits=threads):
        t0 = time.perf_counter()
        oracle.layer_forward(cs, sub)
        return time.perf_counter() - t0


def cpu_baseline(c, inp, T_sample=None):
    """The oracle, as it stands, on a bounded token sample of the same workload: once with
    every core of the affinity mask, once on a single thread."""
    T = min(c.T, T_sample or 2048)
    cores = _cores()
    dt_all = _oracle_seconds(c, inp, T, cores)
    dt_one = _oracle_seconds(c, inp, T, 1)
    return {"value": T / dt_all, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"one layer forward over the first {T} tokens of the workload "
                      f"({dt_all:.1f} s on {cores} cores, fp64 numpy/OpenBLAS)",
            "single_thread": {"value": T / dt_one, "unit": "tokens/s", "cores": 1,
                              "seconds": round(dt_one, 2)}}


# ------------------------------------------------------------------ reference arm (oracle)
def run_reference(args):
    from moe_synth import get_config, make_inputs
    c = get_config(args.config)
    inp = make_inputs(c)
    # size the token sample so that all K + W steps take about two minutes
    per_token_s = 11.0 / 4096 * (c.d * (3 * c.ffn * c.top_k + 3 * c.ffn_shared * c.n_shared +
                                        c.E) + (2 * c.d * c.rank * c.top_k)) / (1024 * (3 * 640 * 8 + 24))
    budget = 120.0 / max(args.steps + args.warmup, 1)
    T_s = int(max(32, min(c.T, budget / max(per_token_s, 1e-9))) // 32 * 32) or 32
    import oracle
    from threadpoolctl import threadpool_limits
    threadpool_limits(limits=_cores())
    sub = dict(inp)
    sub["x"] = inp["x"][:T_s]
    cs = c.with_(T=T_s)
    for _ in range(args.warmup):
        oracle.layer_forward(cs, sub)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        oracle.layer_forward(cs, sub)
        times.append(time.perf_counter() - t0)
    ms = statistics.fmean(times) * 1e3
    v = T_s / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": workload_name(c), "tokens_per_step": T_s},
        "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": _cores(), "kind": "oracle",
                         "sample": f"first {T_s} tokens of the workload per step"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_backward_launches(args):
    """--backward-launches: the backward entry points of one configuration, twice each, untimed
    (a short program for a profiler's launch list; prints one line)."""
    import torch

    import fine_grained_mixture_moe_b200 as moe
    from fine_grained_mixture_moe_b200 import binding as B
    from fine_grained_mixture_moe_b200 import build as _b
    from fine_grained_mixture_moe_b200.layer import MoELayer, upload_weights
    from moe_synth import get_config, make_inputs

    _b.build()
    moe.load()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    c = get_config(args.config)
    inp = make_inputs(c)
    cfg = B.make_config(T=c.T, d=c.d, E=c.E, top_k=c.top_k, n_shared=c.n_shared, ffn=c.ffn,
                        ffn_shared=c.ffn_shared, rank=c.rank, score=c.score, expert=c.expert,
                        dtype=c.dtype, norm_topk=c.norm_topk, capacity_factor=c.capacity_factor,
                        aux_alpha=c.aux_alpha)
    layer = MoELayer(cfg, upload_weights(cfg, inp, dev), dev)
    x = torch.as_tensor(inp["x"]).to(layer.dtype).contiguous().to(dev)
    combine, route, experts, _ = backward_calls(c, cfg, layer, x)
    for _ in range(2):
        combine()
        route()
        experts()
    torch.cuda.synchronize()
    st, info = B.moe_get_device_error()
    if st != 0:
        raise RuntimeError(f"device error in the backward pass: {B.status_str(st)} info={info}")
    return {"backward_launches": c.name, "passes": 2}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="quartz")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-config", default="capacity,sigmoid,lowrank,lowrank_fp8",
                    help="further configurations timed on one GPU beside the headline one "
                         "(comma-separated names, or 'none')")
    ap.add_argument("--backward-launches", action="store_true",
                    help="run the backward entry points of --config twice, untimed, and exit")
    args = ap.parse_args()
    if args.backward_launches:
        print(json.dumps(run_backward_launches(args)), flush=True)
        return
    if args.warmup < 3:
        args.warmup = 3
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
