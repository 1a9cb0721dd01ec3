#!/usr/bin/env python
"""Benchmark of the gated delta-rule hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload kda_prefill] [--no-decode] [--no-cpu-baseline] [--no-extra]

One step = one KDA prefill call (``kda_chunk_fwd``) over the whole synthetic
workload (B=1, H=32, T=4096, d_k=d_v=128, bf16 q/k/v, fp32 gate/beta/state),
inputs resident in HBM.  The same JSON line also carries the decode-step
measurement (256 sequences x 32 heads, state updated in place, 64 steps) as
``decode``, and the other timed prefill configurations (8 packed KDA sequences;
Gated DeltaNet T=65536 with 16 q/k and 32 v heads) as ``prefill_configs``,
each with its own rooflines.  L2 (126 MB) is flushed by writing a 256 MB buffer before every
timed call.  Times are CUDA-event device times on the launching stream; with
N > 1 ranks every rank runs its own copy of the workload (weak scaling, no
data-path collective) and the slowest rank's time is reported.

``--impl reference`` times the fp64 CPU oracle (test infrastructure) on a
bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from gated_delta_rule_87_b200 import workloads as W  # noqa: E402

L2_FLUSH_BYTES = 256 << 20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


# --------------------------------------------------------------------------- #
# algorithmic work per unit (bytes / flops), counted once
# --------------------------------------------------------------------------- #
def prefill_bytes(w: W.Workload, total_tokens: int, num_seqs: int) -> int:
    """q, k (H_qk heads), v, o (H_v heads) in the io dtype, gate and beta in fp32,
    initial and final state in fp32 -- each moved once."""
    e = 2 if w.io_dtype == "bf16" else 4
    per_tok = (2 * w.H_qk * w.d_k + 2 * w.H_v * w.d_v) * e + 4 * w.H_v
    per_tok += 4 * w.H_v * (w.d_k if w.gate == "channel" else 1)
    states = (2 if w.init_state else 1) * num_seqs * w.H_v * w.d_k * w.d_v * 4
    return total_tokens * per_tok + states


def prefill_flops(w: W.Workload, total_tokens: int, C: int = 64) -> float:
    """Fixed chunk-form flop count at C = 64: KDA 15*C*d + 8*d^2 per token-head,
    Gated DeltaNet 7*C*d + 6*d^2 per token-v-head (d = d_k = d_v)."""
    d = w.d_k
    if w.gate == "channel":
        return float(total_tokens) * w.H_v * (15 * C * d + 8 * d * d)
    return float(total_tokens) * w.H_v * (7 * C * d + 6 * d * d)


def kernel_algo_bytes(name: str, w: W.Workload, total_tokens: int, num_seqs: int) -> int:
    """Algorithmic bytes one launch of a library kernel must move.

    chunk_prep_kernel reads every input token once (q, k, v, gate, beta);
    chunk_scan_kernel writes o and reads/writes the states; the single-kernel
    fp32 path moves everything."""
    e = 2 if w.io_dtype == "bf16" else 4
    gate = 4 * w.H_v * (w.d_k if w.gate == "channel" else 1)
    states = (2 if w.init_state else 1) * num_seqs * w.H_v * w.d_k * w.d_v * 4
    if name.startswith("chunk_prep"):
        return total_tokens * ((2 * w.H_qk * w.d_k + w.H_v * w.d_v) * e + gate + 4 * w.H_v)
    if name.startswith("chunk_scan"):
        return total_tokens * w.H_v * w.d_v * e + states
    if name.startswith("plan"):
        return 4 * (num_seqs + 1)
    return prefill_bytes(w, total_tokens, num_seqs)


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes (read + write) per launch from a committed ncu summary, or
    None if the kernel's source changed since the counters were taken."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel, {}).get(workload)
        if not rec:
            return None
        src = os.path.join(ROOT, rec["source"])
        with open(src, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()[:16]
        return rec["bytes"] if sha == rec["source_sha256_16"] else None
    except Exception:
        return None


def decode_bytes_per_head(w: W.Workload) -> int:
    e = 2 if w.io_dtype == "bf16" else 4
    return 2 * w.d_k * w.d_v * 4 + (2 * w.d_k + 2 * w.d_v) * e + 4 * w.d_k + 4


# --------------------------------------------------------------------------- #
# clocks during the timed region
# --------------------------------------------------------------------------- #
class ClockSampler:
    """Samples SM clocks and throttle reasons (NVML, every ~2 ms) while the
    timed region runs.  Reads settings only."""

    REASONS = {  # NVML clocks-event-reason bits
        "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nv = None

    def __enter__(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            self._nv = nv
            self._h = nv.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self._h, nv.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        except Exception:
            self._nv = None
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, bit in self.REASONS.items():
                    if bits & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=2)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- #
# distributed plumbing
# --------------------------------------------------------------------------- #
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a per-rank scalar over all ranks (CPU tensor under gloo)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    on_cpu = dist.get_backend() == "gloo" or device is None
    t = torch.tensor([x], dtype=torch.float64, device="cpu" if on_cpu else device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if dist.get_backend() == "gloo" or device is None:
            dist.barrier()
        else:
            dist.barrier(device_ids=[device.index])


def aggregate_throughput(units_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput of weakly scaled replicas: every rank processes
    its own ``units_per_rank``; the job takes as long as the slowest rank."""
    return units_per_rank * world / (ms_max / 1e3)


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def run_ours(args, world, rank, local):
    import torch

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    peaks = _peaks()
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    w = W.WORKLOADS[args.workload]
    if args.tokens is not None:
        w = w.replace(T=args.tokens)
    main = bench_prefill(w, args, device, world, peaks, stream, flush, with_e2e=True,
                         tokens_override=args.tokens is not None)

    line = {
        "metric": "KDA prefill tokens/s (decode-step state GB/s in 'decode'), % of roofline, 1xB200",
        "value": main["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": main["dtype"],
        "data": "synthetic (seeded normals shaped like the workload)",
        "config": main["config"],
        "roofline": main["roofline"],
        "call_roofline": main["call_roofline"],
        "kernels": main["kernels"],
        "e2e": main["e2e"],
        "gpu_launches": main["launches"],
        "clocks": main["clocks"],
        "step_ms_min_max": main["step_ms_min_max"],
    }
    x_main = main.pop("_inputs")

    if not args.no_decode:
        line["decode"] = bench_decode(args, device, world, peaks, stream, flush)
        line["gpu_launches"] += line["decode"]["launches"]

    # the other timed prefill configurations, each with its own rooflines
    if not args.no_extra and args.tokens is None:
        extra = {}
        for name in EXTRA_PREFILL:
            if name == w.name:
                continue
            r = bench_prefill(W.WORKLOADS[name], args, device, world, peaks, stream, flush,
                              with_e2e=False)
            r.pop("_inputs")
            line["gpu_launches"] += r.pop("launches")
            extra[name] = r
        line["prefill_configs"] = extra

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(x_main, w)

    if world > 1:
        import torch.distributed as dist
        dist.barrier(device_ids=[device.index])
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)


# prefill configurations timed besides the main one (their own sub-objects)
EXTRA_PREFILL = ("kda_prefill", "kda_varlen", "gdn_long")


def bench_prefill(w, args, device, world, peaks, stream, flush, with_e2e=False,
                  tokens_override=False):
    """Device-timed prefill calls on one workload (inputs resident in HBM, L2
    flushed before every call), per-kernel times from the library's trace
    events, rooflines, and optionally the end-to-end time through the public
    API with host buffers."""
    import torch
    import gated_delta_rule_87_b200 as gdr
    x = W.make_prefill(w, seed=0)
    N = x.num_seqs
    T_total = x.total_tokens
    varlen = bool(w.varlen)
    B, T = (1, T_total) if varlen else (w.B, w.T)
    bf = lambda a, shape: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
        torch.bfloat16).reshape(shape)
    f32 = lambda a, shape: torch.from_numpy(np.ascontiguousarray(a)).reshape(shape)
    io_host = bf if w.io_dtype == "bf16" else f32
    host = {
        "q": io_host(x.q, (B, T, w.H_qk, w.d_k)), "k": io_host(x.k, (B, T, w.H_qk, w.d_k)),
        "v": io_host(x.v, (B, T, w.H_v, w.d_v)),
        "g": f32(x.g, (B, T) + x.g.shape[1:]), "beta": f32(x.beta, (B, T, w.H_v)),
    }
    if x.initial_state is not None:
        host["s0"] = f32(x.initial_state, x.initial_state.shape)
    if with_e2e:
        host = {k: v.pin_memory() for k, v in host.items()}
    dev = {k: v.to(device) for k, v in host.items()}
    cu = torch.from_numpy(x.cu_seqlens).to(device) if varlen else None
    s0 = dev.get("s0")
    o = torch.empty((B, T, w.H_v, w.d_v), dtype=dev["q"].dtype, device=device)
    sT = torch.empty((N, w.H_v, w.d_k, w.d_v), dtype=torch.float32, device=device)
    fn = gdr.kda_chunk_fwd if w.gate == "channel" else gdr.gdn_chunk_fwd
    ws = None

    def step(q, k, v, g, beta, s0_):
        nonlocal ws
        _, _, ws = fn(q, k, v, g, beta, s0_, cu, o=o, final_state=sT, workspace=ws)

    for _ in range(args.warmup):
        flush.zero_()
        step(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], s0)
    torch.cuda.synchronize()
    st, code = gdr.check_device_status(ws)
    if st != gdr.KDA_OK:
        raise RuntimeError(f"{w.name}: device status {code}")

    # ---- device-timed steps (inputs resident) ----
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize()
    with ClockSampler(device.index) as clocks:
        for i in range(args.steps):
            flush.zero_()
            evs[i][0].record(stream)
            step(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], s0)
            evs[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world, device)
    per = [a.elapsed_time(b) for a, b in evs]
    ms_local = sum(per) / len(per)
    ms = max_over_ranks(ms_local, world, device)
    tokens = T_total
    value = aggregate_throughput(tokens, ms, world)

    # ---- per-kernel device times: the same calls again, with launch tracing ----
    gdr.trace_enable(True)
    for i in range(args.steps):
        flush.zero_()
        step(dev["q"], dev["k"], dev["v"], dev["g"], dev["beta"], s0)
    torch.cuda.synchronize()
    recs = gdr.trace_read()
    gdr.trace_enable(False)
    per_kernel = {}
    for name, t in recs:
        per_kernel.setdefault(name, []).append(t)
    kern_ms = {k: sum(v) / len(v) for k, v in per_kernel.items()}
    dominant = max(kern_ms, key=kern_ms.get)

    algo_bytes = prefill_bytes(w, T_total, N)
    algo_flops = prefill_flops(w, T_total)
    kb = kernel_algo_bytes(dominant, w, T_total, N)
    achieved = kb / (kern_ms[dominant] / 1e3) / 1e9
    # counters are per launch of the named workload at its own size
    traffic = measured_traffic(dominant, w.name) if not tokens_override else None
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "peak_source": peaks["source"], "kernel": dominant,
                "kernel_us": round(kern_ms[dominant] * 1e3, 2), "algorithmic_bytes": kb}
    call_gbs = algo_bytes / (ms_local / 1e3) / 1e9
    t_roof = max(algo_bytes / (peaks["hbm_gbs"] * 1e9), algo_flops / (peaks["bf16_tflops"] * 1e12))
    call_roofline = {"bound": "hbm" if algo_bytes / peaks["hbm_gbs"] >= algo_flops / peaks["bf16_tflops"] / 1e3 else "tensor",
                     "algorithmic_bytes": algo_bytes, "algorithmic_flops": algo_flops,
                     "achieved_gbs": round(call_gbs, 1),
                     "achieved_tflops": round(algo_flops / (ms_local / 1e3) / 1e12, 2),
                     "roofline_us": round(t_roof * 1e6, 2),
                     "frac": round(t_roof / (ms_local / 1e3), 4),
                     "roofline_tokens_per_s": round(tokens / t_roof, 1),
                     "traffic": {k: measured_traffic(k, w.name) if not tokens_override else None
                                 for k in kern_ms}}
    kernels = {k: {"us": round(v * 1e3, 2), "launches_per_step": len(per_kernel[k]) // args.steps}
               for k, v in kern_ms.items()}
    launches = gdr_launches_per_call(w, varlen) * args.steps

    out = {
        "workload": w.name, "description": w.description,
        "value": round(value, 1), "unit": "tokens/s", "ms_per_step": round(ms, 4),
        "dtype": "bf16" if w.io_dtype == "bf16" else "f32",
        "config": {"workload": w.name, "description": w.description, "B": B, "T": T,
                   "H_qk": w.H_qk, "H_v": w.H_v, "d_k": w.d_k, "d_v": w.d_v,
                   "num_seqs": N, "tokens": T_total, "chunk": 64,
                   "l2": "flushed (256 MB write) before every timed call",
                   "parallelism": f"replicas x{world}, no collective"},
        "roofline": roofline, "call_roofline": call_roofline, "kernels": kernels,
        "clocks": clocks.summary(),
        "step_ms_min_max": [round(min(per), 4), round(max(per), 4)],
        "launches": launches, "_inputs": x,
    }

    # ---- end to end through the public API: pinned host -> device, call, back ----
    # A dense KDA batch goes through kda_chunk_fwd_host (the library's call for
    # prompts in host memory: the copies of one piece overlap the kernels of
    # the previous one); other workloads copy, call and copy back in turn.
    if with_e2e:
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()
        sT_host = torch.empty(sT.shape, dtype=sT.dtype).pin_memory()
        d_in = {k: torch.empty_like(v) for k, v in dev.items()}
        h2d = sum(v.numel() * v.element_size() for v in host.values())
        d2h = o.numel() * o.element_size() + sT.numel() * sT.element_size()
        streamed = w.gate == "channel" and not varlen
        pieces = 4
        buf = None
        e2e_ev = []
        for i in range(max(2, min(args.steps, 10)) + 1):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            if streamed:
                buf = gdr.kda_chunk_fwd_host(host["q"], host["k"], host["v"], host["g"],
                                             host["beta"], host.get("s0"), o=o_host,
                                             final_state=sT_host, device_buffer=buf,
                                             pieces=pieces, stream=stream)
            else:
                for k_, v_ in host.items():
                    d_in[k_].copy_(v_, non_blocking=True)
                step(d_in["q"], d_in["k"], d_in["v"], d_in["g"], d_in["beta"], d_in.get("s0"))
                o_host.copy_(o, non_blocking=True)
                sT_host.copy_(sT, non_blocking=True)
            b.record(stream)
            if i > 0:  # first iteration is a warm-up
                e2e_ev.append((a, b))
        torch.cuda.synchronize()
        if streamed:
            st, code = gdr.check_device_status(buf)
            if st != gdr.KDA_OK:
                raise RuntimeError(f"{w.name}: streamed prefill device status {code}")
        e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev) / len(e2e_ev)
        e2e_ms = max_over_ranks(e2e_ms, world, device)
        out["e2e"] = {"value": round(tokens * world / (e2e_ms / 1e3), 1), "unit": "tokens/s",
                      "ms_per_step": round(e2e_ms, 4), "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h,
                      "call": (f"kda_chunk_fwd_host, {pieces} pieces" if streamed else
                               "copies, then the prefill call, then copies back")}
        del buf
    del dev, o, sT, ws
    torch.cuda.empty_cache()
    return out


def gdr_launches_per_call(w: W.Workload, varlen: bool) -> int:
    """Our kernels per prefill call.  Tensor-core path (bf16, d = 128): prep and
    scan, plus the planning kernel for packed batches.  fp32 path: the chunk
    kernel, plus the cu_seqlens check for packed batches.  (The status reset is
    a memset, not a kernel.)"""
    tc = w.io_dtype == "bf16" and w.d_k == 128 and w.d_v == 128
    if tc:
        return 3 if varlen else 2
    return 1 + (1 if varlen else 0)


def bench_decode(args, device, world, peaks, stream, flush):
    import torch
    import gated_delta_rule_87_b200 as gdr
    w = W.WORKLOADS["kda_decode"]
    x = W.make_decode(w, seed=0)
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
        torch.bfloat16).to(device)
    q, k, v = bf(x.q), bf(x.k), bf(x.v)
    g = torch.from_numpy(x.g).to(device)
    beta = torch.from_numpy(x.beta).to(device)
    state = torch.from_numpy(x.initial_state).to(device)
    o = torch.empty((w.N, w.H_v, w.d_v), dtype=torch.bfloat16, device=device)
    for s in range(3):
        gdr.kda_decode_step(q[s], k[s], v[s], g[s], beta[s], state, o=o)
    torch.cuda.synchronize()
    state.copy_(torch.from_numpy(x.initial_state).to(device))
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, device)
    torch.cuda.synchronize()
    # the 512 MB state exceeds L2, so consecutive steps stream it from HBM
    a.record(stream)
    for s in range(w.steps):
        gdr.kda_decode_step(q[s], k[s], v[s], g[s], beta[s], state, o=o)
    b.record(stream)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / w.steps
    ms = max_over_ranks(ms, world, device)
    per_step = decode_bytes_per_head(w) * w.N * w.H_v
    gbs = per_step / (ms / 1e3) / 1e9
    return {"workload": w.name, "description": w.description, "steps": w.steps,
            "us_per_step": round(ms * 1e3, 2), "bytes_per_step": per_step,
            "value": round(gbs * world, 1), "unit": "GB/s (state read+write and token I/O)",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                         "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                         "traffic": measured_traffic("recurrent_kernel", w.name),
                         "peak_source": peaks["source"],
                         "kernel": "recurrent_kernel"},
            "l2": "state (512 MB) larger than L2; not flushed",
            "launches": w.steps}


def cpu_baseline(x, w, heads=None):
    """The fp64 oracle as it stands, on this host's cores, on a bounded sample."""
    import oracle
    threads = oracle.default_threads()
    if heads is None:
        heads = list(range(w.H_v))
    group = w.H_v // w.H_qk
    hk = [h // group for h in heads]
    args = (x.q32[:, hk], x.k32[:, hk], x.v32[:, heads], x.g[:, heads], x.beta[:, heads],
            None if x.initial_state is None else x.initial_state[:, heads],
            x.cu_seqlens.astype(np.int64))
    t0 = time.perf_counter()
    oracle.gated_delta(*args, threads=threads)
    dt = time.perf_counter() - t0
    tokens_equiv = x.total_tokens * len(heads) / w.H_v
    return {"value": round(tokens_equiv / dt, 2), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{len(heads)} of {w.H_v} heads x {x.total_tokens} tokens of {w.name} "
                      f"(fp64 token loop, {dt:.2f} s); tokens/s counts all {w.H_v} heads "
                      "of a token as one token"}


# --------------------------------------------------------------------------- #
# reference arm: the oracle
# --------------------------------------------------------------------------- #
def run_reference(args, world, rank):
    if rank != 0:
        return
    w = W.WORKLOADS[args.workload]
    x = W.make_prefill(w, seed=0)
    import oracle
    heads = list(range(min(w.H_v, oracle.default_threads())))
    for _ in range(args.warmup):
        cpu_baseline(x, w, heads=heads[:1])
    times = []
    for _ in range(args.steps):
        r = cpu_baseline(x, w, heads=heads)
        times.append(x.total_tokens * len(heads) / w.H_v / r["value"])
    ms = 1e3 * sum(times) / len(times)
    tokens_equiv = x.total_tokens * len(heads) / w.H_v
    value = tokens_equiv / (ms / 1e3)
    line = {
        "impl": "reference",
        "metric": "KDA prefill tokens/s (decode-step state GB/s in 'decode'), % of roofline, 1xB200",
        "value": round(value, 2), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "description": w.description,
                   "sample_heads": len(heads), "tokens": x.total_tokens},
        "cpu_baseline": {"value": round(value, 2), "unit": "tokens/s",
                         "cores": oracle.default_threads(), "kind": "oracle",
                         "sample": f"{len(heads)} of {w.H_v} heads x {x.total_tokens} tokens per step"},
        "e2e": {"value": round(value, 2), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="kda_prefill",
                    choices=[k for k, v in W.WORKLOADS.items() if v.kind == "prefill"])
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the main workload (not the other prefill configurations)")
    ap.add_argument("--tokens", type=int, default=None,
                    help="sequence length of a dense workload in place of its own "
                         "(a smaller case of the same kernels, e.g. for a profiler capture)")
    args = ap.parse_args()
    if args.tokens is not None and (W.WORKLOADS[args.workload].varlen or args.tokens < 1):
        ap.error("--tokens takes a positive length and a dense workload")
    args.warmup = max(args.warmup, 3)
    world, rank, local = dist_setup()
    if args.gpus != world:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE is {world}: launch N ranks with "
                 "torch.distributed.run (one process per GPU)")
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_ours(args, world, rank, local)


if __name__ == "__main__":
    main()
