#!/usr/bin/env python
"""Benchmark: KDA prefill tokens/s (H=32, d=128) and decode GB/s on B200, against the roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload W]

One step = one kda_fwd call (every prefill stage of the hot path: load and gate, decayed
operands, intra-chunk products, UT transform, WY factors, the chunk-serial state pass,
document resets and state I/O) over one batch of the headline workload, long-t65536: B=2,
T=65536, H=32, dk=dv=128, bf16 q/k/v/beta, fp32 log g = -softplus(N(2,1)), fp32 h0 ~ N(0,0.02^2).
Inputs are resident in HBM and larger than L2 (6.4 GB), so no flush is needed between steps.
`value` is tokens/s over all ranks (each rank runs its own batch: weak scaling, no collective
on the data path). The decode step (256 sequences x 32 heads, state in place) and the packed
8-document prefill are timed in the same run and reported under "secondary".

--impl reference times the float64 CPU oracle (the reference arm for this build) on a bounded
sample of the same workload on the host cores; under torchrun only rank 0 runs it.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

METRIC = "KDA prefill tokens/s (H=32,d=128) & decode GB/s; % of B200 roofline"
PROFILE_TRAFFIC = ROOT / "profiles" / "traffic.json"

# Algorithmic bytes per token-head at d = 128 (q, k, v bf16; log g fp32; beta bf16; o bf16)
BYTES_PER_TOKEN_HEAD = 3 * 128 * 2 + 128 * 4 + 2 + 128 * 2
STATE_BYTES = 128 * 128 * 4
# Chunked-form flops per token-head at d = 128, C = 64: 10 C d + 6 d^2 (full tiles)
FLOPS_PER_TOKEN_HEAD = 10 * 64 * 128 + 6 * 128 * 128


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def measured_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        time.sleep(0.3)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------ helpers

KERNEL_SOURCES = {
    "kda_decode_d128": ["kda_decode.cu", "kda_internal.cuh"],
    "kda_decode_tokens_d128": ["kda_decode.cu", "kda_internal.cuh"],
    "kda_out_norm_gated": ["kda_norm.cu", "kda_internal.cuh"],
    "kda_recurrent": ["kda_recurrent.cu", "kda_internal.cuh"],
    "kda_chunk64": ["kda_chunk64.cu", "kda_sm100.cuh", "kda_internal.cuh", "kda_tma.cuh"],
    "kda_chunk64_intra": ["kda_intra.cu", "kda_sm100.cuh", "kda_internal.cuh", "kda_tma.cuh"],
    "kda_chunk_scan": ["kda_scan.cu", "kda_scan.cuh", "kda_sm100.cuh", "kda_internal.cuh",
                       "kda_tma.cuh"],
    "kda_short_conv": ["kda_conv.cu", "kda_internal.cuh"],
}


def source_digest(kernel: str):
    """Digest of the sources a kernel is built from, with their per-file compiler flags (its
    profile is stale once either changes)."""
    from gated_delta_rule_144_b200.build import FILE_FLAGS
    h = hashlib.sha256()
    for name in KERNEL_SOURCES.get(kernel, []):
        p = ROOT / "gated_delta_rule_144_b200" / "csrc" / name
        h.update(name.encode())
        h.update(p.read_bytes() if p.exists() else b"")
        if FILE_FLAGS.get(name):
            h.update(" ".join(FILE_FLAGS[name]).encode())
    return h.hexdigest()[:16]


def committed_traffic(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary, if it is current. For a
    path of several kernels ("a+b"), the sum over its kernels, or None if any is missing."""
    if "+" in kernel:
        parts = [committed_traffic(k, workload) for k in kernel.split("+")]
        return None if any(x is None for x in parts) else sum(parts)
    if not PROFILE_TRAFFIC.exists():
        return None
    try:
        d = json.loads(PROFILE_TRAFFIC.read_text())
        e = d.get(kernel)
        if not e or e.get("source_digest") != source_digest(kernel) \
                or e.get("workload") != workload:
            return None
        return float(e["dram_bytes_per_launch"])
    except (ValueError, KeyError):
        return None


def time_launches(fn, steps, stream):
    """Per-launch CUDA-event timing on the launching stream. Returns (total_ms, [ms...])."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for s, e in ev:
        s.record(stream)
        fn()
        e.record(stream)
    t1.record(stream)
    t1.synchronize()
    return t0.elapsed_time(t1), [s.elapsed_time(e) for s, e in ev]


def time_launches_flushed(fn, steps, stream, scratch):
    """Per-launch CUDA-event timing with L2 flushed before every launch (for workloads whose
    inputs fit in L2): a write over `scratch` (larger than L2) runs between launches, outside
    the event pairs. Returns the list of per-launch ms."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for s, e in ev:
        scratch.zero_()
        s.record(stream)
        fn()
        e.record(stream)
    ev[-1][1].synchronize()
    return [s.elapsed_time(e) for s, e in ev]


def max_over_ranks(x: float, world: int, device):
    from gated_delta_rule_144_b200 import shard
    return shard.max_over_ranks(x, device) if world > 1 else x


def sum_over_ranks(x: float, world: int, device):
    from gated_delta_rule_144_b200 import shard
    return shard.sum_over_ranks(x, device) if world > 1 else x


def barrier(world):
    if world > 1:
        from gated_delta_rule_144_b200 import shard
        shard.barrier()


# ------------------------------------------------------------------------------ our arm

def prefill_bytes(inp) -> int:
    th = inp["T"] * inp["B"] * inp["H"]
    states = inp["N"] * inp["H"] * STATE_BYTES
    return th * BYTES_PER_TOKEN_HEAD + states * (2 if inp["h0"] is not None else 1)


def workspace_for(kda, B, T, H, N, args, dev):
    """The call's workspace, allocated once outside the timed region (None when 0 bytes)."""
    size = (kda.fwd_workspace_size_min if args.fused else kda.fwd_workspace_size)(
        B, T, H, 128, 128, N, torch.bfloat16, args.chunk_size)
    return torch.empty(size, dtype=torch.uint8, device=dev) if size > 0 else None


def run_ours(args):
    import gated_delta_rule_144_b200 as kda
    from gated_delta_rule_144_b200 import synth

    rank, local, world = env_rank()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    stream = torch.cuda.current_stream(dev)
    wl = synth.WORKLOADS[args.workload]

    # ---- headline: prefill on the workload, one batch per rank
    from gated_delta_rule_144_b200 import shard
    inp = synth.prefill_inputs(wl, device=dev, seed=shard.rank_seed(1000 + wl.index, rank))
    B, T, H, dk, dv, N = inp["B"], inp["T"], inp["H"], inp["dk"], inp["dv"], inp["N"]
    o = torch.empty((B, T, H, dv), dtype=inp["q"].dtype, device=dev)
    hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev)
    ws = workspace_for(kda, B, T, H, N, args, dev)

    def step():
        kda.fwd(inp["q"], inp["k"], inp["v"], inp["log_g"], inp["beta"], h0=inp["h0"],
                cu_seqlens=inp["cu_seqlens"], o=o, hT=hT, chunk_size=args.chunk_size,
                workspace=ws, fused=args.fused)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if kda.get_device_error() != 0:
        raise RuntimeError("device error during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    total_ms, per = time_launches(step, args.steps, stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    if kda.get_device_error() != 0:
        raise RuntimeError("device error in the timed region")

    ms_max = max_over_ranks(total_ms, world, dev)
    tokens_rank = B * T
    tokens_all = sum_over_ranks(float(tokens_rank), world, dev)
    value = tokens_all * args.steps / (ms_max / 1e3)
    launch_ms = statistics.fmean(per)
    hbm_peak, tc_peak, peak_kind = measured_peaks()
    bytes_launch = prefill_bytes(inp)
    achieved = bytes_launch / (launch_ms / 1e3) / 1e9
    algo = kda.fwd_algorithm(B, T, H, dk, dv, N, inp["q"].dtype, args.chunk_size,
                             varlen=inp["cu_seqlens"] is not None)
    packed = inp["cu_seqlens"] is not None
    if algo != kda.CHUNK_64:
        kernel_name, launches = "kda_recurrent", 1
    elif args.fused:
        kernel_name, launches = "kda_chunk64", 1 + (1 if packed and 2 <= N <= 2048 else 0)
    else:   # split: intra-chunk kernel + state pass per chunk segment (+ chunk map and document
        # order if packed)
        kernel_name = "kda_chunk64_intra+kda_chunk_scan"
        segs = kda.fwd_split_segments(B, T, H, dk, dv, N, inp["q"].dtype, args.chunk_size,
                                      varlen=packed)
        launches = 2 * segs + ((2 if 2 <= N <= 2048 else 1) if packed else 0)
        if kda.fwd_scan_segments(B, T, H, dk, dv, N, inp["q"].dtype, args.chunk_size,
                                 varlen=packed) >= 3:
            # two-level state pass: intra-chunk kernel, segment 0 and the maps, their chain,
            # the remaining segments
            launches = 5
    traffic = committed_traffic(kernel_name, wl.name)
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                "traffic": traffic, "peak_kind": peak_kind, "kernel": kernel_name,
                "launch": ("one kda_fwd call: intra-chunk kernel then state pass"
                           if "+" in kernel_name else "one kda_fwd call"),
                "algorithmic_bytes_per_launch": bytes_launch,
                "avg_launch_ms": round(launch_ms, 4),
                "flops_per_launch": FLOPS_PER_TOKEN_HEAD * B * T * H,
                "tensor_frac_if_tc": round(FLOPS_PER_TOKEN_HEAD * B * T * H /
                                           (launch_ms / 1e3) / (tc_peak * 1e12), 4)}

    # ---- end to end through the public API with host buffers
    e2e = run_e2e(kda, inp, args, stream, world, dev)

    secondary = {}
    if not args.no_secondary:
        secondary = run_secondary(kda, synth, args, dev, stream, world, rank)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args)

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_max / args.steps, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "B": B, "T": T, "H": H, "dk": dk, "dv": dv,
                       "global_batch": B * world, "seq_len": T, "h0": inp["h0"] is not None,
                       "log_g": "-softplus(N(%g,1))" % wl.decay_mu,
                       "parallelism": "dp%d" % world, "l2": "inputs larger than L2",
                       "chunk_size": args.chunk_size, "path": kernel_name},
            "roofline": roofline, "e2e": e2e, "gpu_launches": args.steps * launches,
            "clocks": clk, "cpu_baseline": cpu, "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(kda, inp, args, stream, world, dev):
    """Same metric through kda.fwd with pinned host inputs copied in and o, hT copied out, every
    step. Steps run as a serving loop would run them: step i's inputs go up on one copy stream and
    its outputs come down on another, so the download of step i overlaps the upload of step i + 1
    (PCIe is full duplex); the device buffers are double-buffered and events order their reuse.
    Every step's copies are inside the timed region."""
    keys = ("q", "k", "v", "log_g", "beta", "h0", "cu_seqlens")
    host = {k: (inp[k].cpu().pin_memory() if inp[k] is not None else None) for k in keys}
    nbuf = 2
    d_in = [{k: (torch.empty_like(inp[k]) if inp[k] is not None else None) for k in keys}
            for _ in range(nbuf)]
    B, T, H, dv, N, dk = inp["B"], inp["T"], inp["H"], inp["dv"], inp["N"], inp["dk"]
    o = [torch.empty((B, T, H, dv), dtype=inp["q"].dtype, device=dev) for _ in range(nbuf)]
    hT = [torch.empty((N, H, dk, dv), dtype=torch.float32, device=dev) for _ in range(nbuf)]
    ws = workspace_for(kda, B, T, H, N, args, dev)   # the calls run in order on `stream`
    o_h = [torch.empty(o[0].shape, dtype=o[0].dtype).pin_memory() for _ in range(nbuf)]
    hT_h = [torch.empty(hT[0].shape, dtype=hT[0].dtype).pin_memory() for _ in range(nbuf)]
    h2d = sum(t.numel() * t.element_size() for t in host.values() if t is not None)
    d2h = o[0].numel() * o[0].element_size() + hT[0].numel() * hT[0].element_size()
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(nbuf)]     # inputs of buffer b uploaded
    ev_done = [torch.cuda.Event() for _ in range(nbuf)]   # the call on buffer b finished
    ev_out = [torch.cuda.Event() for _ in range(nbuf)]    # outputs of buffer b downloaded

    def step(i):
        b = i % nbuf
        s_in.wait_event(ev_done[b])   # the call two steps back has read these inputs
        with torch.cuda.stream(s_in):
            for k in keys:
                if host[k] is not None:
                    d_in[b][k].copy_(host[k], non_blocking=True)
        ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        stream.wait_event(ev_out[b])  # the outputs two steps back have been read
        g = d_in[b]
        kda.fwd(g["q"], g["k"], g["v"], g["log_g"], g["beta"], h0=g["h0"],
                cu_seqlens=g["cu_seqlens"], o=o[b], hT=hT[b], chunk_size=args.chunk_size,
                workspace=ws, fused=args.fused, stream=stream)
        ev_done[b].record(stream)
        s_out.wait_event(ev_done[b])
        with torch.cuda.stream(s_out):
            o_h[b].copy_(o[b], non_blocking=True)
            hT_h[b].copy_(hT[b], non_blocking=True)
        ev_out[b].record(s_out)

    steps = max(1, min(args.steps, args.e2e_steps))
    for i in range(nbuf):   # warm-up: one step on each buffer
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s_in)   # every stream is idle here: the first timed work is the first upload
    for i in range(nbuf, nbuf + steps):
        step(i)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    t1.record(stream)
    t1.synchronize()
    total_ms = t0.elapsed_time(t1)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(total_ms, world, dev)
    tokens_all = sum_over_ranks(float(B * T), world, dev)
    return {"value": round(tokens_all * steps / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "pipelined": "download of step i overlaps upload of step i + 1"}


def run_secondary(kda, synth, args, dev, stream, world, rank):
    out = {}
    hbm_peak, _, _ = measured_peaks()
    from gated_delta_rule_144_b200 import shard
    if args.workload == "long-t65536":
        # the long-context workload with the slow decay its description names (reported, not a
        # target): log g = -softplus(N(-2, 1)), the same shapes, a new draw
        sl = synth.prefill_inputs("long-t65536-slow", device=dev, seed=shard.rank_seed(1099, rank))
        so = torch.empty_like(sl["v"])
        shT = torch.empty((sl["N"], sl["H"], 128, 128), dtype=torch.float32, device=dev)
        sws = workspace_for(kda, sl["B"], sl["T"], sl["H"], sl["N"], args, dev)

        def sstep():
            kda.fwd(sl["q"], sl["k"], sl["v"], sl["log_g"], sl["beta"], h0=sl["h0"], o=so,
                    hT=shT, chunk_size=args.chunk_size, workspace=sws, fused=args.fused)

        for _ in range(max(3, args.warmup)):
            sstep()
        torch.cuda.synchronize()
        barrier(world)
        ssteps = max(args.steps, 5)
        total_ms, _ = time_launches(sstep, ssteps, stream)
        barrier(world)
        ms = max_over_ranks(total_ms, world, dev) / ssteps
        by = prefill_bytes(sl)
        out["long_slow"] = {"workload": "long-t65536-slow", "log_g": "-softplus(N(-2,1))",
                            "ms_per_step": round(ms, 4),
                            "tokens/s": round(sl["B"] * sl["T"] * world / (ms / 1e3), 1),
                            "roofline_frac": round(by / (ms / 1e3) / 1e9 / hbm_peak, 4)}
        del sl, so, shT, sws
        torch.cuda.empty_cache()
    # decode: 256 sequences x 32 heads, fp32 128x128 state updated in place every step
    d = synth.decode_inputs("decode-n256", device=dev, seed=shard.rank_seed(1003, rank))
    od = torch.empty_like(d["v"])

    def dstep():
        kda.decode_step(d["q"], d["k"], d["v"], d["log_g"], d["beta"], d["S"], o=od)

    for _ in range(max(3, args.warmup)):
        dstep()
    torch.cuda.synchronize()
    barrier(world)
    steps = max(args.steps, 20)
    total_ms, per = time_launches(dstep, steps, stream)
    barrier(world)
    ms = max_over_ranks(total_ms, world, dev) / steps
    state = d["S"].numel() * 4
    io = sum(d[k].numel() * d[k].element_size() for k in ("q", "k", "v", "log_g", "beta"))
    io += od.numel() * od.element_size()
    by = 2 * state + io
    gbs = by / (ms / 1e3) / 1e9
    out["decode"] = {"workload": "decode-n256", "N": 256, "H": 32, "dk": 128, "dv": 128,
                     "bytes_per_step": by, "ms_per_step": round(ms, 4),
                     "GB/s": round(gbs * world, 1), "GB/s_per_gpu": round(gbs, 1),
                     "roofline_frac": round(gbs / hbm_peak, 4), "peak": hbm_peak,
                     "kernel": "kda_decode_d128",
                     "traffic": committed_traffic("kda_decode_d128", "decode-n256")}
    del d, od
    # four rows per sequence against the decode state (kda_decode_tokens), in place
    d = synth.decode_tokens_inputs("decode-rows-n256-t4", device=dev,
                                   seed=shard.rank_seed(1053, rank))
    od = torch.empty_like(d["v"])

    def rstep():
        kda.decode_tokens(d["q"], d["k"], d["v"], d["log_g"], d["beta"], d["S"], o=od)

    for _ in range(max(3, args.warmup)):
        rstep()
    torch.cuda.synchronize()
    barrier(world)
    total_ms, per = time_launches(rstep, steps, stream)
    barrier(world)
    ms = max_over_ranks(total_ms, world, dev) / steps
    state = d["S"].numel() * 4
    io = sum(d[k].numel() * d[k].element_size() for k in ("q", "k", "v", "log_g", "beta"))
    io += od.numel() * od.element_size()
    by = 2 * state + io
    gbs = by / (ms / 1e3) / 1e9
    out["decode_rows"] = {"workload": "decode-rows-n256-t4", "N": 256, "T": 4, "H": 32,
                          "bytes_per_step": by, "ms_per_step": round(ms, 4),
                          "GB/s": round(gbs * world, 1), "GB/s_per_gpu": round(gbs, 1),
                          "roofline_frac": round(gbs / hbm_peak, 4), "peak": hbm_peak,
                          "tokens/s": round(256 * 4 * world / (ms / 1e3), 1),
                          "kernel": "kda_decode_tokens_d128",
                          "traffic": committed_traffic("kda_decode_tokens_d128",
                                                       "decode-rows-n256-t4")}
    del d, od
    # packed 8-document prefill (H = 32)
    p = synth.prefill_inputs("packed-8docs", device=dev, seed=shard.rank_seed(1002, rank))
    o = torch.empty_like(p["v"])
    hT = torch.empty((p["N"], p["H"], 128, 128), dtype=torch.float32, device=dev)
    ws = workspace_for(kda, 1, p["T"], p["H"], p["N"], args, dev)

    def pstep():
        kda.fwd(p["q"], p["k"], p["v"], p["log_g"], p["beta"], cu_seqlens=p["cu_seqlens"],
                o=o, hT=hT, chunk_size=args.chunk_size, workspace=ws, fused=args.fused)

    for _ in range(max(3, args.warmup)):
        pstep()
    torch.cuda.synchronize()
    barrier(world)
    total_ms, per = time_launches(pstep, args.steps, stream)
    barrier(world)
    ms = max_over_ranks(total_ms, world, dev) / args.steps
    by = prefill_bytes(p)
    out["packed_prefill"] = {"workload": "packed-8docs", "lengths": p["lengths"],
                             "tokens": p["T"], "ms_per_step": round(ms, 4),
                             "tokens/s": round(p["T"] * world / (ms / 1e3), 1),
                             "roofline_frac": round(by / (ms / 1e3) / 1e9 / hbm_peak, 4)}
    # single-sequence prefill, B=1, T=4096, H=16: its 102 MB of inputs fit in L2, so L2 is
    # flushed (a 256 MiB write) before every timed launch, outside the launch's event pair
    c1 = synth.prefill_inputs("prefill-t4096", device=dev, seed=shard.rank_seed(1001, rank))
    o1 = torch.empty_like(c1["v"])
    h1 = torch.empty((c1["N"], c1["H"], 128, 128), dtype=torch.float32, device=dev)
    ws1 = workspace_for(kda, c1["B"], c1["T"], c1["H"], c1["N"], args, dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def c1step():
        kda.fwd(c1["q"], c1["k"], c1["v"], c1["log_g"], c1["beta"], o=o1, hT=h1,
                chunk_size=args.chunk_size, workspace=ws1, fused=args.fused)

    for _ in range(max(3, args.warmup)):
        c1step()
    torch.cuda.synchronize()
    barrier(world)
    per1 = time_launches_flushed(c1step, max(args.steps, 20), stream, flush)
    barrier(world)
    ms1 = max_over_ranks(statistics.fmean(per1), world, dev)
    by1 = prefill_bytes(c1)
    segs1 = kda.fwd_split_segments(1, c1["T"], c1["H"], 128, 128, 1, c1["q"].dtype,
                                   args.chunk_size)
    pscan1 = kda.fwd_scan_segments(1, c1["T"], c1["H"], 128, 128, 1, c1["q"].dtype,
                                   args.chunk_size)
    ms1_plain = None
    if pscan1 >= 3:
        # the same call with the plain state pass (one chain per SM), for comparison
        prev = os.environ.get("KDA_SCAN_SEGMENTS")
        os.environ["KDA_SCAN_SEGMENTS"] = "0"
        try:
            for _ in range(3):
                c1step()
            torch.cuda.synchronize()
            barrier(world)
            perp = time_launches_flushed(c1step, max(args.steps, 20), stream, flush)
            barrier(world)
            ms1_plain = round(max_over_ranks(statistics.fmean(perp), world, dev), 5)
        finally:
            if prev is None:
                del os.environ["KDA_SCAN_SEGMENTS"]
            else:
                os.environ["KDA_SCAN_SEGMENTS"] = prev
    out["prefill_t4096"] = {"workload": "prefill-t4096", "B": 1, "T": c1["T"], "H": c1["H"],
                            "ms_per_step": round(ms1, 5),
                            "tokens/s": round(c1["T"] * world / (ms1 / 1e3), 1),
                            "bytes_per_step": by1,
                            "roofline_frac": round(by1 / (ms1 / 1e3) / 1e9 / hbm_peak, 4),
                            "l2": "flushed before every launch (256 MiB write)",
                            "ms_plain_state_pass": ms1_plain,
                            "kernel": "kda_chunk64" if args.fused else
                            "kda_chunk64_intra+kda_chunk_scan (two-level state pass, %d "
                            "segments)" % pscan1 if pscan1 >= 3 else
                            "kda_chunk64_intra+kda_chunk_scan (%d segment%s)" % (
                                segs1, "" if segs1 == 1 else "s")}
    del c1, o1, h1, ws1, flush
    # gated per-head RMSNorm epilogue on the same workload: kda_fwd_normed against the plain call
    # followed by the separate norm pass through the Python API
    gen = torch.Generator(device=dev)
    gen.manual_seed(shard.rank_seed(1090, rank))
    gate = torch.randn(o.shape, generator=gen, device=dev).to(o.dtype)
    nw = torch.rand(128, generator=gen, device=dev) + 0.5

    def nstep():
        kda.fwd(p["q"], p["k"], p["v"], p["log_g"], p["beta"], cu_seqlens=p["cu_seqlens"],
                o=o, hT=hT, chunk_size=args.chunk_size, workspace=ws, fused=args.fused,
                out_norm=(gate, nw, 1e-6))

    def ustep():
        pstep()
        kda.out_norm_gated(o, gate, nw, 1e-6, y=o)

    res = {}
    for name, fn in (("normed", nstep), ("separate", ustep)):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        barrier(world)
        total_ms, _ = time_launches(fn, args.steps, stream)
        barrier(world)
        res[name] = round(max_over_ranks(total_ms, world, dev) / args.steps, 4)
    out["packed_prefill_normed"] = {"workload": "packed-8docs", "epilogue": "gated RMSNorm",
                                    "ms_normed_call": res["normed"],
                                    "ms_plain_then_norm": res["separate"],
                                    "ms_plain": out["packed_prefill"]["ms_per_step"]}
    # the input prologue (kda_short_conv): one projection of the packed workload, [1, T, 32 x 128]
    # bf16, W = 4 taps, SiLU, L2 norm per head (how q and k enter the recurrence)
    gen = torch.Generator(device=dev)
    gen.manual_seed(shard.rank_seed(1097, rank))
    px = torch.randn((1, p["T"], 32 * 128), generator=gen, device=dev).to(torch.bfloat16)
    pw = torch.randn((32 * 128, 4), generator=gen, device=dev) * 0.5
    py = torch.empty_like(px)

    def cstep():
        kda.short_conv(px, pw, p["cu_seqlens"], activation="silu", norm_group=128, y=py)

    for _ in range(3):
        cstep()
    torch.cuda.synchronize()
    barrier(world)
    total_ms, _ = time_launches(cstep, max(args.steps, 20), stream)
    barrier(world)
    ms = max_over_ranks(total_ms, world, dev) / max(args.steps, 20)
    by = 2 * px.numel() * 2 + pw.numel() * 4 + p["cu_seqlens"].numel() * 4
    out["prologue"] = {"workload": "packed-8docs (one of q, k, v: 32 heads x 128 channels)",
                       "W": 4, "activation": "silu", "norm_group": 128,
                       "ms_per_call": round(ms, 4), "bytes_per_call": by,
                       "roofline_frac": round(by / (ms / 1e3) / 1e9 / hbm_peak, 4),
                       "kernel": "short_conv_kernel",
                       "traffic": committed_traffic("kda_short_conv", "packed-8docs")}
    del px, pw, py
    # gradients (kda_bwd) on the T=4096, H=16 workload: upstream do and dhT drawn once
    b = synth.prefill_inputs("prefill-t4096", device=dev, seed=shard.rank_seed(1001, rank))
    gen = torch.Generator(device=dev)
    gen.manual_seed(shard.rank_seed(1095, rank))
    bdo = torch.randn(b["v"].shape, generator=gen, device=dev).to(b["v"].dtype)
    bdh = torch.randn((b["N"], b["H"], 128, 128), generator=gen, device=dev)
    bws = torch.empty(kda.bwd_workspace_size(b["B"], b["T"], b["H"], 128, 128, b["N"],
                                             b["q"].dtype), dtype=torch.uint8, device=dev)

    def bstep():
        kda.bwd(b["q"], b["k"], b["v"], b["log_g"], b["beta"], bdo, h0=b["h0"], dhT=bdh,
                workspace=bws)

    bsteps = max(1, min(args.steps, 5))
    for _ in range(3):
        bstep()
    torch.cuda.synchronize()
    barrier(world)
    total_ms, _ = time_launches(bstep, bsteps, stream)
    barrier(world)
    ms = max_over_ranks(total_ms, world, dev) / bsteps
    th = b["B"] * b["T"] * b["H"]
    # algorithmic bytes: q, k, v, do (dtype) and log g, beta read; dq, dk, dv, dlog_g (fp32) and
    # dbeta written; h0, dhT read and dh0 written per chain
    esz = b["q"].element_size()
    states = (2 + (b["h0"] is not None)) * b["N"] * b["H"] * STATE_BYTES
    by = th * (4 * 128 * esz + 128 * 4 + esz + 4 * 128 * 4 + 4) + states
    out["bwd"] = {"workload": "prefill-t4096", "B": b["B"], "T": b["T"], "H": b["H"],
                  "ms_per_step": round(ms, 4),
                  "tokens/s": round(b["B"] * b["T"] * world / (ms / 1e3), 1),
                  "bytes_per_step": by,
                  "roofline_frac": round(by / (ms / 1e3) / 1e9 / hbm_peak, 5),
                  "kernel": "kda_bwd (fp32 CUDA cores, 16 warps per chain: 8 value columns each)"}
    del b, bdo, bdh, bws
    if kda.get_device_error() != 0:
        raise RuntimeError("device error in the secondary runs")
    return out


# ------------------------------------------------------------------------------ CPU oracle

def oracle_sample(wl, tokens):
    """Bounded sample of the workload for the float64 oracle: one sequence, all heads."""
    from gated_delta_rule_144_b200 import synth
    inp = synth.prefill_inputs(wl, device="cpu", B=1, T=tokens)
    f = lambda t: None if t is None else t.float().numpy()
    return {k: f(inp[k]) for k in ("q", "k", "v", "log_g", "beta", "h0")}, inp


def cpu_baseline(wl, args):
    import oracle
    tokens = args.cpu_tokens
    arrays, inp = oracle_sample(wl, tokens)
    t0 = time.perf_counter()
    oracle.kda_fwd(arrays["q"], arrays["k"], arrays["v"], arrays["log_g"], arrays["beta"],
                   h0=arrays["h0"])
    dt = time.perf_counter() - t0
    return {"value": round(tokens / dt, 1), "unit": "tokens/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": "one sequence of %s, first %d tokens, all %d heads (%.1f s)" % (
                wl.name, tokens, inp["H"], dt)}


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return
    import oracle
    from gated_delta_rule_144_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    tokens = args.ref_tokens
    arrays, inp = oracle_sample(wl, tokens)
    run = lambda: oracle.kda_fwd(arrays["q"], arrays["k"], arrays["v"], arrays["log_g"],
                                 arrays["beta"], h0=arrays["h0"])
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = time.perf_counter() - t0
    value = tokens * args.steps / dt
    sample = "one sequence of %s, first %d tokens, all %d heads, per step" % (
        wl.name, tokens, inp["H"])
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 1),
            "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3 / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "B": wl.B, "T": wl.T, "H": wl.H, "dk": wl.dk,
                       "dv": wl.dv, "sample_tokens": tokens},
            "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s",
                             "cores": oracle.max_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """Warm-up plus K launches of one kernel, no timing: the command the ncu captures run."""
    import gated_delta_rule_144_b200 as kda
    from gated_delta_rule_144_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    if args.profile_case == "decode":
        d = synth.decode_inputs("decode-n256", device=dev)
        fn = lambda: kda.decode_step(d["q"], d["k"], d["v"], d["log_g"], d["beta"], d["S"])
    elif args.profile_case == "decode-rows":
        d = synth.decode_tokens_inputs("decode-rows-n256-t4", device=dev)
        fn = lambda: kda.decode_tokens(d["q"], d["k"], d["v"], d["log_g"], d["beta"], d["S"])
    elif args.profile_case == "bwd":
        kw = {} if args.profile_tokens <= 0 else {"T": args.profile_tokens}
        b = synth.prefill_inputs("prefill-t4096", device=dev, **kw)
        gen = torch.Generator(device=dev)
        gen.manual_seed(1095)
        bdo = torch.randn(b["v"].shape, generator=gen, device=dev).to(b["v"].dtype)
        bdh = torch.randn((b["N"], b["H"], 128, 128), generator=gen, device=dev)
        fn = lambda: kda.bwd(b["q"], b["k"], b["v"], b["log_g"], b["beta"], bdo, h0=b["h0"],
                             dhT=bdh)
    elif args.profile_case == "conv":
        p = synth.prefill_inputs("packed-8docs", device=dev)
        gen = torch.Generator(device=dev)
        gen.manual_seed(1097)
        px = torch.randn((1, p["T"], 32 * 128), generator=gen, device=dev).to(torch.bfloat16)
        pw = torch.randn((32 * 128, 4), generator=gen, device=dev) * 0.5
        fn = lambda: kda.short_conv(px, pw, p["cu_seqlens"], activation="silu", norm_group=128)
    elif args.profile_case == "norm":
        p = synth.prefill_inputs("packed-8docs", device=dev)
        o = torch.randn(p["v"].shape, device=dev).to(p["v"].dtype)
        gate = torch.randn(o.shape, device=dev).to(o.dtype)
        nw = torch.rand(128, device=dev) + 0.5
        fn = lambda: kda.out_norm_gated(o, gate, nw, 1e-6)
    else:
        name = args.workload if args.profile_case == "prefill" else "packed-8docs"
        kw = {} if args.profile_tokens <= 0 else {"T": args.profile_tokens}
        p = synth.prefill_inputs(name, device=dev, **kw)
        ws = workspace_for(kda, p["B"], p["T"], p["H"], p["N"], args, dev)
        fn = lambda: kda.fwd(p["q"], p["k"], p["v"], p["log_g"], p["beta"], h0=p["h0"],
                             cu_seqlens=p["cu_seqlens"], chunk_size=args.chunk_size,
                             workspace=ws, fused=args.fused)
    for _ in range(args.warmup + args.steps):
        fn()
    torch.cuda.synchronize()
    st = kda.get_device_error()
    print(json.dumps({"profile_case": args.profile_case, "launches": args.warmup + args.steps,
                      "device_error": st}))
    if st != 0:
        sys.exit(1)


def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[1])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long-t65536")
    ap.add_argument("--chunk-size", type=int, default=0)
    ap.add_argument("--fused", action="store_true",
                    help="run the fused chunked kernel (minimum workspace) instead of the split path")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-tokens", type=int, default=32768)
    ap.add_argument("--ref-tokens", type=int, default=4096)
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile-case",
                    choices=["prefill", "decode", "decode-rows", "packed", "norm", "bwd", "conv"],
                    default=None,
                    help="run only warm-up + steps launches of one case (for ncu captures)")
    ap.add_argument("--profile-tokens", type=int, default=0,
                    help="with --profile-case prefill: tokens per sequence (0 = workload's)")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warm-up raised to 3 (minimum)")
        args.warmup = 3
    _, _, world = env_rank()
    if args.gpus != world and world > 1:
        log("note: --gpus %d but WORLD_SIZE %d; using WORLD_SIZE" % (args.gpus, world))
    if args.profile_case:
        run_profile_case(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
