#!/usr/bin/env python
"""Selective-scan (Mamba S6) benchmark on B200: tokens*channels/s, fwd + bwd.

A step is one training pass of the scan over one batch: ss_fwd (y and the
64-step state checkpoints) followed by ss_bwd (all gradients, including the
deterministic channel/batch reduction), on the Mamba-2.8b layer shape
(batch 4, d_inner 5120, d_state 16, L 4096, bf16 storage, fp32 arithmetic).
With N > 1 ranks each rank runs its own batch (weak scaling) and the
parameter gradients dA, dD, ddelta_bias are all-reduced over NCCL -- the only
exchange data-parallel training of this layer has.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Rank 0 prints one JSON line.  Kernel-only `value` is timed with CUDA events on
the launching stream with inputs resident in HBM (inputs larger than L2);
`e2e` repeats the step through the same public API with host buffers, the
host->device copies of the inputs and device->host copies of every output
inside the timed region.  `roofline` reports the dominant kernel against the
arithmetic unit that bounds it, `cpu_baseline` the fp64 oracle on this host.
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

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "selective-scan tokens*channels/s, fwd+bwd"
UNIT = "tokens*channels/s"
WORKLOAD = "mamba2.8b_layer"

# Algorithmic work per token*channel at d_state N = 16: the operations the definition
# needs, counted per state and per token (an FFMA counts as one FP32 op).
FWD_MUFU_PER_TC = 20      # 16 decays exp(Delta*A) + softplus (exp, log) + SiLU (exp, rcp)
BWD_FP32_PER_TC = 260     # 15 per (t, n) recompute + adjoint ops + ~20 per-token ops
MUFU_PER_SM_CLK = 16      # SFU results per SM per clock (4 per sub-partition)
FP32_PER_SM_CLK = 128     # FP32 lanes per SM per clock (an FFMA counts as one op)


# The sources the selective-scan kernels of the timed step are compiled and
# launched from (the SSD, conv1d and decode kernels are not in that step).
SCAN_SOURCES = ["ss_api.cu", "ss_bwd.cu", "ss_bwd_ch.cu", "ss_device.cuh", "ss_fwd.cu", "ss_internal.h"]


def sources_digest():
    """sha256 over the sources of the timed step's kernels and the ABI header:
    identifies the build a traffic capture was taken from."""
    import hashlib
    csrc = os.path.join(ROOT, "selective_state_space_11_b200", "csrc")
    h = hashlib.sha256()
    for f in SCAN_SOURCES + ["../../include/ss.h"]:
        with open(os.path.join(csrc, f), "rb") as fh:
            h.update(f.encode() + b"\0" + fh.read())
    return h.hexdigest()


def profiled_traffic(workload):
    """DRAM bytes per launch of each pass from the committed ncu capture of this
    workload, or {} when the kernels changed since the capture was taken."""
    path = os.path.join(ROOT, "profiles", f"traffic_{workload}.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return {}
    if rec.get("sources_sha256") != sources_digest():
        return {}
    return rec.get("bytes_per_launch", {})


def peaks(sms):
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    mp = {}
    if os.path.exists(path):
        with open(path) as f:
            mp = json.load(f)
    clk = float(mp.get("sm_max_mhz", 1965.0)) * 1e6
    return dict(
        hbm_gbs=float(mp.get("hbm_gbs", 6650.0)),
        hbm_src="measured" if "hbm_gbs" in mp else "fallback",
        mufu=sms * MUFU_PER_SM_CLK * clk,
        fp32=sms * FP32_PER_SM_CLK * clk,
        clock_mhz=clk / 1e6,
    )


# ---------------------------------------------------------------- clocks ----
class ClockSampler:
    """nvidia-smi samples of this GPU's clocks and throttle reasons."""

    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        t0 = time.time()
        while not self.lines and time.time() - t0 < 5:
            time.sleep(0.01)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self, t_begin, t_end):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.05)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [l for (ts, l) in self.lines if t_begin - 0.03 <= ts <= t_end + 0.03]
        if not rows:  # keep the nearest samples if the region was shorter than a period
            rows = [l for (_, l) in self.lines][-2:]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            f = [x.strip() for x in r.split(",")]
            if len(f) < len(self.FIELDS):
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for nm, v in zip(names, f[4:8]):
                if v.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_uuid(dev):
    import torch
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


# ------------------------------------------------------------- our arm ------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from selective_state_space_11_b200 import build as ssbuild
    ssbuild.build()
    from selective_state_space_11_b200 import dist as ssdist
    from selective_state_space_11_b200 import inputs as gen
    from selective_state_space_11_b200 import ops

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = gen.WORKLOADS[args.workload]
    bsz, dim, N, L = w.batch, w.dim, w.dstate, (args.seqlen or w.seqlen)
    tc_rank = bsz * dim * L
    p = gen.make_inputs(bsz, dim, N, L, w.dtype, w.seed + (7 * rank if world > 1 else 0), device=dev)
    nck = (L + 63) // 64
    y = torch.empty_like(p["u"])
    ck = torch.empty(bsz, dim, nck, N, device=dev, dtype=torch.float32)
    # dA, dD, ddelta_bias packed in one buffer: one all-reduce for N > 1
    pgrad, pviews = ssdist.param_grad_buffer(dim, N, dev)
    gout = dict(du=torch.empty_like(p["u"]), ddelta=torch.empty_like(p["u"]),
                dz=torch.empty_like(p["u"]), **pviews,
                dB=torch.empty(bsz, N, L, device=dev, dtype=torch.float32),
                dC=torch.empty(bsz, N, L, device=dev, dtype=torch.float32))
    ws = torch.empty(ops.lib().ss_bwd_workspace_size(bsz, dim, N, L), device=dev,
                     dtype=torch.uint8)
    fpath, nseg = ops.fwd_path(bsz, dim, L)
    bvariant, ngroups = ops.bwd_path(bsz, dim, L, w.dtype)
    fws_n = ops.lib().ss_fwd_workspace_size(bsz, dim, N, L)
    fws = torch.empty(max(fws_n, 16), device=dev, dtype=torch.uint8)
    # fwd: 1 kernel (3 on the chunk-parallel path); bwd: states, reverse walk, 2 reductions,
    # plus (chunk groups) a second states launch with the carry maps and the group-carry scan
    launches_per_step = (1 if fpath == 0 else 3) + (4 if ngroups == 1 else 6)  # same count on every walk
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                   delta_bias=p["delta_bias"], delta_softplus=True, out=(y, None, ck),
                   workspace=fws)
        if ev is not None:
            ev[1].record(stream)
        ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"], ck, D=p["D"], z=p["z"],
                   delta_bias=p["delta_bias"], delta_softplus=True, workspace=ws, out=gout)
        if ev is not None:
            ev[2].record(stream)
        if world > 1:
            ssdist.allreduce_param_grads(pgrad)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # ---- kernel-only timed region
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(gpu_uuid(dev)) if rank == 0 else None
    if sampler:
        sampler.start()
    barrier()
    torch.cuda.synchronize()
    h0 = time.time()
    t_start.record(stream)
    for i in range(K):
        step(evs[i])
    t_end.record(stream)
    torch.cuda.synchronize()
    h1 = time.time()
    barrier()
    clocks = sampler.stop(h0, h1) if sampler else None
    elapsed_ms = t_start.elapsed_time(t_end)
    # per-pass times: the median over at least 30 steps (the K timed ones, plus
    # more after the timed region when K < 30)
    extra = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(max(0, 30 - K))]
    for e in extra:
        step(e)
    torch.cuda.synchronize()
    evs = evs + extra
    fwd_ms = statistics.median(e[0].elapsed_time(e[1]) for e in evs)
    bwd_ms = statistics.median(e[1].elapsed_time(e[2]) for e in evs)
    if world > 1:
        t = torch.tensor([elapsed_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed_ms = float(t.item())
    value = tc_rank * world * K / (elapsed_ms / 1e3)

    # ---- end to end through the same API with host buffers: pinned host
    # inputs in, every result out, copies overlapped with the kernels of the
    # neighbouring steps (two device slots, copy-in / compute / copy-out streams)
    from selective_state_space_11_b200.streaming import HostStepPipeline
    Ke = max(1, min(K, args.e2e_steps))
    pipe = HostStepPipeline(bsz, dim, L, p["u"].dtype,
                            {"A": p["A"], "D": p["D"], "delta_bias": p["delta_bias"]}, dev,
                            dstate=N, allreduce=ssdist.allreduce_param_grads if world > 1 else None)
    host_in, host_out = HostStepPipeline.host_buffers(bsz, dim, L, p["u"].dtype, dstate=N)
    for k in host_in:
        host_in[k].copy_(p[k].cpu())
    h2d = sum(t.numel() * t.element_size() for t in host_in.values())
    d2h = sum(t.numel() * t.element_size() for t in host_out.values())

    for _ in range(2):  # warm the slots and streams
        pipe.step(host_in, host_out)
    pipe.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(pipe.first_copy_stream())
    for _ in range(Ke):
        pipe.step(host_in, host_out)
    e1.record(pipe.last_copy_stream())
    pipe.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([e2e_ms], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t.item())
    e2e_value = tc_rank * world * Ke / (e2e_ms / 1e3)

    out = None
    if rank == 0:
        sms = torch.cuda.get_device_properties(dev).multi_processor_count
        pk = peaks(sms)
        elt = p["u"].element_size()
        fwd_mufu = FWD_MUFU_PER_TC * tc_rank / (fwd_ms / 1e3)
        bwd_fp32 = BWD_FP32_PER_TC * tc_rank / (bwd_ms / 1e3)
        fwd_bytes = tc_rank * (4 * elt + 64 / 64) + 2 * bsz * N * L * elt
        bwd_bytes = tc_rank * (7 * elt + 64 / 64) + 2 * bsz * N * L * (elt + 4)
        rl = {
            "fwd": {"kernel": ("fwd (chunk-parallel)" if fpath != 0 else
                               "fwd2_kernel (two channels per lane group)" if bsz * dim >= 128 * sms
                               else "fwd_kernel (one channel per lane group)"),
                    "bound": "alu", "unit": "MUFU op/s", "achieved": fwd_mufu, "peak": pk["mufu"],
                    "frac": fwd_mufu / pk["mufu"], "ms": fwd_ms,
                    "hbm_frac": fwd_bytes / (fwd_ms / 1e3) / (pk["hbm_gbs"] * 1e9),
                    "algorithmic_bytes": fwd_bytes},
            "bwd": {"kernel": bwd_pass_name(bvariant, ngroups), "bound": "alu",
                    "unit": "FP32 op/s", "achieved": bwd_fp32, "peak": pk["fp32"],
                    "frac": bwd_fp32 / pk["fp32"], "ms": bwd_ms,
                    "hbm_frac": bwd_bytes / (bwd_ms / 1e3) / (pk["hbm_gbs"] * 1e9),
                    "algorithmic_bytes": bwd_bytes},
        }
        dom = "bwd" if bwd_ms >= fwd_ms else "fwd"
        traffic = profiled_traffic(args.workload) if not args.seqlen else {}
        for k in rl:
            rl[k]["traffic"] = traffic.get(k)
        d = rl[dom]
        roofline = {"bound": "alu", "achieved": d["achieved"], "peak": d["peak"], "unit": d["unit"],
                    "frac": d["frac"], "traffic": d["traffic"], "kernel": d["kernel"],
                    "traffic_basis": ("dram__bytes_read.sum + dram__bytes_write.sum per launch of the pass, "
                                      f"profiles/traffic_{args.workload}.json (same kernel sources)")
                                     if d["traffic"] is not None else "no capture of the current kernels",
                    "peak_basis": f"{sms} SMs x {MUFU_PER_SM_CLK if dom == 'fwd' else FP32_PER_SM_CLK}"
                                  f"/clk x {pk['clock_mhz']:.0f} MHz (derived from unit counts)",
                    "passes": rl}
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "storage_dtype": w.dtype,
            "data": "synthetic",
            "config": {"workload": args.workload if not args.seqlen else
                       f"{args.workload} with L overridden to {L} (profiling capture, not a bench line)",
                       "batch": bsz, "dim": dim, "dstate": N,
                       "seqlen": L, "storage": w.dtype, "tokens_channels_per_gpu_step": tc_rank,
                       "l2": "inputs larger than L2 (4 x %.0f MB per rank)" %
                             (p["u"].numel() * elt / 1e6),
                       "parallelism": f"dp{world}" if world > 1 else "single GPU",
                       "fwd_path": "per-channel" if fpath == 0 else f"chunk-parallel x{nseg}",
                       "bwd_walk": {"variant": bvariant, "chunk_groups": ngroups}},
            "fwd_tc_per_s": tc_rank / (fwd_ms / 1e3), "bwd_tc_per_s": tc_rank / (bwd_ms / 1e3),
            "pass_timing": f"median over {len(evs)} steps (CUDA events around each pass)",
            "roofline": roofline,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": Ke},
            "gpu_launches": launches_per_step * K,
            "clocks": clocks,
        }
    # free the training buffers before the detail measurements
    del p, y, ck, gout, ws, host_in, host_out
    torch.cuda.empty_cache()
    if rank == 0 and not args.no_detail:
        out["detail"] = detail_measurements(args, dev)
    return out


def bwd_pass_name(variant, ngroups):
    """The kernels of one ss_bwd call on the walk variant ss_bwd_path reports."""
    g = f"{ngroups} chunk group{'s' if ngroups > 1 else ''}"
    if variant == 3:
        return ("bwd pass: ch_states_kernel (+ chunk carry maps) + ch_carry_kernel + ch_walk_kernel "
                f"(one thread per channel, {g}) + ch_reduce_bc_kernel + ch_reduce_param_kernel "
                "(timed together)") if ngroups > 1 else (
                "bwd pass: ch_states_kernel + ch_walk_kernel (one thread per channel) + "
                "ch_reduce_bc_kernel + ch_reduce_param_kernel (timed together)")
    walk = "bwd_kernel" if variant == 0 else "bwd2_kernel"
    return ("bwd pass: states_kernel" + (" (+ chunk carry maps) + group_carry_kernel" if ngroups > 1 else "")
            + f" + reverse walk ({walk}, {g}) + reduce_bc_kernel + reduce_param_kernel (timed together)")


def _time_events(fn, iters, warm=3):
    import torch
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(iters):
        fn()
    b.record()
    torch.cuda.synchronize()
    return a.elapsed_time(b) / iters


def detail_measurements(args, dev, only=None):
    """Other rows of the hot path, each on its own workload (not in `value`).
    `only` names one section to run alone (for profiling captures)."""
    import torch

    from selective_state_space_11_b200 import inputs as gen
    from selective_state_space_11_b200 import ops
    res = {}
    def want(name):
        return only is None or only == name

    if want("mamba130m_layer"):
        # fwd-only and fwd+bwd on the Mamba-130m layer shape
        w = gen.WORKLOADS["mamba130m_layer"]
        p = gen.workload_inputs(w.name, device=dev)
        tc = w.batch * w.dim * w.seqlen
        y, fs, ck = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                               delta_bias=p["delta_bias"])
        ws = torch.empty(ops.lib().ss_bwd_workspace_size(w.batch, w.dim, 16, w.seqlen), device=dev,
                         dtype=torch.uint8)
        f_ms = _time_events(lambda: ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"],
                                               z=p["z"], delta_bias=p["delta_bias"],
                                               out=(y, fs, ck)), 20)
        b_ms = _time_events(lambda: ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"],
                                               ck, D=p["D"], z=p["z"], delta_bias=p["delta_bias"],
                                               workspace=ws), 20)
        res["mamba130m_layer"] = {"fwd_ms": f_ms, "bwd_ms": b_ms, "fwd_tc_per_s": tc / f_ms * 1e3,
                                  "fwd_bwd_tc_per_s": tc / (f_ms + b_ms) * 1e3}
        del p, y, fs, ck, ws
    if want("microbench"):
        # the pages' microbenchmark shape: chunk-parallel forward
        w = gen.WORKLOADS["microbench"]
        p = gen.workload_inputs(w.name, device=dev)
        fws = torch.empty(max(16, ops.lib().ss_fwd_workspace_size(1, w.dim, 16, w.seqlen)),
                          device=dev, dtype=torch.uint8)
        y = torch.empty_like(p["u"])
        fs = torch.empty(1, w.dim, 16, device=dev)
        def mfwd():
            ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                       delta_bias=p["delta_bias"], out=(y, fs, None), workspace=fws)
        eager_ms = _time_events(mfwd, 50)
        # at this size a call is shorter than its host-side submission through the
        # Python binding, so the device time is taken from a CUDA graph of 20 calls
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            for _ in range(3):
                mfwd()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(20):
                mfwd()
        m_ms = _time_events(graph.replay, 10) / 20
        del graph
        # the same call with L2 flushed before it: a 256 MB buffer is rewritten
        # between calls (outside the events), so inputs and B/C come from HBM;
        # the flush also covers the host-side submission of the next call
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        fl = []
        for i in range(40):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            mfwd()
            b.record()
            torch.cuda.synchronize()
            if i >= 5:
                fl.append(a.elapsed_time(b))
        del flush
        res["microbench"] = {"fwd_us": m_ms * 1e3, "tokens_per_s": w.seqlen / m_ms * 1e3,
                             "tc_per_s": w.dim * w.seqlen / m_ms * 1e3,
                             "timing": "CUDA graph of 20 calls (device time per call; inputs L2-resident)",
                             "fwd_us_l2_flushed": statistics.median(fl) * 1e3,
                             "l2_flushed_timing": f"median of {len(fl)} calls, each after a 256 MB L2 flush",
                             "fwd_us_eager_python_calls": eager_ms * 1e3,
                             "path": list(ops.fwd_path(1, w.dim, w.seqlen)),
                             "pages_figure_for_context": "~45 M tokens/s, Apple M4 Max (Metal)"}
        del p, y, fs, fws
    if want("long_prefill_decode"):
        # long-context prefill, then decode steps captured in a CUDA graph
        w = gen.WORKLOADS["long_prefill_decode"]
        p = gen.workload_inputs(w.name, device=dev, with_dy=False)
        y = torch.empty_like(p["u"])
        st = torch.empty(1, w.dim, 16, device=dev)
        fws = torch.empty(max(16, ops.lib().ss_fwd_workspace_size(1, w.dim, 16, w.seqlen)),
                          device=dev, dtype=torch.uint8)
        pre_ms = _time_events(lambda: ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                                 D=p["D"], z=p["z"], delta_bias=p["delta_bias"],
                                                 out=(y, st, None), workspace=fws), 10)
        tok = gen.make_decode_tokens(1, w.dim, 16, w.decode_steps, w.dtype, w.seed, device=dev)
        yd = torch.empty(w.decode_steps, 1, w.dim, device=dev, dtype=tok["u"].dtype)
        s = torch.cuda.Stream(dev)
        s.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s):
            for t in range(3):
                ops.ss_state_update(st, tok["u"][t], tok["delta"][t], p["A"], tok["B"][t],
                                    tok["C"][t], D=p["D"], z=tok["z"][t],
                                    delta_bias=p["delta_bias"], y=yd[t])
        torch.cuda.current_stream(dev).wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for t in range(w.decode_steps):
                ops.ss_state_update(st, tok["u"][t], tok["delta"][t], p["A"], tok["B"][t],
                                    tok["C"][t], D=p["D"], z=tok["z"][t],
                                    delta_bias=p["delta_bias"], y=yd[t])
        g_ms = _time_events(g.replay, 10)
        # the same prompt as 8 chained pieces: each piece starts from the previous
        # piece's final state (ss_fwd_with_state)
        npc = 8
        lp = w.seqlen // npc
        pieces = [{k: p[k][..., i * lp:(i + 1) * lp].contiguous() for k in ("u", "delta", "z", "B", "C")}
                  for i in range(npc)]
        ys = [torch.empty_like(q["u"]) for q in pieces]
        sts = [torch.empty(1, w.dim, 16, device=dev) for _ in range(npc)]
        pws = torch.empty(max(16, ops.lib().ss_fwd_workspace_size(1, w.dim, 16, lp)), device=dev,
                          dtype=torch.uint8)

        def chunked():
            h = None
            for q, yq, sq in zip(pieces, ys, sts):
                ops.ss_fwd(q["u"], q["delta"], p["A"], q["B"], q["C"], D=p["D"], z=q["z"],
                           delta_bias=p["delta_bias"], out=(yq, sq, None), workspace=pws, h0=h)
                h = sq

        c_eager_ms = _time_events(chunked, 10)
        # device time of the 8 chained calls, without their host-side submission
        s3 = torch.cuda.Stream(dev)
        s3.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s3):
            chunked()
        torch.cuda.current_stream(dev).wait_stream(s3)
        torch.cuda.synchronize()
        gc8 = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gc8):
            chunked()
        c_ms = _time_events(gc8.replay, 10)
        del gc8
        # the conv-window decode step, 256 steps in a CUDA graph
        cw = gen.make_conv_inputs(1, w.dim, 1, 4, w.dtype, w.seed, device=dev)
        cst = cw["state"].clone()
        cx = tok["u"]
        cu = torch.empty(w.decode_steps, 1, w.dim, device=dev, dtype=cx.dtype)
        s2 = torch.cuda.Stream(dev)
        s2.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(s2):
            for t in range(3):
                ops.conv1d_step(cst, cx[t], cw["w"], bias=cw["bias"], u=cu[t])
        torch.cuda.current_stream(dev).wait_stream(s2)
        torch.cuda.synchronize()
        gc = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gc):
            for t in range(w.decode_steps):
                ops.conv1d_step(cst, cx[t], cw["w"], bias=cw["bias"], u=cu[t])
        cg_ms = _time_events(gc.replay, 10)
        del gc
        res["long_prefill_decode"] = {
            "prefill_ms": pre_ms, "prefill_tc_per_s": w.dim * w.seqlen / pre_ms * 1e3,
            "prefill_path": list(ops.fwd_path(1, w.dim, w.seqlen)),
            "chunked_prefill_ms": c_ms, "chunked_prefill_pieces": npc,
            "chunked_prefill_timing": "CUDA graph of the 8 chained calls (device time)",
            "chunked_prefill_ms_eager_python_calls": c_eager_ms,
            "chunked_prefill_tc_per_s": w.dim * w.seqlen / c_ms * 1e3,
            "chunked_prefill_piece_path": list(ops.fwd_path(1, w.dim, lp)),
            "decode_us_per_step": g_ms * 1e3 / w.decode_steps,
            "conv_decode_us_per_step": cg_ms * 1e3 / w.decode_steps,
            "decode_steps_per_graph": w.decode_steps}
        del g
    if want("packed_documents"):
        # packed documents (seq_idx): the 2.8b layer shape with every row cut into
        # documents of 64..1024 tokens, against the same step unpacked
        w = gen.WORKLOADS["mamba2.8b_layer"]
        p = gen.workload_inputs(w.name, device=dev)
        g = torch.Generator().manual_seed(w.seed)
        rows = []
        for _ in range(w.batch):
            ids, doc = [], 0
            while len(ids) < w.seqlen:
                ids += [doc] * int(torch.randint(64, 1025, (1,), generator=g))
                doc += 1
            rows.append(ids[:w.seqlen])
        seq = torch.tensor(rows, dtype=torch.int32, device=dev)
        y, fs, ck = ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"], D=p["D"], z=p["z"],
                               delta_bias=p["delta_bias"], seq_idx=seq)
        ws = torch.empty(ops.lib().ss_bwd_workspace_size(w.batch, w.dim, 16, w.seqlen), device=dev,
                         dtype=torch.uint8)
        kw = dict(D=p["D"], z=p["z"], delta_bias=p["delta_bias"], seq_idx=seq)
        pf_ms = _time_events(lambda: ops.ss_fwd(p["u"], p["delta"], p["A"], p["B"], p["C"],
                                                out=(y, fs, ck), **kw), 20)
        pb_ms = _time_events(lambda: ops.ss_bwd(p["u"], p["delta"], p["A"], p["B"], p["C"], p["dy"],
                                                ck, workspace=ws, **kw), 20)
        tc = w.batch * w.dim * w.seqlen
        res["packed_documents_mamba2.8b_layer"] = {
            "documents": int(sum(len(set(r)) for r in rows)), "fwd_ms": pf_ms, "bwd_ms": pb_ms,
            "fwd_bwd_tc_per_s": tc / (pf_ms + pb_ms) * 1e3}
        del p, y, fs, ck, ws, seq
    if want("ssd"):
        # Mamba-2 SSD forward on a 2.7b-like layer: 4 x 4096 tokens, 80 heads of 64,
        # ngroups 1, dstate 128, bf16 -- tensor-core flops against the measured
        # cuBLAS bf16 peak
        q = gen.make_ssd_inputs(4, 4096, 80, 64, 1, 128, "bf16", 1005, device=dev)
        sy = torch.empty_like(q["x"])
        sfs = torch.empty(4, 80, 64, 128, device=dev)
        ssd_call = lambda: ops.ssd_fwd(q["x"], q["dt"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"],
                                       dt_bias=q["dt_bias"], out=sy, final_state=sfs)
        s_ms = _time_events(ssd_call, 20)
        # the warp-level mma.sync kernel on the same call, for comparison
        os.environ["SS_SSD_VARIANT"] = "mma"
        try:
            s_ms_mma = _time_events(ssd_call, 20)
        finally:
            os.environ.pop("SS_SSD_VARIANT", None)
        # bytes that must cross HBM: x, z, dt read and y written once; B, C once
        ssd_bytes = 4 * 4096 * (3 * 80 * 64 + 2 * 128 + 80) * 2
        hbm_peak = peaks(1)["hbm_gbs"] * 1e9
        Qc, Pd, Nd = 64, 64, 128
        chunk_flops = 2 * Qc * Qc * Nd + 2 * Qc * Qc * Pd + 2 * Qc * Nd * Pd + 2 * Qc * Nd * Pd
        flops = 4 * 80 * (4096 // Qc) * chunk_flops
        mp = {}
        if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
            with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
                mp = json.load(f)
        bf16_peak = float(mp.get("bf16_tflops", 1590.0)) * 1e12
        res["ssd_fwd_mamba2_2.7b_layer"] = {
            "shape": "batch 4, L 4096, 80 heads x headdim 64, ngroups 1, dstate 128, bf16",
            "fwd_ms": s_ms, "tokens_per_s": 4 * 4096 / s_ms * 1e3,
            "tensor_tflops": flops / (s_ms / 1e3) / 1e12,
            "tensor_frac": flops / (s_ms / 1e3) / bf16_peak,
            "peak_basis": "MEASURED_PEAKS.json bf16_tflops (cuBLAS bf16 GEMM, burst)"
                          if "bf16_tflops" in mp else "fallback 1590 TFLOP/s",
            "hbm_bytes": ssd_bytes, "hbm_gbs": ssd_bytes / (s_ms / 1e3) / 1e9,
            "hbm_frac": ssd_bytes / (s_ms / 1e3) / hbm_peak,
            "mma": "tcgen05.mma kind::f16 (bf16 operands from TMA-loaded smem tiles, fp32 accumulators in TMEM)",
            "kernel": "ssd_tc_kernel",
            "fwd_ms_mma_sync": s_ms_mma,
            "mma_sync_kernel": "ssd_fwd_kernel (warp-level mma.sync m16n8k16, SS_SSD_VARIANT=mma)"}
        # the SSD backward on the same layer: its chunk products run as tcgen05
        # MMAs on fp16 operands, reported against the measured bf16 (= fp16) peak
        dy = gen.make_ssd_inputs(4, 4096, 80, 64, 1, 128, "bf16", 1006, device=dev)["x"]
        sws = torch.empty(ops.lib().ss_ssd_bwd_workspace_size(4, 4096, 80, 64, 1, 128), device=dev,
                          dtype=torch.uint8)
        bwd_call = lambda: ops.ssd_bwd(q["x"], q["dt"], q["A"], q["B"], q["C"], dy, D=q["D"], z=q["z"],
                                       dt_bias=q["dt_bias"], workspace=sws)
        b_ms = _time_events(bwd_call, 5)
        os.environ["SS_SSD_VARIANT"] = "mma"
        try:
            b_ms_mma = _time_events(bwd_call, 5)
        finally:
            os.environ.pop("SS_SSD_VARIANT", None)
        # MACs per chunk: the maps U, V (2 Q P N), the read-out and adjoint products
        # with the state (4 Q P N), C B^T and dout x^T (Q^2 (N + P)), the intra-chunk
        # read-out and G B (2 Q^2 P), dB and dC (2 Q^2 N)
        bwd_mac = 4 * 80 * (4096 // Qc) * (6 * Qc * Pd * Nd + 3 * Qc * Qc * Nd + 3 * Qc * Qc * Pd)
        res["ssd_fwd_mamba2_2.7b_layer"].update({
            "bwd_ms": b_ms, "bwd_tensor_tflops": 2 * bwd_mac / (b_ms / 1e3) / 1e12,
            "bwd_tensor_frac": 2 * bwd_mac / (b_ms / 1e3) / bf16_peak,
            "bwd_peak_basis": "MEASURED_PEAKS.json bf16_tflops (fp16 operands run at the bf16 rate)"
                              if "bf16_tflops" in mp else "fallback 1590 TFLOP/s",
            "bwd_mma": "tcgen05.mma kind::f16 (fp16 operands, fp32 accumulators in TMEM)",
            "bwd_kernels": "ssd_maps_tc_kernel, ssd_pass16_kernel, ssd_grad_tc_kernel, ssd_reduce_bc8_kernel, "
                           "ssd_reduce_param_kernel (fp16 state/adjoint slabs and dB/dC partials)",
            "bwd_ms_mma_sync": b_ms_mma,
            "bwd_mma_sync_kernels": "ssd_maps_kernel, ssd_pass_kernel, ssd_grad_kernel, ssd_reduce_bc_kernel "
                                    "(warp-level tf32 mma.sync, fp32 slabs; SS_SSD_VARIANT=mma)"})
        del q, sy, sfs, dy, sws
    if want("conv1d"):
        # causal conv1d (+ SiLU) feeding the scan, on the Mamba-2.8b layer shape:
        # HBM-bound, reported against the measured copy bandwidth
        w = gen.WORKLOADS["mamba2.8b_layer"]
        c = gen.make_conv_inputs(w.batch, w.dim, w.seqlen, 4, w.dtype, w.seed, device=dev)
        n = w.batch * w.dim * w.seqlen
        elt = c["x"].element_size()
        u = torch.empty_like(c["x"])
        cws = torch.empty(ops.lib().ss_conv1d_bwd_workspace_size(w.batch, w.dim, w.seqlen, 4),
                          device=dev, dtype=torch.uint8)
        cf_ms = _time_events(lambda: ops.conv1d_fwd(c["x"], c["w"], bias=c["bias"], out=u), 20)
        cb_ms = _time_events(lambda: ops.conv1d_bwd(c["x"], c["w"], c["du"], bias=c["bias"],
                                                    workspace=cws), 20)
        hbm = peaks(148)["hbm_gbs"] * 1e9
        res["conv1d_mamba2.8b_layer"] = {
            "fwd_ms": cf_ms, "bwd_ms": cb_ms,
            "fwd_algorithmic_bytes": 2 * elt * n, "bwd_algorithmic_bytes": 3 * elt * n,
            "fwd_hbm_frac": 2 * elt * n / (cf_ms / 1e3) / hbm,
            "bwd_hbm_frac": 3 * elt * n / (cb_ms / 1e3) / hbm,
            "hbm_peak_basis": "MEASURED_PEAKS.json hbm_gbs (measured copy bandwidth)"}
        del c, u, cws
    return res


# ------------------------------------------------------- oracle baseline ----
def oracle_sample(workload, nchan, seed_offset=0):
    """Inputs for an fp64 oracle fwd+bwd over about `nchan` channels at full L:
    the first `nchan` channels of one batch row, or whole batch rows (at most
    the workload's batch) when `nchan` exceeds d_inner.  Returns (inputs, TC, rows, dim)."""
    from selective_state_space_11_b200 import inputs as gen
    w = gen.WORKLOADS[workload]
    if nchan <= w.dim:
        rows, dim = 1, nchan
    else:
        rows, dim = min(w.batch, -(-nchan // w.dim)), w.dim
    p = gen.make_inputs(rows, dim, w.dstate, w.seqlen, w.dtype, w.seed + seed_offset)
    return {k: gen.as_f64(v) for k, v in p.items()}, rows * dim * w.seqlen, rows, dim


def oracle_step(q):
    import oracle
    y, fs, ck = oracle.ss_fwd(q["u"], q["delta"], q["A"], q["B"], q["C"], D=q["D"], z=q["z"],
                              delta_bias=q["delta_bias"])
    oracle.ss_bwd(q["u"], q["delta"], q["A"], q["B"], q["C"], q["dy"], D=q["D"], z=q["z"],
                  delta_bias=q["delta_bias"])


def oracle_threads_step(q):
    import oracle
    return oracle.ss_fwd_bwd_threads(q["u"], q["delta"], q["A"], q["B"], q["C"], q["dy"], D=q["D"],
                                     z=q["z"], delta_bias=q["delta_bias"])[4]


def cpu_baseline(workload, budget_s=8.0):
    """The fp64 oracle on this host: on all cores (the (batch, channel) rows in
    slices, one thread per slice, see oracle.ss_fwd_bwd_threads) and, beside it,
    single-threaded; each on a sample of whole channels at the full L sized to
    about `budget_s` seconds."""
    import oracle
    oracle.build()
    from selective_state_space_11_b200 import inputs as gen
    w = gen.WORKLOADS[workload]
    q, tc, _, _ = oracle_sample(workload, 4)
    t0 = time.perf_counter()
    oracle_step(q)
    per_chan = (time.perf_counter() - t0) / 4
    # single-threaded
    nchan = int(max(4, budget_s / max(per_chan, 1e-6)))
    q, tc, rows, dim = oracle_sample(workload, nchan)
    t0 = time.perf_counter()
    oracle_step(q)
    dt1 = time.perf_counter() - t0
    single = {"value": tc / dt1, "unit": UNIT, "cores": 1,
              "sample": f"fwd+bwd of {rows} batch row(s) x {dim} channels x L={w.seqlen}; {dt1:.1f} s"}
    # all cores
    cores = oracle.host_cores()
    nchan = int(max(cores, budget_s * cores / max(per_chan, 1e-6)))
    q, tc, rows, dim = oracle_sample(workload, nchan)
    t0 = time.perf_counter()
    used = oracle_threads_step(q)
    dt = time.perf_counter() - t0
    return {"value": tc / dt, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"fwd+bwd of {rows} batch row(s) x {dim} channels x L={w.seqlen} of the "
                      f"{workload} shape, fp64, {used} threads over (batch, channel) slices "
                      f"({cores} cores in this process's affinity mask); {dt:.1f} s",
            "single_thread": single}


def run_reference(args):
    """The fp64 oracle as the reference program, on all host cores, on a bounded
    sample of the workload per step (`--ref-channels` channels per core)."""
    import oracle
    oracle.build()
    from selective_state_space_11_b200 import inputs as gen
    w = gen.WORKLOADS[args.workload]
    cores = oracle.host_cores()
    nchan = args.ref_channels * cores
    q, tc, rows, dim = oracle_sample(args.workload, nchan)
    for _ in range(args.warmup):
        oracle_threads_step(q)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        used = oracle_threads_step(q)
    dt = time.perf_counter() - t0
    v = tc * args.steps / dt
    sample = (f"each step: fwd+bwd of {rows} batch row(s) x {dim} channels x L={w.seqlen} of the "
              f"{args.workload} shape, fp64 oracle, {used} threads over (batch, channel) slices")
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": f"{args.workload} sample: {rows} x {dim} channels x L={w.seqlen}",
                       "batch": rows, "dim": dim, "dstate": w.dstate, "seqlen": w.seqlen,
                       "storage": w.dtype, "sample_of": args.workload},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": used, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def launch_plan(gpus, env):
    """How `--gpus N` runs: ("direct", N) in this process when the launcher's
    WORLD_SIZE is N (or it is unset and N == 1); ("spawn", N) to start N ranks
    with torch.distributed.run when no launcher set WORLD_SIZE; ("error", why)
    when the two disagree."""
    if gpus < 1:
        return "error", f"--gpus {gpus}: must be at least 1"
    ws = env.get("WORLD_SIZE")
    if ws is None:
        return ("direct", 1) if gpus == 1 else ("spawn", gpus)
    if int(ws) != gpus:
        return "error", f"--gpus {gpus} but the launcher started WORLD_SIZE={ws} ranks"
    return "direct", gpus


def spawn_ranks(n, argv):
    """Run this script as n ranks (one process per GPU) on this node; rank 0 prints the line."""
    import socket
    import torch
    have = torch.cuda.device_count()
    if have < n:
        print(f"bench.py: --gpus {n} but this node has {have} GPU(s)", file=sys.stderr)
        return 2
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={port}", os.path.abspath(__file__)] + argv
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--ref-channels", type=int, default=8,
                    help="reference arm: channels per host core in each step's sample")
    ap.add_argument("--no-detail", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--detail-only", default=None,
                    choices=["mamba130m_layer", "microbench", "long_prefill_decode",
                             "packed_documents", "ssd", "conv1d"],
                    help="run one detail section alone and print it (profiling captures)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's L (small profiling captures only; the line says so)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    mode, arg = launch_plan(args.gpus, os.environ)
    if mode == "error":
        print(f"bench.py: {arg}", file=sys.stderr)
        return 2
    if mode == "spawn":
        return spawn_ranks(arg, sys.argv[1:])
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    if args.detail_only:
        from selective_state_space_11_b200 import build as ssbuild
        ssbuild.build()
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        if rank == 0:
            print(json.dumps({"detail": detail_measurements(args, dev, only=args.detail_only)}),
                  flush=True)
        return 0
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(args.workload)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
