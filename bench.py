"""Benchmark of the fused attention hot path on B200.

One step = the whole path on one batch of synthetic input: build the block
mask and work order, forward (O and LSE), backward (dQ, dK, dV).  The default
workload is dense MHA B=4, Hq=Hkv=8, S=4096, D=128, non-causal, bf16 inputs
drawn N(0,1) from a fixed seed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME[:MOD]]
    python bench.py --impl reference ...   # the fp64 CPU oracle, timed on the host
    python bench.py --all                  # one line per workload and mod

Prints one JSON line (rank 0).  Throughput counts only unmasked score
elements: 4 D flop each forward, 10 D backward.
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

from synth_inputs import (MOD_NAMES, WORKLOADS, bf16_bits_to_f64, draw_workload,  # noqa: E402
                          mod_params_for, pack_bitmap, pad_offsets)

METRIC = "attention fwd/bwd useful TFLOPS on 1 B200 and % of BF16 tensor peak"
UNIT = "TFLOP/s"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def parse_workload(spec):
    name, _, mod = spec.partition(":")
    w = WORKLOADS[name]
    mod = mod or w.mods[0]
    return w, mod


def rank_workload(w, rank):
    """The replica rank `rank` processes: the same shapes as `w`, its own Q/K/V/dO
    (seed offset by the rank), so N ranks run N independent problems."""
    import dataclasses
    return dataclasses.replace(w, seed=w.seed + rank)


KERNEL_SOURCES = {
    "attn_fwd": ["fwd_sm100.cu", "kernel_common.cuh", "mods.cuh", "sm100.cuh", "exp2_poly.h", "launch.h"],
    "attn_bwd": ["bwd_sm100.cu", "kernel_common.cuh", "mods.cuh", "sm100.cuh", "launch.h"],
}


def kernel_source_hash(kernel):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "tiled_attention_25_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary (the table in
    profiles/traffic.md), if it was taken on the kernel source as it is now
    (else None: the counters are stale)."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    try:
        with open(path) as f:
            lines = f.read().splitlines()
    except OSError:
        return None
    for line in lines:
        cells = [c.strip().strip("`") for c in line.strip().strip("|").split("|")]
        if len(cells) >= 4 and cells[0] == kernel and cells[1] == workload:
            if cells[2] != kernel_source_hash(kernel):
                return None
            try:
                return int(cells[3])
            except ValueError:
                return None
    return None


def max_over_ranks(vals, world, device=None):
    """Element-wise maximum of a list of floats over all ranks of the default
    process group (identity on one rank).  Time-like quantities are reduced
    this way: a multi-GPU step is as slow as its slowest rank."""
    if world <= 1:
        return list(vals)
    import torch
    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(flop_per_rank, world, ms):
    """Whole-job TFLOP/s: every rank processes its own replica of the workload
    (weak scaling, no exchange), so the job's work is world x per-rank work,
    done in the slowest rank's time."""
    return flop_per_rank * world / (ms * 1e-3) / 1e12


def useful_counts(ta, w, mod_name, params):
    mod = MOD_NAMES[mod_name]
    if params.bitmap is not None:
        # a general mask counts its set bits (ANDed with nothing else here),
        # once per batch row and head that shares it
        keep = np.asarray(params.bitmap, dtype=bool)
        n = int(keep.sum()) * (w.B // keep.shape[0]) * (w.Hq // keep.shape[1])
    else:
        n = ta.useful_elements(mod, w.B, w.Hq, w.Sq, w.Skv, window=params.window, doc_offsets=params.doc_offsets)
    return n, ta.useful_flops(n, w.D), ta.useful_flops(n, w.D, backward=True)


# ----------------------------------------------------------------------------- GPU arm

# The parity configurations that get their own entry in the bench line
# (workload:mod), beside the headline workload.
CONFIG_ENTRIES = ("dense:causal", "gqa_long:causal", "score_mods:alibi", "score_mods:softcap",
                  "score_mods:sliding_window", "score_mods:local_boost", "documents:document")


# Variants of the path, each on the same workload (bench.py --variant):
#   det   the backward with the bitwise reproducible dQ (attn_bwd_deterministic)
#   bshd  Q, K, V, O, dO and the gradients stored [B][S][H][D], passed as
#         strided [B][H][S][D] views (attn_fwd_strided / attn_bwd_strided)
#   fp8   the forward with FP8 scores: Q and K rotated and quantised to e4m3
#         (attn_fp8_rotate_quantize, inside the timed forward) and
#         attn_fwd_fp8; forward only (its LSE belongs to the FP8 scores)
VARIANTS = ("det", "bshd", "fp8")


class Problem:
    """One workload's device tensors, mod parameters and block mask."""

    def __init__(self, ta, spec, rank, dev, variant=None):
        import torch
        self.variant = variant
        self.w, self.mod_name = parse_workload(spec)
        w = self.w
        self.mod = MOD_NAMES[self.mod_name]
        self.params = mod_params_for(w, self.mod_name)   # same structure (and flops) on every rank
        bits = draw_workload(rank_workload(w, rank))
        to_dev = lambda b: torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).to(dev)
        self.q, self.k, self.v, self.dout = (to_dev(bits[n]) for n in ("q", "k", "v", "dout"))
        del bits
        doc_t = None
        if self.params.doc_offsets is not None:
            doc_t = torch.from_numpy(pad_offsets(self.params.doc_offsets)[0]).to(dev)
        bm_t = None
        if self.params.bitmap is not None:
            bm_t = torch.from_numpy(pack_bitmap(self.params.bitmap)).to(dev)
        p = self.params
        self.dp = ta.ModParams(softcap=p.softcap, window=p.window, boost=p.boost,
                               boost_radius=p.boost_radius, doc_offsets=doc_t, bitmap=bm_t)
        self.out = torch.empty_like(self.q)
        self.lse = torch.empty(w.B, w.Hq, w.Sq, dtype=torch.float32, device=dev)
        self.dq, self.dk, self.dv = torch.empty_like(self.q), torch.empty_like(self.k), torch.empty_like(self.v)
        self.ws = ta.new_bwd_workspace(w.B, w.Hq, w.Sq, w.D, device=dev, deterministic=variant == "det")
        if variant == "bshd":  # the same values in [B][S][H][D] storage, seen as [B][H][S][D] views
            bshd = lambda t: t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
            self.q, self.k, self.v, self.dout = (bshd(t) for t in (self.q, self.k, self.v, self.dout))
            self.out, self.dq, self.dk, self.dv = (bshd(t) for t in (self.out, self.dq, self.dk, self.dv))
        if variant == "fp8":
            g = torch.Generator().manual_seed(1000 + w.seed)
            self.signs = (torch.randint(0, 2, (w.D,), generator=g, dtype=torch.int8) * 2 - 1).to(dev)
            self.q8 = torch.empty(w.B, w.Hq, w.Sq, w.D, dtype=torch.uint8, device=dev)
            self.k8 = torch.empty(w.B, w.Hkv, w.Skv, w.D, dtype=torch.uint8, device=dev)
            self.qs = torch.empty(w.B, w.Hq, dtype=torch.float32, device=dev)
            self.ks = torch.empty(w.B, w.Hkv, dtype=torch.float32, device=dev)
        nbytes = ta.attn_block_mask_bytes(w.B, w.Sq, w.Skv)
        mbuf = torch.empty(nbytes + 256, dtype=torch.uint8, device=dev)
        off = (-mbuf.data_ptr()) % 256
        self.mask = ta.attn_block_mask_bind(mbuf[off:off + nbytes], w.B, w.Sq, w.Skv)
        self.ta = ta

    def block_mask(self, stream):
        w = self.w
        self.ta.build_block_mask(self.mod, self.dp, w.B, w.Sq, w.Skv, self.mask, stream)

    def forward(self, stream, with_lse=True):
        lse = self.lse if with_lse else None
        kw = dict(scale=self.w.scale, mod_kind=self.mod, mod_params=self.dp, block_mask=self.mask, stream=stream)
        if self.variant == "fp8":
            self.ta.attn_fp8_rotate_quantize(self.q, self.signs, self.q8, self.qs, stream=stream)
            self.ta.attn_fp8_rotate_quantize(self.k, self.signs, self.k8, self.ks, stream=stream)
            self.ta.attn_fwd_fp8(self.q8, self.k8, self.qs, self.ks, self.v, self.out, lse, **kw)
        elif self.variant == "bshd":
            self.ta.attn_fwd_strided(self.q, self.k, self.v, self.out, lse, **kw)
        else:
            self.ta.attn_fwd(self.q, self.k, self.v, self.out, lse, **kw)

    def backward(self, stream):
        args = (self.q, self.k, self.v, self.out, self.lse, self.dout, self.dq, self.dk, self.dv, self.ws)
        kw = dict(scale=self.w.scale, mod_kind=self.mod, mod_params=self.dp, block_mask=self.mask, stream=stream)
        if self.variant == "det":
            self.ta.attn_bwd_deterministic(*args, **kw)
        elif self.variant == "bshd":
            self.ta.attn_bwd_strided(*args, **kw)
        else:
            self.ta.attn_bwd(*args, **kw)


def time_steps(ta, pb, stream, flush, steps, warmup, world, dev, fwd_lse=True, with_bwd=True):
    """Device time of `steps` steps (block mask, forward, backward) after
    `warmup` untimed ones, L2 flushed before each; CUDA events on the launch
    stream; per-step times reduced with the maximum over ranks.  Returns the
    per-phase means and the clock record of the timed region."""
    import torch
    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(times):
        e0, e1, e2, e3 = ev(), ev(), ev(), ev()
        e0.record(stream)
        pb.block_mask(stream)
        e1.record(stream)
        pb.forward(stream, fwd_lse)
        e2.record(stream)
        if with_bwd:
            pb.backward(stream)
        e3.record(stream)
        times.append((e0, e1, e2, e3))

    warm = []
    for _ in range(warmup):
        flush.fill_(1.0)
        step(warm)
    torch.cuda.synchronize()
    st = ta.attn_get_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel status {st} during warm-up")
    sampler = ClockSampler(dev.index if dev.index is not None else 0)
    sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.fill_(1.0)  # L2 flush between steps (outside the timed events)
        step(times)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop()
    st = ta.attn_get_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel status {st} in the timed region")
    # each step's time is the slowest rank's; means, median and minimum follow
    t_mask = max_over_ranks([a.elapsed_time(b) for a, b, _, _ in times], world, dev)
    t_fwd = max_over_ranks([b.elapsed_time(c) for _, b, c, _ in times], world, dev)
    t_bwd = max_over_ranks([c.elapsed_time(d) for _, _, c, d in times], world, dev)
    t_step = max_over_ranks([a.elapsed_time(d) for a, _, _, d in times], world, dev)
    mean = lambda x: sum(x) / len(x)
    return {"ms_step": mean(t_step), "ms_fwd": mean(t_fwd), "ms_bwd": mean(t_bwd), "ms_mask": mean(t_mask),
            "ms_step_median": statistics.median(t_step), "ms_step_min": min(t_step), "clocks": clocks}


# Entries of the other paths the library offers, on parity workloads:
# (workload:mod, variant, work walk)
EXTENSION_ENTRIES = (("dense:none", "det", None), ("dense:none", "bshd", None), ("dense:none", "fp8", None),
                     ("dense:causal", None, "static"), ("documents:document", None, "static"))


def config_entry(ta, spec, rank, world, dev, stream, flush, steps, warmup, peak, variant=None, walk=None):
    """Forward and backward useful TFLOP/s of one parity configuration, timed
    like the headline (own clock record); optionally a variant of the path
    (VARIANTS) or the cluster-launch-control work walk."""
    import torch
    pb = Problem(ta, spec, rank, dev, variant=variant)
    fwd_only = variant == "fp8"
    if walk == "static":
        ta.attn_set_work_walk(ta.WALK_STATIC)
    try:
        t = time_steps(ta, pb, stream, flush, steps, warmup, world, dev, with_bwd=not fwd_only)
    finally:
        ta.attn_set_work_walk(ta.WALK_DEFAULT)
    n_u, f_fwd, f_bwd = useful_counts(ta, pb.w, pb.mod_name, pb.params)
    fwd_tf = f_fwd / (t["ms_fwd"] * 1e-3) / 1e12
    bwd_tf = 0.0 if fwd_only else f_bwd / (t["ms_bwd"] * 1e-3) / 1e12
    w = pb.w
    entry = {"shape": f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} S={w.Sq} D={w.D}", "mod": pb.mod_name,
             "variant": variant,
             "walk": walk or ("static backward (always, for the ordered dQ adds)" if variant == "det"
                              else "cluster launch control"),
             "useful_elements": n_u, "steps": steps, "warmup": warmup,
             "ms_fwd": round(t["ms_fwd"], 4), "ms_block_mask": round(t["ms_mask"], 4),
             "fwd_tflops": round(fwd_tf, 1), "fwd_frac_of_peak": round(fwd_tf / peak, 4), "clocks": t["clocks"]}
    if fwd_only:
        entry["note"] = "forward only: the rotation and e4m3 quantisation of Q and K are inside the timed forward"
    else:
        entry.update({"ms_bwd": round(t["ms_bwd"], 4), "bwd_tflops": round(bwd_tf, 1),
                      "bwd_frac_of_peak": round(bwd_tf / peak, 4),
                      "step_tflops": round(job_throughput(f_fwd + f_bwd, world, t["ms_step"]), 1)})
    del pb
    torch.cuda.empty_cache()
    return entry


def forward_only_entry(ta, pb, stream, flush, steps, warmup, world, dev, peak, with_lse):
    """The forward alone (block mask + forward, no backward), with or without
    the LSE output."""
    t = time_steps(ta, pb, stream, flush, steps, warmup, world, dev, fwd_lse=with_lse, with_bwd=False)
    n_u, f_fwd, _ = useful_counts(ta, pb.w, pb.mod_name, pb.params)
    fwd_tf = f_fwd / (t["ms_fwd"] * 1e-3) / 1e12
    w = pb.w
    return {"shape": f"B={w.B} Hq={w.Hq} Hkv={w.Hkv} S={w.Sq} D={w.D}", "mod": pb.mod_name,
            "lse": with_lse, "useful_elements": n_u, "steps": steps, "warmup": warmup,
            "ms_fwd": round(t["ms_fwd"], 4), "fwd_tflops": round(fwd_tf, 1),
            "fwd_frac_of_peak": round(fwd_tf / peak, 4), "clocks": t["clocks"]}


def run_gpu(args, rank, world, local_rank):
    import torch
    import tiled_attention_25_b200 as ta

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pb = Problem(ta, args.workload, rank, dev)
    w, mod_name, params = pb.w, pb.mod_name, pb.params
    B, Hq, Hkv, Sq, Skv, D = w.B, w.Hq, w.Hkv, w.Sq, w.Skv, w.D
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    launches_per_step = 3 + 1 + 3  # block mask (3), forward (1), backward (3)

    t = time_steps(ta, pb, stream, flush, args.steps, args.warmup, world, dev)
    ms_step, ms_fwd, ms_bwd, ms_mask = t["ms_step"], t["ms_fwd"], t["ms_bwd"], t["ms_mask"]
    clocks = t["clocks"]

    # end-to-end through the same API with pinned host buffers: H2D of the
    # step's inputs, the step, D2H of its results (O, dQ, dK, dV)
    q, k, v, dout, out, lse, dq, dk, dv = pb.q, pb.k, pb.v, pb.dout, pb.out, pb.lse, pb.dq, pb.dk, pb.dv
    ev = lambda: torch.cuda.Event(enable_timing=True)
    if args.no_e2e:
        hq = None
    else:
        hq, hk, hv, hdo = (t_.cpu().pin_memory() for t_ in (q, k, v, dout))
    ho, hdq, hdk, hdv = (torch.empty_like(t_, device="cpu").pin_memory() for t_ in (out, dq, dk, dv))
    e2e_times = []
    for i in range(0 if args.no_e2e else args.warmup + args.steps):
        flush.fill_(1.0)
        a0, a1 = ev(), ev()
        a0.record(stream)
        for d_, h_ in ((q, hq), (k, hk), (v, hv), (dout, hdo)):
            d_.copy_(h_, non_blocking=True)
        pb.block_mask(stream)
        pb.forward(stream)
        pb.backward(stream)
        for h_, d_ in ((ho, out), (hdq, dq), (hdk, dk), (hdv, dv)):
            h_.copy_(d_, non_blocking=True)
        a1.record(stream)
        if i >= args.warmup:
            e2e_times.append((a0, a1))
    torch.cuda.synchronize()
    ms_e2e = sum(a.elapsed_time(b) for a, b in e2e_times) / max(1, len(e2e_times))
    e2e_mode = "serial: H2D, step and D2H in one stream, step by step"
    if getattr(args, "e2e_pipeline", False) and not args.no_e2e:
        mod, dp, mask, ws = pb.mod, pb.dp, pb.mask, pb.ws
        ms_e2e = e2e_pipelined(args, ta, stream, dev, (q, k, v, dout, out, lse, dq, dk, dv),
                               (hq, hk, hv, hdo), (ho, hdq, hdk, hdv),
                               lambda t_, s_: (ta.build_block_mask(mod, dp, B, Sq, Skv, mask, s_),
                                               ta.attn_fwd(t_[0], t_[1], t_[2], t_[4], t_[5], scale=w.scale, mod_kind=mod,
                                                           mod_params=dp, block_mask=mask, stream=s_),
                                               ta.attn_bwd(t_[0], t_[1], t_[2], t_[4], t_[5], t_[3], t_[6], t_[7], t_[8], ws,
                                                           scale=w.scale, mod_kind=mod, mod_params=dp,
                                                           block_mask=mask, stream=s_)))
        e2e_mode = ("pipelined: H2D, step and D2H on three streams with two device buffer sets, so that "
                    "step i's compute overlaps step i+1's H2D and step i-1's D2H (every copy still timed)")
        st = ta.attn_get_status(stream)
        if st != 0:
            raise RuntimeError(f"kernel status {st} in the pipelined end-to-end pass")
    ms_e2e = max_over_ranks([ms_e2e], world, dev)[0]
    h2d = sum(t_.numel() * t_.element_size() for t_ in (q, k, v, dout))
    d2h = sum(t_.numel() * t_.element_size() for t_ in (out, dq, dk, dv))

    n_u, f_fwd, f_bwd = useful_counts(ta, w, mod_name, params)
    peaks, peak_kind = load_peaks()
    peak = float(peaks["bf16_tflops"])
    fwd_tf = f_fwd / (ms_fwd * 1e-3) / 1e12
    bwd_tf = f_bwd / (ms_bwd * 1e-3) / 1e12

    def roof(tf, traffic):
        return {"bound": "tensor", "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                "frac": round(tf / peak, 4), "traffic": traffic, "peak_source": f"{peak_kind} bf16_tflops (burst)"}

    dominant = "backward" if ms_bwd >= ms_fwd else "forward"
    wl = f"{w.name}:{mod_name}"
    traffic_fwd = measured_traffic("attn_fwd", wl)
    traffic_bwd = measured_traffic("attn_bwd", wl)
    line = {
        "metric": METRIC,
        "value": round(job_throughput(f_fwd + f_bwd, world, ms_step), 2),
        "unit": UNIT,
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "ms_per_step_median": round(t["ms_step_median"], 4),
        "ms_per_step_min": round(t["ms_step_min"], 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 Q/K/V/dO, random-free mods)",
        "config": {"workload": f"{w.name}:{mod_name}", "B": B, "Hq": Hq, "Hkv": Hkv, "Sq": Sq, "Skv": Skv,
                   "D": D, "mod": mod_name, "seed": w.seed, "seed_per_rank": "seed + rank (Q/K/V/dO)", "step": "block mask + forward(O, LSE) + backward",
                   "l2": "flushed before every step (256 MiB write, outside the timed events)",
                   "parallelism": f"independent replicas x{world} (no collective on the data path)"},
        "fwd_tflops": round(fwd_tf, 1),
        "bwd_tflops": round(bwd_tf, 1),
        "fwd_frac_of_peak": round(fwd_tf / peak, 4),
        "bwd_frac_of_peak": round(bwd_tf / peak, 4),
        "ms_fwd": round(ms_fwd, 4),
        "ms_bwd": round(ms_bwd, 4),
        "ms_block_mask": round(ms_mask, 4),
        "useful_elements": n_u,
        "roofline": dict(roof(bwd_tf, traffic_bwd) if dominant == "backward" else roof(fwd_tf, traffic_fwd),
                         kernel="attn_bwd_kernel (the backward call: prep, main and dQ cast launches)"
                         if dominant == "backward" else "attn_fwd_kernel"),
        "roofline_forward": roof(fwd_tf, traffic_fwd),
        "roofline_backward": roof(bwd_tf, traffic_bwd),
        "e2e": None if args.no_e2e else {"value": round(job_throughput(f_fwd + f_bwd, world, ms_e2e), 2), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms_e2e, 4),
                "mode": e2e_mode},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if not args.no_configs and not args.all:
        # the other parity configurations, each timed on its own
        configs = {f"{wl}:no_lse_forward": forward_only_entry(ta, pb, stream, flush, args.config_steps, 3,
                                                              world, dev, peak, with_lse=False),
                   f"{wl}:lse_forward": forward_only_entry(ta, pb, stream, flush, args.config_steps, 3,
                                                           world, dev, peak, with_lse=True)}
        del pb, q, k, v, dout, out, lse, dq, dk, dv
        torch.cuda.empty_cache()
        for spec in CONFIG_ENTRIES:
            if spec != wl:
                configs[spec] = config_entry(ta, spec, rank, world, dev, stream, flush, args.config_steps, 3, peak)
        for spec, variant, walk in EXTENSION_ENTRIES:
            name = f"{spec}:{variant or walk}"
            configs[name] = config_entry(ta, spec, rank, world, dev, stream, flush, args.config_steps, 3, peak,
                                         variant=variant, walk=walk)
        line["configs"] = configs
    if rank == 0 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, mod_name, params, seconds=args.cpu_seconds)
    return line


def e2e_pipelined(args, ta, stream, dev, dev_set, host_in, host_out, run_step):
    """End-to-end time per step with the copies overlapped across steps.

    Two device buffer sets alternate.  Step i uploads its inputs into set
    i % 2 on an upload stream (after step i-2's compute has read that set),
    computes on `stream` (after its upload, and after step i-2's outputs in
    that set were read back), and downloads its outputs on a download stream.
    Returns the time from the first timed upload to the last timed download,
    divided by the number of timed steps."""
    import torch
    names = ("q", "k", "v", "dout", "out", "lse", "dq", "dk", "dv")
    sets = [dict(zip(names, dev_set)), {n: torch.empty_like(t) for n, t in zip(names, dev_set)}]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    computed, read_back = [None, None], [None, None]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    for i in range(args.warmup + args.steps):
        b = sets[i & 1]
        if computed[i & 1] is not None:
            s_in.wait_event(computed[i & 1])
        if i == args.warmup:
            start.record(s_in)
        with torch.cuda.stream(s_in):
            for name, h_ in zip(("q", "k", "v", "dout"), host_in):
                b[name].copy_(h_, non_blocking=True)
        uploaded = torch.cuda.Event()
        uploaded.record(s_in)
        stream.wait_event(uploaded)
        if read_back[i & 1] is not None:
            stream.wait_event(read_back[i & 1])
        run_step(tuple(b[n] for n in names), stream)
        done = torch.cuda.Event()
        done.record(stream)
        computed[i & 1] = done
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            for h_, name in zip(host_out, ("out", "dq", "dk", "dv")):
                h_.copy_(b[name], non_blocking=True)
        got = torch.cuda.Event()
        got.record(s_out)
        read_back[i & 1] = got
    end.record(s_out)
    torch.cuda.synchronize()
    return start.elapsed_time(end) / args.steps


# ----------------------------------------------------------------------------- oracle (CPU) arm

def cpu_baseline(w, mod_name, params, seconds=15.0, heads=None):
    """Time the fp64 oracle (as it stands) on whole (b, head) problems of the workload."""
    import oracle
    mod = MOD_NAMES[mod_name]
    bits = draw_workload(w)
    qf, kf, vf, df = (bf16_bits_to_f64(bits[n]) for n in ("q", "k", "v", "dout"))
    G = w.Hq // w.Hkv
    done, flops, t_total = 0, 0.0, 0.0
    for b in range(w.B):
        n_per_head = oracle.useful_elements(mod, params, b + 1, 1, w.Sq, w.Skv) - \
            oracle.useful_elements(mod, params, b, 1, w.Sq, w.Skv)
        for hk in range(w.Hkv):
            if (heads is not None and done >= heads) or (heads is None and t_total >= seconds):
                break
            t0 = time.perf_counter()
            group = [(b, h) for h in range(hk * G, hk * G + G)]
            oracle.attention_forward(qf, kf, vf, w.scale, mod, params, heads=group)
            oracle.attention_backward(qf, kf, vf, df, w.scale, mod, params, groups=[(b, hk)])
            t_total += time.perf_counter() - t0
            done += G
            flops += G * n_per_head * w.D * 14.0
    cores = os.cpu_count()
    return {"value": round(flops / t_total / 1e12, 6), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": f"fp64 numpy oracle, fwd+bwd of {done} of {w.B * w.Hq} (b, head) problems "
                      f"({w.Sq}x{w.Skv}, D={w.D}, {mod_name}), {t_total:.1f} s, BLAS threads = host cores"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w, mod_name = parse_workload(args.workload)
    params = mod_params_for(w, mod_name)
    per_step, step_ms = [], []
    cb = None
    for _ in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        cb = cpu_baseline(w, mod_name, params, heads=1)
        step_ms.append((time.perf_counter() - t0) * 1e3)
        per_step.append(cb["value"])
    vals = per_step[args.warmup:]
    value = sum(vals) / len(vals)
    ms = sum(step_ms[args.warmup:]) / args.steps
    cb["value"] = round(value, 6)
    return {
        "metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": f"{w.name}:{mod_name}", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Sq": w.Sq,
                   "Skv": w.Skv, "D": w.D, "mod": mod_name, "seed": w.seed,
                   "step": "fp64 oracle fwd+bwd of one (b, head) problem of the workload"},
        "cpu_baseline": cb,
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--workload", default="dense:none")
    ap.add_argument("--all", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--e2e-pipeline", action="store_true",
                    help="overlap each step's H2D and D2H with the neighbouring steps' compute")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the headline workload (no per-configuration entries)")
    ap.add_argument("--config-steps", type=int, default=10,
                    help="timed steps of each per-configuration entry")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        if args.all:
            specs = [f"{n}:{m}" for n, w in WORKLOADS.items() for m in w.mods]
            for s in specs:
                args.workload = s
                line = run_gpu(args, rank, world, local_rank)
                if rank == 0:
                    print(json.dumps(line), flush=True)
        else:
            line = run_gpu(args, rank, world, local_rank)
            if rank == 0:
                print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
