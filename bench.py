"""Benchmark of the RotateAttention INT4 forward hot path on B200.

One step = one pass of the whole hot path over one batch of synthetic input:
the fused prologue (ra_rope_rotate_quant) followed by the INT4 attention
(ra_attn_int4), on the Wan-14B-480p-like attention shape (B=1, H=40,
N=32760, D=128, segments 44/42/42, interleaved rotation, 128x64 blocks).

Metric: INT4 attention TOPS = 4 N^2 D H / t, with t the device time of a whole
step.  Prints one JSON line (rank 0).  See --help for options.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched by torch.distributed.run): every rank runs its own
independent batch (weak scaling, no collective on the data path); the step
time is the maximum over ranks.
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "INT4 attn TOPS (4N²DH/t) & % INT8 tensor peak at N=32760,H=40,D=128"
# rope table (two for the interleaved rotation: the fused table and the plain
# one the channel reduce uses), channel reduce, finalize, quantise, attention
def kernels_per_step(rot: int) -> int:
    return 6 if rot == 1 else 5
# (name, p_mode, l_mode) of the attention's ablation switches timed after the step.
ABLATIONS = (("fp32_l", 0, 1), ("local_max", 1, 0), ("local_max_fp32_l", 1, 1),
             ("symmetric_p", 2, 0), ("symmetric_p_fp32_l", 2, 1))


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        return {"hbm_gbs": float(m["hbm_gbs"]), "bf16_tflops": float(m["bf16_tflops"]),
                "bf16_tflops_sustained": float(m.get("bf16_tflops_sustained", m["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self._stop = threading.Event()
        self._t = None

    def _run(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip()
                if out:
                    self.samples.append([s.strip() for s in out.split(",")])
            except Exception:
                pass
            self._stop.wait(0.2)

    def __enter__(self):
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        self._t.join(timeout=10)

    def summary(self):
        sm = [float(s[0]) for s in self.samples if s[0].replace(".", "").isdigit()]
        mx = [float(s[1]) for s in self.samples if s[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for s in self.samples for i in range(4)
                          if len(s) > 3 + i and s[3 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.samples)}


def _workload(name, block_k=None):
    from synth import inputs as si
    wl = si.WORKLOADS[name]
    return wl if block_k is None else wl.with_(block_k=block_k)


def _config(wl, extra=None):
    rot = {0: "none", 1: "interleaved", 2: "half", 3: "full"}[wl.rot]
    c = {"workload": f"{wl.name}: B={wl.B} H={wl.H} N={wl.N} (grid {wl.grid[0]}x{wl.grid[1]}x{wl.grid[2]}) "
                     f"D={wl.D} seg={wl.seg[0]}/{wl.seg[1]}/{wl.seg[2]} rot={rot} blocks {wl.block_q}x{wl.block_k}",
         "B": wl.B, "H": wl.H, "N": wl.N, "D": wl.D, "seg": list(wl.seg), "rot": rot,
         "block_q": wl.block_q, "block_k": wl.block_k,
         "l2": "inputs larger than L2: Q/K/V bf16 = %.2f GB per step" % (3 * wl.B * wl.H * wl.N * wl.D * 2 / 1e9)}
    if extra:
        c.update(extra)
    return c


def cpu_baseline(wl, target_s: float = 15.0, x=None):
    """The oracle, as it stands, on a bounded sample of the workload: the
    prologue of head 0 and the attention of as many 128-row query tiles of head 0
    as fit in about target_s seconds (tiles visited in a strided order so the
    sample spans the sequence); value prorated to the metric's unit."""
    import oracle
    from synth import inputs as si
    if x is None:
        x = si.make_inputs(wl, heads=(0,))
    p = oracle.problem(wl)
    t0 = time.perf_counter()
    h = oracle.prologue_head(p, x["q"][0, 0], x["k"][0, 0], x["v"][0, 0], x["pos"])
    t_pro = time.perf_counter() - t0
    ntiles = -(-wl.N // 128)
    stride = max(1, ntiles // 16)
    order = [t for off in range(stride) for t in range(off, ntiles, stride)]
    rows = 0
    t_att = 0.0
    for tile in order:
        if t_att >= target_s:
            break
        r0 = tile * 128
        r1 = min(r0 + 128, wl.N)
        t0 = time.perf_counter()
        oracle.attention_int4_rows(p, h, r0, r1)
        t_att += time.perf_counter() - t0
        rows += r1 - r0
    t = t_att + t_pro * rows / wl.N
    ops = 4.0 * rows * wl.N * wl.D
    return {"value": ops / t / 1e12, "unit": "TOPS", "cores": oracle.num_threads(), "kind": "oracle",
            "seconds": t,
            "sample": f"head 0 of {wl.name}: prologue of all {wl.N} tokens (prorated to the rows) + "
                      f"attention of {rows} query rows over all {wl.N} keys; {t:.1f} s of CPU time"}


def max_over_ranks(value: float, device) -> float:
    """The largest of every rank's value (all ranks call this in the same
    order); with one rank, the value itself."""
    import torch
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(world: int, ops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job TOPS: every rank runs its own batch of ops_per_rank per step,
    and the step takes the slowest rank's time."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


def _attn_traffic():
    """DRAM bytes per attention launch from the committed ncu summary, or None
    when the attention kernel's sources changed since those counters were taken."""
    import hashlib
    import re
    path = os.path.join(ROOT, "profiles", "launches_wan.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    mt = re.search(r"traffic_bytes_per_launch: (\d+)", text)
    mh = re.search(r"kernel_sources_sha256: ([0-9a-f]{64})", text)
    if not mt or not mh:
        return None
    h = hashlib.sha256()
    for f in ("ra_attn_int4.cu", "ra_common.cuh"):
        with open(os.path.join(ROOT, "int4_quantized_flashattention_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return int(mt.group(1)) if h.hexdigest() == mh.group(1) else None


def run_ours(args, rank, world, local_rank):
    import numpy as np
    import torch

    import __graft_entry__
    __graft_entry__.build()
    import int4_quantized_flashattention_b200 as ra
    from synth import inputs as si

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = _workload(args.workload, args.block_k)
    x = si.make_inputs(wl)
    p = ra.Problem.make(wl.B, wl.H, wl.D, wl.seg, wl.grid, theta=wl.theta, rot=wl.rot,
                        block_q=wl.block_q, block_k=wl.block_k)
    host = {n: torch.from_numpy(x[n + "_bits"]).view(torch.bfloat16).pin_memory() for n in ("q", "k", "v")}
    pos_h = torch.from_numpy(x["pos"]).pin_memory()
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    pos = pos_h.to(dev)
    ws = torch.empty(ra.workspace_bytes(p), dtype=torch.uint8, device=dev)
    codes = ra.rope_rotate_quant(p, q, k, v, pos, workspace=ws)
    out = torch.empty(wl.B, wl.H, wl.N, wl.D, dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ra.rope_rotate_quant(p, q, k, v, pos, out=codes, workspace=ws)
        ra.attn_int4(p, codes, out=out)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ra.sync_status() != 0:
        raise RuntimeError("device status not ok after warm-up")

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
           torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clk:
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        for i in range(args.steps):
            a, b, c = ev[i]
            a.record(stream)
            ra.rope_rotate_quant(p, q, k, v, pos, out=codes, workspace=ws)
            b.record(stream)
            ra.attn_int4(p, codes, out=out)
            c.record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    total_ms = start.elapsed_time(end)
    pro_ms = [a.elapsed_time(b) for a, b, _ in ev]
    att_ms = [b.elapsed_time(c) for _, b, c in ev]
    status = ra.sync_status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    total_ms = max_over_ranks(total_ms, dev)

    # End to end through the public API with host buffers: every step copies its
    # Q/K/V and positions from pinned host memory, runs the prologue and the
    # attention, and copies the output back.  The copies run on their own
    # streams with two device buffer sets, so step i+1's inputs arrive and step
    # i-1's output leaves while step i's kernels run; every copy is inside the
    # timed region.
    out_h = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    dev_in = [dict(q=q, k=k, v=v, pos=pos),
              dict(q=torch.empty_like(q), k=torch.empty_like(k), v=torch.empty_like(v), pos=torch.empty_like(pos))]
    outs = [out, torch.empty_like(out)]
    s_h2d, s_d2h = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_ready, in_free, out_ready, out_free = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(4))

    def e2e_steps(n):
        for i in range(n):
            b = i % 2
            d = dev_in[b]
            with torch.cuda.stream(s_h2d):
                if i >= 2:
                    s_h2d.wait_event(in_free[b])        # the prologue of step i-2 has read them
                for name in ("q", "k", "v"):
                    d[name].copy_(host[name], non_blocking=True)
                d["pos"].copy_(pos_h, non_blocking=True)
                in_ready[b].record(s_h2d)
            stream.wait_event(in_ready[b])
            ra.rope_rotate_quant(p, d["q"], d["k"], d["v"], d["pos"], out=codes, workspace=ws)
            in_free[b].record(stream)
            if i >= 2:
                stream.wait_event(out_free[b])          # step i-2's output has left
            ra.attn_int4(p, codes, out=outs[b])
            out_ready[b].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(out_ready[b])
                out_h.copy_(outs[b], non_blocking=True)
                out_free[b].record(s_d2h)

    e2e_steps(2)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_h2d.wait_event(e0)
    s_d2h.wait_event(e0)
    e2e_steps(args.steps)
    last = torch.cuda.Event()
    last.record(s_d2h)
    stream.wait_event(last)
    e1.record(stream)
    torch.cuda.synchronize(dev)
    if ra.sync_status() != 0:
        raise RuntimeError("device status not ok after the end-to-end steps")
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dev)
    del dev_in, outs
    h2d = sum(host[n].numel() * 2 for n in ("q", "k", "v")) + pos_h.numel() * 4
    d2h = out_h.numel() * 2

    # The bf16 fallback (plain RoPE'd q, k and v in bf16), timed on its own:
    # not part of the INT4 step, reported against the bf16 tensor peak.
    qr, kr = ra.rope_bf16(p, q, k, pos, workspace=ws)
    out_b = torch.empty_like(out)
    # the fallback's key block (a tiling choice that leaves its result unchanged)
    pb = ra.Problem.make(wl.B, wl.H, wl.D, wl.seg, wl.grid, theta=wl.theta, rot=wl.rot,
                         block_q=wl.block_q, block_k=min(wl.block_k, 64))
    for _ in range(2):
        ra.attn_bf16_fallback(pb, qr, kr, v, out=out_b)
    torch.cuda.synchronize(dev)
    fb = []
    for _ in range(max(3, args.steps // 4)):
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        ra.attn_bf16_fallback(pb, qr, kr, v, out=out_b)
        a1.record(stream)
        torch.cuda.synchronize(dev)
        fb.append(a0.elapsed_time(a1))
    if ra.sync_status() != 0:
        raise RuntimeError("device status not ok after the bf16 fallback")
    fb_ms = statistics.median(fb)
    del qr, kr, out_b

    # The fused-Q step: the K/V-only prologue, then the attention kernel that
    # quantises Q itself (no Q codes in HBM).  Timed like the step on the same
    # inputs, after it; its output must equal the step's bit for bit.
    fq = None
    if wl.block_k == 64:
        kv = ra.rope_rotate_quant(p, None, k, v, pos, workspace=ws)
        out_f = torch.empty_like(out)
        for _ in range(2):
            ra.rope_rotate_quant(p, None, k, v, pos, out=kv, workspace=ws)
            ra.attn_int4_qfused(p, q, pos, kv, out=out_f, workspace=ws)
        torch.cuda.synchronize(dev)
        fpro, fatt, fall = [], [], []
        for _ in range(max(3, args.steps // 2)):
            a0, a1, a2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a0.record(stream)
            ra.rope_rotate_quant(p, None, k, v, pos, out=kv, workspace=ws)
            a1.record(stream)
            ra.attn_int4_qfused(p, q, pos, kv, out=out_f, workspace=ws)
            a2.record(stream)
            torch.cuda.synchronize(dev)
            fpro.append(a0.elapsed_time(a1))
            fatt.append(a1.elapsed_time(a2))
            fall.append(a0.elapsed_time(a2))
        if ra.sync_status() != 0:
            raise RuntimeError("device status not ok after the fused-Q step")
        ra.rope_rotate_quant(p, q, k, v, pos, out=codes, workspace=ws)
        ra.attn_int4(p, codes, out=out)
        torch.cuda.synchronize(dev)
        fq = {"ms_per_step": round(statistics.median(fall), 4),
              "prologue_kv_ms": round(statistics.median(fpro), 4),
              "attention_ms": round(statistics.median(fatt), 4),
              "identical_to_step_output": bool(torch.equal(out_f.view(torch.int16), out.view(torch.int16)))}
        del kv, out_f

    # The s8 code layout: the prologue writes one code per byte and the
    # attention loads Q, K and V tiles by TMA straight into its MMA operands
    # (no widening).  Timed like the step, after it; its output must equal
    # the step's bit for bit.
    s8 = None
    if wl.block_k == 64:
        c8 = ra.rope_rotate_quant_s8(p, q, k, v, pos, workspace=ws)
        out_8 = torch.empty_like(out)
        for _ in range(2):
            ra.rope_rotate_quant_s8(p, q, k, v, pos, out=c8, workspace=ws)
            ra.attn_int4_s8(p, c8, out=out_8)
        torch.cuda.synchronize(dev)
        spro, satt, sall = [], [], []
        for _ in range(max(3, args.steps // 2)):
            a0, a1, a2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            a0.record(stream)
            ra.rope_rotate_quant_s8(p, q, k, v, pos, out=c8, workspace=ws)
            a1.record(stream)
            ra.attn_int4_s8(p, c8, out=out_8)
            a2.record(stream)
            torch.cuda.synchronize(dev)
            spro.append(a0.elapsed_time(a1))
            satt.append(a1.elapsed_time(a2))
            sall.append(a0.elapsed_time(a2))
        if ra.sync_status() != 0:
            raise RuntimeError("device status not ok after the s8-layout step")
        ra.rope_rotate_quant(p, q, k, v, pos, out=codes, workspace=ws)
        ra.attn_int4(p, codes, out=out)
        torch.cuda.synchronize(dev)
        s8_att = statistics.median(satt)
        s8 = {"ms_per_step": round(statistics.median(sall), 4),
              "prologue_ms": round(statistics.median(spro), 4),
              "attention_ms": round(s8_att, 4),
              "attention_tops": round(wl.attn_ops() / (s8_att * 1e-3) / 1e12, 1),
              "attention_frac": round(wl.attn_ops() / (s8_att * 1e-3) / 1e12 / (2.0 * _peaks()["bf16_tflops"]), 4),
              "identical_to_step_output": bool(torch.equal(out_8.view(torch.int16), out.view(torch.int16)))}
        del c8, out_8

    # The ablation switches of the attention (block-local max, symmetric P,
    # fp32 denominator), each timed on its own on the same codes; not part of
    # the INT4 step.
    abl = {}
    if wl.block_k in (64, 128) and not args.quick:
        for name, pm, lm in ABLATIONS:
            for _ in range(2):
                ra.attn_int4(p, codes, out=out, p_mode=pm, l_mode=lm)
            torch.cuda.synchronize(dev)
            ts = []
            for _ in range(max(3, args.steps // 8)):
                a0 = torch.cuda.Event(enable_timing=True)
                a1 = torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                ra.attn_int4(p, codes, out=out, p_mode=pm, l_mode=lm)
                a1.record(stream)
                torch.cuda.synchronize(dev)
                ts.append(a0.elapsed_time(a1))
            if ra.sync_status() != 0:
                raise RuntimeError(f"device status not ok after the {name} ablation")
            abl[name] = statistics.median(ts)

    # The prologue under each rotation mode (full D x D Hadamard against the
    # 2x2 rotations), timed on the same inputs after everything else.
    rot_ms = {}
    for rname, rmode in () if args.quick else (("interleaved", ra.ROT_INTERLEAVED), ("half", ra.ROT_HALF), ("full", ra.ROT_FULL),
                         ("none", ra.ROT_NONE)):
        pr = ra.Problem.make(wl.B, wl.H, wl.D, wl.seg, wl.grid, theta=wl.theta, rot=rmode,
                             block_q=wl.block_q, block_k=wl.block_k)
        for _ in range(2):
            ra.rope_rotate_quant(pr, q, k, v, pos, out=codes, workspace=ws)
        torch.cuda.synchronize(dev)
        ts = []
        for _ in range(max(3, args.steps // 4)):
            a0 = torch.cuda.Event(enable_timing=True)
            a1 = torch.cuda.Event(enable_timing=True)
            a0.record(stream)
            ra.rope_rotate_quant(pr, q, k, v, pos, out=codes, workspace=ws)
            a1.record(stream)
            torch.cuda.synchronize(dev)
            ts.append(a0.elapsed_time(a1))
        if ra.sync_status() != 0:
            raise RuntimeError(f"device status not ok after the {rname} prologue")
        rot_ms[rname] = statistics.median(ts)

    ops = wl.attn_ops()
    ms_step = total_ms / args.steps
    value = weak_scaling_value(world, ops, ms_step)
    pk = _peaks()
    int8_peak = 2.0 * pk["bf16_tflops"]        # nominal dense int8 / bf16 ratio on B200 = 2
    att_med = statistics.median(att_ms)
    pro_med = statistics.median(pro_ms)
    achieved = ops / (att_med * 1e-3) / 1e12
    pro_bytes = prologue_bytes(wl)
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "TOPS", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int4", "data": "synthetic (seeded, outlier-structured; no model weights)",
        "config": _config(wl, {"parallelism": f"independent batch per GPU x{world}"}),
        "e2e": {"value": round(weak_scaling_value(world, ops, e2e_ms), 2), "unit": "TOPS",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 4),
                "copies": "H2D and D2H on their own streams, overlapping the previous and next steps' kernels"},
        "roofline": {"bound": "tensor", "kernel": "attn_int4_pair_kernel" if wl.block_k == 128 else "attn_int4_kernel", "achieved": round(achieved, 1),
                     "peak": round(int8_peak, 1), "unit": "TFLOP/s", "frac": round(achieved / int8_peak, 4),
                     "peak_source": f"2 x {pk['source']} bf16 burst {pk['bf16_tflops']} TFLOP/s (int8 ops/s)",
                     "traffic": _attn_traffic() if (args.workload == "wan" and args.block_k is None) else None},
        "prologue": {"ms": round(pro_med, 4), "bytes": pro_bytes,
                     "achieved_gbs": round(pro_bytes / (pro_med * 1e-3) / 1e9, 1),
                     "peak_gbs": pk["hbm_gbs"], "frac": round(pro_bytes / (pro_med * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                     "ratio_to_attention": round(pro_med / att_med, 4)},
        "attention_ms": round(att_med, 4),
        "bf16_fallback": {"ms": round(fb_ms, 4), "tflops": round(ops / (fb_ms * 1e-3) / 1e12, 1),
                          "peak": pk["bf16_tflops"], "frac": round(ops / (fb_ms * 1e-3) / 1e12 / pk["bf16_tflops"], 4),
                          "kernel": "attn_bf16_kernel", "note": "4N^2DH flops of bf16 attention on the RoPE'd inputs"},
        "ablations": {n: {"ms": round(t, 4), "tops": round(ops / (t * 1e-3) / 1e12, 1),
                          "frac": round(ops / (t * 1e-3) / 1e12 / int8_peak, 4)} for n, t in abl.items()},
        "prologue_by_rotation_ms": {n: round(t, 4) for n, t in rot_ms.items()},
        "fused_q": fq,
        "s8_layout": s8,
        "gpu_launches": kernels_per_step(wl.rot) * args.steps,
        "clocks": clk.summary(),
    }
    return res


def prologue_bytes(wl):
    """Algorithmic bytes of the prologue: Q once, K and V twice (bf16), packed
    codes, per-token and per-channel scales, K means, V column sums."""
    B, H, N, D = wl.B, wl.H, wl.N, wl.D
    el = 2 if wl.dtype == "bf16" else 4
    reads = (1 + 2 + 2) * B * H * N * D * el
    nb = -(-N // wl.block_k)
    writes = 3 * B * H * N * D // 2 + 2 * 4 * B * H * N + 3 * 4 * B * H * D + 4 * B * H * nb * D
    return reads + writes


def run_reference(args):
    """The oracle as it stands, on the host cores, one bounded sample per step.

    A whole step of the workload takes the oracle many minutes, so each step
    runs a bounded sample (the prologue of head 0 and as many query tiles as
    fit in the per-step budget, every step within the run's few minutes); the
    line's value is that sample's rate and ms_per_step the time the whole
    step would take at it, marked as extrapolated, with the sample's own time
    beside it."""
    wl = _workload(args.workload, args.block_k)
    import oracle
    oracle.lib()
    from synth import inputs as si
    x = si.make_inputs(wl, heads=(0,))
    # each step is one bounded sample; the whole run stays within a few minutes
    per_step = max(1.0, min(args.ref_seconds, 180.0 / max(1, args.warmup + args.steps)))
    vals = []
    sample_s = []
    base = None
    for i in range(args.warmup + args.steps):
        r = cpu_baseline(wl, target_s=per_step, x=x)
        if i >= args.warmup:
            vals.append(r["value"])
            sample_s.append(r["seconds"])
            base = r
    v = statistics.median(vals)
    ms = 4.0 * wl.N * wl.N * wl.D * wl.H * wl.B / (v * 1e12) * 1e3
    return {"metric": METRIC, "value": round(v, 6), "unit": "TOPS", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 1), "extrapolated": True,
            "sample_ms_per_step": round(1e3 * statistics.median(sample_s), 1),
            "extrapolation": f"ms_per_step = 4 N^2 D H / value: the whole step at the sampled rate; each step "
                             f"ran a {per_step:.1f} s sample ({base['sample']})",
            "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int4", "data": "synthetic (seeded, outlier-structured; no model weights)",
            "config": _config(wl), "impl": "reference",
            "cpu_baseline": {"value": round(v, 6), "unit": "TOPS", "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": round(v, 6), "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan")
    ap.add_argument("--block-k", type=int, default=None, help="override the workload's key block size")
    ap.add_argument("--quick", action="store_true",
                    help="skip the ablation modes and the per-rotation prologue timings (for config sweeps)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=10.0, help="CPU seconds per reference sample")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                res["cpu_baseline"] = cpu_baseline(_workload(args.workload, args.block_k))
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
