#!/usr/bin/env python
"""Benchmark of fused windowed-RoPE attention (forward + backward) on B200.

One step = one pass of the whole hot path over one batch: forward and
backward of every attention block of the workload.  The headline workload is
the attention of all four FlashSwin-T stages at 256 x 256 input with patch 2
(grids 128/64/32/16, heads 3/6/12/24, windows 32/32/32/16, batch 128), one
unshifted and one shifted block per stage (both unshifted at stage 4, whose
window is the whole grid).  Inputs are seeded synthetic bf16 N(0,1) tensors
of the workload's shapes (the pages measure on ImageNet at 256x256; no
dataset is used).

Prints ONE JSON line (rank 0).  `--impl reference` times the fp64 CPU oracle
instead, on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "windowed-RoPE attention fwd+bwd TFLOP/s (% BF16 peak), tokens/s, peak GB"
HEAD_DIM = 32

WORKLOADS = {
    # the attention of all four FlashSwin-T stages at 256x256 input, p=2, batch 128: grids 128/64/32/16,
    # heads 3/6/12/24, windows 32/32/32/16; an unshifted and a shifted (s = M/2) block per stage, both
    # unshifted at stage 4 (the window clamped to the grid)
    "flashswin_t_p2_4stage": dict(stages=[
        dict(B=128, H=128, W=128, heads=3, M=32, shifts=(0, 16)),
        dict(B=128, H=64, W=64, heads=6, M=32, shifts=(0, 16)),
        dict(B=128, H=32, W=32, heads=12, M=32, shifts=(0, 16)),
        dict(B=128, H=16, W=16, heads=24, M=16, shifts=(0, 0)),
    ], qk_scale=1.0),
    # Swin-T stage-1 shape at p=4 (64x64 grid at 256x256 input), window 8, unshifted and shifted blocks
    "swin_t_stage1_p4_m8": dict(B=128, H=64, W=64, heads=3, M=8, shifts=(0, 4), qk_scale=1.0),
    # FlashSwin-T stage 1 at p=2 (128x128 grid), window 32, shifted block
    "flashswin_t_stage1_p2_m32": dict(B=128, H=128, W=128, heads=3, M=32, shifts=(16,), qk_scale=1.0),
    # 512x512 input at p=2, windows 32 and 64 (4096-token windows), Q and K scaled by 3
    "highres_p2_m32": dict(B=16, H=256, W=256, heads=3, M=32, shifts=(16,), qk_scale=3.0),
    "highres_p2_m64": dict(B=16, H=256, W=256, heads=3, M=64, shifts=(32,), qk_scale=3.0),
    # inference forward (no LSE written) at the shape of FlashSwin's inference-throughput figure:
    # p=4 (64x64 grid at 256x256 input), batch 128, windows 8 to 32, unshifted and shifted blocks
    "swin_t_stage1_p4_infer_m8": dict(B=128, H=64, W=64, heads=3, M=8, shifts=(0, 4), qk_scale=1.0, infer=True),
    "swin_t_stage1_p4_infer_m16": dict(B=128, H=64, W=64, heads=3, M=16, shifts=(0, 8), qk_scale=1.0, infer=True),
    "swin_t_stage1_p4_infer_m32": dict(B=128, H=64, W=64, heads=3, M=32, shifts=(0, 16), qk_scale=1.0, infer=True),
    # an 800 x 1333 detection input at p=4: a 200 x 334 grid, not a multiple of the window, worked on
    # padded with zero tokens (200 x 336 at window 8; 224 x 352 at window 32), batch 16
    "swin_t_det_stage1_p4_m8": dict(B=16, H=200, W=334, heads=3, M=8, shifts=(0, 4), qk_scale=1.0),
    "flashswin_t_det_stage1_p4_m32": dict(B=16, H=200, W=334, heads=3, M=32, shifts=(0, 16), qk_scale=1.0),
    # heads of 64 channels (the wide kernels): the FlashSwin-T stage-1 grid at p=2 with 3 heads of d=64,
    # window 32, shifted block; batch 64 keeps each tensor at the size of the d=32 workload's
    "flashswin_stage1_p2_m32_d64": dict(B=64, H=128, W=128, heads=3, M=32, shifts=(16,), qk_scale=1.0, d=64),
    # the low-rank additive bias variant (FlashBias-T: a trainable rank-16 bias factorization, with RoPE
    # here) at the FlashSwin-T stage-1 shapes, p=2 window 32 and p=4 window 8
    "flashbias_t_stage1_p2_m32": dict(B=128, H=128, W=128, heads=3, M=32, shifts=(0, 16), qk_scale=1.0, lrbias=True),
    "flashbias_t_stage1_p4_m8": dict(B=128, H=64, W=64, heads=3, M=8, shifts=(0, 4), qk_scale=1.0, lrbias=True),
}
LRBIAS_RANK = 16
HEADLINE = "flashswin_t_p2_4stage"
SPEC_BF16_TFLOPS = 2250.0  # NVIDIA's dense bf16 figure for one B200: a spec value, not a measurement

# the window-attention block of a Swin layer with its qkv and output projections (inference),
# Swin-T stage 1 at p=4: C = 96 channels in 3 heads, window 8, unshifted and shifted blocks
BLOCK_WORKLOADS = {
    "swin_t_stage1_p4_block_infer_m8": dict(B=128, H=64, W=64, heads=3, M=8, shifts=(0, 4)),
}


def unmasked_pairs(B, H, W, heads, M, s) -> int:
    """Number of (query, key) pairs that attend (same window, same shift-region label), on the
    grid padded to multiples of M (padded tokens attend like the others)."""
    H, W = -(-H // M) * M, -(-W // M) * M

    def sizes(X):
        if s == 0:
            return [[M]] * (X // M)
        out = [[M]] * (X // M - 1)
        out.append([M - s, s])  # last window row/column: two regions of the shifted grid
        return out
    rows, cols = sizes(H), sizes(W)
    per_image = 0
    for rr in rows:
        for cc in cols:
            per_image += sum((a * b) ** 2 for a in rr for b in cc)
    return per_image * B * heads


def _include_closure(root: str, tu: str) -> list:
    """The translation unit and the local headers it includes, directly or not."""
    seen, todo = set(), [tu]
    while todo:
        f = todo.pop()
        path = os.path.join(root, f)
        if f in seen or not os.path.exists(path):
            continue
        seen.add(f)
        with open(path) as fh:
            for line in fh:
                m = re.match(r'\s*#include "([^"/]+)"', line)
                if m:
                    todo.append(m.group(1))
    return sorted(seen)


def kernel_sources_sha256(tu: str) -> str:
    """Hash of a kernel's sources (its translation unit, the local headers it includes)
    and of the build script; stored DRAM traffic is valid only for the build it was
    captured on."""
    pkg = os.path.join(os.path.dirname(os.path.abspath(__file__)), "vision_transformer_windowed_b200")
    root = os.path.join(pkg, "csrc")
    h = hashlib.sha256()
    for f in _include_closure(root, tu):
        h.update(f.encode())
        with open(os.path.join(root, f), "rb") as fh:
            h.update(fh.read())
    with open(os.path.join(pkg, "build.py"), "rb") as fh:
        h.update(fh.read())
    return h.hexdigest()


def measured_traffic(phase: str, workload: str):
    """DRAM bytes per step of the workload's `phase` kernel from the committed ncu capture, or None
    when there is none for this workload or the kernel's sources changed since."""
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "traffic.json")
    try:
        with open(path) as fh:
            recs = json.load(fh).get("records", [])
    except (OSError, ValueError):
        return None
    for rec in recs:
        if rec.get("phase") == phase and rec.get("workload") == workload:
            if rec.get("sources_sha256") != kernel_sources_sha256(rec["source"]):
                return None
            return rec["bytes_per_step"]
    return None


def stages_of(wl) -> list:
    """A workload as a list of stages: one grid shape each, with the shifts of its blocks (and its
    head dimension, 32 unless given)."""
    if "stages" in wl:
        return [dict(st, qk_scale=st.get("qk_scale", wl.get("qk_scale", 1.0)), infer=wl.get("infer", False),
                     d=st.get("d", wl.get("d", HEAD_DIM)), lrbias=wl.get("lrbias", False))
                for st in wl["stages"]]
    return [dict(wl, d=wl.get("d", HEAD_DIM), lrbias=wl.get("lrbias", False))]


def blocks_of(wl) -> list:
    """(stage, shift) of every attention block of one step, in the order the step runs them."""
    return [(st, s) for st in stages_of(wl) for s in st["shifts"]]


def pair_flops(st) -> tuple[float, float]:
    """FLOPs per attending pair of the forward and the backward products: 4 d forward (S and P V)
    and 10 d backward (S again, dP, dV, dK, dQ); with the rank-r low-rank bias the score product
    and the two gradient products that carry the factors contract over d + r channels, so
    4 d + 2 r and 10 d + 6 r."""
    d = st.get("d", HEAD_DIM)
    r = LRBIAS_RANK if st.get("lrbias") else 0
    return 4.0 * d + 2.0 * r, 10.0 * d + 6.0 * r


def workload_flops(wl) -> tuple[float, float]:
    """Useful forward and backward FLOPs of one step (per attending pair: `pair_flops`)."""
    fwd = bwd = 0.0
    for st, s in blocks_of(wl):
        pairs = unmasked_pairs(st["B"], st["H"], st["W"], st["heads"], st["M"], s)
        pf, pb = pair_flops(st)
        fwd += pf * pairs
        bwd += pb * pairs
    return fwd, bwd


def workload_tokens(wl) -> int:
    """Token positions the step's blocks process (B * H * W per block)."""
    return sum(st["B"] * st["H"] * st["W"] for st, _ in blocks_of(wl))


PHASES = ["fwd", "bwd_prep", "bwd_main", "bwd_post", "bwd_dtheta"]


def phase_work(st, s) -> dict:
    """Algorithmic work of one block per kernel phase: flops of its products and the bytes it must
    move.  Windows inside one tile run the whole backward as one kernel (Q, K, V, O, dO read, dQ, dK,
    dV written, LSE and D: 520 B per token-head row, recorded as bwd_main); larger windows run the
    training pair: the forward phase writes the rotated q', k' images (q, k in, images out, 256 B)
    and runs the forward on them (images, v in, o, lse out, 260 B); the backward runs prep / main /
    post with workspace round trips (prep: v, o, dO, lse in, lse2, D and the zeroed dQ' accumulator
    out, 332 B, and the per-window scale pass over lse2, 8 B, timed with it; main: the images, dO, v,
    lse2, D in, dk, dv out, 392 B; post: the dQ' accumulator and q in, dq out, 256 B).  An inference
    forward reads q, k, v and writes o (256 B)."""
    B, H, W, heads, M, d = st["B"], st["H"], st["W"], st["heads"], st["M"], st.get("d", HEAD_DIM)
    rows = B * H * W * heads
    pairs = unmasked_pairs(B, H, W, heads, M, s)
    small = M * M < 128
    pf, pb = pair_flops(st)
    if st.get("lrbias"):  # the bias kernels (plain pipelines at every window size): prep reads dO, o,
        # v and lse, writes lse2 and D and zeroes the fp32 accumulator rows (256 B); main reads q, k, v,
        # dO, lse2 and D and writes dk, dv; post reads the accumulator's dQ' part and q and writes dq;
        # the window sums read the dU / dW shares (the factors themselves stay in L2)
        nbytes = {"fwd": (256 if st.get("infer") else 260) * rows, "bwd_prep": 460 * rows,
                  "bwd_main": 392 * rows, "bwd_post": 256 * rows, "bwd_dtheta": 128 * rows}
        return {"bytes": nbytes, "flops": {"fwd": pf * pairs, "bwd_main": pb * pairs}, "hbm_bound": False}
    if d == 64:  # the wide kernels: prep reads dO, o, v and lse, writes lse2 and D and zeroes the fp32
        # dQ' accumulator; main reads q, k, v, dO, lse2 and D, writes dk, dv (the dQ' additions
        # resolve in L2); post reads the accumulator and q, writes dq
        nbytes = {"fwd": (512 if st.get("infer") else 516) * rows, "bwd_prep": 652 * rows,
                  "bwd_main": 776 * rows, "bwd_post": 512 * rows, "bwd_dtheta": 0}
    else:
        fwd_row = 256 if st.get("infer") else (260 if small else 516)
        nbytes = {"fwd": fwd_row * rows, "bwd_prep": 0 if small else 340 * rows,
                  "bwd_main": (520 if small else 392) * rows, "bwd_post": 0 if small else 256 * rows,
                  "bwd_dtheta": 0}
    flops = {"fwd": pf * pairs, "bwd_main": pb * pairs}
    return {"bytes": nbytes, "flops": flops, "hbm_bound": small and d == 32}


def mufu_ceiling_tflops(flops_per_exp: float, sm_mhz: float, sms: int = 148) -> float:
    """The ceiling one MUFU exp2 per score element puts on a kernel: 16 exp2 per clock per SM
    (the CUDA guide's throughput table for compute capability 10.0) times the SM count and clock,
    times the flops counted per element (4 d forward, 10 d backward)."""
    return flops_per_exp * 16 * sms * sm_mhz * 1e6 / 1e12


def roofline(wl, res, peaks, sm_mhz=None) -> dict:
    """Roofline of the step's dominant kernel (largest share of the step's kernel time): its
    algorithmic work over all launches of one step divided by its measured time per step.  Windows
    inside one tile, and the row passes of the larger-window backward, are bound by HBM (reported in
    GB/s against the measured copy bandwidth); the larger-window attention kernels by the tensor
    cores (TFLOP/s against the measured cuBLAS bf16 peak, the sustained figure since the kernel runs
    inside a long step), with the MUFU ceiling beside it."""
    blocks = blocks_of(wl)
    work = [phase_work(st, s) for st, s in blocks]
    ph = res["phase_ms_per_step"]
    dom = max(ph, key=lambda n: ph[n])
    hbm = all(w["hbm_bound"] for w in work) or dom in ("bwd_prep", "bwd_post", "bwd_dtheta")
    t = ph[dom] * 1e-3
    if hbm:
        nb = sum(w["bytes"][dom] for w in work)
        achieved = nb / t / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                "algorithmic_bytes_per_step": nb, "peak_note": f"HBM copy bandwidth, {peaks['source']}"}
    else:
        fl = sum(w["flops"].get(dom, 0.0) for w in work)
        achieved = fl / t / 1e12
        peak = peaks["bf16_tflops_sustained"]
        roof = {"kernel": dom, "bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "frac_of_burst": achieved / peaks["bf16_tflops"], "traffic": None,
                "algorithmic_flops_per_step": fl, "algorithmic_bytes_per_step": sum(w["bytes"][dom] for w in work),
                "peak_note": f"cuBLAS bf16 sustained (burst {peaks['bf16_tflops']:.1f}), {peaks['source']}"}
        per_exp = pair_flops(blocks[0][0])[0 if dom == "fwd" else 1]
        mhz = sm_mhz or 1965.0
        roof["mufu_ceiling_tflops"] = mufu_ceiling_tflops(per_exp, mhz)
        roof["mufu_note"] = (f"one MUFU exp2 per score element: 16/clk/SM x 148 SMs x {mhz:.0f} MHz x "
                             f"{per_exp:.0f} flops per element")
    roof["launches_per_step"] = len(blocks)
    roof["avg_launch_ms"] = ph[dom] / len(blocks)
    roof["ms_per_step"] = ph[dom]
    return roof


def block_flops(wl) -> float:
    """Useful FLOPs of one block step: the two projections (2 * 4 C^2 per token) and the
    attention forward (4 d per attending pair), at every shift."""
    C = wl["heads"] * HEAD_DIM
    tokens = wl["B"] * wl["H"] * wl["W"]
    pairs = sum(unmasked_pairs(wl["B"], wl["H"], wl["W"], wl["heads"], wl["M"], s) for s in wl["shifts"])
    return 2.0 * 4 * C * C * tokens * len(wl["shifts"]) + 4.0 * HEAD_DIM * pairs


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clock/throttle samples during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def cpu_baseline(tensors, wl, seconds: float = 12.0):
    """Times the fp64 oracle (forward + backward) on host cores over a bounded
    sample of the workload's (batch, window, head) units in every block of the
    step (all of them when they fit in the time budget).  `tensors`: one dict of
    inputs per stage of the workload (a single dict for a one-stage workload)."""
    import numpy as np

    import oracle
    stages = stages_of(wl)
    if isinstance(tensors, dict):
        tensors = [tensors]
    cores = oracle.default_threads()
    nblocks = sum(len(st["shifts"]) for st in stages)
    flops, total_dt, parts, done, full_s = 0.0, 0.0, [], 0, 0.0
    for st, t in zip(stages, tensors):
        B, H, W, heads, M = st["B"], st["H"], st["W"], st["heads"], st["M"]
        nW = -(-H // M) * -(-W // M)  # windows of the grid padded to multiples of M
        n_units = B * nW * heads
        for s in st["shifts"]:
            # units spread over the batch, including windows of the last row/column
            t0 = time.perf_counter()
            probe = np.arange(0, min(n_units, 4 * cores))
            bias = (t["u"], t["w"]) if st.get("lrbias") else None
            oracle.units(t["q"], t["k"], t["v"], t["theta"], M, s, probe, dout=t["dout"], nthreads=cores, bias=bias)
            dt = max(time.perf_counter() - t0, 1e-6)
            budget = seconds / nblocks
            n = int(min(n_units, max(len(probe), len(probe) * budget / dt)))
            ids = np.linspace(0, n_units - 1, n).astype(np.int64)
            t0 = time.perf_counter()
            oracle.units(t["q"], t["k"], t["v"], t["theta"], M, s, ids, dout=t["dout"], nthreads=cores, bias=bias)
            dt = time.perf_counter() - t0
            # useful flops of the sampled units (pairs that attend)
            flops += sum(pair_flops(st)) * unmasked_pairs(B, H, W, heads, M, s) * (n / n_units)
            total_dt += dt
            done += n
            full_s += dt * n_units / n
            where = f"{H}x{W}/M={M} " if len(stages) > 1 else ""
            parts.append(f"{n} of {n_units} at {where}s={s}")
    return {"value": flops / total_dt / 1e12, "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"(batch, window, head) units: {', '.join(parts)}; fwd+bwd, fp64, {total_dt:.1f} s",
            "units_per_s": done / total_dt,
            "full_step_s_extrapolated": full_s,  # equal to the measured time when every unit was sampled
            "seconds": total_dt}


def cpu_stage_inputs(wl) -> list:
    """Seeded CPU inputs of every stage of a workload (with the bias factors when it has them)."""
    from vision_transformer_windowed_b200.inputs import make_bias, make_inputs
    out = []
    for st in stages_of(wl):
        t = make_inputs(st["B"], st["H"], st["W"], st["heads"], st["d"], device="cpu", qk_scale=st["qk_scale"])
        if st.get("lrbias"):
            t.update(make_bias(st["heads"], st["M"], LRBIAS_RANK))
        out.append(t)
    return out


def config_entry(wl, r, peaks, world, name=None) -> dict:
    """Per-workload figures: fwd+bwd and forward-alone throughput, the no-recompute count of
    the backward (8 d per pair instead of 10 d), % of the measured and of the spec bf16 peak,
    the forward's algorithmic HBM rate, peak memory and the backward workspace."""
    blocks = blocks_of(wl)
    fwd_ms = r["phase_ms"]["fwd"] * len(blocks)  # per step
    infer = wl.get("infer", False)
    e = {"tflops": r["tflops"], "ms_per_step": r["ms"],
         "pct_bf16_peak": 100 * r["tflops"] / peaks["bf16_tflops"] / world,
         "pct_bf16_spec": 100 * r["tflops"] / SPEC_BF16_TFLOPS / world,
         "fwd_tflops": r["fwd_flops"] * world / (fwd_ms * 1e-3) / 1e12,
         "tokens_per_s": r["tokens_per_s"], "peak_gb": r["peak_gb"], "phase_ms": r["phase_ms"]}
    e["fwd_pct_bf16_peak"] = 100 * e["fwd_tflops"] / peaks["bf16_tflops"] / world
    # the forward phase's algorithmic bytes (phase_work) over its time
    e["fwd_gbs"] = sum(phase_work(st, s)["bytes"]["fwd"] for st, s in blocks) / (fwd_ms * 1e-3) / 1e9
    if infer:
        e["step"] = "inference forward (no LSE) at every shift"
    else:
        e["tflops_no_recompute"] = (r["fwd_flops"] + 0.8 * r["bwd_flops"]) * world / (r["ms"] * 1e-3) / 1e12
        e["bwd_workspace_gb"] = r["ws_bytes"] / 1e9
    if "phase_ms_per_step" in r:
        e["roofline"] = roofline(wl, r, peaks)
        if name is not None:
            e["roofline"]["traffic"] = measured_traffic(e["roofline"]["kernel"], name)
    return e


def run_block(wl, dev, rank, steps, warmup, peaks):
    """The fused attention block (one kernel) and, for comparison, the same block unfused:
    cuBLAS projections around this library's inference attention forward."""
    import torch

    from vision_transformer_windowed_b200 import dp, ops
    from vision_transformer_windowed_b200.inputs import make_block_inputs
    B, H, W, heads, M = wl["B"], wl["H"], wl["W"], wl["heads"], wl["M"]
    C = heads * HEAD_DIM
    t = make_block_inputs(B, H, W, heads, HEAD_DIM, device=dev)
    x, wqkv, bqkv, wo, bo, th = t["x"], t["w_qkv"], t["b_qkv"], t["w_o"], t["b_o"], t["theta"]
    y = torch.empty_like(x)
    bqkv16, bo16 = bqkv.to(torch.bfloat16), bo.to(torch.bfloat16)

    def fused():
        for s in wl["shifts"]:
            ops.winattn_block_fwd(x, wqkv, bqkv, wo, bo, th, M, s, heads, y=y)

    def unfused():
        for s in wl["shifts"]:
            qkv = torch.nn.functional.linear(x, wqkv, bqkv16).view(B, H, W, 3, heads, HEAD_DIM)
            q, k, v = (qkv[..., i, :, :].contiguous() for i in range(3))
            o, _ = ops.winattn_fwd(q, k, v, th, M, s, need_lse=False)
            y.copy_(torch.nn.functional.linear(o.view(B, H, W, C), wo, bo16))

    def timed(fn):
        for _ in range(warmup):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return dp.max_over_ranks(a.elapsed_time(b) / steps, dev)

    ms = timed(fused)
    ms_unfused = timed(unfused)
    import torch.distributed as dist
    world = dist.get_world_size() if dist.is_initialized() else 1
    fl = block_flops(wl)
    tokens = B * H * W * len(wl["shifts"])
    gbs = tokens * 2 * C * 2 / (ms * 1e-3) / 1e9  # x read and y written once per token
    return {"tflops": fl * world / (ms * 1e-3) / 1e12, "ms_per_step": ms,
            "pct_bf16_peak": 100 * fl / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "tokens_per_s": tokens * world / (ms * 1e-3),
            "hbm_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"],
            "unfused_ms_per_step": ms_unfused,
            "step": "attention block with qkv and output projections, inference, at every shift",
            "unfused": "cuBLAS bf16 projections around the inference attention forward"}


def workload_config(name, wl, world) -> dict:
    """The `config` object of the JSON line: the workload's name and shapes."""
    def shape(st):
        return {"B_per_gpu": st["B"], "H": st["H"], "W": st["W"], "heads": st["heads"], "M": st["M"],
                "shifts": list(st["shifts"])}
    cfg = {"workload": name, "d": stages_of(wl)[0]["d"]}
    if "stages" in wl:
        cfg["stages"] = [shape(st) for st in stages_of(wl)]
    else:
        cfg.update(shape(wl))
    cfg.update({"qk_scale": wl.get("qk_scale", 1.0), "step": "fwd+bwd of every block",
                "parallelism": f"dp{world}"})
    return cfg


def run_reference(args):
    """The fp64 CPU oracle as the reference arm (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import torch

    wl = WORKLOADS[args.workload]
    t = cpu_stage_inputs(wl)
    per_step = max(1.0, args.reference_seconds / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline(t, wl, seconds=per_step)
    vals, secs, last = [], 0.0, None
    for _ in range(args.steps):
        last = cpu_baseline(t, wl, seconds=per_step)
        vals.append(last["value"])
        secs += last["seconds"]
    value = statistics.mean(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, wl, 1),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": last["cores"], "kind": "oracle",
                         "sample": last["sample"] + " per step"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    del torch


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="fswin", choices=["fswin", "reference"])
    ap.add_argument("--workload", default=HEADLINE, choices=sorted(n for n in WORKLOADS if not WORKLOADS[n].get("infer")))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the per-config numbers of the other workloads")
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling runs only)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    if args.batch > 0:
        wl0 = WORKLOADS[args.workload]
        if "stages" in wl0:
            WORKLOADS[args.workload] = dict(wl0, stages=[dict(st, B=args.batch) for st in wl0["stages"]])
        else:
            WORKLOADS[args.workload] = dict(wl0, B=args.batch)
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist

    from vision_transformer_windowed_b200 import _lib, dp, ops
    from vision_transformer_windowed_b200.inputs import make_bias

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    _lib.load()
    peaks = load_peaks()

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    def run_workload(name, steps, warmup, phase=True, clocks=False):
        wl = WORKLOADS[name]
        infer = wl.get("infer", False)
        lrb = wl.get("lrbias", False)
        # per stage: inputs, a backward workspace, and the outputs of each of its blocks
        data = []
        for st in stages_of(wl):
            B, H, W, heads, M = st["B"], st["H"], st["W"], st["heads"], st["M"]
            t = dp.rank_inputs(B, H, W, heads, st["d"], rank, dev, qk_scale=st["qk_scale"])
            if lrb:
                t.update(make_bias(heads, M, LRBIAS_RANK, device=dev))
            blocks = []
            for s in st["shifts"]:
                o = torch.empty_like(t["q"])
                lse = None if infer else torch.empty((B, H, W, heads), device=dev, dtype=torch.float32)
                g = None if infer else (torch.empty_like(t["q"]), torch.empty_like(t["q"]), torch.empty_like(t["q"]),
                                        torch.empty_like(t["theta"]))
                if lrb:
                    g = g + (torch.empty_like(t["u"]), torch.empty_like(t["w"]))
                blocks.append((s, o, lse, g))
            if infer:
                ws = torch.empty(0, dtype=torch.uint8)
            elif lrb:
                ws = ops.alloc_lrbias_workspace(t["q"], M, st["shifts"][0])
            else:
                ws = ops.alloc_workspace(t["q"], M, st["shifts"][0])
            data.append((st, t, blocks, ws))

        def step(evs=None):
            i = 0
            for st, t, blocks, ws in data:
                M = st["M"]
                q, k, v, th, do = t["q"], t["k"], t["v"], t["theta"], t["dout"]
                for s, o, lse, g in blocks:
                    if evs is not None:
                        _lib.fs_set_phase_events([e.cuda_event for e in evs[i][0]])
                    if infer:  # forward only, O only
                        ops.winattn_fwd(q, k, v, th, M, s, o=o, need_lse=False)
                    elif lrb:  # the low-rank bias variant: theta, U and W are shared by the batch
                        ops.winattn_lrbias_fwd(q, k, v, th, t["u"], t["w"], M, s, o=o, lse=lse)
                        if evs is not None:
                            _lib.fs_set_phase_events([e.cuda_event for e in evs[i][1]])
                        dq, dk, dv, dth, du, dw = g
                        ops.winattn_lrbias_bwd(q, k, v, o, do, lse, th, t["u"], t["w"], M, s, workspace=ws, dq=dq,
                                               dk=dk, dv=dv, dtheta=dth, du=du, dw=dw)
                        dp.allreduce_param_grads(dth, du, dw)
                    else:  # the training pair: the forward leaves the rotated q', k' tiles in ws
                        ops.winattn_fwd(q, k, v, th, M, s, o=o, lse=lse, workspace=ws)
                        if evs is not None:
                            _lib.fs_set_phase_events([e.cuda_event for e in evs[i][1]])
                        dq, dk, dv, dth = g
                        ops.winattn_bwd(q, k, v, o, do, lse, th, M, s, workspace=ws, dq=dq, dk=dk, dv=dv, dtheta=dth,
                                        after_train_fwd=True)
                        dp.allreduce_dtheta(dth)  # theta is shared by the whole data-parallel batch
                    i += 1
            if evs is not None:
                _lib.fs_set_phase_events([])

        nblocks = len(blocks_of(wl))
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        evsets = None
        if phase:
            evsets = [[([torch.cuda.Event(enable_timing=True) for _ in range(2)],
                        [torch.cuda.Event(enable_timing=True) for _ in range(5)]) for _ in range(nblocks)]
                      for _ in range(steps)]
            for stp in evsets:  # torch creates the CUDA event on first record
                for fe, be in stp:
                    for e in fe + be:
                        e.record()
            torch.cuda.synchronize()
        sampler = ClockSampler(local) if clocks else None
        barrier()
        torch.cuda.synchronize()
        if sampler:
            sampler.start()
            time.sleep(0.4)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for i in range(steps):
            step(evsets[i] if evsets else None)
        e1.record()
        torch.cuda.synchronize()
        barrier()
        clk = sampler.stop() if sampler else None
        ms = dp.max_over_ranks(e0.elapsed_time(e1) / steps, dev)
        assert _lib.fs_device_status() == 0, "a kernel reported a device-side failure"
        peak_gb = torch.cuda.max_memory_allocated(dev) / 1e9
        fwd_f, bwd_f = workload_flops(wl)
        if infer:
            bwd_f = 0.0
        tokens = workload_tokens(wl)
        res = {"ms": ms, "tflops": (fwd_f + bwd_f) * world / (ms * 1e-3) / 1e12,
               "tokens_per_s": tokens * world / (ms * 1e-3), "peak_gb": peak_gb,
               "fwd_flops": fwd_f, "bwd_flops": bwd_f, "clocks": clk,
               "ws_bytes": sum(x[3].numel() for x in data)}
        if evsets:
            tot = {n: 0.0 for n in PHASES}
            for stp in evsets:
                for fe, be in stp:
                    tot["fwd"] += fe[0].elapsed_time(fe[1])
                    if infer:
                        continue
                    for j in range(4):
                        tot[PHASES[1 + j]] += be[j].elapsed_time(be[j + 1])
            names = ["fwd"] if infer else PHASES
            tot = {n: tot[n] for n in names}
            launches = steps * nblocks
            res["phase_ms"] = {n: tot[n] / launches for n in names}  # average per launch
            res["phase_ms_per_step"] = {n: tot[n] / steps for n in names}
            res["phase_share"] = {n: tot[n] / max(sum(tot.values()), 1e-9) for n in names}
            res["launches_per_kernel"] = launches
        res["data"] = data
        return res

    main_res = run_workload(args.workload, args.steps, args.warmup, phase=True, clocks=True)
    wl = WORKLOADS[args.workload]
    blocks = blocks_of(wl)
    sm_mhz = main_res["clocks"]["sm_mhz"] if main_res["clocks"] else None
    roof = roofline(wl, main_res, peaks, sm_mhz)
    roof["traffic"] = measured_traffic(roof["kernel"], args.workload)  # bytes per step, like "achieved"

    # End to end through the public API with host buffers (pinned), copies inside the timed
    # region.  e2e: every block's inputs (q, k, v, dO, theta) come from pinned host memory on a
    # copy stream, a stage's compute waits only for its own inputs (so the next stage's upload
    # overlaps the current stage's kernels), and each block's d theta (the parameter gradient, the
    # step's result for an optimizer) is read back; O, dQ, dK, dV stay on the device, as they do
    # inside a model.  e2e_all_outputs: the same with O, dQ, dK, dV and d theta all read back and
    # every copy on the compute stream.
    lrb = wl.get("lrbias", False)
    in_keys = ("q", "k", "v", "dout", "theta") + (("u", "w") if lrb else ())
    host = [{k: t[k].cpu().pin_memory() for k in in_keys} for _, t, _, _ in main_res["data"]]
    res_host = {}
    e2e_steps = max(1, min(args.steps, 5))
    torch.cuda.synchronize()
    h2d = sum(x.numel() * x.element_size() for hs in host for x in hs.values())
    copy_stream = torch.cuda.Stream(device=dev)
    d2h = {"result": 0, "all": 0}

    def e2e_step(read_all: bool):
        main = torch.cuda.current_stream(dev)
        nbytes = 0
        staged = []
        if read_all:
            staged = [({k: x.to(dev, non_blocking=True) for k, x in hs.items()}, None) for hs in host]
        else:
            with torch.cuda.stream(copy_stream):
                for hs in host:
                    dvi = {k: x.to(dev, non_blocking=True) for k, x in hs.items()}
                    ev = torch.cuda.Event()
                    ev.record(copy_stream)
                    staged.append((dvi, ev))
        for si, (st, (dvi, ev)) in enumerate(zip(stages_of(wl), staged)):
            if ev is not None:
                main.wait_event(ev)
                for x in dvi.values():
                    x.record_stream(main)  # allocated on the copy stream, used on this one
            M = st["M"]
            for bi, s in enumerate(st["shifts"]):
                if lrb:
                    o, lse = ops.winattn_lrbias_fwd(dvi["q"], dvi["k"], dvi["v"], dvi["theta"], dvi["u"], dvi["w"], M, s)
                    dq, dk, dvv, dth, du, dw = ops.winattn_lrbias_bwd(dvi["q"], dvi["k"], dvi["v"], o, dvi["dout"], lse,
                                                                      dvi["theta"], dvi["u"], dvi["w"], M, s)
                    dp.allreduce_param_grads(dth, du, dw)
                    params = (("dtheta", dth), ("du", du), ("dw", dw))
                else:  # the training pair (ops.window_attention(..., reuse_rotated=True) calls it so)
                    ws = ops.alloc_workspace(dvi["q"], M, s)
                    o, lse = ops.winattn_fwd(dvi["q"], dvi["k"], dvi["v"], dvi["theta"], M, s, workspace=ws)
                    dq, dk, dvv, dth = ops.winattn_bwd(dvi["q"], dvi["k"], dvi["v"], o, dvi["dout"], lse, dvi["theta"],
                                                       M, s, workspace=ws, after_train_fwd=True)
                    dp.allreduce_dtheta(dth)
                    params = (("dtheta", dth),)
                outs = (("o", o), ("dq", dq), ("dk", dk), ("dv", dvv)) + params if read_all else params
                for name, x in outs:
                    key = (si, bi, name)
                    if key not in res_host:
                        res_host[key] = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
                    res_host[key].copy_(x, non_blocking=True)
                    nbytes += x.numel() * x.element_size()
        d2h["all" if read_all else "result"] = nbytes

    def e2e_time(read_all: bool) -> float:
        e2e_step(read_all)
        torch.cuda.synchronize()
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(e2e_steps):
            e2e_step(read_all)
        b.record()
        torch.cuda.synchronize()
        return dp.max_over_ranks(a.elapsed_time(b) / e2e_steps, dev)

    fl = main_res["fwd_flops"] + main_res["bwd_flops"]
    e2e_ms = e2e_time(False)
    e2e = {"value": fl * world / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_ms,
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h["result"],
           "step": "inputs from pinned host memory (uploads overlapped with the previous stage's kernels), "
                   "the parameter gradients (d theta; dU, dW with the bias) of every block read back"}
    e2e_all_ms = e2e_time(True)
    e2e_all = {"value": fl * world / (e2e_all_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "ms_per_step": e2e_all_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h["all"],
               "step": "inputs from pinned host memory; O, dQ, dK, dV and d theta of every block read back; one stream"}

    per_config = {args.workload: config_entry(wl, main_res, peaks, world, args.workload)}
    del main_res["data"], host, res_host
    if not args.no_extra:
        for name in WORKLOADS:
            if name == args.workload:
                continue
            torch.cuda.empty_cache()
            r = run_workload(name, max(3, args.steps // 2), 3, phase=True, clocks=False)
            del r["data"]
            per_config[name] = config_entry(WORKLOADS[name], r, peaks, world, name)

    if not args.no_extra:
        for name, wl_b in BLOCK_WORKLOADS.items():
            torch.cuda.empty_cache()
            per_config[name] = run_block(wl_b, dev, rank, max(3, args.steps // 2), 3, peaks)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(cpu_stage_inputs(wl), wl)
        cpu.pop("seconds", None)

    if rank == 0:
        def launches(st):  # kernels of one block: the forward's, then the backward's
            if st.get("lrbias"):
                return 1 + 6  # prep, main, post, d theta sum, two dU / dW sum levels
            if st["d"] == 64:
                return 1 + 4  # prep, main, post, d theta sum
            if st["M"] * st["M"] < 128:
                return 1 + 2  # the one-tile backward, d theta sum
            return 2 + 5  # q', k' images and the forward; prep, scale, main, post, d theta sum
        nlaunch = sum(launches(st) for st, _ in blocks)
        line = {
            "metric": METRIC, "value": main_res["tflops"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": main_res["ms"], "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(workload_config(args.workload, wl, world),
                           l2="inputs larger than L2 (the largest stage's tensors > 126 MB each)"),
            "pct_bf16_peak": 100 * main_res["tflops"] / peaks["bf16_tflops"] / world,
            "tokens_per_s": main_res["tokens_per_s"], "peak_gb": main_res["peak_gb"],
            # per block: the forward (windows of >= 128 tokens: the rotated q', k' images,
            # then the forward), then the backward's kernels
            "gpu_launches": args.steps * nlaunch,
            "roofline": roof, "clocks": main_res["clocks"], "e2e": e2e, "e2e_all_outputs": e2e_all, "cpu_baseline": cpu,
            "per_config": per_config, "peaks": peaks,
        }
        a, b = per_config.get("highres_p2_m32"), per_config.get("highres_p2_m64")
        if a and b:  # memory flat in M: the same tokens at windows 32 and 64
            line["flat_in_m"] = {"workloads": ["highres_p2_m32", "highres_p2_m64"],
                                 "peak_gb": [a["peak_gb"], b["peak_gb"]],
                                 "peak_diff_mb": abs(a["peak_gb"] - b["peak_gb"]) * 1e3,
                                 "bwd_workspace_gb": [a["bwd_workspace_gb"], b["bwd_workspace_gb"]]}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
