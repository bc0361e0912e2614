#!/usr/bin/env python
"""Benchmark of the hybrid linear/softmax token mixer on B200.

One step = one forward pass of the 720p-shaped 24-layer hybrid stack (18 gated
linear-attention layers, 6 gated softmax anchors at layers 4, 8, ..., 24, three
AttnRes blocks of 8 with the shared-query router) over one batch of synthetic
video tokens: B = 1, N = 19,320 (21 latent frames x 23 x 40 patches), H = 24,
d = 128, D = 3072, bf16 operands with fp32 accumulation and an fp32 residual
stream. Inputs are seeded synthetic tensors (x ~ N(0, 1), weights ~ N(0, 1/D)).

Prints one JSON line: whole-job tokens/s over all GPUs (each GPU runs its own
replica of the stack: the path has no exchange step), device-timed with CUDA
events, max over ranks; an end-to-end figure through the C ABI with the input
copied from pinned host memory and the output read back every step; the
roofline of the dominant kernel from per-launch CUDA events taken in the timed
region; the speed-up over an all-softmax stack of the same shape; clocks
sampled during the timed region; and the fp64 CPU oracle timed on a bounded
sample of the same workload on this host's cores.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "hybrid attn stack tokens/s at N=19,320 (720p shape); HBM GB/s & TC util"
WORKLOAD = dict(name="720p-shaped 24-layer hybrid stack (18 gated linear + 6 gated softmax "
                "anchors, 3 AttnRes blocks of 8, shared-query router)",
                B=1, N=19320, H=24, d=128, L=24, softmax_period=4, attnres_block=8)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
KINDS = ("proj_qkvg", "proj_out", "linear_state", "linear_readout", "anchor", "route", "keys",
         "other", "linear_reduce")


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


def profiled_traffic(kind: str):
    """DRAM bytes per launch of a kernel class from the committed ncu capture
    (profiles/traffic.json), or None when the kernel's source has changed since
    (its hash no longer matches) or no capture exists."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None, None
    with open(path) as f:
        entry = json.load(f).get(kind)
    if entry is None:
        return None, None
    csrc = os.path.join(ROOT, "softmax_attention_video_gated_b200", "csrc")
    h = hashlib.sha256()
    for name in (entry["source"], "common.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    if h.hexdigest()[:16] != entry["source_hash"]:
        return None, None
    return entry["bytes_per_launch"], entry["profile"]


def algorithmic_work(kind: str, wl: dict, n_blocks_routed: int = 1):
    """Algorithmic FLOPs or bytes of one launch of a kernel class.

    GEMMs: 2*M*K*N flops. Linear state pass: K and V read once (2*B*N*D*2 B).
    Linear read-out: Q and G read, Y written (3*B*N*D*2 B). Anchor: 4*B*N^2*D
    flops (S = Q K^T and O = P V). Router: h (fp32) read once, n_b keys and n_b
    summaries read, u written: (4 + 4*n_b + 2)*B*N*D bytes."""
    B, N, D = wl["B"], wl["N"], wl["H"] * wl["d"]
    M = B * N
    if kind == "proj_qkvg":
        # write-gated stacks: the linear layers' projections also produce H logits
        lin = 1.0 - 1.0 / wl["softmax_period"] if wl.get("write_gate") else 0.0
        return "tensor", 2.0 * M * D * (4 * D + lin * wl["H"])
    if kind in ("proj_out", "keys"):
        return "tensor", 2.0 * M * D * D
    if kind == "linear_state":
        # (+ the write-gate logits, one bf16 per token and head, when gated)
        return "hbm", 2.0 * M * D * 2 + (2.0 * M * wl["H"] if wl.get("write_gate") else 0.0)
    if kind == "linear_readout":
        return "hbm", 3.0 * M * D * 2
    if kind == "anchor":
        return "tensor", 4.0 * B * N * N * D
    if kind == "route":
        return "hbm", (4.0 + 4.0 * n_blocks_routed + 2.0) * M * D
    return None, 0.0


class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="sva_clocks_", suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
               "-lms", "200"]
        if self.gpu_id is not None:
            cmd += ["-i", str(self.gpu_id)]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, smax, power, reasons = [], [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax.append(float(parts[2]))
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "power_w_max": max(power) if power else None,
                "samples": len(sm), "reasons": sorted(reasons)}


def gpu_uuid(torch, dev):
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return None


def max_over_ranks(v: float, dist=None, device="cpu") -> float:
    """The maximum of a per-rank value over all ranks (a no-op on one rank)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, tokens_per_rank: int, ms_per_step: float) -> float:
    """Tokens per second of the whole job: every rank runs its own replica of the
    stack on its own tokens, and the slowest rank sets the step time."""
    return world * tokens_per_rank / (ms_per_step * 1e-3)


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# the fp64 oracle on a bounded sample (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample(wl: dict, frac: int):
    """Times the oracle's layer pieces at N_s = N / frac tokens (full D) and
    extrapolates to one pass of the full stack: projections, router and linear
    layers scale with N, the softmax core with N^2. Returns
    (tokens_per_s, stack_seconds_extrapolated, sample_seconds, description)."""
    import numpy as np

    import oracle as O
    import workloads as W

    B, N, H, d = wl["B"], wl["N"], wl["H"], wl["d"]
    D = H * d
    Ns = max(1, N // frac)
    seed = 1236
    x = W.normal((B, Ns, D), 1.0, seed, W.TAG_X, "bf16")
    std = 1.0 / math.sqrt(D)
    wq = W.normal((4 * D, D), std, seed, W.TAG_WQKVG + 1, "bf16")
    wo = W.normal((D, D), std, seed, W.TAG_WO + 1, "bf16")
    wr = W.normal((D, D), std, seed, W.TAG_WR, "bf16")
    s1 = W.normal((B, Ns, D), 1.0, seed, 901, "bf16")
    s2 = W.normal((B, Ns, D), 1.0, seed, 902, "bf16")
    t = {}
    t0 = time.perf_counter()
    qkvg = O.project(x, wq)
    t["proj_qkvg"] = time.perf_counter() - t0
    q, k, v, g = (qkvg[..., i * D:(i + 1) * D] for i in range(4))
    wgl = None
    if wl.get("write_gate"):
        wwg = W.normal((H, D), std, seed, W.TAG_WWG + 1, "bf16")
        t0 = time.perf_counter()
        wgl = O.project(x, wwg)
        t["proj_wgate"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    y = O.linear_attn(q, k, v, g, H, wgate=wgl)
    t["linear"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.softmax_anchor(q, k, v, g, H)
    t["anchor"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.project(y, wo)
    t["proj_out"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.route(x, [s1], wr)
    t["route1"] = time.perf_counter() - t0
    t0 = time.perf_counter()
    O.route(x, [s1, s2], wr)
    t["route2"] = time.perf_counter() - t0
    sample = sum(t.values())
    r = N / Ns
    L = wl["L"]
    n_anchor = L // wl["softmax_period"]
    n_lin = L - n_anchor
    # routed linear layers: 6 in block 2 (one summary), 6 in block 3 (two)
    stack_s = (L * (t["proj_qkvg"] + t["proj_out"]) * r + n_lin * t["linear"] * r
               + n_anchor * t["anchor"] * r * r + 6 * t["route1"] * r + 6 * t["route2"] * r
               + n_lin * t.get("proj_wgate", 0.0) * r)
    desc = (f"fp64 oracle pieces at N_s = N/{frac} = {Ns} tokens, full D = {D}: one QKVG and one "
            f"output projection, one gated linear core, one gated softmax core, one 1-block and "
            f"one 2-block router; extrapolated to the 24-layer stack (x N/N_s, softmax core "
            f"x (N/N_s)^2)")
    return B * N / stack_s, stack_s, sample, desc


# The oracle's sample: N / ORACLE_SAMPLE_FRAC tokens at full width, for both the
# CPU baseline of our arm and every step of the reference arm, so the two report
# one number.
ORACLE_SAMPLE_FRAC = 4


def run_reference(args, wl):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    frac = ORACLE_SAMPLE_FRAC
    for _ in range(args.warmup):
        oracle_sample(wl, frac)
    vals, secs = [], []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, stack_s, sample_s, desc = oracle_sample(wl, frac)
        vals.append(v)
        secs.append(sample_s)
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * wall / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(wl, n_gpus):
    D = wl["H"] * wl["d"]
    return {"workload": wl["name"], "B": wl["B"], "N": wl["N"], "H": wl["H"], "d_head": wl["d"],
            "D": D, "layers": wl["L"], "global_batch": wl["B"] * n_gpus, "seq_len": wl["N"],
            "parallelism": f"replicas{n_gpus}",
            "l2": "inputs larger than L2: every step streams 2.26 GB of weights and "
                  ">1 GB of activations through a 126 MB L2"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def make_stack(torch, sva, W, wl, all_softmax=False, weights=None):
    B, N, H, d, L = wl["B"], wl["N"], wl["H"], wl["d"], wl["L"]
    D = H * d
    seed = 1236
    if weights is None:
        std = 1.0 / math.sqrt(D)
        wq = [W.normal_torch((4 * D, D), std, seed, W.TAG_WQKVG + l, "bf16") for l in range(1, L + 1)]
        wo = [W.normal_torch((D, D), std, seed, W.TAG_WO + l, "bf16") for l in range(1, L + 1)]
        wr = W.normal_torch((D, D), std, seed, W.TAG_WR, "bf16")
        weights = (wq, wo, wr)
    wq, wo, wr = weights[:3]
    wwg = None
    if wl.get("write_gate") and not all_softmax:
        # write-gated linear layers: logits u W_wg^T, W_wg[l] [H, D]
        if len(weights) < 4:
            std = 1.0 / math.sqrt(D)
            weights = weights + ([None if l % wl["softmax_period"] == 0 else
                                  W.normal_torch((H, D), std, seed, W.TAG_WWG + l, "bf16")
                                  for l in range(1, L + 1)],)
        wwg = weights[3]
    st = sva.Stack(wq, wo, wr, B, N, H, softmax_period=wl["softmax_period"],
                   attnres_block=wl["attnres_block"], all_softmax=all_softmax, w_wg=wwg)
    return st, weights


def timed_steps(torch, sva, stack, x, y, ws, steps, profile=True):
    """Runs `steps` stack passes between CUDA events; with profile=True every
    launch is bracketed by its own pair of events (the per-kernel breakdown),
    with profile=False nothing but the two bracketing events is recorded (the
    headline). Returns (ms_total, per-launch records [(kind, ms)], launches)."""
    stream = torch.cuda.current_stream()
    ev_sets = []
    if profile:
        # every event recorded once before use, so the timed pass pays no first-record cost
        cap = 256
        for _ in range(steps):
            evs = [torch.cuda.Event(enable_timing=True) for _ in range(2 * cap)]
            for e in evs:
                e.record(stream)
            ev_sets.append(evs)
        torch.cuda.synchronize()
    else:
        stack.count_launches()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    counts, kinds, kernels = [], [], 0
    start.record(stream)
    for k in range(steps):
        if profile:
            stack.set_profile(ev_sets[k], len(ev_sets[k]) // 2)
        sva.sva_hybrid_stack_fwd(stack, x, y, ws)
        if profile:
            counts.append(stack.prof_count.value)
            kinds.append(list(stack.prof_kind))
        kernels += stack.launch_count.value  # a profiled span may hold 2 kernels
    end.record(stream)
    torch.cuda.synchronize()
    stack.clear_profile()
    recs = []
    for k in range(len(counts)):
        n = min(counts[k], len(ev_sets[k]) // 2)
        for i in range(n):
            recs.append((KINDS[kinds[k][i]], ev_sets[k][2 * i].elapsed_time(ev_sets[k][2 * i + 1])))
    return start.elapsed_time(end), recs, kernels


def summarize(recs, steps, wl, peaks):
    by = {}
    for kind, ms in recs:
        by.setdefault(kind, []).append(ms)
    out = {}
    for kind, v in by.items():
        bound, work = algorithmic_work(kind, wl, 1)
        avg = sum(v) / len(v)
        e = {"launches_per_step": len(v) / steps, "ms_per_step": sum(v) / steps, "avg_launch_ms": avg}
        if bound == "tensor":
            e["achieved"] = work / (avg * 1e-3) / 1e12
            e["unit"] = "TFLOP/s"
            e["frac"] = e["achieved"] / peaks["bf16_tflops_sustained"]
        elif bound == "hbm":
            if kind == "route":
                # routed layers mix 1, 2, ... completed blocks: total bytes over total time
                work = sum(algorithmic_work("route", wl, nb)[1] for nb in routed_blocks(wl))
                work /= max(1, len(routed_blocks(wl)))
            e["achieved"] = work / (avg * 1e-3) / 1e9
            e["unit"] = "GB/s"
            e["frac"] = e["achieved"] / peaks["hbm_gbs"]
        out[kind] = e
    return out


def routed_blocks(wl):
    """Completed blocks each routed linear layer mixes, in layer order."""
    out = []
    blk, per = wl["attnres_block"], wl["softmax_period"]
    for l in range(1, wl["L"] + 1):
        c = (l + blk - 1) // blk if blk > 0 else 1
        if blk > 0 and c >= 2 and not (per > 0 and l % per == 0):
            out.append(c - 1)
    return out


def run_case(args):
    """One kernel class on its own (for sweeps and profiler captures): prints a
    JSON line with the device time per launch and the achieved rate."""
    import torch

    import softmax_attention_video_gated_b200 as sva
    import workloads as W

    peaks = load_peaks()
    B, N, H, d = args.B, args.N, args.H, 128
    D = H * d
    seed = 77
    if args.case in ("anchor", "linear", "linear_wg"):
        q, k, v, g = (W.normal_torch((B, N, D), 1.0, seed, tag, "bf16")
                      for tag in (W.TAG_Q, W.TAG_K, W.TAG_V, W.TAG_G))
        out = torch.empty_like(q)
        if args.case == "anchor":
            ws = sva.workspace(sva._lib().sva_softmax_anchor_workspace_bytes(B, N, H, d, sva.SVA_BF16))
            fn = lambda: sva.sva_softmax_anchor_fwd(q, k, v, g, out, H, ws=ws)  # noqa: E731
            work, unit = 4.0 * B * N * N * D, "TFLOP/s"
        else:
            ws = sva.workspace(sva.sva_linear_attn_workspace_bytes(B, N, H, d, sva.SVA_BF16))
            wg = (W.normal_torch((B, N, H), 1.0, seed, W.TAG_WGATE, "bf16")
                  if args.case == "linear_wg" else None)
            fn = lambda: sva.sva_linear_attn_fwd(q, k, v, g, out, H, ws=ws, wgate=wg)  # noqa: E731
            work, unit = 10.0 * B * N * D + (2.0 * B * N * H if wg is not None else 0.0), "GB/s"
    elif args.case == "gemm":
        M, K, Nout = B * N, D, 4 * D
        x = W.normal_torch((M, K), 1.0, seed, W.TAG_X, "bf16")
        w = W.normal_torch((Nout, K), 1.0 / math.sqrt(K), seed, W.TAG_WQKVG, "bf16")
        y = torch.empty(M, Nout, device="cuda", dtype=torch.bfloat16)
        ws = sva.workspace(256)
        fn = lambda: sva.sva_projection_fwd(x, w, y, ws=ws)  # noqa: E731
        work, unit = 2.0 * M * K * Nout, "TFLOP/s"
    elif args.case == "route":
        # AttnRes router of a linear layer in block nb + 1: u = h + sum_b alpha_b s_b
        M, nb = B * N, args.nb
        hs = W.normal_torch((M, D), 1.0, seed, W.TAG_X, "f32")
        ks = [W.normal_torch((M, D), 1.0, seed, 901 + i, "bf16") for i in range(nb)]
        ss = [W.normal_torch((M, D), 1.0, seed, 911 + i, "bf16") for i in range(nb)]
        u = torch.empty(M, D, device="cuda", dtype=torch.bfloat16)
        ws = sva.workspace(256)
        fn = lambda: sva.sva_attnres_route(hs, ks, ss, u)  # noqa: E731
        work, unit = (4.0 + 4.0 * nb + 2.0) * M * D, "GB/s"
    else:  # proj_out: h += x W_o^T with the bf16 copy of h, as in the stack
        M, K, Nout = B * N, D, D
        x = W.normal_torch((M, K), 1.0, seed, W.TAG_X, "bf16")
        w = W.normal_torch((Nout, K), 1.0 / math.sqrt(K), seed, W.TAG_WO, "bf16")
        hs = W.normal_torch((M, Nout), 1.0, seed, W.TAG_V, "f32")
        hc = torch.empty(M, Nout, device="cuda", dtype=torch.bfloat16)
        ws = sva.workspace(256)
        fn = lambda: sva.sva_projection_residual_fwd(x, w, hs, hc, ws=ws)  # noqa: E731
        work, unit = 2.0 * M * K * Nout, "TFLOP/s"
    for _ in range(args.warmup):
        fn()
    torch.cuda.synchronize()
    st = sva.sva_check_device_status(ws)
    if st != sva.SVA_OK:
        raise RuntimeError(sva.status_string(st))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    rate = work / (ms * 1e-3) / (1e12 if unit == "TFLOP/s" else 1e9)
    peak = peaks["bf16_tflops"] if unit == "TFLOP/s" else peaks["hbm_gbs"]
    print(json.dumps({"case": args.case, "B": B, "N": N, "H": H, "ms_per_launch": ms,
                      "achieved": rate, "unit": unit, "frac_of_burst_peak": rate / peak}), flush=True)
    return 0


# 720p latent grid (23 x 40 patches) at 21 latent frames per 5 s of video; 60 s
# at 16 fps gives 241 latent frames
SWEEP_FRAMES = (21, 41, 81, 161, 241)


def run_sweep(args):
    """The hybrid's advantage over full softmax as the video gets longer: a
    4-layer hybrid group (3 gated linear + 1 gated softmax) against 4 gated
    softmax layers of the same width (D = 3072, H = 24), at 720p token counts
    for 5 s to 60 s of video. One JSON line per length."""
    import torch

    import softmax_attention_video_gated_b200 as sva
    import workloads as W

    H, d, L = 24, 128, 4
    D = H * d
    std = 1.0 / math.sqrt(D)
    wq = [W.normal_torch((4 * D, D), std, 99, W.TAG_WQKVG + l, "bf16") for l in range(1, L + 1)]
    wo = [W.normal_torch((D, D), std, 99, W.TAG_WO + l, "bf16") for l in range(1, L + 1)]
    for frames in SWEEP_FRAMES:
        N = frames * 23 * 40
        x = W.normal_torch((1, N, D), 1.0, 99, W.TAG_X, "bf16")
        y = torch.empty_like(x)
        res, clocks = {}, {}
        for name, all_sm in (("hybrid", False), ("all_softmax", True)):
            st = sva.Stack(wq, wo, None, 1, N, H, attnres_block=0, all_softmax=all_sm)
            ws = sva.workspace(st.workspace_bytes())
            for _ in range(3):
                sva.sva_hybrid_stack_fwd(st, x, y, ws=ws)
            torch.cuda.synchronize()
            sampler = ClockSampler(gpu_uuid(torch, torch.cuda.current_device()))
            sampler.start()
            time.sleep(0.3)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(args.steps):
                sva.sva_hybrid_stack_fwd(st, x, y, ws=ws)
            e1.record()
            torch.cuda.synchronize()
            clocks[name] = sampler.stop()
            if sva.sva_check_device_status(ws) != sva.SVA_OK:
                raise RuntimeError("device status")
            res[name] = e0.elapsed_time(e1) / args.steps
            del ws
        print(json.dumps({"sweep": "720p width, 4-layer group", "latent_frames": frames,
                          "video_seconds_at_16fps": round((4 * (frames - 1) + 1) / 16, 1),
                          "N": N, "hybrid_ms": res["hybrid"], "all_softmax_ms": res["all_softmax"],
                          "speedup": res["all_softmax"] / res["hybrid"],
                          "hybrid_tokens_per_s": N / (res["hybrid"] * 1e-3),
                          "clocks_hybrid": clocks["hybrid"],
                          "clocks_all_softmax": clocks["all_softmax"]}), flush=True)
        del x, y
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-all-softmax", action="store_true")
    ap.add_argument("--case", choices=("anchor", "linear", "linear_wg", "gemm", "proj_out", "route"),
                    help="time one kernel class alone instead of the stack")
    ap.add_argument("--sweep", action="store_true",
                    help="hybrid vs all-softmax 4-layer groups at 5 s .. 60 s of 720p video")
    ap.add_argument("--write-gate", action="store_true",
                    help="time the write-gated variant of the stack's linear layers")
    ap.add_argument("--B", type=int, default=1)
    ap.add_argument("--N", type=int, default=19320)
    ap.add_argument("--H", type=int, default=24)
    ap.add_argument("--nb", type=int, default=2, help="completed blocks the router mixes (--case route)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    wl = dict(WORKLOAD)
    if args.write_gate:
        wl["name"] += ", write-gated linear layers"
        wl["write_gate"] = True
    if args.case:
        return run_case(args)
    if args.sweep:
        return run_sweep(args)
    if args.impl == "reference":
        return run_reference(args, wl)

    import torch

    import softmax_attention_video_gated_b200 as sva
    import workloads as W

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device(f"cuda:{local}"))
    peaks = load_peaks()
    B, N, H, d = wl["B"], wl["N"], wl["H"], wl["d"]
    D = H * d
    x = W.normal_torch((B, N, D), 1.0, 1236 + rank, W.TAG_X, "bf16")
    y = torch.empty_like(x)
    stack, weights = make_stack(torch, sva, W, wl)
    ws = sva.workspace(stack.workspace_bytes())

    def barrier():
        if dist is not None:
            dist.barrier()

    for _ in range(args.warmup):
        sva.sva_hybrid_stack_fwd(stack, x, y, ws)
    st = sva.sva_check_device_status(ws)
    if st != sva.SVA_OK:
        raise RuntimeError(f"device status after warm-up: {sva.status_string(st)}")

    # ---- device-timed region
    sampler = ClockSampler(gpu_uuid(torch, local))
    barrier()
    torch.cuda.synchronize()
    sampler.start()
    time.sleep(0.3)
    ms_total, _, launches = timed_steps(torch, sva, stack, x, y, ws, args.steps, profile=False)
    # ---- per-kernel breakdown: a second pass of as many steps, started right
    # after the timed region (so it runs at the same clocks and power), with
    # every launch bracketed by its own events on the launching stream; the
    # dominant kernel's average launch time there is the roofline's denominator
    n_prof = args.steps
    ms_prof, recs, _ = timed_steps(torch, sva, stack, x, y, ws, n_prof, profile=True)
    clocks = sampler.stop()
    barrier()
    st = sva.sva_check_device_status(ws)
    if st != sva.SVA_OK:
        raise RuntimeError(f"device status after the timed region: {sva.status_string(st)}")
    ms_step = max_over_ranks(ms_total / args.steps, dist, "cuda")
    value = whole_job_rate(world, B * N, ms_step)

    kernels = summarize(recs, n_prof, wl, peaks)
    dom = max((k for k in kernels if k != "other"), key=lambda k: kernels[k]["ms_per_step"])
    bound, work = algorithmic_work(dom, wl, 1)
    de = kernels[dom]
    traffic, traffic_src = profiled_traffic(dom)
    if bound == "tensor":
        roof = {"kernel": dom, "bound": "tensor", "achieved": de["achieved"],
                "peak": peaks["bf16_tflops_sustained"], "unit": "TFLOP/s",
                "frac": de["achieved"] / peaks["bf16_tflops_sustained"],
                "peak_source": f"{peaks['source']} bf16_tflops_sustained (kernel timed inside a long step)",
                "traffic": traffic}
    else:
        roof = {"kernel": dom, "bound": "hbm", "achieved": de["achieved"], "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": de["achieved"] / peaks["hbm_gbs"],
                "peak_source": f"{peaks['source']} hbm_gbs", "traffic": traffic}
    roof["algorithmic_per_launch"] = work
    if traffic is not None:
        roof["traffic_unit"] = "bytes per launch (dram read + write)"
        roof["traffic_source"] = traffic_src

    # ---- end to end through the C ABI's host-batch call: every step copies its
    # input from pinned host memory and its result back, overlapped with the
    # neighbouring steps' passes
    xh = x.cpu().pin_memory()
    yh = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    staging = sva.workspace(sva.sva_hybrid_stack_host_staging_bytes(stack))
    sva.sva_hybrid_stack_fwd_host(stack, [xh, xh], yh, ws=ws, staging=staging)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    sva.sva_hybrid_stack_fwd_host(stack, [xh] * args.steps,
                                  [yh[i % 2] for i in range(args.steps)], ws=ws, staging=staging)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, "cuda")
    barrier()

    # ---- the all-softmax stack of the same shape (quadratic baseline)
    speedup = None
    if not args.no_all_softmax:
        st_all, _ = make_stack(torch, sva, W, wl, all_softmax=True, weights=weights)
        ws_all = sva.workspace(st_all.workspace_bytes())
        sva.sva_hybrid_stack_fwd(st_all, x, y, ws_all)
        # whole steps unprofiled, as the headline; the attention cores from a
        # profiled step of each stack
        ms_all, _, _ = timed_steps(torch, sva, st_all, x, y, ws_all, 2, profile=False)
        _, recs_all, _ = timed_steps(torch, sva, st_all, x, y, ws_all, 1, profile=True)
        del ws_all
        core_h = sum(ms for k, ms in recs
                     if k in ("linear_state", "linear_reduce", "linear_readout", "anchor")) / n_prof
        core_a = sum(ms for k, ms in recs_all if k == "anchor")
        speedup = {"all_softmax_ms_per_step": ms_all / 2,
                   "stack": (ms_all / 2) / (ms_total / args.steps),
                   "attention_cores": core_a / core_h if core_h > 0 else None}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded: x ~ N(0,1), weights ~ N(0,1/D))",
        "config": config_block(wl, world),
        "roofline": roof,
        "e2e": {"value": whole_job_rate(world, B * N, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": xh.numel() * xh.element_size(),
                "d2h_bytes_per_step": yh[0].numel() * yh[0].element_size(),
                "call": "sva_hybrid_stack_fwd_host (copies overlapped with the passes)"},
        "gpu_launches": launches,
        "clocks": clocks,
        "kernels": kernels,
        "kernels_pass": {"steps": n_prof, "ms_per_step": ms_prof / n_prof,
                         "note": "per-launch CUDA events, a second pass of as many steps right after "
                                 "the timed region; clocks: one record over both passes"},
        "speedup_vs_all_softmax": speedup,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # three samples (about 10 s of CPU work), median, as the reference arm
        # takes the median over its steps
        runs = [oracle_sample(wl, ORACLE_SAMPLE_FRAC) for _ in range(3)]
        vals = [r[0] for r in runs]
        v = statistics.median(vals)
        _, stack_s, sample_s, desc = runs[vals.index(v)]
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": blas_threads(),
                                "kind": "oracle", "sample": desc + "; median of 3 samples",
                                "sample_seconds": sum(r[2] for r in runs),
                                "stack_seconds_extrapolated": stack_s}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
