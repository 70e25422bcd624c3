#!/usr/bin/env python
"""Benchmark of the W4A4 NVFP4 linear hot path on B200.

One step = one pass of the whole hot path over one batch, on the 2048px
large-hidden DiT block (the largest configuration that fits one GPU): for
each of its two linears -- the fused QKV + SwiGLU-up projection 6144 -> 55296
and the output projection 24576 -> 6144, M = 16896 tokens (16384 image +
512 text), rank 32 -- the tensor amax, the fused smooth/quantise/pack +
low-rank down-projection, and the block-scaled FP4 GEMM with the low-rank
up-projection and the bf16 cast.  Inputs are synthetic and seeded (per-channel
lognormal(0, 1.5) activation magnitudes, N(0, 0.02) weights), drawn on the GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload block2048|qkv1024] [--table] [--case NAME] [--fp4-peak]

Prints one JSON line.  Under torchrun (N > 1) every rank runs an independent
replica on its own GPU (the path has no cross-GPU exchange); rank 0 prints.
``--impl reference`` times the plain CPU oracle on the host cores instead.
``--workload qkv1024`` runs the FLUX-1024px QKV projection instead (M = 4608,
3072 -> 9216); ``--table`` times every configuration's layers (with the
SwiGLU, rotary and quantising epilogues and FP8 attention); ``--case`` runs
one kernel's small workload for a profiler; ``--fp4-peak`` measures the FP4
tensor-core instruction rate.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "W4A4 linear TFLOPS (act-quant+FP4 GEMM+low-rank)"
MID_EVERY = 10       # steps between per-kernel timing events inside the timed region
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# name -> (description, M, [(layer, K, N)], activation recipe, bias, seed base, L2 sets)
WORKLOADS = {
    "block2048": {
        "workload": "2048px large-hidden DiT block: fused QKV+SwiGLU-up and output linears",
        "M": 16896, "linears": [("qkv_swiglu_up", 6144, 55296), ("out", 24576, 6144)], "r": 32,
        # the fused projection: 3 x 6144 plain QKV features, then 18432 SwiGLU gate/up pairs
        "swiglu": {"qkv_swiglu_up": 18432},
        "act": "lognormal", "activation": "N(0,1) x per-channel lognormal(0,1.5) magnitudes",
        "weight": "N(0,0.02)", "bias": False, "seed": 1004, "l2_sets": 1,
        "l2": "no rotation needed: X2 830 MB and Y1 1.87 GB per step exceed the 126 MB L2, so every kernel "
              "starts on operands another kernel has evicted"},
    "qkv1024": {
        "workload": "FLUX-1024px QKV projection",
        "M": 4608, "linears": [("qkv", 3072, 9216)], "r": 32, "swiglu": {},
        "act": "student_t", "activation": "N(0,1) with 1% Student-t(2)x50 channels",
        "weight": "N(0,0.02)", "bias": True, "seed": 1002, "l2_sets": 3,
        "l2": "3 rotating input/weight/output sets of ~140 MB each (> 126 MB L2)"},
}
DEFAULT_WORKLOAD = "block2048"


def workload_config(name):
    w = WORKLOADS[name]

    def lin(n, k, nn):
        d = {"layer": n, "K": k, "N": nn}
        if n in w["swiglu"]:
            d["epilogue"] = f"SwiGLU: {w['swiglu'][n]} plain outputs, {(nn - w['swiglu'][n]) // 2} silu(gate)*up outputs"
        return d
    return {"workload": w["workload"], "M": w["M"],
            "linears": [lin(n, k, nn) for n, k, nn in w["linears"]], "r": w["r"],
            "bias": w["bias"], "activation": w["activation"], "weight": w["weight"]}


WORKLOAD = workload_config(DEFAULT_WORKLOAD)


def flops_per_step(M, K, N, r):
    """Algorithmic work of one linear: the FP4 product and both low-rank projections."""
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def gemm_flops(M, K, N, r):
    """Algorithmic work of the GEMM kernel: the FP4 product and the low-rank up-projection."""
    return 2.0 * M * N * K + 2.0 * M * r * N


def quant_bytes(M, K, r):
    """Algorithmic bytes of one activation quantisation: the tensor amax reads X
    once (2MK), the quantise pass reads it again and writes the codes (MK/2),
    the scale bytes (MK/16) and U (4Mr), and reads inv_s (4K) and L1t (2Kr)."""
    a0 = 2 * M * K
    a = 2 * M * K + M * K // 2 + M * K // 16 + 4 * M * r + 4 * K + 2 * K * r
    return a0, a


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as fh:
            d = json.load(fh)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


GEMM_SOURCES = ["bit_diffusion_transformer_nvfp4_b200/csrc/gemm.cuh",
                "bit_diffusion_transformer_nvfp4_b200/csrc/gemm2.cuh",
                "bit_diffusion_transformer_nvfp4_b200/csrc/sm100.cuh"]
GEMM_SUMMARY = {"block2048": "gemm_block2048_up_ncu.md", "qkv1024": "gemm_flux1024_qkv_ncu.md"}


def source_hash(paths):
    h = hashlib.sha256()
    for p in paths:
        h.update(open(os.path.join(ROOT, p), "rb").read())
    return h.hexdigest()


def ncu_traffic(kernel_srcs, summary: str):
    """DRAM bytes per launch from the committed ncu summary, if that summary
    was taken on the current kernel sources (hash match); else None."""
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256:\s*([0-9a-f]{16,64})", text)
    if not m or not h:
        return None
    cur = source_hash(kernel_srcs)
    if not cur.startswith(h.group(1)):
        return None
    return float(m.group(1))


class ClockSampler:
    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return []
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        rows = []
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            rows.append(parts)
        return rows

    @staticmethod
    def summarise(rows, sm_floor=300.0):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = []
        power = []
        reasons = set()
        max_mhz = None
        for r in rows:
            try:
                mhz = float(r[1])
                max_mhz = float(r[2])
            except ValueError:
                continue
            if mhz < sm_floor:
                continue
            sm.append(mhz)
            try:
                power.append(float(r[3]))
            except ValueError:
                pass
            for n, v in zip(names, r[4:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max_mhz,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_median": statistics.median(power) if power else None}


# ---------------------------------------------------------------- our arm

def device_linear_inputs(torch, wl, K, N, seed, dev):
    """One linear's seeded synthetic inputs, drawn on the GPU with the
    workload's recipe: activation X [M, K] and a calibration draw [512, K]
    sharing its outlier structure, bf16 weight [N, K] ~ N(0, 0.02), bf16 bias
    ~ N(0, 0.01) or none."""
    M = wl["M"]
    g = torch.Generator(device=dev)
    g.manual_seed(seed)

    def randn(*shape):
        return torch.randn(*shape, generator=g, device=dev, dtype=torch.float32)

    if wl["act"] == "lognormal":
        mags = torch.exp(1.5 * randn(K))
        X = (randn(M, K) * mags).to(torch.bfloat16)
        Xc = (randn(512, K) * mags).to(torch.bfloat16)
    else:  # 1% of the channels replaced by 50 x Student-t(2) = 50 Z / sqrt(E), E ~ Exp(1)
        ch = torch.randperm(K, generator=g, device=dev)[:round(0.01 * K)]

        def draw(m):
            x = randn(m, K)
            e = -torch.log(torch.rand(m, len(ch), generator=g, device=dev).clamp_min(1e-30))
            x[:, ch] = 50.0 * randn(m, len(ch)) / torch.sqrt(e)
            return x.to(torch.bfloat16)
        X, Xc = draw(M), draw(512)
    W = (0.02 * randn(N, K)).to(torch.bfloat16)
    bias = (0.01 * randn(N)).to(torch.bfloat16) if wl["bias"] else None
    return X, Xc, W, bias


class Layer:
    """Device buffers of one linear of the step."""

    def __init__(self, torch, w4, name, M, K, N, r, X, w, dev, n_plain=None):
        self.name, self.M, self.K, self.N, self.r = name, M, K, N, r
        self.n_plain = N if n_plain is None else n_plain   # < N: SwiGLU pairs after the plain rows
        self.X, self.w = X, w
        self.qa = w4.QuantizedActivation(
            torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
            torch.empty(w4.nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=dev),
            torch.empty(1, dtype=torch.float32, device=dev),
            torch.empty(M, 2 * r, dtype=torch.bfloat16, device=dev), M, K, r)
        self.ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, r), dev)
        self.Y = torch.empty(M, self.n_plain, dtype=torch.bfloat16, device=dev)
        self.H = torch.empty(M, (N - self.n_plain) // 2, dtype=torch.bfloat16, device=dev) if self.n_plain < N else None

    def outputs(self):
        return [self.Y] if self.H is None else [self.Y, self.H]


def build_layers(torch, w4, prep, wl, dev):
    """Every linear of the workload (``l2_sets`` copies: rotating buffer sets
    for workloads that would otherwise sit in L2), weights prepared once."""
    sets = []
    packed = []
    for i, (name, K, N) in enumerate(wl["linears"]):
        X, Xc, W, bias = device_linear_inputs(torch, wl, K, N, wl["seed"] + 100 * i, dev)
        if name in wl["swiglu"]:
            # the kernel's row order: per 16 SwiGLU features, the gate rows then the up rows
            order = prep.swiglu_row_order(wl["swiglu"][name], (N - wl["swiglu"][name]) // 2, device=dev)
            W = W[order].contiguous()
            bias = None if bias is None else bias[order].contiguous()
        pk = prep.svdquant_prepare(W, Xc, r=wl["r"], bias=bias)
        del W, Xc
        packed.append((name, K, N, X, pk))
    for s in range(wl["l2_sets"]):
        layers = []
        for name, K, N, X, pk in packed:
            if s > 0:
                X = X.clone()
                pk = w4.PackedWeight(pk.Wq.clone(), pk.Wsf.clone(), pk.t_w.clone(), N, K, pk.inv_s.clone(),
                                     pk.L1t.clone(), pk.L2t.clone(), None if pk.bias is None else pk.bias.clone())
            layers.append(Layer(torch, w4, name, wl["M"], K, N, wl["r"], X, pk, dev, wl["swiglu"].get(name)))
        sets.append(layers)
    return sets


def max_over_ranks(values, world):
    """This rank's device times -> their maximum over all ranks (every rank
    gets the result).  One process per GPU; replicas share nothing else."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_tflops(world, flops_per_rank_step, steps, total_ms):
    """Throughput of the whole job: the units every rank processed over the
    slowest rank's device time."""
    return world * flops_per_rank_step * steps / (total_ms * 1e-3) / 1e12


def count_library_launches(torch, fn):
    """Kernels of this library (names in the ``w4a4`` namespace) that one call
    of ``fn`` launches, from the CUDA activity trace; None if no trace."""
    try:
        from torch.profiler import ProfilerActivity, profile
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            fn()
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if e.device_type.name == "CUDA"]
        n = sum(1 for nm in names if "w4a4::" in nm)
        return n if n > 0 else None
    except Exception:
        return None


def run_ours(args):
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        dist.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=300))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    import bit_diffusion_transformer_nvfp4_b200 as w4
    from bit_diffusion_transformer_nvfp4_b200 import prep
    w4.lib()

    wl = WORKLOADS[args.workload]
    sets = build_layers(torch, w4, prep, wl, dev)
    n_sets = len(sets)
    stream = torch.cuda.current_stream()

    def quant(L):
        w = L.w
        w4.nvfp4_quantize_act(L.X, L.M, L.K, L.K, w.inv_s, w.L1t, L.r, w.t_w, L.qa.Xq, L.qa.Xsf, L.qa.t_x, L.qa.U,
                              L.ws, stream)

    def gemm(L, qa=None, outs=None, st=None):
        w, qa = L.w, qa or L.qa
        Y, H = outs if outs is not None else (L.Y, L.H)
        st = st or stream
        if L.H is None:
            w4.w4a4_gemm(qa.Xq, qa.Xsf, qa.t_x, qa.U, L.M, L.N, L.K, w.Wq, w.Wsf, w.t_w, w.L2t, L.r, w.bias, 0,
                         Y, L.N, st)
        else:
            w4.w4a4_gemm_swiglu(qa.Xq, qa.Xsf, qa.t_x, qa.U, L.M, L.N, L.K, w.Wq, w.Wsf, w.t_w, w.L2t, L.r, w.bias,
                                L.n_plain, Y, L.n_plain, H, H.shape[1], None, None, st)

    def step(i, evs=None):
        for j, L in enumerate(sets[i % n_sets]):
            quant(L)
            if evs is not None:
                evs[2 * j + 1].record(stream)
            gemm(L)
            if evs is not None:
                evs[2 * j + 2].record(stream)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    barrier()
    per_step_launches = None if args.no_profile else count_library_launches(torch, lambda: step(0))
    barrier()
    n_lin = len(wl["linears"])
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    # One event pair brackets the timed steps.  Every MID_EVERY-th step also
    # records events before the first kernel and after each quantiser and
    # GEMM (the per-kernel durations).  An event between two kernels makes
    # the second wait for the first to finish instead of starting its set-up
    # early (programmatic launch), so the other steps go without them.
    ev_first, ev_last = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampled = list(range(0, args.steps, MID_EVERY))
    evs = {i: [torch.cuda.Event(enable_timing=True) for _ in range(2 * n_lin + 1)] for i in sampled}
    t_wall0 = time.time()
    ev_first.record(stream)
    for i in range(args.steps):
        if i in evs:
            evs[i][0].record(stream)
            step(i, evs[i])
        else:
            step(i)
    ev_last.record(stream)
    barrier()
    t_wall1 = time.time()
    clock_rows = sampler.stop()
    total_ms = ev_first.elapsed_time(ev_last)
    quant_ms = [statistics.mean(evs[i][2 * j].elapsed_time(evs[i][2 * j + 1]) for i in sampled) for j in range(n_lin)]
    gemm_ms = [statistics.mean(evs[i][2 * j + 1].elapsed_time(evs[i][2 * j + 2]) for i in sampled)
               for j in range(n_lin)]

    # End to end through the public API with host buffers: every step copies
    # each linear's X in from pinned host memory, runs w4a4_linear on it and
    # copies its Y out to pinned host memory.  Steps are pipelined over three
    # streams (copy in, compute, copy out) and two device buffer sets, as a
    # serving loop would run them: one step's copies overlap its neighbours'
    # work, and events keep the order within a step and the reuse of each
    # buffer set.
    layers0 = sets[0]
    xh = [L.X.cpu().pin_memory() for L in layers0]
    yh = [[[torch.empty_like(o, device="cpu").pin_memory() for o in L.outputs()] for L in layers0] for _ in range(2)]
    bufs = [[(L.X, L.outputs()) for L in layers0]]
    bufs.append([(torch.empty_like(L.X), [torch.empty_like(o) for o in L.outputs()]) for L in layers0])
    # w4a4_linear (quantiser + GEMM in one call) for plain linears; for the
    # SwiGLU projection the two public calls nvfp4_quantize_act and
    # w4a4_gemm_swiglu, with their own activation buffers and workspace
    lin_ws = [w4.new_workspace(w4.w4a4_workspace_bytes(L.M, L.N, L.K, L.r), dev) if L.H is None else None
              for L in layers0]
    e2e_qa = [None if L.H is None else
              (Layer(torch, w4, L.name, L.M, L.K, L.N, L.r, None, L.w, dev, L.n_plain)) for L in layers0]
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    e2e_steps = max(3, min(args.steps, args.e2e_steps))

    def e2e_run(n, e_start=None, e_end=None):
        done_c, done_out = [], []
        if e_start is not None:
            e_start.record(s_in)
        for i in range(n):
            b = bufs[i % 2]
            if i >= 2:
                s_in.wait_event(done_c[i - 2])        # step i-2 no longer reads these X
            with torch.cuda.stream(s_in):
                for (X, _), h in zip(b, xh):
                    X.copy_(h, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            s_c.wait_event(ev_in)
            if i >= 2:
                s_c.wait_event(done_out[i - 2])       # step i-2's outputs have been copied out
            for (X, outs), L, ws, tmp in zip(b, layers0, lin_ws, e2e_qa):
                w = L.w
                if tmp is None:
                    w4.w4a4_linear(X, L.M, L.N, L.K, w.Wq, w.Wsf, w.t_w, w.inv_s, w.L1t, w.L2t, L.r, w.bias, 0,
                                   outs[0], ws, s_c)
                else:
                    w4.nvfp4_quantize_act(X, L.M, L.K, L.K, w.inv_s, w.L1t, L.r, w.t_w, tmp.qa.Xq, tmp.qa.Xsf,
                                          tmp.qa.t_x, tmp.qa.U, tmp.ws, s_c)
                    gemm(L, tmp.qa, outs, s_c)
            ev_c = torch.cuda.Event()
            ev_c.record(s_c)
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                for (_, outs), hs in zip(b, yh[i % 2]):
                    for o, h in zip(outs, hs):
                        h.copy_(o, non_blocking=True)
            ev_out = torch.cuda.Event()
            ev_out.record(s_out)
            done_c.append(ev_c)
            done_out.append(ev_out)
        if e_end is not None:
            e_end.record(s_out)

    e2e_run(2)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    status = w4.w4a4_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}: {w4.w4a4_status_string(status)}")

    total_ms, e2e_ms, *kern = max_over_ranks([total_ms, e2e_ms, *quant_ms, *gemm_ms], world)
    quant_ms, gemm_ms = kern[:n_lin], kern[n_lin:]

    M, r = wl["M"], wl["r"]
    fl = sum(flops_per_step(M, K, N, r) for _, K, N in wl["linears"])
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(world, fl, args.steps, total_ms)
    peaks, peak_kind = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    fp4_peak_sus = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]) * FP4_OVER_BF16
    hbm = peaks["hbm_gbs"]
    rooflines = []
    for j, (name, K, N) in enumerate(wl["linears"]):
        g_fl = gemm_flops(M, K, N, r)
        ach = g_fl / (gemm_ms[j] * 1e-3) / 1e12
        a0, a = quant_bytes(M, K, r)
        qach = (a0 + a) / (quant_ms[j] * 1e-3) / 1e9
        # the GEMM is timed inside a seconds-long loop of steps, as the
        # sustained bf16 figure was measured: its FP4 equivalent is the peak
        rooflines.append({"kernel": f"gemm2_kernel ({name})", "bound": "tensor", "achieved": round(ach, 2),
                          "peak": round(fp4_peak_sus, 1), "unit": "TFLOP/s", "frac": round(ach / fp4_peak_sus, 4),
                          "frac_of_burst": round(ach / fp4_peak, 4), "launch_ms": round(gemm_ms[j], 5),
                          "algorithmic_flops_per_launch": g_fl})
        rooflines.append({"kernel": f"activation quantiser ({name}: tensor amax + quantise pass)", "bound": "hbm",
                          "achieved": round(qach, 1), "peak": hbm, "unit": "GB/s", "frac": round(qach / hbm, 4),
                          "launch_ms": round(quant_ms[j], 5), "algorithmic_bytes_per_call": a0 + a,
                          "bytes_basis": "amax pass 2MK + quantise pass 2MK + MK/2 + MK/16 + 4Mr + 4K + 2Kr"})
    top = max(range(n_lin), key=lambda j: gemm_ms[j])
    dom = dict(rooflines[2 * top])
    dom["traffic"] = ncu_traffic(GEMM_SOURCES, GEMM_SUMMARY[args.workload]) if top == 0 else None
    dom["peak_kind"] = (f"{peak_kind} sustained bf16 {peaks.get('bf16_tflops_sustained')} TFLOP/s x "
                        f"{FP4_OVER_BF16:g} (nominal FP4/BF16 ratio): the kernel runs inside a seconds-long loop "
                        f"under the power cap; frac_of_burst uses the burst figure {peaks['bf16_tflops']} x "
                        f"{FP4_OVER_BF16:g}")
    clocks = ClockSampler.summarise(clock_rows)
    if per_step_launches is None:
        per_step_launches = sum(1 + (2 if 2 * M * K > 64 << 20 else 1) for _, K, _n in wl["linears"])
        launch_basis = "expected per step (no activity trace)"
    else:
        launch_basis = "counted per step from the CUDA activity trace of one step"
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
        "data": "synthetic (seeded, drawn on the GPU)",
        "config": dict(workload_config(args.workload),
                       parallelism=f"replicas x{world}" if world > 1 else "single GPU", l2=wl["l2"]),
        "pct_fp4_peak": round(100.0 * value / (world * fp4_peak_sus), 2),
        "pct_fp4_peak_burst": round(100.0 * value / (world * fp4_peak), 2),
        "fp4_peak_tflops": round(fp4_peak_sus, 1),
        "fp4_peak_burst_tflops": round(fp4_peak, 1),
        "fp4_peak_basis": (f"{peak_kind} sustained bf16 {peaks.get('bf16_tflops_sustained')} TFLOPS x "
                           f"{FP4_OVER_BF16:g} (nominal FP4/BF16 ratio); burst {peaks['bf16_tflops']} x "
                           f"{FP4_OVER_BF16:g}"),
        "roofline": dom,
        "rooflines": rooflines,
        "kernels_ms": {**{f"quant_{n}": round(quant_ms[j], 5) for j, (n, _, _) in enumerate(wl["linears"])},
                       **{f"gemm_{n}": round(gemm_ms[j], 5) for j, (n, _, _) in enumerate(wl["linears"])},
                       "sampled_steps": len(sampled)},
        "e2e": {"value": round(whole_job_tflops(world, fl, 1, e2e_ms), 2), "unit": "TFLOPS",
                "h2d_bytes_per_step": int(sum(2 * M * K for _, K, _ in wl["linears"])),
                "d2h_bytes_per_step": int(sum(o.numel() * 2 for L in layers0 for o in L.outputs())),
                "ms_per_step": round(e2e_ms, 4), "steps": e2e_steps,
                "api": "w4a4_linear; nvfp4_quantize_act + w4a4_gemm_swiglu for the SwiGLU projection",
                "pipelining": "copy-in, compute and copy-out on three streams, two buffer sets"},
        "gpu_launches": per_step_launches * args.steps,
        "gpu_launches_basis": launch_basis,
        "clocks": clocks,
        "wall_s_timed": round(t_wall1 - t_wall0, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(wl, args.cpu_rows, args.cpu_cols)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------- per-configuration table

def run_table(args):
    """Every configuration's layers at full size on one GPU (not the contract
    line): per-kernel device times with L2 flushed before each repetition,
    the whole linear (quantiser + GEMM, one event pair around both), the GEMM
    back to back with warm L2, the MLP block (with the activation amax measured
    by the quantiser or taken from the up-projection's epilogue), config 1 by
    CUDA graph replay, and the denoising block per step and over a 50-step
    trajectory at batch 1, 2 and 4.  One JSON line per row."""
    import torch
    import bit_diffusion_transformer_nvfp4_b200 as w4
    from bit_diffusion_transformer_nvfp4_b200 import prep
    from synth import bf16_bits, config_cases, trajectory_step_activation

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w4.lib()
    s = torch.cuda.current_stream()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    peaks, peak_kind = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    reps = args.table_reps

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(bf16_bits(a).view(np.int16))).to(dev).view(torch.bfloat16)

    def med_us(fns, cold=True):
        """Median device time (us) of each callable in ``fns`` run in sequence,
        one event pair per callable."""
        for _ in range(3):
            for f in fns:
                f()
        torch.cuda.synchronize()
        ts = [[] for _ in fns]
        for _ in range(reps):
            if cold:
                flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
            ev[0].record(s)
            for i, f in enumerate(fns):
                f()
                ev[i + 1].record(s)
            torch.cuda.synchronize()
            for i in range(len(fns)):
                ts[i].append(ev[i].elapsed_time(ev[i + 1]) * 1e3)
        return [statistics.median(t) for t in ts]

    def b2b_us(fn, n=20):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for _ in range(n):
            fn()
        e1.record(s)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n * 1e3

    def tf(fl, us):
        return round(fl / (us * 1e-6) / 1e12, 1)

    def check():
        st = w4.w4a4_device_status()
        if st != 0:
            raise RuntimeError(f"device status {st}: {w4.w4a4_status_string(st)}")

    def emit(row):
        print(json.dumps(row), flush=True)

    swiglu_split = {(4, "qkv_swiglu_up"): 18432}  # the fused projection: plain QKV, then SwiGLU pairs

    def prepare(case, bias=True, n_plain=None):
        W = dev_bf16(case.w)
        Xc = dev_bf16(case.x_cal)
        b = dev_bf16(case.bias) if (bias and case.bias is not None) else None
        if n_plain is not None:  # the kernel's row order for the SwiGLU epilogue
            order = prep.swiglu_row_order(n_plain, (case.N - n_plain) // 2, device=dev)
            W = W[order].contiguous()
            b = None if b is None else b[order].contiguous()
        pk = prep.svdquant_prepare(W, Xc, r=case.r, bias=b)
        del W, Xc
        return pk

    def linear_row(cfg, case, pk, X, epi=0, n_plain=None):
        M, K, N, r = X.shape[0], X.shape[1], pk.N, pk.r
        ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, r), dev)
        qa = w4.quantize_act(X, pk.inv_s, pk.L1t, pk.t_w, workspace=ws)
        Y = torch.empty(M, N if n_plain is None else n_plain, dtype=torch.bfloat16, device=dev)
        H = None if n_plain is None else torch.empty(M, (N - n_plain) // 2, dtype=torch.bfloat16, device=dev)

        def qi():
            w4.nvfp4_quantize_act(X, M, K, X.stride(0), pk.inv_s, pk.L1t, r, pk.t_w, qa.Xq, qa.Xsf, qa.t_x,
                                  qa.U, ws, s)

        def g():
            if n_plain is None:
                w4.gemm(qa, pk, epilogue=epi, Y=Y)
            else:
                w4.gemm_swiglu(qa, pk, n_plain, Y=Y, H=H)

        def both():
            qi()
            g()
        tq, tg = med_us([qi, g])
        (tl,) = med_us([both])
        tgb = b2b_us(g)
        check()
        fl = flops_per_step(M, K, N, r)
        gfl = gemm_flops(M, K, N, r)
        qbytes = 2 * M * K + M * K // 2 + M * K // 16 + 2 * M * 2 * r
        row = {"table": "linear", "config": cfg, "layer": case.name, "M": M, "K": K, "N": N, "r": r,
               "epilogue": "swiglu" if n_plain is not None else ("gelu_tanh" if epi else "none"),
               "quant_us": round(tq, 2), "quant_gbs": round(qbytes / (tq * 1e-6) / 1e9, 1),
               "quant_frac_hbm": round(qbytes / (tq * 1e-6) / 1e9 / peaks["hbm_gbs"], 3),
               "gemm_us": round(tg, 2), "gemm_tflops": tf(gfl, tg), "gemm_frac_fp4": round(tf(gfl, tg) / fp4_peak, 3),
               "gemm_warm_b2b_us": round(tgb, 2), "gemm_warm_b2b_tflops": tf(gfl, tgb),
               "linear_us": round(tl, 2), "linear_tflops": tf(fl, tl),
               "linear_frac_fp4": round(tf(fl, tl) / fp4_peak, 3)}
        emit(row)
        return qa, ws, Y, qi, g

    def quant_next_row(cfg, case, pk, qa, g, epi=0, n_plain=None, next_K=None, next_col=0):
        """The GEMM whose epilogue also writes the next layer's NVFP4 codes and
        scale bytes (w4a4_gemm_quantize_next, given tensor scale), with and
        without storing the bf16 outputs, beside the plain GEMM."""
        M, N = qa.M, pk.N
        n_out = N if n_plain is None else (N - n_plain) // 2
        next_K = n_out if next_K is None else next_K
        t_next = torch.full((1,), 0.01, device=dev)
        s_next = torch.ones(n_out, device=dev)
        nq = torch.empty(M, next_K // 2, dtype=torch.uint8, device=dev)
        nsf = torch.empty(w4.nvfp4_sf_bytes(M, next_K), dtype=torch.uint8, device=dev)
        outs = {}

        def gq(store):
            def f():
                w4.gemm_quantize_next(qa, pk, t_next, next_inv_s=s_next, epilogue=epi, n_plain=n_plain,
                                      store_outputs=store, next_K=next_K, next_col=next_col, next_q=nq,
                                      next_sf=nsf)
            return f
        t_plain, t_store, t_codes = med_us([g, gq(True), gq(False)])
        check()
        gfl = gemm_flops(M, case.K, N, pk.r)
        emit({"table": "quantise_into_epilogue", "config": cfg, "layer": case.name, "M": M, "K": case.K, "N": N,
              "outputs_quantised": n_out, "gemm_us": round(t_plain, 2),
              "gemm_with_next_codes_us": round(t_store, 2), "gemm_next_codes_only_us": round(t_codes, 2),
              "gemm_next_codes_only_tflops": tf(gfl, t_codes)})

    def rope_row(cfg, case, pk, qa, g, n_plain, d_head=128, axes=(16, 56, 56), n_text=512, side=128):
        """The fused projection with the rotary embedding on its query and key
        features (w4a4_gemm_rope; heads of 128, the angles of a text + image
        token sequence) beside the same GEMM with the SwiGLU epilogue alone."""
        from synth import token_positions
        M, N = qa.M, pk.N
        n_rope = 2 * (n_plain // 3)                  # Q and K of the plain Q | K | V features
        tab = prep.rope_table(torch.from_numpy(token_positions(n_text, side, side)).to(dev), axes)
        assert tab.shape[0] == M
        Y = torch.empty(M, n_plain, dtype=torch.bfloat16, device=dev)
        H = torch.empty(M, (N - n_plain) // 2, dtype=torch.bfloat16, device=dev)

        def gr():
            w4.gemm_rope(qa, pk, tab, n_rope, d_head, n_plain=n_plain, Y=Y, H=H)
        t_plain, t_rope = med_us([g, gr])
        check()
        gfl = gemm_flops(M, case.K, N, pk.r)
        emit({"table": "rope_epilogue", "config": cfg, "layer": case.name, "M": M, "K": case.K, "N": N,
              "rotated_outputs": n_rope, "d_head": d_head, "gemm_swiglu_us": round(t_plain, 2),
              "gemm_rope_swiglu_us": round(t_rope, 2), "gemm_rope_swiglu_tflops": tf(gfl, t_rope),
              "gemm_rope_swiglu_frac_fp4": round(tf(gfl, t_rope) / fp4_peak, 3),
              "rope_cost_pct": round(100.0 * (t_rope / t_plain - 1.0), 2)})

    emit({"table": "peaks", "fp4_peak_tflops": round(fp4_peak, 1), "hbm_gbs": peaks["hbm_gbs"],
          "basis": f"{peak_kind}: bf16 burst x {FP4_OVER_BF16:g}; copy bandwidth", "reps": reps,
          "l2": "256 MB buffer zeroed before each repetition"})

    def graph_row(case, pk, X, qa, ws, Y, qi, g):
        """The small layer is launch-bound: quantiser + GEMM replayed as one CUDA graph."""
        M, K, N, r = case.M, case.K, pk.N, pk.r

        def enqueue(st):
            w4.nvfp4_quantize_act(X, M, K, K, pk.inv_s, pk.L1t, r, pk.t_w, qa.Xq, qa.Xsf, qa.t_x, qa.U, ws, st)
            w4.w4a4_gemm(qa.Xq, qa.Xsf, qa.t_x, qa.U, M, N, K, pk.Wq, pk.Wsf, pk.t_w, pk.L2t, r, pk.bias, 0, Y,
                         N, st)

        fl = flops_per_step(M, K, N, r)
        (tpl,) = med_us([lambda: (qi(), g())], cold=False)
        row = {"table": "graph", "config": 1, "layer": case.name, "linear_plain_warm_us": round(tpl, 2),
               "linear_plain_warm_tflops": tf(fl, tpl)}
        try:
            side = torch.cuda.Stream()
            side.wait_stream(s)
            with torch.cuda.stream(side):
                for _ in range(3):
                    enqueue(side)
            s.wait_stream(side)
            torch.cuda.synchronize()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                enqueue(torch.cuda.current_stream())
            tgr = b2b_us(graph.replay, n=200)
            check()
            row.update(linear_graph_us=round(tgr, 2), linear_graph_tflops=tf(fl, tgr))
            del graph
        except Exception as exc:  # report, keep the rest of the table
            row["graph_error"] = str(exc)[:200]
        emit(row)

    # configs 1, 2, 4: independent linears (config 4's fused projection with
    # its SwiGLU epilogue, and quantising its SwiGLU outputs into columns
    # 6144.. of the output projection's 24576-wide activation)
    for cfg in (1, 2, 4):
        for case in config_cases(cfg):
            n_plain = swiglu_split.get((cfg, case.name))
            pk = prepare(case, n_plain=n_plain)
            X = dev_bf16(case.x)
            qa, ws, Y, qi, g = linear_row(cfg, case, pk, X, n_plain=n_plain)
            if cfg == 1:
                graph_row(case, pk, X, qa, ws, Y, qi, g)
            if n_plain is not None:
                rope_row(cfg, case, pk, qa, g, n_plain)
                quant_next_row(cfg, case, pk, qa, g, n_plain=n_plain, next_K=24576, next_col=6144)
            del pk, X, qa, ws, Y
            torch.cuda.empty_cache()

    # config 3: MLP block, GELU between, measured amax vs amax from the up-projection's epilogue
    up, down = config_cases(3)
    pu, pd = prepare(up), prepare(down)
    X = dev_bf16(up.x)
    qa_u, ws_u, H, qi_u, g_u = linear_row(3, up, pu, X, epi=1)
    quant_next_row(3, up, pu, qa_u, g_u, epi=1)
    M = up.M
    ws_d = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, down.K, down.r), dev)
    qa_d = w4.quantize_act(H, pd.inv_s, pd.L1t, pd.t_w, workspace=ws_d)
    Yd = torch.empty(M, down.N, dtype=torch.bfloat16, device=dev)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)

    def qd():
        w4.nvfp4_quantize_act(H, M, down.K, down.K, pd.inv_s, pd.L1t, down.r, pd.t_w, qa_d.Xq, qa_d.Xsf,
                              qa_d.t_x, qa_d.U, ws_d, s)

    def qd_given():
        w4.nvfp4_quantize_act_with_amax(H, M, down.K, down.K, pd.inv_s, pd.L1t, down.r, pd.t_w, amax, qa_d.Xq,
                                        qa_d.Xsf, qa_d.t_x, qa_d.U, ws_d, s)

    def gd():
        w4.gemm(qa_d, pd, Y=Yd)

    def up_amax():
        amax.zero_()
        w4.gemm(qa_u, pu, epilogue=w4.EPI_GELU_TANH, Y=H, next_inv_s=pd.inv_s, next_amax=amax)

    tq, tg = med_us([qd, gd])
    fl_d = flops_per_step(M, down.K, down.N, down.r)
    qbytes = 2 * M * down.K + M * down.K // 2 + M * down.K // 16 + 2 * M * 2 * down.r
    emit({"table": "linear", "config": 3, "layer": down.name, "M": M, "K": down.K, "N": down.N, "r": down.r,
          "input": "GELU output of the up-projection",
          "quant_us": round(tq, 2), "quant_gbs": round(qbytes / (tq * 1e-6) / 1e9, 1),
          "quant_frac_hbm": round(qbytes / (tq * 1e-6) / 1e9 / peaks["hbm_gbs"], 3),
          "gemm_us": round(tg, 2), "gemm_tflops": tf(gemm_flops(M, down.K, down.N, down.r), tg),
          "gemm_frac_fp4": round(tf(gemm_flops(M, down.K, down.N, down.r), tg) / fp4_peak, 3)})
    (tb_meas,) = med_us([lambda: (qi_u(), g_u(), qd(), gd())])
    (tb_fused,) = med_us([lambda: (qi_u(), up_amax(), qd_given(), gd())])
    (t_ua, t_qg) = med_us([up_amax, qd_given])
    check()
    fl_b = flops_per_step(M, up.K, up.N, up.r) + fl_d
    emit({"table": "mlp_block", "config": 3, "M": M,
          "block_us_measured_amax": round(tb_meas, 2), "block_tflops_measured_amax": tf(fl_b, tb_meas),
          "block_us_epilogue_amax": round(tb_fused, 2), "block_tflops_epilogue_amax": tf(fl_b, tb_fused),
          "gemm_up_with_amax_us": round(t_ua, 2), "quant_down_given_amax_us": round(t_qg, 2)})
    del pu, pd, X, qa_u, ws_u, H, ws_d, qa_d, Yd
    torch.cuda.empty_cache()

    # FP8 attention on the sequences of the two block sizes (heads of 128):
    # the three per-tensor E4M3 quantisations and the attention kernel
    for S, H, what in ((4608, 24, "1024px sequence, hidden 3072"), (16896, 48, "2048px sequence, hidden 6144")):
        ga = torch.Generator(device=dev)
        ga.manual_seed(9000 + S)
        q = (1.5 * torch.randn(S, H * 128, generator=ga, device=dev)).to(torch.bfloat16)
        k = (1.5 * torch.randn(S, H * 128, generator=ga, device=dev)).to(torch.bfloat16)
        v = torch.randn(S, H * 128, generator=ga, device=dev).to(torch.bfloat16)
        tq, tk, tv = w4.quantize_fp8(q), w4.quantize_fp8(k), w4.quantize_fp8(v, transpose=True)
        Oa = torch.empty(S, H * 128, dtype=torch.bfloat16, device=dev)
        wsq = torch.empty(w4.fp8_quant_workspace_bytes(S, H * 128), dtype=torch.uint8, device=dev)

        def quant3():
            for x, t, tr in ((q, tq, False), (k, tk, False), (v, tv, True)):
                w4.fp8_quantize(x, S, H * 128, H * 128, tr, t.codes, t.codes.stride(0), t.scale, wsq)

        def att():
            w4.attention(tq, tk, tv, H, O=Oa)
        t_q, t_a = med_us([quant3, att])
        check()
        fl = 4.0 * S * S * 128 * H
        qbytes = 3 * (2 * S * H * 128 + 2 * S * H * 128 + S * H * 128)   # amax read, quantise read, codes
        emit({"table": "attention_fp8", "sequence": what, "S": S, "heads": H, "d_head": 128,
              "attention_us": round(t_a, 1), "attention_tflops": tf(fl, t_a),
              "attention_frac_fp8": round(tf(fl, t_a) / (peaks["bf16_tflops"] * 2.0), 3),
              "fp8_peak_basis": "measured bf16 burst x 2 (nominal FP8/BF16)",
              "quantise_qkv_us": round(t_q, 1), "quantise_qkv_gbs": round(qbytes / (t_q * 1e-6) / 1e9, 1)})
        del q, k, v, tq, tk, tv, Oa, wsq
        torch.cuda.empty_cache()

    # config 5: the denoising block (fused QKV + MLP-up projection on one
    # quantised activation, GELU on the MLP part, MLP-down) per step, and a
    # 50-step trajectory; every step re-quantises a fresh activation
    qkv, mlp, dn = config_cases(5)
    K = qkv.K
    w_cat = np.concatenate([qkv.w, mlp.w], axis=0)
    b_cat = np.concatenate([qkv.bias, mlp.bias])
    x_cal = np.concatenate([trajectory_step_activation(t, 10, K)[0] for t in range(50)], axis=0)
    pf = prep.svdquant_prepare(dev_bf16(w_cat), dev_bf16(x_cal), r=32, bias=dev_bf16(b_cat))
    w_q, w_m = pf.rows(0, qkv.N), pf.rows(qkv.N, w_cat.shape[0])
    pdn = prepare(dn)
    del w_cat
    for B in (1, 2, 4):
        M = 4608 * B
        acts = [dev_bf16(trajectory_step_activation(t, M, K)[0]) for t in range(3)]
        ws1 = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, 32), dev)
        ws2 = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, dn.K, 32), dev)
        qa1 = w4.quantize_act(acts[0], pf.inv_s, pf.L1t, pf.t_w, workspace=ws1)
        Yq = torch.empty(M, qkv.N, dtype=torch.bfloat16, device=dev)
        Hm = torch.empty(M, mlp.N, dtype=torch.bfloat16, device=dev)
        qa2 = w4.quantize_act(Hm, pdn.inv_s, pdn.L1t, pdn.t_w, workspace=ws2)
        Yd = torch.empty(M, dn.N, dtype=torch.bfloat16, device=dev)

        def block(t=0):
            Xs = acts[t % 3]
            w4.nvfp4_quantize_act(Xs, M, K, K, pf.inv_s, pf.L1t, 32, pf.t_w, qa1.Xq, qa1.Xsf, qa1.t_x, qa1.U,
                                  ws1, s)
            w4.gemm(qa1, w_q, Y=Yq)
            w4.gemm(qa1, w_m, epilogue=w4.EPI_GELU_TANH, Y=Hm)
            w4.nvfp4_quantize_act(Hm, M, dn.K, dn.K, pdn.inv_s, pdn.L1t, 32, pdn.t_w, qa2.Xq, qa2.Xsf, qa2.t_x,
                                  qa2.U, ws2, s)
            w4.gemm(qa2, pdn, Y=Yd)

        (t_step,) = med_us([block])
        for t in range(3):
            block(t)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s)
        for t in range(50):
            block(t)
        e1.record(s)
        torch.cuda.synchronize()
        t_traj = e0.elapsed_time(e1)
        check()
        fl = (flops_per_step(M, K, qkv.N, 32) + flops_per_step(M, K, mlp.N, 32)
              + flops_per_step(M, dn.K, dn.N, 32))
        emit({"table": "denoising_block", "config": 5, "batch": B, "M": M,
              "step_us_l2_flushed": round(t_step, 2), "step_tflops": tf(fl, t_step),
              "trajectory_50_steps_ms": round(t_traj, 3), "trajectory_tflops": tf(50 * fl, t_traj * 1e3),
              "trajectory_note": "50 steps back to back, three rotating activations, no L2 flush"})
        del acts, ws1, ws2, qa1, qa2, Yq, Hm, Yd
        torch.cuda.empty_cache()


# ---------------------------------------------------------------- profiling cases

CASES = {
    # name: (what, M, K, N or None, extra)
    "gemm_block2048_up": ("w4a4_gemm_swiglu, the 2048px fused QKV+SwiGLU-up projection", 16896, 6144, 55296, 18432),
    "gemm_block2048_up_small": ("w4a4_gemm_swiglu, the 2048px fused projection at 4096 tokens", 4096, 6144, 55296, 18432),
    "gemm_block2048_out": ("w4a4_gemm, the 2048px output projection", 16896, 24576, 6144, None),
    "gemm_rope_block2048_small": ("w4a4_gemm_rope, the 2048px fused projection at 4096 tokens, the rotary embedding "
                                  "on its 12288 query and key outputs (heads of 128) and SwiGLU on the rest",
                                  4096, 6144, 55296, 18432),
    "gemm_quant_next_block2048_small": ("w4a4_gemm_quantize_next, the 2048px fused projection at 4096 tokens, its "
                                        "SwiGLU outputs quantised into columns 6144.. of a 24576-wide activation",
                                        4096, 6144, 55296, 18432),
    "gemm_flux1024_qkv": ("w4a4_gemm, the FLUX-1024px QKV projection (CTA pairs, 256 x 256 tiles)", 4608, 3072, 9216, None),
    "gemm_row_block": ("w4a4_gemm on a single 128-row block (CTA pairs, 256 x 64 tiles)", 128, 3072, 3072, None),
    "gemm_single_cta": ("w4a4_gemm on a single row block with N > 64 SMs (single-CTA 128 x 192 tiles)", 64, 3072, 19200,
                        None),
    "quant_fused_flux1024": ("nvfp4_quantize_act, single pass (4608 x 3072)", 4608, 3072, None, None),
    "quant_two_pass_block2048": ("nvfp4_quantize_act, two passes (16896 x 6144)", 16896, 6144, None, None),
    "quant_stream_block2048": ("nvfp4_quantize_act_with_amax, streaming pass (16896 x 6144)", 16896, 6144, None, None),
    "attention_fp8_small": ("attention_fp8 on 4096 tokens, 8 heads of 128 (E4M3 operands)", 4096, 1024, None, None),
    "pack_weight_block2048_out": ("nvfp4_pack_weight on an fp32 residual (6144 x 24576)", 6144, 24576, None, None),
}


def run_case(args):
    """One kernel's small workload for an ncu capture: ``--steps`` calls of the
    entry point after ``--warmup`` untimed ones, inputs drawn on the GPU
    (lognormal channel magnitudes), rank 32.  Prints the mean event time per
    call.  Nothing here is a benchmark line."""
    import torch
    import bit_diffusion_transformer_nvfp4_b200 as w4
    what, M, K, N, n_plain = CASES[args.case]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w4.lib()
    st = torch.cuda.current_stream()
    g = torch.Generator(device=dev)
    g.manual_seed(77)
    r = 32
    mags = torch.exp(1.5 * torch.randn(K, generator=g, device=dev))
    inv_s = (1.0 / torch.exp(0.3 * torch.randn(K, generator=g, device=dev))).contiguous()
    L1t = (0.02 * torch.randn(r, K, generator=g, device=dev)).to(torch.bfloat16)
    t_w = torch.full((1,), 0.01, device=dev)
    if args.case.startswith("attention"):
        heads = K // 128
        tq = w4.quantize_fp8((1.5 * torch.randn(M, K, generator=g, device=dev)).to(torch.bfloat16))
        tk = w4.quantize_fp8((1.5 * torch.randn(M, K, generator=g, device=dev)).to(torch.bfloat16))
        tv = w4.quantize_fp8(torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16), transpose=True)
        Oa = torch.empty(M, K, dtype=torch.bfloat16, device=dev)

        def call():
            w4.attention_fp8(tq.codes, tk.codes, tv.codes, 1, M, heads, K, K, M, tq.scale, tk.scale, tv.scale,
                             1.0 / 128 ** 0.5, Oa, K, st)
    elif args.case.startswith("pack_weight"):
        R = 0.02 * torch.randn(M, K, generator=g, device=dev)
        ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, 0), dev)
        Wq = torch.empty(M, K // 2, dtype=torch.uint8, device=dev)
        Wsf = torch.empty(w4.nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=dev)
        tw = torch.empty(1, device=dev)

        def call():
            w4.nvfp4_pack_weight(R, w4.SRC_F32, M, K, K, Wq, Wsf, tw, ws, st)
    else:
        X = (torch.randn(M, K, generator=g, device=dev) * mags).to(torch.bfloat16)
        qa = w4.quantize_act(X, inv_s, L1t, t_w)
        ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, r), dev)
        amax = torch.full((1,), float((X.float() * inv_s).abs().max()), device=dev)
        if args.case.startswith("quant_stream"):
            def call():
                w4.nvfp4_quantize_act_with_amax(X, M, K, K, inv_s, L1t, r, t_w, amax, qa.Xq, qa.Xsf, qa.t_x, qa.U,
                                                ws, st)
        elif args.case.startswith("quant"):
            def call():
                w4.nvfp4_quantize_act(X, M, K, K, inv_s, L1t, r, t_w, qa.Xq, qa.Xsf, qa.t_x, qa.U, ws, st)
        else:
            W = 0.02 * torch.randn(N, K, generator=g, device=dev)
            pw = w4.pack_weight(W)
            del W
            L2t = (0.02 * torch.randn(N, r, generator=g, device=dev)).to(torch.bfloat16)
            if args.case.startswith("gemm_quant_next"):
                Y = torch.empty(M, n_plain, dtype=torch.bfloat16, device=dev)
                H = torch.empty(M, (N - n_plain) // 2, dtype=torch.bfloat16, device=dev)
                t_next = torch.full((1,), 0.01, device=dev)
                nq = torch.empty(M, 24576 // 2, dtype=torch.uint8, device=dev)
                nsf = torch.empty(w4.nvfp4_sf_bytes(M, 24576), dtype=torch.uint8, device=dev)

                def call():
                    w4.w4a4_gemm_quantize_next(qa.Xq, qa.Xsf, qa.t_x, qa.U, M, N, K, pw.Wq, pw.Wsf, pw.t_w, L2t, r,
                                               None, 0, n_plain, Y, n_plain, H, H.shape[1], None, t_next, nq,
                                               nq.stride(0), nsf, 24576, 6144, None, st)
            elif args.case.startswith("gemm_rope"):
                Y = torch.empty(M, n_plain, dtype=torch.bfloat16, device=dev)
                H = torch.empty(M, (N - n_plain) // 2, dtype=torch.bfloat16, device=dev)
                from bit_diffusion_transformer_nvfp4_b200 import prep
                tab = prep.rope_table(torch.arange(M, device=dev), (128,))   # one position axis

                def call():
                    w4.w4a4_gemm_rope(qa.Xq, qa.Xsf, qa.t_x, qa.U, M, N, K, pw.Wq, pw.Wsf, pw.t_w, L2t, r, None,
                                      12288, 128, tab, 128, n_plain, Y, n_plain, H, H.shape[1], None, None, st)
            elif n_plain is None:
                Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

                def call():
                    w4.w4a4_gemm(qa.Xq, qa.Xsf, qa.t_x, qa.U, M, N, K, pw.Wq, pw.Wsf, pw.t_w, L2t, r, None, 0, Y, N,
                                 st)
            else:
                Y = torch.empty(M, n_plain, dtype=torch.bfloat16, device=dev)
                H = torch.empty(M, (N - n_plain) // 2, dtype=torch.bfloat16, device=dev)

                def call():
                    w4.w4a4_gemm_swiglu(qa.Xq, qa.Xsf, qa.t_x, qa.U, M, N, K, pw.Wq, pw.Wsf, pw.t_w, L2t, r, None,
                                        n_plain, Y, n_plain, H, H.shape[1], None, None, st)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(args.steps):
        call()
    e1.record(st)
    torch.cuda.synchronize()
    status = w4.w4a4_device_status()
    print(json.dumps({"case": args.case, "what": what, "M": M, "K": K, "N": N, "calls": args.steps,
                      "warmup": args.warmup, "us_per_call": round(e0.elapsed_time(e1) / args.steps * 1e3, 2),
                      "status": status}), flush=True)
    if status != 0:
        raise RuntimeError(f"device status {status}")


def run_fp4_peak(args):
    """The measured FP4 peak: w4a4_fp4_mma_rate on every SM, CTA pairs
    (256 x 256 x 64 MMAs) and single CTAs (128 x 256 x 64), --fp4-iters MMAs
    per issuer, event-timed launches after warm-up ones; the issuers' own
    cycle counts give the clock.  One JSON line per mode."""
    import torch
    import bit_diffusion_transformer_nvfp4_b200 as w4
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    w4.lib()
    st = torch.cuda.current_stream()
    n_sm = torch.cuda.get_device_properties(dev).multi_processor_count
    cycles = torch.zeros(n_sm, dtype=torch.int64, device=dev)
    peaks, peak_kind = load_peaks()
    for pair in (1, 0):
        issuers = n_sm // 2 if pair else n_sm
        flops = 2.0 * (256 if pair else 128) * 256 * 64
        for _ in range(max(args.warmup, 3)):
            w4.w4a4_fp4_mma_rate(args.fp4_iters, pair, cycles, st)
        torch.cuda.synchronize()
        ms = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            w4.w4a4_fp4_mma_rate(args.fp4_iters, pair, cycles, st)
            e1.record(st)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        status = w4.w4a4_device_status()
        c = cycles[:issuers].cpu().numpy().astype(np.float64)
        t = statistics.median(ms)
        tflops = issuers * args.fp4_iters * flops / (t * 1e-3) / 1e12
        print(json.dumps({"fp4_mma_rate": "pair 256x256x64" if pair else "single 128x256x64",
                          "issuers": issuers, "mmas_per_issuer": args.fp4_iters, "ms": round(t, 4),
                          "tflops": round(tflops, 1),
                          "cycles_per_mma": round(float(np.median(c)) / args.fp4_iters, 2),
                          "sm_mhz_from_cycles": round(float(np.median(c)) / (t * 1e-3) / 1e6, 1),
                          "vs_nominal_fp4_of_measured_bf16": round(tflops / (peaks["bf16_tflops"] * FP4_OVER_BF16), 3),
                          "status": status}), flush=True)
        if status != 0 or not np.all(c > 0):
            raise RuntimeError(f"device status {status}")


# ---------------------------------------------------------------- oracle arms

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_samples(wl, n_rows, n_cols):
    """A bounded sample of every linear of the workload, drawn with the same
    recipe (synth): ``n_rows`` tokens x ``n_cols`` output channels at the
    layer's full K, with the oracle's preparation done (not timed)."""
    from oracle import nvfp4, prep
    from synth import make_linear
    out = []
    act = "lognormal" if wl["act"] == "lognormal" else "student_t"
    for i, (name, K, N) in enumerate(wl["linears"]):
        c = make_linear(name, n_rows, K, n_cols, r=wl["r"], act=act, bias_std=0.01 if wl["bias"] else 0.0,
                        seed=wl["seed"] + 100 * i)
        p = prep.svdquant_prepare(c.w, c.x_cal, c.r, c.alpha)
        wq, wsf, tw, _ = nvfp4.quantize_activation(p["R"], None)
        # a SwiGLU projection's sample: half plain columns, then gate and up quarters
        sw = (n_cols // 2, n_cols // 4) if name in wl["swiglu"] else None
        out.append((c, p, wq, wsf, tw, sw))
    return out


def oracle_step(samples):
    from oracle import linear as olinear
    from oracle import swiglu as oswiglu
    for c, p, wq, wsf, tw, sw in samples:
        y, _ = olinear.w4a4_linear(c.x, p["inv_s"], wq, wsf, tw, p["L1t"], p["L2t"], c.bias)
        if sw is not None:
            oswiglu.split_fused(y, *sw)


def sample_flops(wl, n_rows, n_cols):
    return sum(flops_per_step(n_rows, K, n_cols, wl["r"]) for _, K, _ in wl["linears"])


def sample_text(wl, n_rows, n_cols):
    layers = ", ".join(f"{name} K={K}" for name, K, _ in wl["linears"])
    return (f"{n_rows} of {wl['M']} tokens x {n_cols} output channels of each linear ({layers}), drawn with the "
            f"workload's recipe; the sample's own tensor scale")


def cpu_baseline(wl, n_rows=256, n_cols=1024, min_seconds=10.0):
    """The oracle as it stands on a bounded sample of the workload (numpy fp32
    quantiser, fp64 matmul); throughput counts the sample's FLOPs."""
    samples = oracle_samples(wl, n_rows, n_cols)
    iters = 0
    t0 = time.perf_counter()
    while True:
        oracle_step(samples)
        iters += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    fl = sample_flops(wl, n_rows, n_cols) * iters
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOPS", "cores": cpu_threads(), "kind": "oracle",
            "sample": sample_text(wl, n_rows, n_cols) + f"; repeated {iters}x in {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = WORKLOADS[getattr(args, "workload", DEFAULT_WORKLOAD)]
    samples = oracle_samples(wl, args.ref_rows, args.ref_cols)
    for _ in range(args.warmup):
        oracle_step(samples)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(samples)
    dt = time.perf_counter() - t0
    fl = sample_flops(wl, args.ref_rows, args.ref_cols)
    value = fl * args.steps / dt / 1e12
    sample = "per step: " + sample_text(wl, args.ref_rows, args.ref_cols)
    name = getattr(args, "workload", DEFAULT_WORKLOAD)
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS", "n_gpus": 0,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": dict(workload_config(name), parallelism="host CPU"),
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": cpu_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-rows", type=int, default=256)
    ap.add_argument("--cpu-cols", type=int, default=1024)
    ap.add_argument("--ref-rows", type=int, default=32)
    ap.add_argument("--ref-cols", type=int, default=128)
    ap.add_argument("--e2e-steps", type=int, default=12)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-profile", action="store_true",
                    help="skip the activity trace that counts the library's kernel launches (e.g. under ncu)")
    ap.add_argument("--table", action="store_true",
                    help="time every configuration's layers (one JSON line per row) instead of the benchmark step")
    ap.add_argument("--table-reps", type=int, default=20)
    ap.add_argument("--case", choices=sorted(CASES),
                    help="run one kernel's small profiling workload (--steps calls after --warmup) instead")
    ap.add_argument("--fp4-peak", action="store_true",
                    help="measure the FP4 tensor-core instruction rate (back-to-back MMAs on every SM) instead")
    ap.add_argument("--fp4-iters", type=int, default=100000)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.fp4_peak:
        run_fp4_peak(args)
    elif args.case:
        run_case(args)
    elif args.table:
        run_table(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
