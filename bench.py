#!/usr/bin/env python
"""Benchmark of the W4A4 NVFP4 linear hot path on B200.

One step = one pass of the whole hot path over one batch: tensor amax, fused
smooth/quantise/pack + low-rank down-projection, and the block-scaled FP4 GEMM
with the low-rank up-projection, bias and bf16 cast, on the FLUX-1024px QKV
projection (M = 4608 tokens = 4096 image + 512 text, K = 3072, N = 9216,
rank 32, bf16 bias).  Inputs are synthetic (seeded), shaped like that workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line.  Under torchrun (N > 1) every rank runs an independent
replica on its own GPU (the path has no cross-GPU exchange); rank 0 prints.
``--impl reference`` times the plain CPU oracle on the host cores instead.
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

WORKLOAD = {"workload": "FLUX-1024px QKV projection", "M": 4608, "K": 3072, "N": 9216, "r": 32,
            "bias": True, "activation": "N(0,1) with 1% Student-t(2)x50 channels", "weight": "N(0,0.02)"}
METRIC = "W4A4 linear TFLOPS (act-quant+FP4 GEMM+low-rank)"
L2_SETS = 3          # rotating buffer sets, each ~140 MB, so every step starts L2-cold
MID_EVERY = 10       # steps between per-kernel timing events inside the timed region
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def flops_per_step(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def gemm_flops(M, K, N, r):
    return 2.0 * M * N * K + 2.0 * M * N * (2 * r)  # main GEMM + the hi/lo low-rank pass


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
            for n, v in zip(names, r[4:]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max_mhz,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- our arm

def build_inputs(torch, w4, prep, dev):
    from synth import config_cases, bf16_bits
    case = config_cases(2)[0]
    M, K, N, r = case.M, case.K, case.N, case.r

    def dev_bf16(a):
        return torch.from_numpy(np.ascontiguousarray(bf16_bits(a).view(np.int16))).to(dev).view(torch.bfloat16)

    W = dev_bf16(case.w)
    Xc = dev_bf16(case.x_cal)
    bias = dev_bf16(case.bias)
    packed = prep.svdquant_prepare(W, Xc, r=r, bias=bias)
    del W, Xc
    x_host = np.ascontiguousarray(bf16_bits(case.x).view(np.int16))
    sets = []
    for i in range(L2_SETS):
        X = torch.from_numpy(x_host).to(dev).view(torch.bfloat16)
        w = w4.PackedWeight(packed.Wq.clone(), packed.Wsf.clone(), packed.t_w.clone(), N, K,
                            packed.inv_s.clone(), packed.L1t.clone(), packed.L2t.clone(), packed.bias.clone())
        qa = w4.QuantizedActivation(
            torch.empty(M, K // 2, dtype=torch.uint8, device=dev),
            torch.empty(w4.nvfp4_sf_bytes(M, K), dtype=torch.uint8, device=dev),
            torch.empty(1, dtype=torch.float32, device=dev),
            torch.empty(M, 2 * r, dtype=torch.bfloat16, device=dev), M, K, r)
        ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, r), dev)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        sets.append((X, w, qa, ws, Y))
    return case, x_host, sets


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

    case, x_host, sets = build_inputs(torch, w4, prep, dev)
    M, K, N, r = case.M, case.K, case.N, case.r
    stream = torch.cuda.current_stream()

    def step(i, ev_mid=None):
        X, w, qa, ws, Y = sets[i % L2_SETS]
        w4.nvfp4_quantize_act(X, M, K, K, w.inv_s, w.L1t, r, w.t_w, qa.Xq, qa.Xsf, qa.t_x, qa.U, ws, stream)
        if ev_mid is not None:
            ev_mid.record(stream)
        w4.w4a4_gemm(qa.Xq, qa.Xsf, qa.t_x, qa.U, M, N, K, w.Wq, w.Wsf, w.t_w, w.L2t, r, w.bias, 0, Y, N, stream)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()

    sampler = ClockSampler(local)
    sampler.start()
    for i in range(args.warmup):
        step(i)
    barrier()
    # One event pair brackets the timed steps.  Every MID_EVERY-th step also
    # records events before the quantiser, between the kernels and after the
    # GEMM (the per-kernel durations).  An event between two kernels makes
    # the second wait for the first to finish instead of starting its set-up
    # early (programmatic launch), so the other steps go without them.
    ev_first, ev_last = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampled = list(range(0, args.steps, MID_EVERY))
    evs = {i: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
               torch.cuda.Event(enable_timing=True)) for i in sampled}
    t_wall0 = time.time()
    ev_first.record(stream)
    for i in range(args.steps):
        if i in evs:
            evs[i][0].record(stream)
            step(i, evs[i][1])
            evs[i][2].record(stream)
        else:
            step(i)
    ev_last.record(stream)
    barrier()
    t_wall1 = time.time()
    total_ms = ev_first.elapsed_time(ev_last)
    gemm_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in sampled]
    quant_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in sampled]

    # End to end through the public API with host buffers: every step copies
    # its X in from pinned host memory, runs w4a4_linear and copies its Y out
    # to pinned host memory.  Steps are pipelined over three streams (copy in,
    # compute, copy out) and two device buffer sets, as a serving loop would
    # run them: one step's copies overlap its neighbours' work, and events keep
    # the order within a step and the reuse of each buffer set.
    import torch as _t
    xh = _t.from_numpy(x_host).view(_t.bfloat16).pin_memory()
    yh = [_t.empty(M, N, dtype=_t.bfloat16).pin_memory() for _ in range(2)]
    e2e_steps = max(3, min(args.steps, 50))
    w0 = sets[0][1]
    bufs = [(sets[j][0], sets[j][4]) for j in range(2)]
    lin_ws = w4.new_workspace(w4.w4a4_workspace_bytes(M, N, K, r), dev)
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_run(n, e_start=None, e_end=None):
        done_c, done_out = [], []
        if e_start is not None:
            e_start.record(s_in)
        for i in range(n):
            X, Y = bufs[i % 2]
            if i >= 2:
                s_in.wait_event(done_c[i - 2])        # step i-2 no longer reads this X
            with torch.cuda.stream(s_in):
                X.copy_(xh, non_blocking=True)
            ev_in = torch.cuda.Event()
            ev_in.record(s_in)
            s_c.wait_event(ev_in)
            if i >= 2:
                s_c.wait_event(done_out[i - 2])       # step i-2's Y has been copied out
            w4.w4a4_linear(X, M, N, K, w0.Wq, w0.Wsf, w0.t_w, w0.inv_s, w0.L1t, w0.L2t, r, w0.bias, 0, Y,
                           lin_ws, s_c)
            ev_c = torch.cuda.Event()
            ev_c.record(s_c)
            s_out.wait_event(ev_c)
            with torch.cuda.stream(s_out):
                yh[i % 2].copy_(Y, non_blocking=True)
            ev_out = torch.cuda.Event()
            ev_out.record(s_out)
            done_c.append(ev_c)
            done_out.append(ev_out)
        if e_end is not None:
            e_end.record(s_out)

    e2e_run(4)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_run(e2e_steps, e0, e1)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    clock_rows = sampler.stop()
    status = w4.w4a4_device_status()
    if status != 0:
        raise RuntimeError(f"device status {status}: {w4.w4a4_status_string(status)}")

    total_ms, e2e_ms = max_over_ranks([total_ms, e2e_ms], world)

    fl = flops_per_step(M, K, N, r)
    ms_per_step = total_ms / args.steps
    value = whole_job_tflops(world, fl, args.steps, total_ms)
    peaks, peak_kind = load_peaks()
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    gemm_avg_ms = statistics.mean(gemm_ms)
    g_fl = gemm_flops(M, K, N, r)
    achieved = g_fl / (gemm_avg_ms * 1e-3) / 1e12
    traffic = ncu_traffic(GEMM_SOURCES, "gemm_flux1024_qkv_ncu.md")
    clocks = ClockSampler.summarise(clock_rows)
    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4",
        "data": "synthetic",
        "config": dict(WORKLOAD, parallelism=f"replicas x{world}" if world > 1 else "single GPU",
                       l2=f"{L2_SETS} rotating input/weight/output sets of ~140 MB each (> 126 MB L2)"),
        "pct_fp4_peak": round(100.0 * value / (world * fp4_peak), 2),
        "fp4_peak_tflops": round(fp4_peak, 1),
        "fp4_peak_basis": f"{peak_kind} bf16 burst {peaks['bf16_tflops']} TFLOPS x {FP4_OVER_BF16:g} (nominal FP4/BF16 ratio)",
        "roofline": {"kernel": "gemm2_kernel (CTA-pair block-scaled FP4 + low-rank + bias epilogue)", "bound": "tensor",
                     "achieved": round(achieved, 2), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(achieved / fp4_peak, 4), "traffic": traffic,
                     "peak_kind": f"{peak_kind} (bf16 burst x4)", "launch_ms": round(gemm_avg_ms, 5),
                     "algorithmic_flops_per_launch": g_fl},
        "kernels_ms": {"amax+quant": round(statistics.mean(quant_ms), 5), "gemm": round(gemm_avg_ms, 5),
                       "sampled_steps": len(gemm_ms)},
        "e2e": {"value": round(whole_job_tflops(world, fl, 1, e2e_ms), 2), "unit": "TFLOPS",
                "h2d_bytes_per_step": int(M * K * 2), "d2h_bytes_per_step": int(M * N * 2),
                "ms_per_step": round(e2e_ms, 4), "api": "w4a4_linear",
                "pipelining": "copy-in, compute and copy-out on three streams, two buffer sets"},
        # per step: the single-pass quantiser and the pair GEMM
        "gpu_launches": 2 * args.steps,
        "clocks": clocks,
        "wall_s_timed": round(t_wall1 - t_wall0, 3),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(case, args.cpu_rows, args.cpu_cols)
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

    def prepare(case, bias=True):
        W = dev_bf16(case.w)
        Xc = dev_bf16(case.x_cal)
        b = dev_bf16(case.bias) if (bias and case.bias is not None) else None
        pk = prep.svdquant_prepare(W, Xc, r=case.r, bias=b)
        del W, Xc
        return pk

    def linear_row(cfg, case, pk, X, epi=0):
        M, K, N, r = X.shape[0], X.shape[1], pk.N, pk.r
        ws = w4.new_workspace(w4.nvfp4_quant_workspace_bytes(M, K, r), dev)
        qa = w4.quantize_act(X, pk.inv_s, pk.L1t, pk.t_w, workspace=ws)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)

        def qi():
            w4.nvfp4_quantize_act(X, M, K, X.stride(0), pk.inv_s, pk.L1t, r, pk.t_w, qa.Xq, qa.Xsf, qa.t_x,
                                  qa.U, ws, s)

        def g():
            w4.gemm(qa, pk, epilogue=epi, Y=Y)

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
               "epilogue": "gelu_tanh" if epi else "none",
               "quant_us": round(tq, 2), "quant_gbs": round(qbytes / (tq * 1e-6) / 1e9, 1),
               "quant_frac_hbm": round(qbytes / (tq * 1e-6) / 1e9 / peaks["hbm_gbs"], 3),
               "gemm_us": round(tg, 2), "gemm_tflops": tf(gfl, tg), "gemm_frac_fp4": round(tf(gfl, tg) / fp4_peak, 3),
               "gemm_warm_b2b_us": round(tgb, 2), "gemm_warm_b2b_tflops": tf(gfl, tgb),
               "linear_us": round(tl, 2), "linear_tflops": tf(fl, tl),
               "linear_frac_fp4": round(tf(fl, tl) / fp4_peak, 3)}
        emit(row)
        return qa, ws, Y, qi, g

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

    # configs 1, 2, 4: independent linears
    for cfg in (1, 2, 4):
        for case in config_cases(cfg):
            pk = prepare(case)
            X = dev_bf16(case.x)
            qa, ws, Y, qi, g = linear_row(cfg, case, pk, X)
            if cfg == 1:
                graph_row(case, pk, X, qa, ws, Y, qi, g)
            del pk, X, qa, ws, Y
            torch.cuda.empty_cache()

    # config 3: MLP block, GELU between, measured amax vs amax from the up-projection's epilogue
    up, down = config_cases(3)
    pu, pd = prepare(up), prepare(down)
    X = dev_bf16(up.x)
    qa_u, ws_u, H, qi_u, g_u = linear_row(3, up, pu, X, epi=1)
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
        acts = [dev_bf16(np.concatenate([trajectory_step_activation(t, 4608, K)[0]] * B, axis=0))
                for t in range(3)]
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


# ---------------------------------------------------------------- oracle arms

def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def oracle_prepared(case, cols):
    """Oracle-side preparation (not timed): smoothing, SVD, and the NVFP4
    packing of the weight rows of the sampled output channels under the whole
    residual's tensor scale."""
    from oracle import nvfp4, prep
    p = prep.svdquant_prepare(case.w, case.x_cal, case.r, case.alpha)
    R = p["R"]
    codes, wsf, tw, _ = nvfp4.quantize(R[cols], amax=np.max(np.abs(R)))
    return p, nvfp4.pack(codes), wsf, tw


def sample_indices(case, rows, cols):
    g = np.random.Generator(np.random.PCG64(7))
    return (np.sort(g.choice(case.M, rows, replace=False)), np.sort(g.choice(case.N, cols, replace=False)))


def oracle_step(case, prepared, rows, cols):
    from oracle import linear as olinear
    p, wq, wsf, tw = prepared
    olinear.w4a4_linear(case.x, p["inv_s"], wq, wsf, tw, p["L1t"], p["L2t"][cols],
                        None if case.bias is None else case.bias[cols], rows=rows)


def cpu_baseline(case, n_rows=1024, n_cols=2048, min_seconds=10.0):
    """The oracle as it stands on a bounded sample of the workload: the whole
    activation's tensor scale, then quantisation of ``n_rows`` sampled tokens
    and Y for them on ``n_cols`` sampled output channels (numpy fp32
    quantiser, fp64 matmul).  Throughput counts the sample's FLOPs."""
    rows, cols = sample_indices(case, n_rows, n_cols)
    prepared = oracle_prepared(case, cols)
    iters = 0
    t0 = time.perf_counter()
    while True:
        oracle_step(case, prepared, rows, cols)
        iters += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            break
    fl = flops_per_step(n_rows, case.K, n_cols, case.r) * iters
    return {"value": round(fl / dt / 1e12, 6), "unit": "TFLOPS", "cores": cpu_threads(), "kind": "oracle",
            "sample": f"{n_rows} of {case.M} tokens x {n_cols} of {case.N} output channels, K={case.K}, "
                      f"whole-tensor activation scale; repeated {iters}x in {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from synth import config_cases
    case = config_cases(2)[0]
    rows, cols = sample_indices(case, args.ref_rows, args.ref_cols)
    prepared = oracle_prepared(case, cols)
    for _ in range(args.warmup):
        oracle_step(case, prepared, rows, cols)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(case, prepared, rows, cols)
    dt = time.perf_counter() - t0
    fl = flops_per_step(args.ref_rows, case.K, args.ref_cols, case.r)
    value = fl * args.steps / dt / 1e12
    sample = (f"per step: {args.ref_rows} of {case.M} tokens x {args.ref_cols} of {case.N} output channels, "
              f"K={case.K}, whole-tensor activation scale")
    out = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOPS", "n_gpus": 0,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * dt / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": dict(WORKLOAD, parallelism="host CPU"),
           "cpu_baseline": {"value": round(value, 6), "unit": "TFLOPS", "cores": cpu_threads(), "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-rows", type=int, default=1024)
    ap.add_argument("--cpu-cols", type=int, default=2048)
    ap.add_argument("--ref-rows", type=int, default=256)
    ap.add_argument("--ref-cols", type=int, default=1024)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--table", action="store_true",
                    help="time every configuration's layers (one JSON line per row) instead of the benchmark step")
    ap.add_argument("--table-reps", type=int, default=20)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.table:
        run_table(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
