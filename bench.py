#!/usr/bin/env python
"""Benchmark of the RaBiT residual-binary linear layer on B200 (librabit).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one batch-1 decode pass over the Llama-2-7B-shaped layer set (q, k, v, o
4096x4096; gate, up 11008x4096; down 4096x11008), i.e. seven rabit_gemv calls on seeded
synthetic weights and activations.  The weights of ten independent copies of the set
(about 506 MB of packed signs, more than four times the 126 MB L2) are resident in HBM and
step s uses copy s mod 10, so every step streams its weights from HBM.  The steps of one
copy are captured once in a CUDA graph and replayed.

The printed JSON line carries the metric (packed-weight HBM GB/s of the decode pass), the
roofline of the GEMV kernel, the SM clocks seen during the timed region, an end-to-end
figure through the public Python API with host copies, and, on rank 0 with one GPU, the
secondary measurements of the same metric string (rabit_gemm TFLOP/s at M=2048 on the
Llama-3-8B MLP shapes, rabit_derive_pack GB/s, the Llama-3-70B MLP QAT step, the scale
gradients and the Iterative Residual SVID initialisation of a 4096x4096 layer) plus the
float64 oracle timed on a bounded sample as the CPU baseline.

--impl reference times the float64 CPU oracle (the reference arm of this repository) on the
same workload, metric and unit: each step evaluates a bounded sample of rows of the layer set.
With several GPUs (torchrun), every rank runs its own replica of the workload (weak
scaling, no collective on the data path); the elapsed time is the maximum over ranks.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from bit_gemv_rabit_b200 import inputs  # noqa: E402

METRIC = "residual-binary GEMV HBM GB/s (% of peak) at batch 1; GEMM TFLOP/s at M=2048"
WORKLOAD = "llama2_7b_decode_b1"
COPIES = 10
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=400)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the GEMM / derive / CPU-baseline measurements")
    ap.add_argument("--profile-kernel", choices=["derive", "gemv", "gemv_set", "gemm", "svid", "scale_grads"],
                    default=None,
                    help="run a few launches of one kernel (for an ncu capture) and exit")
    ap.add_argument("--shape", type=int, nargs=3, metavar=("N", "K", "M"), default=(11008, 4096, 1),
                    help="with --profile-kernel: out features, in features, batch/tokens")
    ap.add_argument("--launches", type=int, default=3)
    ap.add_argument("--oracle-table", action="store_true",
                    help="time the float64 CPU oracle on every workload (no GPU) and exit")
    ap.add_argument("--gemm-token-sample", type=int, default=8,
                    help="with --oracle-table: tokens of the GEMM workloads the oracle evaluates")
    return ap.parse_args(argv)


# ----------------------------------------------------------------------------- ranks
def dist_init():
    """(rank, world, local_rank, group-or-None) from the torchrun environment."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))
        return rank, world, local, dist
    return rank, world, local, None


def aggregate(elapsed_ms: float, units: float, dist=None, device=None):
    """Max of the elapsed time and sum of the processed units over ranks."""
    if dist is None:
        return elapsed_ms, units
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    u = torch.tensor([units], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return float(t.item()), float(u.item())


def barrier(dist, device):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.lines = []
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            ident = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            ident = str(device_index)
        self.cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                    "-lms", "200", "-i", ident]

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                                         text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- inputs
def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def sign_bytes(layers) -> int:
    """Packed sign bytes of one decode pass (the work of the dp2a pipe)."""
    return sum(2 * L["N"] * (((L["K"] + 127) // 128) * 128) // 8 for L in layers)


def bf16_tensor(bits: np.ndarray, device) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


def make_layer(rabit, spec, idx, name, N, K, device, batch, P=2):
    seed = inputs.seed_for(spec["cfg"], idx)
    W = inputs.weight(seed, N, K, sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
    a, b = inputs.scales(seed, W, P=P)
    at = torch.from_numpy(a).to(device)
    bt = torch.from_numpy(b).to(device)
    packed = rabit.alloc_packed(N, K, P=P, device=device)
    rabit.rabit_derive_pack(torch.from_numpy(W).to(device), at, bt, packed, P=P)
    x = inputs.activations(seed, batch, K, channel_outlier_frac=spec["x_outliers"])
    return dict(name=name, N=N, K=K, P=P, a=at, b=bt, packed=packed, x_host=x,
                x=bf16_tensor(x, device), y=torch.empty((batch, N), device=device),
                ws=rabit.alloc_gemv_workspace(N, K, P, min(batch, 16), device=device) if batch <= 16 else None)


def layer_tuples(layers, B=None):
    """(packed, a, b, N, K, x, y) of each layer for rabit_gemv_grouped (first B batch rows)."""
    return [(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"][:B] if B else L["x"],
             L["y"][:B] if B else L["y"]) for L in layers]


# Decoder-order grouping of each decode set: the projections that read the same activation
# share one call (q, k, v; gate, up); o and down each follow their own input.
DECODER_GROUPS = {"llama2_7b_decode_b1": [[0, 1, 2], [3], [4, 5], [6]],
                  "llama3_8b_decode": [[0, 1, 2], [3, 4], [5]]}


def decode_schedules(rabit, sets, spec_name, device, B=None, steps=400, warmup=20):
    """Microseconds per set for three schedules of the same matrices: one rabit_gemv per matrix
    (the library picks the kernel by batch), one rabit_gemv_grouped per decoder group, and one
    rabit_gemv_grouped over the whole set (the matrices as independent GEMVs)."""
    base = sets[0]
    ws = rabit.alloc_gemv_grouped_workspace(layer_tuples(base, B), P=base[0]["P"], device=device)
    groups = DECODER_GROUPS[spec_name]

    def per_matrix(ls):
        return lambda: [rabit.rabit_gemv(L["packed"], L["a"], L["b"], L["N"], L["K"],
                                         L["x"][:B] if B else L["x"], L["y"][:B] if B else L["y"],
                                         P=L["P"], workspace=L["ws"]) for L in ls]

    def grouped(ls):
        return lambda: [rabit.rabit_gemv_grouped(layer_tuples([ls[i] for i in g], B), P=ls[0]["P"], workspace=ws)
                        for g in groups]

    def one_call(ls):
        return lambda: rabit.rabit_gemv_grouped(layer_tuples(ls, B), P=ls[0]["P"], workspace=ws)

    out = {}
    for name, mk in (("per_matrix", per_matrix), ("decoder_groups", grouped), ("one_call", one_call)):
        graphs = [capture_graph(mk(ls)) for ls in sets]
        out[name] = round(timed_replays(graphs, steps, warmup, None, device) / steps * 1e3, 2)
        del graphs
    return out


def decode_bytes(layers, batch=1):
    """Algorithmic bytes of one decode pass: packed signs + scales + x + y (per layer)."""
    total = 0
    for L in layers:
        N, K = L["N"], L["K"]
        Kp = ((K + 127) // 128) * 128
        total += 2 * N * Kp // 8 + 4 * 2 * (N + K) + batch * K * 2 + batch * N * 4
    return total


# ----------------------------------------------------------------------------- timing
def capture_graph(fn):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fn()
    torch.cuda.synchronize()
    return g


def timed_replays(graphs, steps, warmup, dist, device, clocks=None):
    """Replay graphs[s % len] for warmup + steps; returns (elapsed ms over the timed steps)."""
    for s in range(warmup):
        graphs[s % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ctx = clocks if clocks is not None else _null()
    with ctx:
        e0.record()
        for s in range(steps):
            graphs[s % len(graphs)].replay()
        e1.record()
        torch.cuda.synchronize()
    barrier(dist, device)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1)


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


# ----------------------------------------------------------------------------- secondary
def bench_gemm(rabit, device, hbm_peak, tf_peak, tf_sustained):
    """rabit_gemm on the Llama-3-8B MLP shapes at M=2048 (the metric's second half)."""
    spec = inputs.WORKLOADS["llama3_8b_mlp_prefill_m2048"]
    M = spec["batches"][0]
    copies = 3
    sets = []
    for c in range(copies):
        layers = []
        for idx, (name, N, K) in enumerate(spec["set"]):
            if c == 0:
                L = make_layer(rabit, spec, idx, name, N, K, device, M)
            else:
                base = sets[0][idx]
                L = dict(base, packed=base["packed"].clone(), x=base["x"].clone(),
                         y=torch.empty_like(base["y"]))
            L["ws"] = rabit.alloc_gemm_workspace(N, K, 2, M, device=device)
            layers.append(L)
        sets.append(layers)

    def step_fn(layers):
        def f():
            for L in layers:
                rabit.rabit_gemm(L["packed"], L["a"], L["b"], L["N"], L["K"], L["x"], L["y"], L["ws"])
        return f

    gws = rabit.alloc_gemm_grouped_workspace(layer_tuples(sets[0]), device=device)

    def grouped_fn(layers):
        return lambda: rabit.rabit_gemm_grouped(layer_tuples(layers), gws)

    steps = 400                                   # about 0.55 s: the clock sampler sees it
    flops = sum(2 * 2 * M * L["N"] * L["K"] for L in sets[0])
    graphs = [capture_graph(step_fn(ls)) for ls in sets]
    ms_per_layer = timed_replays(graphs, steps, 5, None, device)
    del graphs
    graphs = [capture_graph(grouped_fn(ls)) for ls in sets]
    clocks = ClockSampler(device.index)
    ms = timed_replays(graphs, steps, 5, None, device, clocks)
    del graphs
    tflops = flops * steps / (ms * 1e-3) / 1e12
    tflops_per_layer = flops * steps / (ms_per_layer * 1e-3) / 1e12
    fp8 = measure_fp8_tflops(device)
    roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": tf_peak, "unit": "TFLOP/s",
            "frac": round(tflops / tf_peak, 4),
            "peak_note": "measured dense bf16 burst; fp16 operands have the same nominal rate",
            "frac_of_nominal_fp8_dense_4500": round(tflops / 4500.0, 4),
            "sustained_peak": tf_sustained, "frac_of_sustained": round(tflops / tf_sustained, 4)}
    if fp8 is not None:
        roof["fp8_dense_measured_tflops"] = fp8
        roof["frac_of_measured_fp8_dense"] = round(tflops / fp8, 4)
    return {"workload": "llama3_8b_mlp_prefill_m2048", "value": round(tflops, 1), "unit": "TFLOP/s",
            "dtype": "fp16", "ms_per_step": round(ms / steps, 4), "launches_per_step": len(sets[0]) + 1,
            "schedule": "gate, up and down as one rabit_gemm_grouped launch (independent layers, own x each)",
            "per_layer_calls": {"ms_per_step": round(ms_per_layer / steps, 4),
                                "TFLOP_per_s": round(tflops_per_layer, 1)},
            "clocks": clocks.summary(),
            "roofline": roof}


def measure_fp8_tflops(device, n=8192, reps=10):
    """Dense e4m3 GEMM throughput of this part (torch._scaled_mm, n^3, best of reps): the
    denominator for an fp8 fraction.  None when the call is not available."""
    try:
        a = torch.randn((n, n), device=device).to(torch.float8_e4m3fn)
        b = torch.randn((n, n), device=device).to(torch.float8_e4m3fn).t()
        one = torch.ones((), device=device)
        for _ in range(3):
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
        torch.cuda.synchronize()
        best = float("inf")
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch._scaled_mm(a, b, scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
            e1.record()
            torch.cuda.synchronize()
            best = min(best, e0.elapsed_time(e1))
        del a, b
        return round(2.0 * n ** 3 / (best * 1e-3) / 1e12, 1)
    except Exception:
        return None


def bench_decode_sweep(rabit, device, hbm_peak):
    """Llama-3-8B-shaped decode set (q 4096x4096, k/v 1024x4096, gate/up 14336x4096, down
    4096x14336, 0.1% x20 weight outliers) at batch 1, 4, 8 and 16: microseconds per set for the
    per-matrix, decoder-order and one-call schedules, three rotated copies of the packed
    weights (more than L2)."""
    spec = inputs.WORKLOADS["llama3_8b_decode"]
    out = {"workload": "llama3_8b_decode", "copies": 3, "by_batch": {}}
    Bmax = max(spec["batches"])
    base = [make_layer(rabit, spec, idx, name, N, K, device, Bmax)
            for idx, (name, N, K) in enumerate(spec["set"])]
    sets = [base] + [[dict(L, packed=L["packed"].clone()) for L in base] for _ in range(2)]
    torch.cuda.synchronize()
    for B in spec["batches"]:
        sched = decode_schedules(rabit, sets, "llama3_8b_decode", device, B=B, steps=300, warmup=20)
        byts = decode_bytes(base, batch=B)
        out["by_batch"][str(B)] = {k: {"us_per_set": v, "GB_per_s": round(byts / (v * 1e-6) / 1e9, 1),
                                       "hbm_frac": round(byts / (v * 1e-6) / 1e9 / hbm_peak, 4)}
                                   for k, v in sched.items()}
    del sets, base
    torch.cuda.empty_cache()
    return out


def warm_launch_us(rabit, layers, device):
    """Microseconds per launch of each distinct shape, re-reading the same weights 200 times
    in a graph (L2-resident after the first launch: the warm-cache setting of the pages'
    kernel-latency table)."""
    out = {}
    for L in layers:
        key = f"{L['N']}x{L['K']}"
        if key in out:
            continue
        g = capture_graph(lambda L=L: [rabit.rabit_gemv(L["packed"], L["a"], L["b"], L["N"], L["K"],
                                                        L["x"], L["y"], P=L["P"], workspace=L["ws"])
                                       for _ in range(200)])
        out[key] = round(timed_replays([g], 5, 2, None, device) / 5 / 200 * 1e3, 2)
    return out


def bench_gemv_three_path(rabit, device, hbm_peak):
    """The 3-bit variant (three paths) on the same Llama-2-7B decode set, batch 1, ten rotated
    copies (the pages' Table 7 reports 3-bit kernel latencies beside the 2-bit ones)."""
    spec = inputs.WORKLOADS[WORKLOAD]
    base = [make_layer(rabit, spec, idx, name, N, K, device, 1, P=3)
            for idx, (name, N, K) in enumerate(spec["set"])]
    sets = [base] + [[dict(L, packed=L["packed"].clone()) for L in base] for _ in range(COPIES - 1)]
    torch.cuda.synchronize()
    sched = decode_schedules(rabit, sets, WORKLOAD, device, steps=1000, warmup=50)
    algo = sum(3 * L["N"] * (((L["K"] + 127) // 128) * 128) // 8 + 4 * 3 * (L["N"] + L["K"])
               + L["K"] * 2 + L["N"] * 4 for L in base)
    best = sched["one_call"]
    gbs = algo / (best * 1e-6) / 1e9
    return {"workload": "llama2_7b_decode_b1_3path", "value": round(gbs, 1), "unit": "GB/s",
            "us_per_set": best, "schedules_us_per_set": sched,
            "us_per_launch_warm_l2_by_shape": warm_launch_us(rabit, base, device),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4)},
            "note": "3 sign words + 1 padding word per group in HBM; algorithmic bytes count the 3 signs"}


def bench_scale_grads(rabit, device, hbm_peak):
    """QAT backward of the scales on the Llama-3-70B MLP shape (G = dL/dW_hat fp32 28672x8192):
    rabit_scale_grads reads G and the packed signs once (HBM-bound)."""
    spec = inputs.WORKLOADS["llama3_70b_mlp_qat_m4096"]
    name, N, K = spec["set"][0]
    seed = inputs.seed_for(spec["cfg"], 0)
    W = inputs.weight(seed, N, K, sigma=spec["sigma"])
    a, b = inputs.scales(seed, W)
    at, bt = torch.from_numpy(a).to(device), torch.from_numpy(b).to(device)
    packed = rabit.alloc_packed(N, K, device=device)
    rabit.rabit_derive_pack(torch.from_numpy(W).to(device), at, bt, packed)
    del W
    G = torch.empty((N, K), device=device).normal_(generator=torch.Generator(device=device).manual_seed(seed))
    ga, gb = torch.empty((2, N), device=device), torch.empty((2, K), device=device)
    ws = rabit.alloc_scale_grads_workspace(N, K, 2, device=device)
    g = capture_graph(lambda: rabit.rabit_scale_grads(G, packed, at, bt, N, K, ga, gb, ws))
    steps = 20
    ms = timed_replays([g], steps, 3, None, device)
    byts = N * K * 4 + 2 * N * (((K + 127) // 128) * 128) // 8 + 4 * 2 * (N + K) * 2
    gbs = byts * steps / (ms * 1e-3) / 1e9
    return {"workload": "llama3_70b_mlp_scale_grads_28672x8192", "value": round(gbs, 1), "unit": "GB/s",
            "us_per_call": round(ms / steps * 1e3, 2),
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4)}}


SVID_T, SVID_POWER_ITERS = 20, 40
SVID_ALPHA_IN, SVID_ALPHA_OUT = 0.8, 0.65   # the pages' Table 11 intensities, Llama2-7B, 2 bits


def bench_svid_init(rabit, device, hbm_peak):
    """Initialisation of one Llama-2-7B q_proj-shaped layer (4096x4096 fp32 W, seeded
    calibration statistics): Iterative Residual SVID, T = 20, two paths, 40 power steps per
    update.  Algorithmic bytes per update: the residual pass reads W and the other path's
    signs and writes R (fp32) and the new signs; each power step reads R once.  Beside it, the
    same initialisation with the power steps stopped once a step moves u and v by at most 1e-6."""
    spec = inputs.WORKLOADS["llama2_7b_decode_b1"]
    name, N, K = spec["set"][0]
    seed = inputs.seed_for(spec["cfg"], 0)
    W = torch.from_numpy(inputs.weight(seed, N, K, sigma=spec["sigma"])).to(device)
    s_in, s_out = inputs.calibration_stats(seed, N, K)
    si, so = torch.from_numpy(s_in).to(device), torch.from_numpy(s_out).to(device)
    P = 2
    a, b = torch.empty((P, N), device=device), torch.empty((P, K), device=device)
    packed = rabit.alloc_packed(N, K, P=P, device=device)
    ws = rabit.alloc_svid_init_workspace(N, K, P, device=device)

    def timed(tol):
        def run():
            rabit.rabit_svid_init(W, si, so, SVID_ALPHA_IN, SVID_ALPHA_OUT, a, b, packed, ws, P=P, T=SVID_T,
                                  power_iters=SVID_POWER_ITERS, power_tol=tol)
        run()
        torch.cuda.synchronize()
        reps = 3
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            run()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps
    ms = timed(0.0)
    ms_settled = timed(1e-6)
    nk = N * K
    sign_bytes = N * (((K + 127) // 128) * 128) // 8
    per_update = (4 * nk + 4 * nk + (P - 1) * sign_bytes + sign_bytes + SVID_POWER_ITERS * 4 * nk)
    byts = SVID_T * P * per_update
    gbs = byts / (ms * 1e-3) / 1e9
    return {"workload": "llama2_7b_q_proj_4096x4096_svid_init", "T": SVID_T, "P": P,
            "power_iters": SVID_POWER_ITERS, "ms_per_init": round(ms, 3),
            "launches_per_init": 2 + 2 * SVID_T * P,
            "ms_per_init_settled_1e-6": round(ms_settled, 3),
            "value": round(gbs, 1), "unit": "GB/s",
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                         "frac": round(gbs / hbm_peak, 4),
                         "note": "the 67 MB residual is re-read by every power step and fits in L2"}}


def bench_qat_step(rabit, device, hbm_peak, tf_peak, tf_sustained):
    """Llama-3-70B MLP QAT forward: derive_pack of W (fp32 28672x8192) then GEMM at M=4096."""
    spec = inputs.WORKLOADS["llama3_70b_mlp_qat_m4096"]
    name, N, K = spec["set"][0]
    M = spec["batches"][0]
    seed = inputs.seed_for(spec["cfg"], 0)
    W = inputs.weight(seed, N, K, sigma=spec["sigma"])
    a, b = inputs.scales(seed, W)
    Wt, at, bt = (torch.from_numpy(v).to(device) for v in (W, a, b))
    del W
    packed = rabit.alloc_packed(N, K, device=device)
    x = bf16_tensor(inputs.activations(seed, M, K), device)
    y = torch.empty((M, N), device=device)
    ws = rabit.alloc_gemm_workspace(N, K, 2, M, device=device)

    def derive():
        rabit.rabit_derive_pack(Wt, at, bt, packed)

    def step():
        rabit.rabit_derive_pack(Wt, at, bt, packed)
        rabit.rabit_gemm(packed, at, bt, N, K, x, y, ws)

    # backward of the input: the transposed planes, then the GEMM of the transposed layer
    packed_t = rabit.alloc_packed(K, N, device=device)
    dy = bf16_tensor(inputs.activations(seed + 1, M, N), device)
    gx = torch.empty((M, K), device=device)
    ws_t = rabit.alloc_gemm_workspace(K, N, 2, M, device=device)

    def transpose():
        rabit.rabit_transpose_pack(packed, N, K, packed_t)

    def grad_x():
        rabit.rabit_grad_x(packed_t, at, bt, N, K, dy, gx, ws_t)

    derive()
    g_derive = capture_graph(derive)
    g_step = capture_graph(step)
    g_t = capture_graph(transpose)
    g_gx = capture_graph(grad_x)
    steps = 20
    ms_d = timed_replays([g_derive], steps, 5, None, device)
    ms_s = timed_replays([g_step], steps, 3, None, device)
    ms_t = timed_replays([g_t], steps, 5, None, device)
    ms_g = timed_replays([g_gx], steps, 3, None, device)
    d_bytes = N * K * 4 + 2 * N * K // 8 + 4 * 2 * (N + K)
    gbs = d_bytes * steps / (ms_d * 1e-3) / 1e9
    flops = 2 * 2 * M * N * K
    t_bytes = 2 * (2 * N * (((K + 127) // 128) * 128) // 8)          # read and write of two planes
    t_gbs = t_bytes * steps / (ms_t * 1e-3) / 1e9
    gx_tflops = flops * steps / (ms_g * 1e-3) / 1e12
    return {"derive_pack": {"workload": "llama3_70b_mlp_w_fp32_28672x8192", "value": round(gbs, 1),
                            "unit": "GB/s", "us_per_call": round(ms_d / steps * 1e3, 2),
                            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak,
                                         "unit": "GB/s", "frac": round(gbs / hbm_peak, 4)}},
            "qat_step": {"workload": "llama3_70b_mlp_qat_m4096", "ms_per_step": round(ms_s / steps, 4),
                         "derive_plus_gemm_tflops": round(flops / (ms_s / steps * 1e-3) / 1e12, 1)},
            "qat_backward_x": {"workload": "llama3_70b_mlp_qat_m4096 input gradient",
                               "transpose_pack": {"us_per_call": round(ms_t / steps * 1e3, 2),
                                                  "value": round(t_gbs, 1), "unit": "GB/s",
                                                  "roofline": {"bound": "hbm", "achieved": round(t_gbs, 1),
                                                               "peak": hbm_peak, "unit": "GB/s",
                                                               "frac": round(t_gbs / hbm_peak, 4)}},
                               "grad_x": {"ms_per_call": round(ms_g / steps, 4), "value": round(gx_tflops, 1),
                                          "unit": "TFLOP/s",
                                          "roofline": {"bound": "tensor", "achieved": round(gx_tflops, 1),
                                                       "peak": tf_peak, "unit": "TFLOP/s",
                                                       "frac": round(gx_tflops / tf_peak, 4)}}}}


def cpu_baseline(layers, batch, budget_s=12.0):
    """The float64 oracle on a bounded sample of the decode pass: whole passes over the
    layer set (signs precomputed, as the GPU step reads packed signs), repeated until about
    budget_s seconds, at least one pass."""
    import oracle
    threads = oracle.num_threads()
    pass_bytes = sum(2 * L["N"] * (((L["K"] + 127) // 128) * 128) // 8 for L in layers)
    passes, t_total = 0, 0.0
    while passes == 0 or t_total < budget_s:
        t0 = time.perf_counter()
        for L in layers:
            oracle.layer(L["S_cache"], L["a_host"], L["b_host"], L["x_host"], N=L["N"])
        t_total += time.perf_counter() - t0
        passes += 1
    return {"value": round(pass_bytes * passes / t_total / 1e9, 4), "unit": "GB/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{passes} full float64 oracle pass(es) over the {len(layers)} matrices of the "
                      f"layer set at batch {batch} ({t_total:.1f} s); signs derived beforehand"}


def prepare_oracle_inputs(layers, spec):
    import oracle
    oracle.build()
    for idx, L in enumerate(layers):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, L["N"], L["K"], sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
        a, b = inputs.scales(seed, W)
        L["a_host"], L["b_host"] = a, b
        L["S_cache"] = oracle.derive_signs(W, a, b)


def oracle_table(args):
    """The float64 oracle timed on every workload, on this host's cores (a CPU baseline
    only): derive + pack per matrix, the layer at every batch of the decode workloads, and
    for the GEMM workloads the layer on a sample of tokens, scaled to the full token count
    (the layer's cost is linear in the tokens) and labelled as such."""
    import oracle
    oracle.build()
    out = {"kind": "oracle", "cores": oracle.num_threads(), "host": "this host's CPU cores",
           "workloads": {}}
    for wname, spec in inputs.WORKLOADS.items():
        rows = []
        for idx, (name, N, K) in enumerate(spec["set"]):
            seed = inputs.seed_for(spec["cfg"], idx)
            W = inputs.weight(seed, N, K, sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
            a, b = inputs.scales(seed, W)
            t0 = time.perf_counter()
            S = oracle.derive_signs(W, a, b)
            oracle.pack(S)
            t_derive = time.perf_counter() - t0
            del W
            row = {"matrix": f"{name} {N}x{K}", "derive_pack_s": round(t_derive, 3)}
            gemm = max(spec["batches"]) > 16
            for B in spec["batches"]:
                Bs = min(B, args.gemm_token_sample) if gemm else B
                x = inputs.activations(seed, Bs, K, channel_outlier_frac=spec["x_outliers"])
                t0 = time.perf_counter()
                oracle.layer(S, a, b, x)
                t = time.perf_counter() - t0
                if gemm:
                    row[f"layer_m{B}_s"] = round(t * B / Bs, 4)
                    row["token_sample"] = Bs
                else:
                    row[f"layer_b{B}_us"] = round(t * 1e6, 1)
            rows.append(row)
            del S
        out["workloads"][wname] = rows
    print(json.dumps(out), flush=True)
    return 0


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The float64 CPU oracle as the reference arm: each step is a bounded sample of rows."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    spec = inputs.WORKLOADS[WORKLOAD]
    layers = []
    rows_cap = 256
    for idx, (name, N, K) in enumerate(spec["set"]):
        seed = inputs.seed_for(spec["cfg"], idx)
        W = inputs.weight(seed, N, K, sigma=spec["sigma"], outlier_frac=spec["w_outliers"])
        a, b = inputs.scales(seed, W)
        x = inputs.activations(seed, 1, K, channel_outlier_frac=spec["x_outliers"])
        S = oracle.derive_signs(W[:rows_cap], a, b)
        layers.append(dict(N=N, K=K, a=a, b=b, x=x, S=S))
    # size one step (rows per layer) so warmup + steps fit in about two minutes
    t0 = time.perf_counter()
    for L in layers:
        oracle.layer(L["S"][:, :8], L["a"], L["b"], L["x"], rows=np.arange(8), N=L["N"])
    per_row_set = (time.perf_counter() - t0) / 8
    total_steps = max(1, args.steps + args.warmup)
    rows = int(max(1, min(rows_cap, 120.0 / total_steps / max(per_row_set, 1e-9))))
    step_bytes = sum(2 * rows * (((L["K"] + 127) // 128) * 128) // 8 for L in layers)

    def step():
        for L in layers:
            oracle.layer(L["S"][:, :rows], L["a"], L["b"], L["x"], rows=np.arange(rows), N=L["N"])

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    elapsed = time.perf_counter() - t0
    value = step_bytes * args.steps / elapsed / 1e9
    cores = oracle.num_threads()
    sample = (f"float64 oracle output of {rows} row(s) of each of the 7 Llama-2-7B-shaped "
              f"matrices per step, batch 1")
    return {"metric": METRIC, "value": round(value, 6), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(elapsed / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": WORKLOAD, "batch": 1, "matrices": len(layers),
                       "rows_per_matrix_per_step": rows},
            "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ----------------------------------------------------------------------------- main
def main(argv=None):
    args = parse_args(argv)
    if args.oracle_table:
        return oracle_table(args)
    rank, world, local, dist = dist_init()
    try:
        if args.profile_kernel:
            return profile_kernel(args)
        if args.impl == "reference":
            line = run_reference(args, rank, world)
            if line is not None:
                print(json.dumps(line), flush=True)
            return 0
        return run_ours(args, rank, world, local, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


def run_ours(args, rank, world, local, dist):
    from bit_gemv_rabit_b200 import rabit
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl ours needs a CUDA device")
    rabit.load()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    hbm_peak, tf_peak, tf_sustained, peak_kind = peaks()
    spec = inputs.WORKLOADS[WORKLOAD]

    # ---- resident inputs: one seeded layer set, COPIES copies of its packed weights
    base = [make_layer(rabit, spec, idx, name, N, K, device, 1)
            for idx, (name, N, K) in enumerate(spec["set"])]
    sets = [base]
    for c in range(1, COPIES):
        sets.append([dict(L, packed=L["packed"].clone()) for L in base])
    torch.cuda.synchronize()
    step_bytes = decode_bytes(base)

    # One step: the seven matrices of the set as one rabit_gemv_grouped call (three kernels:
    # block maxima, digit images, the sign stream on the tensor cores).
    ws = rabit.alloc_gemv_grouped_workspace(layer_tuples(base), device=device)

    def step_fn(layers):
        def f():
            rabit.rabit_gemv_grouped(layer_tuples(layers), workspace=ws)
        return f

    graphs = [capture_graph(step_fn(ls)) for ls in sets]
    clocks = ClockSampler(device.index) if rank == 0 else None
    elapsed_ms = timed_replays(graphs, args.steps, args.warmup, dist, device, clocks)
    max_ms, total_units = aggregate(elapsed_ms, float(step_bytes) * args.steps, dist, device)
    value = total_units / (max_ms * 1e-3) / 1e9
    launches = 3 * args.steps
    per_call_us = elapsed_ms * 1e3 / args.steps
    achieved = step_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9
    # every bounded device wait of the timed region must have completed
    fault = rabit.rabit_read_fault(clear=True)

    # ---- end to end through the public API: pinned host x in, y back to the host, per step.
    # Each copy of the set keeps its seven x and seven y as views of one device buffer each,
    # so a step is one host-to-device copy, one prepared grouped call (rabit.GemvGroup, the
    # binding's marshalled rabit_gemv_grouped) and one device-to-host copy.
    e2e_steps = min(args.e2e_steps, args.steps)
    x_pinned = torch.from_numpy(np.concatenate([L["x_host"].view(np.int16).reshape(-1) for L in base])
                                ).view(torch.bfloat16).pin_memory()
    n_out = sum(L["N"] for L in base)
    y_pinned = torch.empty(n_out, dtype=torch.float32).pin_memory()
    h2d = x_pinned.numel() * x_pinned.element_size()
    d2h = y_pinned.numel() * y_pinned.element_size()
    e2e_sets = []
    for layers in sets:
        xd = torch.empty(x_pinned.numel(), dtype=torch.bfloat16, device=device)
        yd = torch.empty(n_out, dtype=torch.float32, device=device)
        tup, xo, yo = [], 0, 0
        for L in layers:
            tup.append((L["packed"], L["a"], L["b"], L["N"], L["K"], xd[xo:xo + L["K"]].view(1, L["K"]),
                        yd[yo:yo + L["N"]].view(1, L["N"])))
            xo += L["K"]
            yo += L["N"]
        e2e_sets.append((xd, yd, rabit.GemvGroup(tup, workspace=ws)))
    stream = torch.cuda.current_stream()

    def e2e_step(s):
        xd, yd, group = e2e_sets[s % COPIES]
        xd.copy_(x_pinned, non_blocking=True)
        group.run(stream)
        y_pinned.copy_(yd, non_blocking=True)
        stream.synchronize()

    for s in range(5):
        e2e_step(s)
    barrier(dist, device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for s in range(e2e_steps):
        e2e_step(s)
    e1.record()
    torch.cuda.synchronize()
    e2e_ms, e2e_units = aggregate(e0.elapsed_time(e1), float(step_bytes) * e2e_steps, dist, device)
    e2e_value = e2e_units / (e2e_ms * 1e-3) / 1e9
    fault |= rabit.rabit_read_fault(clear=True)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(max_ms / args.steps, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int16",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "batch": 1,
                   "matrices": [f"{L['name']} {L['N']}x{L['K']}" for L in base],
                   "weights": "2-path packed signs derived on the GPU from seeded fp32 W ~ N(0, 0.02^2)",
                   "l2": f"inputs larger than L2: {COPIES} resident copies of the layer set "
                         f"({COPIES * step_bytes / 1e6:.0f} MB) rotated per step",
                   "schedule": "the 7 matrices as one rabit_gemv_grouped call per step (independent GEMVs, "
                               "each with its own seeded x); per-matrix and decoder-order schedules in "
                               "decode_schedules",
                   "launch": "CUDA graph per copy, programmatic dependent launch between kernels",
                   "parallelism": f"replica x{world}"},
        # The metric's "% of peak": algorithmic bytes of the decode pass over the measured HBM
        # copy bandwidth, per call of the hot path (its three kernels, chained).
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "traffic": None,
                     "kernel": "gemv_tc_kernel (+ gemv_blockmax_kernel, gemv_prep_kernel)",
                     "avg_call_us": round(per_call_us, 3),
                     "peak_kind": f"{peak_kind} HBM copy bandwidth",
                     "achieved_kind": "algorithmic bytes (signs, scales, x, y) per call / average call time"},
        "gpu_launches": launches,
        "fault_word": fault,
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "api": "bit_gemv_rabit_b200.rabit.GemvGroup.run (a prepared rabit_gemv_grouped) over the "
                       "set; one pinned host-to-device copy of the seven x and one device-to-host copy "
                       "of the seven y per step, then a stream sync"},
    }
    if clocks is not None:
        line["clocks"] = clocks.summary()
    if rank == 0 and world == 1 and not args.no_secondary:
        line["us_per_launch_warm_l2_by_shape"] = warm_launch_us(rabit, base, device)
        sched = decode_schedules(rabit, sets, WORKLOAD, device)
        line["decode_schedules"] = {k: {"us_per_set": v, "GB_per_s": round(step_bytes / (v * 1e-6) / 1e9, 1),
                                        "hbm_frac": round(step_bytes / (v * 1e-6) / 1e9 / hbm_peak, 4)}
                                    for k, v in sched.items()}
    traffic = _load_traffic()
    if traffic is not None:
        line["roofline"]["traffic"] = traffic

    if rank == 0 and world == 1 and not args.no_secondary:
        del graphs
        torch.cuda.empty_cache()
        secondary(line, "gemm", lambda: bench_gemm(rabit, device, hbm_peak, tf_peak, tf_sustained))
        secondary(line, "qat_step", lambda: bench_qat_step(rabit, device, hbm_peak, tf_peak, tf_sustained),
                  merge=True)
        secondary(line, "gemv_3path", lambda: bench_gemv_three_path(rabit, device, hbm_peak))
        secondary(line, "scale_grads", lambda: bench_scale_grads(rabit, device, hbm_peak))
        secondary(line, "svid_init", lambda: bench_svid_init(rabit, device, hbm_peak))
        secondary(line, "decode_batch_sweep", lambda: bench_decode_sweep(rabit, device, hbm_peak))
    if rank == 0:
        # parity of the timed configuration: every output of the last timed step against the
        # float64 oracle (normwise, per matrix; the bar is 2e-3 for bf16 activations)
        prepare_oracle_inputs(base, spec)
        line["parity"] = timed_parity(base)
        if world == 1 and not args.no_secondary:
            line["cpu_baseline"] = cpu_baseline(base, 1)
        line["fault_word"] |= rabit.rabit_read_fault(clear=True)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if line["fault_word"] or not line.get("parity", {}).get("ok", True):
        return 1   # a bounded device wait expired, or the timed outputs are out of tolerance
    return 0


def timed_parity(layers, tol=2e-3):
    """Normwise error of each layer's y (from the last timed step) against the oracle."""
    import oracle
    errs = {}
    for L in layers:
        ref = oracle.layer(L["S_cache"], L["a_host"], L["b_host"], L["x_host"])
        y = L["y"].cpu().numpy().astype(np.float64)
        errs[L["name"]] = float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-300))
    worst = max(errs.values())
    return {"normwise_max": worst, "tol": tol, "ok": worst <= tol, "vs": "float64 oracle",
            "outputs": "every row of the 7 layers, last timed step", "by_matrix": errs}


def secondary(line, key, fn, merge=False):
    """Run one secondary measurement into the line.  A failure is recorded under `key` as an
    error string instead of ending the run, so the headline line is always printed."""
    try:
        out = fn()
        if merge:
            line.update(out)
        else:
            line[key] = out
    except Exception as exc:  # noqa: BLE001 -- any failure of a secondary figure
        line[key] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    if torch.cuda.is_available():
        torch.cuda.empty_cache()


def profile_kernel(args):
    """A few launches of one kernel on a seeded layer of the given shape (ncu target); with
    gemv_set, --launches grouped calls over the benchmark's decode layer set."""
    from bit_gemv_rabit_b200 import rabit
    rabit.load()
    device = torch.device("cuda", 0)
    if args.profile_kernel == "gemv_set":
        spec = inputs.WORKLOADS[WORKLOAD]
        layers = [make_layer(rabit, spec, idx, name, N, K, device, 1) for idx, (name, N, K) in enumerate(spec["set"])]
        ws = rabit.alloc_gemv_grouped_workspace(layer_tuples(layers), device=device)
        for _ in range(args.launches):
            rabit.rabit_gemv_grouped(layer_tuples(layers), workspace=ws)
        torch.cuda.synchronize()
        fault = rabit.rabit_read_fault()
        print(f"gemv_set {WORKLOAD} launches={args.launches} fault={fault}")
        return 0 if fault == 0 else 1
    N, K, M = args.shape
    spec = dict(cfg=9, sigma=0.02, w_outliers=0.0, x_outliers=0.0)
    L = make_layer(rabit, spec, 0, "layer", N, K, device, M)
    W = torch.from_numpy(inputs.weight(inputs.seed_for(9, 0), N, K)).to(device)
    ws = rabit.alloc_gemm_workspace(N, K, 2, M, device=device) if args.profile_kernel == "gemm" else None
    if args.profile_kernel == "scale_grads":
        # G = dL/dW_hat, seeded Gaussian (fp32, N x K); --launches calls
        G = torch.randn((N, K), generator=torch.Generator().manual_seed(inputs.seed_for(9, 1)),
                        dtype=torch.float32).to(device)
        ga, gb = torch.empty((2, N), device=device), torch.empty((2, K), device=device)
        ws = rabit.alloc_scale_grads_workspace(N, K, 2, device=device)
    if args.profile_kernel == "svid":
        # one initialisation: T = --launches iterations, 5 power steps per update
        s_in, s_out = inputs.calibration_stats(inputs.seed_for(9, 0), N, K)
        sws = rabit.alloc_svid_init_workspace(N, K, 2, device=device)
        rabit.rabit_svid_init(W, torch.from_numpy(s_in).to(device), torch.from_numpy(s_out).to(device),
                              SVID_ALPHA_IN, SVID_ALPHA_OUT, L["a"], L["b"], L["packed"], sws, P=2,
                              T=args.launches, power_iters=5)
    for _ in range(args.launches if args.profile_kernel != "svid" else 0):
        if args.profile_kernel == "derive":
            rabit.rabit_derive_pack(W, L["a"], L["b"], L["packed"])
        elif args.profile_kernel == "gemv":
            rabit.rabit_gemv(L["packed"], L["a"], L["b"], N, K, L["x"], L["y"], workspace=L["ws"])
        elif args.profile_kernel == "scale_grads":
            rabit.rabit_scale_grads(G, L["packed"], L["a"], L["b"], N, K, ga, gb, ws)
        else:
            rabit.rabit_gemm(L["packed"], L["a"], L["b"], N, K, L["x"], L["y"], ws)
    torch.cuda.synchronize()
    fault = rabit.rabit_read_fault()
    print(f"{args.profile_kernel} N={N} K={K} M={M} launches={args.launches} fault={fault}")
    return 0 if fault == 0 else 1


def _load_traffic():
    """DRAM bytes per decode launch of this workload from the committed ncu summary, or None
    when there is none or the kernel source changed since the counters were taken (the hash
    covers the kernel's own file and the device helpers it includes)."""
    import hashlib
    path = os.path.join(ROOT, "profiles", "gemv_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        if d.get("kernel_sha256") != kernel_source_sha256():
            return None
        return d.get("bytes_per_launch")
    except Exception:
        return None


def kernel_source_sha256():
    import hashlib
    h = hashlib.sha256()
    for rel in ("gemv_tc.cu", "rabit_device.cuh"):
        with open(os.path.join(ROOT, "bit_gemv_rabit_b200", "csrc", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


if __name__ == "__main__":
    sys.exit(main())
