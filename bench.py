#!/usr/bin/env python
"""Benchmark of the MoBiQuant token-routed mixed-bit linear layer on B200.

Metric: "mixed-bit GEMM: decode HBM GB/s & prefill TFLOP/s, % of B200 roofline".
Workload of the headline line: the decode GEMV workload — Llama-7B-shaped
projections (N, K) = (4096, 4096), (11008, 4096), (4096, 11008), each for
T = 1, 4 and 16 tokens (bf16 X ~ N(0,1), fp16 W ~ N(0, 0.02^2) with 0.5%
outlier input columns x10, 3 x 2-bit slices, group 128, router N(0, 1/K)).

One step = the per-token hot path over all nine (shape, T) cases: MoBiRoute
(routing + stable bucketing) and the mixed-bit GEMM that streams only the
slices the batch needs. Packing (MoBiSlice) is the one-time conversion of a
checkpoint; it is timed in the same run and reported under "pack".
value = decode algorithmic bytes of all ranks / max-over-ranks step time, with
decode bytes per GEMV = sum_{s <= k_max} (N*K/4 + N*(K/128)*4) + T*K*2.
Every call of a step reads its own packed copy, and a copy is reused only
after ~270 MB of other traffic, which exceeds twice the 126 MB L2.

--impl reference times the CPU oracle on the machine's host cores on a bounded
sample of the same workload (the only other place this file runs the oracle).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mixed-bit GEMM: decode HBM GB/s & prefill TFLOP/s, % of B200 roofline"
WORKLOAD = ("decode GEMV, Llama-7B projections (N,K) in {(4096,4096),(11008,4096),(4096,11008)} "
            "x T in {1,4,16}, 3x2-bit slices, group 128, route+bucket+GEMM per problem; the nine problems "
            "of a step as one mobi_linear_grouped call")


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


def decode_bytes(N, K, T, kmax, bits=2, widths=None):
    """Algorithmic bytes of one decode GEMM: k_max slices of codes (bits per
    weight, or widths[s] for slice s) and scale/zero words, plus X."""
    if widths is not None:
        return sum(N * K * int(w) // 8 + N * (K // 128) * 4 for w in widths[:kmax]) + T * K * 2
    return kmax * (N * K * bits // 8 + N * (K // 128) * 4) + T * K * 2


# DRAM bytes / algorithmic bytes of the decode step, from one ncu capture of
# each of the step's two decode launches (T <= 8 class: 147277056 read +
# 3972608 written; T = 16 class: 92629760 read + 3942912 written) against the
# step's 228773376 algorithmic bytes. Traffic grows in proportion to the bytes
# streamed, so the step's traffic is its algorithmic bytes times this ratio.
# Valid for the decode kernel as captured.
DECODE_DRAM_RATIO = (147277056 + 3972608 + 92629760 + 3942912) / 228773376


class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the timed region runs."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
        "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
        "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
    }

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop = period_s, threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML unavailable: report no clocks rather than guess
            self.nv = None

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            r = self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
            for name, bit in self.REASONS.items():
                if r & bit:
                    self.reasons.add(name)
        except Exception:
            pass

    def __enter__(self):
        if self.nv:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(v, world):
    """The largest of every rank's v (the slowest rank's time decides the job)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, ms_local, world):
    """(ms per step, whole-job units/s): every rank processes its own replica of
    the step, so the job moves world x units per step in the slowest rank's time."""
    ms = max_over_ranks(ms_local, world)
    return ms, world * units_per_rank_step / (ms * 1e-3)


# ---- the decode workload on the GPU ----------------------------------------------------

class DecodeCase:
    def __init__(self, mobi, wl, N, K, T, codes, sz, dev):
        L = wl.decode(N, K, T)
        self.N, self.K, self.T = N, K, T
        self.X = L.X.to(dev)
        self.X_host = L.X.pin_memory()
        self.Wr = torch.from_numpy(L.Wr).to(dev)
        self.codes, self.sz = codes, sz
        self.k_t = torch.empty(T, dtype=torch.int32, device=dev)
        self.perm = torch.empty(T, dtype=torch.int32, device=dev)
        self.off = torch.empty(4, dtype=torch.int32, device=dev)
        self.Y = torch.empty((T, N), dtype=torch.float32, device=dev)
        self.Y_host = torch.empty((T, N), dtype=torch.float32).pin_memory()
        self.ws_g = torch.empty(mobi.mobi_gemm_workspace_bytes(T, N, K, 3), dtype=torch.uint8, device=dev)
        self.ws_l = torch.empty(max(mobi.mobi_linear_workspace_bytes(T, N, K, 3), 16), dtype=torch.uint8, device=dev)
        self.mobi = mobi

    def gemm(self):
        self.mobi.mobi_gemm(self.X, self.k_t, self.perm, self.off, self.codes, self.sz, self.N, Y=self.Y, ws=self.ws_g)

    def step(self):
        """One layer call through the public API: routing + GEMM (mobi_linear)."""
        self.mobi.mobi_linear(self.X, self.Wr, None, self.codes, self.sz, self.N, Y=self.Y, k_t=self.k_t,
                              perm=self.perm, offsets=self.off, ws=self.ws_l)

    def kmax(self):
        return int(self.k_t.max().item())


def grouped_launches(group_T, group_K):
    """Library kernels of one mobi_linear_grouped call: one routing launch, one
    decode launch per fragment class present (T <= 8, T > 8) and one
    chunk-reduce launch when any problem's K spans more than one chunk."""
    classes = len({1 if T <= 8 else 2 for T in group_T})
    return 1 + classes + (1 if any(K > 1024 for K in group_K) else 0)


def time_graph(step, steps, warmup=3):
    """Capture step() in a CUDA graph and return the mean ms of `steps` replays."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    del graph
    return e0.elapsed_time(e1) / steps


def build_decode_cases(mobi, wl, dev):
    cases = []
    for (N, K) in wl.DECODE_SHAPES:
        L = wl.decode(N, K, 1)
        W = torch.from_numpy(L.W).to(dev)
        for T in wl.DECODE_TOKENS:  # one packed copy per call: rotation beyond L2
            codes, sz = mobi.mobi_pack(W, S=3)
            cases.append(DecodeCase(mobi, wl, N, K, T, codes, sz, dev))
        del W
    torch.cuda.synchronize()
    return cases


def time_pack(mobi, wl, dev, reps=10):
    N, K = 11008, 4096
    W = torch.from_numpy(wl.decode(N, K, 1).W).to(dev)
    codes = torch.empty((3, N, K // 16), dtype=torch.int32, device=dev)
    sz = torch.empty((3, K // 128, N), dtype=torch.int32, device=dev)
    for _ in range(3):
        mobi.mobi_pack(W, 3, codes=codes, sz=sz)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record()
    for _ in range(reps):
        mobi.mobi_pack(W, 3, codes=codes, sz=sz)
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / reps
    nbytes = N * K * 2 + codes.numel() * 4 + sz.numel() * 4
    return {"shape": [N, K], "ms": ms, "GB/s": nbytes / ms / 1e6, "bytes": nbytes,
            "weights_per_s": N * K / ms * 1e3}


def l2_flush_buffer(dev):
    return torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)


def time_full_model(mobi, wl, dev, steps, hbm_peak):
    """Full-model workload: pack the 7 projections x 32 layers of the Llama-2-7B-
    shaped stack (6.5e9 fp16 parameters drawn on the device), then time batch-8
    decode through every projection (224 mobi_linear calls per step, one CUDA
    graph). Returns pack and decode throughput."""
    projs = [(layer, p) for layer in range(wl.LLAMA7B_LAYERS) for p in range(len(wl.LLAMA7B_PROJECTIONS))]
    layers = [wl.full_model_projection(layer, p, T=8, device=dev) for layer, p in projs]
    packed = [(torch.empty((3, L.N, L.K // 16), dtype=torch.int32, device=dev),
               torch.empty((3, L.K // 128, L.N), dtype=torch.int32, device=dev)) for L in layers]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for L, (c, z) in zip(layers[:7], packed[:7]):  # warm-up
        mobi.mobi_pack(L.W, 3, codes=c, sz=z)
    torch.cuda.synchronize()
    e0.record()
    for L, (c, z) in zip(layers, packed):
        mobi.mobi_pack(L.W, 3, codes=c, sz=z)
    e1.record()
    torch.cuda.synchronize()
    pack_ms = e0.elapsed_time(e1)
    params = sum(L.N * L.K for L in layers)
    pack_bytes = sum(L.N * L.K * 2 + c.numel() * 4 + z.numel() * 4 for L, (c, z) in zip(layers, packed))
    dims = [(L.N, L.K) for L in layers]
    for L in layers:
        L.W = None  # free the fp16 stack (13 GB)
    torch.cuda.empty_cache()

    class Call:
        pass
    calls = []
    for L, (c, z), (N, K) in zip(layers, packed, dims):
        k = Call()
        k.X, k.Wr = L.X.to(dev), torch.from_numpy(L.Wr).to(dev)
        k.codes, k.sz, k.N, k.K = c, z, N, K
        k.Y = torch.empty((8, N), dtype=torch.float32, device=dev)
        k.k_t = torch.empty(8, dtype=torch.int32, device=dev)
        k.perm = torch.empty(8, dtype=torch.int32, device=dev)
        k.off = torch.empty(4, dtype=torch.int32, device=dev)
        k.ws = torch.empty(max(mobi.mobi_linear_workspace_bytes(8, N, K, 3), 16), dtype=torch.uint8, device=dev)
        calls.append(k)

    def step():
        for k in calls:
            mobi.mobi_linear(k.X, k.Wr, None, k.codes, k.sz, k.N, Y=k.Y, k_t=k.k_t, perm=k.perm, offsets=k.off,
                             ws=k.ws)
    step()
    torch.cuda.synchronize()
    kmax = [int(k.k_t.max().item()) for k in calls]
    bytes_step = sum(decode_bytes(k.N, k.K, 8, km) for k, km in zip(calls, kmax))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        step()
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for _ in range(3):
        graph.replay()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(steps):
        graph.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    mobi.mobi_sync_check()
    del graph

    # The same step with the seven projections of each layer in one
    # mobi_linear_grouped call (32 calls per step).
    per_layer = len(wl.LLAMA7B_PROJECTIONS)
    layer_probs = []
    for li in range(0, len(calls), per_layer):
        pr = [{"X": k.X, "Wr": k.Wr, "bias": None, "codes": k.codes, "sz": k.sz, "N": k.N, "Y": k.Y, "k_t": k.k_t,
               "perm": k.perm, "offsets": k.off} for k in calls[li:li + per_layer]]
        layer_probs.append(pr)
    gws = torch.empty(max(mobi.mobi_linear_grouped_workspace_bytes(layer_probs[0]), 16), dtype=torch.uint8,
                      device=dev)

    def gstep():
        for pr in layer_probs:  # the layers run one after another on one stream, so they share the scratch
            mobi.mobi_linear_grouped(pr, ws=gws)
    gstep()
    mobi.mobi_sync_check()
    gms = time_graph(gstep, steps)
    mobi.mobi_sync_check()

    # The grouping a real layer allows: q, k, v read the same attention input
    # and gate, up the same MLP input, while o reads the attention output and
    # down the activated MLP product, so a layer is four grouped calls
    # ({q,k,v}, {o}, {gate,up}, {down}; 128 calls per step).
    dep_groups = [(0, 1, 2), (3,), (4, 5), (6,)]
    dep_probs = [[pr[j] for j in g] for pr in layer_probs for g in dep_groups]

    def dstep():
        for pr in dep_probs:
            mobi.mobi_linear_grouped(pr, ws=gws)
    dstep()
    mobi.mobi_sync_check()
    dms = time_graph(dstep, steps)
    mobi.mobi_sync_check()
    out = {"workload": "full model: 7 projections x 32 layers (Llama-2-7B shapes), batch 8, random router per "
                       "projection; pack all, then decode through every projection (224 mobi_linear calls, one "
                       "CUDA graph)",
           "params": params, "pack_ms": round(pack_ms, 3), "pack_GB/s": round(pack_bytes / pack_ms / 1e6, 1),
           "decode_ms_per_step": round(ms, 4), "decode_bytes_per_step": bytes_step,
           "decode_GB/s": round(bytes_step / ms / 1e6, 1), "decode_frac_of_hbm": round(bytes_step / ms / 1e6 / hbm_peak, 4),
           "kmax_histogram": [kmax.count(v) for v in (1, 2, 3)], "steps": steps,
           "grouped_per_layer": {"calls_per_step": len(layer_probs), "decode_ms_per_step": round(gms, 4),
                                 "decode_GB/s": round(bytes_step / gms / 1e6, 1),
                                 "decode_frac_of_hbm": round(bytes_step / gms / 1e6 / hbm_peak, 4),
                                 "note": "all seven projections of a layer in one call: an upper bound, since "
                                         "o and down depend on the others' outputs in a real layer"},
           "grouped_by_dependency": {"groups_per_layer": "{q,k,v}, {o}, {gate,up}, {down}",
                                     "calls_per_step": len(dep_probs), "decode_ms_per_step": round(dms, 4),
                                     "decode_GB/s": round(bytes_step / dms / 1e6, 1),
                                     "decode_frac_of_hbm": round(bytes_step / dms / 1e6 / hbm_peak, 4)}}
    del calls, packed, layers, layer_probs, dep_probs
    torch.cuda.empty_cache()
    return out


def time_prefill(mobi, L, dev, reps, tf_peak, flush):
    """Route + bucket + tcgen05 prefill GEMM on one prefill workload; CUDA events
    per repetition with the L2 flushed (256 MB write) before each one."""
    W = torch.from_numpy(L.W).to(dev)
    codes, sz = mobi.mobi_pack(W, S=3)
    del W
    X = L.X.to(dev)
    Wr = torch.from_numpy(L.Wr).to(dev)
    b = None if L.bias is None else torch.from_numpy(L.bias).to(dev)
    T, N, K = L.T, L.N, L.K
    k_t = torch.empty(T, dtype=torch.int32, device=dev)
    perm = torch.empty(T, dtype=torch.int32, device=dev)
    off = torch.empty(4, dtype=torch.int32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws_r = torch.empty(max(mobi.mobi_route_workspace_bytes(T, K, 3), 16), dtype=torch.uint8, device=dev)
    ws_g = torch.empty(mobi.mobi_gemm_workspace_bytes(T, N, K, 3), dtype=torch.uint8, device=dev)

    def route():
        mobi.mobi_route(X, Wr, b, k_t, perm, off, ws_r)

    def gemm():
        mobi.mobi_gemm(X, k_t, perm, off, codes, sz, N, Y=Y, ws=ws_g)
    for _ in range(3):
        route()
        gemm()
    mobi.mobi_sync_check()
    sumk = int(k_t.sum().item())
    counts = torch.bincount(k_t, minlength=4)[1:].tolist()
    t_route, t_gemm = [], []
    e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for _ in range(reps):
        flush.fill_(1.0)
        e[0].record()
        route()
        e[1].record()
        gemm()
        e[2].record()
        torch.cuda.synchronize()
        t_route.append(e[0].elapsed_time(e[1]))
        t_gemm.append(e[1].elapsed_time(e[2]))
    mobi.mobi_sync_check()
    ms_gemm = statistics.median(t_gemm)
    ms_step = statistics.median([a + b2 for a, b2 in zip(t_route, t_gemm)])
    issued = 2.0 * N * K * sumk
    eff = 2.0 * T * N * K
    return {"workload": L.name, "T": T, "N": N, "K": K, "k_counts": counts, "sum_k": sumk,
            "ms_step": round(ms_step, 4), "ms_gemm": round(ms_gemm, 4), "ms_route": round(statistics.median(t_route), 4),
            "tflops_issued": round(issued / ms_gemm / 1e9, 2), "tflops_effective": round(eff / ms_gemm / 1e9, 2),
            "tflops_issued_step": round(issued / ms_step / 1e9, 2),
            "roofline": {"bound": "tensor", "kernel": "prefill GEMM (gather + tcgen05 prefill kernels)",
                         "achieved": round(issued / ms_gemm / 1e9, 2), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(issued / ms_gemm / 1e9 / tf_peak, 4),
                         "traffic": PREFILL_DRAM_BYTES.get(L.name),
                         "traffic_unit": "bytes per prefill_kernel launch (ncu DRAM read + write)"},
            "reps": reps, "l2": "256 MB flush before each repetition"}


# DRAM bytes (read + write) of one prefill_kernel launch, from one ncu capture
# (dram__bytes_read.sum + dram__bytes_write.sum) of the 11008 x 4096, T = 2048
# workload. The 28672 x 8192 workload has no capture of the current kernel
# (its traffic is reported as null). Valid while the prefill kernel is unchanged.
PREFILL_DRAM_BYTES = {"prefill_11008x4096_T2048": 60248576 + 45078784}


# fp32 FMA peak of the SIMT pipes: 148 SMs x 128 fp32 lanes x 2 FLOP x 1965 MHz
# (the maximum SM clock), the bound of the MLP scorer's hidden layer at prefill.
FP32_SIMT_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def time_route_mlp(mobi, wl, dev, hbm_peak, flush, reps=20):
    """Threshold routing with the MLP scorer (hidden layer, scores, bucketing),
    K=4096, H=128, S=3, at decode (T=16: bound by the W1 read) and prefill
    (T=2048: bound by the fp32 FMAs of the hidden layer). CUDA events around
    each call with the L2 flushed before it; the linear router of the same
    tokens is timed the same way for comparison."""
    out = {}
    for R in (wl.mlp_route_decode(16), wl.mlp_route_prefill()):
        T, K, H = R.T, R.K, R.H
        X = R.X.to(dev)
        W1, b1 = torch.from_numpy(R.W1).to(dev), torch.from_numpy(R.b1).to(dev)
        W2, b2 = torch.from_numpy(R.W2).to(dev), torch.from_numpy(R.b2).to(dev)
        k_t = torch.empty(T, dtype=torch.int32, device=dev)
        perm = torch.empty(T, dtype=torch.int32, device=dev)
        off = torch.empty(4, dtype=torch.int32, device=dev)
        ws = torch.empty(max(mobi.mobi_route_mlp_workspace_bytes(T, K, H), 16), dtype=torch.uint8, device=dev)
        Wr = torch.from_numpy(wl.draw_router(np.random.default_rng(1), K, 3)).to(dev)
        ws_r = torch.empty(max(mobi.mobi_route_workspace_bytes(T, K, 3), 16), dtype=torch.uint8, device=dev)

        def mlp():
            mobi.mobi_route_mlp(X, W1, b1, W2, b2, 1.0, 0.5, k_t=k_t, perm=perm, offsets=off, ws=ws)

        def lin():
            mobi.mobi_route(X, Wr, None, k_t, perm, off, ws_r)
        times = {}
        for name, fn in (("mlp", mlp), ("linear", lin)):
            for _ in range(3):
                fn()
            torch.cuda.synchronize()
            ts = []
            for _ in range(reps):
                flush.sum()  # a read sweep: evicts the inputs without leaving dirty lines to write back
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                fn()
                e1.record()
                torch.cuda.synchronize()
                ts.append(e0.elapsed_time(e1))
            times[name] = statistics.median(ts)
        mlp()
        mobi.mobi_sync_check()
        counts = torch.bincount(k_t, minlength=4)[1:].tolist()
        ms = times["mlp"]
        nbytes = T * K * 2 + K * H * 4 + H * 2 * 4 + T * 4 * 3
        flops = 2.0 * T * K * H + 2.0 * T * H * 2
        r = {"T": T, "K": K, "H": H, "S": 3, "tau": 1.0, "delta": 0.5, "k_counts": counts,
             "us_per_call": round(1e3 * ms, 2), "linear_router_us_per_call": round(1e3 * times["linear"], 2),
             "algorithmic_bytes": nbytes, "flops": flops}
        if T <= 16:
            r["roofline"] = {"bound": "hbm", "achieved": round(nbytes / ms / 1e6, 1), "peak": hbm_peak, "unit": "GB/s",
                             "frac": round(nbytes / ms / 1e6 / hbm_peak, 4), "traffic": None}
        else:
            tf = flops / ms / 1e9
            r["roofline"] = {"bound": "alu", "achieved": round(tf, 2), "peak": round(FP32_SIMT_PEAK_TFLOPS, 1),
                             "unit": "TFLOP/s", "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 x 1965 MHz",
                             "frac": round(tf / FP32_SIMT_PEAK_TFLOPS, 4), "traffic": None}
        out[R.name] = r
        del ws, ws_r
    out["timing"] = f"median of {reps} calls, CUDA events, L2 flushed (256 MB read) before each"
    return out


def time_ckpt(mobi, wl, dev, reps=3):
    """Many-in-one checkpoint I/O: the seven packed projections of one
    Llama-2-7B-shaped layer saved from HBM to one file, then loaded back into
    HBM at 1, 2 and 3 slices (2, 4, 6 bits; each load reads only its slices).
    Host wall time of the calls (each returns once the data is on the device);
    the file was just written, so reads come from the OS page cache."""
    import tempfile
    import time
    tensors = []
    for p in range(len(wl.LLAMA7B_PROJECTIONS)):
        L = wl.full_model_projection(0, p, T=1, device=dev)
        codes, sz = mobi.mobi_pack(L.W, S=3)
        tensors.append((f"layers.0.{wl.LLAMA7B_PROJECTIONS[p][0]}", codes, sz))
        del L
    torch.cuda.synchronize()
    total = sum(c.numel() * 4 + z.numel() * 4 for _, c, z in tensors)
    d = tempfile.mkdtemp(prefix="mobi_ckpt_")
    path = os.path.join(d, "layer0.mobi")
    out = {"workload": "7 packed projections of one Llama-2-7B layer (3 slices) in one checkpoint file",
           "file_bytes_3_slices": total}
    try:
        t_save = []
        for _ in range(reps):
            t0 = time.perf_counter()
            mobi.mobi_ckpt_save(path, tensors)
            t_save.append(time.perf_counter() - t0)
        out["save_GB/s"] = round(total / statistics.median(t_save) / 1e9, 2)
        bufs = [(torch.empty_like(c), torch.empty_like(z)) for _, c, z in tensors]
        with mobi.MobiCheckpoint(path) as ck:
            for k in (1, 2, 3):
                times = []
                for _ in range(reps):
                    r0 = ck.bytes_read
                    t0 = time.perf_counter()
                    for (name, c, z), (bc, bz) in zip(tensors, bufs):
                        ck.load(name, k, device=dev, codes=bc[:k], sz=bz[:k])
                    times.append(time.perf_counter() - t0)
                    nread = ck.bytes_read - r0
                for (name, c, z), (bc, bz) in zip(tensors, bufs):
                    assert torch.equal(bc[:k], c[:k]) and torch.equal(bz[:k], z[:k])
                out[f"load_{2 * k}bit"] = {"bytes_read": nread, "ms": round(1e3 * statistics.median(times), 2),
                                           "GB/s": round(nread / statistics.median(times) / 1e9, 2)}
    finally:
        if os.path.exists(path):
            os.remove(path)
        os.rmdir(d)
    out["timing"] = f"median of {reps}, host wall clock, CRC-32C verified on load"
    return out


def time_generic(mobi, wl, dev, hbm_peak, tf_peak, flush, steps=200):
    """Generic slicing: four 1-bit slices (1..4 bits per weight), G = 128, the
    codes stored at 1 bit per weight. (a) the decode step of the three
    Llama-7B shapes at T = 4 as one mobi_linear_grouped call, router mix 1/4
    each (five packed copies in rotation, so no copy is L2-resident when it is
    read again), beside the same step with four 2-bit slices (same k_max, twice
    the code bytes) and with slices of widths (2, 1, 1, 2) (2, 3, 4, 6 bits);
    (b) the prefill workload's shape (T = 2048, 11008 x 4096) through route +
    prefill GEMM."""
    S = 4
    out = {"slicing": "4 x 1-bit slices, G = 128, codes at 1 bit per weight (32 per word)"}
    # Five packed copies of the three problems, run one after another in each
    # step, so a copy is read again only after 4 x its bytes of other weights
    # (above 200 MB at 1 bit per weight, more than the 126 MB L2).
    copies = 5
    for bits in (1, 2, "mixed"):
        widths = (2, 1, 1, 2) if bits == "mixed" else None
        groups = []
        for r in range(copies):
            probs = []
            for i, (N, K) in enumerate(wl.DECODE_SHAPES):
                L = wl.layer(f"gen_{N}x{K}", N, K, 4, seed=3000 + i, outlier_frac_cols=0.005, S=S, mix=(0.25,) * S)
                codes, sz = (mobi.mobi_pack(torch.from_numpy(L.W).to(dev), widths=widths) if widths else
                             mobi.mobi_pack(torch.from_numpy(L.W).to(dev), S=S, bits=bits))
                probs.append({"X": L.X.to(dev), "Wr": torch.from_numpy(L.Wr).to(dev),
                              "bias": torch.from_numpy(L.bias).to(dev), "codes": codes, "sz": sz, "N": N,
                              "Y": torch.empty((4, N), dtype=torch.float32, device=dev),
                              "k_t": torch.empty(4, dtype=torch.int32, device=dev),
                              "perm": torch.empty(4, dtype=torch.int32, device=dev),
                              "offsets": torch.empty(S + 1, dtype=torch.int32, device=dev)})
            groups.append(probs)
        ws = torch.empty(max(mobi.mobi_linear_grouped_workspace_bytes(groups[0], S=S), 16), dtype=torch.uint8,
                         device=dev)

        def step():
            for probs in groups:
                if widths:
                    mobi.mobi_linear_grouped(probs, S=S, ws=ws, widths=widths)
                else:
                    mobi.mobi_linear_grouped(probs, S=S, ws=ws, bits=bits)
        step()
        mobi.mobi_sync_check()
        kmax = [int(p["k_t"].max().item()) for p in groups[0]]
        nbytes = sum(decode_bytes(p["N"], p["X"].shape[1], 4, km, 2 if widths else bits, widths)
                     for p, km in zip(groups[0], kmax))
        ms = time_graph(step, steps) / copies
        key = {1: "decode_T4_grouped", 2: "decode_T4_grouped_2bit_slices"}.get(bits, "decode_T4_grouped_widths_2_1_1_2")
        prec = [sum(widths[:km]) if widths else bits * km for km in kmax]
        out[key] = {"kmax_per_problem": kmax, "bytes_per_call": nbytes, "ms_per_call": round(ms, 5),
                    "GB/s": round(nbytes / ms / 1e6, 1), "frac_of_hbm": round(nbytes / ms / 1e6 / hbm_peak, 4),
                    "precision_bits_per_weight": prec,
                    "code_bits_read_per_weight": prec,
                    "l2": f"{copies} packed copies in rotation, each read again after ~{(copies - 1) * nbytes / 1e6:.0f} MB"}
        del groups, ws
    L = wl.layer("gen_prefill_11008x4096_T2048", 11008, 4096, 2048, seed=3010, n_outlier_cols=20, S=S,
                 mix=(0.25,) * S)
    W = torch.from_numpy(L.W).to(dev)
    codes, sz = mobi.mobi_pack(W, S=S, bits=1)
    del W
    assert codes.numel() * 4 == mobi.mobi_codes_bytes(11008, 4096, S, bits=1)
    X = L.X.to(dev)
    Wr = torch.from_numpy(L.Wr).to(dev)
    b = torch.from_numpy(L.bias).to(dev)
    T, N, K = L.T, L.N, L.K
    k_t = torch.empty(T, dtype=torch.int32, device=dev)
    perm = torch.empty(T, dtype=torch.int32, device=dev)
    off = torch.empty(S + 1, dtype=torch.int32, device=dev)
    Y = torch.empty((T, N), dtype=torch.float32, device=dev)
    ws_r = torch.empty(max(mobi.mobi_route_workspace_bytes(T, K, S), 16), dtype=torch.uint8, device=dev)
    ws_g = torch.empty(mobi.mobi_gemm_workspace_bytes(T, N, K, S), dtype=torch.uint8, device=dev)
    mobi.mobi_route(X, Wr, b, k_t, perm, off, ws_r)
    for _ in range(3):
        mobi.mobi_gemm(X, k_t, perm, off, codes, sz, N, Y=Y, ws=ws_g, bits=1)
    mobi.mobi_sync_check()
    sumk = int(k_t.sum().item())
    ts = []
    for _ in range(10):
        flush.fill_(1.0)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        mobi.mobi_gemm(X, k_t, perm, off, codes, sz, N, Y=Y, ws=ws_g, bits=1)
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    ms = statistics.median(ts)
    issued = 2.0 * N * K * sumk
    out["prefill_T2048"] = {"k_counts": torch.bincount(k_t, minlength=S + 1)[1:].tolist(), "sum_k": sumk,
                            "ms_gemm": round(ms, 4), "tflops_issued": round(issued / ms / 1e9, 2),
                            "frac_of_bf16_peak": round(issued / ms / 1e9 / tf_peak, 4),
                            "tflops_effective": round(2.0 * T * N * K / ms / 1e9, 2)}
    return out


def run_gpu(args, world, rank):
    import token_adaptive_mixed_b200 as mobi
    from token_adaptive_mixed_b200 import build as mobi_build
    from token_adaptive_mixed_b200 import workloads as wl

    if rank == 0:
        mobi_build.build()
    barrier(world)
    mobi.lib()
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm_peak, tf_peak, tf_sust, peak_kind = peaks()

    if args.only == "route_mlp":
        return {"route_mlp": time_route_mlp(mobi, wl, dev, hbm_peak, l2_flush_buffer(dev))}
    if args.only == "ckpt":
        return {"ckpt": time_ckpt(mobi, wl, dev)}
    if args.only == "generic":
        return {"generic_slicing": time_generic(mobi, wl, dev, hbm_peak, tf_peak, l2_flush_buffer(dev))}
    if args.only == "prefill":
        flush = l2_flush_buffer(dev)
        out = {"prefill": time_prefill(mobi, wl.prefill(), dev, args.prefill_reps, tf_peak, flush)}
        if not args.skip_skewed:
            out["skewed_prefill"] = time_prefill(mobi, wl.skewed_prefill(), dev, args.prefill_reps, tf_peak, flush)
        return out
    cases = build_decode_cases(mobi, wl, dev)
    for c in cases:
        c.step()
    mobi.mobi_sync_check()
    kmax = [c.kmax() for c in cases]
    bytes_step = sum(decode_bytes(c.N, c.K, c.T, km) for c, km in zip(cases, kmax))

    # One step = the nine decode problems through the public API as one
    # mobi_linear_grouped call (one routing launch, one decode launch per
    # fragment class, one chunk reduction), captured in one CUDA graph.
    groups = [cases]
    probs = [[{"X": c.X, "Wr": c.Wr, "bias": None, "codes": c.codes, "sz": c.sz, "N": c.N, "Y": c.Y,
               "k_t": c.k_t, "perm": c.perm, "offsets": c.off} for c in g] for g in groups]
    gws = [torch.empty(max(mobi.mobi_linear_grouped_workspace_bytes(pr), 16), dtype=torch.uint8, device=dev)
           for pr in probs]

    def grouped_step():
        for pr, w in zip(probs, gws):
            mobi.mobi_linear_grouped(pr, ws=w)
    grouped_step()
    mobi.mobi_sync_check()
    launches_per_step = sum(grouped_launches([c.T for c in g], [c.K for c in g]) for g in groups)

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        for _ in range(2):
            grouped_step()
    torch.cuda.current_stream().wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        grouped_step()

    for _ in range(max(args.warmup, 3)):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        e0.record()
        for _ in range(args.steps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms_local = e0.elapsed_time(e1) / args.steps
    ms, rate = whole_job_rate(bytes_step, ms_local, world)
    value = rate / 1e9
    mobi.mobi_sync_check()
    del graph

    # The same nine problems as nine mobi_linear calls (one per problem).
    steps_cmp = min(args.steps, 500)

    def linear_step():
        for c in cases:
            c.step()
    ms_linear = time_graph(linear_step, steps_cmp)

    # Roofline of the dominant kernels (decode GEMM + chunk reduction): the
    # step's grouped GEMM alone (mobi_gemm_grouped, k_t from the routing
    # above), as one CUDA graph.
    gprobs = [[{"X": c.X, "k_t": c.k_t, "codes": c.codes, "sz": c.sz, "N": c.N, "Y": c.Y} for c in g]
              for g in groups]

    def gemm_step():
        for pr, w in zip(gprobs, gws):
            mobi.mobi_gemm_grouped(pr, ws=w)
    ms_gemm = time_graph(gemm_step, steps_cmp)
    mobi.mobi_sync_check()
    achieved = bytes_step / (ms_gemm * 1e-3) / 1e9

    def gemm_calls_step():
        for c in cases:
            c.gemm()
    ms_gemm_calls = time_graph(gemm_calls_step, steps_cmp)

    # End to end through the public API with host buffers (pinned), copies inside
    # every step: the step's nine activation matrices go in as one host-to-device
    # copy from a pinned buffer, the grouped call runs, the nine outputs come
    # back as one device-to-host copy. As a serving loop runs it, the copies
    # have their own streams and the device buffers are doubled, so the input
    # copy of step i+1 and the output copy of step i-1 overlap the compute of
    # step i; the same loop with everything on one stream is reported beside.
    h2d = sum(c.T * c.K * 2 for c in cases)
    d2h = sum(c.T * c.N * 4 for c in cases)
    e2e_steps = max(3, min(args.steps, 200))
    X_host = torch.empty(h2d // 2, dtype=torch.bfloat16).pin_memory()
    Y_host = [torch.empty(d2h // 4, dtype=torch.float32).pin_memory() for _ in range(2)]
    X_dev = [torch.empty(h2d // 2, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    Y_dev = [torch.empty(d2h // 4, dtype=torch.float32, device=dev) for _ in range(2)]
    xo = 0
    for c in cases:
        X_host[xo:xo + c.T * c.K].copy_(c.X_host.reshape(-1))
        xo += c.T * c.K
    bufs = []
    for bi in range(2):
        xo = yo = 0
        views = {}
        for ci, c in enumerate(cases):
            views[ci] = (X_dev[bi][xo:xo + c.T * c.K].view(c.T, c.K), Y_dev[bi][yo:yo + c.T * c.N].view(c.T, c.N))
            xo += c.T * c.K
            yo += c.T * c.N
        bufs.append([[dict(pr, X=views[cases.index(c)][0], Y=views[cases.index(c)][1]) for pr, c in zip(prs, g)]
                     for prs, g in zip(probs, groups)])
    s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_pipelined(nsteps):
        for i in range(nsteps):
            bi = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[bi])  # the compute of step i-2 has read X_dev[bi]
                X_dev[bi].copy_(X_host, non_blocking=True)
                ev_in[bi].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(ev_in[bi])
                if i >= 2:
                    s_cmp.wait_event(ev_out[bi])  # Y_dev[bi] of step i-2 is on the host
                for pr, w in zip(bufs[bi], gws):
                    mobi.mobi_linear_grouped(pr, ws=w, stream=s_cmp)
                ev_cmp[bi].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[bi])
                Y_host[bi].copy_(Y_dev[bi], non_blocking=True)
                ev_out[bi].record(s_out)

    def e2e_serial(nsteps):
        for _ in range(nsteps):
            X_dev[0].copy_(X_host, non_blocking=True)
            for pr, w in zip(bufs[0], gws):
                mobi.mobi_linear_grouped(pr, ws=w)
            Y_host[0].copy_(Y_dev[0], non_blocking=True)

    e2e_pipelined(4)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(s_in)
    e2e_pipelined(e2e_steps)
    t1.record(s_out)
    torch.cuda.synchronize()
    eager_ms, eager_rate = whole_job_rate(bytes_step, t0.elapsed_time(t1) / e2e_steps, world)
    mobi.mobi_sync_check()
    # As a serving loop runs it: the same pipelined steps (copies on their own
    # streams, device buffers doubled) captured as one CUDA graph of 8 steps and
    # replayed, so the host issues one launch per 8 steps; every step still
    # copies its inputs in from pinned memory and its outputs back.
    per_graph = 8
    cap = torch.cuda.Stream()
    cap.wait_stream(torch.cuda.current_stream())
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e, stream=cap):
        s_in.wait_stream(cap)
        s_cmp.wait_stream(cap)
        s_out.wait_stream(cap)
        e2e_pipelined(per_graph)
        cap.wait_stream(s_in)
        cap.wait_stream(s_cmp)
        cap.wait_stream(s_out)
    torch.cuda.synchronize()
    for _ in range(2):
        g_e2e.replay()
    torch.cuda.synchronize()
    reps = max(1, e2e_steps // per_graph)
    t0.record()
    for _ in range(reps):
        g_e2e.replay()
    t1.record()
    torch.cuda.synchronize()
    e2e_ms, e2e_rate = whole_job_rate(bytes_step, t0.elapsed_time(t1) / (reps * per_graph), world)
    e2e_value = e2e_rate / 1e9
    mobi.mobi_sync_check()
    del g_e2e
    e2e_serial(3)
    torch.cuda.synchronize()
    e0.record()
    e2e_serial(e2e_steps)
    e1.record()
    torch.cuda.synchronize()
    serial_ms, serial_rate = whole_job_rate(bytes_step, e0.elapsed_time(e1) / e2e_steps, world)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "bytes_per_step": bytes_step, "kmax_per_call": kmax,
                   "l2": "rotating packed copies, ~270 MB between reuses (> 2x L2)",
                   "timing": "CUDA graph of one step, CUDA events, max over ranks", "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "kernel": "decode GEMM (stream-K mma.sync decode kernel per fragment class "
                                              "+ chunk reduction): the step's mobi_gemm_grouped call as one "
                                              "CUDA graph",
                     "achieved": round(achieved, 2), "peak": hbm_peak, "peak_kind": peak_kind, "unit": "GB/s",
                     "frac": round(achieved / hbm_peak, 4), "frac_of_8TBs_nominal": round(achieved / 8000.0, 4),
                     "traffic": round(bytes_step * DECODE_DRAM_RATIO),
                     "traffic_unit": "bytes per step (ncu DRAM bytes / algorithmic bytes x algorithmic bytes)",
                     "gemm_ms_per_step": round(ms_gemm, 5),
                     "gemm_ms_per_step_nine_calls": round(ms_gemm_calls, 5)},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms, 4),
                "copies": "pinned host buffers; input copy of step i+1 and output copy of step i-1 overlap the "
                          "compute of step i (separate streams, double-buffered device X and Y); 8 such steps "
                          "captured as one CUDA graph and replayed",
                "eager": {"value": round(eager_rate / 1e9, 2), "ms_per_step": round(eager_ms, 4),
                          "copies": "the same pipelined steps issued from Python one by one (host-bound)"},
                "serial": {"value": round(serial_rate / 1e9, 2), "ms_per_step": round(serial_ms, 4),
                           "copies": "one stream, issued from Python: copy in, compute, copy out, step after step"}},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk.summary(),
        "per_problem_calls": {"workload": "the same step as nine mobi_linear calls, one per problem (27 launches)",
                              "ms_per_step": round(ms_linear, 5), "GB/s": round(bytes_step / ms_linear / 1e6, 1),
                              "frac_of_hbm": round(bytes_step / ms_linear / 1e6 / hbm_peak, 4)},
    }
    if rank == 0:
        out["pack"] = time_pack(mobi, wl, dev)
    del cases
    torch.cuda.empty_cache()
    if args.only == "all" and not args.skip_full_model:
        out["full_model"] = time_full_model(mobi, wl, dev, 20, hbm_peak)
    if args.only != "decode":
        torch.cuda.empty_cache()
        flush = l2_flush_buffer(dev)
        out["prefill"] = time_prefill(mobi, wl.prefill(), dev, args.prefill_reps, tf_peak, flush)
        if not args.skip_skewed:
            out["skewed_prefill"] = time_prefill(mobi, wl.skewed_prefill(), dev, args.prefill_reps, tf_peak, flush)
    if args.only == "all" and rank == 0:
        out["route_mlp"] = time_route_mlp(mobi, wl, dev, hbm_peak, l2_flush_buffer(dev))
        out["ckpt"] = time_ckpt(mobi, wl, dev)
        out["generic_slicing"] = time_generic(mobi, wl, dev, hbm_peak, tf_peak, l2_flush_buffer(dev))
    return out


# ---- the oracle on the host cores ------------------------------------------------------

_ORACLE_CASES = {}


def _oracle_case(N, K, T, rows):
    """Inputs of one decode case for the oracle (cached: drawing W is not timed)."""
    import oracle
    from token_adaptive_mixed_b200 import workloads as wl
    key = (N, K, T, rows)
    if key not in _ORACLE_CASES:
        L = wl.decode(N, K, T)
        c_sub, s_sub, _ = oracle.pack(np.ascontiguousarray(L.W[:rows]), S=3)
        _ORACLE_CASES[key] = (L.X, L.Wr, c_sub, s_sub)
    return _ORACLE_CASES[key]


def oracle_decode_sample(budget_s: float, cases_spec, rows_cap=None, nthreads=0):
    """Time the CPU oracle (route + GEMM) on a bounded sample of the decode workload:
    every listed case once, then further passes until `budget_s` of CPU time.
    Returns (bytes credited, seconds, threads, description)."""
    import oracle
    nthreads = nthreads or len(os.sched_getaffinity(0))
    threads = nthreads
    credited, spent, done = 0, 0.0, []
    i = 0
    while i < len(cases_spec) or spent < budget_s:
        N, K, T = cases_spec[i % len(cases_spec)]
        i += 1
        rows = N if rows_cap is None else min(N, rows_cap)
        X, Wr, c_sub, s_sub = _oracle_case(N, K, T, rows)
        t0 = time.perf_counter()
        k, _, _ = oracle.route(X, Wr, nthreads=nthreads)
        oracle.gemm(X, k, c_sub, s_sub, rows, nthreads=nthreads)
        dt = time.perf_counter() - t0
        km = int(k.max())
        credited += km * (rows * K // 4 + rows * (K // 128) * 4) + T * K * 2
        spent += dt
        done.append(f"{rows}/{N}x{K} T={T}")
    return credited, spent, threads, "; ".join(done)


def _timed(fn):
    t0 = time.perf_counter()
    r = fn()
    return r, time.perf_counter() - t0


def cpu_baseline(budget_s=20.0):
    """The oracle on the host cores, following the measurement protocol: all
    threads (OpenMP over output rows; each output's reduction order unchanged)
    on configs 1-3 in full, config 4 on one layer of the stack (pack + batch-8
    decode of its seven projections, extrapolated x32), config 5 packed in full
    with its GEMM on a stated token subset (extrapolated to T = 4096); then one
    thread on a bounded sample. `value` is the decode workload's rate (config 2,
    all threads) in the headline unit."""
    import oracle
    from token_adaptive_mixed_b200 import workloads as wl
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    nt = cores
    proto = {"threads_all": cores}

    def gemm_rate(macs, sec):
        return round(2.0 * macs / sec / 1e9, 3)  # GFLOP/s (fp64)

    # config 1: pack + route + GEMM, T = 16
    L = wl.tiny()
    (c, z, _), tp = _timed(lambda: oracle.pack(L.W, S=3, nthreads=nt))
    (k, _, _), tr = _timed(lambda: oracle.route(L.X, L.Wr, nthreads=nt))
    _, tg = _timed(lambda: oracle.gemm(L.X, k, c, z, L.N, nthreads=nt))
    proto["config1_tiny"] = {"s": round(tp + tr + tg, 4), "pack_s": round(tp, 4), "route_s": round(tr, 4),
                             "gemm_s": round(tg, 4)}
    # config 2: the nine decode problems (route + GEMM), packs timed apart
    dec_bytes, dec_s, pack_s = 0, 0.0, 0.0
    for (N, K) in wl.DECODE_SHAPES:
        L1 = wl.decode(N, K, 1)
        (c, z, _), tp = _timed(lambda: oracle.pack(L1.W, S=3, nthreads=nt))
        pack_s += tp
        for T in wl.DECODE_TOKENS:
            L = wl.decode(N, K, T)
            def run():
                k, _, _ = oracle.route(L.X, L.Wr, nthreads=nt)
                oracle.gemm(L.X, k, c, z, N, nthreads=nt)
                return k
            k, dt = _timed(run)
            dec_bytes += decode_bytes(N, K, T, int(k.max()))
            dec_s += dt
    proto["config2_decode"] = {"s": round(dec_s, 3), "bytes": dec_bytes, "GB/s": round(dec_bytes / dec_s / 1e9, 4),
                               "pack_s_three_shapes": round(pack_s, 3)}
    # config 3: the whole prefill workload
    L = wl.prefill()
    (c, z, _), tp = _timed(lambda: oracle.pack(L.W, S=3, nthreads=nt))
    (k, _, _), tr = _timed(lambda: oracle.route(L.X, L.Wr, L.bias, nthreads=nt))
    _, tg = _timed(lambda: oracle.gemm(L.X, k, c, z, L.N, nthreads=nt))
    macs = L.T * L.N * L.K
    proto["config3_prefill"] = {"s": round(tp + tr + tg, 3), "pack_s": round(tp, 3), "route_s": round(tr, 3),
                                "gemm_s": round(tg, 3), "gemm_GFLOP/s_effective": gemm_rate(macs, tg)}
    # config 4: one layer (7 projections) of the 32-layer stack, extrapolated x32
    lay_pack, lay_dec, params = 0.0, 0.0, 0
    for pi in range(len(wl.LLAMA7B_PROJECTIONS)):
        Lp = wl.full_model_projection(0, pi, T=8, device="cpu")
        W = Lp.W.numpy()
        (c, z, _), tp = _timed(lambda: oracle.pack(W, S=3, nthreads=nt))
        def run():
            k, _, _ = oracle.route(Lp.X, Lp.Wr, nthreads=nt)
            oracle.gemm(Lp.X, k, c, z, Lp.N, nthreads=nt)
        _, td = _timed(run)
        lay_pack += tp
        lay_dec += td
        params += Lp.N * Lp.K
    layers = wl.LLAMA7B_LAYERS
    proto["config4_full_model"] = {"measured": "layer 0 (7 projections), extrapolated x32", "params_layer": params,
                                   "pack_s_layer": round(lay_pack, 3), "decode_s_layer": round(lay_dec, 3),
                                   "pack_s_model": round(lay_pack * layers, 2),
                                   "decode_s_per_step_model": round(lay_dec * layers, 2)}
    # config 5: pack in full, GEMM on a token subset (every bucket), extrapolated to all tokens
    L = wl.skewed_prefill()
    (c, z, _), tp = _timed(lambda: oracle.pack(L.W, S=3, nthreads=nt))
    (k, _, _), tr = _timed(lambda: oracle.route(L.X, L.Wr, L.bias, nthreads=nt))
    sub = np.arange(0, L.T, L.T // 128, dtype=np.int32)
    _, tg = _timed(lambda: oracle.gemm(L.X, k, c, z, L.N, tokens=sub, nthreads=nt))
    proto["config5_skewed_prefill"] = {"pack_s": round(tp, 3), "route_s": round(tr, 3),
                                       "gemm_tokens": int(sub.size), "gemm_s_subset": round(tg, 3),
                                       "gemm_s_all_tokens_extrapolated": round(tg * L.T / sub.size, 2),
                                       "gemm_GFLOP/s_effective": gemm_rate(sub.size * L.N * L.K, tg)}
    # one thread: the decode sample (first 4096 rows of every case) and a 32-token prefill subset
    credited, spent, _, desc = oracle_decode_sample(0.0, [(N, K, T) for (N, K) in wl.DECODE_SHAPES
                                                          for T in wl.DECODE_TOKENS], rows_cap=1024, nthreads=1)
    L = wl.prefill()
    c, z, _ = oracle.pack(L.W[:1024], S=3, nthreads=1)
    k, _, _ = oracle.route(L.X, L.Wr, L.bias, nthreads=1)
    sub = np.arange(0, L.T, L.T // 32, dtype=np.int32)
    _, tg1 = _timed(lambda: oracle.gemm(L.X, k, c, z, 1024, tokens=sub, nthreads=1))
    proto["single_thread"] = {"decode_GB/s": round(credited / spent / 1e9, 4),
                              "decode_sample": "first 1024 rows of each of the nine decode cases",
                              "prefill_gemm_GFLOP/s_effective": gemm_rate(sub.size * 1024 * L.K, tg1),
                              "prefill_sample": "32 tokens x first 1024 rows of config 3"}
    value = dec_bytes / dec_s / 1e9
    return {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "config 2 in full (nine decode problems, oracle route + fp64 GEMM, all threads); the "
                      "protocol below covers configs 1-5 and one thread",
            "protocol": proto}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    from token_adaptive_mixed_b200 import workloads as wl
    import oracle
    oracle.build()
    spec = [(N, K, T) for (N, K) in wl.DECODE_SHAPES for T in wl.DECODE_TOKENS]
    per_step_budget = max(0.2, 150.0 / max(1, args.steps + args.warmup))
    # rows per step sized so one sampled case fits the per-step budget (4096x4096 T=16 ~ 1 s per 1024 rows)
    rows = int(max(16, min(4096, 1024 * per_step_budget)))
    rows -= rows % 16
    for i in range(args.warmup):
        oracle_decode_sample(0.0, [spec[i % len(spec)]], rows_cap=rows)
    tot_b, tot_s = 0, 0.0
    for i in range(args.steps):
        b, s, threads, desc = oracle_decode_sample(0.0, [spec[i % len(spec)]], rows_cap=rows)
        tot_b += b
        tot_s += s
    value = tot_b / tot_s / 1e9
    return {"metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": WORKLOAD, "parallelism": "host cores"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": len(os.sched_getaffinity(0)),
                             "kind": "oracle",
                             "sample": f"per step: oracle route + fp64 GEMM on the first {rows} rows of one decode case, "
                                       f"cycling through the nine cases"},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="mobi", choices=["mobi", "reference"])
    ap.add_argument("--cpu-baseline-seconds", type=float, default=20.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--only", default="all", choices=["all", "decode", "prefill", "route_mlp", "ckpt", "generic"],
                    help="run a subset (profiling); the default runs everything")
    ap.add_argument("--prefill-reps", type=int, default=10)
    ap.add_argument("--skip-skewed", action="store_true")
    ap.add_argument("--skip-full-model", action="store_true")
    args = ap.parse_args()

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out))
        return

    world, rank, _ = dist_setup(args.gpus)
    out = run_gpu(args, world, rank)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline and args.only == "all":
            out["cpu_baseline"] = cpu_baseline(args.cpu_baseline_seconds)
        print(json.dumps(out))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
