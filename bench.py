#!/usr/bin/env python
"""Benchmark of the GPT-OSS MoE FFN layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one whole layer forward (router + top-k, dispatch, gate/up GEMM +
clipped SwiGLU, down GEMM + weighted un-permutation, combine) over one batch
of T synthetic tokens already resident in HBM, through the C ABI call
moe_layer_forward.  Default workload: the GPT-OSS-20B-shaped prefill layer
(T=4096, D=F=2880, E=32, k=4, bf16).  Inputs and weights are seeded synthetic
tensors (random-init weights of that shape); the expert weights (1.6 GB) are
far larger than L2, so consecutive steps cannot be served from L2.

Under torchrun (N > 1) every rank runs an independent replica on its own
tokens (data parallel, weak scaling, no collective on the data path); the
step time is the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (numpy fp64, the plain definition of
the layer) on this host's cores on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "MoE layer tokens/s + TFLOP/s vs TC peak (prefill); GB/s vs HBM peak (decode)"
STAGES = ("router_topk", "dispatch", "gateup_swiglu_gemm", "down_combine_gemm", "combine")


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="gptoss20b_prefill", choices=sorted(W.SPECS))
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-decode", action="store_true", help="skip the decode-regime sweep")
    p.add_argument("--no-mxfp4", action="store_true", help="skip the MXFP4-weight layer")
    p.add_argument("--no-skewed", action="store_true", help="skip the GPT-OSS-120B-shaped skewed layer")
    p.add_argument("--no-glm", action="store_true", help="skip the GLM4-MoE-Lite variant layer")
    p.add_argument("--wfmt", choices=("mxfp4", "mxfp4_a8"), default=None,
                   help="MXFP4 workloads: decode the weights in the GEMM mainloop (mxfp4, the default) or "
                        "multiply them on the block-scaled tensor cores with MXFP8 activations (mxfp4_a8)")
    p.add_argument("--h-split", action="store_true",
                   help="keep the SwiGLU output as two bf16 halves between the expert GEMMs (h_split)")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return dict(bf16_tflops=d["bf16_tflops"], bf16_tflops_sustained=d["bf16_tflops_sustained"],
                    hbm_gbs=d["hbm_gbs"], source="measured")
    return dict(bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, hbm_gbs=6650.0, source="fallback")


def config_of(spec, n_gpus, h_split=False, wfmt=None):
    return {"workload": spec.name, "h_split": h_split, "T_per_gpu": spec.T, "hidden_size": spec.D, "intermediate_size": spec.F,
            "num_local_experts": spec.E, "num_experts_per_tok": spec.k, "swiglu_limit": spec.limit,
            "expert_weights": wfmt or spec.wfmt, "global_tokens": spec.T * n_gpus,
            "parallelism": f"dp{n_gpus} (independent replicas)",
            "l2": "inputs larger than L2: every step streams all expert weights "
                  f"({expert_weight_bytes(spec) / 1e9:.2f} GB) through HBM"}


def expert_weight_bytes(spec):
    n = 3 * spec.E * spec.D * spec.F
    return n * (2 if spec.dtype == "bf16" else 4) if spec.wfmt == "dense" else n // 2 + n // 32


# --------------------------------------------------------------------------- #
# clocks during the timed region (NVML reads only)
# --------------------------------------------------------------------------- #
class ClockSampler:
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.err = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:   # no NVML: report that instead of clocks
            self.nv, self.err, self.max_mhz = None, repr(e), None
        self.t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit and name not in ("gpu_idle",):
                        self.reasons.add(name)
            except Exception as e:
                self.err = repr(e)
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self.t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self.nv is not None:
            self.t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0, "error": self.err}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- #
# CPU oracle timing (the reference arm and the cpu_baseline leg)
# --------------------------------------------------------------------------- #
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count()


def oracle_step(spec, layer, S):
    """The oracle (as it stands) on the first S tokens of the workload: whole layer, every expert decoded."""
    from oracle import moe_oracle as O
    sub = dict(layer)
    sub["x"] = layer["x"][:S]
    t0 = time.perf_counter()
    O.layer_forward(sub, spec.k, spec.limit, spec.alpha)
    return time.perf_counter() - t0


def cpu_baseline(spec, layer, budget_s=20.0):
    S = 32
    dt = oracle_step(spec, layer, S)
    while dt < budget_s / 4 and S < spec.T:
        S = min(spec.T, S * 4)
        dt = oracle_step(spec, layer, S)
    return {"value": S / dt, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"first {S} of {spec.T} tokens through the whole layer (numpy fp64, all "
                      f"{spec.E} experts decoded), {dt:.1f} s"}


def oracle_tokens_step(spec, layer, S):
    """The oracle (as it stands) for the first S tokens, one token at a time (only their experts decoded)."""
    from oracle import moe_oracle as O
    t0 = time.perf_counter()
    O.layer_tokens(layer, np.arange(S), spec.k, spec.limit, spec.alpha)
    return time.perf_counter() - t0


def run_reference(args, rank, world, budget_s=150.0):
    if rank != 0:
        return
    spec = W.SPECS[args.workload]
    layer = W.make_layer(spec, seed=0)
    # size the per-step sample so that warm-up + timed steps fit in about budget_s
    per_step = budget_s / max(1, args.steps + args.warmup)
    S = 1
    dt = oracle_tokens_step(spec, layer, S)
    while S < spec.T and dt * 2.5 < per_step:
        S = min(spec.T, S * 2)
        dt = oracle_tokens_step(spec, layer, S)
    for _ in range(args.warmup):
        oracle_tokens_step(spec, layer, S)
    t = [oracle_tokens_step(spec, layer, S) for _ in range(args.steps)]
    ms = 1e3 * sum(t) / len(t)
    value = S / (ms / 1e3)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config_of(spec, world),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": f"each step: the first {S} of {spec.T} tokens, each through the "
                                       "router and its k experts (numpy fp64; the chosen experts' weights "
                                       "decoded once per step)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "impl": "reference"}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- #
# our arm
# --------------------------------------------------------------------------- #
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from mixture_experts_ffn_12_b200 import _lib, api

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    spec = W.SPECS[args.workload]
    layer = W.make_layer(spec, seed=0)
    if rank > 0:   # each replica routes its own tokens
        layer["x"] = W.make_layer(spec, seed=rank, with_experts=False)["x"]
    d = api.upload_layer(layer, dev)
    if args.wfmt is not None and spec.wfmt != "mxfp4":
        raise SystemExit("--wfmt applies to MXFP4 workloads")
    cfg = api.config_from_spec(spec, h_split=args.h_split, wfmt=args.wfmt)
    moe = api.MoELayer(cfg, d["w_router"], d["b_router"], api.expert_weights_from(d))
    x, T = d["x"], spec.T
    y = torch.empty_like(x)
    moe.workspace(T)
    lib = _lib.load()
    stream = torch.cuda.current_stream(dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dev)

    for _ in range(max(args.warmup, 3)):
        moe(x, y=y)
    torch.cuda.synchronize()
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during warm-up")

    # timed steps: back-to-back layer calls, nothing else on the stream
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(local_rank)
    barrier()
    torch.cuda.synchronize()
    with sampler:
        launches0 = lib.moe_launch_count()
        t0.record(stream)
        for _ in range(K):
            moe(x, y=y)
        t1.record(stream)
        launches = lib.moe_launch_count() - launches0
        torch.cuda.synchronize()
    barrier()
    ms_total = max_over_ranks(t0.elapsed_time(t1))
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during the timed steps")

    # stage times (and the gate/up kernel's time for the roofline) from a separate pass:
    # the library records CUDA events on this stream around each stage, which adds
    # event records between the kernels, so this pass is not the one `value` comes from
    Ks = min(K, 50)
    n = len(STAGES)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(Ks)]
    for row in ev:
        for e in row:
            e.record(stream)   # materialise the handles
    torch.cuda.synchronize()
    handles = [[ctypes_ptr(e.cuda_event) for e in row] for row in ev]
    for i in range(Ks):
        starts = (_lib.ctypes.c_void_p * n)(*handles[i][:n])
        stops = (_lib.ctypes.c_void_p * n)(*handles[i][n:])
        lib.moe_set_stage_events(starts, stops, n)
        moe(x, y=y)
    lib.moe_set_stage_events(None, None, 0)
    torch.cuda.synchronize()
    stage_ms = {name: statistics.mean(ev[i][s].elapsed_time(ev[i][n + s]) for i in range(Ks))
                for s, name in enumerate(STAGES)}

    # end to end through MoELayer.run_host_batches: every step copies its input from
    # pinned host memory and its output back to pinned host memory; the copies of
    # neighbouring steps overlap the forward (three streams, double-buffered).  The same
    # K steps as the device-timed region: the first step's copy in and the last step's
    # copy out (~0.5 ms each at the prefill shape) do not overlap a forward
    Ke = K
    xs_host = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for _ in range(2)]
    for xh in xs_host:
        xh.copy_(x)
    ys_host = [torch.empty(y.shape, dtype=y.dtype, pin_memory=True) for _ in range(2)]
    moe.run_host_batches([xs_host[i % 2] for i in range(3)], [ys_host[i % 2] for i in range(3)])
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    moe.run_host_batches([xs_host[i % 2] for i in range(Ke)], [ys_host[i % 2] for i in range(Ke)])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    ms_e2e = max_over_ranks(e0.elapsed_time(e1))

    # the same layer with h kept as two bf16 halves between the expert GEMMs (the precise form)
    hsplit = None
    if not args.h_split and spec.dtype == "bf16" and spec.wfmt == "dense":
        moe2 = api.MoELayer(api.config_from_spec(spec, h_split=True), d["w_router"], d["b_router"], moe.experts)
        for _ in range(3):
            moe2(x, y=y)
        hsplit = {"ms_per_step": timed_steps(lambda: moe2(x, y=y), stream, max(10, K // 2))}
        del moe2
    decode = decode_sweep(api, moe, spec, layer, dev, stream, max(20, K // 4)) if not args.no_decode else None
    mx = sk = glm = None
    extra = world == 1 and spec.name == W.GPTOSS20B_PREFILL.name
    if extra:
        del d, moe
        torch.cuda.empty_cache()
        if not args.no_mxfp4:
            mx = mxfp4_sweep(api, dev, stream, max(10, K // 10))
        if not args.no_skewed:
            sk = skewed_sweep(api, dev, stream, max(10, K // 2))
        if not args.no_glm:
            glm = glm_sweep(api, dev, stream, max(10, K // 2))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(spec, layer)

    if rank == 0:
        peaks = measured_peaks()
        flops = spec.expert_flops() + spec.router_flops()
        ms_step = ms_total / K
        value = job_throughput(world, T, K, ms_total)
        gu_flops = 4.0 * spec.R * spec.D * spec.F
        gu_ms = stage_ms["gateup_swiglu_gemm"]
        achieved = gu_flops / (gu_ms / 1e3) / 1e12
        # the MXFP4 x MXFP8 GEMMs run kind::mxf8f6f4, whose rate is twice the bf16 one (nominal
        # 4.5 against 2.25 PFLOP/s dense): their peak is the bf16 figure times that ratio
        a8 = args.wfmt == "mxfp4_a8"
        pk, pk_sus = (2.0 if a8 else 1.0) * peaks["bf16_tflops"], (2.0 if a8 else 1.0) * peaks["bf16_tflops_sustained"]
        pk_src = peaks["source"] + (" bf16 burst x 2 (nominal f8f6f4 : bf16 rate)" if a8 else " bf16 burst")
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if spec.dtype == "bf16" else "f32",
            "data": "synthetic (seeded random-init weights and activations of the GPT-OSS-20B MoE layer shape)",
            "config": config_of(spec, world, args.h_split, args.wfmt),
            "tflops": flops / (ms_step / 1e3) / 1e12,
            "roofline": {"bound": "tensor", "kernel": "gateup_swiglu_gemm", "achieved": achieved,
                         "peak": pk, "unit": "TFLOP/s", "frac": achieved / pk, "peak_source": pk_src,
                         "frac_of_sustained": achieved / pk_sus,
                         "flops_per_launch": gu_flops, "ms_per_launch": gu_ms,
                         "traffic": traffic_from_profiles("gateup_swiglu_gemm", spec.name)},
            "stage_ms": stage_ms,
            "layer_tflops_frac": flops / (ms_step / 1e3) / 1e12 / pk,
            "e2e": {"value": job_throughput(world, T, Ke, ms_e2e), "unit": "tokens/s",
                    "h2d_bytes_per_step": x.numel() * x.element_size(),
                    "d2h_bytes_per_step": y.numel() * y.element_size()},
            "gpu_launches": int(launches),
            "clocks": sampler.summary(),
        }
        if hsplit is not None:
            line["h_split"] = hsplit
        if decode is not None:
            line["decode"] = decode
        if mx is not None:
            line["mxfp4"] = mx
        if sk is not None:
            line["skewed"] = sk
        if glm is not None:
            line["glm_variant"] = glm
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def decode_sweep(api, moe, spec, layer, dev, stream, steps, copies=4):
    """Decode regime of the same layer (T = 1, 8, 32, 64): GB/s of the expert weights the step touches.

    Each step replays a CUDA graph of one moe_layer_forward (same kernels, no host launch overhead).
    The replays rotate over `copies` copies of the expert weights (each its own MoELayer and graph),
    so a step's weights were last read `copies` - 1 steps earlier, at least 4 x 199 MB (T = 1) of
    other weights ago: more than L2 holds, so every step streams its weights from HBM.
    Touched bytes = (experts with at least one routed token) x 3 x D x F x element size, plus the
    router weights.
    """
    import torch
    peaks = measured_peaks()
    out = {"weight_copies": copies}
    esz = 2 if spec.dtype == "bf16" else 4
    ew = moe.experts
    layers = [moe]
    for _ in range(copies - 1):
        cp = api.ExpertWeights(*(None if t is None else t.clone() for t in
                                 (ew.w_gate, ew.w_up, ew.w_down, ew.b_gate, ew.b_up, ew.b_down)),
                               *(None if t is None else t.clone() for t in (ew.s_gate, ew.s_up, ew.s_down)))
        layers.append(api.MoELayer(moe.cfg, moe.w_router, moe.b_router, cp))
    for T in W.GPTOSS20B_DECODE_T:
        dspec = W.gptoss20b_decode(T) if spec.name.startswith("gptoss20b") else spec.with_tokens(T)
        x = api.to_torch(W.make_layer(dspec, seed=0, with_experts=False)["x"]).to(dev)
        ids = torch.empty((T, spec.k), dtype=torch.int32, device=dev)
        for _ in range(5):
            moe(x, topk_ids=ids)
        torch.cuda.synchronize()
        touched = int(torch.unique(ids).numel())
        # kernels one layer call launches: 2 = the two-kernel decode layer, more = separate kernels
        from mixture_experts_ffn_12_b200 import _lib
        lib = _lib.load()
        n0 = lib.moe_launch_count()
        moe(x, topk_ids=ids)
        launches = int(lib.moe_launch_count() - n0)
        torch.cuda.synchronize()
        # CUDA-graph replay of the same launches (host launch overhead removed), one graph per copy
        replays = [lyr.graphed(x, topk_ids=torch.empty_like(ids))[0] for lyr in layers]
        for i in range(3 * copies):
            replays[i % copies]()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n = max(steps, 2 * copies)
        a.record(stream)
        for i in range(n):
            replays[i % copies]()
        b.record(stream)
        torch.cuda.synchronize()
        us = 1e3 * a.elapsed_time(b) / n
        nbytes = touched * 3 * spec.D * spec.F * esz + spec.E * spec.D * esz
        gbs = nbytes / (us * 1e-6) / 1e9
        out[f"T{T}"] = {"us_per_step": us, "launches_per_step": launches,
                        "path": "two-kernel decode layer" if launches == 2 else "separate kernels",
                        "experts_touched": touched, "weight_bytes": nbytes, "GB/s": gbs,
                        "hbm_frac": gbs / peaks["hbm_gbs"], "tokens/s": T / (us * 1e-6)}
        del replays
    del layers
    torch.cuda.empty_cache()
    return out


def device_experts(api, spec, dev, seed=0):
    """Dense bf16 expert weights drawn on the device (torch's generator, seeded), with the
    recipe's value laws: W ~ N(0, 1/sqrt(fan_in)), biases N(0, expert_b_std).  Timing only:
    the values do not change the work, and drawing 6.4 GB on the host would take a minute."""
    import math
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(1000003 * (seed + 1) + spec.cfg_id)
    E, D, F = spec.E, spec.D, spec.F

    def w(n, kdim):
        t = torch.empty((E, n, kdim), dtype=torch.bfloat16, device=dev)
        for e in range(E):
            t[e] = (torch.randn((n, kdim), generator=g, device=dev) / math.sqrt(kdim)).to(torch.bfloat16)
        return t

    def b(n):
        return (torch.randn((E, n), generator=g, device=dev) * spec.expert_b_std).to(torch.bfloat16)

    return api.ExpertWeights(w(F, D), w(F, D), w(D, F), b(F), b(F), b(D))


def timed_steps(fn, stream, steps):
    """Mean ms per call of fn over `steps` back-to-back calls, CUDA events on `stream`."""
    import torch
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(stream)
    for _ in range(steps):
        fn()
    b.record(stream)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / steps


def stage_times(fn, stream, steps):
    """Mean ms of each library stage over `steps` calls (separate pass: stage events between kernels)."""
    import torch
    from mixture_experts_ffn_12_b200 import _lib
    lib = _lib.load()
    n = len(STAGES)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n)] for _ in range(steps)]
    for row in ev:
        for e in row:
            e.record(stream)
    torch.cuda.synchronize()
    for i in range(steps):
        hs = [ctypes_ptr(e.cuda_event) for e in ev[i]]
        lib.moe_set_stage_events((_lib.ctypes.c_void_p * n)(*hs[:n]), (_lib.ctypes.c_void_p * n)(*hs[n:]), n)
        fn()
    lib.moe_set_stage_events(None, None, 0)
    torch.cuda.synchronize()
    return {name: statistics.mean(ev[i][j].elapsed_time(ev[i][n + j]) for i in range(steps))
            for j, name in enumerate(STAGES)}


def skewed_sweep(api, dev, stream, steps):
    """The GPT-OSS-120B-shaped skewed-load layer (T = 16384, E = 128, k = 4, Zipf(1.1) router
    bias): step time, tokens/s, TFLOP/s, the touched expert weights and the fraction of the
    roofline max(FLOP / tensor peak, touched bytes / HBM bandwidth)."""
    import torch
    spec = W.GPTOSS120B_SKEWED
    peaks = measured_peaks()
    layer = W.make_layer(spec, seed=0, with_experts=False)
    d = api.upload_layer(layer, dev)
    moe = api.MoELayer(api.config_from_spec(spec), d["w_router"], d["b_router"], device_experts(api, spec, dev))
    x = d["x"]
    y = torch.empty_like(x)
    ids = torch.empty((spec.T, spec.k), dtype=torch.int32, device=dev)
    for _ in range(3):
        moe(x, y=y, topk_ids=ids)
    torch.cuda.synchronize()
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during the skewed-layer warm-up")
    cnt = torch.bincount(ids.flatten().long(), minlength=spec.E)
    touched = int((cnt > 0).sum())
    ms = timed_steps(lambda: moe(x, y=y), stream, steps)
    stage = stage_times(lambda: moe(x, y=y), stream, min(steps, 10))
    # the same layer with h kept as two bf16 halves (the down projection does twice the MMA work)
    moe2 = api.MoELayer(api.config_from_spec(spec, h_split=True), d["w_router"], d["b_router"], moe.experts)
    for _ in range(2):
        moe2(x, y=y)
    ms_split = timed_steps(lambda: moe2(x, y=y), stream, steps)
    del moe2
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during the skewed-layer steps")
    flops = spec.expert_flops() + spec.router_flops()
    nbytes = touched * 3 * spec.D * spec.F * 2
    roof_ms = 1e3 * max(flops / (peaks["bf16_tflops"] * 1e12), nbytes / (peaks["hbm_gbs"] * 1e9))
    out = {"workload": spec.name, "T": spec.T, "us_per_step": 1e3 * ms, "tokens/s": spec.T / (ms * 1e-3),
           "tflops": flops / (ms * 1e-3) / 1e12, "experts_touched": touched,
           "max_expert_rows": int(cnt.max()), "touched_weight_bytes": nbytes,
           "roofline_us": 1e3 * roof_ms, "frac": roof_ms / ms,
           "stage_us": {k: 1e3 * v for k, v in stage.items()}, "us_per_step_h_split": 1e3 * ms_split,
           "weights": "expert weights drawn on the device (same law as the recipe); x and router from the recipe"}
    del moe, d
    torch.cuda.empty_cache()
    return out


def glm_sweep(api, dev, stream, steps):
    """The GLM4-MoE-Lite variant at the GPT-OSS-20B shape (T = 4096, E = 32, k = 4, D = F = 2880,
    a shared expert of 2880): step time, tokens/s and TFLOP/s of the routed and shared experts."""
    import math
    import torch
    spec = W.GLM_GPTOSS20B_SHAPE
    peaks = measured_peaks()
    rng = np.random.default_rng(spec.cfg_id)
    D, E, F, Fs, T = spec.D, spec.E, spec.F, spec.F_shared, spec.T
    x = api.to_torch(W.f32_to_bf16_bits(rng.standard_normal((T, D), dtype=np.float32))).to(dev)
    g = torch.Generator(device=dev)
    g.manual_seed(spec.cfg_id)

    def mat(*shape, std):
        return (torch.randn(shape, generator=g, device=dev) * std).to(torch.bfloat16)

    w_router = mat(E, D, std=1 / math.sqrt(D))
    corr = mat(E, std=spec.correction_b_std)
    ew = api.ExpertWeights(mat(E, F, D, std=1 / math.sqrt(D)), mat(E, F, D, std=1 / math.sqrt(D)),
                           mat(E, D, F, std=1 / math.sqrt(F)), None, None, None)
    params = api.GlmParams(spec.norm_topk_prob, spec.routed_scaling_factor, corr, mat(Fs, D, std=1 / math.sqrt(D)),
                           mat(Fs, D, std=1 / math.sqrt(D)), mat(D, Fs, std=1 / math.sqrt(Fs)))
    cfg = api.glm_config_from_spec(spec)
    y = torch.empty_like(x)
    ws = torch.empty(api.glm_workspace_size(cfg, params, T), dtype=torch.uint8, device=dev)

    def step():
        api.glm_layer_forward(cfg, params, x, w_router, ew, y=y, ws=ws)

    for _ in range(3):
        step()
    torch.cuda.synchronize()
    ms = timed_steps(step, stream, steps)
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during the GLM variant steps")
    flops = 6.0 * T * spec.k * D * F + 6.0 * T * D * Fs + 2.0 * T * D * E
    out = {"workload": spec.name, "T": T, "F_shared": Fs, "us_per_step": 1e3 * ms, "tokens/s": T / (ms * 1e-3),
           "tflops": flops / (ms * 1e-3) / 1e12, "frac": flops / (ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
           "weights": "drawn on the device (x from numpy, both seeded)"}
    del ew, params, ws
    torch.cuda.empty_cache()
    return out


def mxfp4_sweep(api, dev, stream, steps):
    """The same layer with MXFP4 expert weights (GPT-OSS-20B shape, T = 8192): per-step time,
    stage times and the gate/up GEMM's TFLOP/s.  The MXFP4 weights are decoded to bf16 inside
    the GEMM mainloop; the FLOPs counted are the bf16 MMA work (4*R*D*F for gate/up)."""
    import torch
    spec = W.GPTOSS20B_MXFP4
    peaks = measured_peaks()
    layer = W.make_layer(spec, seed=0)
    d = api.upload_layer(layer, dev)
    moe = api.MoELayer(api.config_from_spec(spec), d["w_router"], d["b_router"], api.expert_weights_from(d))
    x = d["x"]
    y = torch.empty_like(x)
    for _ in range(3):
        moe(x, y=y)
    torch.cuda.synchronize()
    us = 1e3 * timed_steps(lambda: moe(x, y=y), stream, steps)
    stage = {k: 1e3 * v for k, v in stage_times(lambda: moe(x, y=y), stream, steps).items()}
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during the MXFP4 steps")
    gu_tf = 4.0 * spec.R * spec.D * spec.F / (stage["gateup_swiglu_gemm"] * 1e-6) / 1e12
    out = {"workload": spec.name, "T": spec.T, "us_per_step": us, "tokens/s": spec.T / (us * 1e-6),
           "stage_us": stage, "gateup_tflops": gu_tf, "gateup_frac": gu_tf / peaks["bf16_tflops"],
           "weight_bytes": 3 * spec.E * spec.D * spec.F // 2 + 3 * spec.E * spec.D * spec.F // 32}
    # the same weights on the block-scaled tensor cores with MXFP8 activations (MOE_W_MXFP4_A8);
    # its peak is the f8f6f4 rate, twice the bf16 one (nominal 4.5 against 2.25 PFLOP/s dense)
    moe8 = api.MoELayer(api.config_from_spec(spec, wfmt="mxfp4_a8"), d["w_router"], d["b_router"], moe.experts)
    for _ in range(3):
        moe8(x, y=y)
    torch.cuda.synchronize()
    us8 = 1e3 * timed_steps(lambda: moe8(x, y=y), stream, steps)
    stage8 = {k: 1e3 * v for k, v in stage_times(lambda: moe8(x, y=y), stream, steps).items()}
    if api.last_device_error() != 0:
        raise RuntimeError("device error word set during the MXFP4 x MXFP8 steps")
    fl = 2.0 * spec.R * spec.D * spec.F
    gu8 = 2 * fl / (stage8["gateup_swiglu_gemm"] * 1e-6) / 1e12
    dn8 = fl / (stage8["down_combine_gemm"] * 1e-6) / 1e12
    peak8 = 2.0 * peaks["bf16_tflops"]
    out["a8"] = {"wfmt": "mxfp4_a8", "us_per_step": us8, "tokens/s": spec.T / (us8 * 1e-6), "stage_us": stage8,
                 "gateup_tflops": gu8, "down_tflops": dn8, "peak_tflops": peak8,
                 "peak_source": peaks["source"] + " bf16 burst x 2 (nominal f8f6f4 : bf16 rate)",
                 "gateup_frac": gu8 / peak8, "down_frac": dn8 / peak8}
    return out


def reduce_max(v: float, device) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_rank: int, steps: int, ms_max: float) -> float:
    """Whole-job tokens/s: every rank processed tokens_per_rank tokens per step; time = slowest rank."""
    return world * tokens_per_rank * steps / (ms_max / 1e3)


def ctypes_ptr(h):
    from mixture_experts_ffn_12_b200 import _lib
    return _lib.ctypes.c_void_p(int(h)).value


def gateup_kernel_sha():
    """Identity of the profiled gate/up kernel build: its source, the device helpers it
    includes, and the lines of gemm_launch.cuh that fix its tile shape and ring depth."""
    import hashlib
    csrc = os.path.join(ROOT, "mixture_experts_ffn_12_b200", "csrc")
    h = hashlib.sha256()
    for name in ("grouped_gemm.cuh", "common.cuh"):
        h.update(open(os.path.join(csrc, name), "rb").read())
    for line in open(os.path.join(csrc, "gemm_launch.cuh")):
        if line.startswith(("constexpr int kStages =", "constexpr int kTNGateUp =")):
            h.update(line.encode())
    return h.hexdigest()[:16]


def traffic_from_profiles(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if it matches the current kernel source."""
    import hashlib
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    sha = gateup_kernel_sha()
    vals = {}
    for line in open(path):
        if ":" in line and line.startswith("- "):
            k, v = line[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("kernel_source_sha256_16") != sha:
        return None
    try:
        return float(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
