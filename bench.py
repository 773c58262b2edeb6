"""Benchmark of the MatMulNBits hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

A step is one Qwen3-1.7B-shaped decode step at M = 1: the 28 x 7 projections
plus the lm_head, 197 calls of mnb_gemv (int4 block-32 asymmetric weights,
fp16 activations and scales), replayed from a CUDA graph with programmatic
dependent launch.  `value` is the weight bytes the step streams per second
(packed nibbles + scales + zero points), inputs already in HBM; the weights
(995 MB) are larger than L2, so no flush is needed.  `e2e` repeats the step
through the same calls with the inputs copied from pinned host memory and
the outputs copied back inside the timed region.  `prefill` times the
tensor-core path (mnb_gemm) on the same model's 196 projections at M = 1024
(TFLOP/s).  Under torchrun every rank runs its own replica (the operator has
no exchange step); time is the max over ranks.

--impl reference times the CPU oracle (tests' reference implementation) on a
bounded sample of the same workload on the host cores.
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
sys.path.insert(0, ROOT)

METRIC = "M=1 GEMV weight GB/s & prefill TFLOP/s on one B200, as % of HBM/TC roofline"
WORKLOAD = ("qwen3-1.7b-shaped decode step, M=1: 28 layers x (q 2048->2048, k/v 2048->1024, "
            "o 2048->2048, gate/up 2048->6144, down 6144->2048) + lm_head 2048->151936; "
            "int4 block 32 asymmetric, fp16 activations and scales, weights N(0,0.02) with 1% outliers x8")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

DECODE_KERNEL = "gemv_resident_kernel"   # the kernel of the decode step's launches (M = 1)
NOMINAL = {"hbm_gbs": 8000.0, "tc_tflops": 2250.0}   # B200 spec sheet: HBM3e, dense fp16/bf16


def ncu_traffic(kernel):
    """DRAM bytes (read + write) per launch of `kernel` from the committed ncu
    summaries under profiles/, which record them in a line
    ``traffic: kernel=<name> source=<file> sha1=<hex> bytes_per_launch=<n>``.
    None unless the kernel's source file still has that hash (the counters
    describe the kernel as it was captured)."""
    import glob
    import hashlib
    import re

    pat = re.compile(r"traffic: kernel=(\S+) source=(\S+) sha1=([0-9a-f]+) bytes_per_launch=(\d+)")
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for m in pat.finditer(open(path).read()):
            if m.group(1) != kernel:
                continue
            src = os.path.join(ROOT, m.group(2))
            if os.path.exists(src) and hashlib.sha1(open(src, "rb").read()).hexdigest() == m.group(3):
                return {"bytes_per_launch": int(m.group(4)), "profile": os.path.relpath(path, ROOT)}
    return None


def job_gbs(world, bytes_per_rank, ms_max):
    """Whole-job throughput: every rank streams bytes_per_rank in the timed step,
    and the step takes the slowest rank's time."""
    return world * bytes_per_rank / (ms_max * 1e-3) / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# --------------------------------------------------------------------------- ranks

def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


class Ranks:
    def __init__(self, world, rank, local, backend):
        import torch
        import torch.distributed as dist

        self.world, self.rank, self.local = world, rank, local
        self.dist = dist if world > 1 else None
        if self.dist:
            import datetime

            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))

    def barrier(self):
        if self.dist:
            self.dist.barrier()

    def max(self, v):
        if not self.dist:
            return v
        import torch

        dev = "cuda" if self.dist.get_backend() == "nccl" else "cpu"
        t = torch.tensor([v], dtype=torch.float64, device=dev)
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.dist:
            self.dist.destroy_process_group()


# --------------------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons with NVML in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index, period=0.005):
        self.samples, self.reasons, self.ok = [], 0, False
        self.period, self.index = period, index
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report it instead of clocks
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            pass

    def __enter__(self):
        if self.ok:
            self._stop = threading.Event()
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok:
            return {"error": getattr(self, "err", "nvml unavailable")}
        names = [n for b, n in self.REASONS.items() if self.reasons & b and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# --------------------------------------------------------------------------- workloads

def build_model(cfg_name, dev, lm_head=True):
    import torch

    import workloads
    from int4_block_quantized_matmulnbits_b200.step import QLinear

    cfg = workloads.CONFIGS[cfg_name]
    lins = []
    linears = workloads.config_linears(cfg_name)
    if not lm_head:
        linears = [l for l in linears if l.name != "lm_head"]
    for lin in linears:
        W = workloads.weight(cfg["seed"], lin.layer, lin.proj, lin.N, lin.K, cfg.get("outliers", False), device=dev)
        lins.append(QLinear.quantize(W, cfg["bs"], cfg["has_zp"], torch.float16, name=f"{lin.name}{lin.layer}"))
        del W
    torch.cuda.synchronize()
    return cfg, lins


def fill(p, seed):
    import workloads

    for i, x in enumerate(p.X):
        x.copy_(workloads.activations(seed, x.shape[0], x.shape[1], x.dtype, tag=i, device=x.device))


def timed_replays(p, steps, warmup, ranks, tag="timed"):
    """Device time of `steps` graph replays (ms, max over ranks).  The timed
    loop sits in an NVTX range named `tag` (for profiler filtering)."""
    import torch

    for _ in range(warmup):
        p.replay()
    torch.cuda.synchronize()
    ranks.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push(tag)
    e0.record(s)
    for _ in range(steps):
        p.replay()
    e1.record(s)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    ranks.barrier()
    return ranks.max(e0.elapsed_time(e1))


def timed_e2e(p, steps, warmup, ranks):
    """Step time with the inputs copied in from pinned host memory and the outputs
    copied back, all inside the timed region (ms per step, max over ranks)."""
    import torch

    hx = torch.empty(p.x_flat.shape, dtype=p.x_flat.dtype, pin_memory=True)
    hx.copy_(p.x_flat.cpu())
    hy = torch.empty(p.y_flat.shape, dtype=p.y_flat.dtype, pin_memory=True)
    s = torch.cuda.current_stream()

    def one():
        p.x_flat.copy_(hx, non_blocking=True)
        p.replay()
        hy.copy_(p.y_flat, non_blocking=True)

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    ranks.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(steps):
        one()
    e1.record(s)
    torch.cuda.synchronize()
    ranks.barrier()
    ms = ranks.max(e0.elapsed_time(e1)) / steps
    return ms, hx.numel() * hx.element_size(), hy.numel() * hy.element_size()


class OracleSample:
    """The CPU oracle on a bounded sample of the decode step: the 7 projections
    of layer 0 at M = 1, weights RTN-quantized by the oracle itself (prepared
    once, outside any timing)."""

    def __init__(self):
        import numpy as np

        import oracle
        import workloads

        self.oracle = oracle
        cfg = workloads.CONFIGS["qwen3_1p7b_decode"]
        self.bs = cfg["bs"]
        self.items = []
        for l in workloads.config_linears("qwen3_1p7b_decode"):
            if l.layer != 0:
                continue
            W = workloads.weight(cfg["seed"], l.layer, l.proj, l.N, l.K, True).numpy()
            pk, sc, zp = oracle.quantize_rtn(W, self.bs, True, np.float16)
            X = workloads.activations(cfg["seed"], 1, l.K, tag=l.proj).float().numpy()
            nbytes = sum(oracle.packed_sizes(l.N, l.K, self.bs, np.float16, True))
            self.items.append((l.name, X, pk, sc, zp, l.K, nbytes))
        self.cores = oracle.num_threads()

    def run(self, i):
        """Projection i % 7 of layer 0; returns (weight bytes, seconds)."""
        name, X, pk, sc, zp, K, nbytes = self.items[i % len(self.items)]
        t0 = time.perf_counter()
        self.oracle.matmul(X, pk, sc, zp, K, self.bs)
        return nbytes, time.perf_counter() - t0

    def measure_for(self, seconds):
        """GB/s over whole passes of the layer until `seconds` of oracle time."""
        tot_b = tot_t = 0.0
        reps = 0
        while tot_t < seconds:
            for i in range(len(self.items)):
                b, t = self.run(i)
                tot_b, tot_t = tot_b + b, tot_t + t
            reps += 1
        return tot_b / tot_t / 1e9, tot_t, reps


# --------------------------------------------------------------------------- arms

def run_reference(args, world, rank):
    if rank != 0:
        return
    sample = OracleSample()
    for i in range(args.warmup):
        sample.run(i)
    tot_b = tot_t = 0.0
    for i in range(args.steps):
        b, t = sample.run(args.warmup + i)
        tot_b, tot_t = tot_b + b, tot_t + t
    gbs = tot_b / tot_t / 1e9
    desc = ("oracle.matmul, one projection of layer 0 of the decode step per step (cycling q, k, v, o, "
            "gate, up, down), M=1")
    out = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1000.0 * tot_t / args.steps, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
           "data": "synthetic", "config": {"workload": WORKLOAD, "M": 1, "sample": desc},
           "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": sample.cores, "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def profile_part(args, dev, ranks):
    """Small cases for ncu captures: the lm_head GEMV alone (180 MB of weights,
    larger than L2), layer 0 of the decode step and the lm_head (8 dependent
    GEMV launches, as in the step), or layer 0 of the prefill at M = 1024 on
    the tensor cores."""
    import torch

    import workloads
    from int4_block_quantized_matmulnbits_b200.step import Pass, QLinear

    cfg = workloads.CONFIGS["qwen3_1p7b_decode"]
    if args.only == "lmhead":
        lin = [l for l in workloads.config_linears("qwen3_1p7b_decode") if l.name == "lm_head"]
        M, kind = 1, "gemv"
    elif args.only == "decode-layer":
        lin = [l for l in workloads.config_linears("qwen3_1p7b_decode") if l.layer in (0, 28)]
        M, kind = 1, "gemv"
    else:
        lin = [l for l in workloads.config_linears("qwen3_1p7b_prefill") if l.layer == 0]
        M, kind = args.m, "gemm"
    lins = []
    for l in lin:
        W = workloads.weight(cfg["seed"], l.layer, l.proj, l.N, l.K, True, device=dev)
        lins.append(QLinear.quantize(W, cfg["bs"], True, torch.float16, name=l.name))
        del W
    p = Pass(lins, M, kind, torch.float16, pdl=(args.only == "decode-layer"))
    fill(p, cfg["seed"])
    torch.cuda.synchronize()
    torch.cuda.empty_cache()    # keep only the live buffers on the device
    for _ in range(args.warmup):
        p.run()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("profiled")
    for _ in range(args.steps):
        p.run()
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()


def oracle_rate(fn, units, seconds=1.5):
    """Units per second of the oracle call fn() repeated for about `seconds`
    (at least once), and the repetitions."""
    t = 0.0
    reps = 0
    while t < seconds or reps == 0:
        t0 = time.perf_counter()
        fn()
        t += time.perf_counter() - t0
        reps += 1
    return units * reps / t, reps


def bench_single_gemv(dev, ranks, hbm, with_oracle):
    """The single fp32 GEMV (M=1, K=1024, N=2048, block 32 with zero points,
    fp32 activations and scales).  Latency: 200 dependent launches on ONE copy
    of the weights (L2-resident, as a lone call in a decoder would be); GB/s:
    200 dependent launches over 200 distinct copies (269 MB, larger than L2)."""
    import numpy as np
    import torch

    import workloads
    from int4_block_quantized_matmulnbits_b200.step import Pass, QLinear

    cfg = workloads.CONFIGS["single_gemv"]
    lin = cfg["linears"][0]
    W = workloads.weight(cfg["seed"], lin.layer, lin.proj, lin.N, lin.K, device=dev)
    one = QLinear.quantize(W, cfg["bs"], cfg["has_zp"], torch.float32, name="single")
    copies = [QLinear.quantize(W, cfg["bs"], cfg["has_zp"], torch.float32, name=f"single{i}") for i in range(200)]
    out = {"weight_bytes": one.nbytes, "launches": 200}
    for key, lins in (("l2_resident", [one] * 200), ("rotated_copies", copies)):
        p = Pass(lins, 1, "gemv", torch.float32, pdl=True)
        fill(p, cfg["seed"])
        p.capture()
        t = timed_replays(p, 20, 3, ranks) / 20
        us = t * 1000.0 / len(lins)
        out[key] = {"us_per_call": round(us, 3), "weight_gbs": round(one.nbytes / (us * 1e-6) / 1e9, 1),
                    "frac_hbm": round(one.nbytes / (us * 1e-6) / 1e9 / hbm, 4)}
        del p
    del copies, one
    if with_oracle:
        import oracle

        Wn = W.cpu().numpy()
        pk, sc, zp = oracle.quantize_rtn(Wn, cfg["bs"], True, np.float32)
        X = workloads.activations(cfg["seed"], 1, lin.K, torch.float32).numpy()
        nbytes = sum(oracle.packed_sizes(lin.N, lin.K, cfg["bs"], np.float32, True))
        gbs, reps = oracle_rate(lambda: oracle.matmul(X, pk, sc, zp, lin.K, cfg["bs"]), nbytes)
        out["cpu_oracle"] = {"weight_gbs": round(gbs / 1e9, 4), "us_per_call": round(nbytes / gbs * 1e6, 1),
                             "cores": oracle.num_threads(), "sample": f"the whole GEMV, {reps} calls"}
    del W
    return out


def oracle_layer_gbs(cfg_name, layer=0, M=1, seconds=1.5):
    """The oracle over one layer's 7 projections of a workload at M tokens:
    weight GB/s (its own RTN of the same seeded weights, prepared untimed)."""
    import numpy as np
    import torch

    import oracle
    import workloads

    cfg = workloads.CONFIGS[cfg_name]
    sdt = np.float16 if cfg["scale"] == "f16" else np.float32
    items = []
    for l in workloads.config_linears(cfg_name):
        if l.layer != layer:
            continue
        W = workloads.weight(cfg["seed"], l.layer, l.proj, l.N, l.K, cfg.get("outliers", False)).numpy()
        q = oracle.quantize_rtn(W, cfg["bs"], cfg["has_zp"], sdt)
        X = workloads.activations(cfg["seed"], M, l.K, torch.float16, tag=l.proj).float().numpy()
        items.append((X, q, l.K))
    nbytes = sum(sum(oracle.packed_sizes(q[0].shape[0], K, cfg["bs"], sdt, cfg["has_zp"])) for _, q, K in items)

    def run():
        for X, (pk, sc, zp), K in items:
            oracle.matmul(X, pk, sc, zp, K, cfg["bs"])

    gbs, reps = oracle_rate(run, nbytes, seconds)
    flops = 2 * M * sum(q[0].shape[0] * K for _, q, K in items)
    return {"weight_gbs": round(gbs / 1e9, 4), "gflops": round(gbs / nbytes * flops / 1e9, 3),
            "cores": oracle.num_threads(), "sample": f"the 7 projections of layer {layer} at M={M}, {reps} passes"}


def bench_step(cfg_name, dev, ranks, hbm, Ms, steps=50):
    """Decode steps (all projections + lm_head, one mnb_gemv each, CUDA graph,
    PDL) of a workload at each M: us per step and weight GB/s."""
    import torch

    from int4_block_quantized_matmulnbits_b200.step import Pass

    cfg, lins = build_model(cfg_name, dev)
    out = {"launches_per_step": len(lins), "weight_bytes_per_step": sum(l.nbytes for l in lins)}
    for M in Ms:
        p = Pass(lins, M, "gemv", torch.float16, pdl=True)
        fill(p, cfg["seed"] + M)
        p.capture()
        t = timed_replays(p, steps, 5, ranks) / steps
        gbs = p.weight_bytes / (t * 1e-3) / 1e9
        out[f"M{M}"] = {"us_per_step": round(t * 1000, 2), "weight_gbs": round(gbs, 1),
                        "frac_hbm": round(gbs / hbm, 4)}
        del p
    return cfg, lins, out


def bench_layout_variant(cfg_name, dev, ranks, hbm, tc_burst, with_oracle):
    """Layout variants at 0.6B shapes: decode steps at M in gemv_M (with the
    lm_head), prefill passes through mnb_gemm at M in gemm_M (no lm_head)."""
    import torch

    import workloads
    from int4_block_quantized_matmulnbits_b200.step import Pass

    cfg = workloads.CONFIGS[cfg_name]
    cfg, lins, out = bench_step(cfg_name, dev, ranks, hbm, cfg["gemv_M"])
    body = [l for l in lins if l.N != workloads.VOCAB]
    for M in cfg["gemm_M"]:
        p = Pass(body, M, "gemm", torch.float16, pdl=True)
        fill(p, cfg["seed"] + M)
        p.capture()
        t = timed_replays(p, 10, 3, ranks) / 10
        tf = p.flops / (t * 1e-3) / 1e12
        out[f"gemm_M{M}"] = {"ms_per_pass": round(t, 4), "tflops": round(tf, 1),
                             "frac_tc_burst": round(tf / tc_burst, 4),
                             "weight_gbs": round(p.weight_bytes / (t * 1e-3) / 1e9, 1)}
        del p
    del lins
    torch.cuda.empty_cache()
    if with_oracle:
        out["cpu_oracle"] = oracle_layer_gbs(cfg_name)
    return out


def bench_embed(dev, ranks, hbm, with_oracle):
    """mnb_embed_gather over the int8 table [151936, 1024] (155.6 MB, larger
    than L2) with fp32 row scales: 4096 uniformly random ids per call into
    fp16 rows; 40 calls per replay, each with its own id set."""
    import torch

    import int4_block_quantized_matmulnbits_b200 as mnb
    import workloads

    e = workloads.EMBED
    table, scales, ids = workloads.embed_inputs(e["seed"], e["V"], e["D"], e["T"])
    table, scales = table.to(dev), scales.to(dev)
    g = torch.Generator(device="cpu").manual_seed(e["seed"] * 7 + 1)
    id_sets = [torch.randint(0, e["V"], (e["T"],), generator=g, dtype=torch.int32).to(dev) for _ in range(40)]
    outs = [torch.empty((e["T"], e["D"]), dtype=torch.float16, device=dev) for _ in range(40)]
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())

    def run():
        for i, o in zip(id_sets, outs):
            mnb.mnb_embed_gather(table, scales, e["V"], e["D"], i, e["T"], o, None, s)

    with torch.cuda.stream(s):
        run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        run()

    class G:
        def replay(self):
            graph.replay()

    t = timed_replays(G(), 20, 3, ranks) / 20
    us = t * 1000.0 / len(id_sets)
    nbytes = e["T"] * (e["D"] + 4 + 4) + e["T"] * e["D"] * 2   # rows, scale, id read; fp16 rows written
    gbs = nbytes / (us * 1e-6) / 1e9
    out = {"ids_per_call": e["T"], "bytes_per_call": nbytes, "us_per_call": round(us, 3), "gbs": round(gbs, 1),
           "frac_hbm": round(gbs / hbm, 4), "calls_per_replay": len(id_sets)}
    if with_oracle:
        import numpy as np

        import oracle

        tn, sn, idn = table.cpu().numpy(), scales.cpu().numpy(), ids.numpy()
        ogbs, reps = oracle_rate(lambda: oracle.embed_gather(tn, sn, idn, np.float16), nbytes)
        out["cpu_oracle"] = {"gbs": round(ogbs / 1e9, 4), "cores": 1,
                             "sample": f"one call of 4096 ids, {reps} calls (the oracle's gather is one thread)"}
    return out


def bench_gptq(dev, ranks, with_oracle):
    """GPTQ of the 1.7B decoder's layer-0 q projection (N = K = 2048) from 2048
    calibration tokens (synthetic, correlated fp16 activations): device time
    of each stage (CUDA events; the factorisation synchronizes its stream once)."""
    import numpy as np
    import torch

    import int4_block_quantized_matmulnbits_b200 as mnb
    import workloads

    cfg = workloads.CONFIGS["qwen3_1p7b_decode"]
    N = K = 2048
    T, bs = 2048, cfg["bs"]
    g = torch.Generator(device="cpu").manual_seed(cfg["seed"] * 1_000_003 + 4242)
    mix = torch.eye(K) + torch.randn((K, K), generator=g) / K ** 0.5
    X = (torch.randn((T, K), generator=g) @ mix).half().to(dev)
    W = workloads.weight(cfg["seed"], 0, 0, N, K, True, device=dev)
    H = torch.empty((K, K), dtype=torch.float32, device=dev)
    U = torch.empty((K, K), dtype=torch.float32, device=dev)
    dead = torch.empty((K,), dtype=torch.uint8, device=dev)
    ws = torch.empty((mnb.mnb_gptq_workspace_bytes(K),), dtype=torch.uint8, device=dev)
    packed = torch.empty((N, K // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((N, K // bs), dtype=torch.float16, device=dev)
    zp = torch.empty((N, K // bs // 2), dtype=torch.uint8, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    times = []
    for rep in range(4):   # the first is warm-up
        torch.cuda.synchronize()
        ev[0].record()
        mnb.mnb_gptq_hessian(X, H)
        ev[1].record()
        mnb.mnb_gptq_prepare(H, U, dead, ws, 0.01)
        ev[2].record()
        mnb.mnb_gptq_quantize(W, U, dead, bs, True, packed, scales, zp)
        ev[3].record()
        torch.cuda.synchronize()
        if rep:
            times.append([ev[i].elapsed_time(ev[i + 1]) for i in range(3)])
    t = np.median(np.array(times), axis=0)
    out = {"projection": "q of layer 0, N = K = 2048, block 32, zero points, fp16 scales", "calib_tokens": T,
           "hessian_ms": round(float(t[0]), 3), "prepare_ms": round(float(t[1]), 3),
           "quantize_ms": round(float(t[2]), 3), "total_ms": round(float(t.sum()), 3),
           "weights_per_s": round(N * K / (float(t.sum()) * 1e-3), 1)}
    # quality: mean squared output error over the calibration inputs, GPTQ's
    # codes against round-to-nearest ones of the same weights (both
    # dequantized by the library)
    rp, rs, rz = torch.empty_like(packed), torch.empty_like(scales), torch.empty_like(zp)
    mnb.mnb_quantize_rtn(W, N, K, bs, True, rp, rs, rz)
    Wd = torch.empty((N, K), dtype=torch.float32, device=dev)
    errs = []
    for cp, cs, cz in ((packed, scales, zp), (rp, rs, rz)):
        mnb.mnb_dequantize(cp, cs, cz, N, K, bs, Wd)
        errs.append(float(((X.float() @ (W - Wd).T) ** 2).mean()))
    out["output_mse"] = {"gptq": errs[0], "rtn": errs[1], "ratio": round(errs[0] / errs[1], 4)}
    del Wd
    if with_oracle:
        import oracle

        Xn = X.float().cpu().numpy()
        Wn = W.cpu().numpy()
        t0 = time.perf_counter()
        Hn = oracle.gptq_hessian(Xn)
        Un, deadn = oracle.gptq_prepare(Hn)
        t1 = time.perf_counter()
        rows = 128
        oracle.gptq_quantize(Wn[:rows], Un.astype(np.float32), bs, True, np.float16, deadn)
        t2 = time.perf_counter()
        total = (t1 - t0) + (t2 - t1) * N / rows
        out["cpu_oracle"] = {"total_s": round(total, 3), "weights_per_s": round(N * K / total, 1),
                             "cores": oracle.num_threads(),
                             "sample": f"Hessian and factor in full (numpy float64), the column loop on {rows} of "
                                       f"{N} rows, scaled to all rows"}
    return out


def run_gpu(args, world, rank, local):
    import torch

    ranks = Ranks(world, rank, local, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    import int4_block_quantized_matmulnbits_b200 as mnb
    from int4_block_quantized_matmulnbits_b200.step import Pass

    if args.only in ("lmhead", "gemm-layer", "decode-layer"):
        profile_part(args, dev, ranks)
        ranks.close()
        return

    peaks, peak_src = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    tc_burst = float(peaks["bf16_tflops"])
    tc_sust = float(peaks.get("bf16_tflops_sustained", tc_burst))

    if args.only == "prefill":   # profiling mode: the M = 1024 prefill pass alone
        cfg, lins = build_model("qwen3_1p7b_decode", dev, lm_head=False)
        pp = Pass(lins, 1024, "gemm", torch.float16, pdl=True)
        fill(pp, cfg["seed"] + 1024)
        pp.capture()
        timed_replays(pp, args.steps, args.warmup, ranks, "prefill")
        ranks.close()
        return

    # ---- decode step, M = 1 (the headline)
    cfg, lins = build_model("qwen3_1p7b_decode", dev)
    dec = Pass(lins, 1, "gemv", torch.float16, pdl=True)
    fill(dec, cfg["seed"])
    dec.capture()
    with ClockSampler(local) as clk:
        ms_total = timed_replays(dec, args.steps, args.warmup, ranks, "decode")
    if args.only == "decode":
        ranks.close()
        return
    ms = ms_total / args.steps
    wbytes = dec.weight_bytes
    value = job_gbs(world, wbytes, ms)
    per_launch_bytes = wbytes / len(lins)
    per_launch_us = ms * 1000.0 / len(lins)
    achieved = per_launch_bytes / (per_launch_us * 1e-6) / 1e9

    # the same 197 GEMVs as ONE persistent launch (mnb_gemv_chain): each GEMV
    # waits for the previous one, as the separate launches do; then with the
    # decoder's own dependencies (k, v read q's input; up reads gate's)
    cdec = Pass(lins, 1, "gemv", torch.float16, pdl=True, chain=True)
    fill(cdec, cfg["seed"])
    cdec.capture()
    with ClockSampler(local) as cclk:
        c_ms = timed_replays(cdec, args.steps, args.warmup, ranks, "decode_chain") / args.steps
    del cdec
    waits = [0 if l.name.rstrip("0123456789") in ("k", "v", "up") else 1 for l in lins]
    gcdec = Pass(lins, 1, "gemv", torch.float16, pdl=True, chain=True, waits=waits)
    fill(gcdec, cfg["seed"])
    gcdec.capture()
    gc_ms = timed_replays(gcdec, args.steps, args.warmup, ranks, "decode_chain_grouped") / args.steps
    del gcdec
    # without a CUDA graph (eager, one host call per launch): the one-launch
    # step against 197 launches issued from Python
    def eager_us(p, n=20):
        for _ in range(3):
            p.run()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(True), torch.cuda.Event(True)
        a.record()
        for _ in range(n):
            p.run()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n * 1000.0

    esep = Pass(lins, 1, "gemv", torch.float16, pdl=True)
    fill(esep, cfg["seed"])
    e_sep_us = eager_us(esep)
    del esep
    echain = Pass(lins, 1, "gemv", torch.float16, pdl=True, chain=True)
    fill(echain, cfg["seed"])
    e_chain_us = eager_us(echain)
    del echain
    one_launch = {"launches_per_step": 1, "us_per_step": round(c_ms * 1000, 2),
                  "eager_us_per_step": round(e_chain_us, 2), "eager_us_per_step_197_launches": round(e_sep_us, 2),
                  "weight_gbs": round(world * wbytes / (c_ms * 1e-3) / 1e9, 1),
                  "frac_hbm": round(wbytes / (c_ms * 1e-3) / 1e9 / hbm, 4), "clocks": cclk.summary(),
                  "waits_per_step": len(lins) - 1,
                  "grouped_us_per_step": round(gc_ms * 1000, 2), "grouped_waits_per_step": sum(waits) - 1,
                  "grouped_weight_gbs": round(world * wbytes / (gc_ms * 1e-3) / 1e9, 1)}

    # the same step with the weights of projections that share an input stored
    # row-concatenated (q|k|v, gate|up): 113 launches, identical bytes and math
    from int4_block_quantized_matmulnbits_b200.step import fuse_decoder

    flins = fuse_decoder(lins)
    fdec = Pass(flins, 1, "gemv", torch.float16, pdl=True)
    fill(fdec, cfg["seed"])
    fdec.capture()
    with ClockSampler(local) as fclk:
        f_ms = timed_replays(fdec, args.steps, args.warmup, ranks, "decode_fused") / args.steps
    assert fdec.weight_bytes == wbytes
    fused = {"launches_per_step": len(flins), "us_per_step": round(f_ms * 1000, 2),
             "weight_gbs": round(world * wbytes / (f_ms * 1e-3) / 1e9, 1),
             "frac_hbm": round(wbytes / (f_ms * 1e-3) / 1e9 / hbm, 4), "clocks": fclk.summary()}
    del fdec

    # the fused layout with the SwiGLU activation in the gate|up launch
    slins = fuse_decoder(lins, swiglu=True)
    sdec = Pass(slins, 1, "gemv", torch.float16, pdl=True)
    fill(sdec, cfg["seed"])
    sdec.capture()
    s_ms = timed_replays(sdec, max(10, args.steps // 4), args.warmup, ranks, "decode_swiglu") / max(10, args.steps // 4)
    fused["with_swiglu_epilogue_us_per_step"] = round(s_ms * 1000, 2)
    del sdec, slins

    # the same step ending in greedy decoding: the lm_head launch also picks the
    # token (mnb_gemv_argmax), as a decoder's step does
    gdec = Pass(lins, 1, "gemv", torch.float16, pdl=True, greedy=True)
    fill(gdec, cfg["seed"])
    gdec.capture()
    g_ms = timed_replays(gdec, max(10, args.steps // 4), args.warmup, ranks, "decode_greedy") / max(10, args.steps // 4)
    greedy = {"launches_per_step": len(lins), "us_per_step": round(g_ms * 1000, 2),
              "weight_gbs": round(job_gbs(world, wbytes, g_ms), 1),
              "frac_hbm": round(wbytes / (g_ms * 1e-3) / 1e9 / hbm, 4)}
    del gdec

    # lm_head alone: one 180 MB launch, the kernel without launch gaps
    lm = lins[-1]
    lmp = Pass([lm], 1, "gemv", torch.float16, pdl=False)
    fill(lmp, cfg["seed"] + 5)
    lmp.capture()
    lm_ms = timed_replays(lmp, 50, 5, ranks) / 50
    lm_gbs = lm.nbytes / (lm_ms * 1e-3) / 1e9
    lmg = Pass([lm], 1, "gemv", torch.float16, pdl=False, greedy=True)
    fill(lmg, cfg["seed"] + 5)
    lmg.capture()
    lmg_ms = timed_replays(lmg, 50, 5, ranks) / 50
    del lmg

    e2e_ms, h2d, d2h = timed_e2e(dec, max(10, args.steps // 4), max(3, args.warmup), ranks)
    e2e_val = job_gbs(world, wbytes, e2e_ms)

    # decode at larger M (same weights)
    by_m = {}
    for M in (2, 4, 8, 16):
        pm = Pass(lins, M, "gemv", torch.float16, pdl=True)
        fill(pm, cfg["seed"] + M)
        pm.capture()
        t = timed_replays(pm, 100, 10, ranks) / 100
        by_m[str(M)] = {"us_per_step": round(t * 1000, 2), "weight_gbs": round(wbytes / (t * 1e-3) / 1e9, 1),
                        "frac_hbm": round(wbytes / (t * 1e-3) / 1e9 / hbm, 4)}
        del pm
    del dec, lmp
    torch.cuda.empty_cache()

    # ---- prefill on the tensor cores, M = 1024 (no lm_head: logits of the last position only)
    body = [l for l in lins if l.name[:7] != "lm_head"]
    prefill = {}
    for M in (1024, 420, 256, 64):
        pp = Pass(body, M, "gemm", torch.float16, pdl=True)
        fill(pp, cfg["seed"] + M)
        pp.capture()
        n = 20 if M == 1024 else 10
        with ClockSampler(local) as pclk:
            t = timed_replays(pp, n, 3, ranks) / n
        tflops = pp.flops / (t * 1e-3) / 1e12
        prefill[str(M)] = {"ms_per_pass": round(t, 4), "tflops": round(tflops, 1),
                           "frac_tc_sustained": round(tflops / tc_sust, 4),
                           "frac_tc_burst": round(tflops / tc_burst, 4),
                           "weight_gbs": round(pp.weight_bytes / (t * 1e-3) / 1e9, 1)}
        if M == 1024:
            prefill["1024"]["clocks"] = pclk.summary()
            prefill["1024"]["gpu_launches"] = n * pp.launches
        del pp
        torch.cuda.empty_cache()
    # the same prefill with q|k|v and gate|up stored row-concatenated (one GEMM
    # per group, 113 launches): identical weights, bytes and FLOPs, larger GEMMs
    fbody = fuse_decoder(body)
    prefill_fused = {}
    for M in (1024, 420, 256, 64):
        pf = Pass(fbody, M, "gemm", torch.float16, pdl=True)
        fill(pf, cfg["seed"] + M)
        pf.capture()
        n = 20 if M == 1024 else 10
        t = timed_replays(pf, n, 3, ranks) / n
        assert pf.flops == sum(2 * M * l.N * l.K for l in body)
        tflops = pf.flops / (t * 1e-3) / 1e12
        prefill_fused[str(M)] = {"launches_per_pass": len(fbody), "ms_per_pass": round(t, 4),
                                 "tflops": round(tflops, 1), "frac_tc_burst": round(tflops / tc_burst, 4),
                                 "frac_tc_sustained": round(tflops / tc_sust, 4)}
        del pf
        torch.cuda.empty_cache()
    del fbody
    # a prompt appended to a cached one: 17-63 new tokens through mnb_matmul,
    # which runs the decode GEMV up to M = 24 and the GEMM above (same shapes as
    # the prefill pass; its weights)
    cached = {}
    for M in (17, 20, 24, 32, 48, 63):
        pc = Pass(body, M, "matmul", torch.float16, pdl=True)
        fill(pc, cfg["seed"] + M)
        pc.capture()
        t = timed_replays(pc, 10, 3, ranks) / 10
        tflops = pc.flops / (t * 1e-3) / 1e12
        cached[str(M)] = {"ms_per_pass": round(t, 4), "tflops": round(tflops, 1),
                          "weight_gbs": round(pc.weight_bytes / (t * 1e-3) / 1e9, 1),
                          "frac_hbm": round(pc.weight_bytes / (t * 1e-3) / 1e9 / hbm, 4),
                          "path": "gemv" if M <= 24 else "gemm"}
        del pc
        torch.cuda.empty_cache()
    # the same GEMM on a 24-layer audio encoder's linears over one clip's audio tokens
    ecfg, elins = build_model("audio_encoder_prefill", dev)
    encoder = {}
    for M in ecfg["gemm_M"]:
        ep = Pass(elins, M, "gemm", torch.float16, pdl=True)
        fill(ep, ecfg["seed"] + M)
        ep.capture()
        t = timed_replays(ep, 10, 3, ranks) / 10
        encoder[str(M)] = {"ms_per_pass": round(t, 4), "tflops": round(ep.flops / (t * 1e-3) / 1e12, 1),
                           "weight_gbs": round(ep.weight_bytes / (t * 1e-3) / 1e9, 1)}
        del ep
    del elins
    n_launches = len(lins)
    del lins, body
    torch.cuda.empty_cache()
    with_oracle = rank == 0 and world == 1
    single = bench_single_gemv(dev, ranks, hbm, with_oracle)
    torch.cuda.empty_cache()
    _, l06, step06 = bench_step("qwen3_0p6b_decode", dev, ranks, hbm, [1], steps=200)
    del l06
    torch.cuda.empty_cache()
    if with_oracle:
        step06["cpu_oracle"] = oracle_layer_gbs("qwen3_0p6b_decode")
        # the prefill's arithmetic on the oracle: layer 0 at 16 of the 1024
        # tokens (the oracle's cost is linear in the token count)
        prefill["1024"]["cpu_oracle"] = oracle_layer_gbs("qwen3_1p7b_decode", M=16)
    variants = {v: bench_layout_variant(v, dev, ranks, hbm, tc_burst, with_oracle)
                for v in ("qwen3_0p6b_bs64", "qwen3_0p6b_nozp")}
    embed = bench_embed(dev, ranks, hbm, with_oracle)
    torch.cuda.empty_cache()
    gptq = bench_gptq(dev, ranks, with_oracle)
    torch.cuda.empty_cache()
    assert mnb.mnb_device_status() == 0, "a GEMM wait timed out"

    cpu = None
    if rank == 0 and world == 1:
        sample = OracleSample()
        gbs, dt, reps = sample.measure_for(10.0)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": sample.cores, "kind": "oracle",
               "sample": f"oracle.matmul over the 7 projections of layer 0 of the decode step at M=1, "
                         f"{reps} passes, {dt:.1f} s wall on {sample.cores} threads"}

    dec_traffic = ncu_traffic(DECODE_KERNEL)
    gemm_traffic = ncu_traffic("gemm_kernel")
    if rank == 0:
        out = {
            "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "M": 1, "launches_per_step": n_launches,
                       "weight_bytes_per_step": wbytes, "graph": True, "pdl": True,
                       "l2": "inputs larger than L2 (weights of one step > 126 MB)",
                       "parallelism": f"replicas x{world}"},
            "roofline": {"bound": "hbm", "kernel": DECODE_KERNEL, "achieved": round(achieved, 1), "peak": hbm,
                         "unit": "GB/s", "frac": round(achieved / hbm, 4),
                         "traffic": (dec_traffic or {}).get("bytes_per_launch"),
                         "traffic_source": (dec_traffic or {}).get("profile"),
                         "peak_source": f"{peak_src} hbm_gbs", "bytes_per_launch": round(per_launch_bytes),
                         "us_per_launch": round(per_launch_us, 3),
                         "frac_of_nominal_8000_gbs": round(achieved / NOMINAL["hbm_gbs"], 4)},
            "lm_head_alone": {"bytes": lm.nbytes, "us": round(lm_ms * 1000, 2), "gbs": round(lm_gbs, 1),
                              "frac_hbm": round(lm_gbs / hbm, 4),
                              "us_with_greedy_argmax": round(lmg_ms * 1000, 2)},
            "decode_greedy": greedy,
            "decode_fused_qkv_gateup": fused,
            "decode_one_launch": one_launch,
            "decode_by_M": by_m,
            "prefill": prefill,
            "prefill_fused_qkv_gateup": prefill_fused,
            "cached_prefill": cached,
            "audio_encoder_prefill": encoder,
            "roofline_prefill": {"bound": "tensor", "kernel": "gemm_kernel", "M": 1024,
                                 "achieved": prefill["1024"]["tflops"], "peak": tc_burst, "unit": "TFLOP/s",
                                 "frac": prefill["1024"]["frac_tc_burst"],
                                 "traffic": (gemm_traffic or {}).get("bytes_per_launch"),
                                 "traffic_of": "layer-0 q projection",
                                 "traffic_source": (gemm_traffic or {}).get("profile"),
                                 "peak_source": f"{peak_src} bf16_tflops, the burst figure: the timed region is a "
                                                f"~0.1 s run of 196 GEMMs (fp16 = bf16 nominal rate)",
                                 "frac_of_nominal_2250_tflops": round(prefill["1024"]["tflops"] / NOMINAL["tc_tflops"], 4)},
            "single_gemv_fp32": single,
            "decode_step_qwen3_0p6b": step06,
            "layout_variants": variants,
            "embed_gather": embed,
            "gptq": gptq,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_val, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5)},
            "gpu_launches": args.steps * n_launches,
            "clocks": clk.summary(),
        }
        print(json.dumps(out), flush=True)
    ranks.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="mnb", choices=["mnb", "reference"])
    ap.add_argument("--only", default="", choices=["", "decode", "prefill", "lmhead", "gemm-layer", "decode-layer"],
                    help="profiling modes: run one part only and print no JSON line")
    ap.add_argument("--m", type=int, default=1024, help="tokens of the gemm-layer profiling mode")
    args = ap.parse_args()
    world, rank, local = dist_setup()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args, world, rank)
        return
    run_gpu(args, world, rank, local)


if __name__ == "__main__":
    main()
