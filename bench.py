#!/usr/bin/env python
"""Benchmark of the sparse-MoE layer forward (moe_layer_forward) on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one moe_layer_forward (router -> top-k -> histogram/LIS/ranks ->
permutation -> grouped expert GEMMs -> combine) over one batch of T tokens held
in device memory. Multi-GPU runs (torchrun, one process per GPU) are data
parallel: every rank holds the same expert weights and its own token batch, no
collective touches the data path (weak scaling); the timing barrier and the
max-over-ranks reduction are the only collectives.

The headline workload is the Mixtral-8x7B-shaped prefill layer (--config picks
another). On one GPU without a variant flag the line also carries the decode and
Switch-style layers under "workloads" (each timed for over a second) and the
headline layer timed again for over a second under "sustained".

Prints ONE JSON line on rank 0. `value` = tokens/s of the whole job from CUDA
events on the launching stream (L2 flushed between steps, outside the timed
events); `e2e` = the same metric through the C-ABI call with the batch copied
from pinned host memory and the output copied back inside the timed region;
`roofline` = the dominant kernel's algorithmic bytes or flops per launch over its
event-timed duration against the measured peaks; `cpu_baseline` = the CPU oracle
timed on a bounded sample of the same workload on this host's cores.
`--impl reference` times that oracle alone (the only other code path that exists).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "MoE-layer tokens/sec at 1 B200; grouped-GEMM TFLOPS and HBM GB/s as % of peak"
UNIT = "tokens/s"
STAGES = ["router", "topk", "histogram_lis_ranks", "permute", "expert_up", "expert_down", "combine"]
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_BF16_TFLOPS = 2250.0  # B200 dense bf16 tensor-core rate from the spec sheet (context beside the measured peak)
L2_FLUSH_BYTES = 256 << 20
# Workloads timed beside the headline one (single-GPU runs without a variant flag), each
# for at least EXTRA_MIN_MS of device time; the headline workload is timed again for
# SUSTAINED_MS when its K steps are shorter than that.
EXTRA_WORKLOADS = ["decode", "switch"]
EXTRA_MIN_MS = 1200.0
SUSTAINED_MS = 1500.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--config", default="mixtral", choices=list(W.CONFIGS),
                    help="workload of the headline line (default: the Mixtral-shaped prefill, the largest "
                         "single-GPU configuration)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU-oracle baseline budget (rank 0, N=1)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the CPU-oracle leg (for profiling runs)")
    ap.add_argument("--no-extra", action="store_true",
                    help="time only the selected workload (no decode / switch keys, no sustained run)")
    ap.add_argument("--replicate", action="store_true",
                    help="R&Q replica dispatch: time moe_layer_forward_replicated (heavy-hitter split alternately "
                         "with a replica expert m) instead of moe_layer_forward")
    ap.add_argument("--floe", type=float, default=None, metavar="S",
                    help="FloE contextual sparsity at target sparsity S: thresholds calibrated on a second "
                         "synthetic batch (untimed), then moe_layer_forward_floe is timed")
    ap.add_argument("--fp8", action="store_true",
                    help="8-bit experts: E4M3 weights with per-channel scales (quantized once, untimed), "
                         "moe_layer_forward_fp8")
    ap.add_argument("--global-lis", action="store_true",
                    help="every step also sums the per-expert counts over all ranks (NCCL all-reduce of m int32) "
                         "and takes the Load Imbalance Score of the whole job's batch (moe_lis_from_counts); "
                         "routing.global_lis reports it")
    ap.add_argument("--router-only", action="store_true",
                    help="time the routing call alone (moe_route / moe_atomic_route) on the workload's inputs; "
                         "an auxiliary line for profiling, not the layer metric")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload_config(cfg) -> dict:
    return {"workload": cfg.name, "tokens": cfg.T, "d_model": cfg.d, "d_ff": cfg.f, "experts": cfg.m, "top_k": cfg.k,
            "shared_experts": cfg.n_shared, "d_ff_shared": cfg.f_shared,
            "ffn": "swiglu" if cfg.act == W.SWIGLU else "relu", "renormalised_gates": bool(cfg.renorm),
            "router_bias_zipf_s": cfg.zipf_s, "description": cfg.note}


# ------------------------------------------------------------------ CPU oracle baseline

def cpu_oracle_sample(cfg, inp, budget_s: float):
    """Time the oracle's full layer forward on the first n tokens, n sized to ~budget_s."""
    import oracle as O

    threads = os.cpu_count() or 1

    def run(n):
        sub = dict(inp)
        sub["x"] = np.ascontiguousarray(inp["x"][:n])
        t0 = time.perf_counter()
        O.layer_forward(cfg, sub, nthreads=threads)
        return time.perf_counter() - t0

    n = 1
    dt = run(n)
    while dt < budget_s / 8 and n < cfg.T:
        n = min(cfg.T, n * 4)
        dt = run(n)
    if dt < budget_s / 2 and n < cfg.T:
        n = min(cfg.T, max(n + 1, int(n * budget_s / max(dt, 1e-6) * 0.8)))
        dt = run(n)
    return {"value": n / dt, "unit": UNIT, "cores": threads, "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"first {n} of {cfg.T} tokens of the {cfg.name} workload; every step of the layer "
                      f"(router, top-k, histogram/LIS, permutation, expert FFNs, combine) in fp64 C, "
                      f"{threads} threads over tokens"}


def cpu_oracle_fp8_sample(cfg, inp, budget_s: float):
    """Time the oracle's 8-bit layer (oracle.layer_forward_fp8) on the first n tokens,
    n sized to ~budget_s; each timed call quantizes the experts its tokens reach."""
    import oracle as O

    def run(n):
        t0 = time.perf_counter()
        O.layer_forward_fp8(cfg, inp, tokens=np.arange(n))
        return time.perf_counter() - t0

    n = 1
    dt = run(n)
    while dt < budget_s / 8 and n < cfg.T:
        n = min(cfg.T, n * 4)
        dt = run(n)
    return {"value": n / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"first {n} of {cfg.T} tokens of the {cfg.name} workload; the 8-bit layer (router, E4M3 "
                      f"quantization of x, of the experts those tokens reach and of h, fp64 expert FFNs, combine) "
                      f"in numpy, one process"}


def run_config(cfg, world: int) -> dict:
    """The `config` object both arms print for a workload: what is computed, how the job
    is split and how the steps are timed, so the two lines describe the same run; an
    arm's own execution details go in its other keys."""
    return dict(workload_config(cfg), parallelism=f"data-parallel token batches x{world} (weak scaling)",
                l2=f"GPU arm: flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, outside the timed events); "
                   "CPU oracle arm: not applicable",
                launch="GPU arm: eager C-ABI call per step")


def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle as O

    cfg = W.CONFIGS[args.config]
    inp = W.make_moe_inputs(cfg)
    threads = os.cpu_count() or 1
    per_step_budget = max(0.2, min(20.0, 150.0 / (args.steps + args.warmup)))
    # size the sample so one step takes about per_step_budget seconds
    n, dt = 1, 0.0
    while True:
        sub = dict(inp)
        sub["x"] = np.ascontiguousarray(inp["x"][:n])
        t0 = time.perf_counter()
        O.layer_forward(cfg, sub, nthreads=threads)
        dt = time.perf_counter() - t0
        if dt >= per_step_budget / 4 or n >= cfg.T:
            break
        n = min(cfg.T, n * 4)
    n = max(1, min(cfg.T, int(n * per_step_budget / max(dt, 1e-9)))) if n < cfg.T else n
    sub = dict(inp)
    sub["x"] = np.ascontiguousarray(inp["x"][:n])
    for _ in range(args.warmup):
        O.layer_forward(cfg, sub, nthreads=threads)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        O.layer_forward(cfg, sub, nthreads=threads)
        times.append(time.perf_counter() - t0)
    sec = sum(times) / len(times)
    value = n / sec
    sample = (f"first {n} of {cfg.T} tokens of the {cfg.name} workload per step; every step of the layer in fp64 C "
              f"on {threads} host threads")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded generator)", "impl": "reference",
            "config": run_config(cfg, args.gpus),
            "execution": {"parallelism": f"one process, {threads} host threads over tokens", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ end-to-end leg

def e2e_pipelined(torch, fwd, x_host, x_devs, out_devs, out_hosts, K, s_comp, dev):
    """K steps through the C-ABI call with the token batch copied in from pinned host
    memory and the output copied back every step. Copies run on their own streams and
    device buffers alternate, so batch i+1's upload and batch i-1's download overlap
    batch i's forward (a serving loop's arrangement). Returns ms per step."""
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]   # upload of the buffer done
    ev_c = [torch.cuda.Event() for _ in range(2)]    # forward done: input free, output ready
    ev_o = [torch.cuda.Event() for _ in range(2)]    # download done: output buffer free
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize(dev)
    start.record(s_in)
    for i in range(K):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_c[b])
            x_devs[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if i >= 2:
                s_comp.wait_event(ev_o[b])
            fwd(x_devs[b], out_devs[b])
            ev_c[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[b])
            out_hosts[b].copy_(out_devs[b], non_blocking=True)
            ev_o[b].record(s_out)
    end.record(s_out)
    torch.cuda.synchronize(dev)
    return start.elapsed_time(end) / K


# ------------------------------------------------------------------ data-parallel ranks

def rank_inputs(cfg, rank: int):
    """Inputs of one data-parallel rank: the expert and router weights are the same
    on every rank (replicate 0); the token batch is the rank's own (replicate = rank)."""
    inp = W.make_moe_inputs(cfg, replicate=0)
    if rank:
        inp["x"] = W.normal(cfg.seed(rank), W.STREAM["x"], (cfg.T, cfg.d), 1.0, cfg.dtype)
    return inp


def global_histogram(counts, dist=None):
    """Sum a rank's per-expert counts over all ranks, in place (identity on one rank):
    the histogram of the whole job's batch, whose LIS is R&Q Definition 1 over every
    rank's tokens together."""
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(counts, op=dist.ReduceOp.SUM)
    return counts


def max_over_ranks(values, dist=None, device=None):
    """Element-wise maximum of a list of floats over all ranks (identity on one rank)."""
    import torch

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


# ------------------------------------------------------------------ clocks (NVML, sampled during timing)

REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
           0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
           0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, device_index: int):
        self.samples, self.masks, self.err = [], 0, None
        self.h = None
        try:
            import pynvml
            import torch

            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: report why
            self.err = f"nvml unavailable: {e}"
        self._stop = threading.Event()
        self._t = None

    def _one(self):
        nv = self.nv
        self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
        try:
            self.masks |= nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except AttributeError:
            self.masks |= nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _loop(self):
        while not self._stop.is_set():
            try:
                self._one()
            except Exception as e:
                self.err = str(e)
                return
            time.sleep(0.004)

    def start(self):
        if self.h is not None:
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()

    def stop(self):
        if self._t is not None:
            self._stop.set()
            self._t.join()
            if not self.samples:
                self._one()

    def report(self):
        if self.h is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": self.err}
        reasons = sorted(name for bit, name in REASONS.items() if self.masks & bit and name != "gpu_idle")
        return {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": float(self.max_mhz), "reasons": reasons, "samples": len(self.samples)}


# ------------------------------------------------------------------ algorithmic cost model

def T_bytes(cfg) -> int:
    """x in and out of one layer step."""
    return cfg.T * cfg.d * (4 if cfg.dtype == W.F32 else 2)


def fused_routing(cfg) -> bool:
    """The library's rule for its one-launch router (logits + top-k + tile ranks in the
    tensor-core epilogue) followed by the one-kernel scatter: bf16, 8192+ tokens,
    m <= 256, k <= 8."""
    return cfg.dtype == W.BF16 and cfg.T >= 8192 and cfg.m <= 256 and cfg.k <= 8


def stage_costs(cfg, active: int, ksplit: int, weight_bytes=None):
    """Algorithmic flops and bytes per launch of each stage (operands read once,
    results written once; weights of ACTIVE experts only). weight_bytes = 1 for
    E4M3 expert weights (activations still enter and leave each stage in bf16)."""
    es = 4 if cfg.dtype == W.F32 else 2
    ew = es if weight_bytes is None else weight_bytes
    T, d, f, m, k = cfg.T, cfg.d, cfg.f, cfg.m, cfg.k
    Tk = T * k
    mats = 2 if cfg.act == W.SWIGLU else 1
    nsh, fsh = cfg.n_shared, cfg.f_shared
    c = {}
    c["router"] = (2.0 * T * d * m, T * d * es + m * d * es + T * m * 4)
    c["topk"] = (0.0, T * m * 4 + Tk * 8)
    c["histogram_lis_ranks"] = (0.0, Tk * 4 + Tk * 8 + (m + 1) * 8)
    c["permute"] = (0.0, Tk * 4 + T * d * es + Tk * d * es)
    tiles = (T + 127) // 128
    # fused routing: x and W_r in, ids, weights, tile ranks and tile counts out; then the
    # scatter reads those back and writes perm / inv_perm / w_perm, counts, offsets and x_perm
    c["router_topk_ranks"] = (2.0 * T * d * m, T * d * es + m * d * es + Tk * 12 + tiles * m * 4)
    c["scatter"] = (0.0, tiles * m * 4 + Tk * 12 + Tk * 12 + (2 * m + 1) * 4 + T * d * es + Tk * d * es)
    c["expert_up"] = (2.0 * mats * f * d * Tk + 2.0 * mats * fsh * d * T * nsh,
                      active * mats * f * d * ew + nsh * mats * fsh * d * ew + Tk * d * es + (T * d * es if nsh else 0)
                      + Tk * f * es + nsh * T * fsh * es)
    fused_k1 = k == 1 and nsh == 0 and ksplit == 1 and cfg.dtype == W.BF16  # down epilogue writes `out` itself
    out_bytes = T * d * es if fused_k1 else ksplit * Tk * d * 4 + nsh * T * d * 4
    c["expert_down"] = (2.0 * d * f * Tk + 2.0 * d * fsh * T * nsh,
                        active * d * f * ew + nsh * d * fsh * ew + Tk * f * es + nsh * T * fsh * es + out_bytes)
    c["combine"] = (0.0, 0.0 if fused_k1 else ksplit * Tk * d * 4 + nsh * T * d * 4 + Tk * 4 + T * d * es)
    layer_flops = 2.0 * T * d * m + c["expert_up"][0] + c["expert_down"][0]
    layer_bytes = m * d * es + (active * (mats + 1) * f * d + nsh * (mats + 1) * fsh * d) * ew + 2 * T * d * es
    return c, layer_flops, layer_bytes


def source_hash(files=None) -> str:
    """Hash of the library sources: the named files of csrc/ (all of them when None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_mixture_experts_08_b200", "csrc")
    for name in sorted(files if files else os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as fh:
            h.update(name.encode() + fh.read())
    return h.hexdigest()[:16]


def traffic_for(workload: str, stage: str):
    """dram bytes per launch from a committed ncu capture, if the sources that define the
    captured kernel (its entry's source_files) are unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            t = json.load(fh)
        e = t[workload][stage]
        ok = e.get("source_hash") == source_hash(e.get("source_files"))
        return e["dram_bytes_per_launch"] if ok else None
    except Exception:
        return None


# ------------------------------------------------------------------ our arm

def _down_ksplit(cfg, cfg_groups, fp8: bool) -> int:
    """The library's static down-projection K split (mirrors its planner; it only
    enters the byte count of the fp32 partial outputs)."""
    plan_ksplit = 1
    avg = cfg.T * cfg.k / cfg_groups.m
    pair = cfg.dtype == W.BF16 and avg > 128  # the library's pair-tile rule (no K split)
    if cfg.dtype == W.BF16 and cfg.n_shared == 0 and not pair:
        bn, cap = 16, (256 if avg >= 256 else 128)  # the library's down-projection tile rule
        while bn < cap and bn < 2.0 * avg:
            bn <<= 1
        tiles = min(cfg_groups.m, cfg.T * cfg.k) * ((cfg.d + 127) // 128) * max(1, math.ceil(avg / bn))
        if tiles < 4 * 148:
            kb = (cfg.f + 63) // 64
            ks = min(16, -(-4 * 148 // tiles), kb)
            kbps = -(-kb // ks)
            plan_ksplit = -(-kb // kbps)
            if fp8:  # the same split re-cut into 128-element k-blocks
                kb8 = (cfg.f + 127) // 128
                ks8 = min(plan_ksplit, kb8)
                plan_ksplit = -(-kb8 // -(-kb8 // ks8))
    return plan_ksplit


def sustained_applies(K: int, ms: float, clocks) -> bool:
    """The sustained tensor peak (a seconds-long GEMM loop under the power cap) is the
    denominator when the timed region is itself seconds long, or when the GPU sat under
    its power cap for it (median SM clock below 90% of max with sw_power_cap active):
    the burst peak was measured at full clock."""
    if K * ms > 1000.0:
        return True
    c = clocks or {}
    med, mx = c.get("sm_mhz"), c.get("sm_max_mhz")
    return bool(med and mx and "sw_power_cap" in (c.get("reasons") or []) and med < 0.9 * mx)


def roofline_for(cfg, stage: str, fl: float, by: float, dom_ms: float, pk: dict, pk_src: str, long_step: bool,
                 fp8: bool, traffic_key: str) -> dict:
    """Roofline object of one kernel: algorithmic flops / bytes per launch over its
    event-timed duration, against the measured peaks; a contraction also states its
    fraction of the nominal dense tensor-core rate (2.25 PFLOP/s bf16, 4.5 E4M3)."""
    sec = dom_ms * 1e-3
    tensor_peak = pk["bf16_tflops_sustained"] if long_step else pk["bf16_tflops"]
    nominal = NOMINAL_BF16_TFLOPS
    if fp8:  # E4M3 contraction: the measured bf16 peak times the nominal dense fp8 / bf16 ratio (4.5 / 2.25)
        tensor_peak *= 2.0
        nominal *= 2.0
    ridge = tensor_peak * 1e12 / (pk["hbm_gbs"] * 1e9)
    if fl > 0 and fl / max(by, 1.0) > ridge and cfg.dtype == W.BF16:
        roof = {"bound": "tensor", "achieved": fl / sec / 1e12, "peak": tensor_peak, "unit": "TFLOP/s"}
        roof["peak_source"] = (f"{pk_src} bf16 ({'sustained' if long_step else 'burst'})"
                               + (" x 2 (nominal fp8 / bf16 dense ratio)" if fp8 else ""))
        roof["frac_of_nominal_dense"] = roof["achieved"] / nominal
        roof["nominal_dense_tflops"] = nominal
        if long_step:  # the burst figure beside it
            roof["frac_of_burst"] = roof["achieved"] / (pk["bf16_tflops"] * (2.0 if fp8 else 1.0))
    else:
        roof = {"bound": "hbm", "achieved": by / sec / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "peak_source": f"{pk_src} hbm copy"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["traffic"] = traffic_for(traffic_key, stage)
    roof["kernel"] = stage
    roof["algorithmic_bytes"] = by
    roof["algorithmic_flops"] = fl
    roof["duration_us"] = dom_ms * 1e3
    return roof


def layer_run(cfg, args, dev, rank: int, world: int, dist, steps, warmup: int, with_e2e: bool,
              min_timed_ms: float = 0.0, sustained_ms: float = 0.0):
    """Everything measured for one coarse-expert workload: warm-up, the per-stage
    pass, `steps` timed steps (None: enough steps for min_timed_ms of device time),
    optionally a second, longer timed run (sustained_ms) and the end-to-end leg.
    Returns a dict of results; rank 0's line is built from it by the caller."""
    import torch

    import sparse_mixture_experts_08_b200 as moe

    inp = rank_inputs(cfg, rank)

    def to_dev(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)

    d_in = {k: to_dev(v) for k, v in inp.items()}
    c = moe.make_config(cfg.T, cfg.d, cfg.f, cfg.m, cfg.k, cfg.n_shared, cfg.f_shared, cfg.dtype, cfg.act,
                        cfg.renorm)
    rep = args.replicate
    floe = args.floe
    fp8 = args.fp8
    if rep and cfg.dtype != W.BF16:
        raise SystemExit("--replicate runs bf16 layers only")
    if fp8 and (rep or floe is not None or cfg.dtype != W.BF16):
        raise SystemExit("--fp8 runs plain bf16 layers (no --replicate / --floe)")
    if floe is not None and (cfg.dtype != W.BF16 or cfg.act != W.SWIGLU or cfg.n_shared):
        raise SystemExit("--floe runs bf16 SwiGLU layers without shared experts")
    if rep:
        ws = moe.replica_workspace(c, device=dev)
    elif floe is not None:
        ws = moe.floe_workspace(c, device=dev)
    elif fp8:
        ws = moe.fp8_workspace(c, device=dev)
        # one-time E4M3 weights (untimed), then the bf16 copies are dropped
        wq = moe.quantize_experts(d_in["w_gate"], d_in.get("w_up"), d_in["w_down"], d_in.get("ws_gate"),
                                  d_in.get("ws_up"), d_in.get("ws_down"))
        for key in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
            d_in.pop(key, None)
        torch.cuda.synchronize(dev)
    else:
        ws = moe.workspace(c, device=dev)
    if floe is not None:  # one-time weight layout and threshold calibration (untimed)
        w_down_t = torch.empty((cfg.m, cfg.f, cfg.d), dtype=torch.bfloat16, device=dev)
        moe.moe_floe_pack_down(c, d_in["w_down"], w_down_t)
        xc = to_dev(W.make_moe_inputs(cfg, replicate=1, weights=False)["x"])
        u_cal = torch.empty((cfg.T, cfg.m * cfg.f), dtype=torch.float32, device=dev)
        thr = torch.empty(cfg.m, dtype=torch.float32, device=dev)
        ws_cal = moe.workspace(c, device=dev)
        moe.moe_floe_calibrate(c, xc, d_in["w_up"], floe, u_cal, thr, ws_cal)
        torch.cuda.synchronize(dev)
        if moe.moe_read_device_status(ws_cal) != moe.OK:
            raise RuntimeError("device status after the FloE calibration is not OK")
        del u_cal
        kept = torch.zeros(cfg.m, dtype=torch.int32, device=dev)
        floe_idx = torch.zeros((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    tdt = torch.float32 if cfg.dtype == W.F32 else torch.bfloat16
    out = torch.empty((cfg.T, cfg.d), dtype=tdt, device=dev)
    counts = torch.empty(cfg.m + (1 if rep else 0), dtype=torch.int32, device=dev)
    lis = moe.lis_buffer(dev)
    lis0 = moe.lis_buffer(dev)
    glob = args.global_lis
    if glob and (rep or floe is not None or fp8):
        raise SystemExit("--global-lis runs the plain layer")
    gcounts = torch.empty(cfg.m, dtype=torch.int32, device=dev)
    glis = moe.lis_buffer(dev)
    s = torch.cuda.Stream(device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd(x=None, o=None):
        if fp8:
            moe.moe_layer_forward_fp8(c, d_in["x"] if x is None else x, d_in["w_router"], d_in["bias"], wq,
                                      out if o is None else o, ws, counts_out=counts, lis_out=lis, stream=s)
            return
        args_ = (c, d_in["x"] if x is None else x, d_in["w_router"], d_in["bias"], d_in["w_gate"], d_in.get("w_up"),
                 d_in["w_down"], d_in.get("ws_gate"), d_in.get("ws_up"), d_in.get("ws_down"),
                 out if o is None else o, ws)
        if rep:
            moe.moe_layer_forward_replicated(*args_, counts_out=counts, lis_before_out=lis0, lis_after_out=lis,
                                             stream=s)
        elif floe is not None:
            moe.moe_layer_forward_floe(c, args_[1], d_in["w_router"], d_in["bias"], d_in["w_gate"], d_in["w_up"],
                                       w_down_t, thr, args_[10], ws, topk_idx_out=floe_idx, kept_out=kept, stream=s)
        else:
            moe.moe_layer_forward(*args_, counts_out=counts, lis_out=lis, stream=s)
            if glob:  # the whole job's histogram and its LIS (an exchange of m int32 per step)
                gcounts.copy_(counts)
                global_histogram(gcounts, dist)
                moe.moe_lis_from_counts(cfg.m, world * cfg.T * cfg.k, gcounts, glis, stream=s)

    with torch.cuda.stream(s):
        n0 = moe.moe_launch_count()
        fwd()
        launches_per_step = moe.moe_launch_count() - n0
        for _ in range(max(warmup, 3)):
            flush.zero_()
            fwd()
    torch.cuda.synchronize(dev)
    st = moe.moe_read_device_status(ws, stream=s)
    if st != moe.OK:
        raise RuntimeError(f"device status after warm-up: {moe.moe_status_string(st)}")
    if floe is not None:  # the FloE call returns no histogram: the same statistics from its routing
        cnt = np.bincount(floe_idx.cpu().numpy().ravel(), minlength=cfg.m).astype(np.int32)
        argmax = int(np.argmax(cnt))
        max_count, lis_v = int(cnt[argmax]), cfg.m * int(cnt[argmax]) / (cfg.T * cfg.k)
    else:
        cnt = counts.cpu().numpy()
        max_count, argmax, lis_v = moe.unpack_lis(lis)
    active = int((cnt > 0).sum())
    ent = cnt[cnt > 0] / cnt.sum()
    entropy = float(-(ent * np.log(ent)).sum())

    # ---- profiling pass (untimed): every stage boundary gets an event, which
    # serialises the kernels; it gives the per-kernel breakdown and picks the
    # dominant kernel, whose boundaries alone are then recorded in the timed region.
    Kp = max(3, min(steps if steps else 50, 50))
    ev_prof = [[torch.cuda.Event(enable_timing=True) for _ in range(8)] for _ in range(Kp)]
    with torch.cuda.stream(s):  # torch creates the CUDA events on first record
        for evs in ev_prof:
            for e in evs:
                e.record(s)
        for i in range(Kp):
            flush.zero_()
            moe.moe_set_stage_events(ev_prof[i])
            fwd()
    torch.cuda.synchronize(dev)
    moe.moe_set_stage_events([])
    stage_ms = {name: sum(ev_prof[i][j].elapsed_time(ev_prof[i][j + 1]) for i in range(Kp)) / Kp
                for j, name in enumerate(STAGES)}
    prof_step_ms = sum(ev_prof[i][0].elapsed_time(ev_prof[i][7]) for i in range(Kp)) / Kp
    dom = max(STAGES, key=lambda n: stage_ms[n])
    jd = STAGES.index(dom)
    if fused_routing(cfg) and not rep:
        # one kernel spans stages 0-1 and one spans 3-4; the two boundaries between them coincide
        stage_ms = {("router_topk_ranks" if n == "router" else "scatter" if n == "permute" else n): v
                    for n, v in stage_ms.items() if n not in ("topk", "histogram_lis_ranks")}
        dom = {"router": "router_topk_ranks", "permute": "scatter"}.get(dom, dom)
    K = steps if steps else max(3, int(math.ceil(min_timed_ms / max(prof_step_ms, 1e-3))))

    def timed(nsteps):
        """nsteps steps, CUDA events on the launching stream, L2 flushed between steps;
        returns (mean step ms, mean dominant-kernel ms, clock report)."""
        ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(nsteps)]
        ev_dom = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(nsteps)]
        with torch.cuda.stream(s):
            for evs in ev_dom:
                for e in evs:
                    e.record(s)
        sampler = ClockSampler(dev.index)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        sampler.start()
        with torch.cuda.stream(s):
            for i in range(nsteps):
                flush.zero_()
                hook = [None] * 8
                hook[jd], hook[jd + 1] = ev_dom[i][0], ev_dom[i][1]
                moe.moe_set_stage_events(hook)
                ev_s[i].record(s)
                fwd()
                ev_e[i].record(s)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        sampler.stop()
        moe.moe_set_stage_events([])
        ms_ = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(nsteps)) / nsteps
        dom_ = sum(ev_dom[i][0].elapsed_time(ev_dom[i][1]) for i in range(nsteps)) / nsteps
        st_ = moe.moe_read_device_status(ws, stream=s)
        if st_ != moe.OK:
            raise RuntimeError(f"device status after the timed steps: {moe.moe_status_string(st_)}")
        return ms_, dom_, sampler.report()

    ms_local, dom_ms, clocks = timed(K)
    sustained = None
    if sustained_ms > 0 and K * ms_local < sustained_ms:
        Ks = int(math.ceil(sustained_ms / max(ms_local, 1e-3)))
        s_ms, s_dom, s_clocks = timed(Ks)
        sustained = {"steps": Ks, "ms_per_step": s_ms, "dom_ms": s_dom, "clocks": s_clocks}

    e2e = None
    if with_e2e:
        # ---- end to end through the C ABI: pinned host batch in, result out, every step
        raw = (lambda t: t.view(torch.int16)) if tdt == torch.bfloat16 else (lambda t: t)
        x_host = torch.from_numpy(inp["x"].view(np.int16) if inp["x"].dtype == np.uint16 else inp["x"]).pin_memory()
        out_hosts = [torch.empty(out.shape, dtype=torch.int16 if tdt == torch.bfloat16 else torch.float32)
                     .pin_memory() for _ in range(2)]
        x_devs = [raw(torch.empty_like(d_in["x"])) for _ in range(2)]
        out_devs = [torch.empty_like(out) for _ in range(2)]
        Ke = max(3, min(K, 100))
        if world > 1:
            dist.barrier()
        # the C ABI takes raw device pointers, so bf16 buffers travel as int16 views
        e2e_local = e2e_pipelined(torch, lambda xd, od: fwd(x=xd, o=od), x_host, x_devs, [raw(o) for o in out_devs],
                                  out_hosts, Ke, s, dev)
        if world > 1:
            dist.barrier()
        e2e = {"ms_local": e2e_local, "h2d": x_host.numel() * x_host.element_size(),
               "d2h": out_hosts[0].numel() * out_hosts[0].element_size()}

    cfg_groups = dataclasses.replace(cfg, m=cfg.m + 1) if rep else cfg  # the replica is one more routed group
    plan_ksplit = _down_ksplit(cfg, cfg_groups, fp8)
    costs, layer_flops, layer_bytes = stage_costs(cfg_groups, active, plan_ksplit, weight_bytes=1 if fp8 else None)
    extra = {}
    if floe is not None:
        # dense up projection: W_up only, u written in fp32; sparse part: the gate and
        # down rows of the kept channels, u and the compact h
        kc = kept.cpu().numpy().astype(np.int64)
        Tk = cfg.T * cfg.k
        costs["expert_up"] = (2.0 * cfg.f * cfg.d * Tk, active * cfg.f * cfg.d * 2 + Tk * cfg.d * 2 + Tk * cfg.f * 4)
        costs["expert_down"] = (4.0 * cfg.d * float(kc.sum()) * max(1.0, Tk / max(active, 1)),
                                float(kc.sum()) * 2 * cfg.d * 2 + Tk * cfg.f * 8 + Tk * cfg.d * 4)
        layer_bytes = (cfg.m * cfg.d + active * cfg.f * cfg.d + float(kc.sum()) * 2 * cfg.d) * 2 + 2 * T_bytes(cfg)
        extra["kept_channel_fraction"] = float(kc[kc > 0].mean() / cfg.f)
    if glob:
        gmx, gam, glv = moe.unpack_lis(glis)
        extra["global_lis"] = {"lis": glv, "max_count": gmx, "heavy_hitter": gam, "ranks": world,
                               "note": "per-expert counts summed over all ranks every step (all-reduce of m int32) "
                                       "and the LIS of the whole job's batch; routing.lis is the rank's own"}
    if rep:
        extra["lis_before_split"] = moe.unpack_lis(lis0)[2]
        extra["heavy_hitter_before_split"] = moe.unpack_lis(lis0)[1]
    return {"K": K, "Kp": Kp, "ms_local": ms_local, "dom": dom, "dom_ms": dom_ms, "clocks": clocks,
            "sustained": sustained, "e2e": e2e, "stage_ms": stage_ms, "costs": costs, "layer_flops": layer_flops,
            "layer_bytes": layer_bytes, "launches_per_step": launches_per_step, "inp": inp, "fp8": fp8,
            "routing": {"lis": lis_v, "max_count": max_count, "heavy_hitter": argmax, "active_experts": active,
                        "reuse_ratio": cfg.T * cfg.k / max(active, 1), "load_entropy": entropy},
            "extra": extra}


def workload_summary(cfg, r: dict, world: int) -> dict:
    """A workload measured beside the headline one: its own step time, tokens/s,
    dominant-kernel roofline (against the peak its timed length calls for), layer
    roofline, stage breakdown, routing statistics and clocks."""
    pk, pk_src = peaks()
    ms = r["ms_local"]
    long_step = sustained_applies(r["K"], ms, r.get("clocks"))
    fl, by = r["costs"][r["dom"]]
    roof = roofline_for(cfg, r["dom"], fl, by, r["dom_ms"], pk, pk_src, long_step, r["fp8"],
                        cfg.name + ("_fp8" if r["fp8"] else ""))
    tensor_peak = (pk["bf16_tflops_sustained"] if long_step else pk["bf16_tflops"]) * (2.0 if r["fp8"] else 1.0)
    t_layer = max(r["layer_flops"] / (tensor_peak * 1e12), r["layer_bytes"] / (pk["hbm_gbs"] * 1e9))
    return {"config": workload_config(cfg), "value": world * cfg.T / (ms * 1e-3), "unit": UNIT, "steps": r["K"],
            "ms_per_step": ms, "timed_region_ms": r["K"] * ms, "roofline": roof,
            "layer_roofline": {"time_us": t_layer * 1e6, "frac": t_layer / (ms * 1e-3), "flops": r["layer_flops"],
                               "bytes": r["layer_bytes"]},
            "stages_us": {k: v * 1e3 for k, v in r["stage_ms"].items()}, "routing": r["routing"],
            "gpu_launches": r["K"] * r["launches_per_step"], "clocks": r["clocks"]}


def ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} needs {args.gpus} ranks (torchrun), found WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    cfg = W.CONFIGS[args.config]
    rep, floe, fp8 = args.replicate, args.floe, args.fp8
    variant = rep or floe is not None or fp8
    r = layer_run(cfg, args, dev, rank, world, dist, args.steps, args.warmup, with_e2e=True,
                  sustained_ms=SUSTAINED_MS if (world == 1 and not variant and not args.no_extra) else 0.0)
    # ---- max over ranks
    ms, e2e_ms = max_over_ranks([r["ms_local"], r["e2e"]["ms_local"]], dist, dev)
    K = r["K"]
    pk, pk_src = peaks()
    long_step = sustained_applies(K, ms, r.get("clocks"))
    fl, by = r["costs"][r["dom"]]
    roof = roofline_for(cfg, r["dom"], fl, by, r["dom_ms"], pk, pk_src, long_step, fp8,
                        cfg.name + ("_fp8" if fp8 else "") + ("_floe" if floe is not None else "")
                        + ("_replicated" if rep else ""))
    tensor_peak = (pk["bf16_tflops_sustained"] if long_step else pk["bf16_tflops"]) * (2.0 if fp8 else 1.0)
    t_layer = max(r["layer_flops"] / (tensor_peak * 1e12), r["layer_bytes"] / (pk["hbm_gbs"] * 1e9))
    variant_note = {}
    if floe is not None:
        variant_note = {"variant": f"FloE contextual sparsity at target sparsity {floe}: thresholds from a second "
                                   "batch; expert_up = dense u = x W_up^T, expert_down = kept lists + kept gate rows + "
                                   "kept down rows"}
    elif fp8:
        variant_note = {"variant": "8-bit experts: E4M3 weights with one fp32 scale per output channel (quantized "
                                   "once, outside the timing); x and h rows quantized per row inside each step; router "
                                   "in bf16",
                        "dtype_note": "expert GEMMs e4m3 x e4m3 with fp32 accumulation; router bf16"}
    elif rep:
        variant_note = {"variant": "R&Q replica dispatch: the heavy-hitter's tasks alternate between it and a replica "
                                   "expert m that computes with its bf16 weights; routing.lis is over the m + 1 experts"}
    line = {"metric": METRIC, "value": world * cfg.T / (ms * 1e-3), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3" if fp8 else "bf16" if cfg.dtype == W.BF16 else "f32",
            "data": "synthetic (seeded generator; x ~ N(0,1), weights ~ N(0, 1/sqrt(fan_in)), Zipf router bias)",
            "config": dict(run_config(cfg, world),
                           **({"expert_weights": "e4m3, per-channel fp32 scales"} if fp8 else {})),
            "roofline": roof,
            "layer_roofline": {"time_us": t_layer * 1e6, "frac": t_layer / (ms * 1e-3),
                               "flops": r["layer_flops"], "bytes": r["layer_bytes"]},
            "stages_us": {k: v * 1e3 for k, v in r["stage_ms"].items()},
            "stages_note": f"per-kernel breakdown from a separate {r['Kp']}-step pass with an event at every stage "
                           "boundary (serialised launches); the timed region records only the dominant kernel's "
                           "boundaries",
            "routing": r["routing"], **variant_note, **r["extra"],
            "e2e": {"value": world * cfg.T / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": r["e2e"]["h2d"],
                    "d2h_bytes_per_step": r["e2e"]["d2h"], "ms_per_step": e2e_ms,
                    "note": "pinned host -> device batch upload and device -> host output download every step, on "
                            "their own streams, overlapped with the neighbouring steps' forward (double-buffered)"},
            "gpu_launches": K * r["launches_per_step"], "launches_per_step": r["launches_per_step"],
            "clocks": r["clocks"]}
    if r["sustained"] is not None:
        su = r["sustained"]
        roof_s = roofline_for(cfg, r["dom"], fl, by, su["dom_ms"], pk, pk_src, True, fp8, cfg.name)
        line["sustained"] = {"steps": su["steps"], "ms_per_step": su["ms_per_step"],
                             "value": cfg.T / (su["ms_per_step"] * 1e-3), "unit": UNIT,
                             "timed_region_ms": su["steps"] * su["ms_per_step"], "roofline": roof_s,
                             "clocks": su["clocks"],
                             "note": "the same workload timed again for over a second after the headline steps, so "
                                     "the clocks settle under the power cap; its roofline uses the sustained peak"}
    inp = r["inp"]
    del r
    if world == 1 and not variant and not args.no_extra:
        # the other single-GPU workloads the targets name, each timed long enough for
        # the clock sampler to see a steady state
        torch.cuda.empty_cache()
        extras = {}
        for name in EXTRA_WORKLOADS:
            if name == cfg.name:
                continue
            xc = W.CONFIGS[name]
            rx = layer_run(xc, args, dev, rank, world, dist, None, args.warmup, with_e2e=False,
                           min_timed_ms=EXTRA_MIN_MS)
            extras[name] = workload_summary(xc, rx, world)
            del rx
            torch.cuda.empty_cache()
        line["workloads"] = extras
    if world > 1:
        dist.barrier()
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = (cpu_oracle_fp8_sample(cfg, inp, args.cpu_seconds) if fp8
                                    else cpu_oracle_sample(cfg, inp, args.cpu_seconds))
        else:
            line["cpu_baseline"] = None
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# ------------------------------------------------------------------ atomic-expert workload

ATOMIC_STAGES = ["router_projections", "grid_topk", "experts", "end"]  # experts: coef + assembly, one launch


def atomic_config(cfg) -> dict:
    return {"workload": cfg.name, "tokens": cfg.T, "d_model": cfg.d, "grid": f"{cfg.Nr}x{cfg.Nc}", "experts": cfg.N,
            "top_k": cfg.K, "activation": "silu" if cfg.act == W.ACT_SILU else "sigmoid", "description": cfg.note}


def atomic_stage_costs(cfg, active: int, ksplit: int):
    T, d, n = cfg.T, cfg.d, cfg.Nr + cfg.Nc
    c = {"router_projections": (2.0 * T * d * n, n * d * 2 + T * d * 2 + ksplit * T * n * 4),
         "grid_topk": (0.0, ksplit * T * n * 4 + T * cfg.K * 8),
         "experts": (4.0 * T * cfg.K * d, 2 * active * d * 2 + 2 * T * d * 2 + 2 * T * cfg.K * 8),
         "end": (0.0, 0.0)}
    layer_flops = 2.0 * T * d * n + 4.0 * T * cfg.K * d
    layer_bytes = n * d * 2 + 2 * active * d * 2 + 2 * T * d * 2
    return c, layer_flops, layer_bytes


def cpu_oracle_atomic(cfg, inp, budget_s: float):
    import oracle as O

    def run(n):
        t0 = time.perf_counter()
        x = np.ascontiguousarray(inp["x"][:n])
        lr, lc = O.atomic_logprobs(x, inp["w_row"], inp["w_col"])
        idx, g = O.atomic_select(lr, lc, cfg.K)
        O.atomic_output(x, inp["w_in"], inp["w_out"], idx, g, cfg.act)
        return time.perf_counter() - t0

    n = 1
    dt = run(n)
    while dt < budget_s / 4 and n < cfg.T:
        n = min(cfg.T, n * 2)
        dt = run(n)
    return {"value": n / dt, "unit": UNIT, "cores": 1, "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"first {n} of {cfg.T} tokens of the {cfg.name} workload; Cartesian router, exact grid top-K "
                      f"(brute-force sort of all {cfg.N} scores per token) and atomic experts, fp64 C, one thread"}


def ours_atomic(args):
    import torch

    import sparse_mixture_experts_08_b200 as moe

    if int(os.environ.get("WORLD_SIZE", "1")) != 1 or args.gpus != 1:
        raise SystemExit("the atomic-expert workload is benchmarked on one GPU")
    cfg = W.CONFIGS[args.config]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    inp = W.make_atomic_inputs(cfg)
    d_in = {k: torch.from_numpy(v.view(np.int16)).to(dev).view(torch.bfloat16) for k, v in inp.items()}
    c = moe.make_atomic_config(cfg.T, cfg.d, cfg.Nr, cfg.Nc, cfg.K, cfg.act)
    ws = moe.workspace(c, device=dev)
    out = torch.empty((cfg.T, cfg.d), dtype=torch.bfloat16, device=dev)
    idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device=dev)
    s = torch.cuda.Stream(device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def fwd(x=None):
        moe.moe_atomic_forward(c, d_in["x"] if x is None else x, d_in["w_row"], d_in["w_col"], d_in["w_in"],
                               d_in["w_out"], out, ws, idx_out=idx, stream=s)

    with torch.cuda.stream(s):
        n0 = moe.moe_launch_count()
        fwd()
        launches_per_step = moe.moe_launch_count() - n0
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            fwd()
    torch.cuda.synchronize(dev)
    if moe.moe_read_device_status(ws, stream=s) != moe.OK:
        raise RuntimeError("device status after warm-up is not OK")
    active = int(np.unique(idx.cpu().numpy()).size)
    Kp = max(3, min(args.steps, 50))
    ev_prof = [[torch.cuda.Event(enable_timing=True) for _ in range(5)] for _ in range(Kp)]
    with torch.cuda.stream(s):
        for evs in ev_prof:
            for e in evs:
                e.record(s)
        for i in range(Kp):
            flush.zero_()
            moe.moe_set_stage_events(ev_prof[i])
            fwd()
    torch.cuda.synchronize(dev)
    moe.moe_set_stage_events([])
    stage_ms = {name: sum(ev_prof[i][j].elapsed_time(ev_prof[i][j + 1]) for i in range(Kp)) / Kp
                for j, name in enumerate(ATOMIC_STAGES)}
    stage_ms.pop("end")  # the library records its last two boundaries together
    dom = max(stage_ms, key=lambda n: stage_ms[n])
    jd = ATOMIC_STAGES.index(dom)
    K = args.steps
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_e = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_dom = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    with torch.cuda.stream(s):
        for evs in ev_dom:
            for e in evs:
                e.record(s)
    sampler = ClockSampler(0)
    torch.cuda.synchronize(dev)
    sampler.start()
    with torch.cuda.stream(s):
        for i in range(K):
            flush.zero_()
            hook = [None] * 5
            hook[jd], hook[jd + 1] = ev_dom[i][0], ev_dom[i][1]
            moe.moe_set_stage_events(hook)
            ev_s[i].record(s)
            fwd()
            ev_e[i].record(s)
    torch.cuda.synchronize(dev)
    sampler.stop()
    moe.moe_set_stage_events([])
    ms = sum(ev_s[i].elapsed_time(ev_e[i]) for i in range(K)) / K
    dom_ms = sum(ev_dom[i][0].elapsed_time(ev_dom[i][1]) for i in range(K)) / K
    # end to end: token batch from pinned host memory, output back, every step (pipelined)
    x_host = torch.from_numpy(inp["x"].view(np.int16)).pin_memory()
    out_hosts = [torch.empty(out.shape, dtype=torch.int16).pin_memory() for _ in range(2)]
    x_devs = [torch.empty_like(d_in["x"]).view(torch.int16) for _ in range(2)]
    out_devs = [torch.empty_like(out) for _ in range(2)]

    def fwd2(xd, od):
        moe.moe_atomic_forward(c, xd.view(torch.bfloat16), d_in["w_row"], d_in["w_col"], d_in["w_in"], d_in["w_out"],
                               od, ws, stream=s)

    Ke = max(3, min(K, 100))
    e2e_ms = e2e_pipelined(torch, lambda xd, od: fwd2(xd, od), x_host, x_devs, [o.view(torch.int16) for o in out_devs],
                           out_hosts, Ke, s, dev)
    pk, pk_src = peaks()
    ksplit = 16  # the router projections' split-K partials per logit (tensor-core tiles)
    costs, layer_flops, layer_bytes = atomic_stage_costs(cfg, active, ksplit)
    fl, by = costs[dom]
    roof = {"bound": "hbm", "achieved": by / (dom_ms * 1e-3) / 1e9, "peak": pk["hbm_gbs"], "unit": "GB/s",
            "peak_source": f"{pk_src} hbm copy"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof.update(traffic=traffic_for(cfg.name, dom), kernel=dom, algorithmic_bytes=by, algorithmic_flops=fl,
                duration_us=dom_ms * 1e3)
    t_layer = max(layer_flops / (pk["bf16_tflops"] * 1e12), layer_bytes / (pk["hbm_gbs"] * 1e9))
    line = {"metric": METRIC, "value": cfg.T / (ms * 1e-3), "unit": UNIT, "n_gpus": 1, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded generator; x ~ N(0,1), router and w_in ~ N(0, 1/sqrt(d)), w_out ~ N(0,1))",
            "config": dict(atomic_config(cfg), parallelism="single GPU",
                           l2=f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write, outside the timed events)",
                           launch="eager C-ABI call per step"),
            "roofline": roof,
            "layer_roofline": {"time_us": t_layer * 1e6, "frac": t_layer / (ms * 1e-3), "flops": layer_flops,
                               "bytes": layer_bytes},
            "stages_us": {k: v * 1e3 for k, v in stage_ms.items()},
            "routing": {"active_experts": active, "reuse_ratio": cfg.T * cfg.K / max(active, 1)},
            "e2e": {"value": cfg.T / (e2e_ms * 1e-3), "unit": UNIT, "h2d_bytes_per_step": x_host.numel() * 2,
                    "d2h_bytes_per_step": out_hosts[0].numel() * 2, "ms_per_step": e2e_ms,
                    "note": "pinned host -> device batch upload and device -> host output download every step, on "
                            "their own streams, overlapped with the neighbouring steps' forward (double-buffered)"},
            "gpu_launches": K * launches_per_step, "launches_per_step": launches_per_step,
            "clocks": sampler.report()}
    line["cpu_baseline"] = None if args.no_cpu_baseline else cpu_oracle_atomic(cfg, inp, args.cpu_seconds)
    print(json.dumps(line), flush=True)
    return 0


def router_only(args):
    """The routing call alone: K steps after W warm-ups, L2 flush between steps outside the events."""
    import torch

    import sparse_mixture_experts_08_b200 as moe

    cfg = W.CONFIGS[args.config]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    s = torch.cuda.Stream(device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
    if isinstance(cfg, W.AtomicWorkload):
        inp = W.make_atomic_inputs(cfg, experts=False)
        c = moe.make_atomic_config(cfg.T, cfg.d, cfg.Nr, cfg.Nc, cfg.K, cfg.act)
        x, wr, wc = bf(inp["x"]), bf(inp["w_row"]), bf(inp["w_col"])
        idx = torch.empty((cfg.T, cfg.K), dtype=torch.int32, device=dev)
        g = torch.empty((cfg.T, cfg.K), dtype=torch.float32, device=dev)
        ws = moe.workspace(c, device=dev)

        def call():
            moe.moe_atomic_route(c, x, wr, wc, None, None, idx, g, ws, stream=s)
    else:
        inp = W.make_moe_inputs(cfg, weights=False)
        c = moe.make_config(cfg.T, cfg.d, cfg.f, cfg.m, cfg.k, cfg.n_shared, cfg.f_shared, cfg.dtype, cfg.act,
                            cfg.renorm)
        conv = bf if cfg.dtype == W.BF16 else (lambda a: torch.from_numpy(a).to(dev))
        x, wr = conv(inp["x"]), conv(inp["w_router"])
        bias = None if inp.get("bias") is None else torch.from_numpy(inp["bias"]).to(dev)
        idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
        w = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
        ws = moe.workspace(c, device=dev)

        def call():
            moe.moe_route(c, x, wr, bias, None, None, idx, w, ws, stream=s)
    with torch.cuda.stream(s):
        n0 = moe.moe_launch_count()
        call()
        launches = moe.moe_launch_count() - n0
        for _ in range(max(args.warmup, 3)):
            flush.zero_()
            call()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    with torch.cuda.stream(s):
        for a, b in ev:
            flush.zero_()
            a.record(s)
            call()
            b.record(s)
    torch.cuda.synchronize(dev)
    if moe.moe_read_device_status(ws, stream=s) != moe.OK:
        raise RuntimeError("device status after the router runs is not OK")
    ms = sum(a.elapsed_time(b) for a, b in ev) / len(ev)
    print(json.dumps({"mode": "router-only", "config": {"workload": cfg.name}, "ms_per_step": ms,
                      "tokens_per_s": cfg.T / (ms * 1e-3), "gpu_launches_per_step": launches}), flush=True)
    return 0


def main():
    args = parse()
    atomic = isinstance(W.CONFIGS[args.config], W.AtomicWorkload)
    if args.router_only:
        return router_only(args)
    if args.impl == "reference":
        if atomic:
            raise SystemExit("--impl reference covers the coarse-expert workloads")
        return reference_arm(args)
    return ours_atomic(args) if atomic else ours(args)


if __name__ == "__main__":
    sys.exit(main())
