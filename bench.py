#!/usr/bin/env python3
"""Benchmark of the delta-rule layer: chunked prefill + decode step on B200.

One step = the whole hot path over one batch of synthetic inputs resident in
HBM:
  * chunked prefill of a Gated DeltaNet batch: B=4 sequences, H=16 heads,
    T=4096 tokens, d_k=d_v=128, bf16 q/k/v, fp32 beta/g, chunk 64, returning o
    and the final fp32 state (dn_chunk_fwd);
  * one recurrent decode step of a serving batch: B=256 sequences, H=32 heads,
    d_k=d_v=128, fp32 state resident in HBM and updated in place, one bf16
    token per sequence (dn_decode_step; token sets cycle through a bank of 16).

value = (prefill tokens + decode tokens) per second = (4*4096 + 256) / step
time, summed over ranks (each rank runs its own copy of the workload: the
heads and sequences are independent, so there is no data-path collective).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--path auto|simt|tc] [--no-cpu-baseline] [--no-e2e]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "delta-rule layer prefill tokens/s + decode tokens/s, % of tensor/HBM roofline"
C = 64


def prefill_flops(B, H, T, dk, dv, chunk=C):
    """Counted FLOPs of the chunked form (each matmul 2mnk, each triangular solve
    C^2 n, full C x C products): 5 C^2 d_k + 3 C^2 d_v + 6 C d_k d_v per chunk."""
    n_chunks = B * H * ((T + chunk - 1) // chunk)
    return n_chunks * (5 * chunk * chunk * dk + 3 * chunk * chunk * dv + 6 * chunk * dk * dv)


def prefill_bytes(B, H, T, dk, dv, esz=2, gate_per_key=False, s0=False, st=True):
    """Algorithmic HBM bytes: q, k, v and o once in their dtype, beta and g fp32
    once, S0 / S_T fp32 once when present."""
    tok = B * H * T
    g = 4 * (dk if gate_per_key else 1)
    b = tok * (esz * (2 * dk + 2 * dv) + 4 + g)
    b += (B * H * dk * dv * 4) * (int(s0) + int(st))
    return b


def decode_bytes(B, H, dk, dv, esz=2):
    """State read + written once (fp32) plus the token vectors and o."""
    return B * H * (2 * dk * dv * 4 + esz * (2 * dk + 2 * dv) + 8)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


def sources_sha256(paths):
    """sha256 over the concatenated contents of the given repo-relative files."""
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_for(kernel_key):
    """DRAM bytes per launch (per call, for a path of several kernels) from a
    committed ncu summary, if none of the sources has changed since it was
    captured (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            tab = json.load(f)
        ent = tab[kernel_key]
        if sources_sha256(ent["sources"]) != ent["sources_sha256"]:
            return None
        return float(ent["dram_bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """SM clock and clock-event (throttle) reasons, polled through NVML from a
    background thread for the whole timed region (nvidia-smi as a fallback).
    The reasons reported are the union over samples."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device_id):
        self.device_id = device_id
        self.samples = []
        self._stop = None

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            if isinstance(self.device_id, str):
                h = pynvml.nvmlDeviceGetHandleByUUID(self.device_id)
            else:
                h = pynvml.nvmlDeviceGetHandleByIndex(int(self.device_id))
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            getr = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons

            def poll():
                while not self._stop.is_set():
                    try:
                        self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM), getr(h)))
                    except Exception:
                        pass
                    self._stop.wait(0.002)
            self._thread = threading.Thread(target=poll, daemon=True)
            self._thread.start()
        except Exception:
            self._thread = None
            self.max_mhz = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0,
                    "source": "nvml"}
        reasons = sorted({name for _, r in self.samples for bit, name in self.REASONS.items() if r & bit})
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples), "source": "nvml"}


def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def max_over_ranks(x, world, device="cuda"):
    """The largest value of x over all ranks (a timing, so the slowest rank wins)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, ms_per_step, world):
    """Whole-job units per second: every rank processes its own units per step
    (weak scaling) and the step time is the slowest rank's."""
    return world * units_per_rank_step / (ms_per_step * 1e-3)


def barrier(world):
    import torch
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# CPU oracle timing (the cpu_baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def oracle_sample_rate(prefill_heads=64, decode_heads=8192, seed_offset=0):
    """Time the fp64 oracle on a bounded sample of the same workload and scale
    to the whole step: returns (tokens/s, seconds per full step, description)."""
    import numpy as np
    import oracle
    from delta_rule_recurrent_02_b200 import workloads as W
    cfg = W.GDN_PREFILL
    inp = W.gen_prefill(1, prefill_heads, cfg.T, cfg.dk, cfg.dv, dtype=cfg.dtype, gate=cfg.gate,
                        seed=cfg.seed + seed_offset, q_norm=True, g_shift=cfg.g_shift)
    f = lambda t: None if t is None else t.double().numpy()
    args = [f(inp[n]) for n in ("q", "k", "v", "beta", "g")]
    t0 = time.perf_counter()
    oracle.delta_rule(*args, None, scale=cfg.scale)
    tp = time.perf_counter() - t0
    dc = W.DECODE
    dinp = W.gen_decode(dc, B=1, H=decode_heads, bank=1)
    dargs = [f(dinp[n][0])[:, :, None] for n in ("q", "k", "v")]
    db = f(dinp["beta"][0])[:, :, None]
    dg = f(dinp["g"][0])[:, :, None]
    S = f(dinp["S"])
    t0 = time.perf_counter()
    oracle.delta_rule(dargs[0], dargs[1], dargs[2], db, dg, S, scale=dc.scale)
    td = time.perf_counter() - t0
    full_p = tp * (cfg.B * cfg.H) / prefill_heads
    full_d = td * (dc.B * dc.H) / decode_heads
    tokens = cfg.B * cfg.T + dc.B
    desc = (f"{prefill_heads} of {cfg.B * cfg.H} prefill heads (T={cfg.T}) in {tp:.2f} s and "
            f"{decode_heads} of {dc.B * dc.H} decode heads in {td:.3f} s, scaled by head count to "
            f"one full step ({full_p + full_d:.1f} s)")
    return tokens / (full_p + full_d), full_p + full_d, desc, (tokens, full_p, full_d)


def oracle_single_thread(prefill_heads=4):
    """The fp64 oracle on one host thread for the small DeltaNet workload (whole)
    and for the bench-size Gated DeltaNet prefill (a sample of heads, scaled to
    all of them): {workload: {"s": seconds, "tokens_per_s": ..., "sample": ...}}."""
    import oracle
    from delta_rule_recurrent_02_b200 import workloads as W
    f = lambda t: None if t is None else t.double().numpy()
    out = {}
    cfg = W.DELTANET_SMALL
    inp = W.gen_prefill_config(cfg)
    t0 = time.perf_counter()
    oracle.delta_rule(*(f(inp[n]) for n in ("q", "k", "v", "beta", "g", "S0")), scale=cfg.scale, nthreads=1)
    s = time.perf_counter() - t0
    out[cfg.name] = {"s": s, "tokens_per_s": cfg.B * cfg.T / s, "sample": "whole workload"}
    cfg = W.GDN_PREFILL
    inp = W.gen_prefill(1, prefill_heads, cfg.T, cfg.dk, cfg.dv, dtype=cfg.dtype, gate=cfg.gate, seed=cfg.seed,
                        q_norm=True, g_shift=cfg.g_shift)
    t0 = time.perf_counter()
    oracle.delta_rule(*(f(inp[n]) for n in ("q", "k", "v", "beta", "g")), None, scale=cfg.scale, nthreads=1)
    s = (time.perf_counter() - t0) * (cfg.B * cfg.H) / prefill_heads
    out[cfg.name] = {"s": s, "tokens_per_s": cfg.B * cfg.T / s,
                     "sample": f"{prefill_heads} of {cfg.B * cfg.H} heads, scaled by head count"}
    return out


def run_reference(args):
    """The reference arm: the fp64 oracle timed as it stands on the host cores."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    vals = []
    desc = ""
    for s in range(args.warmup + args.steps):
        v, secs, desc, _ = oracle_sample_rate(prefill_heads=16, decode_heads=2048, seed_offset=s)
        if s >= args.warmup:
            vals.append(v)
    value = statistics.median(vals)
    tokens = 4 * 4096 + 256
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tokens / value,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(),
                             "nproc": os.cpu_count(), "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def measure_prefill_configs(dn, torch, W, peaks, dev, stream, calls=5, warm=2):
    """Each prefill workload of the method alone (small DeltaNet, long Gated
    DeltaNet, KDA): median of `calls` CUDA-event-timed calls after `warm`, with
    the path the library picks, against the counted FLOPs and algorithmic
    bytes.  The bench-size Gated DeltaNet prefill is the step's own."""
    out = {}
    for cfg in (W.DELTANET_SMALL, W.GDN_LONG, W.KDA_PREFILL):
        inp = W.gen_prefill_config(cfg)
        d = {k: (None if v is None else v.to(dev)) for k, v in inp.items()}
        o = torch.empty((cfg.B, cfg.H, cfg.T, cfg.dv), dtype=W.torch_dtype(cfg.dtype), device=dev)
        S_T = torch.empty((cfg.B, cfg.H, cfg.dk, cfg.dv), dtype=torch.float32, device=dev)
        nws = dn.dn_chunk_fwd_workspace_size(cfg.B, cfg.T, cfg.H, cfg.dk, cfg.dv, chunk=cfg.chunk,
                                             dtype=cfg.dtype, gate=cfg.gate)
        ws = torch.empty(nws, dtype=torch.uint8, device=dev) if nws else None

        def call():
            dn.dn_chunk_fwd(d["q"], d["k"], d["v"], d["beta"], d["g"], d["S0"], o, S_T, chunk=cfg.chunk,
                            scale=cfg.scale, workspace=ws, stream=stream)

        for _ in range(warm):
            call()
        k0 = dn.dn_kernel_launches()
        call()
        launches = dn.dn_kernel_launches() - k0
        ts = []
        for _ in range(calls):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            call()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        dn.dn_device_status(stream)
        ms = statistics.median(ts)
        esz = 2 if cfg.dtype == "bf16" else 4
        fl = prefill_flops(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, cfg.chunk)
        by = prefill_bytes(cfg.B, cfg.H, cfg.T, cfg.dk, cfg.dv, esz=esz, gate_per_key=cfg.gate == "per_key",
                           s0=cfg.s0_std is not None)
        tf = fl / (ms * 1e-3) / 1e12
        gb = by / (ms * 1e-3) / 1e9
        out[cfg.name] = {"ms_per_call": ms, "tokens_per_s": cfg.B * cfg.T / (ms * 1e-3),
                         "path": "tensor cores" if nws else "simt (fp32 CUDA cores)",
                         "kernel_launches_per_call": launches,
                         "counted_flops": fl, "algorithmic_bytes": by,
                         "tensor_tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"],
                         "hbm_gbs": gb, "hbm_frac": gb / peaks["hbm_gbs"],
                         "traffic": (traffic_for("kda_tc" if nws else "chunk_simt_kda")
                                     if cfg is W.KDA_PREFILL else None),
                         "timing": f"median of {calls} calls after {warm}, CUDA events"}
        del d, o, S_T, ws
        torch.cuda.empty_cache()
    out["gated_deltanet_layer_prologue_bf16_B4_H16_T4096_d128"] = measure_gdn_prologue(dn, torch, W, peaks, dev,
                                                                                        stream, calls, warm)
    return out


def measure_gdn_prologue(dn, torch, W, peaks, dev, stream, calls=5, warm=2):
    """The bench-size Gated DeltaNet prefill with the layer's prologue fused in
    (dn_chunk_fwd_gdn: raw q and k normalised inside, beta and g from the raw b,
    a and the per-head A_log, dt_bias), same shape and timing as above."""
    pc = W.GDN_PREFILL
    gen = torch.Generator().manual_seed(pc.seed)
    B, H, T, dk, dv = pc.B, pc.H, pc.T, pc.dk, pc.dv
    q = (torch.randn(B, H, T, dk, generator=gen) * 2).to(torch.bfloat16).to(dev)
    k = (torch.randn(B, H, T, dk, generator=gen) * 2).to(torch.bfloat16).to(dev)
    v = torch.randn(B, H, T, dv, generator=gen).to(torch.bfloat16).to(dev)
    b = torch.randn(B, H, T, generator=gen).to(dev)
    a = torch.randn(B, H, T, generator=gen).to(dev)
    A_log = torch.log(1 + 15 * torch.rand(H, generator=gen)).to(dev)
    dt_bias = torch.randn(H, generator=gen).to(dev)
    o = torch.empty((B, H, T, dv), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((B, H, dk, dv), dtype=torch.float32, device=dev)
    ws = torch.empty(dn.dn_chunk_fwd_workspace_size(B, T, H, dk, dv, path="tc"), dtype=torch.uint8, device=dev)

    def call():
        dn.dn_chunk_fwd_gdn(q, k, v, b, a, A_log, dt_bias, None, o, S_T, scale=pc.scale, workspace=ws,
                            stream=stream)

    for _ in range(warm):
        call()
    ts = []
    for _ in range(calls):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    dn.dn_device_status(stream)
    ms = statistics.median(ts)
    fl = prefill_flops(B, H, T, dk, dv)
    by = prefill_bytes(B, H, T, dk, dv) + 2 * H * 4
    tf = fl / (ms * 1e-3) / 1e12
    gb = by / (ms * 1e-3) / 1e9
    return {"ms_per_call": ms, "tokens_per_s": B * T / (ms * 1e-3), "path": "tensor cores, layer prologue fused",
            "counted_flops": fl, "algorithmic_bytes": by, "tensor_tflops": tf,
            "tensor_frac": tf / peaks["bf16_tflops"], "hbm_gbs": gb, "hbm_frac": gb / peaks["hbm_gbs"],
            "traffic": None, "timing": f"median of {calls} calls after {warm}, CUDA events"}


def _time_calls(torch, call, stream, calls, warm):
    for _ in range(warm):
        call()
    ts = []
    for _ in range(calls):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        call()
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.median(ts)


def measure_next_rows(dn, torch, W, peaks, dev, stream, calls=5, warm=2):
    """The entry points beyond the bench step, each on a synthetic workload of
    the layer's shapes, CUDA-event timed (median of `calls` after `warm`):
    grouped value heads (16 key : 48 value heads), a packed batch of ragged
    sequences, the layer with its prologue and gated RMSNorm fused into the
    prefill and into the decode step, and the generalised (RWKV-7) rule."""
    out = {}
    hbm, tc = peaks["hbm_gbs"], peaks["bf16_tflops"]
    gen = torch.Generator().manual_seed(11)
    unit = lambda x: x / x.norm(dim=-1, keepdim=True)
    d, T, sc = 128, 4096, 128 ** -0.5

    def entry(name, ms, tokens, fl, by, path, bound="hbm"):
        e = {"ms_per_call": ms, "tokens_per_s": tokens / (ms * 1e-3), "path": path, "algorithmic_bytes": by,
             "hbm_gbs": by / (ms * 1e-3) / 1e9, "hbm_frac": by / (ms * 1e-3) / 1e9 / hbm, "bound": bound,
             "timing": f"median of {calls} calls after {warm}, CUDA events"}
        if fl:
            e.update({"counted_flops": fl, "tensor_tflops": fl / (ms * 1e-3) / 1e12,
                      "tensor_frac": fl / (ms * 1e-3) / 1e12 / tc})
        out[name] = e

    # grouped value heads: 16 key heads serve 48 value heads
    Hk, Hv = 16, 48
    q = unit(torch.randn(1, Hk, T, d, generator=gen)).to(torch.bfloat16).to(dev)
    k = unit(torch.randn(1, Hk, T, d, generator=gen)).to(torch.bfloat16).to(dev)
    v = torch.randn(1, Hv, T, d, generator=gen).to(torch.bfloat16).to(dev)
    beta = torch.sigmoid(torch.randn(1, Hv, T, generator=gen)).to(dev)
    g = (-torch.nn.functional.softplus(torch.randn(1, Hv, T, generator=gen) + 2)).to(dev)
    o = torch.empty((1, Hv, T, d), dtype=torch.bfloat16, device=dev)
    S = torch.empty((1, Hv, d, d), device=dev)
    ws = torch.empty(dn.dn_chunk_fwd_workspace_size(1, T, Hv, d, d), dtype=torch.uint8, device=dev)
    ms = _time_calls(torch, lambda: dn.dn_chunk_fwd_gva(q, k, v, beta, g, None, o, S, scale=sc, workspace=ws,
                                                        stream=stream), stream, calls, warm)
    by = Hk * T * d * 2 * 2 + Hv * T * (d * 2 * 2 + 8) + Hv * d * d * 4
    entry("gva_bf16_B1_Hk16_Hv48_T4096_d128", ms, T, prefill_flops(1, Hv, T, d, d), by,
          "tensor cores, q and k read once per key head")
    del q, k, v, beta, g, o, S, ws

    # a packed batch: 8 ragged sequences, 16384 tokens in all, 16 heads
    lens = [4096, 1000, 3000, 64, 1, 4095, 2048, 2080]
    Tt, H, N = sum(lens), 16, len(lens)
    q = unit(torch.randn(1, H, Tt, d, generator=gen)).to(torch.bfloat16).to(dev)
    k = unit(torch.randn(1, H, Tt, d, generator=gen)).to(torch.bfloat16).to(dev)
    v = torch.randn(1, H, Tt, d, generator=gen).to(torch.bfloat16).to(dev)
    beta = torch.sigmoid(torch.randn(1, H, Tt, generator=gen)).to(dev)
    g = (-torch.nn.functional.softplus(torch.randn(1, H, Tt, generator=gen) + 2)).to(dev)
    cu = torch.tensor([0] + [sum(lens[:i + 1]) for i in range(N)], dtype=torch.int32, device=dev)
    o = torch.empty((1, H, Tt, d), dtype=torch.bfloat16, device=dev)
    S = torch.empty((N, H, d, d), device=dev)
    ws = torch.empty(dn.dn_chunk_fwd_varlen_workspace_size(N, Tt, H, d, d), dtype=torch.uint8, device=dev)
    ms = _time_calls(torch, lambda: dn.dn_chunk_fwd_varlen(q, k, v, beta, g, None, o, S, cu, scale=sc, workspace=ws,
                                                           stream=stream), stream, calls, warm)
    fl = sum(prefill_flops(1, H, L, d, d) for L in lens if L)
    by = prefill_bytes(1, H, Tt, d, d, st=False) + N * H * d * d * 4 + (N + 1) * 4
    entry("varlen_bf16_N8_T16384_H16_d128", ms, Tt, fl, by, "tensor cores: chunk tables, WY kernel, state pass")
    del q, k, v, beta, g, o, S, ws, cu

    # the layer's prologue, the rule and the gated RMSNorm in one prefill (bench prefill shape)
    pc = W.GDN_PREFILL
    B, H = pc.B, pc.H
    q = (torch.randn(B, H, T, d, generator=gen) * 2).to(torch.bfloat16).to(dev)
    k = (torch.randn(B, H, T, d, generator=gen) * 2).to(torch.bfloat16).to(dev)
    v = torch.randn(B, H, T, d, generator=gen).to(torch.bfloat16).to(dev)
    b = torch.randn(B, H, T, generator=gen).to(dev)
    a = torch.randn(B, H, T, generator=gen).to(dev)
    A_log = torch.log(1 + 15 * torch.rand(H, generator=gen)).to(dev)
    dt_bias = torch.randn(H, generator=gen).to(dev)
    z = torch.randn(B, T, H, d, generator=gen).to(torch.bfloat16).to(dev)
    nw = torch.ones(d, device=dev)
    y = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=dev)
    S = torch.empty((B, H, d, d), device=dev)
    ws = torch.empty(dn.dn_chunk_fwd_workspace_size(B, T, H, d, d, path="tc"), dtype=torch.uint8, device=dev)
    ms = _time_calls(torch, lambda: dn.dn_chunk_fwd_gdn_ex(q, k, v, b, a, A_log, dt_bias, None, y, S, scale=sc,
                                                           path="tc", z=z, norm_weight=nw, workspace=ws,
                                                           stream=stream), stream, calls, warm)
    by = prefill_bytes(B, H, T, d, d) + B * H * T * d * 2 + d * 4 + 2 * H * 4
    entry("gdn_layer_prologue_norm_bf16_B4_H16_T4096_d128", ms, B * T, prefill_flops(B, H, T, d, d), by,
          "tensor cores, prologue and gated RMSNorm fused")
    del q, k, v, b, a, z, y, S, ws

    # the decode step with the prologue and the gated RMSNorm (decode workload shape)
    dc = W.DECODE
    B, H = dc.B, dc.H
    q = (torch.randn(B, H, d, generator=gen) * 2).to(torch.bfloat16).to(dev)
    k = (torch.randn(B, H, d, generator=gen) * 2).to(torch.bfloat16).to(dev)
    v = torch.randn(B, H, d, generator=gen).to(torch.bfloat16).to(dev)
    b = torch.randn(B, H, generator=gen).to(dev)
    a = torch.randn(B, H, generator=gen).to(dev)
    A_log = torch.log(1 + 15 * torch.rand(H, generator=gen)).to(dev)
    dt_bias = torch.randn(H, generator=gen).to(dev)
    z = torch.randn(B, H, d, generator=gen).to(torch.bfloat16).to(dev)
    Sd = (0.1 * torch.randn(B, H, d, d, generator=gen)).to(dev)
    y = torch.empty((B, H, d), dtype=torch.bfloat16, device=dev)
    ms = _time_calls(torch, lambda: dn.dn_decode_step_gdn_ex(q, k, v, b, a, A_log, dt_bias, Sd, y, scale=sc, z=z,
                                                             norm_weight=nw, stream=stream), stream, calls, warm)
    by = decode_bytes(B, H, d, d) + B * H * d * 2 + d * 4
    entry("decode_step_prologue_norm_bf16_B256_H32_d128", ms, B, None, by,
          "one CTA per head; prologue and gated RMSNorm fused")
    del q, k, v, b, a, z, Sd, y

    # the generalised (RWKV-7) rule: fp32 arithmetic on CUDA cores
    B, H, Tg = 1, 8, 2048
    q = torch.randn(B, H, Tg, d, generator=gen).to(torch.bfloat16).to(dev)
    wl = (-torch.exp(torch.randn(B, H, Tg, d, generator=gen) - 2)).to(dev)
    kp = unit(torch.randn(B, H, Tg, d, generator=gen)).to(torch.bfloat16).to(dev)
    ar = torch.sigmoid(torch.randn(B, H, Tg, d, generator=gen)).to(dev)
    kw = (torch.randn(B, H, Tg, d, generator=gen) / d ** 0.5).to(torch.bfloat16).to(dev)
    v = torch.randn(B, H, Tg, d, generator=gen).to(torch.bfloat16).to(dev)
    o = torch.empty((B, H, Tg, d), dtype=torch.bfloat16, device=dev)
    S = torch.empty((B, H, d, d), device=dev)
    ms = _time_calls(torch, lambda: dn.dn_chunk_fwd_general(q, wl, kp, ar, kw, v, None, o, S, chunk=32, scale=sc,
                                                            stream=stream), stream, 3, 1)
    by = B * H * Tg * (d * 2 * 4 + d * 4 * 2) + B * H * d * d * 4
    entry("general_rule_bf16_B1_H8_T2048_d128", ms, B * Tg, None, by,
          "fp32 on CUDA cores, chunk 32 (per-channel decays exact per pair)", bound="alu")
    del q, wl, kp, ar, kw, v, o, S
    torch.cuda.empty_cache()
    return out


def measure_layer_ops(dn, torch, W, peaks, dev, stream, calls=5, warm=2):
    """The layer steps on either side of the rule at the bench prefill's shape
    (B=4, T=4096, 16 heads of 128), bf16, each against the HBM roofline:
    the causal conv (K=4, SiLU) of q, k and v as three calls on the column
    slices of one [B, T, 3*16*128] projection output, head-major outputs and
    carried states; and the gated RMSNorm of o [B, 16, T, 128] (head-major)
    with z [B, T, 16, 128] into y [B, T, 16, 128]."""
    pc = W.GDN_PREFILL
    B, H, T, d, K = pc.B, pc.H, pc.T, pc.dk, 4
    C3 = 3 * H * d
    gen = torch.Generator().manual_seed(pc.seed + 1)
    proj = torch.randn(B, T, C3, generator=gen).to(torch.bfloat16).to(dev)
    w = (torch.randn(C3, K, generator=gen) * 0.5).to(dev)
    s_in = torch.randn(B, K - 1, C3, generator=gen).to(torch.bfloat16).to(dev)
    ys = [torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    w_parts = [w[i * H * d:(i + 1) * H * d].contiguous() for i in range(3)]
    s_parts = [s_in[:, :, i * H * d:(i + 1) * H * d].contiguous() for i in range(3)]
    s_outs = [torch.empty_like(sp) for sp in s_parts]

    def conv():
        for i in range(3):
            dn.dn_causal_conv1d(proj[:, :, i * H * d:(i + 1) * H * d], w_parts[i], ys[i], s_parts[i], s_outs[i],
                                head_dim=d, stream=stream)

    o = torch.randn(B, H, T, d, generator=gen).to(torch.bfloat16).to(dev)
    z = torch.randn(B, T, H, d, generator=gen).to(torch.bfloat16).to(dev)
    nw = torch.ones(d, device=dev)
    y = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=dev)

    def norm():
        dn.dn_rms_norm_gated(o, z, nw, y, stream=stream)

    def timed(fn):
        for _ in range(warm):
            fn()
        ts = []
        for _ in range(calls):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        dn.dn_device_status(stream)
        return statistics.median(ts)

    out = {}
    conv_bytes = 2 * B * T * C3 * 2 + C3 * K * 4 + 2 * B * (K - 1) * C3 * 2
    norm_bytes = 3 * B * T * H * d * 2 + d * 4
    for name, fn, by, launches in (
            (f"causal_conv1d_qkv_bf16_B{B}_T{T}_C{C3}_K{K}", conv, conv_bytes, 3),
            (f"rms_norm_gated_bf16_B{B}_T{T}_H{H}_d{d}", norm, norm_bytes, 1)):
        ms = timed(fn)
        gb = by / (ms * 1e-3) / 1e9
        out[name] = {"ms_per_call": ms, "algorithmic_bytes": by, "hbm_gbs": gb, "hbm_frac": gb / peaks["hbm_gbs"],
                     "kernel_launches_per_call": launches, "bound": "hbm",
                     "timing": f"median of {calls} calls after {warm}, CUDA events"}
    del proj, w, s_in, ys, o, z, y
    torch.cuda.empty_cache()
    return out


def workload_config():
    return {"workload": "gated_deltanet_prefill_B4_H16_T4096_d128_bf16_chunk64 + "
                        "decode_step_B256_H32_d128_bf16_fp32state",
            "prefill": {"B": 4, "H": 16, "T": 4096, "d_k": 128, "d_v": 128, "chunk": 64,
                        "gate": "scalar", "tokens_per_step": 4 * 4096},
            "decode": {"B": 256, "H": 32, "d_k": 128, "d_v": 128, "gate": "scalar",
                       "tokens_per_step": 256, "token_bank": 16},
            "l2": "no flush: every step streams > 1.3 GB (prefill inputs 274 MB, decode state "
                  "1.07 GB read+write), more than the 126 MB L2",
            "parallelism": "independent replicas, one per GPU"}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--path", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip timing the other prefill workloads (small DeltaNet, long GDN, KDA)")
    ap.add_argument("--profile-case", choices=["prefill", "decode", "kda", "layer_ops"], default=None,
                    help="launch one kernel of the step a few times without timing (for ncu captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.profile_case:
        return run_profile_case(args)

    import torch
    import delta_rule_recurrent_02_b200 as dn
    from delta_rule_recurrent_02_b200 import workloads as W

    world, rank, local = dist_setup()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dn.load_library()
    peaks = load_peaks()

    # ---- inputs (seeded per rank), resident in HBM --------------------------
    pc = W.GDN_PREFILL
    pin = W.gen_prefill(pc.B, pc.H, pc.T, pc.dk, pc.dv, dtype=pc.dtype, gate=pc.gate,
                        seed=pc.seed + 1000 * rank, q_norm=True, g_shift=pc.g_shift)
    dc = W.DECODE
    din = W.gen_decode(dc)
    P = {k: (None if v is None else v.to(dev)) for k, v in pin.items()}
    D = {k: (None if v is None else v.to(dev)) for k, v in din.items()}
    o_p = torch.empty((pc.B, pc.H, pc.T, pc.dv), dtype=torch.bfloat16, device=dev)
    S_T = torch.empty((pc.B, pc.H, pc.dk, pc.dv), dtype=torch.float32, device=dev)
    o_d = torch.empty((dc.B, dc.H, dc.dv), dtype=torch.bfloat16, device=dev)
    S_dec = D["S"]
    stream = torch.cuda.current_stream()
    ws = prefill_workspace(dn, torch, pc, args.path, dev)

    def prefill():
        dn.dn_chunk_fwd(P["q"], P["k"], P["v"], P["beta"], P["g"], None, o_p, S_T, chunk=pc.chunk,
                        scale=pc.scale, path=args.path, workspace=ws, stream=stream)

    def decode(s):
        j = s % dc.bank
        dn.dn_decode_step(D["q"][j], D["k"][j], D["v"][j], D["beta"][j], D["g"][j], S_dec, o_d,
                          scale=dc.scale, stream=stream)

    for s in range(args.warmup):
        k0 = dn.dn_kernel_launches()
        prefill()
        pre_launches = dn.dn_kernel_launches() - k0
        decode(s)
    dn.dn_device_status(stream)
    barrier(world)

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(_smi_id(torch, dev, local))
    with sampler:
        barrier(world)
        launches0 = dn.dn_kernel_launches()
        t_start.record(stream)
        for s in range(args.steps):
            ev[s][0].record(stream)
            prefill()
            ev[s][1].record(stream)
            decode(args.warmup + s)
            ev[s][2].record(stream)
        t_end.record(stream)
        launches = dn.dn_kernel_launches() - launches0
        barrier(world)
    dn.dn_device_status(stream)
    total_ms = max_over_ranks(t_start.elapsed_time(t_end), world)
    pre_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in ev)
    dec_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in ev)
    pre_ms = max_over_ranks(pre_ms, world)
    dec_ms = max_over_ranks(dec_ms, world)
    ms_per_step = total_ms / args.steps
    tokens_step = pc.B * pc.T + dc.B
    value = job_throughput(tokens_step, ms_per_step, world)
    clocks = sampler.summary()

    # ---- roofline per kernel ---------------------------------------------------
    pf = prefill_flops(pc.B, pc.H, pc.T, pc.dk, pc.dv)
    pb = prefill_bytes(pc.B, pc.H, pc.T, pc.dk, pc.dv)
    db = decode_bytes(dc.B, dc.H, dc.dk, dc.dv)
    used_tc = ws is not None          # only the tensor-core path takes a workspace
    # the tensor-core path is one cooperative launch, or the WY kernel then the state pass
    pre_kernel = ("chunk_fused" if pre_launches == 1 else "chunk_wy+chunk_tc") if used_tc else "chunk_simt"
    pre_tflops = pf / (pre_ms * 1e-3) / 1e12
    pre_gbs = pb / (pre_ms * 1e-3) / 1e9
    dec_gbs = db / (dec_ms * 1e-3) / 1e9
    tensor_floor = pf / (peaks["bf16_tflops"] * 1e12)
    hbm_floor = pb / (peaks["hbm_gbs"] * 1e9)
    pre_roof = {"kernel": pre_kernel, "bound": "hbm" if hbm_floor >= tensor_floor else "tensor",
                "achieved": pre_gbs if hbm_floor >= tensor_floor else pre_tflops,
                "peak": peaks["hbm_gbs"] if hbm_floor >= tensor_floor else peaks["bf16_tflops"],
                "unit": "GB/s" if hbm_floor >= tensor_floor else "TFLOP/s",
                "traffic": traffic_for(pre_kernel), "algorithmic_bytes": pb, "counted_flops": pf,
                "tensor_tflops": pre_tflops, "tensor_frac": pre_tflops / peaks["bf16_tflops"],
                "tensor_frac_sustained": pre_tflops / peaks["bf16_tflops_sustained"],
                "hbm_gbs": pre_gbs, "hbm_frac": pre_gbs / peaks["hbm_gbs"],
                "ms_per_launch": pre_ms, "peaks": peaks["source"]}
    pre_roof["frac"] = pre_roof["achieved"] / pre_roof["peak"]
    dec_roof = {"kernel": "decode_step", "bound": "hbm", "achieved": dec_gbs, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": dec_gbs / peaks["hbm_gbs"], "traffic": traffic_for("decode_step"),
                "algorithmic_bytes": db, "ms_per_launch": dec_ms, "peaks": peaks["source"]}
    dominant = pre_roof if pre_ms >= dec_ms else dec_roof
    roofline = {k: dominant[k] for k in ("bound", "achieved", "peak", "unit", "frac", "traffic")}
    roofline["kernel"] = dominant["kernel"]

    # ---- end to end through the C ABI with host buffers -------------------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(dn, torch, W, pin, din, pc, dc, args, stream, dev, world, tokens_step)

    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if used_tc else "f32",
            "data": "synthetic", "config": workload_config(),
            "prefill": {"tokens_per_s": world * pc.B * pc.T / (pre_ms * 1e-3), "roofline": pre_roof},
            "decode": {"tokens_per_s": world * dc.B / (dec_ms * 1e-3), "roofline": dec_roof},
            "roofline": roofline, "e2e": e2e, "gpu_launches": launches,
            "clocks": clocks}
    if world == 1 and not args.no_configs:
        line["other_prefill_workloads"] = measure_prefill_configs(dn, torch, W, peaks, dev, stream)
        line["layer_ops"] = measure_layer_ops(dn, torch, W, peaks, dev, stream)
        line["next_rows"] = measure_next_rows(dn, torch, W, peaks, dev, stream)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        reps = [oracle_sample_rate(seed_offset=r) for r in range(4)]
        v = statistics.median(r[0] for r in reps)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s", "cores": oracle.max_threads(),
                                "nproc": os.cpu_count(), "kind": "oracle",
                                "sample": f"median of {len(reps)} repetitions; each: " + reps[0][2],
                                "single_thread": oracle_single_thread()}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_profile_case(args):
    """Launch the prefill (or the decode step) of the benchmark workload
    args.warmup + args.steps times, with no timing: a small, fixed program for
    ncu captures (one kernel per launch, inputs resident on the device)."""
    import torch
    import delta_rule_recurrent_02_b200 as dn
    from delta_rule_recurrent_02_b200 import workloads as W
    dev = torch.device("cuda", 0)
    if args.profile_case in ("prefill", "kda"):
        pc = W.GDN_PREFILL if args.profile_case == "prefill" else W.KDA_PREFILL
        P = {k: (None if v is None else v.to(dev)) for k, v in W.gen_prefill_config(pc).items()}
        o = torch.empty((pc.B, pc.H, pc.T, pc.dv), dtype=torch.bfloat16, device=dev)
        S_T = torch.empty((pc.B, pc.H, pc.dk, pc.dv), dtype=torch.float32, device=dev)
        ws = prefill_workspace(dn, torch, pc, args.path, dev)
        for _ in range(args.warmup + args.steps):
            dn.dn_chunk_fwd(P["q"], P["k"], P["v"], P["beta"], P["g"], None, o, S_T, chunk=pc.chunk,
                            scale=pc.scale, path=args.path, workspace=ws)
    elif args.profile_case == "layer_ops":
        # the layer's conv (q, k, v slices of one projection row) and gated norm at the
        # bench prefill's shape: 3 conv launches and 1 norm launch per repetition
        pc = W.GDN_PREFILL
        B, H, T, d, K = pc.B, pc.H, pc.T, pc.dk, 4
        C3 = 3 * H * d
        gen = torch.Generator().manual_seed(pc.seed + 1)
        proj = torch.randn(B, T, C3, generator=gen).to(torch.bfloat16).to(dev)
        w = (torch.randn(C3, K, generator=gen) * 0.5).to(dev)
        w_parts = [w[i * H * d:(i + 1) * H * d].contiguous() for i in range(3)]
        s_in = torch.randn(B, K - 1, C3, generator=gen).to(torch.bfloat16).to(dev)
        s_parts = [s_in[:, :, i * H * d:(i + 1) * H * d].contiguous() for i in range(3)]
        s_outs = [torch.empty_like(sp) for sp in s_parts]
        ys = [torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev) for _ in range(3)]
        o = torch.randn(B, H, T, d, generator=gen).to(torch.bfloat16).to(dev)
        z = torch.randn(B, T, H, d, generator=gen).to(torch.bfloat16).to(dev)
        nw = torch.ones(d, device=dev)
        y = torch.empty((B, T, H, d), dtype=torch.bfloat16, device=dev)
        for _ in range(args.warmup + args.steps):
            for i in range(3):
                dn.dn_causal_conv1d(proj[:, :, i * H * d:(i + 1) * H * d], w_parts[i], ys[i], s_parts[i],
                                    s_outs[i], head_dim=d)
            dn.dn_rms_norm_gated(o, z, nw, y)
    else:
        dc = W.DECODE
        D = {k: (None if v is None else v.to(dev)) for k, v in W.gen_decode(dc).items()}
        o = torch.empty((dc.B, dc.H, dc.dv), dtype=torch.bfloat16, device=dev)
        for s in range(args.warmup + args.steps):
            j = s % dc.bank
            dn.dn_decode_step(D["q"][j], D["k"][j], D["v"][j], D["beta"][j], D["g"][j], D["S"], o,
                              scale=dc.scale)
    dn.dn_device_status()
    torch.cuda.synchronize()
    print(json.dumps({"profile_case": args.profile_case, "launches": args.warmup + args.steps}))
    return 0


def _smi_id(torch, dev, local):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return local


def prefill_workspace(dn, torch, pc, path, dev):
    """The prefill's workspace, allocated once like a caller that reuses it (None if the path needs none)."""
    nbytes = dn.dn_chunk_fwd_workspace_size(pc.B, pc.T, pc.H, pc.dk, pc.dv, chunk=pc.chunk, dtype=pc.dtype,
                                            gate=pc.gate, path=path)
    return torch.empty(nbytes, dtype=torch.uint8, device=dev) if nbytes else None


def run_e2e(dn, torch, W, pin, din, pc, dc, args, stream, dev, world, tokens_step):
    """Same step through the C ABI with pinned HOST buffers: per step, copy the
    prefill inputs and the decode token set host->device, run both calls, copy
    o, S_T and the decode output device->host.  The decode state stays
    resident (it is the layer's memory, like weights).

    Steps are double-buffered over three streams, as a server streaming
    requests would run them: step s's uploads (copy stream) overlap step s-1's
    kernels (the caller's stream) and step s-2's downloads (a third stream),
    so the PCIe link's two directions and the GPU work at once.  Every step
    still moves all of its own inputs and results.  The same step run serially
    on one stream is reported beside it (serial_ms_per_step)."""
    hp = {k: (None if v is None else v.pin_memory()) for k, v in pin.items()}
    hd = {k: (None if v is None else v.pin_memory()) for k, v in din.items() if k != "S"}
    S_dec = din["S"].to(dev)
    ws = prefill_workspace(dn, torch, pc, args.path, dev)

    def buffers():
        return dict(P={k: torch.empty_like(v, device=dev) for k, v in hp.items() if v is not None},
                    Dt={k: torch.empty_like(v[0], device=dev) for k, v in hd.items() if v is not None},
                    o_p=torch.empty((pc.B, pc.H, pc.T, pc.dv), dtype=torch.bfloat16, device=dev),
                    S_T=torch.empty((pc.B, pc.H, pc.dk, pc.dv), dtype=torch.float32, device=dev),
                    o_d=torch.empty((dc.B, dc.H, dc.dv), dtype=torch.bfloat16, device=dev),
                    h_o=torch.empty((pc.B, pc.H, pc.T, pc.dv), dtype=torch.bfloat16).pin_memory(),
                    h_S=torch.empty((pc.B, pc.H, pc.dk, pc.dv), dtype=torch.float32).pin_memory(),
                    h_od=torch.empty((dc.B, dc.H, dc.dv), dtype=torch.bfloat16).pin_memory())

    bufs = [buffers(), buffers()]
    h2d = sum(v.numel() * v.element_size() for v in hp.values() if v is not None) + \
        sum(v[0].numel() * v.element_size() for v in hd.values() if v is not None)
    d2h = sum(bufs[0][k].numel() * bufs[0][k].element_size() for k in ("h_o", "h_S", "h_od"))

    def upload(bf, s):
        for k, v in hp.items():
            if v is not None:
                bf["P"][k].copy_(v, non_blocking=True)
        j = s % dc.bank
        for k, v in hd.items():
            if v is not None:
                bf["Dt"][k].copy_(v[j], non_blocking=True)

    def compute(bf, st):
        P, Dt = bf["P"], bf["Dt"]
        dn.dn_chunk_fwd(P["q"], P["k"], P["v"], P["beta"], P["g"], None, bf["o_p"], bf["S_T"], chunk=pc.chunk,
                        scale=pc.scale, path=args.path, workspace=ws, stream=st)
        dn.dn_decode_step(Dt["q"], Dt["k"], Dt["v"], Dt["beta"], Dt["g"], S_dec, bf["o_d"], scale=dc.scale,
                          stream=st)

    def download(bf):
        bf["h_o"].copy_(bf["o_p"], non_blocking=True)
        bf["h_S"].copy_(bf["S_T"], non_blocking=True)
        bf["h_od"].copy_(bf["o_d"], non_blocking=True)

    # ---- serial: one stream, a few steps -----------------------------------------
    def serial_step(s):
        with torch.cuda.stream(stream):
            upload(bufs[0], s)
            compute(bufs[0], stream)
            download(bufs[0])

    for s in range(args.warmup):
        serial_step(s)
    barrier(world)
    torch.cuda.synchronize()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    n_serial = max(1, min(args.steps, 5))
    a.record(stream)
    for s in range(n_serial):
        serial_step(s)
    b.record(stream)
    b.synchronize()
    serial_ms = max_over_ranks(a.elapsed_time(b), world) / n_serial

    # ---- double-buffered over three streams --------------------------------------
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev = lambda: torch.cuda.Event()
    uploaded = [ev() for _ in range(2)]
    computed = [ev() for _ in range(2)]
    downloaded = [ev() for _ in range(2)]
    used = [False, False]

    def pipelined_step(s):
        x = s & 1
        bf = bufs[x]
        with torch.cuda.stream(s_in):
            if used[x]:
                s_in.wait_event(computed[x])      # step s - 2 has read these inputs
            upload(bf, s)
            uploaded[x].record(s_in)
        stream.wait_event(uploaded[x])
        if used[x]:
            stream.wait_event(downloaded[x])      # step s - 2's results are copied out
        compute(bf, stream)
        computed[x].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(computed[x])
            download(bf)
            downloaded[x].record(s_out)
        used[x] = True

    for s in range(args.warmup):
        pipelined_step(s)
    torch.cuda.synchronize()
    barrier(world)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for s in range(args.steps):
        pipelined_step(s)
    s_out.wait_stream(stream)
    s_out.wait_stream(s_in)
    b.record(s_out)
    b.synchronize()
    barrier(world)
    ms = max_over_ranks(a.elapsed_time(b), world) / args.steps
    return {"value": world * tokens_step / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "schedule": "double-buffered over three streams: step s's uploads overlap step s-1's kernels "
                        "and step s-2's downloads",
            "serial_ms_per_step": serial_ms,
            "serial_tokens_per_s": world * tokens_step / (serial_ms * 1e-3)}


if __name__ == "__main__":
    sys.exit(main())
