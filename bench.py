#!/usr/bin/env python
"""Benchmark of the quantized-KV decode path on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

One step = quantize-on-write of the step's new token per sequence (through the
block table) + the fused-dequant decode attention over the whole context, on
the workload "fp8-paged-4x32k": 4 sequences x 32,768 tokens, 8 KV heads, 64
query heads, head_dim 128, FP8 E4M3 cache in 16-token pages at a random
permutation of the pool, per-layer scales calibrated on a 16,384-token sample.
value = KV-scan bytes per step / device time per step (GB/s).  L2 is flushed
before every timed step (a 512 MiB write, then a 256 MiB read so no dirty
lines are left for the timed kernel to write back).

Extra keys report the other rows: the BF16 vs FP8 vs NVFP4 comparison on the
1 x 65,536-token, D 64 workload, the 4 x 126,976-token agent step (2,048-token
prefill chunk written per sequence, then decode), and the calibration abs-max.

Under torchrun (N > 1) every rank runs its own batch of sequences (weak
scaling, no data-path collective); time is the max over ranks.
``--impl reference`` times the CPU oracle instead (rank 0 only), on bounded
samples of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn KV-scan GB/s (frac of HBM peak) & µs/step, BF16 vs FP8 vs NVFP4"
MAIN_WORKLOAD = "fp8-paged-4x32k"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0
L2_FLUSH_BYTES = 512 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default=MAIN_WORKLOAD)
    ap.add_argument("--no-extras", action="store_true", help="main line only")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the bench line: decode time of every sweep cell "
                         "(context x batch x head_dim x format), one JSON line each")
    ap.add_argument("--sweep-formats", default="bf16,fp8,nvfp4")
    ap.add_argument("--sweep-dims", default="64,128")
    return ap.parse_args()


# ------------------------------------------------------------------ plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a float over ranks (plain NCCL/gloo all-reduce of one number)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peak():
    """Dense bf16 tensor-core peak in TFLOP/s: the sustained figure (for a
    kernel timed inside a long run) and the burst one, from MEASURED_PEAKS.json."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops_sustained"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS_SUSTAINED, FALLBACK_BF16_TFLOPS, "fallback"


def source_digest() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "quantized_kv_cache_21_b200", "csrc")
    for name in ("kvq_decode.cu", "kvq_device.cuh"):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per decode launch from the committed ncu summary, if it was
    taken on the current decode source; else None."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d.get(workload)
        if e and e.get("source_digest") == source_digest():
            return int(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """Polls NVML (read-only) for SM clock and throttle reasons while active."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int):
        self.samples, self.active, self.ok = [], False, False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = False
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()

    def _run(self):
        while not self._stop:
            if self.active:
                try:
                    mhz = self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM)
                    rs = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    self.samples.append((mhz, rs))
                except Exception:
                    pass
            time.sleep(0.002)

    def summary(self):
        self._stop = True
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "samples": len(self.samples)}
        mask = 0
        for _, r in self.samples:
            mask |= r
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for b, n in self.REASONS.items() if mask & b),
                "samples": len(self.samples)}


# ------------------------------------------------------------------ GPU timing
class Timer:
    def __init__(self, torch, clocks):
        self.torch, self.clocks = torch, clocks
        self.flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device="cuda")
        self.clean_buf = torch.zeros(L2_FLUSH_BYTES // 2, dtype=torch.uint8, device="cuda")

    def flush(self):
        """Evict L2 (write 512 MiB), then read 256 MiB so L2 holds clean lines:
        the timed step neither hits in L2 nor pays for another kernel's
        dirty-line write-back."""
        self.flush_buf.fill_(1)
        self.clean_buf.max()

    def run(self, parts, K, W):
        """parts: list of callables launched in order each step.  Returns the
        per-step device times (ms) of each part and of the whole step."""
        torch = self.torch
        for _ in range(W):
            self.flush()
            for p in parts:
                p()
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(parts) + 1)]
              for _ in range(K)]
        self.clocks.active = True
        for i in range(K):
            self.flush()
            ev[i][0].record()
            for j, p in enumerate(parts):
                p()
                ev[i][j + 1].record()
        torch.cuda.synchronize()
        self.clocks.active = False
        part_ms = [[ev[i][j].elapsed_time(ev[i][j + 1]) for i in range(K)]
                   for j in range(len(parts))]
        step_ms = [ev[i][0].elapsed_time(ev[i][-1]) for i in range(K)]
        return part_ms, step_ms


def cpu_baseline_sample(w, fmt, seconds, steps=None):
    """The CPU oracle on bounded samples of the workload: one (sequence, KV
    head) unit at a time, quantize-on-write of its step token(s) + float64
    decode attention of its G query heads over the full context.  Inputs are
    host-drawn with the same recipe.  Returns (GB/s, units, seconds)."""
    import numpy as np

    import oracle
    from quantized_kv_cache_21_b200 import workloads as wl
    from quantized_kv_cache_21_b200.scenario import kv_scan_bytes

    G, D, L = w.Hq // w.Hkv, w.D, w.seq_len
    chunk = max(1, w.write_chunk)
    mb = -(-L // 16)
    bt = np.arange(mb, dtype=np.int32)[None, :]
    unit_bytes = kv_scan_bytes(fmt, [L], 1, D)
    done, t_total, u = 0, 0.0, 0
    while True:
        rng = wl.rng_for(w.seed, 5000 + u)
        k = wl.make_tokens(rng, L, 1, D, [(0, 3)] if w.outlier_factor != 1 else [],
                           w.outlier_factor)
        v = wl.make_tokens(rng, L, 1, D)
        q = wl.make_query(rng, 1, G, D)
        n = L if w.calib_tokens is None else w.calib_tokens
        ks = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(k[:n]))
        vs = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(v[:n]))
        kc, vc = oracle.new_cache(fmt, mb, 1, D)
        slots = np.arange(L, dtype=np.int64)
        oracle.write(fmt, k[: L - chunk], v[: L - chunk], slots[: L - chunk], kc, vc, ks, vs)
        t0 = time.perf_counter()
        oracle.write(fmt, k[L - chunk:], v[L - chunk:], slots[L - chunk:], kc, vc, ks, vs)
        oracle.decode_attention(fmt, q, kc, vc, 1, bt, np.array([L], np.int32), ks, vs)
        t_total += time.perf_counter() - t0
        done += 1
        u += 1
        if (steps is not None and done >= steps) or (steps is None and t_total >= seconds):
            break
    return done * unit_bytes / t_total / 1e9, done, t_total, unit_bytes


def run_reference(args):
    """--impl reference: the CPU oracle on this workload (rank 0 only)."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from quantized_kv_cache_21_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    cpu_baseline_sample(w, w.fmt, 0, steps=max(1, args.warmup))  # warm-up units
    gbps, units, secs, unit_bytes = cpu_baseline_sample(w, w.fmt, 0, steps=args.steps)
    ms = secs / units * 1e3
    sample = (f"{units} (sequence, KV head) units of {args.workload}, each: quantize-on-write "
              f"of {max(1, w.write_chunk)} token(s) + float64 decode attention of "
              f"{w.Hq // w.Hkv} query heads over {w.seq_len} tokens ({unit_bytes} KV bytes)")
    line = {"impl": "reference", "metric": METRIC, "value": gbps, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64", "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": gbps, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": gbps, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def workload_config(w, fmt=None):
    return {"workload": w.name, "format": fmt or w.fmt, "num_seqs": w.B, "seq_len": w.seq_len,
            "kv_heads": w.Hkv, "q_heads": w.Hq, "head_dim": w.D, "block_size": 16,
            "block_table": "random permutation" if w.permuted else "in order",
            "l2": "flushed before every timed step (512 MiB write, then 256 MiB read)"}


def roofline(bytes_per_launch, ms_list, peak, peak_kind, traffic):
    ms = statistics.mean(ms_list)
    achieved = bytes_per_launch / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic, "peak_source": peak_kind,
            "kernel": "kvq_decode_kernel", "us_per_launch": ms * 1e3}


def run_sweep(args):
    """Decode-only timing of the sweep cells on one GPU (L2 flushed before every
    timed launch).  Prints one JSON line per cell, then a summary line."""
    import dataclasses
    import torch
    import quantized_kv_cache_21_b200 as kvq
    from quantized_kv_cache_21_b200 import workloads as wl
    from quantized_kv_cache_21_b200.scenario import DecodeScenario

    kvq.lib()
    clocks = ClockSampler(torch.cuda.current_device())
    timer = Timer(torch, clocks)
    peak, peak_kind = measured_hbm_peak()
    K, W = max(3, args.steps), max(3, args.warmup)
    cells = []
    for D in (int(x) for x in args.sweep_dims.split(",")):
        for fmt in args.sweep_formats.split(","):
            for L in wl.SWEEP_LENGTHS:
                for B in wl.SWEEP_BATCHES:
                    w = dataclasses.replace(wl.SWEEP, B=B, D=D, seq_len=L)
                    lens = wl.varlen(wl.rng_for(wl.SWEEP_SEED, wl.sweep_cell_stream(L, B)), B, L)
                    sc = DecodeScenario(w, fmt=fmt, lens=lens)
                    (dms,), _ = timer.run([sc.decode], K, W)
                    assert int(sc.err.item()) == 0
                    us = statistics.median(dms) * 1e3
                    gbps = sc.scan_bytes / (us * 1e-6) / 1e9
                    cell = {"sweep_cell": {"format": fmt, "head_dim": D, "context": L, "batch": B,
                                           "kv_heads": 8, "q_heads": 64,
                                           "lengths": "uniform in [L/2, L]"},
                            "kv_scan_bytes": sc.scan_bytes, "us_per_decode": us, "GBps": gbps,
                            "frac_of_hbm_peak": gbps / peak}
                    print(json.dumps(cell), flush=True)
                    cells.append(cell)
                    del sc
                    torch.cuda.empty_cache()
    heavy = [c for c in cells if c["kv_scan_bytes"] >= 64e6]
    summary = {"sweep_summary": {
        "cells": len(cells), "peak_GBps": peak, "peak_source": peak_kind,
        "byte_heavy_cells (>= 64 MB)": len(heavy),
        "min_frac_byte_heavy": {f: min((c["frac_of_hbm_peak"] for c in heavy
                                        if c["sweep_cell"]["format"] == f), default=None)
                                for f in args.sweep_formats.split(",")},
        "median_frac_byte_heavy": {f: statistics.median([c["frac_of_hbm_peak"] for c in heavy
                                                         if c["sweep_cell"]["format"] == f])
                                   if any(c["sweep_cell"]["format"] == f for c in heavy)
                                   else None for f in args.sweep_formats.split(",")},
        "clocks": clocks.summary()}}
    print(json.dumps(summary))
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    if args.sweep:
        return run_sweep(args)
    import torch
    import quantized_kv_cache_21_b200 as kvq
    from quantized_kv_cache_21_b200 import workloads as wl
    from quantized_kv_cache_21_b200.scenario import DecodeScenario

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    kvq.lib()
    dev_index = torch.cuda.current_device()
    phys = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
    nvml_index = int(phys[dev_index]) if phys and phys[0].strip().isdigit() else dev_index
    clocks = ClockSampler(nvml_index)
    timer = Timer(torch, clocks)
    peak, peak_kind = measured_hbm_peak()
    K, W = args.steps, max(3, args.warmup)

    # ---------------- main line: write + decode step
    w = wl.WORKLOADS[args.workload]
    sc = DecodeScenario(w, device="cuda", seq_offset=rank * w.B)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # The step (write, then decode) is timed as one part: no event between the
    # two launches, so the decode may start its prologue while the write ends.
    def step():
        sc.write()
        sc.decode()

    _, step_ms = timer.run([step], K, W)
    total_ms = sum(step_ms)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    max_total_ms = reduce_max(total_ms, world, device="cuda")

    # ---------------- end to end through the public API with host buffers:
    # one pinned upload of the step's inputs (q, step K, step V) and one pinned
    # download of its results (out, lse) per step, around the write + decode
    nq, nk = sc.q.numel(), sc.step_k.numel()
    up_h = torch.empty(nq + 2 * nk, dtype=torch.bfloat16).pin_memory()
    up_h[:nq].copy_(sc.q.reshape(-1).cpu())
    up_h[nq:nq + nk].copy_(sc.step_k.reshape(-1).cpu())
    up_h[nq + nk:].copy_(sc.step_v.reshape(-1).cpu())
    up_d = torch.empty_like(up_h, device="cuda")
    d_q = up_d[:nq].view(sc.q.shape)
    d_k = up_d[nq:nq + nk].view(sc.step_k.shape)
    d_v = up_d[nq + nk:].view(sc.step_v.shape)
    no, nl = sc.out.numel(), sc.lse.numel()
    down_d = torch.empty(no + nl, dtype=torch.float32, device="cuda")
    down_h = torch.empty(no + nl, dtype=torch.float32).pin_memory()
    d_out, d_lse = down_d[:no].view(sc.out.shape), down_d[no:].view(sc.lse.shape)

    def e2e_step():
        up_d.copy_(up_h, non_blocking=True)
        sc.write(k=d_k, v=d_v)
        sc.decode(q=d_q, out=d_out, lse=d_lse)
        down_h.copy_(down_d, non_blocking=True)

    if world > 1:
        torch.distributed.barrier()
    _, e2e_eager_ms = timer.run([e2e_step], K, W)
    # The same step captured once in a CUDA graph (the same API calls; the
    # write -> decode programmatic dependency is kept as a graph edge) and
    # replayed: what a serving loop does to drop per-call launch overhead.
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            e2e_step()
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        e2e_step()
    torch.cuda.synchronize()
    _, e2e_ms = timer.run([graph.replay], K, W)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    max_e2e_ms = reduce_max(sum(e2e_ms), world, device="cuda") / K
    max_e2e_eager_ms = reduce_max(sum(e2e_eager_ms), world, device="cuda") / K
    assert int(sc.err.item()) == 0, f"device error word {int(sc.err.item())}"
    if rank != 0:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return 0
    ms_per_step = max_total_ms / K
    value = world * sc.scan_bytes / (ms_per_step * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "us_per_step": ms_per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3 (f16 mma, fp32 accumulate)",
            "data": "synthetic: seeded N(0,1) K/V/Q in BF16, 1% outlier channels x16, "
                    "random block table",
            "config": dict(workload_config(w), parallelism=f"dp{world} (sequences per rank)",
                           kv_scan_bytes_per_step=sc.scan_bytes,
                           write_tokens_per_step=int(sc.step_k.shape[0]))}
    line["frac_of_hbm_peak"] = value / world / peak
    # each launch alone (after an L2 flush) for the roofline and the breakdown
    (decode_ms,), _ = timer.run([sc.decode], K, W)
    (write_ms,), _ = timer.run([sc.write], K, W)
    line["roofline"] = roofline(sc.scan_bytes, decode_ms, peak, peak_kind,
                                profiled_traffic(w.name))
    line["step_breakdown_us"] = {"write_alone": statistics.mean(write_ms) * 1e3,
                                 "decode_alone": statistics.mean(decode_ms) * 1e3,
                                 "step": ms_per_step * 1e3}
    line["gpu_launches"] = 2 * K
    line["e2e"] = {"value": world * sc.scan_bytes / (max_e2e_eager_ms * 1e-3) / 1e9,
                   "unit": "GB/s", "h2d_bytes_per_step": up_h.numel() * 2,
                   "d2h_bytes_per_step": down_h.numel() * 4, "us_per_step": max_e2e_eager_ms * 1e3,
                   "copies_per_step": {"h2d": 1, "d2h": 1},
                   "launch": "the API called from Python every step"}
    line["e2e_graph"] = {"value": world * sc.scan_bytes / (max_e2e_ms * 1e-3) / 1e9,
                         "unit": "GB/s", "us_per_step": max_e2e_ms * 1e3,
                         "launch": "CUDA graph of the same calls, replayed each step"}

    del sc
    torch.cuda.empty_cache()

    # ---------------- other rows
    if not args.no_extras:
        wf = wl.WORKLOADS["nvfp4-1x64k"]
        fm = {}
        for fmt in ("bf16", "fp8", "nvfp4"):
            s2 = DecodeScenario(wf, fmt=fmt, device="cuda")
            (dms,), _ = timer.run([s2.decode], K, W)
            a = s2.scan_bytes / (statistics.mean(dms) * 1e-3) / 1e9
            fm[fmt] = {"us_per_step": statistics.mean(dms) * 1e3, "kv_scan_bytes": s2.scan_bytes,
                       "GBps": a, "frac_of_hbm_peak": a / peak}
            assert int(s2.err.item()) == 0
            del s2
            torch.cuda.empty_cache()
        fm["config"] = workload_config(wf, "bf16|fp8|nvfp4")
        fm["speedup_vs_bf16"] = {f: fm["bf16"]["us_per_step"] / fm[f]["us_per_step"]
                                 for f in ("fp8", "nvfp4")}
        line["formats"] = fm

        wa = wl.WORKLOADS["agents-fp8-4x127k"]
        s3 = DecodeScenario(wa, device="cuda")
        Ka = max(3, K // 4)

        def step3():
            s3.write()
            s3.decode()

        _, sms = timer.run([step3], Ka, W)
        (wms,), _ = timer.run([s3.write], Ka, W)
        (dms,), _ = timer.run([s3.decode], Ka, W)
        line["agents"] = {"config": dict(workload_config(wa),
                                         write_tokens_per_step=int(s3.step_k.shape[0])),
                          "us_per_step": statistics.mean(sms) * 1e3,
                          "write_alone_us": statistics.mean(wms) * 1e3,
                          "decode_alone_us": statistics.mean(dms) * 1e3,
                          "decode_GBps": s3.scan_bytes / (statistics.mean(dms) * 1e-3) / 1e9,
                          "decode_frac_of_hbm_peak":
                              s3.scan_bytes / (statistics.mean(dms) * 1e-3) / 1e9 / peak}
        assert int(s3.err.item()) == 0

        # chunked prefill on the same cache: each sequence's 2,048-token chunk
        # (written above) attends causally to its 126,976 cached tokens;
        # tensor-core bound, so reported against the bf16 dense peak
        s3.prefill_setup()
        s3.write()
        (pms,), _ = timer.run([s3.prefill], 3, W)
        assert int(s3.err.item()) == 0
        t_pf = statistics.mean(pms) * 1e-3
        pk_s, pk_b, pk_kind = measured_tensor_peak()
        tf = s3.prefill_flops / t_pf / 1e12
        line["chunked_prefill"] = {
            "config": dict(workload_config(wa), chunk_tokens_per_seq=s3.chunk,
                           attention="causal: query i of the chunk sees positions <= its own"),
            "ms_per_launch": t_pf * 1e3, "algorithmic_flops": s3.prefill_flops,
            "TFLOPs": tf, "peak_TFLOPs": pk_s, "peak": f"{pk_kind} bf16 dense, sustained",
            "frac_of_tensor_peak": tf / pk_s, "frac_of_burst_peak": tf / pk_b,
            "mma": "tcgen05.mma kind::f16 (bf16 for BF16 pages), M=128, fp32 accumulators in "
                   "tensor memory; P enters PV as two 16-bit halves (executed MMA flops = 1.5x "
                   "algorithmic)"}
        del s3
        torch.cuda.empty_cache()

        # the same 4 x 126,976-token, head_dim-128 cache in all three formats:
        # the byte-heavy comparison (decode launches only)
        af = {}
        for fmt in ("bf16", "fp8", "nvfp4"):
            s4 = DecodeScenario(wa, fmt=fmt, device="cuda")
            (dms,), _ = timer.run([s4.decode], max(3, K // 4), W)
            a = s4.scan_bytes / (statistics.mean(dms) * 1e-3) / 1e9
            af[fmt] = {"us_per_step": statistics.mean(dms) * 1e3, "kv_scan_bytes": s4.scan_bytes,
                       "GBps": a, "frac_of_hbm_peak": a / peak}
            assert int(s4.err.item()) == 0
            del s4
            torch.cuda.empty_cache()
        af["config"] = workload_config(wa, "bf16|fp8|nvfp4")
        af["speedup_vs_bf16"] = {f: af["bf16"]["us_per_step"] / af[f]["us_per_step"]
                                 for f in ("fp8", "nvfp4")}
        line["agents_formats"] = af

        # sliding-window mode ("SWA mode" of the MI300X benchmark page: window
        # 4096) on the main workload's cache: decode launches only
        s5 = DecodeScenario(w, device="cuda")
        swa = {}
        for win in (4096,):
            s5.window_ws(win)
            (dms,), _ = timer.run([lambda: s5.decode_window(win)], K, W)
            b5 = s5.window_scan_bytes(win)
            a = b5 / (statistics.mean(dms) * 1e-3) / 1e9
            swa[str(win)] = {"us_per_step": statistics.mean(dms) * 1e3, "kv_scan_bytes": b5,
                             "GBps": a, "frac_of_hbm_peak": a / peak}
        assert int(s5.err.item()) == 0
        line["sliding_window"] = {"config": dict(workload_config(w), window="last 4096 tokens"),
                                  "windows": swa}
        del s5
        torch.cuda.empty_cache()

        x = wl.device_tokens(20264, 0, 65536, 8, 128)
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        (cms,), _ = timer.run([lambda: kvq.kv_calibrate_absmax(x, amax)], K, W)
        cb = x.numel() * 2
        line["calibration"] = {"tensor": "65,536 x 8 x 128 BF16", "bytes": cb,
                               "us": statistics.mean(cms) * 1e3,
                               "GBps": cb / (statistics.mean(cms) * 1e-3) / 1e9}
        del x

    line["clocks"] = clocks.summary()
    if world == 1:
        gbps, units, secs, unit_bytes = cpu_baseline_sample(w, w.fmt, args.cpu_seconds)
        line["cpu_baseline"] = {
            "value": gbps, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{units} (sequence, KV head) units of {w.name} ({unit_bytes} KV bytes "
                      f"each: write of the step token + float64 attention of "
                      f"{w.Hq // w.Hkv} heads over {w.seq_len} tokens), {secs:.1f} s"}
    print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
