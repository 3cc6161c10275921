#!/usr/bin/env python
"""Benchmark of the quantized-KV decode path on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]

One step, on the workload "agents-fp8-4x127k" (4 sequences x 126,976 tokens,
8 KV heads, 64 query heads, head_dim 128, FP8 E4M3 cache in 16-token pages at
a random permutation of the pool, per-layer scales calibrated on a
16,384-token sample): quantize-on-write of a 2,048-token chunk per sequence
through the block table, then the fused-dequant decode attention over the
whole context.  value = KV-scan bytes per step / device time per step (GB/s).
L2 is flushed before every timed step (a 512 MiB write, then a 256 MiB read
so no dirty lines are left for the timed kernel to write back).

Extra keys (compact rows of µs, GB/s and fraction of the HBM peak) report the
other rows: BF16 vs FP8 vs NVFP4 decode on the same 4 x 126,976-token cache
and on the 1 x 65,536-token D=64 workload, the FP8 4 x 32,768-token paged
step, a 4,096-token sliding window, the calibration abs-max and the chunked
prefill of the agent step.

Under torchrun (N > 1) every rank runs its own batch of sequences (weak
scaling, no data-path collective); time is the max over ranks.
``--impl reference`` times the CPU oracle instead (rank 0 only), on all host
cores, over bounded samples of the same workload.
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
MAIN_WORKLOAD = "agents-fp8-4x127k"
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
    ap.add_argument("--cpu-seconds", type=float, default=6.0)
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
    for name in ("kvq_decode.cu", "kvq_device.cuh", "kvq_api.cu"):  # kernel and its work plan
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


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class OracleUnits:
    """(sequence, KV head) units of a workload for the CPU oracle, each with
    its cache already holding the context before the step's chunk.  One
    "round" runs, for every unit, the step the GPU times: quantize-on-write
    of the step's chunk of tokens + float64 decode attention of the KV head's
    G query heads over the whole context.  Units are independent, so a round
    runs them on a pool of host threads (the oracle's C calls release the
    GIL); inputs are host-drawn with the workloads' recipe."""

    def __init__(self, w, fmt, n_units, threads, first_unit=0):
        from concurrent.futures import ThreadPoolExecutor

        self.w, self.fmt, self.threads = w, fmt, threads
        self.G, self.D, self.L = w.Hq // w.Hkv, w.D, w.seq_len
        self.chunk = max(1, w.write_chunk)
        self.mb = -(-self.L // 16)
        self.pool = ThreadPoolExecutor(max_workers=threads)
        self.units = list(self.pool.map(self._prepare, range(first_unit, first_unit + n_units)))

    def _prepare(self, u):
        import numpy as np

        import oracle
        from quantized_kv_cache_21_b200 import workloads as wl

        w, L, D, G, chunk = self.w, self.L, self.D, self.G, self.chunk
        rng = wl.rng_for(w.seed, 5000 + u)
        outl = [(0, 3)] if w.outlier_factor != 1 else []
        k = wl.make_tokens(rng, L, 1, D, outl, w.outlier_factor)
        v = wl.make_tokens(rng, L, 1, D, outl, w.outlier_factor)
        q = wl.make_query(rng, 1, G, D)
        n = L if w.calib_tokens is None else w.calib_tokens
        ks = oracle.scale_from_absmax(self.fmt, oracle.absmax_bf16(k[:n]))
        vs = oracle.scale_from_absmax(self.fmt, oracle.absmax_bf16(v[:n]))
        kc, vc = oracle.new_cache(self.fmt, self.mb, 1, D)
        slots = np.arange(L, dtype=np.int64)
        oracle.write(self.fmt, k[: L - chunk], v[: L - chunk], slots[: L - chunk], kc, vc, ks, vs)
        return dict(k=k[L - chunk:].copy(), v=v[L - chunk:].copy(), slots=slots[L - chunk:].copy(),
                    q=q, kc=kc, vc=vc, ks=ks, vs=vs, bt=np.arange(self.mb, dtype=np.int32)[None],
                    lens=np.array([L], np.int32))

    def _step(self, x):
        import oracle
        oracle.write(self.fmt, x["k"], x["v"], x["slots"], x["kc"], x["vc"], x["ks"], x["vs"])
        oracle.decode_attention(self.fmt, x["q"], x["kc"], x["vc"], 1, x["bt"], x["lens"],
                                x["ks"], x["vs"])

    def round(self) -> float:
        """Wall seconds of one round over all units."""
        t0 = time.perf_counter()
        list(self.pool.map(self._step, self.units))
        return time.perf_counter() - t0

    @property
    def unit_bytes(self) -> int:
        from quantized_kv_cache_21_b200.scenario import kv_scan_bytes
        return kv_scan_bytes(self.fmt, [self.L], 1, self.D)

    def describe(self, rounds: int, secs: float) -> str:
        return (f"{rounds} round(s) of {len(self.units)} (sequence, KV head) unit(s) of "
                f"{self.w.name} on {self.threads} thread(s), {secs:.1f} s; a unit = write of "
                f"{self.chunk} token(s) + float64 attention of {self.G} heads over {self.L} "
                f"tokens ({self.unit_bytes} KV bytes)")

    def close(self):
        self.pool.shutdown()


def cpu_baseline(w, fmt, seconds):
    """The oracle on all host cores (one unit per thread, rounds for about
    `seconds`), then on one core (the first unit's step alone, once)."""
    threads = min(host_cores(), 64)
    ou = OracleUnits(w, fmt, threads, threads)
    rounds, secs = 0, 0.0
    while secs < seconds or rounds == 0:
        secs += ou.round()
        rounds += 1
    allc = (rounds * len(ou.units) * ou.unit_bytes / secs / 1e9, threads,
            ou.describe(rounds, secs))
    t0 = time.perf_counter()
    ou._step(ou.units[0])
    one = ou.unit_bytes / (time.perf_counter() - t0) / 1e9
    ou.close()
    return {"all": allc, "one": (one, 1, "")}


def run_reference(args):
    """--impl reference: the CPU oracle on this workload (rank 0 only), on all
    host cores: one step = one round over one (sequence, KV head) unit per
    thread."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from quantized_kv_cache_21_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    threads = min(host_cores(), 64)
    ou = OracleUnits(w, w.fmt, threads, threads)
    for _ in range(args.warmup):
        ou.round()
    times = [ou.round() for _ in range(args.steps)]
    secs = sum(times)
    gbps = args.steps * threads * ou.unit_bytes / secs / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": gbps, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": secs / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": workload_config(w),
            "cpu_baseline": {"value": gbps, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": ou.describe(args.steps, secs)},
            "e2e": {"value": gbps, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    ou.close()
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


def r4(x):
    """Four significant digits (keeps the JSON line short)."""
    return float(f"{x:.4g}") if x is not None else None


def row(bytes_, ms_list, peak):
    """Compact timing row of a decode-like launch: µs, GB/s, fraction of peak."""
    ms = statistics.mean(ms_list)
    gbps = bytes_ / (ms * 1e-3) / 1e9
    return {"us": r4(ms * 1e3), "GBps": r4(gbps), "frac": r4(gbps / peak)}


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

    # ---------------- main line: quantize-on-write of the step's tokens, then
    # the fused-dequant decode over the whole context, timed as one part (no
    # event between the two launches: the decode's prologue may overlap the
    # write's tail, as in a serving loop)
    w = wl.WORKLOADS[args.workload]
    sc = DecodeScenario(w, device="cuda", seq_offset=rank * w.B)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()

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
    # one pinned upload of the step's inputs (q, the step's K and V tokens)
    # and one pinned download of its results (out, lse) per step
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
    _, e2e_ms = timer.run([e2e_step], K, W)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    max_e2e_serial_ms = reduce_max(sum(e2e_ms), world, device="cuda") / K

    # The same steps as a serving loop runs them: step i + 1's upload (a copy
    # stream, into the other of two device input buffers) overlaps step i's
    # L2 flush, write, decode and download; time per step = elapsed / K.
    up_ds = [up_d, torch.empty_like(up_h, device="cuda")]
    views = [(u[:nq].view(sc.q.shape), u[nq:nq + nk].view(sc.step_k.shape),
              u[nq + nk:].view(sc.step_v.shape)) for u in up_ds]
    copy_stream = torch.cuda.Stream()
    main_stream = torch.cuda.current_stream()

    def e2e_pipelined():
        n = W + K
        up_done = [torch.cuda.Event() for _ in range(n)]
        released = [torch.cuda.Event() for _ in range(n)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(copy_stream):
            up_ds[0].copy_(up_h, non_blocking=True)
            up_done[0].record(copy_stream)
        for i in range(n):
            if i == W:
                timer.clocks.active = True
                t0.record(main_stream)
            if i + 1 < n:  # the next step's inputs, once step i - 1 released that buffer
                with torch.cuda.stream(copy_stream):
                    if i >= 1:
                        copy_stream.wait_event(released[i - 1])
                    up_ds[(i + 1) % 2].copy_(up_h, non_blocking=True)
                    up_done[i + 1].record(copy_stream)
            timer.flush()
            main_stream.wait_event(up_done[i])
            q_i, k_i, v_i = views[i % 2]
            sc.write(k=k_i, v=v_i)
            sc.decode(q=q_i, out=d_out, lse=d_lse)
            released[i].record(main_stream)
            down_h.copy_(down_d, non_blocking=True)
        t1.record(main_stream)
        torch.cuda.synchronize()
        timer.clocks.active = False
        return t0.elapsed_time(t1) / K

    if world > 1:
        torch.distributed.barrier()
    max_e2e_ms = reduce_max(e2e_pipelined(), world, device="cuda")
    if world > 1:
        torch.distributed.barrier()
    assert int(sc.err.item()) == 0, f"device error word {int(sc.err.item())}"
    if rank != 0:
        if world > 1:
            torch.distributed.barrier()
            torch.distributed.destroy_process_group()
        return 0
    ms_per_step = max_total_ms / K
    value = world * sc.scan_bytes / (ms_per_step * 1e-3) / 1e9
    line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": f"{w.fmt} cache (f16 mma, fp32 accumulate)",
            "data": "synthetic: seeded N(0,1) BF16 K/V/Q, 1% outlier channels x16, "
                    "random block table",
            "config": dict(workload_config(w), parallelism=f"dp{world} (sequences per rank)",
                           kv_scan_bytes_per_step=sc.scan_bytes,
                           write_tokens_per_step=int(sc.step_k.shape[0]))}
    # the decode launched alone after a flush: the dominant kernel's roofline
    (decode_ms,), _ = timer.run([sc.decode], K, W)
    (write_ms,), _ = timer.run([sc.write], K, W)
    line["roofline"] = roofline(sc.scan_bytes, decode_ms, peak, peak_kind,
                                profiled_traffic(w.name))
    line["e2e"] = {"value": world * sc.scan_bytes / (max_e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                   "h2d_bytes_per_step": up_h.numel() * 2,
                   "d2h_bytes_per_step": down_h.numel() * 4,
                   "us_per_step": r4(max_e2e_ms * 1e3),
                   "pipelined": "next step's upload under this step's work",
                   "serial_us_per_step": r4(max_e2e_serial_ms * 1e3)}
    line["gpu_launches"] = 2 * K
    line["step_us"] = {"step": r4(ms_per_step * 1e3), "write": r4(statistics.mean(write_ms) * 1e3),
                       "decode": r4(statistics.mean(decode_ms) * 1e3)}
    del sc
    torch.cuda.empty_cache()

    extras = {}
    if not args.no_extras:
        Kx = max(3, K // 2)
        # chunked prefill of the agent step: each sequence's 2,048-token chunk
        # attends causally to its 126,976 cached tokens (tensor-core bound)
        wa = wl.WORKLOADS["agents-fp8-4x127k"]
        s3 = DecodeScenario(wa, device="cuda")
        s3.prefill_setup()
        s3.write()
        (pms,), _ = timer.run([s3.prefill], 3, W)
        assert int(s3.err.item()) == 0
        pk_s, pk_b, pk_kind = measured_tensor_peak()
        tf = s3.prefill_flops / (statistics.mean(pms) * 1e-3) / 1e12
        extras["chunked_prefill_4x127k"] = {
            "ms": r4(statistics.mean(pms)), "TFLOPs": r4(tf),
            "frac_sustained": r4(tf / pk_s), "peak_TFLOPs": pk_s, "peak": pk_kind}
        del s3
        torch.cuda.empty_cache()

        # the calibration abs-max over 65,536 x 8 x 128 BF16
        x = wl.device_tokens(20264, 0, 65536, 8, 128)
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        (cms,), _ = timer.run([lambda: kvq.kv_calibrate_absmax(x, amax)], K, W)
        extras["calibration_64k"] = row(x.numel() * 2, cms, peak)
        del x

        # the FP8 4 x 32,768-token paged workload: the step (4-token write +
        # decode), the decode alone, and a sliding window of 4,096 tokens
        wp = wl.WORKLOADS["fp8-paged-4x32k"]
        s1 = DecodeScenario(wp, device="cuda")

        def step1():
            s1.write()
            s1.decode()

        (s1ms,), _ = timer.run([step1], K, W)
        (d1ms,), _ = timer.run([s1.decode], K, W)
        s1.window_ws(4096)
        (w1ms,), _ = timer.run([lambda: s1.decode_window(4096)], K, W)
        assert int(s1.err.item()) == 0
        extras["swa4096_4x32k"] = row(s1.window_scan_bytes(4096), w1ms, peak)
        extras["paged_4x32k"] = {"step": row(s1.scan_bytes, s1ms, peak),
                                 "decode": row(s1.scan_bytes, d1ms, peak)}
        del s1
        torch.cuda.empty_cache()

        # FP8 attention (E4M3 q and P, both products on E4M3 tensor cores) on
        # the FP8 caches of the agent and the 1 x 65,536-token workloads
        fq = {}
        for key, name in (("4x127k", "agents-fp8-4x127k"), ("1x64k", "nvfp4-1x64k")):
            s4 = DecodeScenario(wl.WORKLOADS[name], fmt="fp8", device="cuda")
            s4.fp8qp_setup()
            (dms,), _ = timer.run([s4.decode_fp8qp], Kx, W)
            assert int(s4.err.item()) == 0
            fq[key] = row(s4.scan_bytes, dms, peak)
            del s4
            torch.cuda.empty_cache()
        extras["fp8_attention"] = fq

        # BF16 vs FP8 vs NVFP4 decode on the byte-heavy 4 x 126,976-token
        # D=128 cache (and the 3-bit PQ3 codec, which needs D=128) and on the
        # 1 x 65,536-token D=64 workload
        for key, name, reps in (("formats_4x127k", "agents-fp8-4x127k", Kx),
                                ("formats_1x64k", "nvfp4-1x64k", K)):
            wf = wl.WORKLOADS[name]
            fm = {}
            fmts = ("bf16", "fp8", "nvfp4", "pq3") if wf.D == 128 else ("bf16", "fp8", "nvfp4")
            for fmt in fmts:
                s2 = DecodeScenario(wf, fmt=fmt, device="cuda")
                (dms,), _ = timer.run([s2.decode], reps, W)
                assert int(s2.err.item()) == 0
                fm[fmt] = row(s2.scan_bytes, dms, peak)
                del s2
                torch.cuda.empty_cache()
            extras[key] = fm

    line["clocks"] = clocks.summary()
    if world == 1 and args.cpu_seconds > 0:
        cb = cpu_baseline(w, w.fmt, args.cpu_seconds)
        gbps, cores, sample = cb["all"]
        line["cpu_baseline"] = {"value": gbps, "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": sample, "one_core_GBps": r4(cb["one"][0])}
    line["peak_GBps"] = {"value": peak, "source": peak_kind}
    line.update(extras)
    print(json.dumps(line))
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
