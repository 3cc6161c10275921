"""Run a few decode (or chunked-prefill) launches of one scenario (for profilers).

    python -m quantized_kv_cache_21_b200.run_decode --workload agents-fp8-4x127k \
        --fmt nvfp4 --seq-len 32768 --launches 4

Builds the named workload's cache (optionally with another format, context
length, batch or head_dim), writes the step's tokens with kv_quantize_write,
then launches kv_decode_attention (with --prefill: kv_prefill_attention of the
step's chunk of new tokens; with --fp8qp: kv_decode_attention_fp8qp over the
FP8 cache) --launches times on the current stream and prints
the device error word and the KV-scan bytes (prefill: algorithmic FLOPs) of one
launch.  Nothing is timed here: bench.py owns timing."""
from __future__ import annotations

import argparse
import dataclasses

import torch

from . import workloads as wl
from .scenario import DecodeScenario


def main(argv=None) -> int:
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--workload", default="fp8-paged-4x32k", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--fmt", choices=["bf16", "fp8", "nvfp4", "pq3"], default=None)
    ap.add_argument("--seq-len", type=int, default=None)
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--head-dim", type=int, choices=[64, 128], default=None)
    ap.add_argument("--launches", type=int, default=4)
    ap.add_argument("--prefill", action="store_true",
                    help="launch the chunk's prefill attention instead of the decode")
    ap.add_argument("--fp8qp", action="store_true",
                    help="launch the FP8 attention (E4M3 q and P) over an FP8 cache")
    args = ap.parse_args(argv)
    w = wl.WORKLOADS[args.workload]
    over = {}
    if args.seq_len is not None:
        over.update(seq_len=args.seq_len, calib_tokens=None)
    if args.batch is not None:
        over["B"] = args.batch
    if args.head_dim is not None:
        over["D"] = args.head_dim
    w = dataclasses.replace(w, **over) if over else w
    sc = DecodeScenario(w, fmt=args.fmt or w.fmt)
    sc.write()  # the step's own tokens, so the scanned cache is complete
    if args.prefill:
        sc.prefill_setup()
    if args.fp8qp:
        sc.fp8qp_setup()
    for _ in range(args.launches):
        if args.prefill:
            sc.prefill()
        elif args.fp8qp:
            sc.decode_fp8qp()
        else:
            sc.decode()
    torch.cuda.synchronize()
    what = (f"prefill chunk {sc.chunk}, FLOPs per launch {sc.prefill_flops}" if args.prefill
            else f"KV-scan bytes per launch {sc.scan_bytes}")
    print(f"workload {w.name} fmt {sc.fmt} B {sc.B} L {sc.L} D {sc.D}: "
          f"device error word {int(sc.err.item())}, {what}")
    return 0 if int(sc.err.item()) == 0 else 1


if __name__ == "__main__":
    raise SystemExit(main())
