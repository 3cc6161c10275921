"""Seeded synthetic inputs shaped like the pages' workloads.

This module holds only input generation: random normal K/V/Q rounded to BF16,
outlier channels, block tables, slot mappings and sequence lengths.  It holds
none of the method's arithmetic (no quantisation, scales or attention), so both
the CUDA path's tests and the CPU oracle can be fed from it.

Recipe (all fp32 draws rounded to BF16 with round-to-nearest-even):
  * K, V, Q ~ N(0, 1).
  * Outlier channels: a seeded set of (kv_head, channel) pairs of K and,
    independently, of V is multiplied by a factor for every token.
  * Block tables: a seeded random permutation of a shared block pool, sliced
    per sequence (sequence b owns blocks perm[b*nb:(b+1)*nb]).
  * Workload sizes follow the agent-context shapes the pages discuss:
    32k-127k-token contexts, 8 KV heads, head_dim 64-128, GQA 8.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

PAGE = 16


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to BF16 (nearest, ties to even); returns uint16 bits.
    Inputs here are finite draws, so NaN handling is not needed."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = 0x7FFF + ((u >> 16) & 1)
    return ((u + rounding) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng_for(seed: int, stream: int) -> np.random.Generator:
    """Independent sub-stream ``stream`` of seed ``seed``."""
    return np.random.default_rng(np.random.SeedSequence(seed, spawn_key=(stream,)))


def outlier_pairs(rng: np.random.Generator, H: int, D: int, per_head: int | None = None,
                  frac: float | None = None) -> list[tuple[int, int]]:
    """Outlier (head, channel) pairs: ``per_head`` channels in every head, or
    round(frac * H * D) pairs drawn over all heads."""
    if per_head is not None:
        return [(h, int(c)) for h in range(H) for c in rng.choice(D, per_head, replace=False)]
    n = int(round((frac or 0.0) * H * D))
    flat = rng.choice(H * D, n, replace=False)
    return [(int(i) // D, int(i) % D) for i in flat]


def make_tokens(rng: np.random.Generator, T: int, H: int, D: int,
                outliers: list[tuple[int, int]] = (), factor: float = 1.0) -> np.ndarray:
    """[T][H][D] BF16 bits, N(0,1) with the listed channels scaled by factor."""
    x = rng.standard_normal((T, H, D), dtype=np.float32)
    for h, c in outliers:
        x[:, h, c] *= np.float32(factor)
    return f32_to_bf16_bits(x)


def make_query(rng: np.random.Generator, B: int, Hq: int, D: int) -> np.ndarray:
    return f32_to_bf16_bits(rng.standard_normal((B, Hq, D), dtype=np.float32))


def permuted_block_table(rng: np.random.Generator, B: int, blocks_per_seq: int,
                         num_blocks: int | None = None) -> np.ndarray:
    """[B][blocks_per_seq] int32: a random permutation of a shared pool."""
    nb = num_blocks if num_blocks is not None else B * blocks_per_seq
    perm = rng.permutation(nb).astype(np.int32)
    return perm[: B * blocks_per_seq].reshape(B, blocks_per_seq)


def identity_block_table(B: int, blocks_per_seq: int) -> np.ndarray:
    return np.arange(B * blocks_per_seq, dtype=np.int32).reshape(B, blocks_per_seq)


def physical_slots(block_table: np.ndarray, b: int, positions: np.ndarray) -> np.ndarray:
    """Physical slot (block * 16 + offset) of the given positions of sequence b."""
    pos = np.asarray(positions, dtype=np.int64)
    return block_table[b, pos // PAGE].astype(np.int64) * PAGE + pos % PAGE


def planar_rotation(rng: np.random.Generator, pairs: int = 64) -> np.ndarray:
    """[pairs][2] fp32 (cos, sin) of seeded angles uniform in [0, 2 pi): the
    random planar rotation a 3-bit rotation codec applies to each head vector
    (an input drawn once per tensor, like a scale)."""
    theta = rng.uniform(0.0, 2.0 * np.pi, size=pairs)
    return np.stack([np.cos(theta), np.sin(theta)], axis=1).astype(np.float32)


def varlen(rng: np.random.Generator, B: int, L: int) -> np.ndarray:
    """Per-sequence lengths uniform in [ceil(L/2), L]."""
    return rng.integers((L + 1) // 2, L + 1, size=B).astype(np.int32)


@dataclass
class Workload:
    """A named workload: sizes plus the outlier recipe.  Seed of a workload is
    fixed by its name so every run draws the same inputs."""
    name: str
    fmt: str
    B: int
    Hkv: int
    Hq: int
    D: int
    seq_len: int
    seed: int
    k_outliers: dict = field(default_factory=dict)
    v_outliers: dict = field(default_factory=dict)
    outlier_factor: float = 1.0
    calib_tokens: int | None = None  # scales from the first N tokens of sequence 0
    permuted: bool = True
    write_chunk: int = 0  # tokens per sequence quantized-on-write each step


WORKLOADS = {
    # 1 sequence x 1024 tokens, 2 KV heads, GQA 4, D 64; two outlier channels
    # per head scaled x20; blocks laid out in order (a contiguous cache).
    "tiny-fp8-1k": Workload("tiny-fp8-1k", "fp8", 1, 2, 8, 64, 1024, 20260,
                            {"per_head": 2}, {"per_head": 2}, 20.0, None, False),
    # 4 x 32,768 tokens, 8 KV heads, 64 query heads, D 128; 1% outlier
    # channels x16; scales from a 16,384-token sample; random block table.
    "fp8-paged-4x32k": Workload("fp8-paged-4x32k", "fp8", 4, 8, 64, 128, 32768, 20261,
                                {"frac": 0.01}, {"frac": 0.01}, 16.0, 16384, True),
    # 1 x 65,536 tokens, 8 KV heads, 64 query heads, D 64, NVFP4 (also run as
    # BF16 and FP8 on the same inputs).
    "nvfp4-1x64k": Workload("nvfp4-1x64k", "nvfp4", 1, 8, 64, 64, 65536, 20262,
                            {}, {}, 1.0, None, True),
    # 4 agents x 126,976 tokens, FP8, D 128; each step writes a 2048-token
    # chunk per sequence, then decodes.
    "agents-fp8-4x127k": Workload("agents-fp8-4x127k", "fp8", 4, 8, 64, 128, 126976, 20263,
                                  {"frac": 0.01}, {"frac": 0.01}, 16.0, 16384, True, 2048),
}

# The sweep: context L in 1k/4k/16k/64k/128k tokens x batch 1/8/32/64, lengths
# uniform in [L/2, L] (varlen), GQA 8 (8 KV heads, 64 query heads), head_dim
# 64 and 128, BF16/FP8/NVFP4; plain N(0,1) K/V.  One cell = this template with
# B, D and seq_len set, and per-sequence lengths drawn with
# varlen(rng_for(SWEEP_SEED, sweep_cell_stream(L, B)), B, L).
SWEEP_LENGTHS = (1024, 4096, 16384, 65536, 131072)
SWEEP_BATCHES = (1, 8, 32, 64)
SWEEP_SEED = 20264
SWEEP = Workload("sweep", "fp8", 1, 8, 64, 128, 1024, SWEEP_SEED)


def sweep_cell_stream(L: int, B: int) -> int:
    """Sub-stream of a sweep cell's length draw (same lengths for every format
    and head_dim)."""
    return 1000 + 10 * SWEEP_LENGTHS.index(L) + SWEEP_BATCHES.index(B)


def device_tokens(seed: int, stream: int, T: int, H: int, D: int,
                  outliers: list[tuple[int, int]] = (), factor: float = 1.0,
                  device: str = "cuda"):
    """[T][H][D] bf16 on the device: N(0, 1) from torch's seeded CUDA generator
    (sub-stream ``stream``), listed channels scaled by ``factor``, rounded to
    BF16 (nearest even).  Used for the large workloads, which are too big to
    draw on the host quickly."""
    import torch

    g = torch.Generator(device=device)
    g.manual_seed(seed * 1000003 + stream)
    x = torch.randn((T, H, D), generator=g, device=device, dtype=torch.float32)
    for h, c in outliers:
        x[:, h, c] *= factor
    return x.to(torch.bfloat16)


def outliers_for(w: "Workload", H: int, D: int, which: str) -> list[tuple[int, int]]:
    """The workload's outlier pairs for K ("k") or V ("v")."""
    spec = w.k_outliers if which == "k" else w.v_outliers
    if not spec:
        return []
    return outlier_pairs(rng_for(w.seed, 100 if which == "k" else 101), H, D,
                         per_head=spec.get("per_head"), frac=spec.get("frac"))
