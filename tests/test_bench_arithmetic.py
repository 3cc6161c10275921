"""The benchmark's algorithmic work counts against brute force: KV-scan bytes
of a decode (every cached token's K and V, block scales included for NVFP4)
and FLOPs of a chunked prefill (4 D Hq per query row and attended key, the
chunk's queries attending causally up to their own positions)."""
import numpy as np
import pytest

from quantized_kv_cache_21_b200.scenario import kv_scan_bytes, prefill_flops


@pytest.mark.parametrize("lens,chunk", [([37, 16, 70], 16), ([5], 9), ([2048, 4096], 2048),
                                        ([0, 1, 3], 2), ([126976] * 4, 2048)])
def test_prefill_flops_brute_force(lens, chunk):
    Hq, D = 12, 64
    keys = 0
    for n in lens:
        for i in range(chunk):
            pos = n - chunk + i
            keys += max(0, pos + 1)  # cache tokens 0..pos
    assert prefill_flops(lens, chunk, Hq, D) == 4 * D * Hq * keys


def test_prefill_flops_of_the_benchmark_step():
    # 4 sequences of 126,976 tokens, their last 2,048 as the chunk, 64 query
    # heads, head_dim 128: 33.81 TFLOP
    assert prefill_flops([126976] * 4, 2048, 64, 128) == 33_810_116_771_840


def test_kv_scan_bytes_brute_force():
    H, D = 3, 128
    lens = np.array([17, 0, 100])
    per_elem = {"bf16": 2.0, "fp8": 1.0, "nvfp4": 0.5 + 1 / 16, "pq3": (4 + 48) / 128}
    for fmt, b in per_elem.items():
        elems = sum(int(n) for n in lens) * H * D * 2  # K and V
        assert kv_scan_bytes(fmt, lens, H, D) == round(elems * b)
