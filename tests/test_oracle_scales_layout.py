"""Pins of the oracle's scales, byte arithmetic, paged layout and quantizers.

The scale formula and the byte figures are the ones printed on the pages
(tests/golden/page_byte_pins.json, each entry cited); the layout is checked by
rebuilding the expected cache bytes with numpy indexing; codes are checked
against the ml_dtypes conversions applied to the same fp32 quotients."""
import json
import os

import ml_dtypes
import numpy as np
import pytest

import oracle
from quantized_kv_cache_21_b200 import workloads as wl

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_byte_pins.json")))
E4M3 = ml_dtypes.float8_e4m3fn
E2M1 = ml_dtypes.float4_e2m1fn


def test_fp8_scale_closed_forms():
    c = GOLD["fp8_scale_constants"]
    assert oracle.fp8_scale(0.0) == np.float32(c["floor"])           # the 1e-12 floor
    assert oracle.fp8_scale(1e-15) == np.float32(c["floor"])
    # amax = 1: 1.05 / 448 = 3/1280 = 0.00234375; fp32 evaluation lands within 1 ulp
    s1 = np.float32(oracle.fp8_scale(1.0))
    assert abs(float(s1) - 0.00234375) <= float(np.spacing(np.float32(0.00234375)))
    # amax = 448: the scale is 1.05 to within 1 ulp
    s448 = np.float32(oracle.fp8_scale(448.0))
    assert abs(float(s448) - 1.05) <= float(np.spacing(np.float32(1.05)))


def test_fp8_scale_headroom_and_monotone():
    amax = np.float32(10.0) ** np.linspace(-10, 6, 3001).astype(np.float32)
    s = np.array([oracle.fp8_scale(a) for a in amax], np.float32)
    assert np.all(np.diff(s) >= 0)
    big = amax > 1e-9
    # 5% headroom: the calibrated maximum maps to 448/1.05 = 426.7, never saturating
    q = amax[big] / s[big]
    assert np.all(q < 427.0) and np.all(q > 426.0)
    codes = oracle.e4m3_encode(q)
    assert np.all(codes < 0x7E)


def test_nvfp4_global_scale():
    for a in [1.0, 3.5, 72.25, 1e-3, 448.0 * 6]:
        g = np.float32(oracle.nvfp4_global_scale(a))
        assert abs(float(g) * 2688.0 - a) <= a * 2.0 ** -23
        # a block holding the tensor maximum gets (about) the largest block scale
        sb = oracle.e4m3_encode([np.float32(a) / (np.float32(6.0) * g)])[0]
        assert sb == 0x7E
    assert oracle.nvfp4_global_scale(0.0) == 0.0


def test_bytes_per_element_pins():
    bpe = GOLD["bytes_per_element"]
    H, D = 8, 128
    assert oracle.kv_bytes_per_token("bf16", H, D) == 2 * H * D * bpe["bf16"]
    assert oracle.kv_bytes_per_token("fp8", H, D) == 2 * H * D * bpe["fp8"]
    nv = GOLD["nvfp4_bits_per_element"]
    assert oracle.kv_bytes_per_token("nvfp4", H, D) == 2 * H * D * nv["value"] / 8
    ratio = oracle.kv_bytes_per_token("fp8", H, D) / oracle.kv_bytes_per_token("nvfp4", H, D)
    assert round(ratio, 1) == nv["smaller_than_fp8"]
    # the head-page sizes the layout actually stores agree with those rates
    for D_ in (64, 128):
        assert oracle.head_page_bytes("nvfp4", D_) * 8 == 16 * D_ * 4.5
        assert oracle.head_page_bytes("fp8", D_) == 16 * D_
        assert oracle.head_page_bytes("bf16", D_) == 32 * D_


def test_cache_size_pins():
    g = GOLD["gb10_128k_context"]
    gib = 2.0 ** 30
    bf = g["bf16_bytes_per_token"] * g["tokens"]
    assert bf / gib == g["bf16_GB"]
    r8 = oracle.kv_bytes_per_token("fp8", 8, 64) / oracle.kv_bytes_per_token("bf16", 8, 64)
    assert bf * r8 / gib == g["fp8_GB"]
    r4 = oracle.kv_bytes_per_token("nvfp4", 8, 64) / oracle.kv_bytes_per_token("bf16", 8, 64)
    # the page's 0.75 GB is the 4.0-bit rate; with the E4M3 block scales it is 4.5 bits
    assert abs(bf * r4 / gib - g["nvfp4_rate_GB"] * 4.5 / 4.0) < 1e-12
    m = GOLD["mi300x_fp16_cache_32k"]
    full = oracle.kv_bytes_per_token("bf16", m["kv_heads"], m["head_dim"]) * m["tokens"]
    # the page's "~134 MB" and "~16 MB" are both the decimal MB figure truncated
    assert int(full / 1e6) == m["full_MB"]
    win = oracle.kv_bytes_per_token("bf16", m["kv_heads"], m["head_dim"]) * m["window"]
    assert int(win / 1e6) == m["window_MB"]


def test_absmax_matches_numpy_and_finds_planted_max():
    rng = wl.rng_for(7, 0)
    x = wl.make_tokens(rng, 300, 3, 64)
    ref = np.abs(wl.bf16_bits_to_f32(x)).max()
    assert oracle.absmax_bf16(x) == ref
    x2 = x.copy()
    x2[123, 1, 17] = wl.f32_to_bf16_bits(np.array([-1234.5], np.float32))[0]
    assert oracle.absmax_bf16(x2) == np.float32(wl.bf16_bits_to_f32(x2[123, 1, 17:18])[0] * -1)
    assert oracle.absmax_bf16(np.zeros(10, np.uint16)) == 0.0


def _expected_fp8_cache(k_bits, slots, nb, H, D, s):
    """FP8 cache bytes rebuilt with numpy indexing and the library E4M3 cast."""
    cache = np.zeros((nb, H, 16, D), np.uint8)
    x = wl.bf16_bits_to_f32(k_bits) / np.float32(s)
    codes = x.astype(E4M3).view(np.uint8)
    sat = np.abs(x) >= 448
    codes[sat] = np.where(x[sat] > 0, 0x7E, 0xFE)
    for t, slot in enumerate(slots):
        if slot >= 0:
            cache[slot // 16, :, slot % 16, :] = codes[t]
    return cache.reshape(-1)


def test_fp8_write_layout_and_codes():
    rng = wl.rng_for(11, 0)
    T, H, D, nb = 40, 3, 64, 5
    k = wl.make_tokens(rng, T, H, D, [(0, 5), (2, 9)], 30.0)
    v = wl.make_tokens(rng, T, H, D)
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    slots[3] = -1  # skipped
    amax = oracle.absmax_bf16(k[:20])  # calibrate on a prefix so later tokens can saturate
    s = oracle.fp8_scale(amax)
    kc, vc = oracle.new_cache("fp8", nb, H, D)
    assert oracle.write("fp8", k, v, slots, kc, vc, s, 1.0) == 0
    assert np.array_equal(kc, _expected_fp8_cache(k, slots, nb, H, D, s))
    assert np.array_equal(vc, _expected_fp8_cache(v, slots, nb, H, D, 1.0))
    # dequantisation returns code * scale at those slots
    ko, _ = oracle.dequantize("fp8", kc, vc, H, D, slots[slots >= 0], s, 1.0)
    codes = kc.reshape(nb, H, 16, D)[slots[slots >= 0] // 16, :, slots[slots >= 0] % 16, :]
    assert np.array_equal(ko, codes.view(E4M3).astype(np.float32) * np.float32(s))
    # an out-of-range slot is reported and not written
    bad = slots.copy()
    bad[0] = nb * 16
    kc2, vc2 = oracle.new_cache("fp8", nb, H, D)
    assert oracle.write("fp8", k, v, bad, kc2, vc2, s, 1.0) == -1


def test_bf16_write_layout():
    rng = wl.rng_for(12, 0)
    T, H, D, nb = 20, 2, 64, 2
    k = wl.make_tokens(rng, T, H, D)
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    kc, vc = oracle.new_cache("bf16", nb, H, D)
    oracle.write("bf16", k, k, slots, kc, vc, 1.0, 1.0)
    want = np.zeros((nb, H, 16, D), np.uint16)
    want[slots // 16, :, slots % 16, :] = k
    assert np.array_equal(kc.view(np.uint16), want.reshape(-1))


@pytest.mark.parametrize("D", [64, 128])
def test_nvfp4_write_layout_and_codes(D):
    rng = wl.rng_for(13, D)
    T, H, nb = 37, 2, 4
    k = wl.make_tokens(rng, T, H, D, [(1, 3)], 16.0)
    k[5, 0, :16] = 0  # an all-zero block
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    amax = oracle.absmax_bf16(k[:10])
    g = np.float32(oracle.nvfp4_global_scale(amax))
    kc, vc = oracle.new_cache("nvfp4", nb, H, D)
    oracle.write("nvfp4", k, k, slots, kc, vc, g, g)
    # rebuild with numpy: per 16-element block, sb = E4M3(bmax / (6 g)),
    # e = E2M1(x / (dec(sb) * g)), two codes per byte (even element low nibble)
    x = wl.bf16_bits_to_f32(k).reshape(T, H, D // 16, 16)
    bmax = np.abs(x).max(axis=-1)
    q = bmax / (np.float32(6.0) * g)
    sb = q.astype(E4M3).view(np.uint8)
    sb[q >= 448] = 0x7E
    den = sb.view(E4M3).astype(np.float32) * g
    with np.errstate(divide="ignore", invalid="ignore"):
        e = (x / den[..., None]).astype(E2M1).view(np.uint8) & 0xF
    e[den == 0] = 0
    e = e.reshape(T, H, D)
    packed = (e[..., 0::2] | (e[..., 1::2] << 4)).astype(np.uint8)  # [T][H][D/2]
    want = np.zeros((nb, H, 9 * D), np.uint8)
    for t, slot in enumerate(slots):
        b, o = slot // 16, slot % 16
        want[b, :, o * D // 2:(o + 1) * D // 2] = packed[t]
        want[b, :, 8 * D + o * D // 16: 8 * D + (o + 1) * D // 16] = sb[t]
    assert np.array_equal(kc, want.reshape(-1))
    # the zero block: scale 0 and codes 0
    b5, o5 = slots[5] // 16, slots[5] % 16
    assert want[b5, 0, 8 * D + o5 * D // 16] == 0
    # dequantisation: e * sb * g
    ko, _ = oracle.dequantize("nvfp4", kc, vc, H, D, slots, g, g)
    ref = (e.view(np.uint8).view(E2M1).astype(np.float32).reshape(T, H, D // 16, 16)
           * sb.view(E4M3).astype(np.float32)[..., None]) * g
    assert np.array_equal(ko, ref.reshape(T, H, D))


def test_nvfp4_zero_global_scale_gives_zero_codes():
    k = np.zeros((3, 1, 64), np.uint16)
    kc, vc = oracle.new_cache("nvfp4", 1, 1, 64, fill=0xAB)
    oracle.write("nvfp4", k, k, np.arange(3), kc, vc, 0.0, 0.0)
    page = kc.reshape(9 * 64)
    assert np.all(page[: 3 * 32] == 0) and np.all(page[512: 512 + 12] == 0)
    assert np.all(page[3 * 32: 512] == 0xAB)  # untouched slots keep their bytes
