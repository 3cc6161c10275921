"""GPU parity of the write side against the oracle, bit for bit: FP8 and NVFP4
codes and block scales (including an exhaustive sweep of every BF16 input
through the E4M3 encoder and every E2M1 rounding case), the paged scatter
(physical and block-table-translated slots), dequantisation, the calibration
abs-max and the per-layer scale."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl

from gpu_common import DEV, cache_bytes, dev_scalar, new_err, to_dev_bits

pytestmark = pytest.mark.gpu


def all_finite_bf16():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = wl.bf16_bits_to_f32(bits)
    return bits[~np.isnan(x)]


def write_both(fmt, k, v, slots, nb, ks, vs, fill=0):
    """Write with the oracle and with the library; return both caches + error word."""
    T, H, D = k.shape
    okc, ovc = oracle.new_cache(fmt, nb, H, D, fill=fill)
    oracle.write(fmt, k, v, slots, okc, ovc, ks, vs)
    cache = kvq.KVCache(fmt, nb, H, D)
    cache.k.fill_(fill)
    cache.v.fill_(fill)
    err = new_err()
    kvq.kv_quantize_write(fmt, to_dev_bits(k), to_dev_bits(v), torch.from_numpy(slots).to(DEV),
                          cache, dev_scalar(ks), dev_scalar(vs), err)
    gk, gv = cache_bytes(cache)
    return okc, ovc, gk, gv, int(err.item()), cache


@pytest.mark.parametrize("scale", [1.0, 0.125, 3.0517578125e-05, 0.0234375, 1e-12, 0.7,
                                   33333.0, oracle.scale_from_absmax("fp8", 7.3),
                                   1.0 / 3.0, 3.0, 7.0, 11.0, 0.3, 3.1415927, 0.0098765, 271.828,
                                   5.5e-7, 1.7e-10,
                                   oracle.scale_from_absmax("fp8", 81.25),
                                   oracle.scale_from_absmax("fp8", 4.6)])
def test_fp8_every_bf16_input(scale):
    """All 65,280 finite BF16 values through x / s -> E4M3 (s = 1 makes it the
    bare encoder; the other scales move every value across binades; scales
    that are not powers of two make x / s a true division; with s = 3, 7, 11
    or 0.3 a reciprocal product x * RN(1/s) would encode some inputs
    differently, e.g. 3.1875 / 3 = 1.0625 is a tie that the product lifts
    above)."""
    bits = all_finite_bf16()
    H, D = 1, 64
    T = bits.size // D  # 65280 = 1020 * 64
    k = bits[: T * D].reshape(T, H, D)
    v = k[::-1].copy()
    slots = np.arange(T, dtype=np.int64)
    okc, ovc, gk, gv, err, _ = write_both("fp8", k, v, slots, -(-T // 16), scale, scale)
    assert err == 0
    assert np.array_equal(gk, okc) and np.array_equal(gv, ovc)


def test_e2m1_every_rounding_case():
    """NVFP4 blocks whose block scale decodes to exactly 1 (g = 1/8, block max
    0.75): every other element is x / 0.125 = 8x, so all BF16 values in
    [-0.75, 0.75] run through the E2M1 encoder, ties and signed zeros included."""
    bits = all_finite_bf16()
    x = wl.bf16_bits_to_f32(bits)
    vals = bits[np.abs(x) <= 0.75]
    per_block = 15
    nblk = -(-vals.size // per_block)
    vals = np.concatenate([vals, np.zeros(nblk * per_block - vals.size, np.uint16)])
    top = wl.f32_to_bf16_bits(np.array([0.75], np.float32))[0]
    blocks = np.concatenate([vals.reshape(nblk, per_block), np.full((nblk, 1), top, np.uint16)], 1)
    D = 64
    nrow = -(-nblk // (D // 16))
    blocks = np.concatenate([blocks, np.zeros((nrow * 4 - nblk, 16), np.uint16)])
    k = blocks.reshape(nrow, 1, D)
    slots = np.arange(nrow, dtype=np.int64)
    okc, ovc, gk, gv, err, _ = write_both("nvfp4", k, k, slots, -(-nrow // 16), 0.125, 0.125)
    assert err == 0
    assert np.array_equal(gk, okc) and np.array_equal(gv, ovc)


def test_e2m1_every_rounding_case_with_an_inexact_divisor():
    """As above with g = 0.1 and a block maximum of BF16(0.825): the block
    scale encodes to 1.375 and every element is divided by 1.375 * fp32(0.1),
    which is not a power of two, so each E2M1 input is a rounded quotient."""
    bits = all_finite_bf16()
    x = wl.bf16_bits_to_f32(bits)
    top = wl.f32_to_bf16_bits(np.array([0.825], np.float32))[0]
    vals = bits[np.abs(x) <= wl.bf16_bits_to_f32(np.array([top]))[0]]
    per_block = 15
    nblk = -(-vals.size // per_block)
    vals = np.concatenate([vals, np.zeros(nblk * per_block - vals.size, np.uint16)])
    blocks = np.concatenate([vals.reshape(nblk, per_block), np.full((nblk, 1), top, np.uint16)], 1)
    D = 128
    nrow = -(-nblk // (D // 16))
    blocks = np.concatenate([blocks, np.zeros((nrow * (D // 16) - nblk, 16), np.uint16)])
    k = blocks.reshape(nrow, 1, D)
    slots = np.arange(nrow, dtype=np.int64)
    g = float(np.float32(0.1))
    okc, ovc, gk, gv, err, _ = write_both("nvfp4", k, k, slots, -(-nrow // 16), g, g)
    assert err == 0
    assert np.array_equal(gk, okc) and np.array_equal(gv, ovc)


def test_e2m1_rounding_with_a_subnormal_divisor():
    """g = 2^-130 (a subnormal fp32 scale) and a block maximum of 6 g: the block
    scale decodes to 1, every element is divided by the subnormal 2^-130, and
    the BF16 subnormals up to 6 g give the quotients k / 8 for k = 0..48, which
    hit every E2M1 tie exactly (1/(2^-130) is not a finite fp32 number, so a
    reciprocal-based division would not do)."""
    g = 2.0 ** -130
    bits = all_finite_bf16()
    x = wl.bf16_bits_to_f32(bits)
    top = wl.f32_to_bf16_bits(np.array([6 * g], np.float32))[0]
    vals = bits[np.abs(x) <= 6 * g]
    assert vals.size == 2 * 49  # +-k * 2^-133 for k = 0..48 (both zeros)
    per_block = 15
    nblk = -(-vals.size // per_block)
    vals = np.concatenate([vals, np.zeros(nblk * per_block - vals.size, np.uint16)])
    blocks = np.concatenate([vals.reshape(nblk, per_block), np.full((nblk, 1), top, np.uint16)], 1)
    D = 64
    nrow = -(-nblk // (D // 16))
    blocks = np.concatenate([blocks, np.zeros((nrow * (D // 16) - nblk, 16), np.uint16)])
    k = blocks.reshape(nrow, 1, D)
    slots = np.arange(nrow, dtype=np.int64)
    okc, ovc, gk, gv, err, _ = write_both("nvfp4", k, k, slots, 1, g, g)
    assert err == 0
    assert np.array_equal(gk, okc) and np.array_equal(gv, ovc)


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("D", [64, 128])
def test_random_write_matches_oracle(fmt, D):
    rng = wl.rng_for(500 + D, 0)
    T, H, nb = 300, 3, 40
    outl = wl.outlier_pairs(rng, H, D, per_head=2)
    k = wl.make_tokens(rng, T, H, D, outl, 20.0)
    v = wl.make_tokens(rng, T, H, D, outl, 20.0)
    k[7, 1, :16] = 0  # an all-zero NVFP4 block
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    slots[11] = -1  # skipped token
    # scales from the first 100 tokens: later outliers saturate
    ks = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(k[:100]))
    vs = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(v[:100]))
    okc, ovc, gk, gv, err, _ = write_both(fmt, k, v, slots, nb, ks, vs, fill=0xA5)
    assert err == 0
    assert np.array_equal(gk, okc) and np.array_equal(gv, ovc)


def test_block_table_translation_matches_physical():
    rng = wl.rng_for(77, 0)
    B, H, D, mb = 3, 2, 128, 9
    nb = B * mb + 2
    bt = wl.permuted_block_table(rng, B, mb, nb)
    T = 90
    seq = rng.integers(0, B, T)
    pos = rng.permutation(mb * 16)[:T]
    k = wl.make_tokens(rng, T, H, D)
    logical = (seq * mb * 16 + pos).astype(np.int64)
    physical = np.array([wl.physical_slots(bt, s, [p])[0] for s, p in zip(seq, pos)], np.int64)
    ks = oracle.fp8_scale(oracle.absmax_bf16(k))
    okc, ovc, gk, gv, err, _ = write_both("fp8", k, k, physical, nb, ks, ks)
    cache = kvq.KVCache("fp8", nb, H, D)
    e2 = new_err()
    kvq.kv_quantize_write("fp8", to_dev_bits(k), to_dev_bits(k), torch.from_numpy(logical).to(DEV),
                          cache, dev_scalar(ks), dev_scalar(ks), e2,
                          block_table=torch.from_numpy(bt).to(DEV))
    tk, tv = cache_bytes(cache)
    assert err == 0 and int(e2.item()) == 0
    assert np.array_equal(tk, okc) and np.array_equal(tv, ovc)


@pytest.mark.parametrize("H,D,T", [(8, 128, 3001), (2, 64, 3001), (32, 128, 1001)])
def test_large_fp8_write_matches_oracle(H, D, T):
    """Writes of a thousand and more tokens (8 tokens per block, grid of
    hundreds of blocks, a ragged last block): logical slots through a block
    table, skipped tokens and one slot past the last sequence, bit-exact
    against the oracle; a bad K scale writes no K byte and still writes V."""
    rng = wl.rng_for(79 + H + D, 0)
    B = 3
    mb = -(-T // (16 * B)) + 2
    nb = B * mb + 1
    bt = wl.permuted_block_table(rng, B, mb, nb)
    outl = wl.outlier_pairs(rng, H, D, per_head=1)
    k = wl.make_tokens(rng, T, H, D, outl, 16.0)
    v = wl.make_tokens(rng, T, H, D, outl, 16.0)
    seq = np.arange(T) % B
    pos = np.arange(T) // B
    logical = (seq * mb * 16 + pos).astype(np.int64)
    physical = np.array([wl.physical_slots(bt, sq, [ps])[0] for sq, ps in zip(seq, pos)], np.int64)
    logical[[5, 1500 % T, T - 1]] = -1
    physical[[5, 1500 % T, T - 1]] = -1
    logical[17] = B * mb * 16 + 3  # a sequence past num_seqs: reported, skipped
    physical[17] = -1
    ks = oracle.fp8_scale(oracle.absmax_bf16(k[:200]))  # later outliers saturate
    vs = oracle.fp8_scale(oracle.absmax_bf16(v[:200]))
    okc, ovc = oracle.new_cache("fp8", nb, H, D, fill=0x5A)
    oracle.write("fp8", k, v, physical, okc, ovc, ks, vs)
    cache = kvq.KVCache("fp8", nb, H, D)
    cache.k.fill_(0x5A)
    cache.v.fill_(0x5A)
    err = new_err()
    kvq.kv_quantize_write("fp8", to_dev_bits(k), to_dev_bits(v), torch.from_numpy(logical).to(DEV),
                          cache, dev_scalar(ks), dev_scalar(vs), err,
                          block_table=torch.from_numpy(bt).to(DEV))
    gk, gv = cache_bytes(cache)
    assert int(err.item()) == kvq.DERR_SLOT
    assert np.array_equal(gk, okc) and np.array_equal(gv, ovc)
    # a bad K scale on a large write: no K byte is written, V still is
    cache.k.fill_(0x5A)
    cache.v.fill_(0x5A)
    e = new_err()
    kvq.kv_quantize_write("fp8", to_dev_bits(k), to_dev_bits(v), torch.from_numpy(logical).to(DEV),
                          cache, dev_scalar(float("nan")), dev_scalar(vs), e,
                          block_table=torch.from_numpy(bt).to(DEV))
    gk, gv = cache_bytes(cache)
    assert int(e.item()) == kvq.DERR_SLOT | kvq.DERR_SCALE
    assert np.all(gk == 0x5A) and np.array_equal(gv, ovc)


def test_bad_slots_and_scales_are_reported_not_written():
    rng = wl.rng_for(78, 0)
    H, D, nb = 1, 64, 2
    k = wl.make_tokens(rng, 4, H, D)
    slots = np.array([0, nb * 16, 5, -3], np.int64)  # one beyond the cache, one skipped
    okc, ovc, gk, gv, err, _ = write_both("fp8", k, k, slots, nb, 0.01, 0.01)
    assert err == kvq.DERR_SLOT
    assert np.array_equal(gk, okc)  # the oracle skips the same token
    # logical slot of a sequence past num_seqs, and a table entry outside the pool
    cache = kvq.KVCache("fp8", nb, H, D)
    bt = torch.tensor([[0, 99]], dtype=torch.int32, device=DEV)
    e = new_err()
    kvq.kv_quantize_write("fp8", to_dev_bits(k[:2]), to_dev_bits(k[:2]),
                          torch.tensor([2 * 32 + 1, 17], dtype=torch.int64, device=DEV), cache,
                          dev_scalar(0.01), dev_scalar(0.01), e, block_table=bt)
    assert int(e.item()) == kvq.DERR_SLOT | kvq.DERR_BLOCK_ID
    assert int(cache.k.count_nonzero().item()) == 0
    # non-positive or non-finite scales: nothing written, error raised
    for bad in (0.0, -1.0, float("nan"), float("inf")):
        cache = kvq.KVCache("fp8", nb, H, D)
        e = new_err()
        kvq.kv_quantize_write("fp8", to_dev_bits(k), to_dev_bits(k),
                              torch.arange(4, dtype=torch.int64, device=DEV), cache,
                              dev_scalar(bad), dev_scalar(0.01), e)
        assert int(e.item()) & kvq.DERR_SCALE
        assert int(cache.k.count_nonzero().item()) == 0
    cache = kvq.KVCache("nvfp4", nb, H, D)
    e = new_err()
    kvq.kv_quantize_write("nvfp4", to_dev_bits(k), to_dev_bits(k),
                          torch.arange(4, dtype=torch.int64, device=DEV), cache,
                          dev_scalar(-0.5), dev_scalar(0.01), e)
    assert int(e.item()) & kvq.DERR_SCALE


def test_host_argument_errors():
    cache = kvq.KVCache("fp8", 2, 1, 64)
    k = torch.zeros(4, 1, 64, dtype=torch.bfloat16, device=DEV)
    s = torch.arange(4, dtype=torch.int64, device=DEV)
    with pytest.raises(kvq.KvqError, match="scale"):
        kvq.kv_quantize_write("fp8", k, k, s, cache, None, None)
    with pytest.raises(kvq.KvqError, match="format"):
        kvq.kv_quantize_write("nvfp4", k, k, s, cache, dev_scalar(1), dev_scalar(1))
    with pytest.raises(kvq.KvqError):
        kvq.KVCache("fp8", 2, 1, 80)


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("D", [64, 128])
def test_dequantize_matches_oracle(fmt, D):
    rng = wl.rng_for(600 + D, 1)
    T, H, nb = 64, 2, 8
    k = wl.make_tokens(rng, T, H, D, [(0, 3)], 12.0)
    v = wl.make_tokens(rng, T, H, D)
    slots = rng.permutation(nb * 16)[:T].astype(np.int64)
    ks = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(k))
    vs = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(v))
    okc, ovc, gk, gv, err, cache = write_both(fmt, k, v, slots, nb, ks, vs)
    assert np.array_equal(gk, okc)
    want_k, want_v = oracle.dequantize(fmt, okc, ovc, H, D, slots, ks, vs)
    ko = torch.empty(T, H, D, device=DEV)
    vo = torch.empty(T, H, D, device=DEV)
    e = new_err()
    kvq.kv_dequantize(fmt, cache, torch.from_numpy(slots).to(DEV), dev_scalar(ks),
                      dev_scalar(vs), ko, vo, e)
    torch.cuda.synchronize()
    assert int(e.item()) == 0
    assert np.array_equal(ko.cpu().numpy().view(np.uint32), want_k.view(np.uint32))
    assert np.array_equal(vo.cpu().numpy().view(np.uint32), want_v.view(np.uint32))


@pytest.mark.parametrize("n,offset", [(1, 0), (7, 1), (8, 0), (1000, 3), (65536 * 8 * 128 // 64, 0),
                                      (123457, 5)])
def test_calibrate_absmax(n, offset):
    rng = wl.rng_for(n, offset)
    x = wl.make_tokens(rng, 1, 1, n + offset).reshape(-1)
    x[offset + n // 2] = wl.f32_to_bf16_bits(np.array([-77.5], np.float32))[0]
    if offset:
        x[:offset] = wl.f32_to_bf16_bits(np.array([1e6] * offset, np.float32))  # outside the range
    want = oracle.absmax_bf16(x[offset:offset + n])
    d = to_dev_bits(x)
    amax = torch.zeros(1, dtype=torch.float32, device=DEV)
    kvq.kv_calibrate_absmax(d[offset:offset + n], amax)
    torch.cuda.synchronize()
    assert amax.item() == want
    # max-accumulation: a second, smaller tensor leaves the maximum
    kvq.kv_calibrate_absmax(d[offset:offset + 1], amax)
    torch.cuda.synchronize()
    assert amax.item() == want


def test_device_scale_matches_host_and_oracle():
    rng = np.random.default_rng(3)
    amax = np.concatenate([[0.0, 1e-15, 1.0, 448.0], rng.lognormal(0, 3, 60)]).astype(np.float32)
    for fmt in ("fp8", "nvfp4", "bf16"):
        d_amax = torch.from_numpy(amax).to(DEV)
        out = torch.empty_like(d_amax)
        for i in range(amax.size):
            kvq.kv_scale_from_absmax_device(fmt, d_amax[i:i + 1], out[i:i + 1])
        torch.cuda.synchronize()
        got = out.cpu().numpy()
        want = np.array([oracle.scale_from_absmax(fmt, a) for a in amax], np.float32)
        assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), fmt
