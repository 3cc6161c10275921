"""GPU parity of the 3-bit planar-rotation codec (PQ3: "AMD MI300X - KV Cache
Compression Benchmark", "Key Results": 52-byte blocks per 128-element
vector, 4.923x against FP16) against the oracle: the written pages (norms
and packed indices) and the dequantised values bit-exact; the fused decode
(scores and outputs computed in the rotated domain, rotated back once per
output) within the attention tolerances of the float64 oracle over the
dequantised cache, over ragged lengths, forced and automatic splits, GQA
ratios, sliding windows, NaN bytes in unwritten slots, a negative sm_scale
and empty sequences; plus the error paths."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl

from gpu_common import DEV, assert_attention_close, new_err, to_dev_bits

pytestmark = pytest.mark.gpu

D = 128


class PQ3Case:
    def __init__(self, B, Hkv, Hq, lens, seed, factor=8.0, permuted=True, extra_blocks=3,
                 fill=0, zero_rows=False):
        rng = wl.rng_for(seed, 0)
        self.B, self.Hkv, self.Hq = B, Hkv, Hq
        self.lens = np.array(lens, np.int32)
        self.max_blocks = max(1, -(-int(self.lens.max(initial=0)) // 16))
        self.num_blocks = B * self.max_blocks + extra_blocks
        self.bt = (wl.permuted_block_table(wl.rng_for(seed, 1), B, self.max_blocks, self.num_blocks)
                   if permuted else wl.identity_block_table(B, self.max_blocks))
        outl = wl.outlier_pairs(rng, Hkv, D, per_head=1)
        self.k = [wl.make_tokens(rng, int(n), Hkv, D, outl, factor) for n in self.lens]
        self.v = [wl.make_tokens(rng, int(n), Hkv, D, outl, factor) for n in self.lens]
        if zero_rows:  # an all-zero vector in every sequence
            for x in self.k + self.v:
                if len(x):
                    x[len(x) // 2] = 0
        self.q = wl.make_query(rng, B, Hq, D)
        self.kp = oracle.pq3_params(wl.planar_rotation(wl.rng_for(seed, 2)))
        self.vp = oracle.pq3_params(wl.planar_rotation(wl.rng_for(seed, 3)))
        self.okc, self.ovc = oracle.new_cache("pq3", self.num_blocks, Hkv, D, fill=fill)
        for b in range(B):
            slots = wl.physical_slots(self.bt, b, np.arange(self.lens[b]))
            oracle.pq3_write(self.k[b], self.v[b], slots, self.okc, self.ovc, self.kp, self.vp)
        self.cache = kvq.KVCache("pq3", self.num_blocks, Hkv, D)
        if fill:
            self.cache.k.fill_(fill)
            self.cache.v.fill_(fill)
        self.d_kp = kvq.pq3_params(self.kp[8:], DEV)
        self.d_vp = kvq.pq3_params(self.vp[8:], DEV)
        self.err = new_err()
        for b in range(B):
            if self.lens[b] == 0:
                continue
            slots = torch.from_numpy(wl.physical_slots(self.bt, b, np.arange(self.lens[b]))).to(DEV)
            kvq.kv_quantize_write("pq3", to_dev_bits(self.k[b]), to_dev_bits(self.v[b]), slots,
                                  self.cache, self.d_kp, self.d_vp, self.err)
        self.d_q = to_dev_bits(self.q)
        self.d_bt = torch.from_numpy(self.bt).to(DEV)
        self.d_lens = torch.from_numpy(self.lens).to(DEV)

    def decode(self, num_splits=0, sm_scale=0.0, window=0):
        msl = self.max_blocks * 16
        ws = kvq.new_workspace(kvq.kv_decode_workspace_size_window(
            "pq3", self.B, self.Hq, self.Hkv, D, msl, window, num_splits))
        out = torch.full((self.B, self.Hq, D), float("nan"), device=DEV)
        lse = torch.full((self.B, self.Hq), float("nan"), device=DEV)
        kvq.kv_decode_attention_window("pq3", self.d_q, self.cache, self.d_bt, self.d_lens, msl,
                                       window, self.d_kp, self.d_vp, out, lse, ws, self.err,
                                       sm_scale, num_splits)
        torch.cuda.synchronize()
        return out.cpu().numpy(), lse.cpu().numpy()

    def reference(self, sm_scale=None, window=0):
        return oracle.pq3_decode_attention(self.q, self.okc, self.ovc, self.Hkv, self.bt,
                                           self.lens, self.kp, self.vp, sm_scale, window=window)


def test_written_pages_are_bit_exact():
    c = PQ3Case(3, 2, 8, [1, 37, 500], seed=9500, factor=16.0, zero_rows=True)
    torch.cuda.synchronize()
    assert int(c.err.item()) == 0
    assert np.array_equal(c.cache.k.cpu().numpy(), c.okc)
    assert np.array_equal(c.cache.v.cpu().numpy(), c.ovc)


def test_dequantize_is_bit_exact():
    c = PQ3Case(2, 3, 6, [40, 200], seed=9510, factor=16.0, zero_rows=True)
    slots = np.concatenate([wl.physical_slots(c.bt, b, np.arange(n)) for b, n in
                            enumerate(c.lens)])
    ko = torch.empty(len(slots), c.Hkv, D, device=DEV)
    vo = torch.empty(len(slots), c.Hkv, D, device=DEV)
    kvq.kv_dequantize("pq3", c.cache, torch.from_numpy(slots).to(DEV), c.d_kp, c.d_vp, ko, vo,
                      c.err)
    torch.cuda.synchronize()
    kf, vf = oracle.pq3_to_f32(c.okc, c.ovc, c.Hkv, c.kp, c.vp)
    kf = kf.view(np.float32).reshape(c.num_blocks, c.Hkv, 16, D)
    vf = vf.view(np.float32).reshape(c.num_blocks, c.Hkv, 16, D)
    want_k = kf[slots // 16, :, slots % 16]
    want_v = vf[slots // 16, :, slots % 16]
    assert np.array_equal(ko.cpu().numpy(), want_k)
    assert np.array_equal(vo.cpu().numpy(), want_v)


@pytest.mark.parametrize("splits", [0, 1, 5])
def test_decode_ragged_batch(splits):
    c = PQ3Case(5, 2, 16, [1, 15, 16, 17, 1001], seed=9520, factor=16.0)
    out, lse = c.decode(splits)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_decode_gqa_ratios(G):
    c = PQ3Case(2, 2, 2 * G, [333, 64], seed=9530 + G)
    out, lse = c.decode()
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("max_len", [16, 100, 700])
def test_decode_many_units_per_cta(max_len):
    """80 short (sequence, KV head) units: CTAs take up to 27 units each in
    turn, some spanning two CTAs, some empty."""
    rng = wl.rng_for(9560 + max_len, 3)
    lens = rng.integers(0, max_len + 1, size=40).tolist()
    c = PQ3Case(40, 2, 16, lens, seed=9570 + max_len, factor=16.0)
    out, lse = c.decode()
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference())


def test_decode_long_context_and_splits():
    c = PQ3Case(1, 1, 8, [20000], seed=9540, factor=16.0)
    ref = c.reference()
    for splits in (0, 3, 97):
        out, lse = c.decode(splits)
        assert_attention_close(out, lse, *ref)


@pytest.mark.parametrize("W", [1, 37, 500])
def test_decode_window(W):
    c = PQ3Case(4, 2, 16, [1, 15, 17, 1001], seed=9550, factor=16.0)
    out, lse = c.decode(window=W)
    assert_attention_close(out, lse, *c.reference(window=W))


def test_decode_nan_bytes_negative_scale_and_empty():
    c = PQ3Case(3, 2, 8, [37, 0, 250], seed=9560, fill=0xFF)
    out, lse = c.decode(2, sm_scale=-0.08)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference(sm_scale=-0.08))
    assert np.all(np.isneginf(lse[1])) and np.all(out[1] == 0)


def test_bad_codebook_and_unsupported_calls():
    c = PQ3Case(1, 1, 8, [100], seed=9570)
    bad = c.d_kp.clone()
    bad[3], bad[4] = bad[4].item(), bad[3].item()  # not ascending
    err = new_err()
    ws = kvq.new_workspace(kvq.kv_decode_workspace_size("pq3", 1, 8, 1, D, 112))
    out = torch.empty(1, 8, D, device=DEV)
    kvq.kv_decode_attention("pq3", c.d_q, c.cache, c.d_bt, c.d_lens, 112, bad, c.d_vp, out, None,
                            ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == kvq.DERR_SCALE
    err.zero_()
    kvq.kv_quantize_write("pq3", to_dev_bits(c.k[0]), to_dev_bits(c.v[0]),
                          torch.arange(100, device=DEV), c.cache, bad, c.d_vp, err)
    torch.cuda.synchronize()
    assert int(err.item()) == kvq.DERR_SCALE
    with pytest.raises(kvq.KvqError, match="head_dim 128"):
        kvq.KVCache("pq3", 4, 1, 64)
    with pytest.raises(kvq.KvqError, match="PQ3"):
        kvq.kv_prefill_attention("pq3", to_dev_bits(np.zeros((1, 1, 8, D), np.uint16)), c.cache,
                                 c.d_bt, c.d_lens, c.d_kp, c.d_vp,
                                 torch.empty(1, 1, 8, D, device=DEV), None)
