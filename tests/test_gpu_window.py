"""Sliding-window decode (kv_decode_attention_window) against the oracle's
windowed float64 attention: each sequence attends to its last W tokens only
("AMD MI300X — KV Cache Compression Benchmark", section "SWA mode").  Windows
shorter than, equal to and longer than the sequences, not multiples of the
16-token page, W = 1, forced and automatic splits, and a window over a long
cache whose pages before the window hold NaN bytes (they must not be read)."""
import numpy as np
import pytest
import torch

import quantized_kv_cache_21_b200 as kvq
import oracle

from gpu_common import DEV, Case, assert_attention_close

pytestmark = pytest.mark.gpu

FMTS = ["bf16", "fp8", "nvfp4"]


def decode_window(c: Case, W: int, num_splits: int = 0, sm_scale: float = 0.0):
    msl = c.max_blocks * 16
    ws = kvq.new_workspace(kvq.kv_decode_workspace_size_window(c.fmt, c.B, c.Hq, c.Hkv, c.D, msl,
                                                               W, num_splits))
    out = torch.full((c.B, c.Hq, c.D), float("nan"), device=DEV)
    lse = torch.full((c.B, c.Hq), float("nan"), device=DEV)
    kvq.kv_decode_attention_window(c.fmt, c.d_q, c.cache, c.d_bt, c.d_lens, msl, W, c.d_ks,
                                   c.d_vs, out, lse, ws, c.err, sm_scale, num_splits)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def reference_window(c: Case, W: int, sm_scale=None):
    return oracle.decode_attention(c.fmt, c.q, c.okc, c.ovc, c.Hkv, c.bt, c.lens, c.ks, c.vs,
                                   sm_scale=sm_scale, window=W)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("W", [1, 16, 37, 500, 4096])
def test_window_ragged_batch(fmt, D, W):
    c = Case(fmt, 5, 2, 16, D, [1, 15, 17, 1001, 3000], seed=6000 + D, factor=16.0)
    out, lse = decode_window(c, W)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *reference_window(c, W))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("splits", [1, 3])
def test_window_forced_splits(fmt, splits):
    c = Case(fmt, 2, 2, 8, 64, [777, 2000], seed=6100, factor=8.0)
    out, lse = decode_window(c, 333, splits)
    assert_attention_close(out, lse, *reference_window(c, 333))


@pytest.mark.parametrize("fmt", FMTS)
def test_window_reads_only_the_window(fmt):
    """A 20,000-token cache with a 1,000-token window: the pages wholly before
    the window are overwritten with 0xFF (NaN codes) after the write; the
    result must still match the oracle (computed before the overwrite)."""
    W = 1000
    c = Case(fmt, 1, 2, 16, 128, [20000], seed=6200, factor=16.0)
    ref = reference_window(c, W)
    first_page = (20000 - W) // 16
    page = kvq.kv_cache_bytes(fmt, 1, c.Hkv, c.D)
    for blk in c.bt[0][:first_page]:
        c.cache.k[int(blk) * page:(int(blk) + 1) * page].fill_(0xFF)
        c.cache.v[int(blk) * page:(int(blk) + 1) * page].fill_(0xFF)
    out, lse = decode_window(c, W)
    assert_attention_close(out, lse, *ref)


def test_window_zero_is_the_full_decode():
    c = Case("fp8", 2, 2, 8, 128, [400, 90], seed=6300)
    a = decode_window(c, 0)
    b = c.decode()
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


def test_negative_window_is_rejected():
    with pytest.raises(kvq.KvqError, match="window"):
        kvq.kv_decode_workspace_size_window("fp8", 1, 8, 1, 64, 100, -1)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 2])
def test_window_negative_scale_and_zero_k(fmt, D, splits):
    """W = 37 starts inside a page, so the window's first page has masked
    tokens before it: with a negative sm_scale, and with an all-zero K (NVFP4
    g = 0, every score 0: out = mean of the window's V, lse = ln min(W, T))."""
    lens = [1, 15, 17, 1001]
    c = Case(fmt, 4, 2, 16, D, lens, seed=6500 + D, factor=16.0)
    out, lse = decode_window(c, 37, splits, sm_scale=-0.08)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *reference_window(c, 37, sm_scale=-0.08))
    z = Case(fmt, 4, 2, 16, D, lens, seed=6510 + D, factor=16.0, zero_k=True)
    out, lse = decode_window(z, 37, splits)
    assert int(z.err.item()) == 0
    ref_out, ref_lse = reference_window(z, 37)
    assert_attention_close(out, lse, ref_out, ref_lse)
    n = np.minimum(np.array(lens, np.float64), 37)
    np.testing.assert_allclose(lse, np.log(n)[:, None] * np.ones((1, z.Hq)), rtol=1e-6, atol=1e-5)
