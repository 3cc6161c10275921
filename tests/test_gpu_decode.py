"""GPU parity of the fused-dequant decode attention against the float64 oracle
(out within 2e-3 max-abs, lse within 1e-5 relative), over formats, head dims,
GQA ratios, ragged lengths, forced and automatic context splits, and the
method's degenerate cases; plus the device-side error reporting."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl

from gpu_common import DEV, Case, assert_attention_close, dev_scalar, new_err, to_dev_bits

pytestmark = pytest.mark.gpu

FMTS = ["bf16", "fp8", "nvfp4"]


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 5])
def test_ragged_batch(fmt, D, splits):
    c = Case(fmt, 5, 2, 16, D, [1, 15, 16, 17, 1001], seed=1000 + D, factor=16.0)
    out, lse = c.decode(num_splits=splits)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_gqa_ratios(fmt, G):
    Hkv = 2
    c = Case(fmt, 2, Hkv, Hkv * G, 128, [333, 64], seed=2000 + G)
    out, lse = c.decode()
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("fmt", FMTS)
def test_long_context_many_splits(fmt):
    c = Case(fmt, 1, 1, 8, 64, [20000], seed=3001, factor=16.0)
    for splits in (0, 3, 97):
        out, lse = c.decode(num_splits=splits)
        assert_attention_close(out, lse, *c.reference())


def test_tiny_fp8_workload():
    """1 sequence x 1024 tokens, 2 KV heads, GQA 4, D 64, two outlier channels
    per head x20, blocks in order."""
    w = wl.WORKLOADS["tiny-fp8-1k"]
    c = Case("fp8", w.B, w.Hkv, w.Hq, w.D, [w.seq_len], seed=w.seed, permuted=False,
             factor=w.outlier_factor, outliers_per_head=2)
    out, lse = c.decode()
    e_out, e_lse = assert_attention_close(out, lse, *c.reference())
    assert e_out < 5e-4


@pytest.mark.parametrize("fmt", FMTS)
def test_empty_and_single_token(fmt):
    c = Case(fmt, 3, 2, 8, 64, [0, 1, 0], seed=4000)
    out, lse = c.decode()
    ref_out, ref_lse = c.reference()
    assert_attention_close(out, lse, ref_out, ref_lse)
    assert np.all(np.isneginf(lse[0])) and np.all(out[0] == 0)
    assert np.all(np.isneginf(lse[2])) and np.all(out[2] == 0)


@pytest.mark.parametrize("fmt", FMTS)
def test_all_sequences_empty(fmt):
    c = Case(fmt, 2, 1, 8, 128, [0, 0], seed=4100)
    out, lse = c.decode(max_seq_len=0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4", "bf16"])
def test_nan_bytes_in_unwritten_slots(fmt):
    """Pages filled with 0xFF (NaN for E4M3 and BF16) before the write: the
    masked tail of a partial last page must not leak into the result."""
    c = Case(fmt, 2, 2, 8, 128, [37, 250], seed=4200, fill=0xFF)
    out, lse = c.decode(num_splits=2)
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_query_is_uniform(fmt):
    c = Case(fmt, 1, 1, 8, 64, [300], seed=4300)
    c.q[:] = 0
    c.d_q.zero_()
    out, lse = c.decode(num_splits=3)
    ref_out, ref_lse = c.reference()
    assert_attention_close(out, lse, ref_out, ref_lse)
    np.testing.assert_allclose(lse, np.log(300), rtol=1e-6)


def test_identical_heads_and_determinism():
    c = Case("fp8", 2, 2, 16, 128, [777, 500], seed=4400)
    c.q[:, 1] = c.q[:, 0]
    c.d_q[:, 1] = c.d_q[:, 0]
    a_out, a_lse = c.decode()
    b_out, b_lse = c.decode()
    assert np.array_equal(a_out, b_out) and np.array_equal(a_lse, b_lse)
    assert np.array_equal(a_out[:, 0], a_out[:, 1])


def test_page_placement_is_invisible():
    """Same tokens at different physical blocks: bit-identical output."""
    a = Case("nvfp4", 2, 2, 16, 64, [300, 129], seed=4500, permuted=False)
    b = Case("nvfp4", 2, 2, 16, 64, [300, 129], seed=4500, permuted=True)
    oa, la = a.decode(num_splits=2)
    ob, lb = b.decode(num_splits=2)
    assert np.array_equal(oa, ob) and np.array_equal(la, lb)


def test_custom_sm_scale():
    c = Case("fp8", 1, 2, 8, 64, [200], seed=4600)
    out, lse = c.decode(sm_scale=0.05)
    assert_attention_close(out, lse, *c.reference(sm_scale=0.05))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 3])
def test_negative_sm_scale(fmt, D, splits):
    """A negative softmax scale is a finite sm_scale the interface accepts:
    the scores change sign, and the masked tail of every partial last page
    (lengths 1, 15, 17, 1001) must still carry no weight."""
    c = Case(fmt, 4, 2, 16, D, [1, 15, 17, 1001], seed=4650 + D, factor=16.0)
    out, lse = c.decode(num_splits=splits, sm_scale=-0.08)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference(sm_scale=-0.08))


def mean_of_v_hat(c: Case):
    """[B][Hq][D]: the mean over each sequence's tokens of the oracle's
    dequantised V at the query head's KV head (the exact result when every
    score is equal)."""
    G = c.Hq // c.Hkv
    out = np.zeros((c.B, c.Hq, c.D))
    for b in range(c.B):
        n = int(c.lens[b])
        if n == 0:
            continue
        slots = wl.physical_slots(c.bt, b, np.arange(n))
        _, v_hat = oracle.dequantize(c.fmt, c.okc, c.ovc, c.Hkv, c.D, slots, c.ks, c.vs)
        mean = v_hat.astype(np.float64).mean(axis=0)  # [Hkv][D]
        out[b] = np.repeat(mean, G, axis=0)
    return out


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 3])
def test_all_zero_k(fmt, D, splits):
    """An all-zero K tensor: its abs-max is 0, so the NVFP4 global scale g is
    0 (the FP8 scale is the 1e-12 floor) and every score is exactly 0.  The
    result is the plain mean of the dequantised V and lse = ln T, also on
    lengths that end inside a page."""
    lens = [1, 15, 17, 1001]
    c = Case(fmt, 4, 2, 16, D, lens, seed=4660 + D, factor=16.0, zero_k=True)
    if fmt == "nvfp4":
        assert c.ks == 0.0
    out, lse = c.decode(num_splits=splits)
    assert int(c.err.item()) == 0
    ref_out, ref_lse = c.reference()
    assert_attention_close(out, lse, ref_out, ref_lse)
    np.testing.assert_allclose(ref_lse, np.log(np.array(lens, np.float64))[:, None]
                               * np.ones((1, c.Hq)), rtol=1e-12)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-6, atol=1e-5)
    assert np.abs(out - mean_of_v_hat(c)).max() <= 2e-3


def test_bad_block_id_and_seq_len_are_reported():
    c = Case("fp8", 2, 1, 8, 64, [40, 40], seed=4700)
    bad = c.d_bt.clone()
    bad[0, 1] = c.num_blocks + 5
    ws = kvq.new_workspace(kvq.kv_decode_workspace_size("fp8", 2, 8, 1, 64, 48, 0))
    out = torch.empty(2, 8, 64, device=DEV)
    lse = torch.empty(2, 8, device=DEV)
    err = new_err()
    kvq.kv_decode_attention("fp8", c.d_q, c.cache, bad, c.d_lens, 48, c.d_ks, c.d_vs, out, lse,
                            ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == kvq.DERR_BLOCK_ID
    # sequence 1 is untouched by the bad entry of sequence 0
    ref_out, ref_lse = c.reference()
    assert np.abs(out[1].cpu().numpy() - ref_out[1]).max() < 2e-3
    # a length beyond max_seq_len
    err.zero_()
    lens = c.d_lens.clone()
    lens[1] = 47
    kvq.kv_decode_attention("fp8", c.d_q, c.cache, c.d_bt, lens, 40, c.d_ks, c.d_vs, out, lse,
                            ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == kvq.DERR_SEQ_LEN
    # a bad scale on the device
    err.zero_()
    kvq.kv_decode_attention("fp8", c.d_q, c.cache, c.d_bt, c.d_lens, 48, dev_scalar(0.0), c.d_vs,
                            out, lse, ws, err)
    torch.cuda.synchronize()
    assert int(err.item()) == kvq.DERR_SCALE


def test_host_side_errors():
    # long enough that the automatic split spreads the one unit over CTAs
    c = Case("fp8", 1, 1, 8, 64, [4000], seed=4800)
    need = kvq.kv_decode_workspace_size("fp8", 1, 8, 1, 64, 4000, 0)
    assert need > 0
    out = torch.empty(1, 8, 64, device=DEV)
    with pytest.raises(kvq.KvqError, match="workspace"):
        kvq.kv_decode_attention("fp8", c.d_q, c.cache, c.d_bt, c.d_lens, 4000, c.d_ks, c.d_vs,
                                out, None, kvq.new_workspace(need - 256 if need > 512 else 0))
    with pytest.raises(kvq.KvqError, match="max_seq_len"):
        kvq.kv_decode_attention("fp8", c.d_q, c.cache, c.d_bt, c.d_lens, 4001, c.d_ks, c.d_vs,
                                out, None, None)
    with pytest.raises(kvq.KvqError):  # GQA ratio must divide
        kvq.kv_decode_workspace_size("fp8", 1, 7, 2, 64, 100, 0)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
def test_variable_lengths_like_the_sweep(fmt, D):
    """Sweep-style batch: lengths uniform in [L/2, L], GQA 8, automatic split."""
    rng = wl.rng_for(5000 + D, 2)
    lens = wl.varlen(rng, 8, 2048).tolist()
    c = Case(fmt, 8, 2, 16, D, lens, seed=5100 + D, factor=16.0)
    out, lse = c.decode()
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("max_len", [16, 100, 700])
def test_many_units_per_cta(fmt, D, max_len):
    """Many short sequences (80 (sequence, KV head) units, lengths uniform in
    [0, max_len]): the automatic split gives each CTA up to 27 units, taken
    in turn, with some units spanning two CTAs and some empty, so the
    per-unit merges inside a CTA meet the cross-CTA ones."""
    rng = wl.rng_for(5200 + D + max_len, 3)
    lens = rng.integers(0, max_len + 1, size=40).tolist()
    c = Case(fmt, 40, 2, 16, D, lens, seed=5300 + D + max_len, factor=16.0)
    out, lse = c.decode()
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference())


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
def test_decode_launched_right_after_a_write(fmt, D):
    """The decode may begin while a kv_quantize_write just before it on the
    stream is finishing: the last 1,200 tokens of every sequence are written
    and the decode launched next, with no other work between, and the result
    must include them."""
    lens = [3000, 2600, 1500]
    c = Case(fmt, 3, 2, 16, D, lens, seed=5300 + D, factor=16.0)
    tail = 1200
    # rewrite the tails with fresh codes from zeroed pages: clear them first
    kb = [torch.from_numpy(wl.physical_slots(c.bt, b, np.arange(n - tail, n))).to(DEV)
          for b, n in enumerate(lens)]
    page = kvq.kv_cache_bytes(fmt, 1, c.Hkv, D)
    for b, n in enumerate(lens):
        for blk in set(int(x) for x in c.bt[b][(n - tail) // 16:]):
            c.cache.k[blk * page:(blk + 1) * page].zero_()
            c.cache.v[blk * page:(blk + 1) * page].zero_()
    # the head of the last page before the tail is zeroed too: write it back
    msl = c.max_blocks * 16
    ws = kvq.new_workspace(kvq.kv_decode_workspace_size(fmt, c.B, c.Hq, c.Hkv, D, msl))
    out = torch.empty((c.B, c.Hq, D), device=DEV)
    lse = torch.empty((c.B, c.Hq), device=DEV)
    heads = [torch.from_numpy(wl.physical_slots(c.bt, b, np.arange((n - tail) // 16 * 16,
                                                                  n - tail))).to(DEV)
             for b, n in enumerate(lens)]
    k_tail = torch.cat([to_dev_bits(c.k[b][n - tail:]) for b, n in enumerate(lens)])
    v_tail = torch.cat([to_dev_bits(c.v[b][n - tail:]) for b, n in enumerate(lens)])
    k_head = torch.cat([to_dev_bits(c.k[b][(n - tail) // 16 * 16:n - tail])
                        for b, n in enumerate(lens)])
    v_head = torch.cat([to_dev_bits(c.v[b][(n - tail) // 16 * 16:n - tail])
                        for b, n in enumerate(lens)])
    kvq.kv_quantize_write(fmt, k_head, v_head, torch.cat(heads), c.cache, c.d_ks, c.d_vs, c.err)
    slots = torch.cat(kb)
    torch.cuda.synchronize()
    # write, then decode: adjacent launches on one stream
    kvq.kv_quantize_write(fmt, k_tail, v_tail, slots, c.cache, c.d_ks, c.d_vs, c.err)
    kvq.kv_decode_attention(fmt, c.d_q, c.cache, c.d_bt, c.d_lens, msl, c.d_ks, c.d_vs, out, lse,
                            ws, c.err)
    torch.cuda.synchronize()
    assert int(c.err.item()) == 0
    assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), *c.reference())


def test_bounded_wait_times_out_and_reports():
    """The bounded mbarrier wait behind every kernel's waits: a completed phase
    passes with no error; a phase nothing completes gives up after about two
    seconds with DERR_TIMEOUT in the error word, and the context stays usable
    (a decode right after it matches the oracle)."""
    import time

    err = new_err()
    kvq.kvq_selftest_bounded_wait(err, True)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    t0 = time.monotonic()
    kvq.kvq_selftest_bounded_wait(err, False)
    torch.cuda.synchronize()
    dt = time.monotonic() - t0
    assert int(err.item()) == kvq.DERR_TIMEOUT
    assert 1.0 < dt < 20.0, f"wait gave up after {dt:.2f} s"
    c = Case("fp8", 2, 2, 16, 128, [300, 77], seed=7700)
    out, lse = c.decode()
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *c.reference())


def test_decode_from_two_host_threads_on_one_stream():
    """Two host threads launch decodes of different formats and head dims on
    one shared stream at the same time (the library's per-device launch state
    is shared between them); every result matches the oracle."""
    import threading

    cases = [Case("fp8", 2, 2, 16, 128, [3000, 1200], seed=7800, factor=16.0),
             Case("nvfp4", 3, 2, 16, 64, [900, 17, 2500], seed=7801, factor=16.0)]
    stream = torch.cuda.Stream()
    outs = []
    for c in cases:
        msl = c.max_blocks * 16
        ws = kvq.new_workspace(kvq.kv_decode_workspace_size(c.fmt, c.B, c.Hq, c.Hkv, c.D, msl))
        outs.append((torch.full((c.B, c.Hq, c.D), float("nan"), device=DEV),
                     torch.full((c.B, c.Hq), float("nan"), device=DEV), ws, msl))
    torch.cuda.synchronize()
    start = threading.Barrier(2)
    errors = []

    def run(i):
        try:
            c = cases[i]
            out, lse, ws, msl = outs[i]
            start.wait()
            for _ in range(3):
                kvq.kv_decode_attention(c.fmt, c.d_q, c.cache, c.d_bt, c.d_lens, msl, c.d_ks,
                                        c.d_vs, out, lse, ws, c.err, stream=stream)
        except Exception as e:  # surfaced by the main thread
            errors.append(e)

    threads = [threading.Thread(target=run, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    for c, (out, lse, _, _) in zip(cases, outs):
        assert int(c.err.item()) == 0
        assert_attention_close(out.cpu().numpy(), lse.cpu().numpy(), *c.reference())
