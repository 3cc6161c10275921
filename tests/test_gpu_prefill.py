"""Chunked-prefill attention (kv_prefill_attention) against the oracle's
float64 prefill: the chunk's Tq newest tokens of each sequence attend causally
to the cache up to their own position ("Dual R9700 model and spec-decode
campaign", fixed knobs: long-prefill-token-threshold 2048 with prefix caching).

Covered: the three formats at head_dim 64 and 128; GQA groups of 1, 3, 8 and
16 query heads (3: padding rows in every CTA; 16: 8 query tokens per CTA);
ragged chunks (several 64-key blocks, a partial last page, a partial last query
block) and a sequence shorter than the chunk (its first queries attend to
nothing); a chunk of one token against the decode; bad block ids and lengths
reported through the error word; host-side argument errors; and, at the
benchmark's full size (4 x 126,976 tokens, 2,048-token chunks, FP8, head_dim
128), sampled rows recomputed by the oracle from its own pages."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl
from quantized_kv_cache_21_b200.scenario import DecodeScenario

from gpu_common import DEV, Case, assert_attention_close, new_err, to_dev_bits

pytestmark = pytest.mark.gpu

FMTS = ["bf16", "fp8", "nvfp4"]


def chunk_q(c: Case, Tq: int, seed: int) -> np.ndarray:
    return wl.make_query(wl.rng_for(seed, 9), c.B * Tq, c.Hq, c.D).reshape(c.B, Tq, c.Hq, c.D)


def run(c: Case, q: np.ndarray, err=None, lens=None, sm_scale=0.0):
    B, Tq, Hq, D = q.shape
    out = torch.full((B, Tq, Hq, D), float("nan"), device=DEV)
    lse = torch.full((B, Tq, Hq), float("nan"), device=DEV)
    kvq.kv_prefill_attention(c.fmt, to_dev_bits(q), c.cache, c.d_bt,
                             c.d_lens if lens is None else lens, c.d_ks, c.d_vs, out, lse,
                             c.err if err is None else err, sm_scale)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def reference(c: Case, q: np.ndarray, sm_scale=None):
    return oracle.prefill_attention(c.fmt, q, c.okc, c.ovc, c.Hkv, c.bt, c.lens, c.ks, c.vs,
                                    sm_scale)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 3, 8, 16])
def test_prefill_matches_oracle(fmt, D, G):
    Tq = 40
    c = Case(fmt, 3, 2, 2 * G, D, [29, 301, 700], seed=7000 + D + G, factor=16.0)
    q = chunk_q(c, Tq, 7001 + G)
    out, lse = run(c, q)
    assert int(c.err.item()) == 0
    assert_attention_close(out, lse, *reference(c, q))


@pytest.mark.parametrize("fmt", FMTS)
def test_prefill_long_context(fmt):
    """4,100 and 5,000 cached tokens, 128-token chunks: ~80 key blocks per CTA."""
    Tq = 128
    c = Case(fmt, 2, 2, 16, 128, [4100, 5000], seed=7100, factor=16.0)
    q = chunk_q(c, Tq, 7101)
    out, lse = run(c, q)
    assert int(c.err.item()) == 0
    rows = np.array([[b, i, j] for b in range(2) for i in (0, 1, 63, 64, 127)
                     for j in (0, 5, 15)], np.int32)
    ref_out, ref_lse = oracle.prefill_attention(fmt, q, c.okc, c.ovc, c.Hkv, c.bt, c.lens, c.ks,
                                                c.vs, rows=rows)
    sel = (rows[:, 0], rows[:, 1], rows[:, 2])
    assert_attention_close(out[sel], lse[sel], ref_out[sel], ref_lse[sel])


def test_chunk_of_one_token_is_the_decode():
    c = Case("fp8", 3, 2, 16, 128, [1, 90, 1000], seed=7200, factor=8.0)
    q = chunk_q(c, 1, 7201)
    out, lse = run(c, q)
    c.q = q[:, 0].copy()
    c.d_q = to_dev_bits(c.q)
    d_out, d_lse = c.decode()
    ref_out, ref_lse = c.reference()
    assert_attention_close(out[:, 0], lse[:, 0], ref_out, ref_lse)
    assert_attention_close(d_out, d_lse, ref_out, ref_lse)


def test_sm_scale_and_no_lse():
    c = Case("nvfp4", 2, 1, 8, 64, [70, 33], seed=7300)
    q = chunk_q(c, 17, 7301)
    for sm in (-0.2, 0.3):  # a negative scale flips which key dominates
        out, lse = run(c, q, sm_scale=sm)
        assert_attention_close(out, lse, *reference(c, q, sm_scale=sm))
    out2 = torch.full(q.shape, float("nan"), device=DEV)
    kvq.kv_prefill_attention("nvfp4", to_dev_bits(q), c.cache, c.d_bt, c.d_lens, c.d_ks, c.d_vs,
                             out2, None, c.err, 0.3)
    torch.cuda.synchronize()
    assert np.array_equal(out2.cpu().numpy(), out)


def test_bad_block_id_and_length_are_reported():
    c = Case("fp8", 2, 2, 16, 64, [200, 150], seed=7400)
    q = chunk_q(c, 20, 7401)
    bt = c.bt.copy()
    bt[0, 3] = c.num_blocks + 7  # a page of sequence 0 points outside the pool
    err = new_err()
    out = torch.full(q.shape, float("nan"), device=DEV)
    lse = torch.full(q.shape[:3], float("nan"), device=DEV)
    kvq.kv_prefill_attention("fp8", to_dev_bits(q), c.cache, torch.from_numpy(bt).to(DEV),
                             c.d_lens, c.d_ks, c.d_vs, out, lse, err)
    torch.cuda.synchronize()
    assert int(err.item()) & kvq.DERR_BLOCK_ID
    assert np.all(np.isfinite(out.cpu().numpy()))
    # sequence 1 is untouched by the bad page
    ref_out, ref_lse = reference(c, q)
    assert_attention_close(out.cpu().numpy()[1], lse.cpu().numpy()[1], ref_out[1], ref_lse[1])
    # a length past max_blocks * 16: reported, that sequence's rows are empty
    err2 = new_err()
    lens = torch.tensor([200, c.max_blocks * 16 + 1], dtype=torch.int32, device=DEV)
    o2, l2 = run(c, q, err=err2, lens=lens)
    assert int(err2.item()) & kvq.DERR_SEQ_LEN
    assert np.all(o2[1] == 0) and np.all(np.isneginf(l2[1]))
    assert_attention_close(o2[0], l2[0], ref_out[0], ref_lse[0])


def test_host_argument_errors():
    c = Case("fp8", 1, 1, 8, 64, [40], seed=7500)
    q = to_dev_bits(chunk_q(c, 4, 7501))
    out = torch.empty((1, 4, 8, 64), device=DEV)
    with pytest.raises(kvq.KvqError, match="multiple"):
        c2 = Case("fp8", 1, 3, 3, 64, [40], seed=7502)
        q2 = to_dev_bits(wl.make_query(wl.rng_for(1, 1), 4, 4, 64).reshape(1, 4, 4, 64))
        kvq.kv_prefill_attention("fp8", q2, c2.cache, c2.d_bt, c2.d_lens, c2.d_ks, c2.d_vs,
                                 torch.empty((1, 4, 4, 64), device=DEV), None)
    with pytest.raises(kvq.KvqError, match="query heads per KV head"):
        q3 = torch.zeros((1, 1, 256, 64), dtype=torch.bfloat16, device=DEV)
        kvq.kv_prefill_attention("fp8", q3, c.cache, c.d_bt, c.d_lens, c.d_ks, c.d_vs,
                                 torch.empty((1, 1, 256, 64), device=DEV), None)
    with pytest.raises(kvq.KvqError, match="scale"):
        kvq.kv_prefill_attention("fp8", q, c.cache, c.d_bt, c.d_lens, None, None, out, None)
    # an empty chunk launches nothing
    kvq.kv_prefill_attention("fp8", q[:, :0], c.cache, c.d_bt, c.d_lens, c.d_ks, c.d_vs,
                             out[:, :0], None)


def test_full_size_sampled_rows():
    """The benchmark's prefill step (4 x 126,976 FP8 tokens, head_dim 128, 64
    query heads, a 2,048-token chunk written then attended to), as bench.py
    launches it; sampled (sequence, query, head) rows are recomputed by the
    oracle from its own pages of the same BF16 tokens."""
    w = wl.WORKLOADS["agents-fp8-4x127k"]
    sc = DecodeScenario(w)
    sc.prefill_setup()
    sc.write()
    sc.prefill()
    torch.cuda.synchronize()
    assert int(sc.err.item()) == 0
    ks, vs = float(sc.d_ks.item()), float(sc.d_vs.item())
    T, G, D = sc.chunk, sc.Hq // sc.H, sc.D
    out = sc.out_chunk
    lse = sc.lse_chunk
    for b, h in [(0, 0), (3, 5)]:
        n = int(sc.lens[b])
        k, v = sc.tokens(b)
        kb = k[:n, h:h + 1].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        vb = v[:n, h:h + 1].contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        del k, v
        used = -(-n // 16)
        okc, ovc = oracle.new_cache(sc.fmt, used, 1, D)
        oracle.write(sc.fmt, kb, vb, np.arange(n, dtype=np.int64), okc, ovc, ks, vs)
        q = sc.q_chunk[b:b + 1, :, h * G:(h + 1) * G].contiguous()
        qb = q.view(torch.int16).cpu().numpy().view(np.uint16)
        bt = np.arange(used, dtype=np.int32)[None, :]
        rows = np.array([[0, i, j] for i in (0, 1, 1000, T - 1) for j in (0, G - 1)], np.int32)
        ref_out, ref_lse = oracle.prefill_attention(sc.fmt, qb, okc, ovc, 1, bt,
                                                    np.array([n], np.int32), ks, vs, rows=rows)
        got_o = out[b, rows[:, 1], h * G + rows[:, 2]].cpu().numpy()
        got_l = lse[b, rows[:, 1], h * G + rows[:, 2]].cpu().numpy()
        assert_attention_close(got_o, got_l, ref_out[0, rows[:, 1], rows[:, 2]],
                               ref_lse[0, rows[:, 1], rows[:, 2]])
