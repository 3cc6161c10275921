"""Pins of the oracle's float64 chunked-prefill attention: against torch's
scaled_dot_product_attention in float64 with an explicit causal mask (an
independent library routine) on the oracle's own dequantised values, and
closed forms (a chunk that starts the sequence: its first query sees one
token; q = 0 gives the running mean of V; queries before the sequence start
are empty).  A consistency check ties the chunk's last query to the decode of
the same sequence."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_21_b200 import workloads as wl

from test_oracle_attention import build_case, dequant_seq


def chunk_queries(seed, B, Tq, Hq, D, zero=False):
    q = wl.make_query(wl.rng_for(seed, 7), B * Tq, Hq, D).reshape(B, Tq, Hq, D)
    return np.zeros_like(q) if zero else q


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("D", [64, 128])
def test_matches_torch_sdpa_float64_with_a_causal_mask(fmt, D):
    B, H, Hq, Tq = 3, 2, 8, 16
    lens = [37, 16, 70]
    c = build_case(fmt, B, H, Hq, D, lens, seed=300 + D, factor=8.0)
    q = chunk_queries(301 + D, B, Tq, Hq, D)
    out, lse = oracle.prefill_attention(fmt, q, c["kc"], c["vc"], H, c["bt"], c["lens"],
                                        c["ks"], c["vs"])
    G = Hq // H
    for b in range(B):
        T = lens[b]
        kd, vd = dequant_seq(fmt, c, b)  # [T][H][D] fp32
        k = torch.from_numpy(kd.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
        v = torch.from_numpy(vd.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
        qq = torch.from_numpy(wl.bf16_bits_to_f32(q[b]).astype(np.float64)).permute(1, 0, 2)
        pos = T - Tq + torch.arange(Tq)[:, None]  # [Tq][1] query positions
        allowed = torch.arange(T)[None, :] <= pos  # [Tq][T]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, k, v, attn_mask=allowed)
        scores = (qq @ k.transpose(1, 2)) / math.sqrt(D)
        ref_lse = torch.logsumexp(scores.masked_fill(~allowed, -math.inf), dim=-1)
        np.testing.assert_allclose(out[b], ref.permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[b], ref_lse.T.numpy(), rtol=1e-13, atol=1e-13)


def test_chunk_that_starts_the_sequence():
    """len = Tq: query i sits at position i, so query 0 sees token 0 only
    (out = its V, lse = its score) and q = 0 gives the mean of V over
    tokens 0..i with lse = ln(i + 1)."""
    H, Hq, D, Tq = 2, 4, 64, 24
    c = build_case("fp8", 1, H, Hq, D, [Tq], seed=41)
    kd, vd = dequant_seq("fp8", c, 0)
    q = chunk_queries(42, 1, Tq, Hq, D)
    out, lse = oracle.prefill_attention("fp8", q, c["kc"], c["vc"], H, c["bt"], c["lens"],
                                        c["ks"], c["vs"])
    for j in range(Hq):
        h = j // (Hq // H)
        assert np.array_equal(out[0, 0, j], vd[0, h].astype(np.float64))
        s = np.dot(wl.bf16_bits_to_f32(q[0, 0, j]).astype(np.float64),
                   kd[0, h].astype(np.float64)) / math.sqrt(D)
        assert abs(lse[0, 0, j] - s) <= 1e-12 * max(1, abs(s))
    qz = chunk_queries(42, 1, Tq, Hq, D, zero=True)
    out, lse = oracle.prefill_attention("fp8", qz, c["kc"], c["vc"], H, c["bt"], c["lens"],
                                        c["ks"], c["vs"])
    for i in range(Tq):
        for j in range(Hq):
            h = j // (Hq // H)
            mean = vd[: i + 1, h].astype(np.float64).mean(axis=0)
            np.testing.assert_allclose(out[0, i, j], mean, rtol=1e-12, atol=1e-12)
            assert abs(lse[0, i, j] - math.log(i + 1)) <= 1e-12


def test_queries_before_the_sequence_start_are_empty():
    """A sequence shorter than the chunk: its first Tq - len queries sit at
    negative positions and attend to nothing (out = 0, lse = -inf)."""
    H, Hq, D, Tq = 2, 8, 64, 20
    c = build_case("nvfp4", 1, H, Hq, D, [7], seed=43)
    q = chunk_queries(44, 1, Tq, Hq, D)
    out, lse = oracle.prefill_attention("nvfp4", q, c["kc"], c["vc"], H, c["bt"], c["lens"],
                                        c["ks"], c["vs"])
    assert np.all(out[0, : Tq - 7] == 0.0) and np.all(lse[0, : Tq - 7] == -np.inf)
    assert np.all(np.isfinite(lse[0, Tq - 7:]))


def test_rows_subset_and_last_query_equals_decode():
    B, H, Hq, D, Tq = 2, 2, 8, 128, 9
    lens = [33, 50]
    c = build_case("fp8", B, H, Hq, D, lens, seed=45)
    q = chunk_queries(46, B, Tq, Hq, D)
    out, lse = oracle.prefill_attention("fp8", q, c["kc"], c["vc"], H, c["bt"], c["lens"],
                                        c["ks"], c["vs"])
    rows = np.array([[1, 8, 3], [0, 0, 7], [1, 2, 0]], np.int32)
    o2, l2 = oracle.prefill_attention("fp8", q, c["kc"], c["vc"], H, c["bt"], c["lens"],
                                      c["ks"], c["vs"], rows=rows)
    for b, i, j in rows:
        assert np.array_equal(o2[b, i, j], out[b, i, j]) and l2[b, i, j] == lse[b, i, j]
    assert np.isnan(l2[0, 1, 0])
    od, ld = oracle.decode_attention("fp8", q[:, Tq - 1], c["kc"], c["vc"], H, c["bt"],
                                     c["lens"], c["ks"], c["vs"])
    assert np.array_equal(od, out[:, Tq - 1]) and np.array_equal(ld, lse[:, Tq - 1])
