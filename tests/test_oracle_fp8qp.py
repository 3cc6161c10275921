"""Pins of the oracle's FP8-attention variant (E4M3 Q with q_scale, E4M3 P
with prob_scale, P quantized page by page against the page's largest score;
"FP8 KV calibration guide", paragraphs on the Radiance calibrator and on the
Q/K/V-only sidecar and probability scales).  Each check ties it to something
other than itself:
  * pages whose scores are all equal reduce it to exact attention (the
    regular float64 oracle, itself pinned to torch SDPA): scores, the page
    structure and the cross-page merge;
  * q = 0: every score 0, so out = dec(E4M3(1/prob_scale)) * prob_scale *
    mean(V_hat) and lse = ln T (closed form, with the calibrator's prob_scale);
  * against exact attention with the same E4M3 query, out stays within the
    E4M3 rounding bound on P (relative 2^-4 per weight), and lse is exact
    (the normaliser uses the unquantized probabilities);
  * the decision-boundary bound amb is 0 for eps = 0 and grows with eps."""
import numpy as np
import pytest

import oracle
from quantized_kv_cache_21_b200 import workloads as wl

E4M3_VALUES = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))  # finite, non-negative


def e4m3_query(rng, B, Hq, D, span=6):
    """BF16 bits of a query whose values are E4M3 values (exact in BF16), so
    with q_scale = 1 the quantized query equals the query."""
    mags = E4M3_VALUES[(E4M3_VALUES >= 2.0 ** -span) & (E4M3_VALUES <= 2.0 ** 2)]
    x = rng.choice(mags, size=(B, Hq, D)) * rng.choice([-1.0, 1.0], size=(B, Hq, D))
    return wl.f32_to_bf16_bits(x.astype(np.float32))


def fp8_cache(rng, k_rows, v_rows):
    """FP8 cache holding the given BF16 K/V rows ([T][1][D]) at slots 0..T-1."""
    T, H, D = k_rows.shape
    ks = oracle.fp8_scale(oracle.absmax_bf16(k_rows))
    vs = oracle.fp8_scale(oracle.absmax_bf16(v_rows))
    nb = -(-T // 16)
    kc, vc = oracle.new_cache("fp8", nb, H, D)
    oracle.write("fp8", k_rows, v_rows, np.arange(T), kc, vc, ks, vs)
    return kc, vc, ks, vs, np.arange(nb, dtype=np.int32)[None]


@pytest.mark.parametrize("T", [16, 37, 160])
@pytest.mark.parametrize("q_scale", [1.0, 0.25])
def test_equal_scores_within_pages_is_exact_attention(T, q_scale):
    """K rows repeat within each 16-token page, so every score of a page is
    equal: each p is exactly 1, and with prob_scale = 2^-8 its E4M3 code is
    exact.  The query is q_scale times E4M3 values, so its E4M3 codes are
    exact too.  The variant is then exact attention over the same query."""
    rng = wl.rng_for(71, T)
    D, Hq = 64, 4
    npg = -(-T // 16)
    page_k = wl.make_tokens(rng, npg, 1, D, [(0, 3)], 8.0)
    k = np.repeat(page_k, 16, axis=0)[:T]
    v = wl.make_tokens(rng, T, 1, D, [(0, 5)], 8.0)
    kc, vc, ks, vs, bt = fp8_cache(rng, k, v)
    q = wl.f32_to_bf16_bits(oracle.bf16_to_f32(e4m3_query(rng, 1, Hq, D)) * np.float32(q_scale))
    lens = np.array([T], np.int32)
    out, lse, _ = oracle.decode_attention_fp8qp(q, kc, vc, 1, bt, lens, ks, vs, q_scale,
                                                2.0 ** -8)
    ref_out, ref_lse = oracle.decode_attention("fp8", q, kc, vc, 1, bt, lens, ks, vs)
    # the regular oracle rounds each dequantised element to fp32 (its
    # definition), this variant scales the float64 sums of code products:
    # they agree to the fp32 rounding of one element (2^-24 relative)
    _, v_hat = oracle.dequantize("fp8", kc, vc, 1, D, np.arange(T), ks, vs)
    np.testing.assert_allclose(out, ref_out, rtol=0, atol=1e-6 * np.abs(v_hat).max())
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-6)
    # the pages really have different scores (the merge across pages matters)
    assert np.ptp(ref_lse) > 0 or npg == 1


def test_zero_query_closed_form():
    rng = wl.rng_for(72, 0)
    T, D, Hq = 50, 128, 8
    k = wl.make_tokens(rng, T, 1, D, [(0, 1)], 16.0)
    v = wl.make_tokens(rng, T, 1, D, [(0, 2)], 16.0)
    kc, vc, ks, vs, bt = fp8_cache(rng, k, v)
    q = np.zeros((1, Hq, D), np.uint16)
    ps = oracle.fp8_scale(1.0)  # the calibrator's formula at an observed maximum of 1
    assert ps == np.float32(1.05) / np.float32(448.0)
    out, lse, _ = oracle.decode_attention_fp8qp(q, kc, vc, 1, bt, np.array([T], np.int32), ks,
                                                vs, 0.01, ps)
    # 1 / ps = 426.67 lies between the E4M3 values 416 and 448, nearer 416
    c = 416.0 * ps
    _, v_hat = oracle.dequantize("fp8", kc, vc, 1, D, np.arange(T), ks, vs)
    # (v_hat from dequantize is rounded to fp32 per element: 2^-24 relative)
    np.testing.assert_allclose(out[0], np.repeat(c * v_hat.astype(np.float64).mean(axis=0), Hq,
                                                 axis=0), rtol=0, atol=1e-7 * np.abs(v_hat).max())
    np.testing.assert_allclose(lse, np.log(T), rtol=1e-14)


@pytest.mark.parametrize("T,seed", [(1, 0), (15, 1), (333, 2), (2048, 3)])
def test_within_the_p_rounding_bound_of_exact_attention(T, seed):
    rng = wl.rng_for(73, seed)
    D, Hq = 128, 8
    k = wl.make_tokens(rng, T, 1, D, [(0, 7)], 16.0)
    v = wl.make_tokens(rng, T, 1, D, [(0, 9)], 16.0)
    kc, vc, ks, vs, bt = fp8_cache(rng, k, v)
    q = e4m3_query(rng, 1, Hq, D, span=4)
    lens = np.array([T], np.int32)
    ps = oracle.fp8_scale(1.0)
    out, lse, _ = oracle.decode_attention_fp8qp(q, kc, vc, 1, bt, lens, ks, vs, 1.0, ps)
    ref_out, ref_lse = oracle.decode_attention("fp8", q, kc, vc, 1, bt, lens, ks, vs)
    _, v_hat = oracle.dequantize("fp8", kc, vc, 1, D, np.arange(T), ks, vs)
    vmax = np.abs(v_hat).max()
    # E4M3 rounding of p / ps: relative 2^-4 in the normal range, plus at most
    # half the smallest subnormal step (2^-10 * ps) per weight below it, plus
    # the fp32 rounding of the regular oracle's dequantised elements
    bound = (2.0 ** -4 + 2.0 ** -10 * ps + 1e-6) * vmax
    err = np.abs(out - ref_out).max()
    assert err <= bound, (err, bound)
    assert err > 0 or T == 1  # P really is quantized
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-6)  # fp32 rounding of k_hat, as above


def test_boundary_bound_grows_with_eps():
    rng = wl.rng_for(74, 0)
    T, D, Hq = 700, 64, 8
    k = wl.make_tokens(rng, T, 1, D)
    v = wl.make_tokens(rng, T, 1, D)
    kc, vc, ks, vs, bt = fp8_cache(rng, k, v)
    q = wl.make_query(rng, 1, Hq, D)
    qs = oracle.fp8_scale(oracle.absmax_bf16(q))
    lens = np.array([T], np.int32)
    ps = oracle.fp8_scale(1.0)
    amb = [oracle.decode_attention_fp8qp(q, kc, vc, 1, bt, lens, ks, vs, qs, ps, eps=e)[2]
           for e in (0.0, 1e-5, 1e-3)]
    assert np.all(amb[0] == 0)
    assert np.all(amb[1] <= amb[2]) and amb[2].sum() > 0
