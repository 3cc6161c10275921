"""Pins of the oracle's float64 decode attention: against torch's
scaled_dot_product_attention in float64 (an independent library routine) on the
oracle's own dequantised values, closed forms (single token, constant V, q = 0,
one dominant key, empty sequence), the split/merge identity, and invariance to
where pages sit in the pool."""
import math

import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_21_b200 import workloads as wl


def build_case(fmt, B, H, Hq, D, lens, seed, permuted=True, factor=1.0):
    rng = wl.rng_for(seed, 0)
    nbps = max(1, -(-max(lens) // 16))
    nb = B * nbps + 3
    bt = (wl.permuted_block_table(wl.rng_for(seed, 1), B, nbps, nb) if permuted
          else wl.identity_block_table(B, nbps))
    kc, vc = oracle.new_cache(fmt, nb, H, D)
    outl = wl.outlier_pairs(rng, H, D, per_head=1)
    k_all, v_all = [], []
    for b in range(B):
        k = wl.make_tokens(rng, lens[b], H, D, outl, factor)
        v = wl.make_tokens(rng, lens[b], H, D, outl, factor)
        k_all.append(k)
        v_all.append(v)
    kcat = np.concatenate(k_all) if k_all else np.zeros((0, H, D), np.uint16)
    vcat = np.concatenate(v_all) if v_all else np.zeros((0, H, D), np.uint16)
    ks = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(kcat)) if kcat.size else 1.0
    vs = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(vcat)) if vcat.size else 1.0
    for b in range(B):
        slots = wl.physical_slots(bt, b, np.arange(lens[b]))
        oracle.write(fmt, k_all[b], v_all[b], slots, kc, vc, ks, vs)
    q = wl.make_query(rng, B, Hq, D)
    return dict(q=q, kc=kc, vc=vc, bt=bt, lens=np.array(lens, np.int32), ks=ks, vs=vs, H=H, D=D)


def dequant_seq(fmt, c, b):
    slots = wl.physical_slots(c["bt"], b, np.arange(c["lens"][b]))
    return oracle.dequantize(fmt, c["kc"], c["vc"], c["H"], c["D"], slots, c["ks"], c["vs"])


@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4"])
@pytest.mark.parametrize("D", [64, 128])
def test_matches_torch_sdpa_float64(fmt, D):
    B, H, Hq = 3, 2, 8
    c = build_case(fmt, B, H, Hq, D, [37, 16, 70], seed=100 + D, factor=8.0)
    out, lse = oracle.decode_attention(fmt, c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                       c["ks"], c["vs"])
    G = Hq // H
    for b in range(B):
        kd, vd = dequant_seq(fmt, c, b)  # [T][H][D] fp32
        k = torch.from_numpy(kd.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
        v = torch.from_numpy(vd.astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
        q = torch.from_numpy(wl.bf16_bits_to_f32(c["q"][b]).astype(np.float64))[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)[:, 0, :]
        scores = (q @ k.transpose(1, 2))[:, 0, :] / math.sqrt(D)
        ref_lse = torch.logsumexp(scores, dim=-1)
        np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(lse[b], ref_lse.numpy(), rtol=1e-13, atol=1e-13)


def test_closed_forms():
    H, Hq, D = 2, 4, 64
    # single token: out = v_hat, lse = the one score
    c = build_case("fp8", 1, H, Hq, D, [1], seed=5)
    out, lse = oracle.decode_attention("fp8", c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                       c["ks"], c["vs"])
    kd, vd = dequant_seq("fp8", c, 0)
    for j in range(Hq):
        h = j // (Hq // H)
        assert np.array_equal(out[0, j], vd[0, h].astype(np.float64))
        s = np.dot(wl.bf16_bits_to_f32(c["q"][0, j]).astype(np.float64),
                   kd[0, h].astype(np.float64)) / math.sqrt(D)
        assert abs(lse[0, j] - s) <= 1e-12 * max(1, abs(s))
    # q = 0: uniform weights -> mean of V, lse = ln T
    c = build_case("nvfp4", 1, H, Hq, D, [45], seed=6)
    c["q"][:] = 0
    out, lse = oracle.decode_attention("nvfp4", c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                       c["ks"], c["vs"])
    kd, vd = dequant_seq("nvfp4", c, 0)
    for j in range(Hq):
        np.testing.assert_allclose(out[0, j], vd[:, j // 2].astype(np.float64).mean(0),
                                   rtol=1e-13, atol=1e-13)
        assert abs(lse[0, j] - math.log(45)) < 1e-13


def test_constant_v_and_dominant_key():
    H, Hq, D, T = 1, 2, 64, 50
    rng = wl.rng_for(9, 0)
    k = wl.make_tokens(rng, T, H, D)
    v = np.tile(wl.make_tokens(rng, 1, H, D), (T, 1, 1))
    bt = wl.identity_block_table(1, 4)
    kc, vc = oracle.new_cache("bf16", 4, H, D)
    oracle.write("bf16", k, v, wl.physical_slots(bt, 0, np.arange(T)), kc, vc, 1, 1)
    q = wl.make_query(rng, 1, Hq, D)
    out, _ = oracle.decode_attention("bf16", q, kc, vc, H, bt, np.array([T], np.int32), 1, 1)
    np.testing.assert_allclose(out[0, 0], wl.bf16_bits_to_f32(v[0, 0]), rtol=1e-14)
    # a key aligned with q and 80x longer than the rest dominates by > 50 nats
    qv = wl.bf16_bits_to_f32(q[0, 0])
    k2 = wl.make_tokens(rng, T, H, D)
    k2[17, 0] = wl.f32_to_bf16_bits(qv * 40)
    v2 = wl.make_tokens(rng, T, H, D)
    oracle.write("bf16", k2, v2, wl.physical_slots(bt, 0, np.arange(T)), kc, vc, 1, 1)
    out, _ = oracle.decode_attention("bf16", q, kc, vc, H, bt, np.array([T], np.int32), 1, 1)
    np.testing.assert_allclose(out[0, 0], wl.bf16_bits_to_f32(v2[17, 0]), rtol=1e-15, atol=1e-15)


def test_empty_sequence():
    c = build_case("fp8", 2, 1, 2, 64, [0, 5], seed=3)
    out, lse = oracle.decode_attention("fp8", c["q"], c["kc"], c["vc"], 1, c["bt"], c["lens"],
                                       c["ks"], c["vs"])
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(lse[1]))


def test_split_merge_identity():
    H, Hq, D = 2, 4, 128
    c = build_case("fp8", 1, H, Hq, D, [300], seed=21, factor=10.0)
    out, lse = oracle.decode_attention("fp8", c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                       c["ks"], c["vs"])
    for cuts in ([0, 16, 160, 300], [0, 1, 2, 299, 300], [0, 150, 150, 300]):
        for j in range(Hq):
            parts = [oracle.attention_range("fp8", c["q"][0, j], c["kc"], c["vc"], H, D,
                                            c["bt"][0], j // 2, a, b, c["ks"], c["vs"],
                                            1 / math.sqrt(D)) for a, b in zip(cuts, cuts[1:])]
            o, l_ = oracle.merge(np.stack([p[0] for p in parts]), [p[1] for p in parts],
                                 [p[2] for p in parts])
            np.testing.assert_allclose(o, out[0, j], rtol=1e-13, atol=1e-13)
            assert abs(l_ - lse[0, j]) < 1e-12


def test_page_placement_invariance():
    H, Hq, D = 2, 4, 64
    a = build_case("nvfp4", 2, H, Hq, D, [33, 64], seed=44, permuted=False)
    b = build_case("nvfp4", 2, H, Hq, D, [33, 64], seed=44, permuted=True)
    oa = oracle.decode_attention("nvfp4", a["q"], a["kc"], a["vc"], H, a["bt"], a["lens"],
                                 a["ks"], a["vs"])
    ob = oracle.decode_attention("nvfp4", b["q"], b["kc"], b["vc"], H, b["bt"], b["lens"],
                                 b["ks"], b["vs"])
    assert np.array_equal(oa[0], ob[0]) and np.array_equal(oa[1], ob[1])


# ---- sliding-window mode ("AMD MI300X — KV Cache Compression Benchmark",
# section "SWA mode": attention over the most recent `window` tokens)

@pytest.mark.parametrize("fmt", ["bf16", "fp8", "nvfp4"])
def test_window_matches_torch_sdpa_on_the_last_tokens(fmt):
    """torch float64 SDPA over only the last W dequantised tokens (W < len,
    W = len, W > len, and a W that is not a multiple of the page size)."""
    B, H, Hq, D = 4, 2, 8, 64
    c = build_case(fmt, B, H, Hq, D, [100, 37, 16, 70], seed=700, factor=8.0)
    G = Hq // H
    for W in (1, 17, 37, 64, 500):
        out, lse = oracle.decode_attention(fmt, c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                           c["ks"], c["vs"], window=W)
        for b in range(B):
            n = int(c["lens"][b])
            t0 = max(0, n - W)
            kd, vd = dequant_seq(fmt, c, b)
            k = torch.from_numpy(kd[t0:].astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
            v = torch.from_numpy(vd[t0:].astype(np.float64)).permute(1, 0, 2).repeat_interleave(G, 0)
            q = torch.from_numpy(wl.bf16_bits_to_f32(c["q"][b]).astype(np.float64))[:, None, :]
            ref = torch.nn.functional.scaled_dot_product_attention(q, k, v)[:, 0, :]
            scores = (q @ k.transpose(1, 2))[:, 0, :] / math.sqrt(D)
            np.testing.assert_allclose(out[b], ref.numpy(), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(lse[b], torch.logsumexp(scores, -1).numpy(), rtol=1e-12)


def test_window_equals_full_attention_over_a_truncated_cache():
    """A windowed decode over the cache equals a full decode over a cache that
    holds only those last W tokens (the page's truncated-cache form), with the
    tokens at other pages and offsets."""
    fmt, B, H, Hq, D, W = "fp8", 2, 2, 8, 128, 45
    c = build_case(fmt, B, H, Hq, D, [200, 30], seed=701, factor=4.0)
    out_w, lse_w = oracle.decode_attention(fmt, c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                           c["ks"], c["vs"], window=W)
    rng = wl.rng_for(702, 0)
    for b in range(B):
        n = int(c["lens"][b])
        t0 = max(0, n - W)
        # the raw codes of the last W tokens, rewritten at positions 0.. of a
        # fresh randomly permuted table (codes are copied, not re-quantized)
        m = n - t0
        nbps = -(-m // 16)
        bt2 = wl.permuted_block_table(rng, 1, nbps, nbps + 5)
        kc2, vc2 = oracle.new_cache(fmt, nbps + 5, H, D)
        page = oracle.head_page_bytes(fmt, D)
        src = wl.physical_slots(c["bt"], b, np.arange(t0, n))
        dst = wl.physical_slots(bt2, 0, np.arange(m))
        for s_, d_ in zip(src, dst):
            for h in range(H):
                so = (s_ // 16 * H + h) * page + (s_ % 16) * D
                do = (d_ // 16 * H + h) * page + (d_ % 16) * D
                kc2[do:do + D] = c["kc"][so:so + D]
                vc2[do:do + D] = c["vc"][so:so + D]
        out_f, lse_f = oracle.decode_attention(fmt, c["q"][b:b + 1], kc2, vc2, H, bt2,
                                               np.array([m], np.int32), c["ks"], c["vs"])
        assert np.array_equal(out_w[b], out_f[0]) and np.array_equal(lse_w[b], lse_f[0])


def test_window_of_one_token_returns_the_last_value():
    fmt, H, Hq, D = "bf16", 1, 4, 64
    c = build_case(fmt, 1, H, Hq, D, [50], seed=703)
    out, lse = oracle.decode_attention(fmt, c["q"], c["kc"], c["vc"], H, c["bt"], c["lens"],
                                       c["ks"], c["vs"], window=1)
    kd, vd = dequant_seq(fmt, c, 0)
    q = wl.bf16_bits_to_f32(c["q"][0]).astype(np.float64)
    for j in range(Hq):
        np.testing.assert_array_equal(out[0, j], vd[-1, 0].astype(np.float64))
        assert lse[0, j] == pytest.approx(q[j] @ kd[-1, 0].astype(np.float64) / math.sqrt(D),
                                          rel=1e-12)
