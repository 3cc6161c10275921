"""Pins of the oracle's 3-bit planar-rotation codec (PQ3; "AMD MI300X - KV
Cache Compression Benchmark", "Key Results": 52-byte blocks, 4.923x against
FP16, reconstruction cosine similarity 0.983, the PlanarQuant rotation's 256
FMAs; the repository's Lloyd-Max codebook generator).  Each check ties it to
something other than itself: the textbook Lloyd-Max quantizers of N(0, 1) and
their optimality conditions integrated with scipy, numpy's f16 rounding, exact
float64 rotations and nearest-centroid search, closed-form rotations, scale
invariance, the page's byte counts and cosine similarity, an explicit bit
layout, and torch SDPA for the attention over the dequantised values."""
import numpy as np
import pytest
import torch
from scipy import integrate
from scipy.stats import norm

import oracle
from quantized_kv_cache_21_b200 import workloads as wl


def test_lloyd_max_matches_the_textbook_quantizers():
    # Max (1960), Table: optimum quantizers for a unit-variance Gaussian
    np.testing.assert_allclose(oracle.lloyd_max_gaussian(2), [-0.7979, 0.7979], atol=1e-4)
    np.testing.assert_allclose(np.abs(oracle.lloyd_max_gaussian(4))[2:], [0.4528, 1.510],
                               atol=1e-3)
    np.testing.assert_allclose(oracle.lloyd_max_gaussian(8)[4:],
                               [0.2451, 0.7560, 1.344, 2.152], atol=1e-3)
    assert oracle.lloyd_max_gaussian(2)[1] == pytest.approx(np.sqrt(2 / np.pi), abs=1e-12)


def test_lloyd_max_optimality_conditions_and_mse():
    c = oracle.lloyd_max_gaussian(8)
    t = np.concatenate([[-np.inf], (c[:-1] + c[1:]) / 2, [np.inf]])
    mse = 0.0
    for k in range(8):  # each centroid is the mean of its cell (scipy quadrature)
        mass = norm.cdf(t[k + 1]) - norm.cdf(t[k])
        mean = integrate.quad(lambda x: x * norm.pdf(x), t[k], t[k + 1])[0] / mass
        assert c[k] == pytest.approx(mean, abs=1e-9)
        mse += integrate.quad(lambda x: (x - c[k]) ** 2 * norm.pdf(x), t[k], t[k + 1])[0]
    assert mse == pytest.approx(0.03455, abs=2e-5)  # the 3-bit Gaussian distortion


def test_codebook_is_f16_rounded_and_symmetric():
    cb = oracle.pq3_codebook()
    want = (oracle.lloyd_max_gaussian(8) / np.sqrt(128.0)).astype(np.float16).astype(np.float32)
    assert np.array_equal(cb, want)
    assert np.array_equal(cb[:4], -cb[4:][::-1]) and np.all(np.diff(cb) > 0)


def params(seed):
    return oracle.pq3_params(wl.planar_rotation(wl.rng_for(seed, 0)))


def exact_y(x_bits, nrm, pr):
    """The rotated unit vector in float64 (exact products of the fp32 inputs)."""
    u = oracle.bf16_to_f32(x_bits).astype(np.float64) / np.float64(nrm)
    c, s = pr[8::2].astype(np.float64), pr[9::2].astype(np.float64)
    y = np.empty(128)
    y[0::2] = c * u[0::2] - s * u[1::2]
    y[1::2] = s * u[0::2] + c * u[1::2]
    return y


def test_encode_is_nearest_centroid_of_the_rotated_unit_vector():
    pr = params(1)
    cb = pr[:8].astype(np.float64)
    rng = wl.rng_for(75, 0)
    x = wl.make_tokens(rng, 200, 1, 128, [(0, 5)], 16.0)[:, 0]
    checked = 0
    for row in x:
        nrm, idx = oracle.pq3_encode_row(row, pr)
        ref = np.linalg.norm(oracle.bf16_to_f32(row).astype(np.float64))
        assert nrm == pytest.approx(ref, rel=1e-6)
        y = exact_y(row, nrm, pr)
        dist = np.abs(y[:, None] - cb[None, :])
        best = np.argmin(dist, axis=1)
        # where two centroids are (nearly) equally near, fp32 rounding decides
        sdist = np.sort(dist, axis=1)
        clear = sdist[:, 1] - sdist[:, 0] > 1e-6
        assert np.array_equal(idx[clear], best[clear])
        checked += clear.sum()
    assert checked > 200 * 120


def test_closed_form_rotations_and_scale_invariance():
    rng = wl.rng_for(76, 0)
    x = wl.make_tokens(rng, 1, 1, 128)[0, 0]
    cb = oracle.pq3_codebook()
    ident = oracle.pq3_params(np.tile([1.0, 0.0], (64, 1)))
    quarter = oracle.pq3_params(np.tile([0.0, 1.0], (64, 1)))  # 90 degrees
    n0, i0 = oracle.pq3_encode_row(x, ident)
    n1, i1 = oracle.pq3_encode_row(x, quarter)
    u = oracle.bf16_to_f32(x) / np.float32(n0)
    thr = (cb[:-1] + cb[1:]) / np.float32(2)
    assert np.array_equal(i0, np.searchsorted(thr, u, side="left"))  # no rotation: y = u
    y = np.empty(128, np.float32)
    y[0::2], y[1::2] = -u[1::2], u[0::2]  # y = (-u1, u0), exact
    assert np.array_equal(i1, np.searchsorted(thr, y, side="left"))
    # decode with no rotation is norm * centroid
    np.testing.assert_array_equal(oracle.pq3_decode_row(n0, i0, ident),
                                  np.float32(n0) * cb[i0])
    # doubling a BF16 vector doubles its norm exactly and keeps every index
    x2 = wl.f32_to_bf16_bits(oracle.bf16_to_f32(x) * np.float32(2))
    pr = params(2)
    (na, ia), (nb, ib) = oracle.pq3_encode_row(x, pr), oracle.pq3_encode_row(x2, pr)
    assert nb == 2 * na and np.array_equal(ia, ib)
    # an all-zero vector: norm 0, indices 0, decodes to 0
    nz, iz = oracle.pq3_encode_row(np.zeros(128, np.uint16), pr)
    assert nz == 0.0 and not iz.any()
    assert not oracle.pq3_decode_row(nz, iz, pr).any()


def test_block_bytes_and_reconstruction_match_the_page():
    # 52-byte blocks: a 128-element FP16 vector is 256 bytes, 4.923x
    assert oracle.head_page_bytes("pq3", 128) == 16 * 52
    assert round(256 / 52, 3) == 4.923
    # reconstruction cosine similarity on Gaussian vectors: the page's 0.983
    pr = params(3)
    rng = wl.rng_for(77, 0)
    x = wl.make_tokens(rng, 2000, 1, 128)[:, 0]
    cos = []
    for row in x:
        nrm, idx = oracle.pq3_encode_row(row, pr)
        xh = oracle.pq3_decode_row(nrm, idx, pr).astype(np.float64)
        xf = oracle.bf16_to_f32(row).astype(np.float64)
        cos.append(xh @ xf / np.linalg.norm(xh) / np.linalg.norm(xf))
    assert np.mean(cos) == pytest.approx(0.983, abs=0.003)


def test_bit_layout_of_a_page():
    """A 16-token head page: the 16 fp32 norms, then 16 rows of 48 bytes.  A
    row is 8 little-endian 32-bit words of the indices' low 2 bits (word w:
    indices 16w + k at bits 4k and 16w + 8 + k at bits 4k + 2, k < 8), then
    4 words of their high bits (word v: indices 32v + 8j + k at bit
    4k + (2, 3, 0, 1)[j]); rebuilt here with numpy shifts and sums."""
    pr = params(6)
    rng = wl.rng_for(79, 0)
    x = wl.make_tokens(rng, 1, 1, 128, [(0, 7)], 16.0)
    nrm, idx = oracle.pq3_encode_row(x[0, 0], pr)
    kc, vc = oracle.new_cache("pq3", 1, 1, 128)
    oracle.pq3_write(x, x, np.array([3]), kc, vc, pr, pr)
    assert kc[12:16].view(np.float32)[0] == np.float32(nrm)  # slot 3's norm
    idx = idx.astype(np.uint64)
    low = (idx & 3).reshape(8, 2, 8)  # [word][half][k]: index 16 w + 8 half + k
    low_words = (low << (4 * np.arange(8, dtype=np.uint64) + 2 * np.arange(2, dtype=np.uint64)[:, None])).sum(axis=(1, 2))
    high = (idx >> 2).reshape(4, 4, 8)  # [word][j][k]: index 32 v + 8 j + k
    slot_of_j = np.array([2, 3, 0, 1], dtype=np.uint64)[:, None]
    high_words = (high << (4 * np.arange(8, dtype=np.uint64) + slot_of_j)).sum(axis=(1, 2))
    want = np.concatenate([low_words, high_words]).astype("<u4").view(np.uint8)
    assert want.size == 48
    assert np.array_equal(kc[64 + 3 * 48: 64 + 4 * 48], want)
    # every other byte of the page is untouched
    rest = np.delete(kc, np.r_[12:16, 64 + 3 * 48: 64 + 4 * 48])
    assert not rest.any()


@pytest.mark.parametrize("T", [1, 17, 300])
def test_attention_over_the_dequantised_cache_is_sdpa(T):
    rng = wl.rng_for(78, T)
    H, Hq, D = 2, 8, 128
    k = wl.make_tokens(rng, T, H, D, [(0, 3)], 8.0)
    v = wl.make_tokens(rng, T, H, D, [(1, 9)], 8.0)
    q = wl.make_query(rng, 1, Hq, D)
    kp, vp = params(4), params(5)
    nb = -(-T // 16)
    kc, vc = oracle.new_cache("pq3", nb, H, D)
    oracle.pq3_write(k, v, np.arange(T), kc, vc, kp, vp)
    bt = np.arange(nb, dtype=np.int32)[None]
    out, lse = oracle.pq3_decode_attention(q, kc, vc, H, bt, np.array([T], np.int32), kp, vp)
    kf, vf = oracle.pq3_to_f32(kc, vc, H, kp, vp)
    kh = kf.view(np.float32).reshape(nb, H, 16, D).transpose(1, 0, 2, 3).reshape(H, -1, D)[:, :T]
    vh = vf.view(np.float32).reshape(nb, H, 16, D).transpose(1, 0, 2, 3).reshape(H, -1, D)[:, :T]
    # each row of the dequantised cache is the codec's decode of that token
    nrm, idx = oracle.pq3_encode_row(k[T - 1, 1], kp)
    np.testing.assert_array_equal(kh[1, T - 1], oracle.pq3_decode_row(nrm, idx, kp))
    qt = torch.from_numpy(oracle.bf16_to_f32(q).astype(np.float64)).view(1, H, Hq // H, D)
    kt = torch.from_numpy(kh.astype(np.float64))[None, :, None]
    vt = torch.from_numpy(vh.astype(np.float64))[None, :, None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.expand(1, H, Hq // H, T, D).reshape(1, H, Hq // H, T, D)[:, :, 0],
        vt.expand(1, H, Hq // H, T, D).reshape(1, H, Hq // H, T, D)[:, :, 0], scale=D ** -0.5)
    np.testing.assert_allclose(out[0], ref.reshape(Hq, D).numpy(), rtol=0, atol=1e-10)
