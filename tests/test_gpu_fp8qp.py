"""GPU parity of the FP8-attention variant (kv_decode_attention_fp8qp: E4M3
Q with q_scale and E4M3 P with prob_scale over the FP8 cache, QK and PV on
E4M3 tensor cores) against the oracle's float64 definition of the same
method ("FP8 KV calibration guide": the calibrator's Q scale; other attention
paths accept probability scales).

Tolerance: lse within 1e-5 relative (the normaliser uses the unquantized
probabilities); out within 2e-3 max-abs plus, per element, the oracle's bound
for P codes whose decision input lies within relative EPS of an E4M3
rounding boundary (the kernel decides on its own fp32 p, the oracle on its
float64 p).  Formats, head dims, GQA ratios, ragged and empty sequences,
forced and automatic splits, NaN bytes in unwritten slots, a negative
sm_scale, the q = 0 closed form and the device-side scale check."""
import numpy as np
import pytest
import torch

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl

from gpu_common import DEV, LSE_RTOL, OUT_ATOL, Case, dev_scalar, new_err

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -12  # relative distance to a rounding boundary within which either P code is valid


def scales(c: Case):
    qs = oracle.fp8_scale(oracle.absmax_bf16(c.q)) if c.q.size else 1.0
    return qs, oracle.fp8_scale(1.0)


def run(c: Case, num_splits=0, sm_scale=0.0, qs=None, ps=None, err=None):
    q_s, p_s = scales(c)
    qs = q_s if qs is None else qs
    ps = p_s if ps is None else ps
    msl = c.max_blocks * 16
    ws = kvq.new_workspace(kvq.kv_decode_workspace_size("fp8", c.B, c.Hq, c.Hkv, c.D, msl,
                                                        num_splits))
    out = torch.full((c.B, c.Hq, c.D), float("nan"), device=DEV)
    lse = torch.full((c.B, c.Hq), float("nan"), device=DEV)
    kvq.kv_decode_attention_fp8qp(c.d_q, c.cache, c.d_bt, c.d_lens, msl, c.d_ks, c.d_vs,
                                  dev_scalar(qs), dev_scalar(ps), out, lse, ws,
                                  c.err if err is None else err, sm_scale, num_splits)
    torch.cuda.synchronize()
    return out.cpu().numpy(), lse.cpu().numpy()


def reference(c: Case, sm_scale=None, qs=None, ps=None):
    q_s, p_s = scales(c)
    return oracle.decode_attention_fp8qp(c.q, c.okc, c.ovc, c.Hkv, c.bt, c.lens, c.ks, c.vs,
                                         q_s if qs is None else qs, p_s if ps is None else ps,
                                         sm_scale, eps=EPS)


def assert_close(out, lse, ref_out, ref_lse, amb):
    empty = np.isneginf(ref_lse)
    assert np.all(np.isneginf(lse[empty])) and np.all(out[empty] == 0)
    ok = ~empty
    assert np.all(np.isfinite(out[ok])) and np.all(np.isfinite(lse[ok]))
    excess = np.abs(out[ok] - ref_out[ok]) - amb[ok]
    assert excess.max(initial=0.0) <= OUT_ATOL, (
        f"out error beyond the boundary bound: {excess.max():.3e} > {OUT_ATOL}")
    err_lse = (np.abs(lse[ok] - ref_lse[ok]) / np.maximum(np.abs(ref_lse[ok]), 1.0)).max(initial=0)
    assert err_lse <= LSE_RTOL, f"lse relative error {err_lse:.3e}"
    return np.abs(out[ok] - ref_out[ok]).max(initial=0.0), err_lse


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("splits", [0, 1, 5])
def test_ragged_batch(D, splits):
    c = Case("fp8", 5, 2, 16, D, [1, 15, 16, 17, 1001], seed=8000 + D, factor=16.0)
    out, lse = run(c, splits)
    assert int(c.err.item()) == 0
    assert_close(out, lse, *reference(c))


@pytest.mark.parametrize("G", [1, 4, 8, 16])
def test_gqa_ratios(G):
    c = Case("fp8", 2, 2, 2 * G, 128, [333, 64], seed=8100 + G)
    out, lse = run(c)
    assert_close(out, lse, *reference(c))


def test_long_context_many_splits():
    c = Case("fp8", 1, 1, 8, 64, [20000], seed=8200, factor=16.0)
    ref = reference(c)
    outs = []
    for splits in (0, 3, 97):
        out, lse = run(c, splits)
        assert_close(out, lse, *ref)
        outs.append(out)
    # P is quantized per cache page, so the split changes only the fp32 merge order
    assert np.abs(outs[0] - outs[2]).max() < 1e-4


@pytest.mark.parametrize("max_len", [16, 100, 700])
def test_many_units_per_cta(max_len):
    """80 short (sequence, KV head) units: CTAs take up to 27 units each in
    turn, some spanning two CTAs, some empty."""
    rng = wl.rng_for(8250 + max_len, 3)
    lens = rng.integers(0, max_len + 1, size=40).tolist()
    c = Case("fp8", 40, 2, 16, 128, lens, seed=8260 + max_len, factor=16.0)
    out, lse = run(c)
    assert int(c.err.item()) == 0
    assert_close(out, lse, *reference(c))


def test_empty_and_single_token():
    c = Case("fp8", 3, 2, 8, 64, [0, 1, 0], seed=8300)
    out, lse = run(c)
    assert_close(out, lse, *reference(c))
    assert np.all(np.isneginf(lse[0])) and np.all(out[0] == 0)


def test_nan_bytes_in_unwritten_slots():
    c = Case("fp8", 2, 2, 8, 128, [37, 250], seed=8400, fill=0xFF)
    out, lse = run(c, 2)
    assert_close(out, lse, *reference(c))


def test_negative_sm_scale():
    c = Case("fp8", 4, 2, 16, 128, [1, 15, 17, 1001], seed=8500, factor=16.0)
    out, lse = run(c, 3, sm_scale=-0.08)
    assert_close(out, lse, *reference(c, sm_scale=-0.08))


def test_zero_query_closed_form():
    """q = 0: every score is 0 and every p is 1, so out = dec(E4M3(1 /
    prob_scale)) * prob_scale * mean(V_hat) and lse = ln T."""
    T = 300
    c = Case("fp8", 1, 1, 8, 64, [T], seed=8600)
    c.q[:] = 0
    c.d_q.zero_()
    ps = oracle.fp8_scale(1.0)
    out, lse = run(c, 3, qs=0.01, ps=ps)
    ref_out, ref_lse, amb = reference(c, qs=0.01, ps=ps)
    assert_close(out, lse, ref_out, ref_lse, amb)
    np.testing.assert_allclose(lse, np.log(T), rtol=1e-6)
    _, v_hat = oracle.dequantize("fp8", c.okc, c.ovc, 1, 64, wl.physical_slots(c.bt, 0, np.arange(T)),
                                 c.ks, c.vs)
    want = 416.0 * ps * v_hat.astype(np.float64).mean(axis=0)  # E4M3(426.67) = 416
    assert np.abs(out[0] - want).max() <= OUT_ATOL


def test_bad_scales_are_reported():
    c = Case("fp8", 1, 2, 8, 64, [200], seed=8700)
    for qs, ps in ((0.0, 0.01), (0.01, -1.0), (float("inf"), 0.01)):
        err = new_err()
        run(c, qs=qs, ps=ps, err=err)
        assert int(err.item()) == kvq.DERR_SCALE


def test_only_the_fp8_cache_is_accepted():
    c = Case("bf16", 1, 1, 8, 64, [40], seed=8800)
    out = torch.empty(1, 8, 64, device=DEV)
    with pytest.raises(kvq.KvqError, match="FP8 cache"):
        kvq.kv_decode_attention_fp8qp(c.d_q, c.cache, c.d_bt, c.d_lens, 48, c.d_ks, c.d_vs,
                                      dev_scalar(1.0), dev_scalar(1.0), out, None, None)
