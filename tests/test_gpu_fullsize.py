"""Parity at the benchmark's full sizes, in the launch configuration bench.py
times (automatic work split, one decode launch after the step's write).

For sampled (sequence, KV head) units the oracle recomputes everything from
the same BF16 inputs: its own calibration abs-max and scales (compared bit
for bit with the device's), its own quantized pages (compared bit for bit
with the device cache, gathered through the block table) and float64
attention over its own dequantised values (out within 2e-3, lse within 1e-5
relative).  Nothing the CUDA path produced is fed to the oracle."""
import numpy as np
import pytest
import torch

import oracle
from quantized_kv_cache_21_b200 import workloads as wl
from quantized_kv_cache_21_b200.scenario import DecodeScenario

from gpu_common import LSE_RTOL, OUT_ATOL

pytestmark = pytest.mark.gpu


def bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_scales(sc: DecodeScenario):
    """The oracle's abs-max and scales over the same calibration sample."""
    w = sc.w
    ks, vs = [], []
    for b in range(sc.B if w.calib_tokens is None else 1):
        k, v = sc.tokens(b)
        n = int(sc.lens[b]) if w.calib_tokens is None else w.calib_tokens
        ks.append(oracle.absmax_bf16(bits(k[:n])))
        vs.append(oracle.absmax_bf16(bits(v[:n])))
    return (oracle.scale_from_absmax(sc.fmt, max(ks)), oracle.scale_from_absmax(sc.fmt, max(vs)))


def device_pages(sc: DecodeScenario, b: int, h: int, which: str) -> np.ndarray:
    """The device cache's head pages of (sequence b, KV head h), in order."""
    page = oracle.head_page_bytes(sc.fmt, sc.D)
    buf = (sc.cache.k if which == "k" else sc.cache.v).view(sc.num_blocks, sc.H, page)
    used = -(-int(sc.lens[b]) // 16)  # pages holding the sequence's tokens
    idx = torch.from_numpy(sc.bt[b][:used].astype(np.int64)).to(buf.device)
    return buf[idx, h].cpu().numpy().reshape(-1)


def check_unit(sc: DecodeScenario, b: int, h: int, ks: float, vs: float):
    L, D, G = int(sc.lens[b]), sc.D, sc.Hq // sc.H
    k, v = sc.tokens(b)
    kb, vb = bits(k[:L, h:h + 1]), bits(v[:L, h:h + 1])
    used = -(-L // 16)
    okc, ovc = oracle.new_cache(sc.fmt, used, 1, D)
    oracle.write(sc.fmt, kb, vb, np.arange(L, dtype=np.int64), okc, ovc, ks, vs)
    # codes and block scales: bit for bit, page by page (bytes past the length
    # in the last page are compared too: both sides leave them zero)
    assert np.array_equal(device_pages(sc, b, h, "k"), okc), "K pages differ"
    assert np.array_equal(device_pages(sc, b, h, "v"), ovc), "V pages differ"
    q = bits(sc.q[b:b + 1, h * G:(h + 1) * G])
    ref_out, ref_lse = oracle.decode_attention(
        sc.fmt, q, okc, ovc, 1, np.arange(used, dtype=np.int32)[None], np.array([L], np.int32),
        ks, vs)
    out = sc.out[b, h * G:(h + 1) * G].cpu().numpy()
    lse = sc.lse[b, h * G:(h + 1) * G].cpu().numpy()
    e_out = np.abs(out - ref_out[0]).max()
    e_lse = (np.abs(lse - ref_lse[0]) / np.maximum(np.abs(ref_lse[0]), 1.0)).max()
    assert e_out <= OUT_ATOL, f"out error {e_out:.3e}"
    assert e_lse <= LSE_RTOL, f"lse error {e_lse:.3e}"
    return e_out, e_lse


@pytest.mark.parametrize("name,fmt,units", [
    ("fp8-paged-4x32k", "fp8", [(0, 0), (3, 7), (2, 4)]),
    ("nvfp4-1x64k", "nvfp4", [(0, 0), (0, 5)]),
    ("nvfp4-1x64k", "fp8", [(0, 3)]),
    ("nvfp4-1x64k", "bf16", [(0, 6)]),
    ("agents-fp8-4x127k", "fp8", [(1, 2), (3, 7)]),
])
def test_full_size_units(name, fmt, units):
    sc = DecodeScenario(wl.WORKLOADS[name], fmt=fmt)
    sc.step()  # the bench's step: write the step's tokens, then decode
    torch.cuda.synchronize()
    assert int(sc.err.item()) == 0
    ks, vs = oracle_scales(sc)
    got = sc.scales.cpu().numpy()
    if fmt != "bf16":
        assert got[0] == np.float32(ks) and got[1] == np.float32(vs), "scales differ"
    for b, h in units:
        check_unit(sc, b, h, ks, vs)


# Sweep cells (context x batch, lengths uniform in [L/2, L], GQA 8) at their
# full sizes, the byte-heavy corners included, built exactly as bench.py
# --sweep builds them; two sampled (sequence, KV head) units each.
@pytest.mark.parametrize("fmt,D,L,B,units", [
    ("fp8", 128, 131072, 8, [(0, 0), (7, 5)]),
    ("nvfp4", 128, 65536, 8, [(3, 2), (6, 7)]),
    ("nvfp4", 64, 65536, 32, [(0, 1), (31, 6)]),
    ("fp8", 64, 16384, 64, [(13, 3), (63, 0)]),
    ("bf16", 128, 16384, 32, [(5, 4)]),
    ("fp8", 128, 1024, 1, [(0, 0), (0, 7)]),
])
def test_full_size_sweep_cells(fmt, D, L, B, units):
    import dataclasses
    w = dataclasses.replace(wl.SWEEP, B=B, D=D, seq_len=L)
    lens = wl.varlen(wl.rng_for(wl.SWEEP_SEED, wl.sweep_cell_stream(L, B)), B, L)
    sc = DecodeScenario(w, fmt=fmt, lens=lens)
    sc.step()
    torch.cuda.synchronize()
    assert int(sc.err.item()) == 0
    ks, vs = oracle_scales(sc)
    got = sc.scales.cpu().numpy()
    if fmt != "bf16":
        assert got[0] == np.float32(ks) and got[1] == np.float32(vs), "scales differ"
    for b, h in units:
        check_unit(sc, b, h, ks, vs)
