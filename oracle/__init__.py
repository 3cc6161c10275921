"""CPU oracle for the quantized KV-cache decode path (test infrastructure).

This package is a plain, slow, obviously-correct CPU restatement of what the
library computes, used only to check it.  Only the tests, the smoke check and
the benchmark's CPU-baseline leg may import it; the product path never does,
and it never imports the product package.  The arithmetic lives in
``kvq_oracle.c`` (plain C, fp32 where the method fixes fp32, float64 for the
attention); this module is argument marshalling over numpy arrays.

Sources of each definition (cited by page title and section):
  * "FP8 KV calibration guide", paragraph on the Radiance calibrator: per-layer
    abs-max of BF16 K/V, OCP E4M3, scale = max(amax * 1.05 / 448, 1e-12).
  * "I Tested NVFP4 vs FP8 KV Cache on Blackwell", "What you'll learn": E4M3 at
    one byte per number; NVFP4 = block-scaled 4-bit float with FP8 block
    scales, 4.5 bits per number.
  * "FP8 KV calibration guide", paragraphs on the calibrator (Q maxima too)
    and on probability scales: the FP8-attention variant with E4M3 Q and P.
  * OCP 8-bit FP (E4M3) and OCP MX (E2M1) format definitions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.c")
_LIB = os.path.join(_HERE, "libkvq_oracle.so")

FORMATS = {"bf16": 0, "fp8": 1, "nvfp4": 2, "pq3": 3, "f32": 4}
PAGE = 16


def build(force: bool = False) -> str:
    """Compile the oracle with the host C compiler (strict IEEE: no fast-math,
    no FMA contraction, so fp32 steps round exactly as written)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-Wall", "-o", _LIB, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        f32, f64, i32, i64, u8, u16 = (ctypes.c_float, ctypes.c_double, ctypes.c_int,
                                       ctypes.c_int64, ctypes.c_uint8, ctypes.c_uint16)
        P = ctypes.c_void_p
        L.orc_e4m3_decode.restype = f32
        L.orc_e4m3_decode.argtypes = [u8]
        L.orc_e2m1_decode.restype = f32
        L.orc_e2m1_decode.argtypes = [u8]
        for name in ("orc_e4m3_encode", "orc_e4m3_encode_nearest", "orc_e2m1_encode",
                     "orc_e2m1_encode_nearest"):
            getattr(L, name).restype = u8
            getattr(L, name).argtypes = [f32]
        for name in ("orc_e4m3_encode_array", "orc_e2m1_encode_array"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [P, P, i64, i32]
        for name in ("orc_e4m3_decode_array", "orc_e2m1_decode_array"):
            getattr(L, name).restype = None
            getattr(L, name).argtypes = [P, P, i64]
        L.orc_absmax_bf16.restype = f32
        L.orc_absmax_bf16.argtypes = [P, i64]
        L.orc_fp8_scale.restype = f32
        L.orc_fp8_scale.argtypes = [f32]
        L.orc_nvfp4_global_scale.restype = f32
        L.orc_nvfp4_global_scale.argtypes = [f32]
        L.orc_head_page_bytes.restype = i64
        L.orc_head_page_bytes.argtypes = [i32, i32]
        L.orc_kv_bytes_per_token.restype = f64
        L.orc_kv_bytes_per_token.argtypes = [i32, i32, i32]
        L.orc_write.restype = i32
        L.orc_write.argtypes = [i32, P, P, i64, i32, i32, P, i64, P, P, f32, f32]
        L.orc_dequantize.restype = i32
        L.orc_dequantize.argtypes = [i32, P, P, i64, i32, i32, P, i64, f32, f32, P, P]
        L.orc_attention_range.restype = i32
        L.orc_attention_range.argtypes = [i32, P, P, P, i64, i32, i32, P, i32, i64, i64, f32,
                                          f32, f64, P, P, P]
        L.orc_decode_attention.restype = i32
        L.orc_decode_attention.argtypes = [i32, P, P, P, i64, i32, i32, P, i32, P, i32, i32,
                                           f32, f32, f64, P, i64, P, P]
        L.orc_decode_attention_window.restype = i32
        L.orc_decode_attention_window.argtypes = [i32, P, P, P, i64, i32, i32, P, i32, P, i32,
                                                  i32, f32, f32, f64, i32, P, i64, P, P]
        L.orc_merge.restype = None
        L.orc_prefill_attention.restype = i32
        L.orc_prefill_attention.argtypes = [i32, P, P, P, i64, i32, i32, P, i32, P, i32, i32,
                                            i32, f32, f32, f64, P, i64, P, P]
        L.orc_merge.argtypes = [i32, i32, P, P, P, P, P]
        L.orc_lloyd_max_gaussian.restype = None
        L.orc_lloyd_max_gaussian.argtypes = [i32, P]
        L.orc_pq3_codebook.restype = None
        L.orc_pq3_codebook.argtypes = [P]
        L.orc_pq3_encode_row.restype = None
        L.orc_pq3_encode_row.argtypes = [P, P, P, P]
        L.orc_pq3_decode_row.restype = None
        L.orc_pq3_decode_row.argtypes = [f32, P, P, P]
        L.orc_pq3_write.restype = i32
        L.orc_pq3_write.argtypes = [P, P, i64, i32, P, i64, P, P, P, P]
        L.orc_pq3_to_f32.restype = None
        L.orc_pq3_to_f32.argtypes = [P, P, i64, i32, P, P, P, P]
        L.orc_decode_attention_fp8qp.restype = i32
        L.orc_decode_attention_fp8qp.argtypes = [P, P, P, i64, i32, i32, P, i32, P, i32, i32,
                                                 f32, f32, f32, f32, f64, f64, P, i64, P, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# --------------------------------------------------------------------------- codecs

def e4m3_decode(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_e4m3_decode_array(_p(c), _p(out), c.size)
    return out


def e2m1_decode(codes) -> np.ndarray:
    c = _c(codes, np.uint8)
    out = np.empty(c.shape, np.float32)
    lib().orc_e2m1_decode_array(_p(c), _p(out), c.size)
    return out


def e4m3_encode(x, brute_force: bool = False) -> np.ndarray:
    a = _c(x, np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().orc_e4m3_encode_array(_p(a), _p(out), a.size, int(brute_force))
    return out


def e2m1_encode(x, brute_force: bool = False) -> np.ndarray:
    a = _c(x, np.float32)
    out = np.empty(a.shape, np.uint8)
    lib().orc_e2m1_encode_array(_p(a), _p(out), a.size, int(brute_force))
    return out


def bf16_to_f32(bits) -> np.ndarray:
    """Exact widening of BF16 bit patterns (uint16) to float32."""
    b = _c(bits, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------- scales

def absmax_bf16(x_bits) -> float:
    x = _c(x_bits, np.uint16)
    return float(lib().orc_absmax_bf16(_p(x), x.size))


def fp8_scale(amax: float) -> float:
    return float(np.float32(lib().orc_fp8_scale(float(np.float32(amax)))))


def nvfp4_global_scale(amax: float) -> float:
    return float(np.float32(lib().orc_nvfp4_global_scale(float(np.float32(amax)))))


def scale_from_absmax(fmt: str, amax: float) -> float:
    if fmt == "fp8":
        return fp8_scale(amax)
    if fmt == "nvfp4":
        return nvfp4_global_scale(amax)
    return 1.0


# --------------------------------------------------------------------------- cache

def head_page_bytes(fmt: str, D: int) -> int:
    return int(lib().orc_head_page_bytes(FORMATS[fmt], D))


def kv_bytes_per_token(fmt: str, H: int, D: int) -> float:
    return float(lib().orc_kv_bytes_per_token(FORMATS[fmt], H, D))


def new_cache(fmt: str, num_blocks: int, H: int, D: int, fill: int = 0):
    """A zero-filled (K, V) pair of byte buffers in the paged layout."""
    nbytes = num_blocks * H * head_page_bytes(fmt, D)
    return (np.full(nbytes, fill, np.uint8), np.full(nbytes, fill, np.uint8))


def write(fmt: str, k_bits, v_bits, slot_mapping, k_cache, v_cache, k_scale, v_scale) -> int:
    """Quantize-on-write of BF16 K/V rows ([T][H][D] uint16 bit patterns) into
    the caches at the given physical slots.  Returns 0, or -1 if a slot lay
    beyond the cache."""
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    T, H, D = k.shape
    sm = _c(slot_mapping, np.int64)
    nb = k_cache.size // (H * head_page_bytes(fmt, D))
    return int(lib().orc_write(FORMATS[fmt], _p(k), _p(v), T, H, D, _p(sm), nb, _p(k_cache),
                               _p(v_cache), float(k_scale), float(v_scale)))


def dequantize(fmt: str, k_cache, v_cache, H: int, D: int, slots, k_scale, v_scale):
    s = _c(slots, np.int64)
    nb = k_cache.size // (H * head_page_bytes(fmt, D))
    ko = np.empty((s.size, H, D), np.float32)
    vo = np.empty((s.size, H, D), np.float32)
    rc = lib().orc_dequantize(FORMATS[fmt], _p(k_cache), _p(v_cache), nb, H, D, _p(s), s.size,
                              float(k_scale), float(v_scale), _p(ko), _p(vo))
    if rc:
        raise ValueError("slot out of range")
    return ko, vo


def decode_attention(fmt: str, q_bits, k_cache, v_cache, H: int, block_table, seq_lens,
                     k_scale, v_scale, sm_scale=None, pairs=None, window=0):
    """Float64 decode attention.  q_bits: [B][Hq][D] BF16 bit patterns;
    block_table [B][max_blocks] int32; seq_lens [B] int32.  Returns
    (out [B][Hq][D], lse [B][Hq]) in float64.  With ``pairs`` (an [n][2] array
    of (b, j)), only those rows are computed and the rest are NaN.  With
    ``window`` > 0, sequence b attends only to its last ``window`` tokens (the
    sliding-window mode of the MI300X benchmark page, section "SWA mode")."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    bt = _c(block_table, np.int32)
    sl = _c(seq_lens, np.int32)
    nb = k_cache.size // (H * head_page_bytes(fmt, D))
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    if pairs is None:
        pp, npairs = None, 0
    else:
        pr = _c(pairs, np.int32).reshape(-1, 2)
        pp, npairs = _p(pr), pr.shape[0]
    rc = lib().orc_decode_attention_window(FORMATS[fmt], _p(q), _p(k_cache), _p(v_cache), nb,
                                           H, D, _p(bt), bt.shape[1], _p(sl), B, Hq,
                                           float(k_scale), float(v_scale), float(sm_scale),
                                           int(window), pp, npairs, _p(out), _p(lse))
    if rc:
        raise ValueError(f"oracle attention failed ({rc})")
    return out, lse


def prefill_attention(fmt: str, q_bits, k_cache, v_cache, H: int, block_table, seq_lens,
                      k_scale, v_scale, sm_scale=None, rows=None):
    """Float64 chunked-prefill attention.  q_bits: [B][Tq][Hq][D] BF16 bit
    patterns, the Tq newest tokens of each sequence; seq_lens [B] counts them.
    Query token i of sequence b (position seq_lens[b] - Tq + i) attends to the
    cache tokens up to and including its own position.  Returns (out
    [B][Tq][Hq][D], lse [B][Tq][Hq]) in float64; with ``rows`` (an [n][3]
    array of (b, i, j)) only those rows are computed and the rest are NaN."""
    q = _c(q_bits, np.uint16)
    B, Tq, Hq, D = q.shape
    bt = _c(block_table, np.int32)
    sl = _c(seq_lens, np.int32)
    nb = k_cache.size // (H * head_page_bytes(fmt, D))
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.full((B, Tq, Hq, D), np.nan)
    lse = np.full((B, Tq, Hq), np.nan)
    if rows is None:
        rp, nr = None, 0
    else:
        rr = _c(rows, np.int32).reshape(-1, 3)
        rp, nr = _p(rr), rr.shape[0]
    rc = lib().orc_prefill_attention(FORMATS[fmt], _p(q), _p(k_cache), _p(v_cache), nb, H, D,
                                     _p(bt), bt.shape[1], _p(sl), B, Tq, Hq, float(k_scale),
                                     float(v_scale), float(sm_scale), rp, nr, _p(out), _p(lse))
    if rc:
        raise ValueError(f"oracle prefill attention failed ({rc})")
    return out, lse


def attention_range(fmt: str, q_row_bits, k_cache, v_cache, H: int, D: int, bt_row, kv_head,
                    t0, t1, k_scale, v_scale, sm_scale):
    """Unnormalised partial attention over tokens [t0, t1): (o_unnorm, m, l)."""
    q = _c(q_row_bits, np.uint16)
    bt = _c(bt_row, np.int32)
    nb = k_cache.size // (H * head_page_bytes(fmt, D))
    o = np.empty(D, np.float64)
    m = ctypes.c_double()
    l = ctypes.c_double()
    rc = lib().orc_attention_range(FORMATS[fmt], _p(q), _p(k_cache), _p(v_cache), nb, H, D,
                                   _p(bt), int(kv_head), int(t0), int(t1), float(k_scale),
                                   float(v_scale), float(sm_scale), _p(o), ctypes.byref(m),
                                   ctypes.byref(l))
    if rc:
        raise ValueError("oracle attention_range failed")
    return o, m.value, l.value


def merge(o_parts, m_parts, l_parts):
    o = _c(o_parts, np.float64)
    m = _c(m_parts, np.float64)
    l = _c(l_parts, np.float64)
    n, D = o.shape
    out = np.empty(D, np.float64)
    lse = ctypes.c_double()
    lib().orc_merge(n, D, _p(o), _p(m), _p(l), _p(out), ctypes.byref(lse))
    return out, lse.value


def decode_attention_fp8qp(q_bits, k_cache, v_cache, H: int, block_table, seq_lens, k_scale,
                           v_scale, q_scale, prob_scale, sm_scale=None, pairs=None, eps=0.0):
    """Float64 decode attention with E4M3 Q and E4M3 P over an FP8 cache
    (orc_decode_attention_fp8qp): Q quantized with q_scale, P quantized page by
    page relative to the page's largest score with prob_scale.  Returns (out
    [B][Hq][D], lse [B][Hq], amb [B][Hq][D]); amb bounds how far each output
    can move if the P codes within relative ``eps`` of a rounding boundary
    took the other neighbour.  With ``pairs`` only those (b, j) rows are
    computed."""
    q = _c(q_bits, np.uint16)
    B, Hq, D = q.shape
    bt = _c(block_table, np.int32)
    sl = _c(seq_lens, np.int32)
    nb = k_cache.size // (H * head_page_bytes("fp8", D))
    if sm_scale is None:
        sm_scale = 1.0 / np.sqrt(D)
    out = np.full((B, Hq, D), np.nan)
    lse = np.full((B, Hq), np.nan)
    amb = np.full((B, Hq, D), np.nan)
    if pairs is None:
        pp, npairs = None, 0
    else:
        pr = _c(pairs, np.int32).reshape(-1, 2)
        pp, npairs = _p(pr), pr.shape[0]
    rc = lib().orc_decode_attention_fp8qp(_p(q), _p(k_cache), _p(v_cache), nb, H, D, _p(bt),
                                          bt.shape[1], _p(sl), B, Hq, float(k_scale),
                                          float(v_scale), float(q_scale), float(prob_scale),
                                          float(sm_scale), float(eps), pp, npairs, _p(out),
                                          _p(lse), _p(amb))
    if rc:
        raise ValueError(f"oracle fp8 q/p attention failed ({rc})")
    return out, lse, amb


# --------------------------------------------------------------------------- PQ3 codec
# The 3-bit planar-rotation codec of 128-element vectors ("AMD MI300X - KV
# Cache Compression Benchmark", "Key Results": 52-byte blocks, 4.923x against
# FP16); see kvq_oracle.c for the reading the oracle takes.
PQ3_D = 128
PQ3_PARAMS = 136  # 8 codebook values + 64 (cos, sin) pairs


def lloyd_max_gaussian(n: int) -> np.ndarray:
    """Centroids of the n-level Lloyd-Max quantizer of N(0, 1) (float64)."""
    c = np.empty(n, np.float64)
    lib().orc_lloyd_max_gaussian(n, _p(c))
    return c


def pq3_codebook() -> np.ndarray:
    cb = np.empty(8, np.float32)
    lib().orc_pq3_codebook(_p(cb))
    return cb


def pq3_params(cos_sin) -> np.ndarray:
    """The parameter block of one tensor: the codebook, then the 64 given
    (cos, sin) pairs (fp32)."""
    cs = _c(cos_sin, np.float32).reshape(64, 2)
    return np.concatenate([pq3_codebook(), cs.reshape(-1)]).astype(np.float32)


def pq3_encode_row(x_bits, params):
    """(norm, indices[128]) of one 128-element BF16 row."""
    x = _c(x_bits, np.uint16).reshape(PQ3_D)
    pr = _c(params, np.float32)
    nrm = np.empty(1, np.float32)
    idx = np.empty(PQ3_D, np.uint8)
    lib().orc_pq3_encode_row(_p(x), _p(pr), _p(nrm), _p(idx))
    return float(nrm[0]), idx


def pq3_decode_row(nrm, idx, params) -> np.ndarray:
    i = _c(idx, np.uint8).reshape(PQ3_D)
    pr = _c(params, np.float32)
    out = np.empty(PQ3_D, np.float32)
    lib().orc_pq3_decode_row(float(np.float32(nrm)), _p(i), _p(pr), _p(out))
    return out


def pq3_write(k_bits, v_bits, slot_mapping, k_cache, v_cache, k_params, v_params) -> int:
    """Quantize-on-write of BF16 K/V rows ([T][H][128]) into PQ3 caches (byte
    buffers of num_blocks * H * 832 bytes) at the given physical slots."""
    k = _c(k_bits, np.uint16)
    v = _c(v_bits, np.uint16)
    T, H, D = k.shape
    assert D == PQ3_D
    sm = _c(slot_mapping, np.int64)
    nb = k_cache.size // (H * head_page_bytes("pq3", D))
    kp, vp = _c(k_params, np.float32), _c(v_params, np.float32)
    return int(lib().orc_pq3_write(_p(k), _p(v), T, H, _p(sm), nb, _p(k_cache), _p(v_cache),
                                   _p(kp), _p(vp)))


def pq3_to_f32(k_cache, v_cache, H: int, k_params, v_params):
    """The dequantised caches in the "f32" format ([blocks][H][16][128] fp32,
    as byte buffers) the attention oracle reads."""
    nb = k_cache.size // (H * head_page_bytes("pq3", PQ3_D))
    ko = np.empty(nb * H * PAGE * PQ3_D, np.float32)
    vo = np.empty(nb * H * PAGE * PQ3_D, np.float32)
    kp, vp = _c(k_params, np.float32), _c(v_params, np.float32)
    lib().orc_pq3_to_f32(_p(k_cache), _p(v_cache), nb, H, _p(kp), _p(vp), _p(ko), _p(vo))
    return ko.view(np.uint8), vo.view(np.uint8)


def pq3_decode_attention(q_bits, k_cache, v_cache, H: int, block_table, seq_lens, k_params,
                         v_params, sm_scale=None, pairs=None, window=0):
    """Float64 decode attention over the dequantised PQ3 cache."""
    kf, vf = pq3_to_f32(k_cache, v_cache, H, k_params, v_params)
    return decode_attention("f32", q_bits, kf, vf, H, block_table, seq_lens, 1.0, 1.0,
                            sm_scale=sm_scale, pairs=pairs, window=window)
