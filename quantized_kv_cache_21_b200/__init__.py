"""Quantized KV-cache decode attention for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libkvq.so`` (declared in
``include/kvq.h``): the functions below have the same names as the C entry
points and only marshal arguments (torch tensors -> device pointers, the
current CUDA stream).  Every step of the computation runs in the library's
CUDA kernels; there is no Python or CPU fallback, and importing the compute
functions without the built library raises.

Formats: ``"bf16"``, ``"fp8"`` (OCP E4M3 with a per-layer fp32 scale),
``"nvfp4"`` (16-element E2M1 blocks along head_dim, E4M3 block scales and an
fp32 per-tensor scale; 4.5 bits per element) and ``"pq3"`` (3-bit
planar-rotation codec of 128-element vectors, 52 bytes each; its "scale" is a
136-float parameter block, see ``pq3_params``).
"""
from __future__ import annotations

import ctypes
import os

import torch

from .build import LIB as _LIB_PATH

FORMATS = {"bf16": 0, "fp8": 1, "nvfp4": 2, "pq3": 3}
BLOCK_SIZE = 16

DERR_BLOCK_ID = 0x1
DERR_SLOT = 0x2
DERR_SCALE = 0x4
DERR_SEQ_LEN = 0x8
DERR_TIMEOUT = 0x10

EXPORTS = ("kvq_status_string", "kvq_last_error", "kv_cache_bytes", "kv_scale_from_absmax",
           "kv_pq3_codebook",
           "kv_scale_from_absmax_device", "kv_calibrate_absmax", "kv_quantize_write",
           "kv_decode_workspace_size", "kv_decode_attention", "kv_decode_attention_static_ws",
           "kv_decode_attention_window", "kv_decode_workspace_size_window",
           "kv_decode_attention_fp8qp",
           "kv_prefill_attention", "kv_dequantize", "kvq_selftest_bounded_wait")


class KvqError(RuntimeError):
    pass


class _Cache(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_blocks", ctypes.c_int64), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libkvq.so from this package directory (built by build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise KvqError(f"{_LIB_PATH} is missing; run `python -m quantized_kv_cache_21_b200.build`")
        L = ctypes.CDLL(_LIB_PATH)
        i32, i64, f32, P, sz = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p,
                                ctypes.c_size_t)
        CP = ctypes.POINTER(_Cache)
        L.kvq_status_string.restype = ctypes.c_char_p
        L.kvq_status_string.argtypes = [ctypes.c_int]
        L.kvq_last_error.restype = ctypes.c_char_p
        L.kvq_last_error.argtypes = []
        sigs = {
            "kv_cache_bytes": [i32, i64, i32, i32, ctypes.POINTER(i64)],
            "kv_scale_from_absmax": [i32, f32, ctypes.POINTER(f32)],
            "kv_pq3_codebook": [P],
            "kv_scale_from_absmax_device": [i32, P, P, P],
            "kv_calibrate_absmax": [P, i64, P, P],
            "kv_quantize_write": [i32, P, P, i64, P, P, i32, i32, CP, P, P, P, P],
            "kv_decode_workspace_size": [i32, i32, i32, i32, i32, i32, i32, ctypes.POINTER(sz)],
            "kv_decode_attention": [i32, P, CP, P, i32, P, i32, i32, i32, i32, P, P, f32, P, P,
                                    P, sz, P, P],
            "kv_decode_attention_static_ws": [i32, P, CP, P, i32, P, i32, i32, i32, i32, P, P,
                                              f32, P, P, P, P],
            "kv_decode_attention_window": [i32, P, CP, P, i32, P, i32, i32, i32, i32, i32, P, P,
                                           f32, P, P, P, sz, P, P],
            "kv_decode_workspace_size_window": [i32, i32, i32, i32, i32, i32, i32, i32,
                                                ctypes.POINTER(sz)],
            "kv_decode_attention_fp8qp": [P, CP, P, i32, P, i32, i32, i32, i32, P, P, P, P, f32,
                                          P, P, P, sz, P, P],
            "kv_prefill_attention": [i32, P, CP, P, i32, P, i32, i32, i32, P, P, f32, P, P, P,
                                     P],
            "kv_dequantize": [i32, CP, P, i64, P, P, P, P, P, P],
            "kvq_selftest_bounded_wait": [P, i32, P],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.restype = ctypes.c_int
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int) -> None:
    if status != 0:
        L = lib()
        raise KvqError(f"{L.kvq_status_string(status).decode()}: {L.kvq_last_error().decode()}")


def _fmt(fmt) -> int:
    return FORMATS[fmt] if isinstance(fmt, str) else int(fmt)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream=None) -> int:
    """The CUDA stream handle to launch on: the given torch stream, else the
    current one (read without building a torch.cuda.Stream object)."""
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


class KVCache:
    """One layer's paged K/V cache: two device byte buffers in the layout of
    include/kvq.h, sized by their compressed bytes."""

    def __init__(self, fmt, num_blocks: int, num_kv_heads: int, head_dim: int,
                 device="cuda", k: torch.Tensor | None = None, v: torch.Tensor | None = None):
        self.fmt = _fmt(fmt)
        self.num_blocks, self.num_kv_heads, self.head_dim = num_blocks, num_kv_heads, head_dim
        nbytes = kv_cache_bytes(self.fmt, num_blocks, num_kv_heads, head_dim)
        self.k = k if k is not None else torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self.v = v if v is not None else torch.zeros(nbytes, dtype=torch.uint8, device=device)
        self._c = _Cache(self.fmt, BLOCK_SIZE, num_blocks, num_kv_heads, head_dim,
                         self.k.data_ptr(), self.v.data_ptr())

    @property
    def c(self):
        return ctypes.byref(self._c)

    @property
    def nbytes(self) -> int:
        return self.k.numel() + self.v.numel()


def kv_cache_bytes(fmt, num_blocks: int, num_kv_heads: int, head_dim: int) -> int:
    out = ctypes.c_int64()
    _check(lib().kv_cache_bytes(_fmt(fmt), num_blocks, num_kv_heads, head_dim, ctypes.byref(out)))
    return out.value


def kv_scale_from_absmax(fmt, amax: float) -> float:
    out = ctypes.c_float()
    _check(lib().kv_scale_from_absmax(_fmt(fmt), float(amax), ctypes.byref(out)))
    return out.value


def kv_pq3_codebook() -> list:
    """The PQ3 codebook (8 ascending f16-representable values, see include/kvq.h)."""
    out = (ctypes.c_float * 8)()
    _check(lib().kv_pq3_codebook(ctypes.cast(out, ctypes.c_void_p)))
    return list(out)


def pq3_params(cos_sin, device="cuda") -> torch.Tensor:
    """The 136-float PQ3 parameter block of one tensor on the device: the
    codebook, then the 64 (cos, sin) pairs of its planar rotation."""
    rot = torch.as_tensor(cos_sin, dtype=torch.float32).reshape(-1)
    assert rot.numel() == 128
    cb = torch.tensor(kv_pq3_codebook(), dtype=torch.float32)
    return torch.cat([cb, rot]).to(device)


def kv_scale_from_absmax_device(fmt, d_amax: torch.Tensor, d_scale: torch.Tensor, stream=None):
    _check(lib().kv_scale_from_absmax_device(_fmt(fmt), _ptr(d_amax), _ptr(d_scale),
                                             _stream(stream)))


def kv_calibrate_absmax(x: torch.Tensor, d_amax: torch.Tensor, stream=None):
    """Max-accumulate max|x| of a BF16 tensor into the fp32 device scalar d_amax."""
    assert x.dtype == torch.bfloat16 and x.is_contiguous()
    _check(lib().kv_calibrate_absmax(_ptr(x), x.numel(), _ptr(d_amax), _stream(stream)))


def kv_quantize_write(fmt, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                      cache: KVCache, k_scale: torch.Tensor | None, v_scale: torch.Tensor | None,
                      d_err: torch.Tensor | None = None, block_table: torch.Tensor | None = None,
                      stream=None):
    """k, v: BF16 [T][Hkv][D].  slot_mapping: int64 [T] physical slots, or with
    block_table ([B][max_blocks] int32) logical slots seq*max_blocks*16 + pos."""
    assert k.dtype == torch.bfloat16 and v.dtype == torch.bfloat16
    assert slot_mapping.dtype == torch.int64
    T = k.shape[0]
    B, MB = (block_table.shape[0], block_table.shape[1]) if block_table is not None else (0, 0)
    _check(lib().kv_quantize_write(_fmt(fmt), _ptr(k), _ptr(v), T, _ptr(slot_mapping),
                                   _ptr(block_table), B, MB, cache.c, _ptr(k_scale),
                                   _ptr(v_scale), _ptr(d_err), _stream(stream)))


def kv_decode_workspace_size(fmt, num_seqs: int, num_q_heads: int, num_kv_heads: int,
                             head_dim: int, max_seq_len: int, num_splits: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(lib().kv_decode_workspace_size(_fmt(fmt), num_seqs, num_q_heads, num_kv_heads,
                                          head_dim, max_seq_len, num_splits, ctypes.byref(out)))
    return out.value


def new_workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled workspace (the counters it holds must start at zero)."""
    return torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)


def kv_decode_attention(fmt, q: torch.Tensor, cache: KVCache, block_table: torch.Tensor,
                        seq_lens: torch.Tensor, max_seq_len: int, k_scale, v_scale,
                        out: torch.Tensor, lse: torch.Tensor | None, workspace: torch.Tensor | None,
                        d_err: torch.Tensor | None = None, sm_scale: float = 0.0,
                        num_splits: int = 0, stream=None):
    """q: BF16 [B][Hq][D]; block_table int32 [B][max_blocks]; seq_lens int32 [B];
    out fp32 [B][Hq][D]; lse fp32 [B][Hq] or None."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous()
    assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
    assert out.dtype == torch.float32
    B, Hq, _ = q.shape
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib().kv_decode_attention(_fmt(fmt), _ptr(q), cache.c, _ptr(block_table),
                                     block_table.shape[1], _ptr(seq_lens), B, Hq, max_seq_len,
                                     num_splits, _ptr(k_scale), _ptr(v_scale), float(sm_scale),
                                     _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _ptr(d_err),
                                     _stream(stream)))


def kv_decode_attention_static_ws(fmt, q: torch.Tensor, cache: KVCache,
                                  block_table: torch.Tensor, seq_lens: torch.Tensor,
                                  max_seq_len: int, k_scale, v_scale, out: torch.Tensor,
                                  lse: torch.Tensor | None, d_err: torch.Tensor | None = None,
                                  sm_scale: float = 0.0, num_splits: int = 0, stream=None):
    """kv_decode_attention with the library's built-in scratch instead of a
    caller workspace, for callers that cannot allocate device memory at the
    call (see include/kvq.h).  Calls on one device share that scratch: keep
    them ordered on one stream."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous()
    assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
    assert out.dtype == torch.float32
    B, Hq, _ = q.shape
    _check(lib().kv_decode_attention_static_ws(_fmt(fmt), _ptr(q), cache.c, _ptr(block_table),
                                               block_table.shape[1], _ptr(seq_lens), B, Hq,
                                               max_seq_len, num_splits, _ptr(k_scale),
                                               _ptr(v_scale), float(sm_scale), _ptr(out),
                                               _ptr(lse), _ptr(d_err), _stream(stream)))


def kv_decode_workspace_size_window(fmt, num_seqs: int, num_q_heads: int, num_kv_heads: int,
                                    head_dim: int, max_seq_len: int, window: int,
                                    num_splits: int = 0) -> int:
    out = ctypes.c_size_t()
    _check(lib().kv_decode_workspace_size_window(_fmt(fmt), num_seqs, num_q_heads, num_kv_heads,
                                                 head_dim, max_seq_len, window, num_splits,
                                                 ctypes.byref(out)))
    return out.value


def kv_decode_attention_window(fmt, q: torch.Tensor, cache: KVCache, block_table: torch.Tensor,
                               seq_lens: torch.Tensor, max_seq_len: int, window: int, k_scale,
                               v_scale, out: torch.Tensor, lse: torch.Tensor | None,
                               workspace: torch.Tensor | None, d_err: torch.Tensor | None = None,
                               sm_scale: float = 0.0, num_splits: int = 0, stream=None):
    """kv_decode_attention over each sequence's last ``window`` tokens only
    (sliding-window mode; see include/kvq.h)."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous()
    assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
    assert out.dtype == torch.float32
    B, Hq, _ = q.shape
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib().kv_decode_attention_window(_fmt(fmt), _ptr(q), cache.c, _ptr(block_table),
                                            block_table.shape[1], _ptr(seq_lens), B, Hq,
                                            max_seq_len, window, num_splits, _ptr(k_scale),
                                            _ptr(v_scale), float(sm_scale), _ptr(out), _ptr(lse),
                                            _ptr(workspace), ws_bytes, _ptr(d_err),
                                            _stream(stream)))


def kv_decode_attention_fp8qp(q: torch.Tensor, cache: KVCache, block_table: torch.Tensor,
                              seq_lens: torch.Tensor, max_seq_len: int, k_scale, v_scale,
                              q_scale, prob_scale, out: torch.Tensor, lse: torch.Tensor | None,
                              workspace: torch.Tensor | None, d_err: torch.Tensor | None = None,
                              sm_scale: float = 0.0, num_splits: int = 0, stream=None):
    """FP8 attention over an FP8 cache: q and the softmax probabilities in
    E4M3 too (q_scale, prob_scale: device fp32 scalars; see include/kvq.h).
    Shapes and the workspace as kv_decode_attention with the "fp8" format."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous()
    assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
    assert out.dtype == torch.float32
    B, Hq, _ = q.shape
    ws_bytes = workspace.numel() if workspace is not None else 0
    _check(lib().kv_decode_attention_fp8qp(_ptr(q), cache.c, _ptr(block_table),
                                           block_table.shape[1], _ptr(seq_lens), B, Hq,
                                           max_seq_len, num_splits, _ptr(k_scale), _ptr(v_scale),
                                           _ptr(q_scale), _ptr(prob_scale), float(sm_scale),
                                           _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes,
                                           _ptr(d_err), _stream(stream)))


def kv_prefill_attention(fmt, q: torch.Tensor, cache: KVCache, block_table: torch.Tensor,
                         seq_lens: torch.Tensor, k_scale, v_scale, out: torch.Tensor,
                         lse: torch.Tensor | None, d_err: torch.Tensor | None = None,
                         sm_scale: float = 0.0, stream=None):
    """Chunked-prefill attention (see include/kvq.h).  q: BF16 [B][Tq][Hq][D],
    the Tq newest tokens of each sequence, already in the cache; seq_lens int32
    [B] counts them; out fp32 [B][Tq][Hq][D]; lse fp32 [B][Tq][Hq] or None."""
    assert q.dtype == torch.bfloat16 and q.is_contiguous() and q.dim() == 4
    assert block_table.dtype == torch.int32 and seq_lens.dtype == torch.int32
    assert out.dtype == torch.float32 and out.is_contiguous()
    B, Tq, Hq, _ = q.shape
    _check(lib().kv_prefill_attention(_fmt(fmt), _ptr(q), cache.c, _ptr(block_table),
                                      block_table.shape[1], _ptr(seq_lens), B, Tq, Hq,
                                      _ptr(k_scale), _ptr(v_scale), float(sm_scale), _ptr(out),
                                      _ptr(lse), _ptr(d_err), _stream(stream)))


def kv_dequantize(fmt, cache: KVCache, slots: torch.Tensor, k_scale, v_scale,
                  k_out: torch.Tensor, v_out: torch.Tensor, d_err: torch.Tensor | None = None,
                  stream=None):
    assert slots.dtype == torch.int64
    _check(lib().kv_dequantize(_fmt(fmt), cache.c, _ptr(slots), slots.numel(), _ptr(k_scale),
                               _ptr(v_scale), _ptr(k_out), _ptr(v_out), _ptr(d_err),
                               _stream(stream)))


def kvq_selftest_bounded_wait(d_err: torch.Tensor, arrive: bool, stream=None):
    """Run the bounded-wait self-test (see include/kvq.h): arrive=False makes
    the wait run out (about 2 s) and set DERR_TIMEOUT in d_err."""
    assert d_err.dtype == torch.int32
    _check(lib().kvq_selftest_bounded_wait(_ptr(d_err), int(bool(arrive)), _stream(stream)))
