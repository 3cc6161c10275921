"""kv_decode_attention_static_ws: the decode entry point that allocates
nothing, for callers that cannot allocate device memory where they run a
decode step (a fixed memory pool they must not bypass, no room for a
cudaMalloc's latency, no scratch handed to them).  It uses a fixed 8 MiB
scratch array built into the library instead of a caller workspace.

Checked through the C ABI against the float64 CPU oracle and against the
regular entry point (caller workspace) on two calls in a row, within the
attention tolerance the other parity tests use, and for its size limit.  This file is collected last so a
run that stops at the first failure has run every other test first."""
import ctypes

import numpy as np
import pytest
import torch

import quantized_kv_cache_21_b200 as kvq

from gpu_common import (DEV, LSE_RTOL, OUT_ATOL, Case, assert_attention_close, new_err,
                        to_dev_bits)

pytestmark = pytest.mark.gpu

KVQ_ERR_WORKSPACE = 3


def call_static(c: Case, out, lse, err):
    """The new entry point, called through the C ABI with raw pointers."""
    L = kvq.lib()
    P = ctypes.c_void_p
    return L.kv_decode_attention_static_ws(
        kvq.FORMATS[c.fmt], P(c.d_q.data_ptr()), c.cache.c, P(c.d_bt.data_ptr()), c.max_blocks,
        P(c.d_lens.data_ptr()), c.B, c.Hq, c.max_blocks * 16, 0, P(c.d_ks.data_ptr()),
        P(c.d_vs.data_ptr()), ctypes.c_float(0.0), P(out.data_ptr()), P(lse.data_ptr()),
        P(err.data_ptr()), P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("fmt,D,lens", [("fp8", 128, [5000, 17, 2049]),
                                        ("nvfp4", 64, [1, 3000, 700, 64])])
def test_static_scratch_matches_caller_workspace(fmt, D, lens):
    c = Case(fmt, len(lens), 2, 16, D, lens, seed=9100 + D, factor=16.0)
    # this problem does use scratch on the regular path
    assert kvq.kv_decode_workspace_size(fmt, c.B, c.Hq, c.Hkv, D, c.max_blocks * 16) > 0
    ref_out, ref_lse = c.decode()  # regular entry point, caller workspace
    assert int(c.err.item()) == 0
    ora_out, ora_lse = c.reference()  # the CPU oracle, float64
    for _ in range(2):  # two calls in a row share the one built-in array
        out = torch.full((c.B, c.Hq, D), float("nan"), device=DEV)
        lse = torch.full((c.B, c.Hq), float("nan"), device=DEV)
        err = new_err()
        assert call_static(c, out, lse, err) == 0, kvq.lib().kvq_last_error()
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        o, l = out.cpu().numpy(), lse.cpu().numpy()
        # the float64 oracle first, then the regular entry point
        assert_attention_close(o, l, ora_out, ora_lse)
        assert np.abs(o - ref_out).max() <= OUT_ATOL
        assert (np.abs(l - ref_lse) / np.maximum(np.abs(ref_lse), 1.0)).max() <= LSE_RTOL


def test_static_scratch_rejects_oversized_problems():
    # 256 sequences x 8 KV heads of one page each need ~8.9 MB of workspace
    B, Hkv, Hq, D = 256, 8, 64, 128
    cache = kvq.KVCache("fp8", B, Hkv, D)
    assert kvq.kv_decode_workspace_size("fp8", B, Hq, Hkv, D, 16) > 8 << 20
    q = to_dev_bits(np.zeros((B, Hq, D), np.uint16))
    bt = torch.arange(B, dtype=torch.int32, device=DEV).reshape(B, 1)
    lens = torch.full((B,), 16, dtype=torch.int32, device=DEV)
    one = torch.ones(1, dtype=torch.float32, device=DEV)
    out = torch.full((B, Hq, D), 7.0, device=DEV)
    err = new_err()
    L = kvq.lib()
    P = ctypes.c_void_p
    st = L.kv_decode_attention_static_ws(
        kvq.FORMATS["fp8"], P(q.data_ptr()), cache.c, P(bt.data_ptr()), 1, P(lens.data_ptr()), B,
        Hq, 16, 0, P(one.data_ptr()), P(one.data_ptr()), ctypes.c_float(0.0), P(out.data_ptr()),
        None, P(err.data_ptr()), P(torch.cuda.current_stream().cuda_stream))
    assert st == KVQ_ERR_WORKSPACE
    assert b"built-in scratch" in L.kvq_last_error()
    torch.cuda.synchronize()
    assert bool((out == 7.0).all())  # nothing was launched
