"""The C-ABI library: it builds for sm_100a, loads, exports every function the
public header declares, and its pure host functions agree with the oracle.
No kernel is launched here (no GPU needed)."""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+char\s*\*|kvq_status)\s+(\w+)\s*\(", text, flags=re.M)


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kvq.lib()


def test_header_symbols_are_exported(L):
    names = header_functions()
    assert len(names) >= 10
    assert set(names) == set(kvq.EXPORTS)
    for n in names:
        assert hasattr(L, n), n
    # the oracle is not linked into the product library
    assert not hasattr(ctypes.CDLL(kbuild.LIB), "orc_e4m3_encode")


def test_library_is_sm100a_only():
    # the fatbin carries sm_100a SASS only: nvcc was asked for that gencode
    assert kbuild.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(L):
    assert L.kvq_status_string(0) == b"ok"
    assert b"invalid" in L.kvq_status_string(1)


def test_cache_bytes_match_oracle_layout(L):
    for fmt in ("bf16", "fp8", "nvfp4"):
        for D in (64, 128):
            got = kvq.kv_cache_bytes(fmt, 37, 3, D)
            assert got == 37 * 3 * oracle.head_page_bytes(fmt, D)
    with pytest.raises(kvq.KvqError):
        kvq.kv_cache_bytes("fp8", 4, 2, 96)
    with pytest.raises(kvq.KvqError):
        kvq.kv_cache_bytes(7, 4, 2, 64)


def test_host_scale_matches_oracle_bit_exact(L):
    rng = np.random.default_rng(0)
    amax = np.concatenate([[0.0, 1e-15, 1e-9, 1.0, 448.0, 2688.0, 72.25],
                           rng.lognormal(0, 4, 2000)]).astype(np.float32)
    for a in amax:
        assert np.float32(kvq.kv_scale_from_absmax("fp8", a)) == np.float32(oracle.fp8_scale(a))
        assert (np.float32(kvq.kv_scale_from_absmax("nvfp4", a))
                == np.float32(oracle.nvfp4_global_scale(a)))
        assert kvq.kv_scale_from_absmax("bf16", a) == 1.0
    for bad in (-1.0, float("nan"), float("inf")):
        with pytest.raises(kvq.KvqError):
            kvq.kv_scale_from_absmax("fp8", bad)


def test_prefill_argument_checks_run_on_the_host(L):
    """kv_prefill_attention validates its arguments before touching the device:
    these calls return their status codes on a machine without a GPU (the cache
    pointers are never dereferenced)."""
    fake = 1 << 20  # 256-byte aligned, never dereferenced
    cache = kvq._Cache(kvq.FORMATS["fp8"], 16, 8, 2, 64, fake, fake)
    cp = ctypes.byref(cache)

    def call(B=1, Tq=4, Hq=8, q=fake, out=fake, bt=fake, lens=fake, ks=fake, vs=fake, fmt=1):
        return L.kv_prefill_attention(fmt, q, cp, bt, 4, lens, B, Tq, Hq, ks, vs, 0.0, out, None,
                                      None, None)

    assert call(Hq=3) == 1                  # not a multiple of the 2 KV heads
    assert call(Hq=2 * 129) == 2            # 129 query heads per KV head
    assert call(B=-1) == 1
    assert call(Tq=-1) == 1
    assert call(Tq=0) == 0                  # an empty chunk launches nothing
    assert call(B=0) == 0
    assert call(q=None) == 1
    assert call(q=fake + 8) == 1            # q not 16-byte aligned
    assert call(out=fake + 4) == 1
    assert call(bt=None) == 1
    assert call(ks=None) == 1               # quantized formats need both scales
    assert call(fmt=2) == 1                 # cache format differs from fmt


def test_header_is_plain_c99_and_links(L, tmp_path):
    """include/kvq.h compiles as C99 with warnings as errors (no CUDA or C++
    headers needed) and a C program links against libkvq.so and calls its
    host functions."""
    import shutil
    import subprocess

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(
        '#include <stdio.h>\n#include "kvq.h"\n'
        "int main(void) {\n"
        "  float s = 0.f; int64_t n = 0;\n"
        "  kvq_status a = kv_scale_from_absmax(KVQ_FMT_FP8_E4M3, 448.0f, &s);\n"
        "  kvq_status b = kv_cache_bytes(KVQ_FMT_NVFP4, 37, 3, 128, &n);\n"
        '  printf("%d %a %d %lld\\n", (int)a, (double)s, (int)b, (long long)n);\n'
        "  return 0;\n}\n")
    exe = tmp_path / "abi"
    libdir = os.path.dirname(kbuild.LIB)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I",
                    os.path.join(ROOT, "include"), str(src), "-L", libdir, "-lkvq",
                    f"-Wl,-rpath,{libdir}", "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert out[0] == "0" and out[2] == "0"
    assert float.fromhex(out[1]) == float(np.float32(oracle.fp8_scale(448.0)))
    assert int(out[3]) == 37 * 3 * oracle.head_page_bytes("nvfp4", 128)


def test_pq3_codebook_matches_the_oracle(L):
    """The library's own Lloyd-Max solver gives the oracle's codebook, bit for
    bit (8 ascending f16-representable values)."""
    import numpy as np
    cb = np.array(kvq.kv_pq3_codebook(), np.float32)
    assert np.array_equal(cb, oracle.pq3_codebook())
    assert np.array_equal(cb, cb.astype(np.float16).astype(np.float32))
    with pytest.raises(kvq.KvqError, match="PQ3"):
        kvq.kv_scale_from_absmax("pq3", 1.0)
    assert kvq.kv_cache_bytes("pq3", 3, 2, 128) == 3 * 2 * 832
    with pytest.raises(kvq.KvqError, match="head_dim 128"):
        kvq.kv_cache_bytes("pq3", 3, 2, 64)
