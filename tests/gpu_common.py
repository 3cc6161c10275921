"""Shared helpers of the GPU parity tests: move seeded inputs to the device,
run the library through its binding, and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl

DEV = "cuda"
OUT_ATOL = 2e-3   # max-abs error on attention outputs (fp32 vs float64 oracle)
LSE_RTOL = 1e-5   # relative error on the log-sum-exp, relative to max(|lse|, 1)


def to_dev_bits(bits: np.ndarray, dtype=torch.bfloat16) -> torch.Tensor:
    """uint16 BF16 bit patterns -> a device bf16 tensor with the same bits."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(DEV).view(dtype)


def dev_scalar(x: float) -> torch.Tensor:
    return torch.tensor([x], dtype=torch.float32, device=DEV)


def new_err() -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def cache_bytes(cache: kvq.KVCache):
    torch.cuda.synchronize()
    return cache.k.cpu().numpy(), cache.v.cpu().numpy()


class Case:
    """A decode problem: BF16 K/V written into both a GPU cache (by the
    library) and an oracle cache (by the oracle), plus the query."""

    def __init__(self, fmt, B, Hkv, Hq, D, lens, seed, permuted=True, factor=8.0,
                 outliers_per_head=1, extra_blocks=3, fill=0, calib_tokens=None, zero_k=False):
        """zero_k: K is all zeros (its abs-max is 0, so the NVFP4 global scale
        g is 0 and every score is 0)."""
        rng = wl.rng_for(seed, 0)
        self.fmt, self.B, self.Hkv, self.Hq, self.D = fmt, B, Hkv, Hq, D
        self.lens = np.array(lens, np.int32)
        self.max_blocks = max(1, -(-int(self.lens.max(initial=0)) // 16))
        self.num_blocks = B * self.max_blocks + extra_blocks
        if permuted:
            self.bt = wl.permuted_block_table(wl.rng_for(seed, 1), B, self.max_blocks,
                                              self.num_blocks)
        else:
            self.bt = wl.identity_block_table(B, self.max_blocks)
        outl = wl.outlier_pairs(rng, Hkv, D, per_head=outliers_per_head) if factor != 1 else []
        self.k = [wl.make_tokens(rng, int(n), Hkv, D, outl, factor) for n in self.lens]
        if zero_k:
            self.k = [np.zeros_like(k) for k in self.k]
        self.v = [wl.make_tokens(rng, int(n), Hkv, D, outl, factor) for n in self.lens]
        self.q = wl.make_query(rng, B, Hq, D)
        kc = np.concatenate(self.k) if self.k else np.zeros((0, Hkv, D), np.uint16)
        vc = np.concatenate(self.v) if self.v else np.zeros((0, Hkv, D), np.uint16)
        if calib_tokens is not None:
            kc, vc = kc[:calib_tokens], vc[:calib_tokens]
        self.ks = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(kc)) if kc.size else 1.0
        self.vs = oracle.scale_from_absmax(fmt, oracle.absmax_bf16(vc)) if vc.size else 1.0
        # oracle cache
        self.okc, self.ovc = oracle.new_cache(fmt, self.num_blocks, Hkv, D, fill=fill)
        for b in range(B):
            slots = wl.physical_slots(self.bt, b, np.arange(self.lens[b]))
            oracle.write(fmt, self.k[b], self.v[b], slots, self.okc, self.ovc, self.ks, self.vs)
        # GPU cache, written by the library from the same BF16 inputs
        self.cache = kvq.KVCache(fmt, self.num_blocks, Hkv, D)
        if fill:
            self.cache.k.fill_(fill)
            self.cache.v.fill_(fill)
        self.d_ks, self.d_vs = dev_scalar(self.ks), dev_scalar(self.vs)
        self.err = new_err()
        for b in range(B):
            if self.lens[b] == 0:
                continue
            slots = torch.from_numpy(wl.physical_slots(self.bt, b, np.arange(self.lens[b]))).to(DEV)
            kvq.kv_quantize_write(fmt, to_dev_bits(self.k[b]), to_dev_bits(self.v[b]), slots,
                                  self.cache, self.d_ks, self.d_vs, self.err)
        self.d_q = to_dev_bits(self.q)
        self.d_bt = torch.from_numpy(self.bt).to(DEV)
        self.d_lens = torch.from_numpy(self.lens).to(DEV)

    def decode(self, num_splits=0, max_seq_len=None, sm_scale=0.0, err=None):
        msl = int(self.max_blocks * 16 if max_seq_len is None else max_seq_len)
        ws = kvq.new_workspace(kvq.kv_decode_workspace_size(self.fmt, self.B, self.Hq, self.Hkv,
                                                            self.D, msl, num_splits))
        out = torch.full((self.B, self.Hq, self.D), float("nan"), device=DEV)
        lse = torch.full((self.B, self.Hq), float("nan"), device=DEV)
        kvq.kv_decode_attention(self.fmt, self.d_q, self.cache, self.d_bt, self.d_lens, msl,
                                self.d_ks, self.d_vs, out, lse, ws,
                                err if err is not None else self.err, sm_scale, num_splits)
        torch.cuda.synchronize()
        return out.cpu().numpy(), lse.cpu().numpy()

    def reference(self, sm_scale=None, pairs=None):
        return oracle.decode_attention(self.fmt, self.q, self.okc, self.ovc, self.Hkv, self.bt,
                                       self.lens, self.ks, self.vs, sm_scale, pairs)


def assert_attention_close(out, lse, ref_out, ref_lse, atol=OUT_ATOL, rtol=LSE_RTOL):
    """out within atol (max-abs) and lse within rtol (relative) of the oracle;
    empty sequences must give exactly 0 and -inf."""
    empty = np.isneginf(ref_lse)
    assert np.all(np.isneginf(lse[empty])), "lse of empty rows must be -inf"
    assert np.all(out[empty] == 0), "out of empty rows must be 0"
    ok = ~empty
    err_out = np.abs(out[ok] - ref_out[ok]).max(initial=0.0)
    err_lse = (np.abs(lse[ok] - ref_lse[ok]) / np.maximum(np.abs(ref_lse[ok]), 1.0)).max(
        initial=0.0)
    assert np.all(np.isfinite(out[ok])) and np.all(np.isfinite(lse[ok]))
    assert err_out <= atol, f"out max-abs error {err_out:.3e} > {atol}"
    assert err_lse <= rtol, f"lse relative error {err_lse:.3e} > {rtol}"
    return err_out, err_lse
