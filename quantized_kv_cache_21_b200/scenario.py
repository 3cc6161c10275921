"""Device-resident decode workloads driven through the library's binding.

A ``DecodeScenario`` builds one layer's paged cache for a named workload
(seeded synthetic K/V, random block table, calibrated scales), then exposes the
per-step work of a decode step: quantize-on-write of the step's new tokens
(``write_chunk`` per sequence, through the block table) followed by the fused
decode attention over the whole context.  Everything runs in libkvq kernels;
torch only allocates memory and provides the stream and the RNG.
"""
from __future__ import annotations

import numpy as np
import torch

import quantized_kv_cache_21_b200 as kvq
from quantized_kv_cache_21_b200 import workloads as wl

BYTES_PER_ELEM = {"bf16": 2.0, "fp8": 1.0, "nvfp4": 4.5 / 8, "pq3": 52 / 128}


def kv_scan_bytes(fmt: str, lens, H: int, D: int) -> int:
    """Algorithmic bytes one decode step must read from the cache: every
    cached token's K and V for every KV head (NVFP4 block scales and PQ3
    norms included: 52 bytes per 128-element PQ3 vector)."""
    return int(round(sum(int(n) for n in lens) * H * 2 * D * BYTES_PER_ELEM[fmt]))


def prefill_flops(lens, chunk: int, Hq: int, D: int) -> int:
    """Algorithmic FLOPs of a chunked prefill: 2 D (QK) + 2 D (PV) per (query
    row, attended key).  The chunk is the last `chunk` tokens of each sequence;
    query i of a sequence of length n sits at position n - chunk + i and
    attends to n - chunk + i + 1 keys (none if that is not positive)."""
    keys = 0
    for n in lens:
        n = int(n)
        first = n - chunk + 1  # keys of the chunk's first query
        if first >= 1:
            keys += chunk * (first - 1) + chunk * (chunk + 1) // 2
        else:  # queries before the sequence start attend to nothing
            m = max(0, n)
            keys += m * (m + 1) // 2
    return 4 * D * Hq * keys


class DecodeScenario:
    def __init__(self, w: wl.Workload, fmt: str | None = None, device: str = "cuda",
                 seq_offset: int = 0, lens=None):
        """lens: optional per-sequence lengths (each in [chunk, seq_len]); by
        default every sequence holds seq_len tokens."""
        self.w = w
        self.fmt = fmt or w.fmt
        self.device = device
        B, H, Hq, D, L = w.B, w.Hkv, w.Hq, w.D, w.seq_len
        self.B, self.H, self.Hq, self.D, self.L = B, H, Hq, D, L
        self.chunk = max(1, w.write_chunk)
        self.mb = -(-L // wl.PAGE)
        self.num_blocks = B * self.mb
        rng = wl.rng_for(w.seed, 1)
        self.bt = (wl.permuted_block_table(rng, B, self.mb) if w.permuted
                   else wl.identity_block_table(B, self.mb))
        self.lens = (np.full(B, L, np.int32) if lens is None
                     else np.asarray(lens, dtype=np.int32).reshape(B))
        assert self.lens.max(initial=0) <= L and self.lens.min(initial=L) >= self.chunk
        self.out_k = wl.outliers_for(w, H, D, "k")
        self.out_v = wl.outliers_for(w, H, D, "v")
        self.seq_offset = seq_offset  # a rank's sequences draw distinct sub-streams
        dev = device

        self.cache = kvq.KVCache(self.fmt, self.num_blocks, H, D, device=dev)
        self.d_bt = torch.from_numpy(self.bt).to(dev)
        self.d_lens = torch.from_numpy(self.lens).to(dev)
        self.err = torch.zeros(1, dtype=torch.int32, device=dev)
        self.amax = torch.zeros(2, dtype=torch.float32, device=dev)
        self.scales = torch.ones(2, dtype=torch.float32, device=dev)
        self.d_ks, self.d_vs = self.scales[0:1], self.scales[1:2]

        # calibration: the first calib_tokens tokens of sequence 0, or all tokens
        # (PQ3 instead takes its codebook and a seeded planar rotation per tensor)
        if self.fmt == "pq3":
            self.d_ks = kvq.pq3_params(wl.planar_rotation(wl.rng_for(w.seed, 2)), dev)
            self.d_vs = kvq.pq3_params(wl.planar_rotation(wl.rng_for(w.seed, 3)), dev)
        elif self.fmt != "bf16":
            for b in range(B if w.calib_tokens is None else 1):
                k, v = self.tokens(b)
                n = int(self.lens[b]) if w.calib_tokens is None else w.calib_tokens
                kvq.kv_calibrate_absmax(k[:n].contiguous(), self.amax[0:1])
                kvq.kv_calibrate_absmax(v[:n].contiguous(), self.amax[1:2])
                del k, v
            kvq.kv_scale_from_absmax_device(self.fmt, self.amax[0:1], self.d_ks)
            kvq.kv_scale_from_absmax_device(self.fmt, self.amax[1:2], self.d_vs)

        # fill the context (all but the step's chunk), keep the chunk for the step
        step_k, step_v = [], []
        for b in range(B):
            k, v = self.tokens(b)
            n = int(self.lens[b])
            ctx = n - self.chunk
            if ctx > 0:
                slots = torch.from_numpy(wl.physical_slots(self.bt, b, np.arange(ctx))).to(dev)
                kvq.kv_quantize_write(self.fmt, k[:ctx], v[:ctx], slots, self.cache, self.d_ks,
                                      self.d_vs, self.err)
            step_k.append(k[ctx:n].clone())
            step_v.append(v[ctx:n].clone())
            del k, v
        self.step_k = torch.cat(step_k).contiguous()
        self.step_v = torch.cat(step_v).contiguous()
        # logical slots (seq * max_blocks * 16 + position) of the step's tokens,
        # translated through the block table inside the write kernel
        logical = np.concatenate([b * self.mb * wl.PAGE + np.arange(int(n) - self.chunk, int(n))
                                  for b, n in enumerate(self.lens)])
        self.step_slots = torch.from_numpy(logical.astype(np.int64)).to(dev)

        g = torch.Generator(device=dev)
        g.manual_seed(w.seed * 7919 + 17 + seq_offset)
        self.q = torch.randn((B, Hq, D), generator=g, device=dev).to(torch.bfloat16)
        self.out = torch.empty((B, Hq, D), dtype=torch.float32, device=dev)
        self.lse = torch.empty((B, Hq), dtype=torch.float32, device=dev)
        self.ws = kvq.new_workspace(
            kvq.kv_decode_workspace_size(self.fmt, B, Hq, H, D, L), device=dev)
        torch.cuda.synchronize()

    def tokens(self, b: int):
        """BF16 K and V ([L][H][D]) of sequence b (deterministic per workload)."""
        s = 2 * (b + self.seq_offset)
        k = wl.device_tokens(self.w.seed, s, self.L, self.H, self.D, self.out_k,
                             self.w.outlier_factor, self.device)
        v = wl.device_tokens(self.w.seed, s + 1, self.L, self.H, self.D, self.out_v,
                             self.w.outlier_factor, self.device)
        return k, v

    @property
    def scan_bytes(self) -> int:
        return kv_scan_bytes(self.fmt, self.lens, self.H, self.D)

    def write(self, stream=None, k=None, v=None):
        kvq.kv_quantize_write(self.fmt, self.step_k if k is None else k,
                              self.step_v if v is None else v, self.step_slots, self.cache,
                              self.d_ks, self.d_vs, self.err, block_table=self.d_bt,
                              stream=stream)

    def decode(self, stream=None, q=None, out=None, lse=None):
        kvq.kv_decode_attention(self.fmt, self.q if q is None else q, self.cache, self.d_bt,
                                self.d_lens, self.L, self.d_ks, self.d_vs,
                                self.out if out is None else out,
                                self.lse if lse is None else lse, self.ws, self.err,
                                stream=stream)

    def decode_window(self, window: int, stream=None, out=None, lse=None):
        """Sliding-window decode over each sequence's last ``window`` tokens
        (needs a workspace sized for the window: window_workspace())."""
        kvq.kv_decode_attention_window(self.fmt, self.q, self.cache, self.d_bt, self.d_lens,
                                       self.L, window, self.d_ks, self.d_vs,
                                       self.out if out is None else out,
                                       self.lse if lse is None else lse,
                                       self.window_ws(window), self.err, stream=stream)

    def window_ws(self, window: int):
        ws = getattr(self, "_wws", {})
        if window not in ws:
            ws[window] = kvq.new_workspace(kvq.kv_decode_workspace_size_window(
                self.fmt, self.B, self.Hq, self.H, self.D, self.L, window), device=self.device)
            self._wws = ws
        return ws[window]

    def window_scan_bytes(self, window: int) -> int:
        return kv_scan_bytes(self.fmt, np.minimum(self.lens, window), self.H, self.D)

    # ---- FP8 attention (E4M3 q and P) over the FP8 cache
    def fp8qp_setup(self):
        """Per-layer E4M3 scales of q (calibrated on the step's query with the
        library's abs-max and scale kernels) and of P (the same formula at an
        observed maximum of 1)."""
        if hasattr(self, "d_qs"):
            return
        assert self.fmt == "fp8", "FP8 attention runs on the FP8 cache"
        amax = torch.zeros(1, dtype=torch.float32, device=self.device)
        kvq.kv_calibrate_absmax(self.q.contiguous(), amax)
        self.d_qs = torch.empty(1, dtype=torch.float32, device=self.device)
        kvq.kv_scale_from_absmax_device("fp8", amax, self.d_qs)
        self.d_ps = torch.tensor([kvq.kv_scale_from_absmax("fp8", 1.0)], dtype=torch.float32,
                                 device=self.device)

    def decode_fp8qp(self, stream=None, out=None, lse=None):
        kvq.kv_decode_attention_fp8qp(self.q, self.cache, self.d_bt, self.d_lens, self.L,
                                      self.d_ks, self.d_vs, self.d_qs, self.d_ps,
                                      self.out if out is None else out,
                                      self.lse if lse is None else lse, self.ws, self.err,
                                      stream=stream)

    def step(self, stream=None):
        self.write(stream)
        self.decode(stream)

    # ---- chunked prefill: the step's chunk of new tokens attends to the cache
    def prefill_setup(self):
        """Seeded BF16 queries of the step's chunk ([B][chunk][Hq][D]) and their
        output buffers (created on first use)."""
        if hasattr(self, "q_chunk"):
            return
        B, Hq, D, dev = self.B, self.Hq, self.D, self.device
        g = torch.Generator(device=dev)
        g.manual_seed(self.w.seed * 7919 + 29 + self.seq_offset)
        self.q_chunk = torch.randn((B, self.chunk, Hq, D), generator=g,
                                   device=dev).to(torch.bfloat16)
        self.out_chunk = torch.empty((B, self.chunk, Hq, D), dtype=torch.float32, device=dev)
        self.lse_chunk = torch.empty((B, self.chunk, Hq), dtype=torch.float32, device=dev)

    def prefill(self, stream=None):
        """Attention of the chunk's queries over the cache (after write())."""
        kvq.kv_prefill_attention(self.fmt, self.q_chunk, self.cache, self.d_bt, self.d_lens,
                                 self.d_ks, self.d_vs, self.out_chunk, self.lse_chunk, self.err,
                                 stream=stream)

    @property
    def prefill_flops(self) -> int:
        """Algorithmic FLOPs of the chunk prefill (see prefill_flops)."""
        return prefill_flops(self.lens, self.chunk, self.Hq, self.D)
