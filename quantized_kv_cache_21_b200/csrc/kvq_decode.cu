// kvq_decode.cu -- decode-step attention over the paged, quantized KV cache
// with the dequantisation fused into the scan.
//
// What it computes: for every sequence b and query head j (KV head
// j / (Hq/Hkv)), softmax(sm_scale * q . k_hat_t) . v_hat_t over the cached
// tokens, and the log-sum-exp of the scaled scores.  Quantized formats are
// those of "I Tested NVFP4 vs FP8 KV Cache on Blackwell" ("What you'll learn":
// E4M3 one byte per number; NVFP4 block-scaled E2M1, 4.5 bits per number) and
// the FP8 KV calibration guide's per-layer E4M3 scale.  That page's chapter
// "The Missing Fused Dequant Kernel" is the reason the dequantisation lives
// inside this scan: the codes are read once from HBM and decoded in
// registers, so the step time follows the compressed bytes.
//
// Design (one launch per decode step):
//   * Work = the virtual page space units x pmax, where a unit is (sequence,
//     KV head, group of <= 8 query heads) and pmax = ceil(max_seq_len / 16)
//     (plus some empty pages at each unit's end when units straddle CTAs, so
//     a CTA whose range holds a unit boundary scans fewer pages).
//     It is cut evenly over persistent CTAs (one per SM), so every SM streams
//     the same number of pages whatever the batch shape (stream-K style); a
//     CTA walks its range unit by unit ("segments").
//   * Each of the CTA's warps takes every NW-th page of that range and streams
//     it through its own ring of shared-memory stages: the warp issues one TMA
//     tensor copy per K/V tile (plus the NVFP4 block scales) into a stage,
//     completion tracked by that stage's mbarrier, and refills the stage as
//     soon as its contents are in registers.  Block ids are gathered 32 pages
//     ahead (one coalesced load per 32 pages).  Tiles are 128/64/32-byte
//     swizzled so the fragment reads are bank-conflict free.  A warp only
//     waits on barriers of its own stages, one phase at a time.
//   * The G (<= 8) query heads sharing a KV head make QK^T and PV small
//     contractions, run on tensor cores with mma.sync m16n8k16 and fp32
//     accumulation: S^T[16 tokens][8 heads] = K_codes . Q^T, then
//     O^T[16 dims][8 heads] += V_codes^T . P^T.  Codes are decoded exactly
//     into f16 (E4M3, and E2M1 x E4M3 block scale) with packed cvt
//     instructions; BF16 pages feed the bf16 MMA directly.  The per-layer
//     scale (FP8 s, NVFP4 g) is folded into the softmax scale for K and into
//     the final normalisation for V, so no dequantised value is ever rounded.
//   * P is split into a 16-bit high part and a 16-bit residual (two MMAs) so
//     the probabilities keep ~22 bits: rounding P to one 16-bit value would
//     cost up to 2^-11 relative on outputs whose V reaches hundreds.
//   * Online softmax in the exp2 domain per warp (rescale skipped when no
//     running max moved).  At a segment end the consumer warps merge through
//     shared memory; a unit split over several CTAs is merged by the last of
//     them to arrive (atomic ticket, nobody waits), which writes out and lse.
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
// P is fed to the MMA as p * 2^kPLog2 (computed directly as 2^(s - m + 12)),
// so small probabilities stay clear of the f16 subnormals; l and O carry the
// same factor.  A warp's running max m lags the true max by at most
// kRescaleGap (log2 units): p <= 2^3, P <= 2^15 < 65504, the largest f16.
constexpr float kPLog2 = 12.0f;
constexpr float kRescaleGap = 3.0f;
constexpr float kETop = kPLog2 + kRescaleGap;  // e = s - m + kPLog2 above this moves m

// --------------------------------------------------------------------------
// Per-(format, head_dim) fragment layouts.
//
// Fragment mapping used by every format (lane = 4*gid + tig):
//   QK: A = K tile (rows = 16 tokens, k = head_dim), B = Q^T (n = 8 heads).
//       Thread (gid, tig) supplies tokens gid and gid+8 and D/4 head-dim
//       elements k_elem(tig, i); k-step s uses elements 4s..4s+3 of that list
//       (the same list indexes Q, so the contraction is over all of D).
//   PV: A = V^T tile (rows = 16 head-dim elements, k = 16 tokens),
//       B = P^T (n = 8 heads).  Thread supplies tokens 2tig, 2tig+1, 2tig+8,
//       2tig+9 and D/8 elements v_elem(gid, i); m-tile j uses elements 2j
//       (row gid) and 2j+1 (row gid+8).
// Stage layout: K tile(s), V tile(s) [, K block scales, V block scales], each
// at an offset aligned to its swizzle repeat.
// --------------------------------------------------------------------------
template <int FMT, int D>
struct Fmt;

// ---- FP8 E4M3, head_dim 128: rows of 128 B, 128-byte swizzle.
template <>
struct Fmt<1, 128> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 4096, TX = 4096, V_OFF = 2048;
  __device__ static int k_elem(int tig, int i) { return 32 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 16 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap*, const CUtensorMap*,
                               int h, int blk, const DecodeParams&) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void prefetch(const CUtensorMap* mk, const CUtensorMap* mv, int h, int blk,
                                  const DecodeParams&) {
    tma_prefetch_l2_4d(mk, 0, 0, h, blk);
    tma_prefetch_l2_4d(mv, 0, 0, h, blk);
  }
  // Raw stage words of this thread: K rows gid, gid+8 (32 codes each), V
  // rows 2tig, 2tig+1, 2tig+8, 2tig+9 (16 codes each).
  struct Raw {
    uint4 k[4], v[4];
  };
  static constexpr bool kLateV = false;
  static constexpr bool kStream = false;
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = gid + 8 * rr;
      r.k[2 * rr] = lds128(st + swz128(row, 32 * tig));
      r.k[2 * rr + 1] = lds128(st + swz128(row, 32 * tig + 16));
    }
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
    const uint8_t* sv = st + V_OFF;
    r.v[0] = lds128(sv + swz128(2 * tig, 16 * gid));
    r.v[1] = lds128(sv + swz128(2 * tig + 1, 16 * gid));
    r.v[2] = lds128(sv + swz128(2 * tig + 8, 16 * gid));
    r.v[3] = lds128(sv + swz128(2 * tig + 9, 16 * gid));
  }
  __device__ static void conv_k(const Raw& r, uint32_t ka[8][4]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint4 a = r.k[2 * rr], c = r.k[2 * rr + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) e4m3x4_to_f16x2x2(w[s], ka[s][rr], ka[s][2 + rr]);
    }
  }
  __device__ static void conv_v(const Raw& r, uint32_t va[8][4]) {
    const uint4 X = r.v[0], Y = r.v[1], Z = r.v[2], W = r.v[3];
    const uint32_t x[4] = {X.x, X.y, X.z, X.w}, y[4] = {Y.x, Y.y, Y.z, Y.w};
    const uint32_t z[4] = {Z.x, Z.y, Z.z, Z.w}, w[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
    for (int wi = 0; wi < 4; ++wi) {
      e4m3x4_to_f16x2x2(prmt(x[wi], y[wi], 0x5140), va[2 * wi][0], va[2 * wi][1]);
      e4m3x4_to_f16x2x2(prmt(z[wi], w[wi], 0x5140), va[2 * wi][2], va[2 * wi][3]);
      e4m3x4_to_f16x2x2(prmt(x[wi], y[wi], 0x7362), va[2 * wi + 1][0], va[2 * wi + 1][1]);
      e4m3x4_to_f16x2x2(prmt(z[wi], w[wi], 0x7362), va[2 * wi + 1][2], va[2 * wi + 1][3]);
    }
  }
};

// ---- FP8 E4M3, head_dim 64: rows of 64 B, 64-byte swizzle.
template <>
struct Fmt<1, 64> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 2048, TX = 2048, V_OFF = 1024;
  __device__ static int k_elem(int tig, int i) { return 16 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 8 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap*, const CUtensorMap*,
                               int h, int blk, const DecodeParams&) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void prefetch(const CUtensorMap* mk, const CUtensorMap* mv, int h, int blk,
                                  const DecodeParams&) {
    tma_prefetch_l2_4d(mk, 0, 0, h, blk);
    tma_prefetch_l2_4d(mv, 0, 0, h, blk);
  }
  struct Raw {
    uint4 k[2];
    uint2 v[4];
  };
  static constexpr bool kLateV = false;
  static constexpr bool kStream = false;
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) r.k[rr] = lds128(st + swz64(gid + 8 * rr, 16 * tig));
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
    const uint8_t* sv = st + V_OFF;
    r.v[0] = lds64(sv + swz64(2 * tig, 8 * gid));
    r.v[1] = lds64(sv + swz64(2 * tig + 1, 8 * gid));
    r.v[2] = lds64(sv + swz64(2 * tig + 8, 8 * gid));
    r.v[3] = lds64(sv + swz64(2 * tig + 9, 8 * gid));
  }
  __device__ static void conv_k(const Raw& r, uint32_t ka[4][4]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint4 a = r.k[rr];
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) e4m3x4_to_f16x2x2(w[s], ka[s][rr], ka[s][2 + rr]);
    }
  }
  __device__ static void conv_v(const Raw& r, uint32_t va[4][4]) {
    const uint2 X = r.v[0], Y = r.v[1], Z = r.v[2], W = r.v[3];
    const uint32_t x[2] = {X.x, X.y}, y[2] = {Y.x, Y.y}, z[2] = {Z.x, Z.y}, w[2] = {W.x, W.y};
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
      e4m3x4_to_f16x2x2(prmt(x[wi], y[wi], 0x5140), va[2 * wi][0], va[2 * wi][1]);
      e4m3x4_to_f16x2x2(prmt(z[wi], w[wi], 0x5140), va[2 * wi][2], va[2 * wi][3]);
      e4m3x4_to_f16x2x2(prmt(x[wi], y[wi], 0x7362), va[2 * wi + 1][0], va[2 * wi + 1][1]);
      e4m3x4_to_f16x2x2(prmt(z[wi], w[wi], 0x7362), va[2 * wi + 1][2], va[2 * wi + 1][3]);
    }
  }
};

// ---- BF16, head_dim 64: rows of 128 B, 128-byte swizzle; no decode needed.
template <>
struct Fmt<0, 64> {
  static constexpr bool kBF16 = true;
  static constexpr int STAGE = 4096, TX = 4096, V_OFF = 2048;
  __device__ static int k_elem(int tig, int i) { return 16 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 8 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap*, const CUtensorMap*,
                               int h, int blk, const DecodeParams&) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void prefetch(const CUtensorMap* mk, const CUtensorMap* mv, int h, int blk,
                                  const DecodeParams&) {
    tma_prefetch_l2_4d(mk, 0, 0, h, blk);
    tma_prefetch_l2_4d(mv, 0, 0, h, blk);
  }
  struct Raw {
    uint4 k[4], v[4];
  };
  static constexpr bool kLateV = false;
  static constexpr bool kStream = false;
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = gid + 8 * rr;
      r.k[2 * rr] = lds128(st + swz128(row, 32 * tig));
      r.k[2 * rr + 1] = lds128(st + swz128(row, 32 * tig + 16));
    }
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
    const uint8_t* sv = st + V_OFF;
    r.v[0] = lds128(sv + swz128(2 * tig, 16 * gid));
    r.v[1] = lds128(sv + swz128(2 * tig + 1, 16 * gid));
    r.v[2] = lds128(sv + swz128(2 * tig + 8, 16 * gid));
    r.v[3] = lds128(sv + swz128(2 * tig + 9, 16 * gid));
  }
  __device__ static void conv_k(const Raw& r, uint32_t ka[4][4]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint4 a = r.k[2 * rr], c = r.k[2 * rr + 1];
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        ka[s][rr] = w[2 * s];
        ka[s][2 + rr] = w[2 * s + 1];
      }
    }
  }
  __device__ static void conv_v(const Raw& r, uint32_t va[4][4]) {
    const uint4 X = r.v[0], Y = r.v[1], Z = r.v[2], W = r.v[3];
    const uint32_t x[4] = {X.x, X.y, X.z, X.w}, y[4] = {Y.x, Y.y, Y.z, Y.w};
    const uint32_t z[4] = {Z.x, Z.y, Z.z, Z.w}, w[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][0] = prmt(x[j], y[j], 0x5410);
      va[j][1] = prmt(x[j], y[j], 0x7632);
      va[j][2] = prmt(z[j], w[j], 0x5410);
      va[j][3] = prmt(z[j], w[j], 0x7632);
    }
  }
};

// ---- BF16, head_dim 128: two 64-element half tiles, each 128-byte swizzled.
template <>
struct Fmt<0, 128> {
  static constexpr bool kBF16 = true;
  static constexpr int STAGE = 8192, TX = 8192, V_OFF = 4096;
  __device__ static int k_elem(int tig, int i) {
    return i < 16 ? 16 * tig + i : 64 + 16 * tig + (i - 16);
  }
  __device__ static int v_elem(int gid, int i) {
    return i < 8 ? 8 * gid + i : 64 + 8 * gid + (i - 8);
  }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap*, const CUtensorMap*,
                               int h, int blk, const DecodeParams&) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + 2048, mk, bar, 64, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF + 2048, mv, bar, 64, 0, h, blk);
  }
  __device__ static void prefetch(const CUtensorMap* mk, const CUtensorMap* mv, int h, int blk,
                                  const DecodeParams&) {
    tma_prefetch_l2_4d(mk, 0, 0, h, blk);
    tma_prefetch_l2_4d(mk, 64, 0, h, blk);
    tma_prefetch_l2_4d(mv, 0, 0, h, blk);
    tma_prefetch_l2_4d(mv, 64, 0, h, blk);
  }
  struct Raw {
    uint4 k[8], v[8];
  };
  // 64 raw registers would not fit beside the accumulators: K is read and
  // used first, V read after the QK product (kLateV), then the stage refilled.
  static constexpr bool kLateV = true;
  static constexpr bool kStream = false;
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const int row = gid + 8 * rr;
        r.k[4 * hf + 2 * rr] = lds128(st + 2048 * hf + swz128(row, 32 * tig));
        r.k[4 * hf + 2 * rr + 1] = lds128(st + 2048 * hf + swz128(row, 32 * tig + 16));
      }
    }
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint8_t* sv = st + V_OFF + 2048 * hf;
      r.v[4 * hf] = lds128(sv + swz128(2 * tig, 16 * gid));
      r.v[4 * hf + 1] = lds128(sv + swz128(2 * tig + 1, 16 * gid));
      r.v[4 * hf + 2] = lds128(sv + swz128(2 * tig + 8, 16 * gid));
      r.v[4 * hf + 3] = lds128(sv + swz128(2 * tig + 9, 16 * gid));
    }
  }
  __device__ static void conv_k(const Raw& r, uint32_t ka[8][4]) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint4 a = r.k[4 * hf + 2 * rr], c = r.k[4 * hf + 2 * rr + 1];
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          ka[4 * hf + s][rr] = w[2 * s];
          ka[4 * hf + s][2 + rr] = w[2 * s + 1];
        }
      }
    }
  }
  __device__ static void conv_v(const Raw& r, uint32_t va[8][4]) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint4 X = r.v[4 * hf], Y = r.v[4 * hf + 1], Z = r.v[4 * hf + 2], W = r.v[4 * hf + 3];
      const uint32_t x[4] = {X.x, X.y, X.z, X.w}, y[4] = {Y.x, Y.y, Y.z, Y.w};
      const uint32_t z[4] = {Z.x, Z.y, Z.z, Z.w}, w[4] = {W.x, W.y, W.z, W.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        va[4 * hf + j][0] = prmt(x[j], y[j], 0x5410);
        va[4 * hf + j][1] = prmt(x[j], y[j], 0x7632);
        va[4 * hf + j][2] = prmt(z[j], w[j], 0x5410);
        va[4 * hf + j][3] = prmt(z[j], w[j], 0x7632);
      }
    }
  }
};

// Interleave the E2M1 nibbles of two tokens: byte j of lo = (x_j low nibble,
// y_j low nibble), byte j of hi = (x_j high nibble, y_j high nibble).
__device__ __forceinline__ void nib_interleave(uint32_t x, uint32_t y, uint32_t& lo,
                                               uint32_t& hi) {
  lo = (x & 0x0F0F0F0Fu) | ((y << 4) & 0xF0F0F0F0u);
  hi = ((x >> 4) & 0x0F0F0F0Fu) | (y & 0xF0F0F0F0u);
}

// f16x2 pair (scale of token a, scale of token b) from two E4M3 bytes.
__device__ __forceinline__ uint32_t scale_pair(uint32_t sa, uint32_t sb) {
  uint32_t lo, hi;
  e4m3x4_to_f16x2x2(sa | (sb << 8), lo, hi);
  return lo;
}

// ---- NVFP4, head_dim 64: a head page is 18 rows of 32 B, 16 code rows
// (32-byte swizzle) then 2 rows of block scales (4 per token), fetched as one
// box; the swizzle leaves rows 16-17 in place, so scales sit at byte 512.
template <>
struct Fmt<2, 64> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 1536, TX = 1152, V_OFF = 768, KSF = 512, VSF = V_OFF + 512;
  __device__ static int k_elem(int tig, int i) { return 16 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 8 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap*, const CUtensorMap*,
                               int h, int blk, const DecodeParams&) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void prefetch(const CUtensorMap* mk, const CUtensorMap* mv, int h, int blk,
                                  const DecodeParams&) {
    tma_prefetch_l2_4d(mk, 0, 0, h, blk);
    tma_prefetch_l2_4d(mv, 0, 0, h, blk);
  }
  // Raw stage words: K code rows gid, gid+8 (16 codes each) and their block
  // scale (block tig); V code rows 2tig, 2tig+1, 2tig+8, 2tig+9 (8 codes
  // each, block gid/2) and the four scales.
  struct Raw {
    uint2 k[2];
    uint32_t v[4], ks[2], vs[4];
  };
  static constexpr bool kLateV = false;
  static constexpr bool kStream = false;
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = gid + 8 * rr;
      r.k[rr] = lds64(st + swz32(row, 8 * tig));
      r.ks[rr] = st[KSF + row * 4 + tig];
    }
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
    const uint8_t* sv = st + V_OFF;
    const uint8_t* ss = st + VSF;
    const int t0 = 2 * tig, t2 = 2 * tig + 8, blk = gid >> 1;
    r.v[0] = lds32(sv + swz32(t0, 4 * gid));
    r.v[1] = lds32(sv + swz32(t0 + 1, 4 * gid));
    r.v[2] = lds32(sv + swz32(t2, 4 * gid));
    r.v[3] = lds32(sv + swz32(t2 + 1, 4 * gid));
    r.vs[0] = ss[t0 * 4 + blk];
    r.vs[1] = ss[(t0 + 1) * 4 + blk];
    r.vs[2] = ss[t2 * 4 + blk];
    r.vs[3] = ss[(t2 + 1) * 4 + blk];
  }
  __device__ static void conv_k(const Raw& r, uint32_t ka[4][4]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const uint32_t sc = scale_pair(r.ks[rr], r.ks[rr]);
      uint32_t f[8];
      e2m1x8_to_f16x2x4(r.k[rr].x, f);
      e2m1x8_to_f16x2x4(r.k[rr].y, f + 4);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        ka[s][rr] = hmul2(f[2 * s], sc);
        ka[s][2 + rr] = hmul2(f[2 * s + 1], sc);
      }
    }
  }
  __device__ static void conv_v(const Raw& r, uint32_t va[4][4]) {
    const uint32_t sxy = scale_pair(r.vs[0], r.vs[1]);
    const uint32_t szw = scale_pair(r.vs[2], r.vs[3]);
    uint32_t lo, hi, L[4], H[4];
    nib_interleave(r.v[0], r.v[1], lo, hi);
    e2m1x8_to_f16x2x4(lo, L);
    e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][0] = hmul2(L[j], sxy);
      va[j][1] = hmul2(H[j], sxy);
    }
    nib_interleave(r.v[2], r.v[3], lo, hi);
    e2m1x8_to_f16x2x4(lo, L);
    e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][2] = hmul2(L[j], szw);
      va[j][3] = hmul2(H[j], szw);
    }
  }
};

// ---- NVFP4, head_dim 128: 18 rows of 64 B per head page, 16 code rows
// (64-byte swizzle) then 2 scale rows (8 per token), one box; the scales stay
// in place at byte 1024.  V starts at the next 512-byte swizzle repeat.
template <>
struct Fmt<2, 128> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 3072, TX = 2304, V_OFF = 1536, KSF = 1024, VSF = V_OFF + 1024;
  __device__ static int k_elem(int tig, int i) { return 32 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 16 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap*, const CUtensorMap*,
                               int h, int blk, const DecodeParams&) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void prefetch(const CUtensorMap* mk, const CUtensorMap* mv, int h, int blk,
                                  const DecodeParams&) {
    tma_prefetch_l2_4d(mk, 0, 0, h, blk);
    tma_prefetch_l2_4d(mv, 0, 0, h, blk);
  }
  // Raw stage words: K code rows gid, gid+8 (32 codes each) with their two
  // block scales (blocks 2tig, 2tig+1, one 16-bit load); V code rows 2tig,
  // 2tig+1, 2tig+8, 2tig+9 (16 codes each, block gid) and the four scales.
  struct Raw {
    uint4 k[2];
    uint2 v[4];
    uint32_t ks[2], vs[4];
  };
  static constexpr bool kLateV = false;
  // K decoded per pair of k-steps right at its MMAs and V four m-tiles at a
  // time after the softmax, so no whole page of fragments is live at once
  // (154 registers instead of 164; the 4 x 126,976-token decode 180 -> 174 us)
  static constexpr bool kStream = true;
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = gid + 8 * rr;
      r.k[rr] = lds128(st + swz64(row, 16 * tig));
      r.ks[rr] = *reinterpret_cast<const uint16_t*>(st + KSF + row * 8 + 2 * tig);
    }
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
    const uint8_t* sv = st + V_OFF;
    const uint8_t* ss = st + VSF;
    const int t0 = 2 * tig, t2 = 2 * tig + 8;
    r.v[0] = lds64(sv + swz64(t0, 8 * gid));
    r.v[1] = lds64(sv + swz64(t0 + 1, 8 * gid));
    r.v[2] = lds64(sv + swz64(t2, 8 * gid));
    r.v[3] = lds64(sv + swz64(t2 + 1, 8 * gid));
    r.vs[0] = ss[t0 * 8 + gid];
    r.vs[1] = ss[(t0 + 1) * 8 + gid];
    r.vs[2] = ss[t2 * 8 + gid];
    r.vs[3] = ss[(t2 + 1) * 8 + gid];
  }
  __device__ static void conv_k(const Raw& r, uint32_t ka[8][4]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      uint32_t s01, unused;
      e4m3x4_to_f16x2x2(r.ks[rr], s01, unused);  // (scale of block 2tig, of 2tig+1)
      const uint32_t sc0 = prmt(s01, s01, 0x1010), sc1 = prmt(s01, s01, 0x3232);
      const uint4 c = r.k[rr];
      uint32_t f[16];
      e2m1x8_to_f16x2x4(c.x, f);
      e2m1x8_to_f16x2x4(c.y, f + 4);
      e2m1x8_to_f16x2x4(c.z, f + 8);
      e2m1x8_to_f16x2x4(c.w, f + 12);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t sc = s < 4 ? sc0 : sc1;
        ka[s][rr] = hmul2(f[2 * s], sc);
        ka[s][2 + rr] = hmul2(f[2 * s + 1], sc);
      }
    }
  }
  // k-steps 2w and 2w+1 only: code word w of both rows (blocks 2tig for
  // w < 2, 2tig+1 after), the same values conv_k puts in ka[2w], ka[2w+1]
  __device__ static void conv_k_pair(const Raw& r, int w, uint32_t a0[4], uint32_t a1[4]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      uint32_t s01, unused;
      e4m3x4_to_f16x2x2(r.ks[rr], s01, unused);
      const uint32_t sc = w < 2 ? prmt(s01, s01, 0x1010) : prmt(s01, s01, 0x3232);
      const uint4 c = r.k[rr];
      const uint32_t word = w == 0 ? c.x : w == 1 ? c.y : w == 2 ? c.z : c.w;
      uint32_t f[4];
      e2m1x8_to_f16x2x4(word, f);
      a0[rr] = hmul2(f[0], sc);
      a0[2 + rr] = hmul2(f[1], sc);
      a1[rr] = hmul2(f[2], sc);
      a1[2 + rr] = hmul2(f[3], sc);
    }
  }
  // m-tiles 4wi .. 4wi+3 only: the values conv_v puts in va[4wi .. 4wi+3]
  __device__ static void conv_v_half(const Raw& r, int wi, uint32_t va[4][4]) {
    const uint32_t sxy = scale_pair(r.vs[0], r.vs[1]);
    const uint32_t szw = scale_pair(r.vs[2], r.vs[3]);
    const uint32_t x = wi ? r.v[0].y : r.v[0].x, y = wi ? r.v[1].y : r.v[1].x;
    const uint32_t z = wi ? r.v[2].y : r.v[2].x, w = wi ? r.v[3].y : r.v[3].x;
    uint32_t lo, hi, L[4], H[4];
    nib_interleave(x, y, lo, hi);
    e2m1x8_to_f16x2x4(lo, L);
    e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][0] = hmul2(L[j], sxy);
      va[j][1] = hmul2(H[j], sxy);
    }
    nib_interleave(z, w, lo, hi);
    e2m1x8_to_f16x2x4(lo, L);
    e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][2] = hmul2(L[j], szw);
      va[j][3] = hmul2(H[j], szw);
    }
  }
  __device__ static void conv_v(const Raw& r, uint32_t va[8][4]) {
    const uint32_t sxy = scale_pair(r.vs[0], r.vs[1]);
    const uint32_t szw = scale_pair(r.vs[2], r.vs[3]);
    const uint32_t x[2] = {r.v[0].x, r.v[0].y}, y[2] = {r.v[1].x, r.v[1].y};
    const uint32_t z[2] = {r.v[2].x, r.v[2].y}, w[2] = {r.v[3].x, r.v[3].y};
#pragma unroll
    for (int wi = 0; wi < 2; ++wi) {
      uint32_t lo, hi, L[4], H[4];
      nib_interleave(x[wi], y[wi], lo, hi);
      e2m1x8_to_f16x2x4(lo, L);
      e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        va[4 * wi + j][0] = hmul2(L[j], sxy);
        va[4 * wi + j][1] = hmul2(H[j], sxy);
      }
      nib_interleave(z[wi], w[wi], lo, hi);
      e2m1x8_to_f16x2x4(lo, L);
      e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        va[4 * wi + j][2] = hmul2(L[j], szw);
        va[4 * wi + j][3] = hmul2(H[j], szw);
      }
    }
  }
};

// ---- PQ3 (3-bit planar-rotation codec of 128-element vectors), head_dim 128:
// a head page is 16 fp32 norms and 16 rows of 48 index bytes (832 B), fetched
// whole by bulk copies, K's page then V's.  A row is two bit planes: 8 words
// of the indices' low 2 bits (word w: index 16w + k at bits 4k, 4k+1 and
// 16w + 8 + k at bits 4k+2, 4k+3) and 4 words of their high bits (word v:
// index 32v + 8j + k at bit 4k + (2, 3, 0, 1)[j]).  Two masks and an OR turn
// a low word and its high bits into 8 byte-permute selectors (one index a
// nibble); two permutes over the codebook's low and high bytes (tl, th) then
// give four exact f16 codebook values.
template <>
struct Fmt<3, 128> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 1664, TX = 1664, V_OFF = 832, PAGE = 832;
  static constexpr bool kLateV = false;
  static constexpr bool kStream = false;
  __device__ static int k_elem(int tig, int i) { return 32 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 16 * gid + i; }
  __device__ static const uint8_t* page(const uint8_t* base, const DecodeParams& p, int h,
                                        int blk) {
    return base + (static_cast<size_t>(blk) * p.Hkv + h) * PAGE;
  }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap*, const CUtensorMap*,
                               const CUtensorMap*, const CUtensorMap*, int h, int blk,
                               const DecodeParams& p) {
    mbar_arrive_expect_tx(bar, TX);
    bulk_load(st, page(p.kc, p, h, blk), PAGE, bar);
    bulk_load(st + V_OFF, page(p.vc, p, h, blk), PAGE, bar);
  }
  __device__ static void prefetch(const CUtensorMap*, const CUtensorMap*, int h, int blk,
                                  const DecodeParams& p) {
    bulk_prefetch_l2(page(p.kc, p, h, blk), PAGE);
    bulk_prefetch_l2(page(p.vc, p, h, blk), PAGE);
  }
  // Raw stage words: K rows gid, gid+8 (low words 2tig, 2tig+1 and high word
  // tig: indices of head-dim elements 32tig .. 32tig+31) and their norms; V
  // rows 2tig, 2tig+1, 2tig+8, 2tig+9 (low word gid and high word gid / 2:
  // elements 16gid .. 16gid+15) and the V norms of tokens gid, gid+8 (the
  // token rows of P).
  struct Raw {
    uint2 kl[2];
    uint32_t kh[2], vl[4], vh[4];
    float nk[2], nv[2];
  };
  __device__ static void load_raw_k(const uint8_t* st, int gid, int tig, Raw& r) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      const int row = gid + 8 * rr;
      const uint8_t* rw = st + 64 + 48 * row;
      r.kl[rr] = *reinterpret_cast<const uint2*>(rw + 8 * tig);
      r.kh[rr] = *reinterpret_cast<const uint32_t*>(rw + 32 + 4 * tig);
      r.nk[rr] = reinterpret_cast<const float*>(st)[row];
    }
  }
  __device__ static void load_raw_v(const uint8_t* st, int gid, int tig, Raw& r) {
    const uint8_t* sv = st + V_OFF;
    const int rows[4] = {2 * tig, 2 * tig + 1, 2 * tig + 8, 2 * tig + 9};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint8_t* rw = sv + 64 + 48 * rows[i];
      r.vl[i] = *reinterpret_cast<const uint32_t*>(rw + 4 * gid);
      r.vh[i] = *reinterpret_cast<const uint32_t*>(rw + 32 + 4 * (gid >> 1));
    }
    r.nv[0] = reinterpret_cast<const float*>(sv)[gid];
    r.nv[1] = reinterpret_cast<const float*>(sv)[gid + 8];
  }
  // Selectors of a low word w and its high bits h (bit 4k+2: index k, bit
  // 4k+3: index 8+k): nibble k of a = index k, nibble k of b = index 8+k.
  __device__ static void selectors(uint32_t w, uint32_t h, uint32_t& a, uint32_t& b) {
    a = (w & 0x33333333u) | (h & 0x44444444u);
    b = ((w >> 2) & 0x33333333u) | ((h >> 1) & 0x44444444u);
  }
  // Bytes [c[n0], c[n1], c[n2], c[n3]] of the selector's low 16 bits, low
  // bytes in lo and high bytes in hi.
  __device__ static void lookup(uint32_t sel, const uint32_t tl[2], const uint32_t th[2],
                                uint32_t& lo, uint32_t& hi) {
    lo = prmt(tl[0], tl[1], sel);
    hi = prmt(th[0], th[1], sel);
  }
  // A fragments of QK: k-step s takes elements 32tig + 4s .. +3, selector
  // half s of (a0, b0, a1, b1) in turn.
  __device__ static void conv_k(const Raw& r, uint32_t ka[8][4], const uint32_t tl[2],
                                const uint32_t th[2]) {
#pragma unroll
    for (int rr = 0; rr < 2; ++rr) {
      uint32_t sel[4];
      selectors(r.kl[rr].x, r.kh[rr], sel[0], sel[1]);       // elements 0-7, 8-15
      selectors(r.kl[rr].y, r.kh[rr] << 2, sel[2], sel[3]);  // elements 16-23, 24-31
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        uint32_t lo, hi;
        lookup((s & 1) ? sel[s >> 1] >> 16 : sel[s >> 1], tl, th, lo, hi);
        ka[s][rr] = prmt(lo, hi, 0x5140);      // elements 4s, 4s+1
        ka[s][2 + rr] = prmt(lo, hi, 0x7362);  // elements 4s+2, 4s+3
      }
    }
  }
  // A fragments of PV: m-tile jj takes head-dim elements 16gid + 2jj, +1 of
  // tokens 2tig, 2tig+1 (va[jj][0], [1]) and 2tig+8, 2tig+9 (va[jj][2], [3]).
  // Selector byte jj & 3 of a row holds both elements' indices; one permute
  // puts two token rows' bytes side by side.
  __device__ static void conv_v(const Raw& r, uint32_t va[8][4], const uint32_t tl[2],
                                const uint32_t th[2], int gid) {
    const int hs = 2 * (gid & 1);  // odd gid: the high word's upper 16 indices
    uint32_t sa[4], sb[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) selectors(r.vl[i], r.vh[i] << hs, sa[i], sb[i]);
#pragma unroll
    for (int jj = 0; jj < 8; ++jj) {
      const uint32_t pick = (jj & 3) | ((4 + (jj & 3)) << 4);
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {  // token rows (2tig, 2tig+1), then (2tig+8, 2tig+9)
        const uint32_t x = jj < 4 ? sa[2 * pr] : sb[2 * pr];
        const uint32_t y = jj < 4 ? sa[2 * pr + 1] : sb[2 * pr + 1];
        uint32_t lo, hi;
        lookup(prmt(x, y, pick), tl, th, lo, hi);
        va[jj][2 * pr] = prmt(lo, hi, 0x6240);      // element 2jj of both rows
        va[jj][2 * pr + 1] = prmt(lo, hi, 0x7351);  // element 2jj+1
      }
    }
  }
};

// Kernel shape per format: warps per CTA (NW, one CTA per SM) and ring stages
// per warp (NSW).  Each warp owns NSW stages (~150-170 KB of ring per SM in
// all) and refills a stage only after consuming it, so every mbarrier wait is
// exactly one phase ahead; NW warp-partial slots serve the segment merge.
// The quantized head_dim-64 pages are small and their scan is bound by
// instruction latency, so those kernels run 16 warps (128 registers each).
template <int FMT, int D>
struct Shape {
  static constexpr int NW = (FMT != 0 && D == 64) ? 16 : ((FMT == 0 || FMT == 3) && D == 128) ? 10 : 12;
  static constexpr int STAGE = Fmt<FMT, D>::STAGE;
  static constexpr int NSW = (FMT == 2 && D == 64) ? 7 : (FMT == 1 && D == 64) ? 5 : FMT == 3 ? 6
                             : STAGE <= 2048 ? 6 : STAGE <= 3072 ? 4 : STAGE <= 4096 ? 3 : 2;
  static constexpr int WPART = 16 + 8 * D;  // floats of one partial: m[8], l[8], o[8][D]
};

template <bool BF>
__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  if constexpr (BF)
    mma_bf16(c, a, b0, b1);
  else
    mma_f16(c, a, b0, b1);
}

// The CTA that holds virtual page g when V pages are split evenly over C CTAs
// (CTA c owns [c*V/C, (c+1)*V/C)).
__device__ __forceinline__ int cta_of(int64_t g, int64_t V, int C) {
  return static_cast<int>(((g + 1) * C - 1) / V);
}

struct UnitView {
  int b, h, grp, len;
  int first;   // absolute page of the attended range's first token (window mode)
  int ps, pe;  // this CTA's page range of the unit (relative to first), clipped
};

// First page of the attended tokens of a sequence of length len: with a
// sliding window, the tokens [len - window, len) ("AMD MI300X — KV Cache
// Compression Benchmark", section "SWA mode"); else page 0.
__device__ __forceinline__ int window_first(const DecodeParams& p, int len) {
  return (p.window > 0 && len > p.window) ? (len - p.window) / kPage : 0;
}

__device__ __forceinline__ int ps_of(const DecodeParams& p, int u, int64_t vbeg) {
  const int64_t base = static_cast<int64_t>(u) * p.pmax;
  return vbeg > base ? static_cast<int>(vbeg - base) : 0;
}

__device__ __forceinline__ UnitView unit_view(const DecodeParams& p, int u, int64_t vbeg,
                                              int64_t vend) {
  UnitView v;
  v.grp = u % p.n_groups;
  v.h = (u / p.n_groups) % p.Hkv;
  v.b = u / (p.n_groups * p.Hkv);
  int len = __ldg(p.seq_lens + v.b);
  if (len < 0 || len > p.max_seq_len) len = 0;  // reported by the unit's first CTA
  v.len = len;
  v.first = window_first(p, len);
  const int64_t base = static_cast<int64_t>(u) * p.pmax;
  const int npages = (len + kPage - 1) / kPage - v.first;
  v.ps = ps_of(p, u, vbeg);
  const int pe = static_cast<int>((vend < base + p.pmax ? vend : base + p.pmax) - base);
  v.pe = pe < npages ? pe : npages;
  if (v.pe < v.ps) v.pe = v.ps;
  return v;
}

// The units a CTA's range covers, built once at kernel start (one load round):
// kend[i] = items (cached pages) of units u0..u0+i, len[i] = length of u0+i.
constexpr int kMaxUnits = 64;
struct UnitTable {
  int n, total;
  int kend[kMaxUnits];
  int len[kMaxUnits];
  int first[kMaxUnits];
};

// Block id and KV head of the CTA's item k, or blk = -1 past the last item.
__device__ __forceinline__ void item_block(const DecodeParams& p, const UnitTable& tab, int u0,
                                           int64_t vbeg, int64_t vend, int k, int& blk, int& h) {
  blk = -1;
  h = 0;
  if (k >= tab.total) return;
  int i = 0, k0 = 0, first = 0;
  if (tab.n <= kMaxUnits) {
    int lo = 0, hi = tab.n - 1;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (tab.kend[mid] > k)
        hi = mid;
      else
        lo = mid + 1;
    }
    i = lo;
    k0 = i ? tab.kend[i - 1] : 0;
    first = tab.first[i];
  } else {  // long unit lists: walk them
    for (;;) {
      const UnitView uv = unit_view(p, u0 + i, vbeg, vend);
      first = uv.first;
      if (k < k0 + uv.pe - uv.ps) break;
      k0 += uv.pe - uv.ps;
      ++i;
    }
  }
  const int u = u0 + i;
  h = (u / p.n_groups) % p.Hkv;
  const int b = u / (p.n_groups * p.Hkv);
  blk = __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks + first + ps_of(p, u, vbeg) +
              (k - k0));
}

// Merge the per-CTA partials of unit u (slots u + c for c in [c_first,
// c_first + n)) into out / lse; threads t of nthreads share the float4
// columns.  Partials are read kBatch at a time, all loads of a batch in
// flight together (one pass when n <= kBatch), folded with a running max.
template <int D, int WPART, bool kRot>
__device__ __forceinline__ void final_merge(const DecodeParams& p, int u, int b, int h, int grp,
                                            int c_first, int n, float vs, int t, int nthreads) {
  const float kInf = __int_as_float(0x7f800000);
  constexpr int kBatch = 8;  // partials whose loads are in flight together
  const float* up = p.ws_part + (static_cast<size_t>(u) + c_first) * WPART;
  for (int col = t; col < 2 * D; col += nthreads) {  // float4 columns of [8][D]
    const int hh = col / (D / 4), d4 = (col - hh * (D / 4)) * 4;
    const int qi = grp * 8 + hh;
    if (qi >= p.G) continue;
    float M = -kInf, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s0 = 0; s0 < n; s0 += kBatch) {
      float m[kBatch], l[kBatch];
      float4 v4[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        if (s0 + i < n) {
          const float* ps = up + (s0 + i) * WPART;
          m[i] = __ldcg(ps + hh);
          l[i] = __ldcg(ps + 8 + hh);
          v4[i] = __ldcg(reinterpret_cast<const float4*>(ps + 16 + hh * D + d4));
        } else {
          m[i] = -kInf;
          l[i] = 0.f;
          v4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      float Mn = M;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) Mn = fmaxf(Mn, m[i]);
      if (Mn == -kInf) continue;  // nothing cached so far
      const float a = fast_exp2(M - Mn);  // 0 while M = -inf
      L *= a;
      acc.x *= a;
      acc.y *= a;
      acc.z *= a;
      acc.w *= a;
#pragma unroll
      for (int i = 0; i < kBatch; ++i) {
        const float e = fast_exp2(m[i] - Mn);  // 0 for an empty partial (m = -inf)
        L += e * l[i];
        acc.x += e * v4[i].x;
        acc.y += e * v4[i].y;
        acc.z += e * v4[i].z;
        acc.w += e * v4[i].w;
      }
      M = Mn;
    }
    const float sc = L > 0.f ? vs / L : 0.f;
    const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + qi;
    if constexpr (kRot) {  // PQ3: rotate the pairs (d4, d4+1), (d4+2, d4+3) back
      const float c0 = __ldg(p.v_scale + 8 + d4), s0 = __ldg(p.v_scale + 9 + d4);
      const float c1 = __ldg(p.v_scale + 10 + d4), s1 = __ldg(p.v_scale + 11 + d4);
      acc = make_float4(fmaf(c0, acc.x, s0 * acc.y), fmaf(c0, acc.y, -(s0 * acc.x)),
                        fmaf(c1, acc.z, s1 * acc.w), fmaf(c1, acc.w, -(s1 * acc.z)));
    }
    *reinterpret_cast<float4*>(p.out + row * D + d4) =
        make_float4(acc.x * sc, acc.y * sc, acc.z * sc, acc.w * sc);
    if (d4 == 0 && p.lse) p.lse[row] = L > 0.f ? (M + log2f(L) - kPLog2) * kLn2 : -kInf;
  }
}

template <int FMT, int D, bool QP>
__global__ void __launch_bounds__(Shape<FMT, D>::NW * 32, 1)
    kvq_decode_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                      const __grid_constant__ CUtensorMap mks,
                      const __grid_constant__ CUtensorMap mvs, const DecodeParams p) {
  using F = Fmt<FMT, D>;
  using S = Shape<FMT, D>;
  constexpr int NW = S::NW, NSW = S::NSW, KS = D / 16, MT = D / 16;
  constexpr int NT = NW * 32;
  const float kInf = __int_as_float(0x7f800000);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* rings = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
  float* slots = reinterpret_cast<float*>(rings + static_cast<size_t>(NW) * NSW * F::STAGE);
  uint64_t* bars_all = reinterpret_cast<uint64_t*>(slots + NW * S::WPART);
  __shared__ UnitTable tab;
  __shared__ int s_last;  // this CTA completes the unit's cross-CTA merge
  __shared__ float s_wt[NW][8];  // segment merge: warp weights per head
  __shared__ float s_ml[2][8];   // segment merge: max and weighted sum per head

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int c = blockIdx.x, C = gridDim.x;
  const int64_t V = static_cast<int64_t>(p.units) * p.pmax;
  if (tid == 0) {
    tma_prefetch_desc(&mk);
    tma_prefetch_desc(&mv);
  }
  uint8_t* ring = rings + static_cast<size_t>(warp) * NSW * F::STAGE;
  uint64_t* bars = bars_all + warp * NSW;

  if (V == 0) {  // nothing cached anywhere: every output is empty
    for (int64_t i = static_cast<int64_t>(c) * blockDim.x + tid;
         i < static_cast<int64_t>(p.B) * p.Hq * D; i += static_cast<int64_t>(C) * blockDim.x) {
      p.out[i] = 0.f;
      if (p.lse && i % D == 0) p.lse[i / D] = -kInf;
    }
    return;
  }
  const int64_t vbeg = static_cast<int64_t>(c) * V / C, vend = static_cast<int64_t>(c + 1) * V / C;
  if (vbeg >= vend) return;
  const int u0 = static_cast<int>(vbeg / p.pmax), u1 = static_cast<int>((vend - 1) / p.pmax);
  const int nu = u1 - u0 + 1;

  // Scales: FP8 needs s > 0, NVFP4 g >= 0 (0 = an all-zero tensor); both finite.
  float ks = 1.f, vs = 1.f;
  bool scale_ok = true;
  // PQ3: the K and V codebooks (the parameter blocks' first 8 values, f16
  // values by contract) as byte tables for the index lookups, and the
  // check that each is finite and ascending
  uint32_t tkl[2] = {0u, 0u}, tkh[2] = {0u, 0u}, tvl[2] = {0u, 0u}, tvh[2] = {0u, 0u};
  if constexpr (FMT == 1 || FMT == 2) {
    ks = __ldg(p.k_scale);
    vs = __ldg(p.v_scale);
    if (FMT == 1)
      scale_ok = ks > 0.f && vs > 0.f && ks < kInf && vs < kInf;
    else
      scale_ok = ks >= 0.f && vs >= 0.f && ks < kInf && vs < kInf;
  } else if constexpr (FMT == 3) {
#pragma unroll
    for (int kv = 0; kv < 2; ++kv) {
      const float* cb = kv ? p.v_scale : p.k_scale;
      float v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) v[k] = __ldg(cb + k);
#pragma unroll
      for (int k = 0; k < 7; ++k) scale_ok = scale_ok && v[k] < v[k + 1];
      scale_ok = scale_ok && v[0] > -kInf && v[7] < kInf;
      const uint32_t w01 = pack_f16x2(v[0], v[1]), w23 = pack_f16x2(v[2], v[3]);
      const uint32_t w45 = pack_f16x2(v[4], v[5]), w67 = pack_f16x2(v[6], v[7]);
      uint32_t* tl = kv ? tvl : tkl;
      uint32_t* th = kv ? tvh : tkh;
      tl[0] = prmt(w01, w23, 0x6420);  // low bytes of c0 .. c3
      tl[1] = prmt(w45, w67, 0x6420);
      th[0] = prmt(w01, w23, 0x7531);  // high bytes
      th[1] = prmt(w45, w67, 0x7531);
    }
  }
  // FP8 attention: the E4M3 scales of q and P (both > 0 and finite).  The
  // output takes prob_scale, and the 2^kPLog2 that l carries (see pv_page).
  float qs = 1.f, inv_ps = 1.f, vs_out = vs;
  if constexpr (QP) {
    qs = __ldg(p.q_scale);
    const float ps = __ldg(p.prob_scale);
    scale_ok = scale_ok && qs > 0.f && qs < kInf && ps > 0.f && ps < kInf;
    inv_ps = __fdiv_rn(1.f, ps);
    vs_out = vs * ps * 4096.f;  // 2^kPLog2
  }

  // Scores are scaled by c = sm_scale * k_scale * log2(e) in the softmax
  // below, and masked tokens carry a raw score of -inf, so c must be positive:
  // a negative sm_scale is moved into Q's sign (exact), and c = 0 (an all-zero
  // NVFP4 K tensor, g = 0, whose scores are all 0) becomes a tiny positive c
  // with the same result.
  const float c_raw = p.sm_scale * qs * ks * kLog2e;
  const uint32_t q_sign = c_raw < 0.f ? (QP ? 0x80808080u : 0x80008000u) : 0u;
  const float c_log2 = fmaxf(fabsf(c_raw), 1e-30f);

  // Query fragments (B operand of QK) of unit u; padded heads are 0.  The
  // thread's head-dim elements come in 16-byte runs of 8.
  uint32_t qb[KS][2];
  // PQ3: the scores are q . (|k| R^T c[idx]) = |k| (R q) . c[idx]: q is rotated
  // once, q' = R q (fp32), and enters QK as a 16-bit high part (qb) and its
  // residual (qbl), so the product keeps ~22 bits of q'
  uint32_t qbl[FMT == 3 ? KS : 1][2];
  // FP8 attention: the E4M3 query as the A operand of QK (rows = heads, row
  // gid; the padding rows gid+8 are zero): per 32-element k-step s, a0 holds
  // head-dim elements k_elem(tig, 8s .. 8s+3) and a2 elements 8s+4 .. 8s+7.
  uint32_t qa[QP ? D / 32 : 1][2];
  // Format-specific decode of a stage's words into MMA fragments (PQ3 also
  // needs its codebook tables).
  auto conv_k_any = [&](const typename F::Raw& raw, uint32_t ka[KS][4]) {
    if constexpr (FMT == 3)
      F::conv_k(raw, ka, tkl, tkh);
    else
      F::conv_k(raw, ka);
  };
  auto conv_v_any = [&](const typename F::Raw& raw, uint32_t va[MT][4]) {
    if constexpr (FMT == 3)
      F::conv_v(raw, va, tvl, tvh, gid);
    else
      F::conv_v(raw, va);
  };
  // q of unit u in two steps: fetch_q issues the loads of the thread's
  // head-dim runs (zero for padded heads), conv_q builds the fragments, so
  // the first unit's loads overlap the other prologue loads.
  using QRaw = uint4[D / 32];
  auto fetch_q = [&](int u, QRaw& w) {
    const int grp = u % p.n_groups, h = (u / p.n_groups) % p.Hkv, b = u / (p.n_groups * p.Hkv);
    const int qi = grp * 8 + gid;
    const bool hv = qi < p.G;
    const uint16_t* qrow = p.q + (static_cast<size_t>(b) * p.Hq + h * p.G + (hv ? qi : 0)) * D;
#pragma unroll
    for (int s = 0; s < D / 32; ++s)
      w[s] = hv ? __ldg(reinterpret_cast<const uint4*>(qrow + F::k_elem(tig, 8 * s)))
                : make_uint4(0u, 0u, 0u, 0u);
  };
  auto conv_q = [&](const QRaw& w) {
    if constexpr (QP) {
      // q_hat = E4M3(q / q_scale): IEEE fp32 division, round to nearest even,
      // saturating (the rounding of the cache write)
#pragma unroll
      for (int s = 0; s < D / 32; ++s) {
        const uint32_t ws[4] = {w[s].x, w[s].y, w[s].z, w[s].w};
        uint32_t e[4];
#pragma unroll
        for (int x = 0; x < 4; ++x)
          e[x] = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(ws[x]), qs), __fdiv_rn(bf16_hi(ws[x]), qs));
        qa[s][0] = (e[0] | (e[1] << 16)) ^ q_sign;
        qa[s][1] = (e[2] | (e[3] << 16)) ^ q_sign;
      }
    } else if constexpr (FMT == 3) {
      const float* rot = p.k_scale + 8;
#pragma unroll
      for (int i = 0; i < D / 4; i += 8) {
        const uint32_t ws[4] = {w[i / 8].x, w[i / 8].y, w[i / 8].z, w[i / 8].w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {  // the pair of head-dim elements 2j, 2j+1
          const int j = F::k_elem(tig, i) / 2 + x;
          const float cs = __ldg(rot + 2 * j), sn = __ldg(rot + 2 * j + 1);
          const float a = bf16_lo(ws[x]), b = bf16_hi(ws[x]);
          const float y0 = fmaf(cs, a, -(sn * b)), y1 = fmaf(sn, a, cs * b);
          const uint32_t hi = pack_f16x2(y0, y1);
          float h0, h1;
          unpack_f16x2(hi, h0, h1);
          qb[i / 4 + x / 2][x & 1] = hi ^ q_sign;
          qbl[i / 4 + x / 2][x & 1] = pack_f16x2(y0 - h0, y1 - h1) ^ q_sign;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < D / 4; i += 8) {
        const uint32_t ws[4] = {w[i / 8].x, w[i / 8].y, w[i / 8].z, w[i / 8].w};
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          uint32_t v = ws[x];
          if constexpr (!F::kBF16) v = pack_f16x2(bf16_lo(v), bf16_hi(v));
          qb[i / 4 + x / 2][x & 1] = v ^ q_sign;
        }
      }
    }
  };
  auto load_q = [&](int u) {
    QRaw w;
    fetch_q(u, w);
    conv_q(w);
  };
  QRaw q0raw;
  fetch_q(u0, q0raw);  // in flight while the unit table is built

  // Block ids of this warp's first 64 local items, loaded now on the guess
  // that they lie in unit u0 (they do unless its segment is shorter), so they
  // share one memory round trip with q, the scales and seq_lens instead of
  // waiting for the unit table.  Clamped to max_blocks - 1, the
  // loads stay in the table row; a wrong guess is discarded below.
  const int g0 = warp + lane * NW, g1 = warp + (32 + lane) * NW;
  int spec0, spec1;
  {
    const int32_t* bt0 = p.block_table +
                         static_cast<size_t>(u0 / (p.n_groups * p.Hkv)) * p.max_blocks;
    const int ps0 = ps_of(p, u0, vbeg);
    spec0 = __ldg(bt0 + min(ps0 + g0, p.max_blocks - 1));
    spec1 = __ldg(bt0 + min(ps0 + g1, p.max_blocks - 1));
  }

  // ---- unit table: lane i of warp 0 looks at unit u0 + i (32 at a time)
  if (warp == 0) {
    int run = 0;
    for (int base = 0; base < nu; base += 32) {
      const int i = base + lane;
      int n_i = 0, len_i = 0, first_i = 0;
      if (i < nu) {
        const UnitView uv = unit_view(p, u0 + i, vbeg, vend);
        n_i = scale_ok ? uv.pe - uv.ps : 0;
        len_i = uv.len;
        first_i = uv.first;
      }
      int x = n_i;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, off);
        if (lane >= off) x += y;
      }
      if (i < nu && i < kMaxUnits) {
        tab.kend[i] = run + x;
        tab.len[i] = len_i;
        tab.first[i] = first_i;
      }
      run += __shfl_sync(0xffffffffu, x, 31);
    }
    if (lane == 0) {
      tab.n = nu;
      tab.total = run;
    }
  }
  // The scales' check is reported here, after the table, so that no thread
  // waits on the scale loads before the other prologue loads are issued.
  if (c == 0 && tid == 0 && !scale_ok) set_err(p.d_err, kErrScale);
  conv_q(q0raw);
  // Ask L2 for the page of this warp's first stage (the guessed block id)
  // while the unit table is built; a wrong guess only costs a prefetch.  Only
  // the first: prefetching the pages of all NSW stages measured slower on the
  // head_dim-64 decodes (1 x 65,536 tokens: NVFP4 30.7 against 28.7 us).
  if (p.window <= 0 && lane == 0 && spec0 >= 0 && spec0 < p.num_blocks)
    F::prefetch(&mk, &mv, (u0 / p.n_groups) % p.Hkv, spec0, p);
  if (lane < NSW) mbar_init(&bars[lane], 1);  // each warp its own stages
  mbar_init_fence();
  __syncthreads();
  // Everything read so far (q, tables, scales) predates a preceding cache
  // write of this stream; its cache stores must be visible before the first
  // page copy (this launch may overlap that write's tail).
  griddep_wait();
  const int total = tab.total;
  const int n_local = warp < total ? (total - warp + NW - 1) / NW : 0;

  // Block ids of this warp's local items [chunk, chunk + 64): lane L holds
  // items chunk + L (cur) and chunk + 32 + L (nxt).
  int chunk = 0;
  int cur_blk, cur_h, nxt_blk, nxt_h;
  {
    // the guess assumes the unit's pages start at page 0 (no window)
    const int k_first = p.window > 0 ? 0 : tab.kend[0], h0 = (u0 / p.n_groups) % p.Hkv;
    if (g0 < k_first) {
      cur_blk = spec0;
      cur_h = h0;
    } else {
      item_block(p, tab, u0, vbeg, vend, g0, cur_blk, cur_h);
    }
    if (g1 < k_first) {
      nxt_blk = spec1;
      nxt_h = h0;
    } else {
      item_block(p, tab, u0, vbeg, vend, g1, nxt_blk, nxt_h);
    }
  }

  // Issue the copies of local item i into stage stg (= i % NSW; all lanes
  // call).  The lane holding item i's block id in the window issues them, so
  // no shuffle is needed; ok_win (one ballot per window) says which items of
  // the window have a valid block id.  stage_ok (warp-uniform) records which
  // stages hold a valid page; a bad block id completes its stage's phase with
  // no data.
  unsigned ok_win = __ballot_sync(0xffffffffu, cur_blk >= 0 && cur_blk < p.num_blocks);
  unsigned stage_ok = 0;
  auto issue = [&](int i, int stg) {
    if (i >= chunk + 32) {  // slide the id window by 32 items
      chunk += 32;
      cur_blk = nxt_blk;
      cur_h = nxt_h;
      item_block(p, tab, u0, vbeg, vend, warp + (chunk + 32 + lane) * NW, nxt_blk, nxt_h);
      ok_win = __ballot_sync(0xffffffffu, cur_blk >= 0 && cur_blk < p.num_blocks);
    }
    const int src = i - chunk;
    const unsigned ok = (ok_win >> src) & 1u;
    stage_ok = (stage_ok & ~(1u << stg)) | (ok << stg);
    if (lane == src) {
      uint64_t* bar = &bars[stg];
      fence_proxy_async_smem();  // the warp's reads of this stage precede the copy
      if (ok) {
        F::issue(ring + stg * F::STAGE, bar, &mk, &mv, &mks, &mvs, cur_h, cur_blk, p);
      } else {
        set_err(p.d_err, kErrBlockId);
        mbar_arrive(bar);  // completes the phase with no data; the page is skipped
      }
    }
  };
  // Prologue: lane i fills stage i with local item i (its own cur_blk), the
  // lanes' copies issued together rather than one after another.
  {
    const int n0 = min(NSW, n_local);
    stage_ok = ok_win & ((1u << n0) - 1u);
    if (lane < n0) {
      uint64_t* bar = &bars[lane];
      if ((ok_win >> lane) & 1u) {
        F::issue(ring + lane * F::STAGE, bar, &mk, &mv, &mks, &mvs, cur_h, cur_blk, p);
      } else {
        set_err(p.d_err, kErrBlockId);
        mbar_arrive(bar);  // completes the phase with no data; the page is skipped
      }
    }
  }

  int k_base = 0, j = 0;  // j = this warp's next local item
  int st = 0, ph = 0;     // its stage (j % NSW) and barrier phase parity ((j / NSW) & 1)
  // FP8 attention: S[head][token] = Q_hat K^T on E4M3 tensor cores, the K
  // codes as read from the stage forming the B operand (column = token gid
  // for tokens 0-7, gid+8 for tokens 8-15); this thread gets head gid's
  // scores of tokens 2tig, 2tig+1 (r[0], r[1]) and 2tig+8, 2tig+9 (r[2], r[3]).
  auto qk_page = [&](const typename F::Raw& raw, float r[4]) {
    if constexpr (QP) {
      constexpr int NR = sizeof(raw.k) / sizeof(raw.k[0]) / 2;  // uint4 per row
      float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int t = 0; t < 2; ++t) {  // n-tile t: tokens 8t .. 8t+7, this thread's row gid + 8t
        uint32_t w[4 * NR];
#pragma unroll
        for (int i = 0; i < NR; ++i) {
          const uint4 x = raw.k[NR * t + i];
          w[4 * i] = x.x;
          w[4 * i + 1] = x.y;
          w[4 * i + 2] = x.z;
          w[4 * i + 3] = x.w;
        }
#pragma unroll
        for (int s = 0; s < D / 32; ++s)
          mma_e4m3_k32(t ? s1 : s0, qa[s][0], 0u, qa[s][1], 0u, w[2 * s], w[2 * s + 1]);
      }
      r[0] = s0[0];
      r[1] = s0[1];
      r[2] = s1[0];
      r[3] = s1[1];
      return;
    }
    uint32_t ka[KS][4];
    conv_k_any(raw, ka);
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      if (s & 1)
        mma16816<F::kBF16>(sb, ka[s], qb[s][0], qb[s][1]);
      else
        mma16816<F::kBF16>(sa, ka[s], qb[s][0], qb[s][1]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) r[i] = sa[i] + sb[i];
  };

  for (int si = 0; si < nu; ++si) {
    const int u = u0 + si;
    const int grp = u % p.n_groups, h = (u / p.n_groups) % p.Hkv, b = u / (p.n_groups * p.Hkv);
    int n_items, len, first;
    if (nu <= kMaxUnits) {
      n_items = tab.kend[si] - (si ? tab.kend[si - 1] : 0);
      len = tab.len[si];
      first = tab.first[si];
    } else {
      const UnitView uv = unit_view(p, u, vbeg, vend);
      n_items = scale_ok ? uv.pe - uv.ps : 0;
      len = uv.len;
      first = uv.first;
    }
    const int ps = ps_of(p, u, vbeg);
    const int c_first = cta_of(static_cast<int64_t>(u) * p.pmax, V, C);
    const int c_last = cta_of(static_cast<int64_t>(u + 1) * p.pmax - 1, V, C);
    if (c == c_first && tid == 0 && h == 0 && grp == 0) {
      const int raw = __ldg(p.seq_lens + b);
      if (raw < 0 || raw > p.max_seq_len) set_err(p.d_err, kErrSeqLen);
    }
    if (si > 0) load_q(u);

    // Online softmax state of this thread's heads 2tig, 2tig+1 (log2 domain).
    // n = kPLog2 - m; it starts huge but finite, so the first page with a
    // cached token moves m, and masked scores (-inf) give e = -inf, not NaN.
    float m0 = -kInf, m1 = -kInf, l0 = 0.f, l1 = 0.f;
    float n0 = 1e30f, n1 = 1e30f;
    // FP8 attention: running reference max mq and normaliser lq of head gid
    float mq = -kInf, lq = 0.f;
    int kb = 0;  // PQ3: exponent of the V-norm scale P carries (see below)
    float o[MT][4];
#pragma unroll
    for (int jj = 0; jj < MT; ++jj) o[jj][0] = o[jj][1] = o[jj][2] = o[jj][3] = 0.f;

    const int k_end = k_base + n_items;
    // valid tokens of the segment's last page (only that page can be partial)
    const int n_last = len - (first + ps + n_items - 1) * kPage;
    // window mode: tokens of the window's first page before its start are
    // masked (only the unit's relative page 0 can hold such tokens)
    const int n_skip = (p.window > 0 && len > p.window) ? len - p.window - first * kPage : 0;

    // Softmax of a page, part 1: turn the raw scores r into exponents e = s -
    // m + kPLog2 (s = c_log2 r).  The running max m moves only when a score passes m +
    // kRescaleGap (one vote, no reduction, on most pages); p = 2^(s - m) then
    // stays <= 2^kRescaleGap, which keeps P = p 2^kPLog2 inside f16.
    // Raw scores of the tokens outside [t_lo, t_hi) of the page become -inf
    // (only edge pages: the window's first page, the segment's last page, a
    // page with a bad block id).
    auto mask_scores = [&](float r[4], int t_lo, int t_hi) {
      if constexpr (QP) {  // r: tokens 2tig, 2tig+1, 2tig+8, 2tig+9
        const int t0 = 2 * tig;
        if (!(t0 >= t_lo && t0 < t_hi)) r[0] = -kInf;
        if (!(t0 + 1 >= t_lo && t0 + 1 < t_hi)) r[1] = -kInf;
        if (!(t0 + 8 >= t_lo && t0 + 8 < t_hi)) r[2] = -kInf;
        if (!(t0 + 9 >= t_lo && t0 + 9 < t_hi)) r[3] = -kInf;
      } else {  // r: tokens gid (r[0], r[1]) and gid+8 (r[2], r[3])
        if (!(gid >= t_lo && gid < t_hi)) r[0] = r[1] = -kInf;
        if (!(gid + 8 >= t_lo && gid + 8 < t_hi)) r[2] = r[3] = -kInf;
      }
    };
    auto softmax_e = [&](float r[4], float e[4]) {
      if constexpr (QP) {
        // FP8 attention: r holds head gid's raw scores of tokens 2tig,
        // 2tig+1, 2tig+8, 2tig+9.  P is quantized against the page's own
        // largest score mp, p = 2^(s - mp), P_hat = E4M3(p / prob_scale);
        // the page then enters the running sums with weight f = 2^(mp - mq).
        float rmax = fmaxf(fmaxf(r[0], r[1]), fmaxf(r[2], r[3]));
        rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 1));
        rmax = fmaxf(rmax, __shfl_xor_sync(0xffffffffu, rmax, 2));
        const bool live = rmax != -kInf;  // the page holds an attended token
        const float mp = live ? rmax * c_log2 : -kInf;
        // the running reference moves only when a page max passes it by
        // more than kRescaleGap, so f <= 2^kRescaleGap
        if (__any_sync(0xffffffffu, mp > mq + kRescaleGap)) {
          const float mn = fmaxf(mq, mp);
          const float a = fast_exp2(mq - mn);  // 0 while mq = -inf
          lq *= a;
          const float a0 = __shfl_sync(0xffffffffu, a, 8 * tig);  // head 2tig
          const float a1 = __shfl_sync(0xffffffffu, a, 8 * tig + 4);  // head 2tig+1
#pragma unroll
          for (int jj = 0; jj < MT; ++jj) {
            o[jj][0] *= a0;
            o[jj][1] *= a1;
            o[jj][2] *= a0;
            o[jj][3] *= a1;
          }
          mq = mn;
        }
        const float f = live ? fast_exp2(mp - mq) : 0.f;
        const float mpc = live ? mp : 0.f;
        float pp[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) pp[i] = fast_exp2(fmaf(r[i], c_log2, -mpc));
        lq = fmaf(f * 4096.f, (pp[0] + pp[1]) + (pp[2] + pp[3]), lq);  // l carries 2^kPLog2
        // the decision on fp32 p times fp32(1 / prob_scale), round to nearest even
        const uint32_t lo = f32x2_to_e4m3x2(pp[0] * inv_ps, pp[1] * inv_ps);
        const uint32_t hi = f32x2_to_e4m3x2(pp[2] * inv_ps, pp[3] * inv_ps);
        e[0] = __uint_as_float(lo | (hi << 16));  // B operand of PV: tokens 2tig.. of head gid
        e[1] = __shfl_sync(0xffffffffu, f, 8 * tig);      // weight of head 2tig
        e[2] = __shfl_sync(0xffffffffu, f, 8 * tig + 4);  // weight of head 2tig+1
        return;
      }
      e[0] = fmaf(r[0], c_log2, n0);
      e[1] = fmaf(r[1], c_log2, n1);
      e[2] = fmaf(r[2], c_log2, n0);
      e[3] = fmaf(r[3], c_log2, n1);
      if (__any_sync(0xffffffffu, e[0] > kETop || e[2] > kETop || e[1] > kETop || e[3] > kETop)) {
        const float s0 = r[0] * c_log2, s1 = r[1] * c_log2, s2 = r[2] * c_log2,
                    s3 = r[3] * c_log2;
        float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float a0 = fast_exp2(m0 - mn0), a1 = fast_exp2(m1 - mn1);  // 0 while m = -inf
        l0 *= a0;
        l1 *= a1;
#pragma unroll
        for (int jj = 0; jj < MT; ++jj) {
          o[jj][0] *= a0;
          o[jj][1] *= a1;
          o[jj][2] *= a0;
          o[jj][3] *= a1;
        }
        m0 = mn0;
        m1 = mn1;
        n0 = kPLog2 - m0;
        n1 = kPLog2 - m1;
        e[0] = s0 + n0;
        e[1] = s1 + n1;
        e[2] = s2 + n0;
        e[3] = s3 + n1;
      }
    };
    // The V operand of a page's PV product, from the stage words in registers.
    // FP8 attention: per head-dim row, the codes of tokens 2tig, 2tig+1,
    // 2tig+8, 2tig+9 (the token order of P_hat), a byte transpose of the
    // thread's four token rows: va[jj][0], va[jj][1] (rows gid, gid+8).
    auto prep_v = [&](const typename F::Raw& raw, uint32_t va[MT][4]) {
      if constexpr (QP) {
        constexpr int NWD = D / 32;  // 32-bit words of a thread's run of one token row
#pragma unroll
        for (int k = 0; k < NWD; ++k) {
          uint32_t x[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) x[i] = reinterpret_cast<const uint32_t*>(&raw.v[i])[k];
          const uint32_t xyl = prmt(x[0], x[1], 0x5140), ztl = prmt(x[2], x[3], 0x5140);
          const uint32_t xyh = prmt(x[0], x[1], 0x7362), zth = prmt(x[2], x[3], 0x7362);
          va[2 * k][0] = prmt(xyl, ztl, 0x5410);  // head-dim byte 0 of word k
          va[2 * k][1] = prmt(xyl, ztl, 0x7632);  // byte 1
          va[2 * k + 1][0] = prmt(xyh, zth, 0x5410);  // byte 2
          va[2 * k + 1][1] = prmt(xyh, zth, 0x7632);  // byte 3
        }
      } else {
        conv_v_any(raw, va);
      }
    };
    // Softmax of a page, part 2, and O^T += V^T P^T.  Tokens at or past
    // n_valid are zeroed in V (only the unit's last page can hold unwritten
    // slots, possibly NaN codes).
    auto pv_page = [&](const float e[4], uint32_t va[MT][4], int n_valid) {
      if constexpr (QP) {
        // FP8 attention: O^T += f * (V^T P_hat^T) on E4M3 tensor cores, each
        // page into a fresh accumulator weighted by its f.
        if (n_valid < kPage) {
          const uint32_t msk =
              (2 * tig < n_valid ? 0x000000FFu : 0u) | (2 * tig + 1 < n_valid ? 0x0000FF00u : 0u) |
              (2 * tig + 8 < n_valid ? 0x00FF0000u : 0u) |
              (2 * tig + 9 < n_valid ? 0xFF000000u : 0u);
#pragma unroll
          for (int jj = 0; jj < MT; ++jj) {
            va[jj][0] &= msk;
            va[jj][1] &= msk;
          }
        }
        const uint32_t pq = __float_as_uint(e[0]);
#pragma unroll
        for (int jj = 0; jj < MT; ++jj) {
          float acc[4];
          mma_e4m3_k16(acc, va[jj][0], va[jj][1], pq);
          o[jj][0] = fmaf(e[1], acc[0], o[jj][0]);
          o[jj][1] = fmaf(e[2], acc[1], o[jj][1]);
          o[jj][2] = fmaf(e[1], acc[2], o[jj][2]);
          o[jj][3] = fmaf(e[2], acc[3], o[jj][3]);
        }
        return;
      }
      const float q0 = fast_exp2(e[0]), q1 = fast_exp2(e[1]), q2 = fast_exp2(e[2]),
                  q3 = fast_exp2(e[3]);
      l0 += q0 + q2;  // l and O carry the factor 2^kPLog2, removed at normalisation
      l1 += q1 + q3;
      if (n_valid < kPage) {
        const uint32_t m01 = (2 * tig < n_valid ? 0x0000FFFFu : 0u) |
                             (2 * tig + 1 < n_valid ? 0xFFFF0000u : 0u);
        const uint32_t m23 = (2 * tig + 8 < n_valid ? 0x0000FFFFu : 0u) |
                             (2 * tig + 9 < n_valid ? 0xFFFF0000u : 0u);
#pragma unroll
        for (int jj = 0; jj < MT; ++jj) {
          va[jj][0] &= m01;
          va[jj][1] &= m01;
          va[jj][2] &= m23;
          va[jj][3] &= m23;
        }
      }
      // P^T fragments: high part + residual, transposed in registers
      uint32_t x0h, x1h, x0l, x1l;
      float h0, h1, h2, h3;  // the high parts as fp32
      if constexpr (F::kBF16) {
        x0h = pack_bf16x2(q0, q1);
        x1h = pack_bf16x2(q2, q3);
        unpack_bf16x2(x0h, h0, h1);
        unpack_bf16x2(x1h, h2, h3);
        x0l = pack_bf16x2(q0 - h0, q1 - h1);
        x1l = pack_bf16x2(q2 - h2, q3 - h3);
      } else {
        x0h = pack_f16x2(q0, q1);
        x1h = pack_f16x2(q2, q3);
        unpack_f16x2(x0h, h0, h1);
        unpack_f16x2(x1h, h2, h3);
        x0l = pack_f16x2(q0 - h0, q1 - h1);
        x1l = pack_f16x2(q2 - h2, q3 - h3);
      }
      const uint32_t bh0 = movmatrix_t(x0h), bh1 = movmatrix_t(x1h);
      const uint32_t bl0 = movmatrix_t(x0l), bl1 = movmatrix_t(x1l);
#pragma unroll
      for (int jj = 0; jj < MT; ++jj) {
        mma16816<F::kBF16>(o[jj], va[jj], bh0, bh1);
        mma16816<F::kBF16>(o[jj], va[jj], bl0, bl1);
      }
    };

    if constexpr (QP) {
      // FP8 attention: the same page loop, the page's work in the lambdas above
      for (int k = warp + j * NW; k < k_end; k += NW, ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], ph))) {
          if (lane == 0) set_err(p.d_err, kErrTimeout);
          for (int i = j + 1; i < j + NSW && i < n_local; ++i)  // drain copies in flight
            mbar_wait_bounded(&bars[i % NSW], (i / NSW) & 1);
          j = n_local;
          break;
        }
        const bool valid = (stage_ok >> st) & 1u;
        typename F::Raw raw;
        if (valid) {
          F::load_raw_k(ring + st * F::STAGE, gid, tig, raw);
          F::load_raw_v(ring + st * F::STAGE, gid, tig, raw);
        }
        __syncwarp();
        if (j + NSW < n_local) issue(j + NSW, st);  // item j + NSW reuses stage st
        if (++st == NSW) {
          st = 0;
          ph ^= 1;
        }
        if (!valid) continue;
        float r[4], e[4];
        uint32_t va[MT][4];
        qk_page(raw, r);
        prep_v(raw, va);
        // valid tokens [t_lo, t_hi) of an edge page: the window's first page
        // starts late, the segment's last page may end early
        const bool first_w = n_skip > 0 && ps == 0 && k == k_base;
        int t_hi = kPage;
        if (first_w || k == k_end - 1) {
          t_hi = (k == k_end - 1 && n_last < kPage) ? n_last : kPage;
          mask_scores(r, first_w ? n_skip : 0, t_hi);
        }
        softmax_e(r, e);
        pv_page(e, va, t_hi);
      }
    } else {
      for (int k = warp + j * NW; k < k_end; k += NW, ++j) {
        const uint8_t* sp = ring + st * F::STAGE;
        // all lanes agree on the outcome so the warp stays converged
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], ph))) {
          if (lane == 0) set_err(p.d_err, kErrTimeout);
          for (int i = j + 1; i < j + NSW && i < n_local; ++i)  // drain copies in flight
            mbar_wait_bounded(&bars[i % NSW], (i / NSW) & 1);
          j = n_local;
          break;
        }
        const bool valid = (stage_ok >> st) & 1u;

        // The stage's words go to registers first, so the stage is refilled with
        // local item j + NSW before any decode or math on this one (for BF16
        // head_dim 128, after the QK product: see kLateV).
        typename F::Raw raw;
        uint32_t ka[KS][4], va[MT][4];
        float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
        // ---- S^T = K Q^T on tensor cores (two accumulator chains)
        auto qk = [&]() {
          if constexpr (F::kStream) {
  #pragma unroll
            for (int w = 0; w < KS / 2; ++w) {
              uint32_t a0[4], a1[4];
              F::conv_k_pair(raw, w, a0, a1);
              mma16816<F::kBF16>(sa, a0, qb[2 * w][0], qb[2 * w][1]);
              mma16816<F::kBF16>(sb, a1, qb[2 * w + 1][0], qb[2 * w + 1][1]);
            }
            return;
          }
          conv_k_any(raw, ka);
  #pragma unroll
          for (int s = 0; s < KS; ++s) {
            if constexpr (FMT == 3) {  // q' high part and residual, two chains
              mma16816<false>(sa, ka[s], qb[s][0], qb[s][1]);
              mma16816<false>(sb, ka[s], qbl[s][0], qbl[s][1]);
            } else if (s & 1) {
              mma16816<F::kBF16>(sb, ka[s], qb[s][0], qb[s][1]);
            } else {
              mma16816<F::kBF16>(sa, ka[s], qb[s][0], qb[s][1]);
            }
          }
        };
        if constexpr (F::kLateV) {
          if (valid) {
            F::load_raw_k(sp, gid, tig, raw);
            qk();
            F::load_raw_v(sp, gid, tig, raw);
          }
        } else if (valid) {
          F::load_raw_k(sp, gid, tig, raw);
          F::load_raw_v(sp, gid, tig, raw);
        }
        __syncwarp();
        if (j + NSW < n_local) issue(j + NSW, st);  // item j + NSW reuses stage st
        if (++st == NSW) {
          st = 0;
          ph ^= 1;
        }
        if (!valid) continue;
        if constexpr (!F::kLateV) qk();
        if constexpr (!F::kStream) conv_v_any(raw, va);

        // raw scores r = q . k_code (the scale c_log2 is applied below)
        float r0 = sa[0] + sb[0], r1 = sa[1] + sb[1], r2 = sa[2] + sb[2], r3 = sa[3] + sb[3];
        if constexpr (FMT == 3) {  // times the K norms of tokens gid, gid+8
          r0 *= raw.nk[0];
          r1 *= raw.nk[0];
          r2 *= raw.nk[1];
          r3 *= raw.nk[1];
        }
        uint32_t vm01 = 0xFFFFFFFFu, vm23 = 0xFFFFFFFFu;  // V token masks of a partial page
        if (k == k_end - 1 && n_last < kPage) {  // last, partial page: mask tokens past the length
          const int n_valid = n_last;
          if (gid >= n_valid) r0 = r1 = -kInf;
          if (gid + 8 >= n_valid) r2 = r3 = -kInf;
          if constexpr (FMT == 3) {  // unwritten norms may be NaN
            if (gid >= n_valid) raw.nv[0] = 0.f;
            if (gid + 8 >= n_valid) raw.nv[1] = 0.f;
          }
          const uint32_t m01 = (2 * tig < n_valid ? 0x0000FFFFu : 0u) |
                               (2 * tig + 1 < n_valid ? 0xFFFF0000u : 0u);
          const uint32_t m23 = (2 * tig + 8 < n_valid ? 0x0000FFFFu : 0u) |
                               (2 * tig + 9 < n_valid ? 0xFFFF0000u : 0u);
          vm01 = m01;
          vm23 = m23;
          if constexpr (!F::kStream) {
  #pragma unroll
            for (int jj = 0; jj < MT; ++jj) {  // unwritten slots may hold NaN codes
              va[jj][0] &= m01;
              va[jj][1] &= m01;
              va[jj][2] &= m23;
              va[jj][3] &= m23;
            }
          }
        }
        if (n_skip > 0 && ps == 0 && k == k_base) {  // window's first page: tokens before it
          if (gid < n_skip) r0 = r1 = -kInf;
          if (gid + 8 < n_skip) r2 = r3 = -kInf;
        }

        // ---- online softmax (log2 domain); this thread: heads 2tig, 2tig+1.
        // The running max m moves only when a score passes m + kRescaleGap
        // (one vote, no reduction, on most pages); p = 2^(s - m) then stays
        // <= 2^kRescaleGap, which keeps P = p * 2^kPLog2 inside f16.
        // e = s - m + kPLog2 with s = c_log2 * r: 2^e = p * 2^kPLog2 = P as fed to the MMA
        float e0 = fmaf(r0, c_log2, n0), e1 = fmaf(r1, c_log2, n1);
        float e2 = fmaf(r2, c_log2, n0), e3 = fmaf(r3, c_log2, n1);
        if (__any_sync(0xffffffffu, e0 > kETop || e2 > kETop || e1 > kETop || e3 > kETop)) {
          const float s0 = r0 * c_log2, s1 = r1 * c_log2, s2 = r2 * c_log2, s3 = r3 * c_log2;
          float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
  #pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
          }
          const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
          const float a0 = fast_exp2(m0 - mn0), a1 = fast_exp2(m1 - mn1);  // 0 while m = -inf
          l0 *= a0;
          l1 *= a1;
  #pragma unroll
          for (int jj = 0; jj < MT; ++jj) {
            o[jj][0] *= a0;
            o[jj][1] *= a1;
            o[jj][2] *= a0;
            o[jj][3] *= a1;
          }
          m0 = mn0;
          m1 = mn1;
          n0 = kPLog2 - m0;
          n1 = kPLog2 - m1;
          e0 = s0 + n0;
          e1 = s1 + n1;
          e2 = s2 + n0;
          e3 = s3 + n1;
        }
        float q0 = fast_exp2(e0), q1 = fast_exp2(e1), q2 = fast_exp2(e2), q3 = fast_exp2(e3);
        l0 += q0 + q2;  // l and O carry the factor 2^kPLog2, removed at normalisation
        l1 += q1 + q3;
        if constexpr (FMT == 3) {
          // P also carries the V norms of its tokens (gid, gid+8), over a
          // warp-uniform power of two 2^(kb - 126) at or above every V norm of
          // the segment so far (kb: the largest biased fp32 exponent), which
          // keeps it below 2^15 in f16; O takes the factor back at the segment
          // end, and is rescaled (exactly) when kb grows
          const int e_0 = (__float_as_int(raw.nv[0]) >> 23) & 0xFF;
          const int e_1 = (__float_as_int(raw.nv[1]) >> 23) & 0xFF;
          const int ep = min(__reduce_max_sync(0xffffffffu, max(e_0, e_1)), 252);
          if (ep > kb) {
            const int dd = 127 + kb - ep;
            const float a = dd >= 1 ? __int_as_float(dd << 23) : 0.f;
#pragma unroll
            for (int jj = 0; jj < MT; ++jj) {
              o[jj][0] *= a;
              o[jj][1] *= a;
              o[jj][2] *= a;
              o[jj][3] *= a;
            }
            kb = ep;
          }
          const float sc = __int_as_float((253 - kb) << 23);  // 2^(126 - kb)
          const float g0 = raw.nv[0] * sc, g1 = raw.nv[1] * sc;
          q0 *= g0;
          q1 *= g0;
          q2 *= g1;
          q3 *= g1;
        }

        // ---- P^T fragments: high part + residual, transposed in registers
        uint32_t x0h, x1h, x0l, x1l;
        float h0, h1, h2, h3;  // the high parts as fp32
        if constexpr (F::kBF16) {
          x0h = pack_bf16x2(q0, q1);
          x1h = pack_bf16x2(q2, q3);
          unpack_bf16x2(x0h, h0, h1);
          unpack_bf16x2(x1h, h2, h3);
          x0l = pack_bf16x2(q0 - h0, q1 - h1);
          x1l = pack_bf16x2(q2 - h2, q3 - h3);
        } else {
          x0h = pack_f16x2(q0, q1);
          x1h = pack_f16x2(q2, q3);
          unpack_f16x2(x0h, h0, h1);
          unpack_f16x2(x1h, h2, h3);
          x0l = pack_f16x2(q0 - h0, q1 - h1);
          x1l = pack_f16x2(q2 - h2, q3 - h3);
        }
        const uint32_t bh0 = movmatrix_t(x0h), bh1 = movmatrix_t(x1h);
        const uint32_t bl0 = movmatrix_t(x0l), bl1 = movmatrix_t(x1l);

        // ---- O^T += V^T P^T
        if constexpr (F::kStream) {  // V decoded four m-tiles at a time
          const bool part = k == k_end - 1 && n_last < kPage;
  #pragma unroll
          for (int wi = 0; wi < MT / 4; ++wi) {
            uint32_t v4[4][4];
            F::conv_v_half(raw, wi, v4);
            if (part) {
  #pragma unroll
              for (int x = 0; x < 4; ++x) {  // unwritten slots may hold NaN codes
                v4[x][0] &= vm01;
                v4[x][1] &= vm01;
                v4[x][2] &= vm23;
                v4[x][3] &= vm23;
              }
            }
  #pragma unroll
            for (int x = 0; x < 4; ++x) {
              mma16816<F::kBF16>(o[4 * wi + x], v4[x], bh0, bh1);
              mma16816<F::kBF16>(o[4 * wi + x], v4[x], bl0, bl1);
            }
          }
        } else {
  #pragma unroll
          for (int jj = 0; jj < MT; ++jj) {
            mma16816<F::kBF16>(o[jj], va[jj], bh0, bh1);
            mma16816<F::kBF16>(o[jj], va[jj], bl0, bl1);
          }
        }
      }
    }
    k_base = k_end;

    if constexpr (FMT == 3) {  // O back to absolute units: times 2^(kb - 126)
      const float a = __int_as_float((kb + 1) << 23);
#pragma unroll
      for (int jj = 0; jj < MT; ++jj) {
        o[jj][0] *= a;
        o[jj][1] *= a;
        o[jj][2] *= a;
        o[jj][3] *= a;
      }
    }
    // ---- segment end: warp partials -> shared slots, merged by the CTA
    float* wp = slots + warp * S::WPART;  // m[8], l[8], o[8][D]
    if constexpr (QP) {  // head gid's sums are spread over the tig lanes
      lq += __shfl_xor_sync(0xffffffffu, lq, 1);
      lq += __shfl_xor_sync(0xffffffffu, lq, 2);
      if (tig == 0) {
        wp[gid] = mq;
        wp[8 + gid] = lq;
      }
    } else {
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
      }
      if (gid == 0) {
        wp[2 * tig] = m0;
        wp[2 * tig + 1] = m1;
        wp[8 + 2 * tig] = l0;
        wp[8 + 2 * tig + 1] = l1;
      }
    }
#pragma unroll
    for (int jj = 0; jj < MT; ++jj) {
      const int d0 = F::v_elem(gid, 2 * jj), d1 = F::v_elem(gid, 2 * jj + 1);
      wp[16 + (2 * tig) * D + d0] = o[jj][0];
      wp[16 + (2 * tig + 1) * D + d0] = o[jj][1];
      wp[16 + (2 * tig) * D + d1] = o[jj][2];
      wp[16 + (2 * tig + 1) * D + d1] = o[jj][3];
    }
    __syncthreads();
    // per head: the max M over the warps, each warp's weight 2^(m_w - M) and
    // the weighted sum L, once (8 threads), for all D outputs of the head
    if (tid < 8) {
      float M = -kInf;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, slots[w * S::WPART + tid]);
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float e = M == -kInf ? 0.f : fast_exp2(slots[w * S::WPART + tid] - M);
        s_wt[w][tid] = e;
        L += e * slots[w * S::WPART + 8 + tid];
      }
      s_ml[0][tid] = M;
      s_ml[1][tid] = L;
    }
    __syncthreads();
    const bool alone = c_first == c_last;
    float* gpart = p.ws_part + (static_cast<size_t>(u) + c) * S::WPART;
    if constexpr (FMT == 3) {
      // PQ3: O holds R_v (out); an output pair (2j, 2j+1) is rotated back,
      // out_2j = cos_j a + sin_j b, out_2j+1 = cos_j b - sin_j a
      for (int idx = tid; idx < 4 * D; idx += NT) {
        const int hh = idx / (D / 2), d = 2 * (idx - hh * (D / 2));
        const float M = s_ml[0][hh], L = s_ml[1][hh];
        float a0 = 0.f, a1 = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          a0 += s_wt[w][hh] * slots[w * S::WPART + 16 + hh * D + d];
          a1 += s_wt[w][hh] * slots[w * S::WPART + 16 + hh * D + d + 1];
        }
        if (alone) {
          const int qi = grp * 8 + hh;
          if (qi < p.G) {
            const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + qi;
            const float cs = __ldg(p.v_scale + 8 + d), sn = __ldg(p.v_scale + 9 + d);
            const float sc = L > 0.f ? vs_out / L : 0.f;
            p.out[row * D + d] = fmaf(cs, a0, sn * a1) * sc;
            p.out[row * D + d + 1] = fmaf(cs, a1, -(sn * a0)) * sc;
            if (d == 0 && p.lse) p.lse[row] = L > 0.f ? (M + log2f(L) - kPLog2) * kLn2 : -kInf;
          }
        } else {
          gpart[16 + hh * D + d] = a0;
          gpart[16 + hh * D + d + 1] = a1;
          if (d == 0) {
            gpart[hh] = M;
            gpart[8 + hh] = L;
          }
        }
      }
    } else
    for (int idx = tid; idx < 8 * D; idx += NT) {
      const int hh = idx / D, d = idx - hh * D;
      const float M = s_ml[0][hh], L = s_ml[1][hh];
      float acc = 0.f;
#pragma unroll
      for (int w = 0; w < NW; ++w) acc += s_wt[w][hh] * slots[w * S::WPART + 16 + hh * D + d];
      if (alone) {
        const int qi = grp * 8 + hh;
        if (qi < p.G) {
          const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + qi;
          p.out[row * D + d] = L > 0.f ? acc * (vs_out / L) : 0.f;
          if (d == 0 && p.lse) p.lse[row] = L > 0.f ? (M + log2f(L) - kPLog2) * kLn2 : -kInf;
        }
      } else {
        gpart[16 + hh * D + d] = acc;
        if (d == 0) {
          gpart[hh] = M;
          gpart[8 + hh] = L;
        }
      }
    }
    if (!alone) {
      // ---- the last CTA of the unit to get here merges all its partials.
      // The barrier orders the CTA's partial stores before thread 0's
      // release; its acquire, then the barrier, orders the merge's loads
      // after every other CTA's release.
      __syncthreads();
      if (tid == 0) {
        const unsigned t = atom_add_acq_rel_gpu(p.ws_cnt + u, 1u);
        s_last = (t == static_cast<unsigned>(c_last - c_first));
      }
      __syncthreads();
      if (s_last) {
        final_merge<D, S::WPART, FMT == 3>(p, u, b, h, grp, c_first, c_last - c_first + 1, vs_out,
                                           tid, NT);
        if (tid == 0) p.ws_cnt[u] = 0u;  // ready for the next launch
      }
    }
    __syncthreads();  // slots and s_last are reused by the next segment
  }
}

template <int FMT, int D>
size_t smem_bytes() {
  using S = Shape<FMT, D>;
  return 1024 + static_cast<size_t>(S::NW) * S::NSW * S::STAGE +
         sizeof(float) * S::NW * S::WPART + 8 * static_cast<size_t>(S::NW) * S::NSW;
}

template <int FMT, int D, bool QP = false>
cudaError_t launch_t(const CUtensorMap* maps, const DecodeParams& p, int ctas,
                     cudaStream_t stream) {
  using S = Shape<FMT, D>;
  const size_t smem = smem_bytes<FMT, D>();
  static std::atomic<bool> attr_done[kMaxDevices];  // per instantiation and device ordinal
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kvq_decode_kernel<FMT, D, QP>),
                                   smem, attr_done);
  if (e != cudaSuccess) return e;
  // Programmatic stream serialization: the launch may begin while a
  // preceding kv_quantize_write of this stream finishes (see griddep_wait).
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(S::NW * 32);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kvq_decode_kernel<FMT, D, QP>, maps[0], maps[1], maps[2], maps[3],
                            p);
}

template <int FMT, int D>
void config_t(DecodeConfig* c) {
  c->warps = Shape<FMT, D>::NW;
  c->stages = Shape<FMT, D>::NSW;
  c->stage_bytes = Fmt<FMT, D>::STAGE;
  c->smem_bytes = smem_bytes<FMT, D>();
  c->part_floats = Shape<FMT, D>::WPART;
  // measured on the 4 x 126,976 and 8 x 65,536-token decodes (optimum ~96-128
  // pages; PQ3 pages take about three times as long as FP8 pages)
  c->merge_pages = FMT == 3 ? 64 : 128;
}

}  // namespace

bool decode_config(int fmt, int D, DecodeConfig* cfg) {
  switch (fmt * 1000 + D) {
    case 64: config_t<0, 64>(cfg); return true;
    case 128: config_t<0, 128>(cfg); return true;
    case 1064: config_t<1, 64>(cfg); return true;
    case 1128: config_t<1, 128>(cfg); return true;
    case 2064: config_t<2, 64>(cfg); return true;
    case 2128: config_t<2, 128>(cfg); return true;
    case 3128: config_t<3, 128>(cfg); return true;
  }
  return false;
}

cudaError_t launch_decode(int fmt, int D, const CUtensorMap* maps, const DecodeParams& p,
                          int ctas, cudaStream_t stream, bool fp8_qp) {
  if (fp8_qp) {
    if (fmt != 1) return cudaErrorInvalidValue;
    return D == 128 ? launch_t<1, 128, true>(maps, p, ctas, stream)
                    : launch_t<1, 64, true>(maps, p, ctas, stream);
  }
  switch (fmt * 1000 + D) {
    case 64: return launch_t<0, 64>(maps, p, ctas, stream);
    case 128: return launch_t<0, 128>(maps, p, ctas, stream);
    case 1064: return launch_t<1, 64>(maps, p, ctas, stream);
    case 1128: return launch_t<1, 128>(maps, p, ctas, stream);
    case 2064: return launch_t<2, 64>(maps, p, ctas, stream);
    case 2128: return launch_t<2, 128>(maps, p, ctas, stream);
    case 3128: return launch_t<3, 128>(maps, p, ctas, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
