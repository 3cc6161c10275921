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
//   * Grid (split, KV head x head group, sequence).  A CTA owns a contiguous
//     range of 16-token pages of one (sequence, KV head); its warps take the
//     range's pages round-robin.
//   * Each warp streams its pages through a private ring of shared-memory
//     stages filled by TMA tensor copies (one per K/V tile, swizzled so the
//     fragment reads below are bank-conflict free), completion tracked by one
//     mbarrier per stage.  No other warp touches the ring, so there is no
//     CTA-wide synchronisation in the loop.
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
//   * Online softmax in the exp2 domain per warp; warps are merged through
//     shared memory; splits are merged by the last CTA of each (sequence, KV
//     head) to arrive (atomic ticket, nobody waits), which writes out and lse.
//     With one split the CTA writes the result directly.
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

constexpr float kLn2 = 0.6931471805599453f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kPScale = 4096.0f;  // P is fed to the MMA as p * 2^12 (exact)
constexpr int kMaxSplits = 512;

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
                               int h, int blk) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void load_k(const uint8_t* st, int gid, int tig, uint32_t ka[8][4]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = gid + 8 * r;
      const uint4 a = lds128(st + swz128(row, 32 * tig));
      const uint4 c = lds128(st + swz128(row, 32 * tig + 16));
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int s = 0; s < 8; ++s) e4m3x4_to_f16x2x2(w[s], ka[s][r], ka[s][2 + r]);
    }
  }
  __device__ static void load_v(const uint8_t* st, int gid, int tig, uint32_t va[8][4]) {
    const uint8_t* sv = st + V_OFF;
    const uint4 X = lds128(sv + swz128(2 * tig, 16 * gid));
    const uint4 Y = lds128(sv + swz128(2 * tig + 1, 16 * gid));
    const uint4 Z = lds128(sv + swz128(2 * tig + 8, 16 * gid));
    const uint4 W = lds128(sv + swz128(2 * tig + 9, 16 * gid));
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
                               int h, int blk) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void load_k(const uint8_t* st, int gid, int tig, uint32_t ka[4][4]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const uint4 a = lds128(st + swz64(gid + 8 * r, 16 * tig));
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) e4m3x4_to_f16x2x2(w[s], ka[s][r], ka[s][2 + r]);
    }
  }
  __device__ static void load_v(const uint8_t* st, int gid, int tig, uint32_t va[4][4]) {
    const uint8_t* sv = st + V_OFF;
    const uint2 X = lds64(sv + swz64(2 * tig, 8 * gid));
    const uint2 Y = lds64(sv + swz64(2 * tig + 1, 8 * gid));
    const uint2 Z = lds64(sv + swz64(2 * tig + 8, 8 * gid));
    const uint2 W = lds64(sv + swz64(2 * tig + 9, 8 * gid));
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
                               int h, int blk) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
  }
  __device__ static void load_k(const uint8_t* st, int gid, int tig, uint32_t ka[4][4]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = gid + 8 * r;
      const uint4 a = lds128(st + swz128(row, 32 * tig));
      const uint4 c = lds128(st + swz128(row, 32 * tig + 16));
      const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        ka[s][r] = w[2 * s];
        ka[s][2 + r] = w[2 * s + 1];
      }
    }
  }
  __device__ static void load_v(const uint8_t* st, int gid, int tig, uint32_t va[4][4]) {
    const uint8_t* sv = st + V_OFF;
    const uint4 X = lds128(sv + swz128(2 * tig, 16 * gid));
    const uint4 Y = lds128(sv + swz128(2 * tig + 1, 16 * gid));
    const uint4 Z = lds128(sv + swz128(2 * tig + 8, 16 * gid));
    const uint4 W = lds128(sv + swz128(2 * tig + 9, 16 * gid));
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
                               int h, int blk) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + 2048, mk, bar, 64, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF + 2048, mv, bar, 64, 0, h, blk);
  }
  __device__ static void load_k(const uint8_t* st, int gid, int tig, uint32_t ka[8][4]) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int row = gid + 8 * r;
        const uint4 a = lds128(st + 2048 * hf + swz128(row, 32 * tig));
        const uint4 c = lds128(st + 2048 * hf + swz128(row, 32 * tig + 16));
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, c.x, c.y, c.z, c.w};
#pragma unroll
        for (int s = 0; s < 4; ++s) {
          ka[4 * hf + s][r] = w[2 * s];
          ka[4 * hf + s][2 + r] = w[2 * s + 1];
        }
      }
    }
  }
  __device__ static void load_v(const uint8_t* st, int gid, int tig, uint32_t va[8][4]) {
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      const uint8_t* sv = st + V_OFF + 2048 * hf;
      const uint4 X = lds128(sv + swz128(2 * tig, 16 * gid));
      const uint4 Y = lds128(sv + swz128(2 * tig + 1, 16 * gid));
      const uint4 Z = lds128(sv + swz128(2 * tig + 8, 16 * gid));
      const uint4 W = lds128(sv + swz128(2 * tig + 9, 16 * gid));
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

// ---- NVFP4, head_dim 64: code rows of 32 B (32-byte swizzle) + 4 scale bytes.
template <>
struct Fmt<2, 64> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 1280, TX = 1152, V_OFF = 512, KSF = 1024, VSF = 1152;
  __device__ static int k_elem(int tig, int i) { return 16 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 8 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap* mks,
                               const CUtensorMap* mvs, int h, int blk) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
    tma_load_3d(st + KSF, mks, bar, 0, h, blk);
    tma_load_3d(st + VSF, mvs, bar, 0, h, blk);
  }
  __device__ static void load_k(const uint8_t* st, int gid, int tig, uint32_t ka[4][4]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = gid + 8 * r;
      const uint2 c = lds64(st + swz32(row, 8 * tig));
      const uint32_t sc = scale_pair(st[KSF + row * 4 + tig], st[KSF + row * 4 + tig]);
      uint32_t f[8];
      e2m1x8_to_f16x2x4(c.x, f);
      e2m1x8_to_f16x2x4(c.y, f + 4);
#pragma unroll
      for (int s = 0; s < 4; ++s) {
        ka[s][r] = hmul2(f[2 * s], sc);
        ka[s][2 + r] = hmul2(f[2 * s + 1], sc);
      }
    }
  }
  __device__ static void load_v(const uint8_t* st, int gid, int tig, uint32_t va[4][4]) {
    const uint8_t* sv = st + V_OFF;
    const uint8_t* ss = st + VSF;
    const int t0 = 2 * tig, t2 = 2 * tig + 8, blk = gid >> 1;
    const uint32_t X = lds32(sv + swz32(t0, 4 * gid));
    const uint32_t Y = lds32(sv + swz32(t0 + 1, 4 * gid));
    const uint32_t Z = lds32(sv + swz32(t2, 4 * gid));
    const uint32_t W = lds32(sv + swz32(t2 + 1, 4 * gid));
    const uint32_t sxy = scale_pair(ss[t0 * 4 + blk], ss[(t0 + 1) * 4 + blk]);
    const uint32_t szw = scale_pair(ss[t2 * 4 + blk], ss[(t2 + 1) * 4 + blk]);
    uint32_t lo, hi, L[4], H[4];
    nib_interleave(X, Y, lo, hi);
    e2m1x8_to_f16x2x4(lo, L);
    e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][0] = hmul2(L[j], sxy);
      va[j][1] = hmul2(H[j], sxy);
    }
    nib_interleave(Z, W, lo, hi);
    e2m1x8_to_f16x2x4(lo, L);
    e2m1x8_to_f16x2x4(hi, H);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      va[j][2] = hmul2(L[j], szw);
      va[j][3] = hmul2(H[j], szw);
    }
  }
};

// ---- NVFP4, head_dim 128: code rows of 64 B (64-byte swizzle) + 8 scale bytes.
template <>
struct Fmt<2, 128> {
  static constexpr bool kBF16 = false;
  static constexpr int STAGE = 2560, TX = 2304, V_OFF = 1024, KSF = 2048, VSF = 2176;
  __device__ static int k_elem(int tig, int i) { return 32 * tig + i; }
  __device__ static int v_elem(int gid, int i) { return 16 * gid + i; }
  __device__ static void issue(uint8_t* st, uint64_t* bar, const CUtensorMap* mk,
                               const CUtensorMap* mv, const CUtensorMap* mks,
                               const CUtensorMap* mvs, int h, int blk) {
    mbar_arrive_expect_tx(bar, TX);
    tma_load_4d(st, mk, bar, 0, 0, h, blk);
    tma_load_4d(st + V_OFF, mv, bar, 0, 0, h, blk);
    tma_load_3d(st + KSF, mks, bar, 0, h, blk);
    tma_load_3d(st + VSF, mvs, bar, 0, h, blk);
  }
  __device__ static void load_k(const uint8_t* st, int gid, int tig, uint32_t ka[8][4]) {
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int row = gid + 8 * r;
      const uint4 c = lds128(st + swz64(row, 16 * tig));
      const uint32_t s01 = scale_pair(st[KSF + row * 8 + 2 * tig], st[KSF + row * 8 + 2 * tig + 1]);
      const uint32_t sc0 = prmt(s01, s01, 0x1010), sc1 = prmt(s01, s01, 0x3232);
      uint32_t f[16];
      e2m1x8_to_f16x2x4(c.x, f);
      e2m1x8_to_f16x2x4(c.y, f + 4);
      e2m1x8_to_f16x2x4(c.z, f + 8);
      e2m1x8_to_f16x2x4(c.w, f + 12);
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        const uint32_t sc = s < 4 ? sc0 : sc1;
        ka[s][r] = hmul2(f[2 * s], sc);
        ka[s][2 + r] = hmul2(f[2 * s + 1], sc);
      }
    }
  }
  __device__ static void load_v(const uint8_t* st, int gid, int tig, uint32_t va[8][4]) {
    const uint8_t* sv = st + V_OFF;
    const uint8_t* ss = st + VSF;
    const int t0 = 2 * tig, t2 = 2 * tig + 8;
    const uint2 X = lds64(sv + swz64(t0, 8 * gid));
    const uint2 Y = lds64(sv + swz64(t0 + 1, 8 * gid));
    const uint2 Z = lds64(sv + swz64(t2, 8 * gid));
    const uint2 W = lds64(sv + swz64(t2 + 1, 8 * gid));
    const uint32_t sxy = scale_pair(ss[t0 * 8 + gid], ss[(t0 + 1) * 8 + gid]);
    const uint32_t szw = scale_pair(ss[t2 * 8 + gid], ss[(t2 + 1) * 8 + gid]);
    const uint32_t x[2] = {X.x, X.y}, y[2] = {Y.x, Y.y}, z[2] = {Z.x, Z.y}, w[2] = {W.x, W.y};
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

// Kernel shape per format: warps per CTA and stages per warp.
template <int FMT, int D>
struct Shape {
  static constexpr int NW = 4;
  static constexpr int NS = Fmt<FMT, D>::STAGE <= 1280 ? 8
                            : Fmt<FMT, D>::STAGE <= 2560 ? 6
                            : Fmt<FMT, D>::STAGE <= 4096 ? 4
                                                        : 3;
};

template <bool BF>
__device__ __forceinline__ void mma16816(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  if constexpr (BF)
    mma_bf16(c, a, b0, b1);
  else
    mma_f16(c, a, b0, b1);
}

template <int FMT, int D>
__device__ __forceinline__ void drain(uint64_t* bars, int from, int to) {
  constexpr int NS = Shape<FMT, D>::NS;
  for (int k = from; k < to; ++k) mbar_wait_bounded(&bars[k % NS], (k / NS) & 1);
}

template <int FMT, int D>
__global__ void __launch_bounds__(Shape<FMT, D>::NW * 32, 1)
    kvq_decode_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mv,
                      const __grid_constant__ CUtensorMap mks,
                      const __grid_constant__ CUtensorMap mvs, const DecodeParams p) {
  using F = Fmt<FMT, D>;
  constexpr int NW = Shape<FMT, D>::NW, NS = Shape<FMT, D>::NS;
  constexpr int KS = D / 16, MT = D / 16;
  const float kInf = __int_as_float(0x7f800000);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ int s_last;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  uint8_t* stages = smem + static_cast<size_t>(warp) * NS * F::STAGE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + static_cast<size_t>(NW) * NS * F::STAGE) +
                   warp * NS;

  const int split = blockIdx.x;
  const int h = blockIdx.y / p.n_groups, grp = blockIdx.y % p.n_groups;
  const int b = blockIdx.z;
  const int unit = (b * p.Hkv + h) * p.n_groups + grp;

  // Scales: FP8 needs s > 0, NVFP4 g >= 0 (0 = an all-zero tensor); both finite.
  float ks = 1.f, vs = 1.f;
  bool scale_ok = true;
  if constexpr (FMT != 0) {
    ks = __ldg(p.k_scale);
    vs = __ldg(p.v_scale);
    if (FMT == 1)
      scale_ok = ks > 0.f && vs > 0.f && ks < kInf && vs < kInf;
    else
      scale_ok = ks >= 0.f && vs >= 0.f && ks < kInf && vs < kInf;
  }
  int len = __ldg(p.seq_lens + b);
  if (len < 0 || len > p.max_seq_len) {
    if (tid == 0 && split == 0 && grp == 0) set_err(p.d_err, kErrSeqLen);
    len = 0;
  }
  if (!scale_ok) {
    if (tid == 0 && split == 0 && blockIdx.y == 0 && b == 0) set_err(p.d_err, kErrScale);
    len = 0;
  }

  const int n_pages = (len + kPage - 1) / kPage;
  const int pg0 = split * p.pages_per_split;
  const int pg1 = min(pg0 + p.pages_per_split, n_pages);
  const int first = pg0 + warp;
  const int n_my = first < pg1 ? (pg1 - first + NW - 1) / NW : 0;
  const int32_t* bt = p.block_table + static_cast<size_t>(b) * p.max_blocks;

  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
    mbar_init_fence();
  }
  __syncwarp();

  // Issue the copies of this warp's i-th page into stage i % NS (lane 0).
  auto issue = [&](int i) {
    const int blk = __ldg(bt + first + i * NW);
    uint64_t* bar = &bars[i % NS];
    if (blk >= 0 && blk < p.num_blocks) {
      F::issue(stages + (i % NS) * F::STAGE, bar, &mk, &mv, &mks, &mvs, h, blk);
    } else {
      set_err(p.d_err, kErrBlockId);
      mbar_arrive(bar);  // completes the phase with no data; the page is skipped
    }
  };
  if (lane == 0) {
    const int n0 = n_my < NS ? n_my : NS;
    for (int i = 0; i < n0; ++i) issue(i);
  }

  // Query fragments (B operand of QK), head gid of this group; padded heads 0.
  const float c_log2 = p.sm_scale * ks * kLog2e;
  uint32_t qb[KS][2];
  {
    const int qi = grp * 8 + gid;
    const bool hv = qi < p.G;
    const uint16_t* qrow = p.q + (static_cast<size_t>(b) * p.Hq + h * p.G + (hv ? qi : 0)) * D;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int e0 = F::k_elem(tig, 4 * s + 2 * half);
        const uint32_t a = hv ? __ldg(qrow + e0) : 0u;
        const uint32_t c = hv ? __ldg(qrow + e0 + 1) : 0u;
        if constexpr (F::kBF16)
          qb[s][half] = a | (c << 16);
        else
          qb[s][half] = pack_f16x2(__uint_as_float(a << 16), __uint_as_float(c << 16));
      }
    }
  }

  float m0 = -kInf, m1 = -kInf, l0 = 0.f, l1 = 0.f;
  float o[MT][4];
#pragma unroll
  for (int j = 0; j < MT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;

  for (int i = 0; i < n_my; ++i) {
    const int st = i % NS;
    const int page = first + i * NW;
    const int blk = __ldg(bt + page);
    // all lanes agree on the outcome so the warp stays converged
    if (!__all_sync(0xffffffffu, mbar_wait_bounded(&bars[st], (i / NS) & 1))) {
      if (lane == 0) set_err(p.d_err, kErrTimeout);
      drain<FMT, D>(bars, i + 1, min(i + NS, n_my));
      break;
    }
    if (blk < 0 || blk >= p.num_blocks) {  // reported at issue time; skip
      __syncwarp();
      if (lane == 0 && i + NS < n_my) issue(i + NS);
      continue;
    }
    const uint8_t* sp = stages + st * F::STAGE;
    const int n_valid = min(kPage, len - page * kPage);

    // ---- S^T = K Q^T on tensor cores (two accumulator chains)
    uint32_t ka[KS][4];
    F::load_k(sp, gid, tig, ka);
    float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      if (s & 1)
        mma16816<F::kBF16>(sb, ka[s], qb[s][0], qb[s][1]);
      else
        mma16816<F::kBF16>(sa, ka[s], qb[s][0], qb[s][1]);
    }
    uint32_t va[MT][4];
    F::load_v(sp, gid, tig, va);

    // The stage is now in registers: hand it back to TMA for page i + NS.
    __syncwarp();
    if (lane == 0 && i + NS < n_my) {
      fence_proxy_async_smem();
      issue(i + NS);
    }

    float s0 = (sa[0] + sb[0]) * c_log2, s1 = (sa[1] + sb[1]) * c_log2;
    float s2 = (sa[2] + sb[2]) * c_log2, s3 = (sa[3] + sb[3]) * c_log2;
    if (n_valid < kPage) {  // last, partial page: mask tokens past the length
      if (gid >= n_valid) s0 = s1 = -kInf;
      if (gid + 8 >= n_valid) s2 = s3 = -kInf;
      const uint32_t m01 = (2 * tig < n_valid ? 0x0000FFFFu : 0u) |
                           (2 * tig + 1 < n_valid ? 0xFFFF0000u : 0u);
      const uint32_t m23 = (2 * tig + 8 < n_valid ? 0x0000FFFFu : 0u) |
                           (2 * tig + 9 < n_valid ? 0xFFFF0000u : 0u);
#pragma unroll
      for (int j = 0; j < MT; ++j) {  // unwritten slots may hold NaN codes
        va[j][0] &= m01;
        va[j][1] &= m01;
        va[j][2] &= m23;
        va[j][3] &= m23;
      }
    }

    // ---- online softmax (log2 domain); this thread: heads 2tig, 2tig+1
    float mx0 = fmaxf(s0, s2), mx1 = fmaxf(s1, s3);
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
    }
    const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
    const float a0 = fast_exp2(m0 - mn0), a1 = fast_exp2(m1 - mn1);
    m0 = mn0;
    m1 = mn1;
    const float p0 = fast_exp2(s0 - mn0), p1 = fast_exp2(s1 - mn1);
    const float p2 = fast_exp2(s2 - mn0), p3 = fast_exp2(s3 - mn1);
    l0 = l0 * a0 + (p0 + p2);
    l1 = l1 * a1 + (p1 + p3);
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      o[j][0] *= a0;
      o[j][1] *= a1;
      o[j][2] *= a0;
      o[j][3] *= a1;
    }

    // ---- P^T fragments: high part + residual, transposed in registers
    const float q0 = p0 * kPScale, q1 = p1 * kPScale, q2 = p2 * kPScale, q3 = p3 * kPScale;
    uint32_t x0h, x1h, x0l, x1l;
    float r0, r1, r2, r3;
    if constexpr (F::kBF16) {
      x0h = pack_bf16x2(q0, q1);
      x1h = pack_bf16x2(q2, q3);
      unpack_bf16x2(x0h, r0, r1);
      unpack_bf16x2(x1h, r2, r3);
      x0l = pack_bf16x2(q0 - r0, q1 - r1);
      x1l = pack_bf16x2(q2 - r2, q3 - r3);
    } else {
      x0h = pack_f16x2(q0, q1);
      x1h = pack_f16x2(q2, q3);
      unpack_f16x2(x0h, r0, r1);
      unpack_f16x2(x1h, r2, r3);
      x0l = pack_f16x2(q0 - r0, q1 - r1);
      x1l = pack_f16x2(q2 - r2, q3 - r3);
    }
    const uint32_t bh0 = movmatrix_t(x0h), bh1 = movmatrix_t(x1h);
    const uint32_t bl0 = movmatrix_t(x0l), bl1 = movmatrix_t(x1l);

    // ---- O^T += V^T P^T
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      mma16816<F::kBF16>(o[j], va[j], bh0, bh1);
      mma16816<F::kBF16>(o[j], va[j], bl0, bl1);
    }
  }

  // ---- warp partial -> shared memory (this warp's own, now idle, stages)
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  __syncwarp();
  float* wml = reinterpret_cast<float*>(stages);  // m[8], l[8], o[8][D]
  if (gid == 0) {
    wml[2 * tig] = m0;
    wml[2 * tig + 1] = m1;
    wml[8 + 2 * tig] = l0;
    wml[8 + 2 * tig + 1] = l1;
  }
  float* wo = wml + 16;
#pragma unroll
  for (int j = 0; j < MT; ++j) {
    const int d0 = F::v_elem(gid, 2 * j), d1 = F::v_elem(gid, 2 * j + 1);
    wo[(2 * tig) * D + d0] = o[j][0];
    wo[(2 * tig + 1) * D + d0] = o[j][1];
    wo[(2 * tig) * D + d1] = o[j][2];
    wo[(2 * tig + 1) * D + d1] = o[j][3];
  }
  __syncthreads();

  // ---- merge the warps: (M, L, O) of the CTA for each of the 8 heads
  constexpr int WSTRIDE = NS * F::STAGE / 4;  // floats between warp partials
  const float* base = reinterpret_cast<const float*>(smem);
  for (int idx = tid; idx < 8 * D; idx += NW * 32) {
    const int hh = idx / D, d = idx - hh * D;
    float M = -kInf;
#pragma unroll
    for (int w = 0; w < NW; ++w) M = fmaxf(M, base[w * WSTRIDE + hh]);
    float L = 0.f, acc = 0.f;
    if (M != -kInf) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float e = fast_exp2(base[w * WSTRIDE + hh] - M);
        L += e * base[w * WSTRIDE + 8 + hh];
        acc += e * base[w * WSTRIDE + 16 + hh * D + d];
      }
    }
    if (p.num_splits == 1) {
      const int qi = grp * 8 + hh;
      if (qi < p.G) {
        const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + qi;
        p.out[row * D + d] = L > 0.f ? acc * (vs / (L * kPScale)) : 0.f;
        if (d == 0 && p.lse) p.lse[row] = L > 0.f ? (M + log2f(L)) * kLn2 : -kInf;
      }
    } else {
      const size_t pi = (static_cast<size_t>(unit) * p.num_splits + split) * 8 + hh;
      p.ws_o[pi * D + d] = acc;
      if (d == 0) {
        p.ws_ml[pi * 2] = M;
        p.ws_ml[pi * 2 + 1] = L;
      }
    }
  }
  if (p.num_splits == 1) return;

  // ---- split-K merge by the last CTA of this (sequence, KV head, group)
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned t = atomicAdd(p.ws_cnt + unit, 1u);
    s_last = (t == static_cast<unsigned>(p.num_splits - 1));
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  const int S = p.num_splits;
  const size_t ubase = static_cast<size_t>(unit) * S * 8;
  float* wgt = reinterpret_cast<float*>(smem);  // [8][S] weights, then M[8], L[8]
  float* hM = wgt + 8 * kMaxSplits;
  float* hL = hM + 8;
  // per head: M = max_s m_s, L = sum_s 2^(m_s - M) l_s (one warp per head)
  for (int hh = warp; hh < 8; hh += NW) {
    float M = -kInf;
    for (int s = lane; s < S; s += 32) M = fmaxf(M, __ldcg(p.ws_ml + (ubase + s * 8 + hh) * 2));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float L = 0.f;
    for (int s = lane; s < S; s += 32) {
      const float ms = __ldcg(p.ws_ml + (ubase + s * 8 + hh) * 2);
      const float e = M != -kInf ? fast_exp2(ms - M) : 0.f;
      wgt[hh * kMaxSplits + s] = e;
      L += e * __ldcg(p.ws_ml + (ubase + s * 8 + hh) * 2 + 1);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) L += __shfl_xor_sync(0xffffffffu, L, off);
    if (lane == 0) {
      hM[hh] = M;
      hL[hh] = L;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < 8 * D; idx += NW * 32) {
    const int hh = idx / D, d = idx - hh * D;
    const int qi = grp * 8 + hh;
    if (qi >= p.G) continue;
    float acc = 0.f;
    for (int s = 0; s < S; ++s)
      acc += wgt[hh * kMaxSplits + s] * __ldcg(p.ws_o + (ubase + s * 8 + hh) * D + d);
    const float L = hL[hh];
    const size_t row = static_cast<size_t>(b) * p.Hq + h * p.G + qi;
    p.out[row * D + d] = L > 0.f ? acc * (vs / (L * kPScale)) : 0.f;
    if (d == 0 && p.lse) p.lse[row] = L > 0.f ? (hM[hh] + log2f(L)) * kLn2 : -kInf;
  }
  if (tid == 0) p.ws_cnt[unit] = 0u;  // leave the counter ready for the next launch
}

template <int FMT, int D>
size_t smem_bytes() {
  using F = Fmt<FMT, D>;
  constexpr int NW = Shape<FMT, D>::NW, NS = Shape<FMT, D>::NS;
  size_t stages = static_cast<size_t>(NW) * NS * F::STAGE;
  size_t merge = (8 * kMaxSplits + 16) * sizeof(float);
  size_t body = stages > merge ? stages : merge;
  return 1024 + body + static_cast<size_t>(NW) * NS * 8;
}

template <int FMT, int D>
cudaError_t launch_t(const CUtensorMap* maps, const DecodeParams& p, cudaStream_t stream) {
  constexpr int NW = Shape<FMT, D>::NW;
  const size_t smem = smem_bytes<FMT, D>();
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kvq_decode_kernel<FMT, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(p.num_splits, p.Hkv * p.n_groups, p.B);
  kvq_decode_kernel<FMT, D><<<grid, NW * 32, smem, stream>>>(maps[0], maps[1], maps[2], maps[3], p);
  return cudaGetLastError();
}

template <int FMT, int D>
int occupancy_t() {
  constexpr int NW = Shape<FMT, D>::NW;
  const size_t smem = smem_bytes<FMT, D>();
  cudaFuncSetAttribute(kvq_decode_kernel<FMT, D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kvq_decode_kernel<FMT, D>, NW * 32, smem) !=
      cudaSuccess)
    return 0;
  return n;
}

template <int FMT, int D>
void config_t(DecodeConfig* c) {
  c->warps = Shape<FMT, D>::NW;
  c->stages = Shape<FMT, D>::NS;
  c->stage_bytes = Fmt<FMT, D>::STAGE;
  c->smem_bytes = smem_bytes<FMT, D>();
}

}  // namespace

bool decode_config(int fmt, int D, DecodeConfig* cfg) {
  if (D != 64 && D != 128) return false;
  switch (fmt * 1000 + D) {
    case 64: config_t<0, 64>(cfg); return true;
    case 128: config_t<0, 128>(cfg); return true;
    case 1064: config_t<1, 64>(cfg); return true;
    case 1128: config_t<1, 128>(cfg); return true;
    case 2064: config_t<2, 64>(cfg); return true;
    case 2128: config_t<2, 128>(cfg); return true;
  }
  return false;
}

int decode_ctas_per_sm(int fmt, int D) {
  static int cache[3][2] = {{-1, -1}, {-1, -1}, {-1, -1}};
  const int di = D == 64 ? 0 : 1;
  if (fmt < 0 || fmt > 2) return 0;
  if (cache[fmt][di] >= 0) return cache[fmt][di];
  int n = 0;
  switch (fmt * 1000 + D) {
    case 64: n = occupancy_t<0, 64>(); break;
    case 128: n = occupancy_t<0, 128>(); break;
    case 1064: n = occupancy_t<1, 64>(); break;
    case 1128: n = occupancy_t<1, 128>(); break;
    case 2064: n = occupancy_t<2, 64>(); break;
    case 2128: n = occupancy_t<2, 128>(); break;
  }
  cache[fmt][di] = n;
  return n;
}

cudaError_t launch_decode(int fmt, int D, const CUtensorMap* maps, const DecodeParams& p,
                          cudaStream_t stream) {
  switch (fmt * 1000 + D) {
    case 64: return launch_t<0, 64>(maps, p, stream);
    case 128: return launch_t<0, 128>(maps, p, stream);
    case 1064: return launch_t<1, 64>(maps, p, stream);
    case 1128: return launch_t<1, 128>(maps, p, stream);
    case 2064: return launch_t<2, 64>(maps, p, stream);
    case 2128: return launch_t<2, 128>(maps, p, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
