// kvq_quant.cu -- calibration abs-max, per-layer scale, quantize-on-write into
// the paged cache (FP8 E4M3, NVFP4, BF16) and dequantisation of chosen slots.
//
// Formulas ("FP8 KV calibration guide", Radiance calibrator paragraph; NVFP4
// per "I Tested NVFP4 vs FP8 KV Cache on Blackwell", "What you'll learn", with
// 16-element E2M1 blocks along head_dim and an E4M3 block scale):
//   FP8  : s = max(amax * 1.05 / 448, 1e-12); code = E4M3_rne_sat(x / s)
//   NVFP4: g = amax / 2688; per block sb = E4M3_rne_sat(bmax / (6 g)),
//          code_i = E2M1_rne_sat(x_i / (E4M3(sb) * g))  (+0 if that is 0)
// All divisions are IEEE fp32 divisions (no reciprocal approximation), so
// codes and scales are bit-identical to a plain CPU evaluation.
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {

namespace {

#define kInf __int_as_float(0x7f800000)

// Resolve token t's slot: physical slot, or logical (seq * max_blocks * 16 +
// position) translated through the block table.  Returns -1 to skip.
__device__ __forceinline__ int64_t resolve_slot(const QuantParams& p, int64_t t) {
  int64_t s = __ldg(p.slot_mapping + t);
  if (s < 0) return -1;
  if (p.block_table) {
    const int64_t span = static_cast<int64_t>(p.max_blocks) * kPage;
    const int64_t seq = s / span, pos = s - seq * span;
    if (seq >= p.num_seqs) {
      set_err(p.d_err, kErrSlot);
      return -1;
    }
    const int32_t blk = __ldg(p.block_table + seq * p.max_blocks + pos / kPage);
    if (blk < 0 || blk >= p.num_blocks) {
      set_err(p.d_err, kErrBlockId);
      return -1;
    }
    s = static_cast<int64_t>(blk) * kPage + pos % kPage;
  }
  if (s / kPage >= p.num_blocks) {
    set_err(p.d_err, kErrSlot);
    return -1;
  }
  return s;
}

// The write kernels give each block `tpb` (<= kTokPerBlock) tokens, grid-
// strided: the block's first threads resolve the tokens' slots in parallel
// (one dependent load chain per block), then every thread takes chunks of
// the tokens' 2 (K, V) x H rows x (D/8 or D/16) columns, kBatch (NVFP4:
// kBatchNv) at a time with all their loads issued before any convert or store.
constexpr int kTokPerBlock = 8;
constexpr int kBatch = 4;
constexpr int kBatchNv = 2;  // NVFP4 chunks hold 2x the registers

struct TokSlots {
  int64_t slot[kTokPerBlock];
};

__device__ __forceinline__ void block_slots(const QuantParams& p, int64_t t0, int tpb,
                                            TokSlots& s) {
  if (threadIdx.x < tpb)
    s.slot[threadIdx.x] = t0 + threadIdx.x < p.T ? resolve_slot(p, t0 + threadIdx.x) : -1;
  __syncthreads();
}

// Chunk ii of the block's tokens: token tt, K or V (kv), head h, column c.
struct Chunk {
  int64_t t, slot;
  int kv, h, c;
};
__device__ __forceinline__ Chunk chunk_of(const TokSlots& ts, int64_t t0, int ii, int n,
                                          int per_kv, int lg) {
  Chunk q;
  const int tt = ii / n, i = ii - tt * n;
  q.t = t0 + tt;
  q.slot = ts.slot[tt];
  q.kv = i >= per_kv;
  const int j = i - q.kv * per_kv;
  q.h = j >> lg;
  q.c = j & ((1 << lg) - 1);
  return q;
}

// One chunk = 8 elements of one (K|V, head) row of a token.
__global__ void quantize_fp8_kernel(const QuantParams p, int tpb) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int lg = p.D == 128 ? 4 : 3, per_kv = p.H << lg, n = 2 * per_kv, total = tpb * n;
  const float ks = __ldg(p.k_scale), vs = __ldg(p.v_scale);
  const bool ok_k = ks > 0.f && ks < kInf, ok_v = vs > 0.f && vs < kInf;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !(ok_k && ok_v)) set_err(p.d_err, kErrScale);
  __shared__ TokSlots ts;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * tpb; t0 < p.T;
       t0 += static_cast<int64_t>(gridDim.x) * tpb) {
    block_slots(p, t0, tpb, ts);
    for (int ii0 = threadIdx.x; ii0 < total; ii0 += kBatch * blockDim.x) {
      uint4 x[kBatch];
      uint8_t* dst[kBatch];
      float sc[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        dst[u] = nullptr;
        const int ii = ii0 + u * blockDim.x;
        if (ii >= total) continue;
        const Chunk q = chunk_of(ts, t0, ii, n, per_kv, lg);
        if (q.slot < 0 || !(q.kv ? ok_v : ok_k)) continue;
        sc[u] = q.kv ? vs : ks;
        x[u] = __ldg(reinterpret_cast<const uint4*>((q.kv ? p.v : p.k) +
                                                    (q.t * p.H + q.h) * p.D + 8 * q.c));
        dst[u] = (q.kv ? p.vc : p.kc) +
                 ((q.slot / kPage * p.H + q.h) * kPage + q.slot % kPage) * p.D + 8 * q.c;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        if (!dst[u]) continue;
        const uint32_t w[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
        uint32_t code[4];
#pragma unroll
        for (int e = 0; e < 4; ++e)
          code[e] = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(w[e]), sc[u]),
                                    __fdiv_rn(bf16_hi(w[e]), sc[u]));
        *reinterpret_cast<uint2*>(dst[u]) =
            make_uint2(code[0] | (code[1] << 16), code[2] | (code[3] << 16));
      }
    }
    __syncthreads();  // ts is rewritten for the next tokens
  }
}

// One chunk = one 16-element block of one (K|V, head) row of a token.
__global__ void quantize_nvfp4_kernel(const QuantParams p, int tpb) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int lg = p.D == 128 ? 3 : 2, per_kv = p.H << lg, n = 2 * per_kv, total = tpb * n;
  const float gk = __ldg(p.k_scale), gv = __ldg(p.v_scale);
  const bool ok_k = gk >= 0.f && gk < kInf, ok_v = gv >= 0.f && gv < kInf;
  if (blockIdx.x == 0 && threadIdx.x == 0 && !(ok_k && ok_v)) set_err(p.d_err, kErrScale);
  __shared__ TokSlots ts;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * tpb; t0 < p.T;
       t0 += static_cast<int64_t>(gridDim.x) * tpb) {
    block_slots(p, t0, tpb, ts);
    for (int ii0 = threadIdx.x; ii0 < total; ii0 += kBatchNv * blockDim.x) {
      uint4 x0[kBatchNv], x1[kBatchNv];
      uint8_t* page[kBatchNv];
      float gg[kBatchNv];
      int o[kBatchNv], blk16[kBatchNv];
#pragma unroll
      for (int u = 0; u < kBatchNv; ++u) {
        page[u] = nullptr;
        const int ii = ii0 + u * blockDim.x;
        if (ii >= total) continue;
        const Chunk q = chunk_of(ts, t0, ii, n, per_kv, lg);
        if (q.slot < 0 || !(q.kv ? ok_v : ok_k)) continue;
        gg[u] = q.kv ? gv : gk;
        const uint4* src = reinterpret_cast<const uint4*>((q.kv ? p.v : p.k) +
                                                          (q.t * p.H + q.h) * p.D + 16 * q.c);
        x0[u] = __ldg(src);
        x1[u] = __ldg(src + 1);
        page[u] = (q.kv ? p.vc : p.kc) +
                  (q.slot / kPage * p.H + q.h) * static_cast<int64_t>(9 * p.D);
        o[u] = static_cast<int>(q.slot % kPage);
        blk16[u] = q.c;
      }
#pragma unroll
      for (int u = 0; u < kBatchNv; ++u) {
        if (!page[u]) continue;
        const float g = gg[u];
        const uint32_t w[8] = {x0[u].x, x0[u].y, x0[u].z, x0[u].w,
                               x1[u].x, x1[u].y, x1[u].z, x1[u].w};
        float v[16];
        float bmax = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          v[2 * e] = bf16_lo(w[e]);
          v[2 * e + 1] = bf16_hi(w[e]);
          bmax = fmaxf(bmax, fmaxf(fabsf(v[2 * e]), fabsf(v[2 * e + 1])));
        }
        uint32_t sb = 0, codes_lo = 0, codes_hi = 0;
        if (g > 0.f) {
          sb = f32x2_to_e4m3x2(__fdiv_rn(bmax, __fmul_rn(6.0f, g)), 0.f) & 0xFFu;
          const float den = __fmul_rn(e4m3_to_f32(sb), g);
          if (den != 0.f) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              codes_lo |= f32x2_to_e2m1x2(__fdiv_rn(v[2 * e], den),
                                          __fdiv_rn(v[2 * e + 1], den))
                          << (8 * e);
              codes_hi |= f32x2_to_e2m1x2(__fdiv_rn(v[8 + 2 * e], den),
                                          __fdiv_rn(v[9 + 2 * e], den))
                          << (8 * e);
            }
          }
        }
        *reinterpret_cast<uint2*>(page[u] + o[u] * (p.D / 2) + 8 * blk16[u]) =
            make_uint2(codes_lo, codes_hi);
        page[u][8 * p.D + o[u] * (p.D / 16) + blk16[u]] = static_cast<uint8_t>(sb);
      }
    }
    __syncthreads();  // ts is rewritten for the next tokens
  }
}

// One chunk = 8 elements (16 bytes) of one (K|V, head) row of a token.
__global__ void write_bf16_kernel(const QuantParams p, int tpb) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int lg = p.D == 128 ? 4 : 3, per_kv = p.H << lg, n = 2 * per_kv, total = tpb * n;
  __shared__ TokSlots ts;
  for (int64_t t0 = static_cast<int64_t>(blockIdx.x) * tpb; t0 < p.T;
       t0 += static_cast<int64_t>(gridDim.x) * tpb) {
    block_slots(p, t0, tpb, ts);
    for (int ii0 = threadIdx.x; ii0 < total; ii0 += kBatch * blockDim.x) {
      uint4 x[kBatch];
      uint8_t* dst[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        dst[u] = nullptr;
        const int ii = ii0 + u * blockDim.x;
        if (ii >= total) continue;
        const Chunk q = chunk_of(ts, t0, ii, n, per_kv, lg);
        if (q.slot < 0) continue;
        x[u] = __ldg(reinterpret_cast<const uint4*>((q.kv ? p.v : p.k) +
                                                    (q.t * p.H + q.h) * p.D + 8 * q.c));
        dst[u] = (q.kv ? p.vc : p.kc) +
                 (((q.slot / kPage * p.H + q.h) * kPage + q.slot % kPage) * p.D + 8 * q.c) * 2;
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u)
        if (dst[u]) *reinterpret_cast<uint4*>(dst[u]) = x[u];
    }
    __syncthreads();  // ts is rewritten for the next tokens
  }
}

// One thread = 8 elements of one (slot, K|V, head) row.
__global__ void dequantize_kernel(int fmt, const uint8_t* kc, const uint8_t* vc,
                                  int64_t num_blocks, int H, int D, const int64_t* slots,
                                  int64_t n, const float* ks, const float* vs, float* ko,
                                  float* vo, int* d_err) {
  const int cpr = D / 8;
  const int64_t total = n * 2 * H * cpr;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % cpr);
  int64_t r = idx / cpr;
  const int h = static_cast<int>(r % H);
  r /= H;
  const int kv = static_cast<int>(r & 1);
  const int64_t i = r >> 1;
  const int64_t slot = __ldg(slots + i);
  if (slot < 0 || slot / kPage >= num_blocks) {
    if (c == 0 && h == 0 && kv == 0) set_err(d_err, kErrSlot);
    return;
  }
  const int64_t blk = slot / kPage;
  const int o = static_cast<int>(slot % kPage);
  float* out = (kv ? vo : ko) + (i * H + h) * D + 8 * c;
  float v[8];
  if (fmt == 0) {
    const uint16_t* src = reinterpret_cast<const uint16_t*>(kv ? vc : kc) +
                          ((blk * H + h) * kPage + o) * D + 8 * c;
    const uint4 x = *reinterpret_cast<const uint4*>(src);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      v[2 * k] = bf16_lo(w[k]);
      v[2 * k + 1] = bf16_hi(w[k]);
    }
  } else if (fmt == 1) {
    const float s = __ldg(kv ? vs : ks);
    const uint8_t* src = (kv ? vc : kc) + ((blk * H + h) * kPage + o) * D + 8 * c;
    const uint2 x = *reinterpret_cast<const uint2*>(src);
    const uint32_t w[2] = {x.x, x.y};
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      uint32_t lo, hi;
      e4m3x4_to_f16x2x2(w[k], lo, hi);
      float a, b, cc, d;
      unpack_f16x2(lo, a, b);
      unpack_f16x2(hi, cc, d);
      v[4 * k] = __fmul_rn(a, s);
      v[4 * k + 1] = __fmul_rn(b, s);
      v[4 * k + 2] = __fmul_rn(cc, s);
      v[4 * k + 3] = __fmul_rn(d, s);
    }
  } else {
    const float g = __ldg(kv ? vs : ks);
    const uint8_t* page = (kv ? vc : kc) + (blk * H + h) * static_cast<int64_t>(9 * D);
    const uint32_t codes = *reinterpret_cast<const uint32_t*>(page + o * (D / 2) + 4 * c);
    const float sb = e4m3_to_f32(page[8 * D + o * (D / 16) + (8 * c) / 16]);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __fmul_rn(__fmul_rn(e2m1_to_f32(codes >> (4 * k)), sb), g);
  }
  reinterpret_cast<float4*>(out)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(out)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// ------------------------------------------------------------------ PQ3
// 3-bit planar-rotation codec of 128-element vectors ("AMD MI300X - KV Cache
// Compression Benchmark", "Key Results": 52-byte blocks, 4.923x against FP16;
// the planar rotation's 256 FMAs; a Lloyd-Max codebook).  Head page: 16 fp32
// norms, then 16 rows of 48 bytes of 3-bit indices in two bit planes (see
// the writer below).  Parameter block of a tensor:
// 8 ascending codebook values, then 64 (cos, sin) pairs.
constexpr int kPq3Page = 832;

// The codebook must be finite and ascending; anything else is a bad scale.
__device__ __forceinline__ bool pq3_params_ok(const float* cb) {
  bool ok = true;
#pragma unroll
  for (int k = 0; k < 7; ++k) ok = ok && cb[k] < cb[k + 1];
  return ok && cb[0] > -kInf && cb[7] < kInf;
}

// One warp per (token, K|V, head) row; lane l holds elements 4l .. 4l+3.
// Every fp32 step is the format's fixed one: the sum of squares as a
// pairwise tree in index order (elements, then pairs, then the lanes'
// butterfly), sqrt and division rounded to nearest, the rotation's explicit
// roundings, and the index as the count of thresholds below y.
__global__ void quantize_pq3_kernel(const QuantParams p) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const int64_t rows = p.T * 2 * p.H;
  for (int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += nwarps) {
    const int64_t t = r / (2 * p.H);
    const int rem = static_cast<int>(r - t * 2 * p.H), kv = rem / p.H, h = rem - kv * p.H;
    int64_t slot = -1;
    if (lane == 0) slot = resolve_slot(p, t);  // errors reported once
    slot = __shfl_sync(0xffffffffu, slot, 0);
    if (slot < 0) continue;
    const float* prm = kv ? p.v_scale : p.k_scale;
    float cb[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) cb[k] = __ldg(prm + k);
    if (!pq3_params_ok(cb)) {
      if (lane == 0) set_err(p.d_err, kErrScale);
      continue;
    }
    const uint16_t* x = (kv ? p.v : p.k) + (t * p.H + h) * 128;
    const uint2 w = *reinterpret_cast<const uint2*>(x + 4 * lane);
    const float x0 = bf16_lo(w.x), x1 = bf16_hi(w.x), x2 = bf16_lo(w.y), x3 = bf16_hi(w.y);
    float ss = __fadd_rn(__fadd_rn(__fmul_rn(x0, x0), __fmul_rn(x1, x1)),
                         __fadd_rn(__fmul_rn(x2, x2), __fmul_rn(x3, x3)));
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) ss = __fadd_rn(ss, __shfl_xor_sync(0xffffffffu, ss, off));
    const float nrm = __fsqrt_rn(ss);
    uint32_t code = 0;  // this lane's 4 indices, 3 bits each
    if (nrm != 0.f) {
      const float u[4] = {__fdiv_rn(x0, nrm), __fdiv_rn(x1, nrm), __fdiv_rn(x2, nrm),
                          __fdiv_rn(x3, nrm)};
      float thr[7];
#pragma unroll
      for (int k = 0; k < 7; ++k) thr[k] = __fmul_rn(__fadd_rn(cb[k], cb[k + 1]), 0.5f);
#pragma unroll
      for (int pr = 0; pr < 2; ++pr) {  // pairs j = 2 lane + pr: elements 2j, 2j+1
        const int j = 2 * lane + pr;
        const float c = __ldg(prm + 8 + 2 * j), sn = __ldg(prm + 9 + 2 * j);
        const float u0 = u[2 * pr], u1 = u[2 * pr + 1];
        const float y[2] = {__fmaf_rn(c, u0, -__fmul_rn(sn, u1)),
                            __fmaf_rn(sn, u0, __fmul_rn(c, u1))};
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          uint32_t k = 0;
#pragma unroll
          for (int q = 0; q < 7; ++q) k += y[e] > thr[q] ? 1u : 0u;
          code |= k << (3 * (2 * pr + e));
        }
      }
    }
    // The row's two bit planes (12 little-endian words): low word w holds
    // the low 2 bits of indices 16w + e at bit 4 (e % 8) + 2 (e / 8), high
    // word v (words 8..11) bit 2 of indices 32v + e at bit 4 (e % 8) +
    // (2, 3, 0, 1)[e / 8].  Lane l's indices 4l .. 4l+3 fall in low word l / 4
    // and high word l / 8; the lanes of a word OR their disjoint bits.
    uint32_t low = 0, high = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t ix = (code >> (3 * q)) & 7u;
      const int el = 4 * (lane & 3) + q, eh = 4 * (lane & 7) + q;
      low |= (ix & 3u) << (4 * (el & 7) + 2 * (el >> 3));
      high |= (ix >> 2) << (4 * (eh & 7) + ((eh >> 3) ^ 2));
    }
    low |= __shfl_xor_sync(0xffffffffu, low, 1);
    low |= __shfl_xor_sync(0xffffffffu, low, 2);
    high |= __shfl_xor_sync(0xffffffffu, high, 1);
    high |= __shfl_xor_sync(0xffffffffu, high, 2);
    high |= __shfl_xor_sync(0xffffffffu, high, 4);
    uint8_t* page = (kv ? p.vc : p.kc) +
                    ((slot / kPage) * p.H + h) * static_cast<int64_t>(kPq3Page);
    const int o = static_cast<int>(slot % kPage);
    uint32_t* row = reinterpret_cast<uint32_t*>(page + 64 + 48 * o);
    if ((lane & 3) == 0) row[lane >> 2] = low;
    if ((lane & 7) == 0) row[8 + (lane >> 3)] = high;
    if (lane == 0) *reinterpret_cast<float*>(page + 4 * o) = nrm;
  }
}

// The dequantised fp32 row of a PQ3 slot: x_hat_2j = nrm * fma(cos, Y0, sin *
// Y1), x_hat_2j+1 = nrm * fma(cos, Y1, -(sin * Y0)).  One warp per (slot, K|V,
// head) row, lane l writing elements 4l .. 4l+3.
__global__ void dequantize_pq3_kernel(const uint8_t* kc, const uint8_t* vc, int64_t num_blocks,
                                      int H, const int64_t* slots, int64_t n, const float* ks,
                                      const float* vs, float* ko, float* vo, int* d_err) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (r >= n * 2 * H) return;
  const int h = static_cast<int>(r % H), kv = static_cast<int>((r / H) & 1);
  const int64_t i = r / (2 * H);
  const int64_t slot = __ldg(slots + i);
  if (slot < 0 || slot / kPage >= num_blocks) {
    if (lane == 0 && h == 0 && kv == 0) set_err(d_err, kErrSlot);
    return;
  }
  const float* prm = kv ? vs : ks;
  const uint8_t* page = (kv ? vc : kc) + ((slot / kPage) * H + h) * static_cast<int64_t>(kPq3Page);
  const int o = static_cast<int>(slot % kPage);
  const float nrm = *reinterpret_cast<const float*>(page + 4 * o);
  const uint32_t* row = reinterpret_cast<const uint32_t*>(page + 64 + 48 * o);
  // indices 4 lane .. 4 lane + 3 from the row's bit planes (see the writer)
  const uint32_t low = row[lane >> 2], high = row[8 + (lane >> 3)];
  uint32_t code = 0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int el = 4 * (lane & 3) + q, eh = 4 * (lane & 7) + q;
    const uint32_t ix = ((low >> (4 * (el & 7) + 2 * (el >> 3))) & 3u) |
                        (((high >> (4 * (eh & 7) + ((eh >> 3) ^ 2))) & 1u) << 2);
    code |= ix << (3 * q);
  }
  float v[4];
#pragma unroll
  for (int pr = 0; pr < 2; ++pr) {
    const int j = 2 * lane + pr;
    const float c = __ldg(prm + 8 + 2 * j), sn = __ldg(prm + 9 + 2 * j);
    const float y0 = __ldg(prm + ((code >> (6 * pr)) & 7u));
    const float y1 = __ldg(prm + ((code >> (6 * pr + 3)) & 7u));
    v[2 * pr] = __fmul_rn(nrm, __fmaf_rn(c, y0, __fmul_rn(sn, y1)));
    v[2 * pr + 1] = __fmul_rn(nrm, __fmaf_rn(c, y1, -__fmul_rn(sn, y0)));
  }
  float* out = (kv ? vo : ko) + (i * H + h) * 128 + 4 * lane;
  *reinterpret_cast<float4*>(out) = make_float4(v[0], v[1], v[2], v[3]);
}

// Per-16-bit-lane max of the magnitude bits of 8 BF16 values.
__device__ __forceinline__ uint32_t absmax8(const uint4 a) {
  const uint32_t k = 0x7FFF7FFFu;
  return __vmaxu2(__vmaxu2(a.x & k, a.y & k), __vmaxu2(a.z & k, a.w & k));
}

// Abs-max of BF16 values as the max of their 15 magnitude bits (exact and
// order-free: for non-NaN BF16, magnitude order equals integer order).
__global__ void absmax_kernel(const uint16_t* x, int64_t n, int64_t head, float* d_amax) {
  uint32_t m = 0;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t nthreads = static_cast<int64_t>(gridDim.x) * blockDim.x;
  // scalar head (until 16-byte alignment) and tail
  for (int64_t i = tid; i < head && i < n; i += nthreads) m = max(m, (uint32_t)(x[i] & 0x7FFFu));
  const int64_t nvec = (n - head) / 8;
  const uint4* xv = reinterpret_cast<const uint4*>(x + head);
  uint32_t mm = 0;
  int64_t i = tid;
  for (; i + 3 * nthreads < nvec; i += 4 * nthreads) {
    const uint4 a = __ldcs(xv + i), b = __ldcs(xv + i + nthreads);
    const uint4 c = __ldcs(xv + i + 2 * nthreads), d = __ldcs(xv + i + 3 * nthreads);
    mm = __vmaxu2(mm, absmax8(a));
    mm = __vmaxu2(mm, absmax8(b));
    mm = __vmaxu2(mm, absmax8(c));
    mm = __vmaxu2(mm, absmax8(d));
  }
  for (; i < nvec; i += nthreads) mm = __vmaxu2(mm, absmax8(__ldcs(xv + i)));
  m = max(m, max(mm & 0xFFFFu, mm >> 16));
  for (int64_t k = head + nvec * 8 + tid; k < n; k += nthreads) m = max(m, (uint32_t)(x[k] & 0x7FFFu));
  m = __reduce_max_sync(0xffffffffu, m);
  __shared__ uint32_t wmax[32];
  if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    uint32_t v = threadIdx.x < (blockDim.x >> 5) ? wmax[threadIdx.x] : 0u;
    v = __reduce_max_sync(0xffffffffu, v);
    if (threadIdx.x == 0 && v) atomicMax(reinterpret_cast<unsigned*>(d_amax), v << 16);
  }
}

__global__ void scale_kernel(int fmt, const float* d_amax, float* d_scale) {
  const float amax = *d_amax;
  float s = 1.0f;
  if (fmt == 1) {
    s = __fdiv_rn(__fmul_rn(amax, 1.05f), 448.0f);
    if (s < 1e-12f) s = 1e-12f;
  } else if (fmt == 2) {
    s = __fdiv_rn(amax, 2688.0f);
  }
  *d_scale = s;
}

unsigned grid_for(int64_t total, int threads) {
  return static_cast<unsigned>((total + threads - 1) / threads);
}

}  // namespace

cudaError_t launch_quantize(int fmt, const QuantParams& p, cudaStream_t stream) {
  if (p.T == 0) return cudaSuccess;
  // Tokens per block: as many as keep >= 4 blocks per SM (so a short write
  // stays spread over SMs, a long one pays one slot lookup chain per block).
  const int threads = 256;
  int tpb = 1;
  while (tpb < kTokPerBlock && p.T / (2 * tpb) >= 4 * static_cast<int64_t>(num_sms())) tpb *= 2;
  const int64_t blocks = (p.T + tpb - 1) / tpb;
  const unsigned grid = static_cast<unsigned>(blocks < (1 << 20) ? blocks : (1 << 20));
  if (fmt == 3) {  // one warp per row
    const int64_t rows = p.T * 2 * p.H;
    const int64_t cap = static_cast<int64_t>(num_sms()) * 16;
    const int64_t b = (rows + 7) / 8;
    quantize_pq3_kernel<<<static_cast<unsigned>(b < cap ? b : cap), threads, 0, stream>>>(p);
  } else if (fmt == 1) {
    quantize_fp8_kernel<<<grid, threads, 0, stream>>>(p, tpb);
  } else if (fmt == 2) {
    quantize_nvfp4_kernel<<<grid, threads, 0, stream>>>(p, tpb);
  } else {
    write_bf16_kernel<<<grid, threads, 0, stream>>>(p, tpb);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(int fmt, const uint8_t* kc, const uint8_t* vc, int64_t num_blocks,
                              int H, int D, const int64_t* slots, int64_t n, const float* ks,
                              const float* vs, float* ko, float* vo, int* d_err,
                              cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  if (fmt == 3) {
    dequantize_pq3_kernel<<<grid_for(n * 2 * H * 32, threads), threads, 0, stream>>>(
        kc, vc, num_blocks, H, slots, n, ks, vs, ko, vo, d_err);
    return cudaGetLastError();
  }
  dequantize_kernel<<<grid_for(n * 2 * H * (D / 8), threads), threads, 0, stream>>>(
      fmt, kc, vc, num_blocks, H, D, slots, n, ks, vs, ko, vo, d_err);
  return cudaGetLastError();
}

cudaError_t launch_absmax(const uint16_t* x, int64_t n, float* d_amax, cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const uintptr_t addr = reinterpret_cast<uintptr_t>(x);
  int64_t head = static_cast<int64_t>(((16 - (addr & 15)) & 15) / 2);
  if (head > n) head = n;
  const int threads = 512;
  const int64_t per_cta = static_cast<int64_t>(threads) * 8 * 4;
  int64_t blocks = (n + per_cta - 1) / per_cta;
  const int64_t cap = static_cast<int64_t>(num_sms()) * 4;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  absmax_kernel<<<static_cast<unsigned>(blocks), threads, 0, stream>>>(x, n, head, d_amax);
  return cudaGetLastError();
}

cudaError_t launch_scale(int fmt, const float* d_amax, float* d_scale, cudaStream_t stream) {
  scale_kernel<<<1, 1, 0, stream>>>(fmt, d_amax, d_scale);
  return cudaGetLastError();
}

}  // namespace kvq
