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

// One thread = 8 elements of one (token, K|V, head) row.
__global__ void quantize_fp8_kernel(const QuantParams p) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int cpr = p.D / 8;  // chunks per row
  const int64_t total = p.T * 2 * p.H * cpr;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % cpr);
  int64_t r = idx / cpr;
  const int h = static_cast<int>(r % p.H);
  r /= p.H;
  const int kv = static_cast<int>(r & 1);
  const int64_t t = r >> 1;
  const float s = __ldg(kv ? p.v_scale : p.k_scale);
  if (!(s > 0.f && s < kInf)) {
    if (idx == 0 || idx == cpr * p.H) set_err(p.d_err, kErrScale);
    return;
  }
  const int64_t slot = resolve_slot(p, t);
  if (slot < 0) return;
  const uint16_t* src = (kv ? p.v : p.k) + (t * p.H + h) * p.D + 8 * c;
  const uint4 x = __ldg(reinterpret_cast<const uint4*>(src));
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
  uint32_t code[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    code[i] = f32x2_to_e4m3x2(__fdiv_rn(bf16_lo(w[i]), s), __fdiv_rn(bf16_hi(w[i]), s));
  uint8_t* dst = (kv ? p.vc : p.kc) +
                 ((slot / kPage * p.H + h) * kPage + slot % kPage) * p.D + 8 * c;
  *reinterpret_cast<uint2*>(dst) = make_uint2(code[0] | (code[1] << 16), code[2] | (code[3] << 16));
}

// One thread = one 16-element block of one (token, K|V, head) row.
__global__ void quantize_nvfp4_kernel(const QuantParams p) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int bpr = p.D / 16;  // blocks per row
  const int64_t total = p.T * 2 * p.H * bpr;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int blk16 = static_cast<int>(idx % bpr);
  int64_t r = idx / bpr;
  const int h = static_cast<int>(r % p.H);
  r /= p.H;
  const int kv = static_cast<int>(r & 1);
  const int64_t t = r >> 1;
  const float g = __ldg(kv ? p.v_scale : p.k_scale);
  if (!(g >= 0.f && g < kInf)) {
    if (idx == 0 || idx == bpr * p.H) set_err(p.d_err, kErrScale);
    return;
  }
  const int64_t slot = resolve_slot(p, t);
  if (slot < 0) return;
  const uint16_t* src = (kv ? p.v : p.k) + (t * p.H + h) * p.D + 16 * blk16;
  const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(src));
  const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(src) + 1);
  const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
  float v[16];
  float bmax = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    v[2 * i] = bf16_lo(w[i]);
    v[2 * i + 1] = bf16_hi(w[i]);
    bmax = fmaxf(bmax, fmaxf(fabsf(v[2 * i]), fabsf(v[2 * i + 1])));
  }
  uint32_t sb = 0, codes_lo = 0, codes_hi = 0;
  if (g > 0.f) {
    sb = f32x2_to_e4m3x2(__fdiv_rn(bmax, __fmul_rn(6.0f, g)), 0.f) & 0xFFu;
    const float den = __fmul_rn(e4m3_to_f32(sb), g);
    if (den != 0.f) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        codes_lo |= f32x2_to_e2m1x2(__fdiv_rn(v[2 * i], den), __fdiv_rn(v[2 * i + 1], den))
                    << (8 * i);
        codes_hi |= f32x2_to_e2m1x2(__fdiv_rn(v[8 + 2 * i], den), __fdiv_rn(v[9 + 2 * i], den))
                    << (8 * i);
      }
    }
  }
  uint8_t* page = (kv ? p.vc : p.kc) + (slot / kPage * p.H + h) * static_cast<int64_t>(9 * p.D);
  const int o = static_cast<int>(slot % kPage);
  *reinterpret_cast<uint2*>(page + o * (p.D / 2) + 8 * blk16) = make_uint2(codes_lo, codes_hi);
  page[8 * p.D + o * (p.D / 16) + blk16] = static_cast<uint8_t>(sb);
}

// One thread = 8 elements (16 bytes) of one (token, K|V, head) row.
__global__ void write_bf16_kernel(const QuantParams p) {
  griddep_launch_dependents();  // a following decode may start its prologue
  const int cpr = p.D / 8;
  const int64_t total = p.T * 2 * p.H * cpr;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= total) return;
  const int c = static_cast<int>(idx % cpr);
  int64_t r = idx / cpr;
  const int h = static_cast<int>(r % p.H);
  r /= p.H;
  const int kv = static_cast<int>(r & 1);
  const int64_t t = r >> 1;
  const int64_t slot = resolve_slot(p, t);
  if (slot < 0) return;
  const uint16_t* src = (kv ? p.v : p.k) + (t * p.H + h) * p.D + 8 * c;
  uint8_t* dst = (kv ? p.vc : p.kc) +
                 (((slot / kPage * p.H + h) * kPage + slot % kPage) * p.D + 8 * c) * 2;
  *reinterpret_cast<uint4*>(dst) = __ldg(reinterpret_cast<const uint4*>(src));
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
  const int threads = 256;
  if (fmt == 1) {
    quantize_fp8_kernel<<<grid_for(p.T * 2 * p.H * (p.D / 8), threads), threads, 0, stream>>>(p);
  } else if (fmt == 2) {
    quantize_nvfp4_kernel<<<grid_for(p.T * 2 * p.H * (p.D / 16), threads), threads, 0, stream>>>(p);
  } else {
    write_bf16_kernel<<<grid_for(p.T * 2 * p.H * (p.D / 8), threads), threads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequantize(int fmt, const uint8_t* kc, const uint8_t* vc, int64_t num_blocks,
                              int H, int D, const int64_t* slots, int64_t n, const float* ks,
                              const float* vs, float* ko, float* vo, int* d_err,
                              cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
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
