// kvq_prefill.cu -- chunked-prefill attention over the quantized paged cache.
//
// A long prompt is fed in chunks of a fixed token budget, each chunk attending
// to the prefix already in the cache ("Dual R9700 model and spec-decode
// campaign", fixed knobs: long-prefill-token-threshold 2048 with prefix
// caching; "FP8 KV calibration guide", first paragraph: TTFT at ~126k context
// with FP8 KV).  The Tq newest tokens of sequence b (already written to the
// cache) are its queries: query i sits at position p = len_b - Tq + i and
// attends to the cache tokens [0, p].
//
// Work: one CTA per (sequence b, KV head h, block of QT query tokens).  Its 128
// rows are (query token, query head) pairs of the KV head's GQA group (row r =
// token r / G, head r % G), so one decoded K/V tile serves the whole group.
// 8 warps; warp w owns rows [16w, 16w + 16), one m16 tile.
//
// Keys go in blocks of 64 (4 cache pages).  The 256 threads load the next
// block's codes into registers while the current block is computed, then
// decode them exactly into f16 (BF16 pages: bf16) tiles in shared memory:
// E4M3 with cvt.f16x2.e4m3x2, E2M1 with cvt.f16x2.e2m1x2 times the E4M3 block
// scale (an exact f16 product).  Tiles are [64 keys][D] with 16-byte chunks
// XOR-swizzled by key & 7, so the ldmatrix row reads are bank-conflict free.
// S = Q K^T and O += P V run on mma.sync.m16n8k16 with fp32 accumulation; the
// S accumulators become the P operand in registers (the C layout of two n8
// tiles is the A layout of one k16 step).  P enters PV as a 16-bit high part
// plus its 16-bit residual (two MMAs), so P keeps ~22 bits (f16) / 16 (bf16).
// Online softmax in the exp2 domain; the per-layer K scale is folded into the
// score scale and the V scale into the final normalisation, so no decoded
// value is rounded.  Causal mask: key position <= the row's position, applied
// only to blocks that reach past a row's position or hold a bad page.
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kRows = 128, kWarps = 8, kThreads = kWarps * 32, kKeys = 64;
constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t r[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t r[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// Byte offset of 16-byte chunk c of key row k in a [64][D] 16-bit tile.
template <int D>
__device__ __forceinline__ int tile_off(int k, int c) {
  return k * (2 * D) + ((c ^ (k & 7)) << 4);
}

// One thread's share of a 64-key block: page pg = tid / 64 of the block, row
// (token) li / 4 of the page, elements [(li % 4) * D/4, +D/4) of the row, for
// K and for V.  R 16-byte words of codes per tensor; NVFP4 adds the block
// scales of those elements (D/64 bytes).
template <int FMT, int D>
struct Share {
  static constexpr int R = FMT == 0 ? D / 32 : (FMT == 1 ? D / 64 : 1);
  uint4 k[R], v[R];
  uint32_t ksf, vsf;
};

template <int FMT, int D>
__device__ __forceinline__ void load_share(const PrefillParams& p, int b, int h, int kb, int tid,
                                           Share<FMT, D>& s, int npages, bool& bad) {
  const int pg = tid >> 6, li = tid & 63, row = li >> 2, part = li & 3;
  const int page = kb * 4 + pg;
#pragma unroll
  for (int i = 0; i < Share<FMT, D>::R; ++i) s.k[i] = s.v[i] = make_uint4(0u, 0u, 0u, 0u);
  s.ksf = s.vsf = 0u;
  bad = false;
  if (page >= npages) return;
  const int blk = __ldg(p.block_table + static_cast<size_t>(b) * p.max_blocks + page);
  if (blk < 0 || blk >= p.num_blocks) {
    bad = true;
    return;
  }
  const int64_t hp = static_cast<int64_t>(blk) * p.Hkv + h;
  if constexpr (FMT == 0) {  // BF16 page: [16][D] x 2 B
    const size_t off = hp * (32 * D) + row * (2 * D) + part * (D / 2);
#pragma unroll
    for (int i = 0; i < Share<FMT, D>::R; ++i) {
      s.k[i] = __ldg(reinterpret_cast<const uint4*>(p.kc + off) + i);
      s.v[i] = __ldg(reinterpret_cast<const uint4*>(p.vc + off) + i);
    }
  } else if constexpr (FMT == 1) {  // FP8 page: [16][D] x 1 B
    const size_t off = hp * (16 * D) + row * D + part * (D / 4);
#pragma unroll
    for (int i = 0; i < Share<FMT, D>::R; ++i) {
      s.k[i] = __ldg(reinterpret_cast<const uint4*>(p.kc + off) + i);
      s.v[i] = __ldg(reinterpret_cast<const uint4*>(p.vc + off) + i);
    }
  } else {  // NVFP4 page: [16][D/2] codes, then [16][D/16] E4M3 block scales
    const size_t base = hp * (9 * D);
    const size_t co = base + row * (D / 2) + part * (D / 8);
    const size_t so = base + 16 * (D / 2) + row * (D / 16) + part * (D / 64);
    if constexpr (D == 128) {
      s.k[0] = __ldg(reinterpret_cast<const uint4*>(p.kc + co));
      s.v[0] = __ldg(reinterpret_cast<const uint4*>(p.vc + co));
      s.ksf = __ldg(reinterpret_cast<const uint16_t*>(p.kc + so));
      s.vsf = __ldg(reinterpret_cast<const uint16_t*>(p.vc + so));
    } else {
      const uint2 a = __ldg(reinterpret_cast<const uint2*>(p.kc + co));
      const uint2 c = __ldg(reinterpret_cast<const uint2*>(p.vc + co));
      s.k[0] = make_uint4(a.x, a.y, 0u, 0u);
      s.v[0] = make_uint4(c.x, c.y, 0u, 0u);
      s.ksf = __ldg(p.kc + so);
      s.vsf = __ldg(p.vc + so);
    }
  }
}

// Decode one tensor's share into D/32 16-byte chunks of 16-bit values.
template <int FMT, int D>
__device__ __forceinline__ void decode_share(const uint4* w, uint32_t sf, uint4 out[D / 32]) {
  if constexpr (FMT == 0) {
#pragma unroll
    for (int i = 0; i < D / 32; ++i) out[i] = w[i];
  } else if constexpr (FMT == 1) {
    const uint32_t* b = reinterpret_cast<const uint32_t*>(w);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      e4m3x4_to_f16x2x2(b[2 * i], out[i].x, out[i].y);
      e4m3x4_to_f16x2x2(b[2 * i + 1], out[i].z, out[i].w);
    }
  } else {
    const uint32_t* b = reinterpret_cast<const uint32_t*>(w);
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      // chunk i holds elements [8i, 8i + 8) of the share: 4 code bytes, block
      // scale i / 2 of the share (one 16-element block spans two chunks)
      uint32_t s2, unused;
      const uint32_t sb = (sf >> (8 * (i >> 1))) & 0xFFu;
      e4m3x4_to_f16x2x2(sb | (sb << 8), s2, unused);
      uint32_t f[4];
      e2m1x8_to_f16x2x4(b[i], f);
      out[i] = make_uint4(hmul2(f[0], s2), hmul2(f[1], s2), hmul2(f[2], s2), hmul2(f[3], s2));
    }
  }
}

template <int FMT, int D>
__device__ __forceinline__ void store_share(const Share<FMT, D>& s, int tid, uint8_t* sk,
                                            uint8_t* sv) {
  const int pg = tid >> 6, li = tid & 63, key = pg * 16 + (li >> 2), c0 = (li & 3) * (D / 32);
  uint4 ck[D / 32], cv[D / 32];
  decode_share<FMT, D>(s.k, s.ksf, ck);
  decode_share<FMT, D>(s.v, s.vsf, cv);
#pragma unroll
  for (int i = 0; i < D / 32; ++i) {
    *reinterpret_cast<uint4*>(sk + tile_off<D>(key, c0 + i)) = ck[i];
    *reinterpret_cast<uint4*>(sv + tile_off<D>(key, c0 + i)) = cv[i];
  }
}

template <int FMT>
__device__ __forceinline__ void mma16(float c[4], const uint32_t a[4], uint32_t b0, uint32_t b1) {
  if constexpr (FMT == 0)
    mma_bf16(c, a, b0, b1);
  else
    mma_f16(c, a, b0, b1);
}

// (x, y) as a 16-bit pair (f16, or bf16 for the BF16 format) and the pair of
// what rounding left over, so that hi + lo carries ~22 (f16) / 16 (bf16) bits.
template <int FMT>
__device__ __forceinline__ void split_pair(float x, float y, uint32_t& hi, uint32_t& lo) {
  float hx, hy;
  if constexpr (FMT == 0) {
    hi = pack_bf16x2(x, y);
    unpack_bf16x2(hi, hx, hy);
    lo = pack_bf16x2(x - hx, y - hy);
  } else {
    hi = pack_f16x2(x, y);
    unpack_f16x2(hi, hx, hy);
    lo = pack_f16x2(x - hx, y - hy);
  }
}

template <int FMT, int D>
__global__ void __launch_bounds__(kThreads, 1) kvq_prefill_kernel(const PrefillParams p) {
  constexpr int KS = D / 16, NT = D / 8;
  const float kInf = __int_as_float(0x7f800000);
  __shared__ __align__(128) uint8_t sk[kKeys * 2 * D];
  __shared__ __align__(128) uint8_t sv[kKeys * 2 * D];
  __shared__ int s_bad[4];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const int qb = blockIdx.x % p.n_qblk;
  const int h = (blockIdx.x / p.n_qblk) % p.Hkv;
  const int b = blockIdx.x / (p.n_qblk * p.Hkv);

  float ks = 1.f, vs = 1.f;
  bool ok = true;
  if constexpr (FMT != 0) {
    ks = __ldg(p.k_scale);
    vs = __ldg(p.v_scale);
    if (FMT == 1)
      ok = ks > 0.f && vs > 0.f && ks < kInf && vs < kInf;
    else
      ok = ks >= 0.f && vs >= 0.f && ks < kInf && vs < kInf;
    if (!ok && blockIdx.x == 0 && tid == 0) set_err(p.d_err, kErrScale);
  }
  int len = __ldg(p.seq_lens + b);
  if (len < 0 || static_cast<int64_t>(len) > static_cast<int64_t>(p.max_blocks) * kPage) {
    if (qb == 0 && h == 0 && tid == 0) set_err(p.d_err, kErrSeqLen);
    len = 0;
  }
  if (!ok) len = 0;

  // The thread's two rows (gid and gid + 8 of the warp's tile): query index,
  // position (INT_MAX for padding rows, which are computed but not stored).
  const int r0 = warp * 16 + gid, r1 = r0 + 8;
  int qi[2], pos[2], qh[2];
  bool valid[2];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int r = e ? r1 : r0, tok = r / p.G;
    qi[e] = qb * p.QT + tok;
    qh[e] = h * p.G + r % p.G;
    valid[e] = tok < p.QT && qi[e] < p.Tq;
    pos[e] = valid[e] ? len - p.Tq + qi[e] : 0x7fffffff;
  }
  // Keys the CTA needs: [0, last position of its queries]
  const int q_last = min(p.Tq, (qb + 1) * p.QT) - 1;
  const int n_keys = max(0, len - p.Tq + q_last + 1);
  const int npages = (n_keys + kPage - 1) / kPage;
  const int nblk = (n_keys + kKeys - 1) / kKeys;

  // Query fragments (A operand of QK): rows r0 / r1, k-step s, columns
  // 16s + 2tig (+1) and 16s + 8 + 2tig (+1).
  uint32_t qa[KS][4];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const uint16_t* qrow =
        p.q + ((static_cast<size_t>(b) * p.Tq + (valid[e] ? qi[e] : 0)) * p.Hq + qh[e]) * D;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      uint32_t lo = 0u, hi = 0u;
      if (valid[e]) {
        lo = __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * s + 2 * tig));
        hi = __ldg(reinterpret_cast<const uint32_t*>(qrow + 16 * s + 8 + 2 * tig));
        if constexpr (FMT != 0) {
          lo = pack_f16x2(bf16_lo(lo), bf16_hi(lo));
          hi = pack_f16x2(bf16_lo(hi), bf16_hi(hi));
        }
      }
      qa[s][e] = lo;
      qa[s][2 + e] = hi;
    }
  }

  float o[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m[2] = {-kInf, -kInf}, l[2] = {0.f, 0.f};
  const float c_log2 = p.sm_scale * ks * kLog2e;
  const uint32_t sk_base = smem_u32(sk), sv_base = smem_u32(sv);
  const int min_pos = min(pos[0], pos[1]);

  Share<FMT, D> nxt;
  bool nbad = false;
  if (nblk > 0) {
    load_share<FMT, D>(p, b, h, 0, tid, nxt, npages, nbad);
    store_share<FMT, D>(nxt, tid, sk, sv);
    if ((tid & 63) == 0) {
      s_bad[tid >> 6] = nbad;
      if (nbad) set_err(p.d_err, kErrBlockId);
    }
  }
  __syncthreads();

  for (int kb = 0; kb < nblk; ++kb) {
    if (kb + 1 < nblk) load_share<FMT, D>(p, b, h, kb + 1, tid, nxt, npages, nbad);
    const int key0 = kb * kKeys;
    const bool any_bad = s_bad[0] | s_bad[1] | s_bad[2] | s_bad[3];

    // ---- S = Q K^T for 64 keys: n tile j = keys key0 + 8j .. + 7
    float sacc[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
#pragma unroll
      for (int s = 0; s < KS; s += 2) {
        uint32_t f[4];
        const int key = 8 * j + (lane & 7), c = 2 * s + (lane >> 3);
        ldsm_x4(sk_base + tile_off<D>(key, c), f);
        mma16<FMT>(sacc[j], qa[s], f[0], f[1]);
        mma16<FMT>(sacc[j], qa[s + 1], f[2], f[3]);
      }
    }
    // ---- scale, mask, running max
    const bool need_mask = __any_sync(0xffffffffu, key0 + kKeys - 1 > min_pos) || any_bad;
    float mx[2] = {-kInf, -kInf};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        float v = sacc[j][x] * c_log2;
        if (need_mask) {
          const int kp = key0 + 8 * j + 2 * tig + (x & 1);
          if (kp > pos[x >> 1] || s_bad[j >> 1]) v = -kInf;
        }
        sacc[j][x] = v;
        mx[x >> 1] = fmaxf(mx[x >> 1], v);
      }
    }
    float alpha[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 1));
      mx[e] = fmaxf(mx[e], __shfl_xor_sync(0xffffffffu, mx[e], 2));
      const float mn = fmaxf(m[e], mx[e]);
      alpha[e] = mn == -kInf ? 1.f : fast_exp2(m[e] - mn);
      m[e] = mn;
    }
    float ps[2] = {0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float mm = m[x >> 1];
        const float pv = mm == -kInf ? 0.f : fast_exp2(sacc[j][x] - mm);
        sacc[j][x] = pv;
        ps[x >> 1] += pv;
      }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) l[e] = l[e] * alpha[e] + ps[e];
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      o[j][0] *= alpha[0];
      o[j][1] *= alpha[0];
      o[j][2] *= alpha[1];
      o[j][3] *= alpha[1];
    }
    // ---- O += P V: k step s = keys key0 + 16s .. + 15 (n tiles 2s, 2s + 1 of S)
#pragma unroll
    for (int s = 0; s < 4; ++s) {
      uint32_t ph[4], pl[4];
      split_pair<FMT>(sacc[2 * s][0], sacc[2 * s][1], ph[0], pl[0]);
      split_pair<FMT>(sacc[2 * s][2], sacc[2 * s][3], ph[1], pl[1]);
      split_pair<FMT>(sacc[2 * s + 1][0], sacc[2 * s + 1][1], ph[2], pl[2]);
      split_pair<FMT>(sacc[2 * s + 1][2], sacc[2 * s + 1][3], ph[3], pl[3]);
      const int mi = lane >> 3, key = 16 * s + 8 * (mi & 1) + (lane & 7);
#pragma unroll
      for (int j = 0; j < NT; j += 2) {
        uint32_t f[4];
        ldsm_x4_t(sv_base + tile_off<D>(key, j + (mi >> 1)), f);
        mma16<FMT>(o[j], ph, f[0], f[1]);
        mma16<FMT>(o[j], pl, f[0], f[1]);
        mma16<FMT>(o[j + 1], ph, f[2], f[3]);
        mma16<FMT>(o[j + 1], pl, f[2], f[3]);
      }
    }
    __syncthreads();  // every warp is done with this block's tiles
    if (kb + 1 < nblk) {
      store_share<FMT, D>(nxt, tid, sk, sv);
      if ((tid & 63) == 0) {
        s_bad[tid >> 6] = nbad;
        if (nbad) set_err(p.d_err, kErrBlockId);
      }
    }
    __syncthreads();
  }

  // ---- normalise and store
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 1);
    l[e] += __shfl_xor_sync(0xffffffffu, l[e], 2);
    if (!valid[e]) continue;
    const size_t row = (static_cast<size_t>(b) * p.Tq + qi[e]) * p.Hq + qh[e];
    const float sc = l[e] > 0.f ? vs / l[e] : 0.f;
    float* orow = p.out + row * D;
#pragma unroll
    for (int j = 0; j < NT; ++j)
      *reinterpret_cast<float2*>(orow + 8 * j + 2 * tig) =
          make_float2(o[j][2 * e] * sc, o[j][2 * e + 1] * sc);
    if (tig == 0 && p.lse) p.lse[row] = l[e] > 0.f ? (m[e] + log2f(l[e])) * kLn2 : -kInf;
  }
}

template <int FMT, int D>
cudaError_t launch_t(const PrefillParams& p, int64_t ctas, cudaStream_t stream) {
  kvq_prefill_kernel<FMT, D><<<static_cast<unsigned>(ctas), kThreads, 0, stream>>>(p);
  return cudaGetLastError();
}

}  // namespace

int prefill_rows() { return kRows; }

cudaError_t launch_prefill(int fmt, int D, const PrefillParams& p, int64_t ctas,
                           cudaStream_t stream) {
  if (fmt == 0) return D == 128 ? launch_t<0, 128>(p, ctas, stream) : launch_t<0, 64>(p, ctas, stream);
  if (fmt == 1) return D == 128 ? launch_t<1, 128>(p, ctas, stream) : launch_t<1, 64>(p, ctas, stream);
  return D == 128 ? launch_t<2, 128>(p, ctas, stream) : launch_t<2, 64>(p, ctas, stream);
}

}  // namespace kvq
