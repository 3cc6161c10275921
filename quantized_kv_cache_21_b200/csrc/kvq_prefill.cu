// kvq_prefill.cu -- chunked-prefill attention over the quantized paged cache,
// on the fifth-generation tensor cores (tcgen05, accumulators in tensor memory).
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
// token r / G, head r % G), so one decoded K/V tile serves the whole group and
// the 128 rows are exactly one M = 128 tensor-core tile.  128 threads; thread r
// owns row r, which is also lane r of the CTA's tensor memory, so the softmax
// of a row needs no cross-thread reduction.
//
// Per 64-key block (4 cache pages):
//   1. the threads have decoded the block's K and V exactly into f16 (BF16
//      pages: bf16) tiles in shared memory, in the 128-byte-swizzled layouts the
//      tensor core reads (E4M3 with cvt.f16x2.e4m3x2, E2M1 with cvt.f16x2.e2m1x2
//      times the E4M3 block scale: exact f16 products);
//   2. one thread issues S = Q K^T (M 128, N 64, K = head_dim, in steps of 16)
//      into tensor memory and commits it to an mbarrier;
//   3. meanwhile every thread loads the next block's codes into registers;
//   4. each thread reads its row of S from tensor memory, masks (causal: key
//      position <= row position; bad pages), and updates its running max
//      lazily: the reference max moves only when a score exceeds it by more
//      than 2^8, and only then is its row of O (in tensor memory) rescaled, so
//      P stays <= 256;
//   5. P is written back over the row's S in tensor memory as a 16-bit high
//      part and its residual (two K-major A operands, two 16-bit values per
//      column), and one thread issues O += P_hi V + P_lo V with A read from
//      tensor memory (M 128, N = head_dim, K 64; V read MN-major straight
//      from its tile);
//   6. while that runs, the next block's K is decoded into its tile; after the
//      PV commit, V.
// Q is staged once.  Online softmax in the exp2 domain; the per-layer K scale
// is folded into the score scale and the V scale into the final normalisation.
// Every mbarrier wait is bounded (about 2 s, then KVQ error bit 0x10), and the
// tensor memory is freed on every path.
#include <math.h>

#include "kvq_device.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kRows = 128, kThreads = 128, kKeys = 64;
constexpr float kLog2e = 1.4426950408889634f, kLn2 = 0.6931471805599453f;
constexpr float kGap = 8.f;  // lazy rescale: P <= 2^kGap

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem]; acc = 0 overwrites D.
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(
          d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]: A (K-major, 16-bit elements packed two per
// 32-bit column, row i in lane i) read from tensor memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b,
                                          uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n}\n" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrive once on bar when every MMA this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float v[32]) {
  uint32_t* r = reinterpret_cast<uint32_t*>(v);
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float v[32]) {
  const uint32_t* r = reinterpret_cast<const uint32_t*>(v);
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, "
      "%28, %29, %30, %31, %32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, 128-byte swizzle (sm_100 format: start
// address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29, stride byte
// offset >> 4 in 32-45, version 1 in 46-47, layout 2 = 128B swizzle in 61-63).
__device__ __forceinline__ uint64_t sdesc(const void* p, uint32_t lbo, uint32_t sbo) {
  return static_cast<uint64_t>((smem_u32(p) & 0x3FFFFu) >> 4) |
         (static_cast<uint64_t>(lbo >> 4) << 16) | (static_cast<uint64_t>(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}
// Instruction descriptor, kind::f16: fp32 accumulator (bit 4), A/B type in
// bits 7-9 / 10-12 (0 f16, 1 bf16), B major in bit 16 (1 = MN-major), N >> 3
// in bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc(uint32_t ab, uint32_t b_mn, uint32_t n, uint32_t m) {
  return (1u << 4) | (ab << 7) | (ab << 10) | (b_mn << 16) | ((n >> 3) << 17) | ((m >> 4) << 24);
}

// Byte offset of 16-byte chunk c of row r in a [rows][128 B] swizzled tile.
__device__ __forceinline__ int sw128(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

// ------------------------------------------------------------------ K/V blocks
// One thread's share of a 64-key block: key t / 2 (page key / 16 of the block,
// token key % 16 of the page), elements [(t % 2) D/2, +D/2) of that key's K and
// V rows.  R 16-byte words of codes per tensor; NVFP4 adds the D/32 block
// scales of those elements.
template <int FMT, int D>
struct Share {
  static constexpr int R = FMT == 0 ? D / 16 : (FMT == 1 ? D / 32 : D / 64);
  uint4 k[R], v[R];
  uint32_t ksf, vsf;
};

template <int FMT, int D>
__device__ __forceinline__ void load_share(const PrefillParams& p, int b, int h, int kb, int tid,
                                           Share<FMT, D>& s, int npages, bool& bad) {
  const int key = tid >> 1, half = tid & 1, row = key & 15;
  const int page = kb * 4 + (key >> 4);
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
  size_t off;
  if constexpr (FMT == 0)
    off = hp * (32 * D) + row * (2 * D) + half * D;  // [16][D] BF16
  else if constexpr (FMT == 1)
    off = hp * (16 * D) + row * D + half * (D / 2);  // [16][D] E4M3
  else
    off = hp * (9 * D) + row * (D / 2) + half * (D / 4);  // [16][D/2] E2M1 codes
#pragma unroll
  for (int i = 0; i < Share<FMT, D>::R; ++i) {
    s.k[i] = __ldg(reinterpret_cast<const uint4*>(p.kc + off) + i);
    s.v[i] = __ldg(reinterpret_cast<const uint4*>(p.vc + off) + i);
  }
  if constexpr (FMT == 2) {  // then [16][D/16] E4M3 block scales
    const size_t so = hp * (9 * D) + 8 * D + row * (D / 16) + half * (D / 32);
    if constexpr (D == 128) {
      s.ksf = __ldg(reinterpret_cast<const uint32_t*>(p.kc + so));
      s.vsf = __ldg(reinterpret_cast<const uint32_t*>(p.vc + so));
    } else {
      s.ksf = __ldg(reinterpret_cast<const uint16_t*>(p.kc + so));
      s.vsf = __ldg(reinterpret_cast<const uint16_t*>(p.vc + so));
    }
  }
}

// Decode one tensor's share into D/16 16-byte chunks of 16-bit values.
template <int FMT, int D>
__device__ __forceinline__ uint4 decode_chunk(const uint4* w, uint32_t sf, int i) {
  if constexpr (FMT == 0) {
    return w[i];
  } else if constexpr (FMT == 1) {
    const uint32_t* b = reinterpret_cast<const uint32_t*>(w);
    uint4 o;
    e4m3x4_to_f16x2x2(b[2 * i], o.x, o.y);
    e4m3x4_to_f16x2x2(b[2 * i + 1], o.z, o.w);
    return o;
  } else {
    // chunk i: elements [8i, 8i + 8) = code word i; its 16-element block is i / 2
    const uint32_t* b = reinterpret_cast<const uint32_t*>(w);
    uint32_t s2, unused;
    const uint32_t sb = (sf >> (8 * (i >> 1))) & 0xFFu;
    e4m3x4_to_f16x2x2(sb | (sb << 8), s2, unused);
    uint32_t f[4];
    e2m1x8_to_f16x2x4(b[i], f);
    return make_uint4(hmul2(f[0], s2), hmul2(f[1], s2), hmul2(f[2], s2), hmul2(f[3], s2));
  }
}

// Store a decoded share into a [D/64 atoms][64 keys][128 B] tile (the K-major
// B operand of QK for K; the MN-major B operand of PV for V).
template <int FMT, int D>
__device__ __forceinline__ void store_tile(const uint4* w, uint32_t sf, int tid, uint8_t* tile) {
  const int key = tid >> 1, half = tid & 1;
#pragma unroll
  for (int i = 0; i < D / 16; ++i) {
    const int gc = half * (D / 16) + i;  // 16-byte chunk of the key's D values
    *reinterpret_cast<uint4*>(tile + (gc >> 3) * (kKeys * 128) + sw128(key, gc & 7)) =
        decode_chunk<FMT, D>(w, sf, i);
  }
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

template <int D>
__host__ __device__ constexpr uint32_t tmem_cols() {
  return D == 128 ? 256u : 128u;  // O (D columns) + S (64 columns), a power of two
}
template <int D>
constexpr size_t smem_bytes() {
  // Q [D/64][128][128 B], K and V [D/64][64][128 B], plus 1 KB to align the
  // tiles to the 1024-byte swizzle repeat (P lives in tensor memory)
  return (D / 64) * (16384 + 2 * 8192) + 1024;
}

template <int FMT, int D>
__global__ void __launch_bounds__(kThreads, 2) kvq_prefill_kernel(const PrefillParams p) {
  constexpr int KA = D / 64;
  constexpr uint32_t kCols = tmem_cols<D>(), kColO = 0, kColS = D;
  constexpr uint32_t kAB = FMT == 0 ? 1u : 0u;
  constexpr uint32_t kIdQK = idesc(kAB, 0, kKeys, kRows), kIdPV = idesc(kAB, 1, D, kRows);
  const float kInf = __int_as_float(0x7f800000);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sQ = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                           ~static_cast<uintptr_t>(1023));
  uint8_t* sK = sQ + KA * 16384;
  uint8_t* sV = sK + KA * 8192;
  __shared__ uint64_t bar_s, bar_o;
  __shared__ uint32_t s_tmem;
  __shared__ int s_bad[4];

  const int tid = threadIdx.x, warp = tid >> 5;
  const int qb = blockIdx.x % p.n_qblk;
  const int h = (blockIdx.x / p.n_qblk) % p.Hkv;
  const int b = blockIdx.x / (p.n_qblk * p.Hkv);

  if (warp == 0) {
    tmem_alloc(&s_tmem, kCols);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_s, 1);
    mbar_init(&bar_o, 1);
    mbar_init_fence();
  }

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

  // This thread's row: query index, query head, position (INT_MAX for padding
  // rows, which are computed but not stored).
  const int tok = tid / p.G;
  const int qi = qb * p.QT + tok, qh = h * p.G + tid % p.G;
  const bool valid = tok < p.QT && qi < p.Tq;
  const int pos = valid ? len - p.Tq + qi : 0x7fffffff;
  const int q_last = min(p.Tq, (qb + 1) * p.QT) - 1;
  const int n_keys = max(0, len - p.Tq + q_last + 1);
  const int npages = (n_keys + kPage - 1) / kPage;
  const int nblk = (n_keys + kKeys - 1) / kKeys;

  // Scores are scaled by c = sm_scale * k_scale * log2(e) after the running max
  // of the raw ones is taken, so c must not be negative: a negative sm_scale is
  // moved into Q's sign (exact).  c = 0 (an all-zero NVFP4 K tensor, whose
  // scores are all 0) becomes a tiny positive c with the same result.
  const float c_log2 = p.sm_scale * ks * kLog2e;
  const uint32_t q_sign = c_log2 < 0.f ? 0x80008000u : 0u;
  const float c_abs = fmaxf(fabsf(c_log2), 1e-30f);
  // Q row -> sQ (K-major A tile: [D/64][128 rows][128 B])
  {
    const uint4* qrow = reinterpret_cast<const uint4*>(
        p.q + ((static_cast<size_t>(b) * p.Tq + (valid ? qi : 0)) * p.Hq + qh) * D);
#pragma unroll
    for (int c = 0; c < D / 8; ++c) {
      uint4 w = valid ? __ldg(qrow + c) : make_uint4(0u, 0u, 0u, 0u);
      if constexpr (FMT != 0) {
        w.x = pack_f16x2(bf16_lo(w.x), bf16_hi(w.x));
        w.y = pack_f16x2(bf16_lo(w.y), bf16_hi(w.y));
        w.z = pack_f16x2(bf16_lo(w.z), bf16_hi(w.z));
        w.w = pack_f16x2(bf16_lo(w.w), bf16_hi(w.w));
      }
      w.x ^= q_sign;
      w.y ^= q_sign;
      w.z ^= q_sign;
      w.w ^= q_sign;
      *reinterpret_cast<uint4*>(sQ + (c >> 3) * 16384 + sw128(tid, c & 7)) = w;
    }
  }
  Share<FMT, D> nxt;
  bool nbad = false;
  if (nblk > 0) {
    load_share<FMT, D>(p, b, h, 0, tid, nxt, npages, nbad);
    store_tile<FMT, D>(nxt.k, nxt.ksf, tid, sK);
    store_tile<FMT, D>(nxt.v, nxt.vsf, tid, sV);
    if ((tid & 31) == 0) {
      s_bad[tid >> 5] = nbad;
      if (nbad) set_err(p.d_err, kErrBlockId);
    }
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tm = s_tmem;
  const uint32_t tm_row = tm + (static_cast<uint32_t>(warp * 32) << 16);

  float m_ref = -kInf, l = 0.f;
  uint32_t ph = 0;
  bool failed = false;
  for (int kb = 0; kb < nblk; ++kb) {
    const int key0 = kb * kKeys;
    // ---- S = Q K^T into tensor memory
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < D / 16; ++s)
        tc_mma(tm + kColS, sdesc(sQ + (s >> 2) * 16384 + (s & 3) * 32, 16, 1024),
               sdesc(sK + (s >> 2) * 8192 + (s & 3) * 32, 16, 1024), kIdQK, s > 0);
      tc_commit(&bar_s);
    }
    if (kb + 1 < nblk) load_share<FMT, D>(p, b, h, kb + 1, tid, nxt, npages, nbad);
    const bool got_s = mbar_wait_bounded(&bar_s, ph);
    if (__syncthreads_or(!got_s)) {
      failed = true;
      break;
    }
    tc_fence_after();
    float sv[64];
    tmem_ld32(tm_row + kColS, sv);
    tmem_ld32(tm_row + kColS + 32, sv + 32);
    tmem_wait_ld();

    // ---- mask, lazy running max (scores stay raw; c_abs > 0 scales them)
    const bool any_bad = s_bad[0] | s_bad[1] | s_bad[2] | s_bad[3];
    if (key0 + kKeys - 1 > pos || any_bad) {
#pragma unroll
      for (int k = 0; k < kKeys; ++k)
        if (key0 + k > pos || s_bad[k >> 4]) sv[k] = -kInf;
    }
    float t[32];  // max as a tree: depth 6 instead of a chain of 64
#pragma unroll
    for (int i = 0; i < 32; ++i) t[i] = fmaxf(sv[i], sv[i + 32]);
#pragma unroll
    for (int w = 16; w >= 1; w >>= 1)
#pragma unroll
      for (int i = 0; i < w; ++i) t[i] = fmaxf(t[i], t[i + w]);
    const float mx = t[0] * c_abs;
    float m_new = m_ref;
    if (mx > m_ref + kGap || (m_ref == -kInf && mx > -kInf)) m_new = mx;
    const bool resc = m_new != m_ref && m_ref != -kInf;
    const float alpha = resc ? fast_exp2(m_ref - m_new) : 1.f;
    if (__any_sync(0xffffffffu, resc)) {  // rows whose reference moved: O *= alpha
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        float o[32];
        tmem_ld32(tm_row + kColO + 32 * c, o);
        tmem_wait_ld();
#pragma unroll
        for (int x = 0; x < 32; ++x) o[x] *= alpha;
        tmem_st32(tm_row + kColO + 32 * c, o);
      }
      tmem_wait_st();
    }
    m_ref = m_new;
    // p = 2^(s c - m); a row with nothing unmasked yet has s = -inf throughout
    const float neg_m = m_ref == -kInf ? 0.f : -m_ref;
    // P's two 16-bit halves replace this row's S in tensor memory (S is in
    // registers now): columns [S, S + 32) high parts, [S + 32, S + 64) residuals
    float ps8[8];
    uint32_t phi[32], plo[32];
#pragma unroll
    for (int c = 0; c < 8; ++c) {  // keys 8c .. 8c + 7
      float pc[8];
#pragma unroll
      for (int x = 0; x < 8; ++x) pc[x] = fast_exp2(fmaf(sv[8 * c + x], c_abs, neg_m));
#pragma unroll
      for (int x = 0; x < 4; ++x)
        split_pair<FMT>(pc[2 * x], pc[2 * x + 1], phi[4 * c + x], plo[4 * c + x]);
      ps8[c] = ((pc[0] + pc[1]) + (pc[2] + pc[3])) + ((pc[4] + pc[5]) + (pc[6] + pc[7]));
    }
    tmem_st32(tm_row + kColS, reinterpret_cast<const float*>(phi));
    tmem_st32(tm_row + kColS + 32, reinterpret_cast<const float*>(plo));
    const float ps = ((ps8[0] + ps8[1]) + (ps8[2] + ps8[3])) + ((ps8[4] + ps8[5]) + (ps8[6] + ps8[7]));
    l = l * alpha + ps;
    tmem_wait_st();
    tc_fence_before();
    __syncthreads();

    // ---- O += P V (both halves of P)
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s = 0; s < kKeys / 16; ++s) {  // 16 keys = 8 columns of packed P
        const uint64_t bv = sdesc(sV + s * 2048, kKeys * 128, 1024);
        tc_mma_ts(tm + kColO, tm + kColS + 8 * s, bv, kIdPV, kb > 0 || s > 0);
        tc_mma_ts(tm + kColO, tm + kColS + 32 + 8 * s, bv, kIdPV, 1u);
      }
      tc_commit(&bar_o);
    }
    // the next block's K while PV runs (QK of this block is complete)
    if (kb + 1 < nblk) store_tile<FMT, D>(nxt.k, nxt.ksf, tid, sK);
    const bool got_o = mbar_wait_bounded(&bar_o, ph);
    if (__syncthreads_or(!got_o)) {
      failed = true;
      break;
    }
    ph ^= 1u;
    if (kb + 1 < nblk) {
      store_tile<FMT, D>(nxt.v, nxt.vsf, tid, sV);
      if ((tid & 31) == 0) {
        s_bad[tid >> 5] = nbad;
        if (nbad) set_err(p.d_err, kErrBlockId);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
  }

  if (failed) {
    if (tid == 0) set_err(p.d_err, kErrTimeout);
    // let whatever this CTA issued finish (bounded) before its memory goes away
    mbar_wait_bounded(&bar_s, ph);
    mbar_wait_bounded(&bar_o, ph);
  } else {
    tc_fence_after();
    // ---- out = O * vs / l, lse = (m + log2 l) ln 2
    const bool live = nblk > 0 && l > 0.f;
    const float sc = live ? vs / l : 0.f;
    float* orow = p.out + ((static_cast<size_t>(b) * p.Tq + (valid ? qi : 0)) * p.Hq + qh) * D;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      float o[32];
      if (nblk > 0) {
        tmem_ld32(tm_row + kColO + 32 * c, o);
        tmem_wait_ld();
      }
      if (valid) {
#pragma unroll
        for (int x = 0; x < 32; x += 4)
          *reinterpret_cast<float4*>(orow + 32 * c + x) =
              live ? make_float4(o[x] * sc, o[x + 1] * sc, o[x + 2] * sc, o[x + 3] * sc)
                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (valid && p.lse)
      p.lse[(static_cast<size_t>(b) * p.Tq + qi) * p.Hq + qh] =
          live ? (m_ref + log2f(l)) * kLn2 : -kInf;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tm, kCols);
  }
}

template <int FMT, int D>
cudaError_t launch_t(const PrefillParams& p, int64_t ctas, cudaStream_t stream) {
  static std::atomic<bool> attr_done[kMaxDevices];  // per instantiation and device ordinal
  constexpr size_t smem = smem_bytes<D>();
  cudaError_t e = ensure_smem_attr(reinterpret_cast<const void*>(kvq_prefill_kernel<FMT, D>),
                                   smem, attr_done);
  if (e != cudaSuccess) return e;
  kvq_prefill_kernel<FMT, D><<<static_cast<unsigned>(ctas), kThreads, smem, stream>>>(p);
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
