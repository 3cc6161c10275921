// kvq_api.cu -- the C ABI declared in include/kvq.h: argument checks, the
// context-split plan, TMA descriptors for the paged cache, and launches.
#include <cudaTypedefs.h>
#include <math.h>

#include <cmath>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

thread_local char g_err[512] = "";

kvq_status fail(kvq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

kvq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(KVQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// 0 = unknown, 1 = supported (sm_100), 2 = not supported.
std::atomic<int> g_dev_ok[64];

kvq_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(KVQ_ERR_UNSUPPORTED, "device ordinal %d", dev);
  int st = g_dev_ok[dev].load(std::memory_order_relaxed);
  if (st == 0) {
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    st = (major == 10 && minor == 0) ? 1 : 2;
    g_dev_ok[dev].store(st, std::memory_order_relaxed);
  }
  if (st != 1) return fail(KVQ_ERR_UNSUPPORTED, "device %d is not compute capability 10.0 (B200)", dev);
  return KVQ_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int64_t head_page_bytes(int fmt, int D) {
  if (fmt == KVQ_FMT_BF16) return 32LL * D;
  if (fmt == KVQ_FMT_FP8_E4M3) return 16LL * D;
  if (fmt == KVQ_FMT_PQ3) return 16LL * 52;  // per token: fp32 norm + 48 index bytes
  return 9LL * D;
}

kvq_status check_cache(int32_t fmt, const kvq_cache* c) {
  if (fmt < 0 || fmt > 3) return fail(KVQ_ERR_UNSUPPORTED, "unknown format %d", fmt);
  if (!c) return fail(KVQ_ERR_INVALID_ARG, "cache is NULL");
  if (c->fmt != fmt) return fail(KVQ_ERR_INVALID_ARG, "cache format %d != fmt %d", c->fmt, fmt);
  if (c->block_size != KVQ_BLOCK_SIZE)
    return fail(KVQ_ERR_UNSUPPORTED, "block_size %d (only 16)", c->block_size);
  if (c->head_dim != 64 && c->head_dim != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", c->head_dim);
  if (fmt == KVQ_FMT_PQ3 && c->head_dim != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "PQ3 needs head_dim 128 (got %d)", c->head_dim);
  if (c->num_kv_heads < 1) return fail(KVQ_ERR_INVALID_ARG, "num_kv_heads %d", c->num_kv_heads);
  if (c->num_blocks < 1 || c->num_blocks > 0x7fffffffLL)
    return fail(KVQ_ERR_INVALID_ARG, "num_blocks %lld", (long long)c->num_blocks);
  if (!c->k || !c->v) return fail(KVQ_ERR_INVALID_ARG, "cache k/v is NULL");
  if (!aligned(c->k, 256) || !aligned(c->v, 256))
    return fail(KVQ_ERR_INVALID_ARG, "cache k/v must be 256-byte aligned");
  return KVQ_OK;
}

// ---------------------------------------------------------------- work plan
// The decode work is the virtual page space units x pmax (unit = sequence, KV
// head, group of 8 query heads), cut evenly over `ctas` persistent CTAs.  A
// unit that straddles CTAs is finished by a merge of its per-CTA partials.
struct Plan {
  int G, n_groups, units, pmax, ctas;
  size_t off_part, ws_bytes;
};

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

kvq_status make_plan(int32_t fmt, int32_t B, int32_t Hq, int32_t Hkv, int32_t D,
                     int32_t max_seq_len, int32_t num_splits, Plan* pl, int32_t window = 0) {
  kvq::DecodeConfig cfg;
  if (fmt < 0 || fmt > 3 || !kvq::decode_config(fmt, D, &cfg))
    return fail(KVQ_ERR_UNSUPPORTED, "format %d / head_dim %d", fmt, D);
  if (B < 0 || Hkv < 1 || Hq < Hkv || Hq % Hkv != 0)
    return fail(KVQ_ERR_INVALID_ARG, "num_seqs %d, num_q_heads %d, num_kv_heads %d", B, Hq, Hkv);
  if (max_seq_len < 0) return fail(KVQ_ERR_INVALID_ARG, "max_seq_len %d", max_seq_len);
  if (num_splits < 0) return fail(KVQ_ERR_INVALID_ARG, "num_splits %d", num_splits);
  pl->G = Hq / Hkv;
  pl->n_groups = (pl->G + 7) / 8;
  const int64_t units = (int64_t)B * Hkv * pl->n_groups;
  if (units > 0x7fffffff) return fail(KVQ_ERR_UNSUPPORTED, "too many (sequence, head) units");
  pl->units = (int)units;
  pl->pmax = (max_seq_len + KVQ_BLOCK_SIZE - 1) / KVQ_BLOCK_SIZE;
  if (window < 0) return fail(KVQ_ERR_INVALID_ARG, "window %d", window);
  if (window > 0) {  // a window's tokens span at most ceil(window / 16) + 1 pages
    const int wp = (window + KVQ_BLOCK_SIZE - 1) / KVQ_BLOCK_SIZE + 1;
    if (wp < pl->pmax) pl->pmax = wp;
  }
  const int64_t V = units * pl->pmax;
  const int sms = kvq::num_sms();
  int64_t ctas;
  if (V == 0) {
    ctas = units < sms ? units : sms;
  } else if (num_splits > 0) {
    ctas = units * num_splits;
  } else {
    ctas = V / (2 * cfg.warps);  // at least two pages per consumer warp
    if (ctas > sms) ctas = sms;
    // With fewer units than CTAs, a whole number of CTAs per unit keeps
    // every CTA inside one unit: a CTA whose range held two units would scan
    // them in turn, with a merge between (~8-10 us), and end last.  The other
    // way is to keep all CTAs and pad each unit's share with merge_pages
    // empty pages (below).
    if (ctas > units && ctas % units != 0) {
      const int64_t whole = ctas / units * units;
      bool take_whole;
      if (fmt == KVQ_FMT_BF16) {
        // BF16 pages stream at the HBM rate whatever the CTA count: whole
        // CTAs if that leaves out at most a tenth of them or costs each at
        // most ~96 more pages (4 x 32,768 tokens: 90.2 us whole, 92.2 padded)
        take_whole = whole * 10 >= ctas * 9 || V / whole - V / ctas <= 96;
      } else {
        // the quantized page loops are bound by instruction issue, so every
        // SM counts: whole CTAs unless the padded split gives each CTA at
        // least 5% fewer pages.  4 x 32,768 tokens on 148 SMs pads (512
        // against 471 pages a CTA; FP8 55.4 -> 54.0 us, NVFP4 59.5 -> 56.3);
        // 4 x 16,384 (256 against 249; 34.8 whole, 36.9 padded) and 8 units
        // of 65,536 tokens (228 against 228) stay whole.
        const int64_t per_whole = (V + whole - 1) / whole;
        const int64_t per_pad = (V + units * cfg.merge_pages + ctas - 1) / ctas;
        take_whole = per_pad * 105 >= per_whole * 100;
      }
      if (take_whole) ctas = whole;
    }
  }
  if (V > 0 && ctas > V) ctas = V;
  if (ctas > 4096) ctas = 4096;
  if (ctas < 1) ctas = 1;
  pl->ctas = (int)ctas;
  // Where units straddle CTAs, a CTA whose range holds a unit boundary stops
  // there for the first unit's merge and starts the next unit.  Each unit's
  // share of the partition gets merge_pages empty pages at its end, so such
  // a CTA scans about that many fewer pages and ends with the others (the
  // 4 x 126,976-token FP8 decode 167.9 -> 163.8 us).  The padding holds no work.
  if (V > 0 && num_splits == 0 && ctas > units && ctas % units != 0) pl->pmax += cfg.merge_pages;
  // A unit that straddles CTAs is finished from per-CTA partials (one slot
  // per (unit, CTA) pair) with an arrival counter per unit.
  bool spans = false;
  if (V > 0 && ctas > 1) spans = !(ctas <= units && units % ctas == 0);
  if (spans) {
    pl->off_part = align_up(sizeof(unsigned) * (size_t)units, 256);
    pl->ws_bytes = pl->off_part + sizeof(float) * (size_t)cfg.part_floats * (units + ctas);
  } else {
    pl->off_part = 0;
    pl->ws_bytes = 0;
  }
  return KVQ_OK;
}

// ---------------------------------------------------------------- TMA maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

kvq_status encode(CUtensorMap* m, CUtensorMapDataType dt, cuuint32_t rank, void* base,
                  const cuuint64_t* dims, const cuuint64_t* strides, const cuuint32_t* box,
                  CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return fail(KVQ_ERR_CUDA, "cuTensorMapEncodeTiled unavailable");
  const cuuint32_t es[5] = {1, 1, 1, 1, 1};
  auto call = [&] {
    return fn(m, dt, rank, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  };
  CUresult r = call();
  if (r == CUDA_ERROR_INVALID_CONTEXT) {
    // A host thread that has made no CUDA runtime call yet has no current
    // context, and the encoder (a driver call) needs one: make the current
    // device's primary context current, as the runtime's own launch would.
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess && cudaSetDevice(dev) == cudaSuccess) r = call();
  }
  if (r != CUDA_SUCCESS) return fail(KVQ_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return KVQ_OK;
}

// Descriptors for one cache buffer: [0] = codes/values tile of a head page,
// [1] = NVFP4 block-scale run of a head page (same as [0] otherwise).
kvq_status make_maps(int fmt, const kvq_cache* c, void* buf, CUtensorMap* tile, CUtensorMap* sf) {
  const cuuint64_t D = c->head_dim, H = c->num_kv_heads, nb = c->num_blocks;
  if (fmt == KVQ_FMT_PQ3) {  // head pages are fetched whole with bulk copies: no map
    memset(tile, 0, sizeof(*tile));
    memset(sf, 0, sizeof(*sf));
    return KVQ_OK;
  }
  if (fmt == KVQ_FMT_FP8_E4M3) {
    const cuuint64_t dims[4] = {D, 16, H, nb};
    const cuuint64_t str[3] = {D, 16 * D, 16 * D * H};
    const cuuint32_t box[4] = {(cuuint32_t)D, 16, 1, 1};
    kvq_status s = encode(tile, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, buf, dims, str, box,
                          D == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
    *sf = *tile;
    return s;
  }
  if (fmt == KVQ_FMT_BF16) {
    const cuuint64_t dims[4] = {D, 16, H, nb};
    const cuuint64_t str[3] = {2 * D, 32 * D, 32 * D * H};
    const cuuint32_t box[4] = {64, 16, 1, 1};
    kvq_status s = encode(tile, CU_TENSOR_MAP_DATA_TYPE_UINT16, 4, buf, dims, str, box,
                          CU_TENSOR_MAP_SWIZZLE_128B);
    *sf = *tile;
    return s;
  }
  // NVFP4: a head page is 16 rows of D/2 code bytes followed by 16 * D/16
  // scale bytes, i.e. 18 rows of D/2 bytes: one box covers codes and scales.
  const cuuint64_t dims[4] = {D / 2, 18, H, nb};
  const cuuint64_t str[3] = {D / 2, 9 * D, 9 * D * H};
  const cuuint32_t box[4] = {(cuuint32_t)(D / 2), 18, 1, 1};
  kvq_status s = encode(tile, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, buf, dims, str, box,
                        D == 64 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B);
  *sf = *tile;
  return s;
}

// The four tensor maps of a cache (K tile, V tile, K scales, V scales), from
// a small per-thread cache keyed by everything they encode: a decode step
// reuses the maps of the previous step instead of re-encoding them.
struct MapEntry {
  int32_t fmt, H, D;
  int64_t nb;
  const void* k;
  const void* v;
  int dev;
  CUtensorMap maps[4];
};
kvq_status cached_maps(int fmt, const kvq_cache* c, const CUtensorMap** out) {
  constexpr int kEntries = 8;
  thread_local MapEntry entries[kEntries];
  thread_local int n_used = 0, next = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  for (int i = 0; i < n_used; ++i) {
    const MapEntry& e = entries[i];
    if (e.fmt == fmt && e.H == c->num_kv_heads && e.D == c->head_dim && e.nb == c->num_blocks &&
        e.k == c->k && e.v == c->v && e.dev == dev) {
      *out = e.maps;
      return KVQ_OK;
    }
  }
  MapEntry& e = entries[next];
  e.k = nullptr;  // invalid until both encodes succeed
  kvq_status s = make_maps(fmt, c, c->k, &e.maps[0], &e.maps[2]);
  if (s != KVQ_OK) return s;
  s = make_maps(fmt, c, c->v, &e.maps[1], &e.maps[3]);
  if (s != KVQ_OK) return s;
  e.fmt = fmt;
  e.H = c->num_kv_heads;
  e.D = c->head_dim;
  e.nb = c->num_blocks;
  e.k = c->k;
  e.v = c->v;
  e.dev = dev;
  *out = e.maps;
  if (n_used < kEntries) ++n_used;
  next = (next + 1) % kEntries;
  return KVQ_OK;
}

}  // namespace

namespace kvq {
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

cudaError_t ensure_smem_attr(const void* func, size_t bytes, std::atomic<bool>* done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < kMaxDevices;
  if (tracked && done[dev].load(std::memory_order_acquire)) return cudaSuccess;
  e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess && tracked) done[dev].store(true, std::memory_order_release);
  return e;
}

int num_sms() {
  static std::atomic<int> cached[64];  // per device ordinal; 0 = not yet asked
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && (n = cached[dev].load(std::memory_order_relaxed)) > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64) cached[dev].store(n, std::memory_order_relaxed);
  return n;
}
}  // namespace kvq

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported";
    case KVQ_ERR_WORKSPACE: return "workspace missing or too small";
    case KVQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* kvq_last_error(void) { return g_err; }

kvq_status kv_cache_bytes(int32_t fmt, int64_t num_blocks, int32_t num_kv_heads,
                          int32_t head_dim, int64_t* bytes) {
  if (fmt < 0 || fmt > 3) return fail(KVQ_ERR_UNSUPPORTED, "unknown format %d", fmt);
  if (head_dim != 64 && head_dim != 128) return fail(KVQ_ERR_UNSUPPORTED, "head_dim %d", head_dim);
  if (fmt == KVQ_FMT_PQ3 && head_dim != 128)
    return fail(KVQ_ERR_UNSUPPORTED, "PQ3 needs head_dim 128 (got %d)", head_dim);
  if (num_blocks < 0 || num_kv_heads < 1 || !bytes)
    return fail(KVQ_ERR_INVALID_ARG, "num_blocks/num_kv_heads/bytes");
  *bytes = num_blocks * num_kv_heads * head_page_bytes(fmt, head_dim);
  return KVQ_OK;
}

kvq_status kv_pq3_codebook(float* cb) {
  if (!cb) return fail(KVQ_ERR_INVALID_ARG, "cb is NULL");
  // Lloyd's algorithm on the standard normal density: the thresholds are the
  // midpoints of neighbouring centroids, each centroid the density's mean
  // over its cell, iterated to a fixed point from evenly spaced centroids.
  const double inv_sqrt2pi = 0.3989422804014327, inv_sqrt2 = 0.7071067811865476;
  auto pdf = [&](double x) { return std::isinf(x) ? 0.0 : inv_sqrt2pi * std::exp(-0.5 * x * x); };
  auto cdf = [&](double x) { return 0.5 * std::erfc(-x * inv_sqrt2); };
  double c[8];
  for (int k = 0; k < 8; ++k) c[k] = (k - 3.5) * 0.5;
  for (int it = 0; it < 100000; ++it) {
    double t[9];
    t[0] = -INFINITY;
    t[8] = INFINITY;
    for (int k = 1; k < 8; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
    double moved = 0.0;
    for (int k = 0; k < 8; ++k) {
      const double m = (pdf(t[k]) - pdf(t[k + 1])) / (cdf(t[k + 1]) - cdf(t[k]));
      moved = std::fmax(moved, std::fabs(m - c[k]));
      c[k] = m;
    }
    if (moved < 1e-15) break;
  }
  // scale to one coordinate of a unit vector in 128 dimensions, then round to
  // the nearest f16 value (11 significant bits, ties to even)
  for (int k = 0; k < 8; ++k) {
    const double v = c[k] / std::sqrt(128.0);
    int e = 0;
    std::frexp(v, &e);
    const double ulp = std::ldexp(1.0, e - 11);
    cb[k] = static_cast<float>(std::nearbyint(v / ulp) * ulp);  // default rounding: to even
  }
  return KVQ_OK;
}

kvq_status kv_scale_from_absmax(int32_t fmt, float amax, float* scale) {
  if (fmt == KVQ_FMT_PQ3)
    return fail(KVQ_ERR_UNSUPPORTED, "PQ3 has no abs-max scale (see kv_pq3_codebook)");
  if (fmt < 0 || fmt > 2) return fail(KVQ_ERR_UNSUPPORTED, "unknown format %d", fmt);
  if (!scale) return fail(KVQ_ERR_INVALID_ARG, "scale is NULL");
  if (!(amax >= 0.0f) || isinf(amax)) return fail(KVQ_ERR_INVALID_ARG, "amax must be finite, >= 0");
  volatile float a = amax;  // keep the fp32 evaluation order literal
  if (fmt == KVQ_FMT_FP8_E4M3) {
    volatile float t = a * 1.05f;
    float s = t / 448.0f;
    if (s < 1e-12f) s = 1e-12f;
    *scale = s;
  } else if (fmt == KVQ_FMT_NVFP4) {
    *scale = a / 2688.0f;
  } else {
    *scale = 1.0f;
  }
  return KVQ_OK;
}

kvq_status kv_scale_from_absmax_device(int32_t fmt, const float* d_amax, float* d_scale,
                                       kvq_stream stream) {
  if (fmt == KVQ_FMT_PQ3)
    return fail(KVQ_ERR_UNSUPPORTED, "PQ3 has no abs-max scale (see kv_pq3_codebook)");
  if (fmt < 0 || fmt > 2) return fail(KVQ_ERR_UNSUPPORTED, "unknown format %d", fmt);
  if (!d_amax || !d_scale) return fail(KVQ_ERR_INVALID_ARG, "d_amax/d_scale is NULL");
  kvq_status s = check_device();
  if (s != KVQ_OK) return s;
  cudaError_t e = kvq::launch_scale(fmt, d_amax, d_scale, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e, "scale kernel");
}

kvq_status kv_calibrate_absmax(const void* x, int64_t n, float* d_amax, kvq_stream stream) {
  if (n < 0) return fail(KVQ_ERR_INVALID_ARG, "n %lld", (long long)n);
  if (!d_amax || !aligned(d_amax, 4)) return fail(KVQ_ERR_INVALID_ARG, "d_amax NULL or misaligned");
  if (n > 0 && (!x || !aligned(x, 2))) return fail(KVQ_ERR_INVALID_ARG, "x NULL or misaligned");
  kvq_status s = check_device();
  if (s != KVQ_OK) return s;
  cudaError_t e = kvq::launch_absmax(static_cast<const uint16_t*>(x), n, d_amax,
                                     static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e, "absmax kernel");
}

kvq_status kv_quantize_write(int32_t fmt, const void* k, const void* v, int64_t num_tokens,
                             const int64_t* slot_mapping, const int32_t* block_table,
                             int32_t num_seqs, int32_t max_blocks, const kvq_cache* cache,
                             const float* d_k_scale, const float* d_v_scale, int32_t* d_err,
                             kvq_stream stream) {
  kvq_status s = check_cache(fmt, cache);
  if (s != KVQ_OK) return s;
  if (num_tokens < 0) return fail(KVQ_ERR_INVALID_ARG, "num_tokens %lld", (long long)num_tokens);
  if (num_tokens > 0) {
    if (!k || !v || !aligned(k, 16) || !aligned(v, 16))
      return fail(KVQ_ERR_INVALID_ARG, "k/v NULL or not 16-byte aligned");
    if (!slot_mapping) return fail(KVQ_ERR_INVALID_ARG, "slot_mapping is NULL");
  }
  if (block_table && (num_seqs < 1 || max_blocks < 1))
    return fail(KVQ_ERR_INVALID_ARG, "block_table given with num_seqs %d, max_blocks %d",
                num_seqs, max_blocks);
  if (fmt != KVQ_FMT_BF16 && (!d_k_scale || !d_v_scale))
    return fail(KVQ_ERR_INVALID_ARG, "quantized formats need d_k_scale and d_v_scale");
  s = check_device();
  if (s != KVQ_OK) return s;
  kvq::QuantParams p;
  p.k = static_cast<const uint16_t*>(k);
  p.v = static_cast<const uint16_t*>(v);
  p.T = num_tokens;
  p.H = cache->num_kv_heads;
  p.D = cache->head_dim;
  p.slot_mapping = slot_mapping;
  p.block_table = block_table;
  p.num_seqs = num_seqs;
  p.max_blocks = max_blocks;
  p.num_blocks = cache->num_blocks;
  p.kc = static_cast<uint8_t*>(cache->k);
  p.vc = static_cast<uint8_t*>(cache->v);
  p.k_scale = d_k_scale;
  p.v_scale = d_v_scale;
  p.d_err = d_err;
  cudaError_t e = kvq::launch_quantize(fmt, p, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e, "quantize kernel");
}

kvq_status kv_decode_workspace_size(int32_t fmt, int32_t num_seqs, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t max_seq_len,
                                    int32_t num_splits, size_t* bytes) {
  if (!bytes) return fail(KVQ_ERR_INVALID_ARG, "bytes is NULL");
  kvq_status s = check_device();
  if (s != KVQ_OK) return s;
  Plan pl;
  s = make_plan(fmt, num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len, num_splits, &pl);
  if (s != KVQ_OK) return s;
  *bytes = pl.ws_bytes;
  return KVQ_OK;
}

kvq_status kv_decode_workspace_size_window(int32_t fmt, int32_t num_seqs, int32_t num_q_heads,
                                           int32_t num_kv_heads, int32_t head_dim,
                                           int32_t max_seq_len, int32_t window,
                                           int32_t num_splits, size_t* bytes) {
  if (!bytes) return fail(KVQ_ERR_INVALID_ARG, "bytes is NULL");
  kvq_status s = check_device();
  if (s != KVQ_OK) return s;
  Plan pl;
  s = make_plan(fmt, num_seqs, num_q_heads, num_kv_heads, head_dim, max_seq_len, num_splits, &pl,
                window);
  if (s != KVQ_OK) return s;
  *bytes = pl.ws_bytes;
  return KVQ_OK;
}

kvq_status kv_decode_attention(int32_t fmt, const void* q, const kvq_cache* cache,
                               const int32_t* block_table, int32_t max_blocks,
                               const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                               int32_t max_seq_len, int32_t num_splits, const float* d_k_scale,
                               const float* d_v_scale, float sm_scale, float* out, float* lse,
                               void* workspace, size_t workspace_bytes, int32_t* d_err,
                               kvq_stream stream) {
  return kv_decode_attention_window(fmt, q, cache, block_table, max_blocks, seq_lens, num_seqs,
                                    num_q_heads, max_seq_len, 0, num_splits, d_k_scale, d_v_scale,
                                    sm_scale, out, lse, workspace, workspace_bytes, d_err, stream);
}

}  // extern "C"

namespace {
// The decode launches behind kv_decode_attention, its window mode and its FP8
// attention variant (d_q_scale / d_prob_scale non-NULL: E4M3 Q and P).
kvq_status decode_impl(int32_t fmt, const void* q, const kvq_cache* cache,
                       const int32_t* block_table, int32_t max_blocks, const int32_t* seq_lens,
                       int32_t num_seqs, int32_t num_q_heads, int32_t max_seq_len, int32_t window,
                       int32_t num_splits, const float* d_k_scale, const float* d_v_scale,
                       const float* d_q_scale, const float* d_prob_scale, float sm_scale,
                       float* out, float* lse, void* workspace, size_t workspace_bytes,
                       int32_t* d_err, kvq_stream stream) {
  const bool qp = d_q_scale || d_prob_scale;
  kvq_status s = check_cache(fmt, cache);
  if (s != KVQ_OK) return s;
  const int D = cache->head_dim, Hkv = cache->num_kv_heads;
  if (num_seqs < 0) return fail(KVQ_ERR_INVALID_ARG, "num_seqs %d", num_seqs);
  if (num_seqs == 0) return KVQ_OK;
  if (!q || !aligned(q, 16)) return fail(KVQ_ERR_INVALID_ARG, "q NULL or not 16-byte aligned");
  if (!aligned(out, 16)) return fail(KVQ_ERR_INVALID_ARG, "out must be 16-byte aligned");
  if (!block_table || !seq_lens) return fail(KVQ_ERR_INVALID_ARG, "block_table/seq_lens NULL");
  if (!out || !aligned(out, 4)) return fail(KVQ_ERR_INVALID_ARG, "out NULL or misaligned");
  if (max_blocks < 1) return fail(KVQ_ERR_INVALID_ARG, "max_blocks %d", max_blocks);
  if (max_seq_len < 0 || (int64_t)max_seq_len > (int64_t)max_blocks * KVQ_BLOCK_SIZE)
    return fail(KVQ_ERR_INVALID_ARG, "max_seq_len %d exceeds max_blocks * 16", max_seq_len);
  if (fmt != KVQ_FMT_BF16 && (!d_k_scale || !d_v_scale))
    return fail(KVQ_ERR_INVALID_ARG, "quantized formats need d_k_scale and d_v_scale");
  if (qp) {
    if (fmt != KVQ_FMT_FP8_E4M3)
      return fail(KVQ_ERR_UNSUPPORTED, "FP8 attention needs an FP8 cache (format %d given)", fmt);
    if (!d_q_scale || !d_prob_scale)
      return fail(KVQ_ERR_INVALID_ARG, "FP8 attention needs d_q_scale and d_prob_scale");
    if (window != 0) return fail(KVQ_ERR_UNSUPPORTED, "FP8 attention has no window mode");
  }
  if (sm_scale == 0.0f) sm_scale = 1.0f / sqrtf((float)D);
  if (!isfinite(sm_scale)) return fail(KVQ_ERR_INVALID_ARG, "sm_scale not finite");
  s = check_device();
  if (s != KVQ_OK) return s;
  Plan pl;
  s = make_plan(fmt, num_seqs, num_q_heads, Hkv, D, max_seq_len, num_splits, &pl, window);
  if (s != KVQ_OK) return s;
  if (pl.ws_bytes > 0) {
    if (!workspace || !aligned(workspace, 256))
      return fail(KVQ_ERR_WORKSPACE, "workspace NULL or not 256-byte aligned (%zu bytes needed)",
                  pl.ws_bytes);
    if (workspace_bytes < pl.ws_bytes)
      return fail(KVQ_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", workspace_bytes,
                  pl.ws_bytes);
  }
  const CUtensorMap* maps = nullptr;
  s = cached_maps(fmt, cache, &maps);
  if (s != KVQ_OK) return s;

  kvq::DecodeParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.k_scale = d_k_scale;
  p.v_scale = d_v_scale;
  p.q_scale = d_q_scale;
  p.prob_scale = d_prob_scale;
  p.kc = static_cast<const uint8_t*>(cache->k);
  p.vc = static_cast<const uint8_t*>(cache->v);
  p.out = out;
  p.lse = lse;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_cnt = pl.ws_bytes ? reinterpret_cast<unsigned*>(ws) : nullptr;
  p.ws_part = pl.ws_bytes ? reinterpret_cast<float*>(ws + pl.off_part) : nullptr;
  p.d_err = d_err;
  p.num_blocks = cache->num_blocks;
  p.max_blocks = max_blocks;
  p.B = num_seqs;
  p.Hq = num_q_heads;
  p.Hkv = Hkv;
  p.G = pl.G;
  p.n_groups = pl.n_groups;
  p.units = pl.units;
  p.pmax = pl.pmax;
  p.max_seq_len = max_seq_len;
  p.window = window;
  p.sm_scale = sm_scale;
  cudaError_t e =
      kvq::launch_decode(fmt, D, maps, p, pl.ctas, static_cast<cudaStream_t>(stream), qp);
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e, "decode kernel");
}
}  // namespace

extern "C" {

kvq_status kv_decode_attention_window(int32_t fmt, const void* q, const kvq_cache* cache,
                                      const int32_t* block_table, int32_t max_blocks,
                                      const int32_t* seq_lens, int32_t num_seqs,
                                      int32_t num_q_heads, int32_t max_seq_len, int32_t window,
                                      int32_t num_splits, const float* d_k_scale,
                                      const float* d_v_scale, float sm_scale, float* out,
                                      float* lse, void* workspace, size_t workspace_bytes,
                                      int32_t* d_err, kvq_stream stream) {
  return decode_impl(fmt, q, cache, block_table, max_blocks, seq_lens, num_seqs, num_q_heads,
                     max_seq_len, window, num_splits, d_k_scale, d_v_scale, nullptr, nullptr,
                     sm_scale, out, lse, workspace, workspace_bytes, d_err, stream);
}

kvq_status kv_decode_attention_fp8qp(const void* q, const kvq_cache* cache,
                                     const int32_t* block_table, int32_t max_blocks,
                                     const int32_t* seq_lens, int32_t num_seqs,
                                     int32_t num_q_heads, int32_t max_seq_len, int32_t num_splits,
                                     const float* d_k_scale, const float* d_v_scale,
                                     const float* d_q_scale, const float* d_prob_scale,
                                     float sm_scale, float* out, float* lse, void* workspace,
                                     size_t workspace_bytes, int32_t* d_err, kvq_stream stream) {
  if (cache && cache->fmt != KVQ_FMT_FP8_E4M3)
    return fail(KVQ_ERR_UNSUPPORTED, "FP8 attention needs an FP8 cache (format %d given)",
                cache->fmt);
  if (!d_q_scale || !d_prob_scale)
    return fail(KVQ_ERR_INVALID_ARG, "FP8 attention needs d_q_scale and d_prob_scale");
  return decode_impl(KVQ_FMT_FP8_E4M3, q, cache, block_table, max_blocks, seq_lens, num_seqs,
                     num_q_heads, max_seq_len, 0, num_splits, d_k_scale, d_v_scale, d_q_scale,
                     d_prob_scale, sm_scale, out, lse, workspace, workspace_bytes, d_err, stream);
}

kvq_status kv_prefill_attention(int32_t fmt, const void* q, const kvq_cache* cache,
                                const int32_t* block_table, int32_t max_blocks,
                                const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_tokens,
                                int32_t num_q_heads, const float* d_k_scale,
                                const float* d_v_scale, float sm_scale, float* out, float* lse,
                                int32_t* d_err, kvq_stream stream) {
  kvq_status s = check_cache(fmt, cache);
  if (s != KVQ_OK) return s;
  if (fmt == KVQ_FMT_PQ3) return fail(KVQ_ERR_UNSUPPORTED, "no chunked prefill for PQ3");
  const int D = cache->head_dim, Hkv = cache->num_kv_heads;
  if (num_seqs < 0 || num_q_tokens < 0)
    return fail(KVQ_ERR_INVALID_ARG, "num_seqs %d / num_q_tokens %d", num_seqs, num_q_tokens);
  if (num_q_heads < 1 || num_q_heads % Hkv != 0)
    return fail(KVQ_ERR_INVALID_ARG, "num_q_heads %d not a multiple of num_kv_heads %d",
                num_q_heads, Hkv);
  const int G = num_q_heads / Hkv;
  if (G > kvq::prefill_rows())
    return fail(KVQ_ERR_UNSUPPORTED, "%d query heads per KV head (at most %d)", G,
                kvq::prefill_rows());
  if (num_seqs == 0 || num_q_tokens == 0) return KVQ_OK;
  if (!q || !aligned(q, 16)) return fail(KVQ_ERR_INVALID_ARG, "q NULL or not 16-byte aligned");
  if (!out || !aligned(out, 16)) return fail(KVQ_ERR_INVALID_ARG, "out NULL or not 16-byte aligned");
  if (!block_table || !seq_lens) return fail(KVQ_ERR_INVALID_ARG, "block_table/seq_lens NULL");
  if (max_blocks < 1) return fail(KVQ_ERR_INVALID_ARG, "max_blocks %d", max_blocks);
  if (fmt != KVQ_FMT_BF16 && (!d_k_scale || !d_v_scale))
    return fail(KVQ_ERR_INVALID_ARG, "quantized formats need d_k_scale and d_v_scale");
  if (sm_scale == 0.0f) sm_scale = 1.0f / sqrtf((float)D);
  if (!isfinite(sm_scale)) return fail(KVQ_ERR_INVALID_ARG, "sm_scale not finite");
  s = check_device();
  if (s != KVQ_OK) return s;
  kvq::PrefillParams p;
  p.q = static_cast<const uint16_t*>(q);
  p.block_table = block_table;
  p.seq_lens = seq_lens;
  p.kc = static_cast<const uint8_t*>(cache->k);
  p.vc = static_cast<const uint8_t*>(cache->v);
  p.k_scale = d_k_scale;
  p.v_scale = d_v_scale;
  p.out = out;
  p.lse = lse;
  p.d_err = d_err;
  p.num_blocks = cache->num_blocks;
  p.max_blocks = max_blocks;
  p.B = num_seqs;
  p.Tq = num_q_tokens;
  p.Hq = num_q_heads;
  p.Hkv = Hkv;
  p.G = G;
  p.QT = kvq::prefill_rows() / G;
  p.n_qblk = (num_q_tokens + p.QT - 1) / p.QT;
  p.sm_scale = sm_scale;
  const int64_t ctas = static_cast<int64_t>(p.n_qblk) * Hkv * num_seqs;
  if (ctas > 0x7fffffffLL) return fail(KVQ_ERR_INVALID_ARG, "problem too large (%lld CTAs)",
                                       (long long)ctas);
  cudaError_t e = kvq::launch_prefill(fmt, D, p, ctas, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e, "prefill kernel");
}

kvq_status kv_dequantize(int32_t fmt, const kvq_cache* cache, const int64_t* slots, int64_t n,
                         const float* d_k_scale, const float* d_v_scale, float* k_out,
                         float* v_out, int32_t* d_err, kvq_stream stream) {
  kvq_status s = check_cache(fmt, cache);
  if (s != KVQ_OK) return s;
  if (n < 0) return fail(KVQ_ERR_INVALID_ARG, "n %lld", (long long)n);
  if (n > 0 && (!slots || !k_out || !v_out || !aligned(k_out, 16) || !aligned(v_out, 16)))
    return fail(KVQ_ERR_INVALID_ARG, "slots/k_out/v_out NULL or outputs not 16-byte aligned");
  if (fmt != KVQ_FMT_BF16 && (!d_k_scale || !d_v_scale))
    return fail(KVQ_ERR_INVALID_ARG, "quantized formats need d_k_scale and d_v_scale");
  s = check_device();
  if (s != KVQ_OK) return s;
  cudaError_t e = kvq::launch_dequantize(
      fmt, static_cast<const uint8_t*>(cache->k), static_cast<const uint8_t*>(cache->v),
      cache->num_blocks, cache->num_kv_heads, cache->head_dim, slots, n, d_k_scale, d_v_scale,
      k_out, v_out, d_err, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? KVQ_OK : cuda_fail(e, "dequantize kernel");
}

}  // extern "C"
