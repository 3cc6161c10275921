/*
 * kvq_oracle.c -- plain, slow, obviously-correct CPU oracle for the quantized
 * KV-cache decode path (calibration abs-max, FP8/NVFP4/BF16 quantize-on-write
 * into a paged cache, dequantisation, and float64 decode attention).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library calls, links or
 * includes this file; only the tests, the smoke check and the benchmark's
 * CPU-baseline leg load it.  It shares no source with the CUDA path: the two
 * agree only on the documented data layout and the formulas below.
 *
 * Every step follows the definitions as written, in the order written, with no
 * blocking, fusion or reordering.  Sources:
 *   [FP8-KV] "FP8 KV calibration guide" (thetechpanda.github.io,
 *            radiance-R9700-vllm-experiments), the paragraph on the Radiance
 *            calibrator: per-layer abs-max of BF16 K/V activations, OCP E4M3
 *            convention, scale = max(observed_absolute_max * 1.05 / 448, 1e-12);
 *            and the paragraph on storage: BF16 uses 2 bytes per element, FP8 one.
 *   [NVFP4]  "I Tested NVFP4 vs FP8 KV Cache on Blackwell (One Refused to Boot)",
 *            "What you'll learn": E4M3 at one byte per number; NVFP4 is a
 *            block-scaled 4-bit float with FP8 scale factors, 4.5 bits per
 *            number.  The block recipe used here (16-element E2M1 blocks along
 *            head_dim, E4M3 block scale = block_absmax / (6 g), FP32 per-tensor
 *            g = tensor_absmax / (448 * 6)) is the recipe this library
 *            implements; the page fixes only the format family and its size.
 *   [FP8-KV], the paragraphs on the calibrator (it observes Q as well as K and
 *            V maxima) and on the Q/K/V-only sidecar (other attention paths
 *            accept probability scales): the FP8-attention variant at the end
 *            of this file, with E4M3 Q and E4M3 P.
 *   OCP 8-bit floating point specification (E4M3: bias 7, no infinities,
 *            S.1111.111 is NaN, max finite 448) and the OCP MX specification
 *            (E2M1: bias 1, magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6, no NaN/Inf).
 *
 * Parity status: every function here is pinned by a test that checks it
 * against something other than itself (library conversions, brute force,
 * closed forms, the pages' byte counts); see the tests directory.
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Format ids used by this oracle's C interface. */
#define ORC_BF16 0
#define ORC_FP8 1
#define ORC_NVFP4 2
#define ORC_F32 4 /* plain fp32 values, the dequantised form of another format */

#define ORC_PAGE 16 /* tokens per cache page (block size) */

/* ------------------------------------------------------------------------ */
/* BF16                                                                     */
/* ------------------------------------------------------------------------ */

/* A BF16 value is the upper half of an IEEE binary32; widening is exact. */
static float bf16_to_f32(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

float orc_bf16_to_f32(uint16_t b) { return bf16_to_f32(b); }

/* ------------------------------------------------------------------------ */
/* E4M3 (OCP FP8, "FN" flavour): 1 sign, 4 exponent bits (bias 7), 3 mantissa */
/* ------------------------------------------------------------------------ */

/* Decode from the bit fields.  exponent 0: (m/8) * 2^-6 (subnormal);
 * otherwise (1 + m/8) * 2^(e-7); S.1111.111 is NaN; there are no infinities. */
float orc_e4m3_decode(uint8_t c) {
  int s = (c >> 7) & 1;
  int e = (c >> 3) & 0xF;
  int m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = ((double)m / 8.0) * ldexp(1.0, -6);
  else
    v = (1.0 + (double)m / 8.0) * ldexp(1.0, e - 7);
  return (float)(s ? -v : v);
}

/* Round a non-negative double q to the nearest integer, ties to even. */
static double round_half_even(double q) {
  double f = floor(q);
  double r = q - f;
  if (r > 0.5) return f + 1.0;
  if (r < 0.5) return f;
  return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Encode by arithmetic on the binade: round to nearest, ties to even,
 * saturating to +-448 (satfinite); the sign is kept for results that round to
 * zero.  NaN inputs are outside the contract (returns the NaN code). */
uint8_t orc_e4m3_encode(float x) {
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  if (isnan(x)) return (uint8_t)(sign | 0x7F);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  if (a < ldexp(1.0, -6)) {
    /* subnormal range: step 2^-9; a result of 8 steps is the smallest normal */
    double q = round_half_even(a / ldexp(1.0, -9));
    return (uint8_t)(sign | (uint8_t)q); /* q in 0..8; 8 == code 0x08 */
  }
  int e2;
  frexp(a, &e2); /* a = f * 2^e2, f in [0.5, 1) -> binade exponent e2-1 */
  int e = e2 - 1;
  double q = round_half_even(a / ldexp(1.0, e - 3)); /* in [8, 16] */
  if (q == 16.0) {
    q = 8.0;
    e += 1;
  }
  int code = ((e + 7) << 3) | ((int)q - 8);
  if (code > 0x7E) code = 0x7E; /* cannot happen below 448; kept for clarity */
  return (uint8_t)(sign | code);
}

/* Brute force: scan the finite codes of the input's sign in increasing value
 * and keep the nearest one.  "Nearer" is decided against the exact midpoint of
 * the two candidates (representable in double), so huge inputs do not tie on
 * rounded distances; at a midpoint the code with mantissa LSB 0 wins.  Inputs
 * beyond the largest finite value therefore land on +-448 (satfinite). */
uint8_t orc_e4m3_encode_nearest(float x) {
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs((double)x);
  int best = 0;
  for (int c = 1; c <= 0x7E; c++) {
    double mid = ((double)orc_e4m3_decode((uint8_t)best) + (double)orc_e4m3_decode((uint8_t)c)) / 2;
    if (a > mid || (a == mid && (c & 1) == 0)) best = c;
  }
  return (uint8_t)(sign | best);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (OCP MX FP4): 1 sign (bit 3), 2 exponent bits (bias 1), 1 mantissa   */
/* ------------------------------------------------------------------------ */

float orc_e2m1_decode(uint8_t c) {
  int s = (c >> 3) & 1;
  int e = (c >> 1) & 3;
  int m = c & 1;
  double v = (e == 0) ? 0.5 * m : (1.0 + 0.5 * m) * ldexp(1.0, e - 1);
  return (float)(s ? -v : v);
}

uint8_t orc_e2m1_encode(float x) {
  uint8_t sign = signbit(x) ? 0x8 : 0x0;
  double a = fabs((double)x);
  if (isnan(x)) return (uint8_t)(sign | 0x7); /* outside the contract */
  if (a >= 6.0) return (uint8_t)(sign | 0x7);
  if (a < 1.0) {
    double q = round_half_even(a / 0.5); /* 0, 1 or 2 (2 == code 2 == 1.0) */
    return (uint8_t)(sign | (uint8_t)q);
  }
  int e2;
  frexp(a, &e2);
  int e = e2 - 1;                                     /* 0, 1 or 2 */
  double q = round_half_even(a / ldexp(1.0, e - 1)); /* in [2, 4] */
  if (q == 4.0) {
    q = 2.0;
    e += 1;
  }
  int code = ((e + 1) << 1) | ((int)q - 2);
  if (code > 7) code = 7;
  return (uint8_t)(sign | code);
}

/* Brute force over the 8 magnitudes, as for E4M3. */
uint8_t orc_e2m1_encode_nearest(float x) {
  uint8_t sign = signbit(x) ? 0x8 : 0x0;
  double a = fabs((double)x);
  int best = 0;
  for (int c = 1; c <= 7; c++) {
    double mid = ((double)orc_e2m1_decode((uint8_t)best) + (double)orc_e2m1_decode((uint8_t)c)) / 2;
    if (a > mid || (a == mid && (c & 1) == 0)) best = c;
  }
  return (uint8_t)(sign | best);
}

/* Array forms for exhaustive sweeps.  which: 0 = arithmetic, 1 = brute force. */
void orc_e4m3_encode_array(const float* x, uint8_t* out, int64_t n, int which) {
  for (int64_t i = 0; i < n; i++)
    out[i] = which ? orc_e4m3_encode_nearest(x[i]) : orc_e4m3_encode(x[i]);
}
void orc_e2m1_encode_array(const float* x, uint8_t* out, int64_t n, int which) {
  for (int64_t i = 0; i < n; i++)
    out[i] = which ? orc_e2m1_encode_nearest(x[i]) : orc_e2m1_encode(x[i]);
}
void orc_e4m3_decode_array(const uint8_t* c, float* out, int64_t n) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_decode(c[i]);
}
void orc_e2m1_decode_array(const uint8_t* c, float* out, int64_t n) {
  for (int64_t i = 0; i < n; i++) out[i] = orc_e2m1_decode(c[i] & 0xF);
}

/* ------------------------------------------------------------------------ */
/* Calibration and scales                                                   */
/* ------------------------------------------------------------------------ */

/* [FP8-KV] calibrator: the observed absolute maximum of a BF16 tensor. */
float orc_absmax_bf16(const uint16_t* x, int64_t n) {
  float m = 0.0f;
  for (int64_t i = 0; i < n; i++) {
    float a = fabsf(bf16_to_f32(x[i]));
    if (a > m) m = a;
  }
  return m;
}

/* [FP8-KV]: scale = max(observed_absolute_max * 1.05 / 448, 1e-12), evaluated
 * in fp32 left to right. */
float orc_fp8_scale(float amax) {
  float s = (amax * 1.05f) / 448.0f;
  if (s < 1e-12f) s = 1e-12f;
  return s;
}

/* NVFP4 per-tensor scale g = absmax / (448 * 6), fp32 (448 * 6 = 2688 exactly). */
float orc_nvfp4_global_scale(float amax) { return amax / (448.0f * 6.0f); }

/* ------------------------------------------------------------------------ */
/* Paged cache layout                                                       */
/* ------------------------------------------------------------------------ */
/*
 * K and V are separate buffers with identical layout.  A cache slot is
 * block * 16 + offset.  For head h of block blk the "head page" holds the 16
 * tokens of that block for that head:
 *   BF16 : uint16 [blk][h][16][D]
 *   FP8  : uint8  [blk][h][16][D]   (E4M3 codes)
 *   NVFP4: bytes  [blk][h][ 16*D/2 codes | 16*D/16 block scales ]  (9*D bytes)
 *          codes  [16][D/2]: element 2j in the low nibble, 2j+1 in the high one
 *          scales [16][D/16]: one E4M3 byte per 16-element block along D
 */
static int64_t head_page_index(int64_t blk, int h, int H) { return blk * H + h; }

/* Dequantised value of element (blk, h, o, d) as the fp32 the method defines:
 *   BF16 : the BF16 value;
 *   FP8  : fp32(dec_e4m3(code) * s);
 *   NVFP4: fp32(fp32(dec_e2m1(e) * dec_e4m3(sb)) * g)  (inner product exact). */
static float dequant_elem(int fmt, const void* cache, int64_t blk, int h, int o, int d, int H,
                          int D, float scale) {
  int64_t hp = head_page_index(blk, h, H);
  if (fmt == ORC_F32) {
    return ((const float*)cache)[(hp * ORC_PAGE + o) * D + d];
  } else if (fmt == ORC_BF16) {
    const uint16_t* c = (const uint16_t*)cache;
    return bf16_to_f32(c[(hp * ORC_PAGE + o) * D + d]);
  } else if (fmt == ORC_FP8) {
    const uint8_t* c = (const uint8_t*)cache;
    return orc_e4m3_decode(c[(hp * ORC_PAGE + o) * D + d]) * scale;
  } else {
    const uint8_t* base = (const uint8_t*)cache + hp * (int64_t)(9 * D);
    uint8_t byte = base[o * (D / 2) + d / 2];
    uint8_t e = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
    uint8_t sb = base[ORC_PAGE * (D / 2) + o * (D / 16) + d / 16];
    float elem = orc_e2m1_decode(e) * orc_e4m3_decode(sb);
    return elem * scale;
  }
}

int64_t orc_head_page_bytes(int fmt, int D) {
  if (fmt == ORC_F32) return (int64_t)ORC_PAGE * D * 4;
  if (fmt == 3) return (int64_t)ORC_PAGE * 52; /* PQ3, D = 128 (see below) */
  if (fmt == ORC_BF16) return (int64_t)ORC_PAGE * D * 2;
  if (fmt == ORC_FP8) return (int64_t)ORC_PAGE * D;
  return (int64_t)9 * D;
}

/* Bytes of one token's K and V for H heads of width D in the given format. */
double orc_kv_bytes_per_token(int fmt, int H, int D) {
  double per_elem = (fmt == ORC_BF16) ? 2.0 : (fmt == ORC_FP8) ? 1.0 : 4.5 / 8.0;
  return 2.0 * H * D * per_elem;
}

/* ------------------------------------------------------------------------ */
/* Quantize-on-write                                                        */
/* ------------------------------------------------------------------------ */

/* Quantize one [D] row of BF16 values into head page (blk, h) at offset o. */
static void write_row(int fmt, const uint16_t* x, void* cache, int64_t blk, int h, int o, int H,
                      int D, float scale) {
  int64_t hp = head_page_index(blk, h, H);
  if (fmt == ORC_BF16) {
    uint16_t* c = (uint16_t*)cache;
    for (int d = 0; d < D; d++) c[(hp * ORC_PAGE + o) * D + d] = x[d];
  } else if (fmt == ORC_FP8) {
    /* [FP8-KV]: code = E4M3(x / scale), fp32 division, RNE, satfinite. */
    uint8_t* c = (uint8_t*)cache;
    for (int d = 0; d < D; d++) {
      float v = bf16_to_f32(x[d]) / scale;
      c[(hp * ORC_PAGE + o) * D + d] = orc_e4m3_encode(v);
    }
  } else {
    /* NVFP4, one 16-element block at a time along D. */
    uint8_t* base = (uint8_t*)cache + hp * (int64_t)(9 * D);
    float g = scale;
    for (int blk16 = 0; blk16 < D / 16; blk16++) {
      float bmax = 0.0f;
      for (int i = 0; i < 16; i++) {
        float a = fabsf(bf16_to_f32(x[blk16 * 16 + i]));
        if (a > bmax) bmax = a;
      }
      uint8_t sb;
      float den;
      if (g > 0.0f) {
        sb = orc_e4m3_encode(bmax / (6.0f * g));
        den = orc_e4m3_decode(sb) * g;
      } else {
        sb = 0; /* g == 0: an all-zero tensor; every code is +0 */
        den = 0.0f;
      }
      base[ORC_PAGE * (D / 2) + o * (D / 16) + blk16] = sb;
      for (int i = 0; i < 16; i += 2) {
        int d = blk16 * 16 + i;
        uint8_t e0 = 0, e1 = 0;
        if (den != 0.0f) {
          e0 = orc_e2m1_encode(bf16_to_f32(x[d]) / den);
          e1 = orc_e2m1_encode(bf16_to_f32(x[d + 1]) / den);
        }
        base[o * (D / 2) + d / 2] = (uint8_t)(e0 | (e1 << 4));
      }
    }
  }
}

/* Write tokens [0, T) of k, v ([T][H][D] BF16) to the slots slot_mapping[t]
 * (block = slot / 16, offset = slot % 16).  A negative slot skips the token.
 * Returns 0, or -1 if a slot lies beyond the cache (nothing is written for it). */
int orc_write(int fmt, const uint16_t* k, const uint16_t* v, int64_t T, int H, int D,
              const int64_t* slot_mapping, int64_t num_blocks, void* k_cache, void* v_cache,
              float k_scale, float v_scale) {
  int rc = 0;
  for (int64_t t = 0; t < T; t++) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t blk = slot / ORC_PAGE;
    int o = (int)(slot % ORC_PAGE);
    if (blk >= num_blocks) {
      rc = -1;
      continue;
    }
    for (int h = 0; h < H; h++) {
      write_row(fmt, k + (t * H + h) * D, k_cache, blk, h, o, H, D, k_scale);
      write_row(fmt, v + (t * H + h) * D, v_cache, blk, h, o, H, D, v_scale);
    }
  }
  return rc;
}

/* Dequantise the listed slots into k_out, v_out ([n][H][D] fp32). */
int orc_dequantize(int fmt, const void* k_cache, const void* v_cache, int64_t num_blocks, int H,
                   int D, const int64_t* slots, int64_t n, float k_scale, float v_scale,
                   float* k_out, float* v_out) {
  for (int64_t i = 0; i < n; i++) {
    int64_t slot = slots[i];
    if (slot < 0 || slot / ORC_PAGE >= num_blocks) return -1;
    int64_t blk = slot / ORC_PAGE;
    int o = (int)(slot % ORC_PAGE);
    for (int h = 0; h < H; h++)
      for (int d = 0; d < D; d++) {
        k_out[(i * H + h) * D + d] = dequant_elem(fmt, k_cache, blk, h, o, d, H, D, k_scale);
        v_out[(i * H + h) * D + d] = dequant_elem(fmt, v_cache, blk, h, o, d, H, D, v_scale);
      }
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* Decode attention, float64                                                */
/* ------------------------------------------------------------------------ */

/*
 * Softmax attention of one query head over context tokens [t0, t1) of
 * sequence b, over the dequantised cache values, in float64:
 *   s_t = sm_scale * sum_d q_d * k_hat_{t,d}
 *   m   = max_t s_t,   l = sum_t exp(s_t - m),   o_unnorm = sum_t exp(s_t - m) v_hat_t
 * Token t of the sequence lives in block block_table[b][t / 16] at offset
 * t % 16.  Query head j reads KV head j / (Hq / H).  An empty range returns
 * m = -inf, l = 0, o_unnorm = 0.  Returns -1 if a block id is out of range.
 */
int orc_attention_range(int fmt, const uint16_t* q_row, const void* k_cache, const void* v_cache,
                        int64_t num_blocks, int H, int D, const int32_t* bt_row, int kv_head,
                        int64_t t0, int64_t t1, float k_scale, float v_scale, double sm_scale,
                        double* o_unnorm, double* m_out, double* l_out) {
  int64_t n = t1 - t0;
  for (int d = 0; d < D; d++) o_unnorm[d] = 0.0;
  if (n <= 0) {
    *m_out = -INFINITY;
    *l_out = 0.0;
    return 0;
  }
  double* s = (double*)malloc(sizeof(double) * (size_t)n);
  if (!s) return -2;
  double m = -INFINITY;
  for (int64_t t = t0; t < t1; t++) {
    int64_t blk = bt_row[t / ORC_PAGE];
    if (blk < 0 || blk >= num_blocks) {
      free(s);
      return -1;
    }
    int o = (int)(t % ORC_PAGE);
    double acc = 0.0;
    for (int d = 0; d < D; d++)
      acc += (double)bf16_to_f32(q_row[d]) *
             (double)dequant_elem(fmt, k_cache, blk, kv_head, o, d, H, D, k_scale);
    s[t - t0] = sm_scale * acc;
    if (s[t - t0] > m) m = s[t - t0];
  }
  double l = 0.0;
  for (int64_t t = t0; t < t1; t++) {
    double p = exp(s[t - t0] - m);
    l += p;
    int64_t blk = bt_row[t / ORC_PAGE];
    int o = (int)(t % ORC_PAGE);
    for (int d = 0; d < D; d++)
      o_unnorm[d] += p * (double)dequant_elem(fmt, v_cache, blk, kv_head, o, d, H, D, v_scale);
  }
  free(s);
  *m_out = m;
  *l_out = l;
  return 0;
}

/*
 * Decode step over a sliding window ("AMD MI300X — KV Cache Compression
 * Benchmark", section "SWA mode": only the most recent `window` tokens of the
 * cache are attended to).  Sequence b attends to its tokens
 * [max(0, len_b - window), len_b); window <= 0 means the whole context.
 * Otherwise as orc_decode_attention below.
 */
int orc_decode_attention_window(int fmt, const uint16_t* q, const void* k_cache,
                                const void* v_cache, int64_t num_blocks, int H, int D,
                                const int32_t* block_table, int max_blocks,
                                const int32_t* seq_lens, int B, int Hq, float k_scale,
                                float v_scale, double sm_scale, int32_t window,
                                const int32_t* pairs, int64_t n_pairs, double* out, double* lse) {
  int G = Hq / H;
  int64_t total = pairs ? n_pairs : (int64_t)B * Hq;
  for (int64_t i = 0; i < total; i++) {
    int b = pairs ? pairs[2 * i] : (int)(i / Hq);
    int j = pairs ? pairs[2 * i + 1] : (int)(i % Hq);
    int64_t len = seq_lens[b];
    int64_t t0 = (window > 0 && len > window) ? len - window : 0;
    double m, l;
    double* o = out + ((int64_t)b * Hq + j) * D;
    int rc = orc_attention_range(fmt, q + ((int64_t)b * Hq + j) * D, k_cache, v_cache, num_blocks,
                                 H, D, block_table + (int64_t)b * max_blocks, j / G, t0, len,
                                 k_scale, v_scale, sm_scale, o, &m, &l);
    if (rc) return rc;
    if (l > 0.0) {
      for (int d = 0; d < D; d++) o[d] /= l;
      lse[(int64_t)b * Hq + j] = m + log(l);
    } else {
      lse[(int64_t)b * Hq + j] = -INFINITY;
    }
  }
  return 0;
}

/*
 * Full decode step: out[b][j][:] = o_unnorm / l and lse[b][j] = m + ln(l) for
 * every sequence b and query head j (natural log, scaled-score units).  A
 * sequence of length 0 gives out = 0 and lse = -inf.  q is [B][Hq][D] BF16;
 * block_table is [B][max_blocks]; out is [B][Hq][D], lse [B][Hq] (float64).
 * If pairs is non-NULL, only the n_pairs (b, j) pairs listed in it (as
 * pairs[2i], pairs[2i+1]) are computed; other outputs are left untouched.
 */
int orc_decode_attention(int fmt, const uint16_t* q, const void* k_cache, const void* v_cache,
                         int64_t num_blocks, int H, int D, const int32_t* block_table,
                         int max_blocks, const int32_t* seq_lens, int B, int Hq, float k_scale,
                         float v_scale, double sm_scale, const int32_t* pairs, int64_t n_pairs,
                         double* out, double* lse) {
  return orc_decode_attention_window(fmt, q, k_cache, v_cache, num_blocks, H, D, block_table,
                                     max_blocks, seq_lens, B, Hq, k_scale, v_scale, sm_scale, 0,
                                     pairs, n_pairs, out, lse);
}

/*
 * Chunked-prefill attention: the Tq newest tokens of each sequence, already
 * written to the cache, attend causally to the cache.  Long prompts are fed
 * in chunks of a fixed token budget with the earlier prefix reused from the
 * cache ("Dual R9700 model and spec-decode campaign", fixed knobs:
 * long-prefill-token-threshold 2048 with prefix caching; "FP8 KV calibration
 * guide", first paragraph: TTFT at ~126k context with FP8 KV).
 *   Sequence b holds len_b = seq_lens[b] tokens; its query token i
 *   (0 <= i < Tq) sits at position p = len_b - Tq + i and attends to the
 *   cache tokens [0, p] (itself included), with the same scores, softmax and
 *   GQA mapping as a decode query.  A query with p < 0 (a sequence shorter
 *   than the chunk) attends to nothing: out = 0, lse = -inf.
 * q is [B][Tq][Hq][D] BF16; out is [B][Tq][Hq][D] and lse [B][Tq][Hq]
 * (float64).  If rows is non-NULL only the n_rows (b, i, j) triples listed in
 * it (rows[3r], rows[3r + 1], rows[3r + 2]) are computed; other outputs are
 * left untouched.
 */
int orc_prefill_attention(int fmt, const uint16_t* q, const void* k_cache, const void* v_cache,
                          int64_t num_blocks, int H, int D, const int32_t* block_table,
                          int max_blocks, const int32_t* seq_lens, int B, int Tq, int Hq,
                          float k_scale, float v_scale, double sm_scale, const int32_t* rows,
                          int64_t n_rows, double* out, double* lse) {
  int G = Hq / H;
  int64_t total = rows ? n_rows : (int64_t)B * Tq * Hq;
  for (int64_t r = 0; r < total; r++) {
    int b = rows ? rows[3 * r] : (int)(r / ((int64_t)Tq * Hq));
    int i = rows ? rows[3 * r + 1] : (int)((r / Hq) % Tq);
    int j = rows ? rows[3 * r + 2] : (int)(r % Hq);
    int64_t row = ((int64_t)b * Tq + i) * Hq + j;
    int64_t p = (int64_t)seq_lens[b] - Tq + i;
    double m, l;
    double* o = out + row * D;
    int rc = orc_attention_range(fmt, q + row * D, k_cache, v_cache, num_blocks, H, D,
                                 block_table + (int64_t)b * max_blocks, j / G, 0, p + 1, k_scale,
                                 v_scale, sm_scale, o, &m, &l);
    if (rc) return rc;
    if (l > 0.0) {
      for (int d = 0; d < D; d++) o[d] /= l;
      lse[row] = m + log(l);
    } else {
      lse[row] = -INFINITY;
    }
  }
  return 0;
}

/*
 * Merge of n partial results (o_unnorm_i, m_i, l_i) of disjoint context
 * ranges into the full one:
 *   M = max_i m_i,  L = sum_i exp(m_i - M) l_i,
 *   out = sum_i exp(m_i - M) o_unnorm_i / L,  lse = M + ln L.
 * Parts with m_i = -inf (empty ranges) contribute nothing.
 */
void orc_merge(int n, int D, const double* o_parts, const double* m_parts, const double* l_parts,
               double* out, double* lse) {
  double M = -INFINITY;
  for (int i = 0; i < n; i++)
    if (m_parts[i] > M) M = m_parts[i];
  for (int d = 0; d < D; d++) out[d] = 0.0;
  if (M == -INFINITY) {
    *lse = -INFINITY;
    return;
  }
  double L = 0.0;
  for (int i = 0; i < n; i++) {
    if (m_parts[i] == -INFINITY) continue;
    double w = exp(m_parts[i] - M);
    L += w * l_parts[i];
    for (int d = 0; d < D; d++) out[d] += w * o_parts[(int64_t)i * D + d];
  }
  for (int d = 0; d < D; d++) out[d] /= L;
  *lse = M + log(L);
}

/* ------------------------------------------------------------------------ */
/* FP8 attention over an FP8 cache: E4M3 Q and E4M3 P                       */
/* ------------------------------------------------------------------------ */
/*
 * [FP8-KV], paragraph on the Radiance calibrator: it observes the BF16 Q, K
 * and V activation maxima and writes per-layer E4M3 scales with the formula of
 * orc_fp8_scale; and the paragraph on the Q/K/V-only sidecar: other attention
 * paths also accept a probability scale (prob_scale).  With Q and the softmax
 * probabilities P in E4M3 as well as K and V, both attention products take
 * E4M3 operands.  The pages fix no more than that; this is the plain reading
 * the oracle takes, step by step:
 *   1. q_hat_d = E4M3(q_d / q_scale)  (fp32 division, RNE, satfinite, as the
 *      cache write);
 *   2. s_t = sm_scale * q_scale * k_scale * sum_d dec(q_hat_d) dec(k_{t,d});
 *   3. P is quantized page by page (the cache's 16-token blocks), relative to
 *      the page's largest score m_i, so that each page's largest probability
 *      is 1: p_t = exp(s_t - m_i), p_hat_t = dec(E4M3(p_t / prob_scale)) *
 *      prob_scale (the decision taken on fp32(p_t) * fp32(1 / prob_scale));
 *   4. the normaliser uses the unquantized probabilities, and pages merge by
 *      log-sum-exp: M = max_i m_i,
 *        out = sum_i exp(m_i - M) sum_{t in i} p_hat_t v_hat_t
 *              / sum_i exp(m_i - M) sum_{t in i} p_t,
 *        lse = M + ln(sum_i exp(m_i - M) sum_{t in i} p_t).
 * Only the FP8 cache format takes this path (its K and V are E4M3 already).
 *
 * Where floating point decides a code, the GPU decides on its own fp32 p_t,
 * which can differ from this float64 p_t in the last bits.  For the checks,
 * amb (if not NULL, [B][Hq][D] like out) receives a bound on how far each
 * output can move if every p_t whose fp32(p_t) * fp32(1 / prob_scale) lies
 * within relative distance eps of an E4M3 rounding boundary took the other
 * neighbouring code:
 *   amb_d = sum over such t of exp(m_i - M) * |other - chosen| * prob_scale *
 *           |v_hat_{t,d}| / L.
 */

/* The two E4M3 neighbours of a finite x in [0, 448]: lo <= x <= hi (equal
 * when x is representable). */
static void e4m3_neighbours(double x, double* lo, double* hi) {
  double best_lo = 0.0, best_hi = 448.0;
  for (int c = 0; c <= 0x7E; c++) {
    double v = (double)orc_e4m3_decode((uint8_t)c);
    if (v <= x && v > best_lo) best_lo = v;
    if (v >= x && v < best_hi) best_hi = v;
  }
  *lo = best_lo;
  *hi = best_hi;
}

int orc_decode_attention_fp8qp(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                               int64_t num_blocks, int H, int D, const int32_t* block_table,
                               int max_blocks, const int32_t* seq_lens, int B, int Hq,
                               float k_scale, float v_scale, float q_scale, float prob_scale,
                               double sm_scale, double eps, const int32_t* pairs,
                               int64_t n_pairs, double* out, double* lse, double* amb) {
  int G = Hq / H;
  int64_t total = pairs ? n_pairs : (int64_t)B * Hq;
  float inv_ps = 1.0f / prob_scale;
  for (int64_t i = 0; i < total; i++) {
    int b = pairs ? pairs[2 * i] : (int)(i / Hq);
    int j = pairs ? pairs[2 * i + 1] : (int)(i % Hq);
    int kv = j / G;
    int64_t len = seq_lens[b];
    const uint16_t* q_row = q + ((int64_t)b * Hq + j) * D;
    const int32_t* bt_row = block_table + (int64_t)b * max_blocks;
    int64_t row = (int64_t)b * Hq + j;
    double* o = out + row * D;
    for (int d = 0; d < D; d++) o[d] = 0.0;
    if (amb)
      for (int d = 0; d < D; d++) amb[row * D + d] = 0.0;
    if (len <= 0) {
      lse[row] = -INFINITY;
      continue;
    }
    double* qh = (double*)malloc(sizeof(double) * (size_t)D);
    double* s = (double*)malloc(sizeof(double) * (size_t)len);
    double* w = (double*)malloc(sizeof(double) * (size_t)len);
    if (!qh || !s || !w) {
      free(qh);
      free(s);
      free(w);
      return -2;
    }
    /* step 1: the quantized query */
    for (int d = 0; d < D; d++) {
      float x = bf16_to_f32(q_row[d]) / q_scale;
      qh[d] = (double)orc_e4m3_decode(orc_e4m3_encode(x));
    }
    /* step 2: scores over the E4M3 values */
    for (int64_t t = 0; t < len; t++) {
      int64_t blk = bt_row[t / ORC_PAGE];
      if (blk < 0 || blk >= num_blocks) {
        free(qh);
        free(s);
        free(w);
        return -1;
      }
      int off = (int)(t % ORC_PAGE);
      const uint8_t* krow = k_cache + ((blk * H + kv) * ORC_PAGE + off) * (int64_t)D;
      double acc = 0.0;
      for (int d = 0; d < D; d++) acc += qh[d] * (double)orc_e4m3_decode(krow[d]);
      s[t] = sm_scale * (double)q_scale * (double)k_scale * acc;
    }
    /* M: the largest score (the largest page maximum) */
    double M = -INFINITY;
    for (int64_t t = 0; t < len; t++)
      if (s[t] > M) M = s[t];
    /* steps 3-4, page by page */
    double L = 0.0;
    for (int64_t p0 = 0; p0 < len; p0 += ORC_PAGE) {
      int64_t p1 = p0 + ORC_PAGE < len ? p0 + ORC_PAGE : len;
      double mi = -INFINITY;
      for (int64_t t = p0; t < p1; t++)
        if (s[t] > mi) mi = s[t];
      double f = exp(mi - M);
      for (int64_t t = p0; t < p1; t++) {
        double p = exp(s[t] - mi);
        float x = (float)p * inv_ps;
        uint8_t code = orc_e4m3_encode(x);
        double chosen = (double)orc_e4m3_decode(code);
        L += f * p;
        int64_t blk = bt_row[t / ORC_PAGE];
        int off = (int)(t % ORC_PAGE);
        const uint8_t* vrow = v_cache + ((blk * H + kv) * ORC_PAGE + off) * (int64_t)D;
        for (int d = 0; d < D; d++) {
          double v = (double)orc_e4m3_decode(vrow[d]) * (double)v_scale;
          o[d] += f * chosen * (double)prob_scale * v;
        }
        /* a rounding boundary within relative eps of x: the other neighbour
         * is a possible code too */
        double lo, hi;
        e4m3_neighbours((double)x, &lo, &hi);
        double other = chosen == lo ? hi : lo;
        int near = (double)x < 448.0 && fabs((double)x - 0.5 * (lo + hi)) <= eps * (double)x;
        w[t] = near ? f * fabs(other - chosen) * (double)prob_scale : 0.0;
      }
    }
    for (int d = 0; d < D; d++) o[d] /= L;
    lse[row] = M + log(L);
    if (amb)
      for (int64_t t = 0; t < len; t++) {
        if (w[t] == 0.0) continue;
        int64_t blk = bt_row[t / ORC_PAGE];
        int off = (int)(t % ORC_PAGE);
        const uint8_t* vrow = v_cache + ((blk * H + kv) * ORC_PAGE + off) * (int64_t)D;
        for (int d = 0; d < D; d++)
          amb[row * D + d] += w[t] * fabs((double)orc_e4m3_decode(vrow[d]) * (double)v_scale) / L;
      }
    free(qh);
    free(s);
    free(w);
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* PQ3: 3-bit planar-rotation codec of 128-element vectors (52-byte blocks)  */
/* ------------------------------------------------------------------------ */
/*
 * [MI300X] "AMD MI300X - KV Cache Compression Benchmark", "Key Results": the
 * 3-bit methods share one 52-byte block layout at 4.923x compression against
 * FP16 (a 128-element FP16 vector is 256 bytes; 256 / 52 = 4.923), with a
 * reconstruction cosine similarity of 0.983; PlanarQuant needs the fewest
 * FMAs (256 against 16,384 for a dense 128 x 128 rotation), and the
 * repository lists a Lloyd-Max solver and codebook generator.  The page fixes
 * no more; the plain reading this oracle takes:
 *   block  = one 128-element head vector: its fp32 L2 norm (4 bytes) and 128
 *            3-bit codebook indices (48 bytes);
 *   rotate = 64 planar rotations of the coordinate pairs (2j, 2j+1) by
 *            seeded angles, given as fp32 (cos_j, sin_j) (4 multiplies a
 *            pair: the 256 FMAs);
 *   codebook = the 8-level Lloyd-Max quantizer of N(0, 1/128), the law of
 *            one coordinate of a random unit vector in 128 dimensions
 *            (Gaussian approximation), rounded to f16 values;
 *   encode = u = x / |x|, y = R u, index = nearest codebook value;
 *   decode = |x| * R^T c[index].
 * Every fp32 step of the encode is fixed so the indices are exact:
 *   ss  = sum of x_i^2 as a pairwise tree in index order (level 1 adds
 *         elements 2i and 2i+1, each further level adds adjacent sums);
 *   nrm = sqrt(ss) rounded to nearest; u_i = x_i / nrm (IEEE division);
 *   y_2j = fmaf(c_j, u_2j, -(s_j * u_2j+1)), y_2j+1 = fmaf(s_j, u_2j, c_j * u_2j+1);
 *   index = number of thresholds t_k = (c_k + c_k+1) / 2 (fp32) below y
 *         (y equal to a threshold takes the lower index);
 *   nrm = 0 (an all-zero vector) stores norm 0 and indices 0.
 * The dequantised element (fp32): with Y0 = c[i_2j], Y1 = c[i_2j+1],
 *   x_hat_2j = nrm * fmaf(c_j, Y0, s_j * Y1), x_hat_2j+1 = nrm * fmaf(c_j, Y1, -(s_j * Y0)).
 * Layout of a 16-token head page (832 bytes): the 16 norms (fp32), then 16
 * rows of 48 index bytes.  A row is two bit planes of its 128 indices, as a
 * little-endian bit string of 384 bits (the page fixes only the 3 bits an
 * index; the planes let a reader turn indices into byte-permute selectors
 * with a few masks):
 *   low plane, bits 0..255: the low 2 bits of index i = 16w + e (e < 16) at
 *     bit 32w + 4 (e % 8) + 2 (e / 8);
 *   high plane, bits 256..383: bit 2 of index i = 32v + e (e < 32) at bit
 *     256 + 32v + 4 (e % 8) + {2, 3, 0, 1}[e / 8].
 * The per-layer parameter block of a tensor (K or V): 8 codebook values then
 * the 64 (cos, sin) pairs, 136 fp32.
 */
#define ORC_PQ3 3
#define ORC_PQ3_D 128
#define ORC_PQ3_PAGE_BYTES (ORC_PAGE * 4 + ORC_PAGE * 48)

/* Standard normal density and distribution function. */
static double std_pdf(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * 3.14159265358979323846); }
static double std_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* The n-level Lloyd-Max quantizer of N(0, 1): centroids c_0 < ... < c_{n-1}
 * satisfying both conditions (each threshold is the midpoint of its two
 * centroids; each centroid is the mean of the density over its cell),
 * reached by Lloyd's fixed-point iteration from equally spaced centroids. */
void orc_lloyd_max_gaussian(int n, double* c) {
  for (int k = 0; k < n; k++) c[k] = -2.0 + 4.0 * (k + 0.5) / n;
  for (int it = 0; it < 100000; it++) {
    double change = 0.0;
    for (int k = 0; k < n; k++) {
      double lo = k == 0 ? -INFINITY : 0.5 * (c[k - 1] + c[k]);
      double hi = k == n - 1 ? INFINITY : 0.5 * (c[k] + c[k + 1]);
      double mass = std_cdf(hi) - std_cdf(lo);
      double mean = (std_pdf(lo) - std_pdf(hi)) / mass; /* E[X | lo < X < hi] */
      change = fmax(change, fabs(mean - c[k]));
      c[k] = mean;
    }
    if (change < 1e-15) break;
  }
}

/* Round a double to the nearest f16 value (ties to even), as a double; the
 * values here are normal f16 numbers (|v| in [2^-14, 65504]). */
static double round_to_f16(double v) {
  int e;
  frexp(v, &e);                   /* v = f * 2^e, f in [0.5, 1) */
  double ulp = ldexp(1.0, e - 11); /* 11 significant bits */
  return round_half_even(fabs(v) / ulp) * ulp * (v < 0 ? -1.0 : 1.0);
}

/* The PQ3 codebook: the 8-level Lloyd-Max centroids scaled by 1/sqrt(128),
 * rounded to f16, as fp32. */
void orc_pq3_codebook(float* cb) {
  double c[8];
  orc_lloyd_max_gaussian(8, c);
  for (int k = 0; k < 8; k++) cb[k] = (float)round_to_f16(c[k] / sqrt(128.0));
}

/* Pairwise-tree fp32 sum of squares of a 128-element BF16 row. */
static float pq3_sum_squares(const uint16_t* x) {
  float s[ORC_PQ3_D];
  for (int i = 0; i < ORC_PQ3_D; i++) {
    float v = bf16_to_f32(x[i]);
    s[i] = v * v; /* exact: a BF16 square has at most 16 significant bits */
  }
  for (int n = ORC_PQ3_D; n > 1; n /= 2)
    for (int i = 0; i < n / 2; i++) s[i] = s[2 * i] + s[2 * i + 1];
  return s[0];
}

/* Encode one row: norm and 128 indices (one byte each here). */
static void pq3_encode(const uint16_t* x, const float* params, float* nrm_out, uint8_t* idx) {
  const float* cb = params;
  const float* rot = params + 8;
  float nrm = sqrtf(pq3_sum_squares(x));
  *nrm_out = nrm;
  if (nrm == 0.0f) {
    for (int i = 0; i < ORC_PQ3_D; i++) idx[i] = 0;
    return;
  }
  float thr[7];
  for (int k = 0; k < 7; k++) thr[k] = (cb[k] + cb[k + 1]) / 2.0f;
  for (int j = 0; j < ORC_PQ3_D / 2; j++) {
    float c = rot[2 * j], s = rot[2 * j + 1];
    float u0 = bf16_to_f32(x[2 * j]) / nrm, u1 = bf16_to_f32(x[2 * j + 1]) / nrm;
    float y[2];
    y[0] = fmaf(c, u0, -(s * u1));
    y[1] = fmaf(s, u0, c * u1);
    for (int h = 0; h < 2; h++) {
      int k = 0;
      while (k < 7 && y[h] > thr[k]) k++;
      idx[2 * j + h] = (uint8_t)k;
    }
  }
}

/* The dequantised fp32 row of a norm and 128 indices. */
static void pq3_decode(float nrm, const uint8_t* idx, const float* params, float* out) {
  const float* cb = params;
  const float* rot = params + 8;
  for (int j = 0; j < ORC_PQ3_D / 2; j++) {
    float c = rot[2 * j], s = rot[2 * j + 1];
    float y0 = cb[idx[2 * j]], y1 = cb[idx[2 * j + 1]];
    out[2 * j] = nrm * fmaf(c, y0, s * y1);
    out[2 * j + 1] = nrm * fmaf(c, y1, -(s * y0));
  }
}

/* Bit positions (in the row's 384-bit string) of index i's three bits:
 * bit k of the index at pq3_bit(i, k). */
static int pq3_bit(int i, int k) {
  static const int high_slot[4] = {2, 3, 0, 1};
  if (k < 2) {
    const int e = i % 16;
    return 32 * (i / 16) + 4 * (e % 8) + 2 * (e / 8) + k;
  }
  const int e = i % 32;
  return 256 + 32 * (i / 32) + 4 * (e % 8) + high_slot[e / 8];
}

static void pq3_pack(const uint8_t* idx, uint8_t* bytes48) {
  for (int b = 0; b < 48; b++) bytes48[b] = 0;
  for (int i = 0; i < ORC_PQ3_D; i++)
    for (int k = 0; k < 3; k++)
      if ((idx[i] >> k) & 1) {
        const int b = pq3_bit(i, k);
        bytes48[b / 8] |= (uint8_t)(1u << (b % 8));
      }
}

static void pq3_unpack(const uint8_t* bytes48, uint8_t* idx) {
  for (int i = 0; i < ORC_PQ3_D; i++) {
    int v = 0;
    for (int k = 0; k < 3; k++) {
      const int b = pq3_bit(i, k);
      v |= ((bytes48[b / 8] >> (b % 8)) & 1) << k;
    }
    idx[i] = (uint8_t)v;
  }
}

/* Encode / decode one row (exposed for the checks). */
void orc_pq3_encode_row(const uint16_t* x, const float* params, float* nrm, uint8_t* idx) {
  pq3_encode(x, params, nrm, idx);
}
void orc_pq3_decode_row(float nrm, const uint8_t* idx, const float* params, float* out) {
  pq3_decode(nrm, idx, params, out);
}

/* Quantize-on-write of tokens [0, T) of k, v ([T][H][128] BF16) to the
 * physical slots slot_mapping[t] (negative: skip).  Returns -1 if a slot lies
 * beyond the cache (nothing written for it), else 0. */
int orc_pq3_write(const uint16_t* k, const uint16_t* v, int64_t T, int H,
                  const int64_t* slot_mapping, int64_t num_blocks, uint8_t* k_cache,
                  uint8_t* v_cache, const float* k_params, const float* v_params) {
  int rc = 0;
  for (int64_t t = 0; t < T; t++) {
    int64_t slot = slot_mapping[t];
    if (slot < 0) continue;
    int64_t blk = slot / ORC_PAGE;
    int o = (int)(slot % ORC_PAGE);
    if (blk >= num_blocks) {
      rc = -1;
      continue;
    }
    for (int h = 0; h < H; h++)
      for (int kv = 0; kv < 2; kv++) {
        const uint16_t* x = (kv ? v : k) + (t * H + h) * ORC_PQ3_D;
        uint8_t* page = (kv ? v_cache : k_cache) + (blk * H + h) * (int64_t)ORC_PQ3_PAGE_BYTES;
        float nrm;
        uint8_t idx[ORC_PQ3_D];
        pq3_encode(x, kv ? v_params : k_params, &nrm, idx);
        memcpy(page + 4 * o, &nrm, 4);
        pq3_pack(idx, page + ORC_PAGE * 4 + 48 * o);
      }
  }
  return rc;
}

/* Dequantise the whole PQ3 cache into fp32 caches [num_blocks][H][16][128]
 * (the float format the attention oracle reads). */
void orc_pq3_to_f32(const uint8_t* k_cache, const uint8_t* v_cache, int64_t num_blocks, int H,
                    const float* k_params, const float* v_params, float* k_out, float* v_out) {
  for (int64_t hp = 0; hp < num_blocks * H; hp++)
    for (int kv = 0; kv < 2; kv++) {
      const uint8_t* page = (kv ? v_cache : k_cache) + hp * (int64_t)ORC_PQ3_PAGE_BYTES;
      float* dst = (kv ? v_out : k_out) + hp * ORC_PAGE * ORC_PQ3_D;
      for (int o = 0; o < ORC_PAGE; o++) {
        float nrm;
        uint8_t idx[ORC_PQ3_D];
        memcpy(&nrm, page + 4 * o, 4);
        pq3_unpack(page + ORC_PAGE * 4 + 48 * o, idx);
        pq3_decode(nrm, idx, kv ? v_params : k_params, dst + o * ORC_PQ3_D);
      }
    }
}
