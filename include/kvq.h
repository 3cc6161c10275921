/*
 * kvq.h -- C ABI of libkvq: attention over a quantized, paged KV cache on
 * NVIDIA B200 (sm_100a).
 *
 * The library computes the decode-time hot path the pages describe:
 *   1. a calibration abs-max reduction and the per-layer FP8 scale
 *      ("FP8 KV calibration guide", paragraph on the Radiance calibrator:
 *      scale = max(observed_absolute_max * 1.05 / 448, 1e-12), OCP E4M3);
 *   2. quantize-on-write of BF16 K/V into a paged cache as FP8 E4M3 or NVFP4
 *      ("I Tested NVFP4 vs FP8 KV Cache on Blackwell", "What you'll learn":
 *      E4M3 at one byte per number; NVFP4 is a block-scaled 4-bit float with
 *      FP8 block scales, 4.5 bits per number), or as plain BF16;
 *   3. decode-step attention that scans the cache with the dequantisation
 *      fused into the scan (same page, chapter "The Missing Fused Dequant
 *      Kernel": without that fusion, halving the bytes gave no speedup), with
 *      grouped-query heads, online softmax and split-K over the context merged
 *      by log-sum-exp in the same launch;
 *   4. dequantisation of chosen slots, for checking.
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The
 *     library allocates no device memory at run time.  The host state it
 *     keeps is small and safe to share between threads: per device ordinal,
 *     the capability check, the SM count and whether each kernel's shared-
 *     memory limit has been raised; per calling thread, the text of the last
 *     error and the TMA descriptors of the last few caches it decoded (keyed
 *     by device, buffer addresses and geometry, so a reused address with the
 *     same geometry encodes the same descriptor).  The only device state is
 *     the fixed scratch array of kv_decode_attention_static_ws (below).
 *   - Every call is asynchronous on the given stream (a cudaStream_t passed
 *     as kvq_stream; NULL means the legacy default stream) and never
 *     synchronises.
 *   - Host-side argument errors return a status and launch nothing;
 *     kvq_last_error() then describes the failing argument (per thread).
 *   - Problems only visible on the device (a block id outside the pool, a
 *     slot beyond the cache, a non-positive or non-finite scale, a sequence
 *     length above the stated maximum) are OR-ed into the caller's int32
 *     error word d_err as KVQ_DERR_* bits; the offending page, token or
 *     sequence is skipped.  The caller zeroes d_err and reads it after its own
 *     synchronisation.  No kernel traps.
 *   - There is no default scale: every quantized format needs the caller's
 *     scale (a scale silently falling back to 1.0 is the failure mode the
 *     "FP4 kv path for a single 5090" discussion reports for long contexts).
 *   - Only devices of compute capability 10.0 (B200) are accepted; any other
 *     returns KVQ_ERR_UNSUPPORTED.
 *
 * Cache layout (block size 16 tokens; a slot is block * 16 + offset).  K and
 * V are two buffers with the same layout.  For KV head h of block b the
 * "head page" holds the 16 tokens of b for h:
 *   KVQ_FMT_BF16     : bf16  [num_blocks][num_kv_heads][16][head_dim]
 *   KVQ_FMT_FP8_E4M3 : uint8 [num_blocks][num_kv_heads][16][head_dim]
 *   KVQ_FMT_NVFP4    : bytes [num_blocks][num_kv_heads][9 * head_dim], each
 *                      head page = codes [16][head_dim/2] (E2M1; element 2j
 *                      in the low nibble, 2j+1 in the high one) followed by
 *                      block scales [16][head_dim/16] (one E4M3 byte per
 *                      16-element block along head_dim): 4.5 bits/element.
 * Pages are sized by their compressed bytes, never padded to BF16 size (the
 * FP8 KV calibration guide attributes an earlier flat FP8 capacity to
 * BF16-sized padded pages).
 *
 * Scales (one fp32 device scalar for K and one for V, per layer):
 *   FP8  : s; code = E4M3(x / s) (fp32 division, round to nearest even,
 *          saturating to +-448); value = code * s.
 *   NVFP4: g (per-tensor); per 16-element block sb = E4M3(block_absmax /
 *          (6 g)), element code = E2M1(x / (E4M3_value(sb) * g)) (saturating
 *          to +-6; all codes +0 when that divisor is 0);
 *          value = E2M1_value(code) * E4M3_value(sb) * g.
 *   BF16 : scales are ignored and may be NULL.
 *
 * KVQ_FMT_PQ3 ("AMD MI300X - KV Cache Compression Benchmark", "Key Results":
 * 3-bit methods with one 52-byte block per 128-element vector, 4.923x against
 * FP16; PlanarQuant's rotation needs 256 FMAs; the repository generates a
 * Lloyd-Max codebook).  Each 128-element head vector x (one token, one KV
 * head, K or V) is stored as its fp32 L2 norm and 128 3-bit indices:
 *   u = x / |x|; y = R u with R = 64 planar rotations of the coordinate
 *   pairs (2j, 2j+1) by (cos_j, sin_j); index_i = the nearest of 8 codebook
 *   values c_0 < ... < c_7 to y_i; value = |x| * R^T c[index].
 * The encode's fp32 steps are fixed, so indices are exact: sum of squares as
 * a pairwise tree in index order, sqrt and division rounded to nearest,
 * y_2j = fma(cos_j, u_2j, -(sin_j * u_2j+1)), y_2j+1 = fma(sin_j, u_2j,
 * cos_j * u_2j+1), index = the number of thresholds (c_k + c_k+1) / 2 below
 * y; an all-zero x stores norm 0 and indices 0.
 *   Head page (832 bytes): 16 fp32 norms, then 16 rows of 48 bytes.  A row
 *   is 12 little-endian 32-bit words in two bit planes: words 0-7 hold the
 *   low 2 bits of the indices (word w: index 16w + k at bits 4k, 4k+1 and
 *   index 16w + 8 + k at bits 4k+2, 4k+3, k < 8), words 8-11 their high bits
 *   (word 8 + v: bit 2 of index 32v + 8j + k at bit 4k + (2, 3, 0, 1)[j]).
 *   The "scale" of a PQ3 tensor (d_k_scale, d_v_scale) is a device array of
 *   136 fp32: the 8 codebook values (f16-representable, ascending; see
 *   kv_pq3_codebook), then the 64 (cos, sin) pairs.
 *   kv_decode_attention, its window mode, kv_quantize_write, kv_dequantize
 *   and kv_cache_bytes accept PQ3; kv_prefill_attention and
 *   kv_scale_from_absmax(_device) do not (KVQ_ERR_UNSUPPORTED).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVQ_BLOCK_SIZE 16

typedef enum kvq_format {
  KVQ_FMT_BF16 = 0,
  KVQ_FMT_FP8_E4M3 = 1,
  KVQ_FMT_NVFP4 = 2,
  KVQ_FMT_PQ3 = 3 /* 3-bit planar-rotation codec, head_dim 128 only (see below) */
} kvq_format;

typedef enum kvq_status {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1, /* a null pointer, bad size, misaligned buffer */
  KVQ_ERR_UNSUPPORTED = 2, /* not sm_100, unsupported format/head_dim/GQA ratio */
  KVQ_ERR_WORKSPACE = 3,   /* workspace missing or smaller than required */
  KVQ_ERR_CUDA = 4         /* a CUDA runtime call or a launch failed */
} kvq_status;

/* Bits OR-ed into the caller's device error word. */
#define KVQ_DERR_BLOCK_ID 0x1 /* block_table entry outside [0, num_blocks) */
#define KVQ_DERR_SLOT 0x2     /* slot beyond the cache or its sequence */
#define KVQ_DERR_SCALE 0x4    /* scale <= 0 (FP8), < 0 (NVFP4), or not finite */
#define KVQ_DERR_SEQ_LEN 0x8  /* seq_lens[b] < 0 or > max_seq_len */
#define KVQ_DERR_TIMEOUT 0x10 /* a bounded wait on a shared-memory copy expired */

/* A cudaStream_t. */
typedef void* kvq_stream;

/* Description of one layer's paged K/V cache.  k and v are device buffers of
 * kv_cache_bytes() bytes each, 256-byte aligned. */
typedef struct kvq_cache {
  int32_t fmt;          /* kvq_format */
  int32_t block_size;   /* must be KVQ_BLOCK_SIZE */
  int64_t num_blocks;   /* blocks in the pool */
  int32_t num_kv_heads; /* Hkv >= 1 */
  int32_t head_dim;     /* 64 or 128 */
  void* k;
  void* v;
} kvq_cache;

/* Text for a status code (static storage). */
const char* kvq_status_string(kvq_status status);

/* Detail of the last non-OK status returned on the calling thread. */
const char* kvq_last_error(void);

/* Bytes of ONE of the two cache buffers (K or V) for the given geometry:
 * num_blocks * num_kv_heads * head-page bytes, a head page being 32*head_dim
 * bytes (BF16), 16*head_dim (FP8), 9*head_dim (NVFP4) or 832 (PQ3, head_dim
 * 128). */
kvq_status kv_cache_bytes(int32_t fmt, int64_t num_blocks, int32_t num_kv_heads,
                          int32_t head_dim, int64_t* bytes);

/* Host, pure.  The per-layer scale from an abs-max:
 *   FP8  : max(amax * 1.05 / 448, 1e-12), fp32, evaluated left to right
 *          ("FP8 KV calibration guide", Radiance calibrator paragraph);
 *   NVFP4: g = amax / (448 * 6);
 *   BF16 : 1.
 * amax must be finite and >= 0. */
kvq_status kv_scale_from_absmax(int32_t fmt, float amax, float* scale);

/* Host, pure.  The PQ3 codebook: the 8-level Lloyd-Max quantizer of N(0, 1/128)
 * (one coordinate of a random unit vector in 128 dimensions, Gaussian
 * approximation; "AMD MI300X - KV Cache Compression Benchmark", repository
 * structure: Lloyd-Max solver and codebook generator), each value rounded to
 * the nearest f16, written to cb[8] in ascending order.  KVQ_ERR_INVALID_ARG
 * if cb is NULL. */
kvq_status kv_pq3_codebook(float* cb);

/* Device version of kv_scale_from_absmax: reads *d_amax, writes *d_scale
 * (bit-identical to the host function), so calibration, scale and
 * quantize-on-write chain on the stream without a host round trip. */
kvq_status kv_scale_from_absmax_device(int32_t fmt, const float* d_amax, float* d_scale,
                                       kvq_stream stream);

/* Calibration abs-max ("FP8 KV calibration guide": the calibrator observes the
 * BF16 K/V activation maxima).  x: n BF16 values (2-byte aligned, any
 * length).  *d_amax is MAX-ACCUMULATED: max(*d_amax, max |x|); the caller
 * zeroes it once, so several batches (or K and V of several layers, each with
 * its own word) can be observed in turn.  The result is exact (order-free). */
kvq_status kv_calibrate_absmax(const void* x, int64_t n, float* d_amax, kvq_stream stream);

/* Quantize-on-write.  k, v: BF16 [num_tokens][num_kv_heads][head_dim]
 * (16-byte aligned).  Token t goes to the slot named by slot_mapping[t]
 * (int64; negative = skip the token):
 *   block_table == NULL: slot_mapping holds PHYSICAL slots block*16+offset;
 *   block_table != NULL: slot_mapping holds LOGICAL slots seq*(max_blocks*16)
 *     + position, translated in the kernel through block_table
 *     [num_seqs][max_blocks] (int32): block_table[seq][position/16]*16 +
 *     position%16 (the paged scatter a chunked prefill performs).
 * d_k_scale / d_v_scale: device fp32 scalars (FP8: s, NVFP4: g; unused for
 * BF16).  Bad slots or table entries set KVQ_DERR_SLOT / KVQ_DERR_BLOCK_ID and
 * that token is skipped; a bad scale sets KVQ_DERR_SCALE and nothing is
 * written for that tensor. */
kvq_status kv_quantize_write(int32_t fmt, const void* k, const void* v, int64_t num_tokens,
                             const int64_t* slot_mapping, const int32_t* block_table,
                             int32_t num_seqs, int32_t max_blocks, const kvq_cache* cache,
                             const float* d_k_scale, const float* d_v_scale, int32_t* d_err,
                             kvq_stream stream);

/* Workspace bytes kv_decode_attention needs for this problem size (0 when it
 * needs none).  num_splits: 0 = let the library spread the context over the
 * SMs (the usual choice); > 0 cuts every (sequence, KV head) into about that
 * many pieces, each on its own CTA, merged by log-sum-exp.  The same
 * arguments must be given to kv_decode_attention. */
kvq_status kv_decode_workspace_size(int32_t fmt, int32_t num_seqs, int32_t num_q_heads,
                                    int32_t num_kv_heads, int32_t head_dim, int32_t max_seq_len,
                                    int32_t num_splits, size_t* bytes);

/* Decode-step attention over the quantized cache, one query token per
 * sequence, dequantisation fused into the scan.
 *   q          : BF16 [num_seqs][num_q_heads][head_dim], 16-byte aligned.
 *   block_table: int32 [num_seqs][max_blocks]; token t of sequence b is in
 *                block block_table[b][t/16] at offset t%16.
 *   seq_lens   : int32 [num_seqs], each in [0, max_seq_len].
 *   num_q_heads: a multiple of num_kv_heads; query head j reads KV head
 *                j / (num_q_heads / num_kv_heads) (grouped-query attention).
 *   max_seq_len: an upper bound on seq_lens (<= max_blocks * 16); sizes the
 *                context split.
 *   sm_scale   : softmax scale; 0 means 1/sqrt(head_dim).
 *   out        : fp32 [num_seqs][num_q_heads][head_dim] = softmax(s) . V_hat.
 *   lse        : fp32 [num_seqs][num_q_heads] = ln sum_t exp(s_t) of the
 *                scaled scores s_t = sm_scale * q . k_hat_t.  May be NULL.
 *   A sequence of length 0 gives out = 0 and lse = -inf.
 *   workspace  : device scratch of kv_decode_workspace_size() bytes
 *                (256-byte aligned) holding the split partials and one
 *                counter per (sequence, KV head).  It must be zero-filled
 *                before its FIRST use; every call leaves the counters zero
 *                again, so it can be reused without clearing.  Calls that
 *                share a workspace must not overlap on the GPU.
 * Values are fp32-accumulated; results match float64 attention over the same
 * dequantised values to about 1e-4 absolute on out and 1e-6 relative on lse.
 * Stream ordering: the launch allows programmatic dependent launch.  When the
 * previous operation on the stream is a kv_quantize_write, the decode may
 * start its prologue (reading q, block_table, seq_lens and the scales) while
 * that write finishes, and waits for the write's cache stores before reading
 * any cache page; those four inputs must therefore not be produced by that
 * write's kernel (they never are).  After any other operation the launch is
 * an ordinary stream-ordered one.  kv_quantize_write's kernels likewise let
 * a following programmatic-dependent launch begin early: such a kernel must
 * wait on its grid dependency before reading the cache. */
kvq_status kv_decode_attention(int32_t fmt, const void* q, const kvq_cache* cache,
                               const int32_t* block_table, int32_t max_blocks,
                               const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
                               int32_t max_seq_len, int32_t num_splits, const float* d_k_scale,
                               const float* d_v_scale, float sm_scale, float* out, float* lse,
                               void* workspace, size_t workspace_bytes, int32_t* d_err,
                               kvq_stream stream);

/* kv_decode_attention in sliding-window mode ("AMD MI300X — KV Cache
 * Compression Benchmark", section "SWA mode": attention over the most recent
 * `window` tokens of a truncated or windowed cache).  Sequence b attends to
 * its tokens [max(0, seq_lens[b] - window), seq_lens[b]) only; window = 0 is
 * kv_decode_attention itself.  The work is split over the window's pages
 * only, so a short window over a long cache reads ~window tokens per
 * sequence.  Same arguments, layouts and errors as kv_decode_attention;
 * window < 0 is KVQ_ERR_INVALID_ARG.  The workspace must hold
 * kv_decode_workspace_size_window() bytes for the same arguments. */
kvq_status kv_decode_attention_window(int32_t fmt, const void* q, const kvq_cache* cache,
                                      const int32_t* block_table, int32_t max_blocks,
                                      const int32_t* seq_lens, int32_t num_seqs,
                                      int32_t num_q_heads, int32_t max_seq_len, int32_t window,
                                      int32_t num_splits, const float* d_k_scale,
                                      const float* d_v_scale, float sm_scale, float* out,
                                      float* lse, void* workspace, size_t workspace_bytes,
                                      int32_t* d_err, kvq_stream stream);

/* FP8 attention over an FP8 cache: kv_decode_attention with the query and the
 * softmax probabilities in E4M3 too, so both attention products run on E4M3
 * tensor cores ("FP8 KV calibration guide": the calibrator observes the BF16
 * Q, K and V activation maxima and writes per-layer E4M3 scales with the same
 * formula, and other attention paths accept a probability scale, prob_scale).
 *   d_q_scale    : device fp32 scalar, the query's E4M3 scale (the per-layer
 *                  formula of kv_scale_from_absmax on Q's abs-max):
 *                  q_hat = E4M3(q / q_scale) (fp32 division, nearest even,
 *                  saturating).
 *   d_prob_scale : device fp32 scalar, P's E4M3 scale (the same formula at an
 *                  observed maximum of 1 gives 1.05 / 448).
 * P is quantized page by page: within each 16-token cache page the
 * probabilities are taken against the page's largest score (so each page's
 * largest p is 1), P_hat = E4M3(p * fp32(1 / prob_scale)); the page then
 * enters the softmax sums with weight exp(page max - running max), and the
 * normaliser uses the unquantized p.  Results therefore differ from
 * kv_decode_attention by the E4M3 rounding of q and of P (about 2^-4
 * relative per probability); the split over CTAs does not change them.
 * Other arguments, layouts, the workspace (kv_decode_workspace_size with
 * KVQ_FMT_FP8_E4M3 and the same sizes) and the errors are those of
 * kv_decode_attention.  The cache must be FP8 (KVQ_ERR_UNSUPPORTED
 * otherwise); d_q_scale / d_prob_scale NULL is KVQ_ERR_INVALID_ARG, and a
 * non-positive or non-finite value on the device sets KVQ_DERR_SCALE. */
kvq_status kv_decode_attention_fp8qp(const void* q, const kvq_cache* cache,
                                     const int32_t* block_table, int32_t max_blocks,
                                     const int32_t* seq_lens, int32_t num_seqs,
                                     int32_t num_q_heads, int32_t max_seq_len, int32_t num_splits,
                                     const float* d_k_scale, const float* d_v_scale,
                                     const float* d_q_scale, const float* d_prob_scale,
                                     float sm_scale, float* out, float* lse, void* workspace,
                                     size_t workspace_bytes, int32_t* d_err, kvq_stream stream);

/* Workspace bytes kv_decode_attention_window needs (as
 * kv_decode_workspace_size, with the window). */
kvq_status kv_decode_workspace_size_window(int32_t fmt, int32_t num_seqs, int32_t num_q_heads,
                                           int32_t num_kv_heads, int32_t head_dim,
                                           int32_t max_seq_len, int32_t window,
                                           int32_t num_splits, size_t* bytes);

/* Chunked-prefill attention over the paged cache: the attention of a prompt
 * chunk's own tokens, after kv_quantize_write has put them in the cache.
 * Long prompts are fed in chunks of a fixed token budget that attend to the
 * prefix already cached ("Dual R9700 model and spec-decode campaign", fixed
 * knobs: long-prefill-token-threshold 2048 with prefix caching; "FP8 KV
 * calibration guide", first paragraph: TTFT at ~126k context with FP8 KV).
 *   q          [num_seqs][num_q_tokens][num_q_heads][head_dim] BF16: the
 *              num_q_tokens newest tokens of each sequence.  Device, 16-byte
 *              aligned.
 *   seq_lens   [num_seqs] int32: cached tokens of each sequence, the chunk
 *              included.  Query i of sequence b sits at position
 *              p = seq_lens[b] - num_q_tokens + i and attends to the cache
 *              tokens [0, p] (causal, itself included); a query with p < 0
 *              attends to nothing (out = 0, lse = -inf).
 *   block_table, max_blocks, cache, d_k_scale, d_v_scale, sm_scale: as for
 *              kv_decode_attention (GQA: query head j reads KV head
 *              j / (num_q_heads / num_kv_heads)).
 *   out        [num_seqs][num_q_tokens][num_q_heads][head_dim] fp32, 16-byte
 *              aligned; lse [num_seqs][num_q_tokens][num_q_heads] fp32 (natural
 *              log of the scaled scores) or NULL.
 * Scores, softmax and dequantisation are those of kv_decode_attention; the
 * result matches float64 attention over the dequantised cache within the same
 * tolerances.  No workspace.  num_q_heads / num_kv_heads must be at most 128
 * (KVQ_ERR_UNSUPPORTED otherwise).  Device-side problems set d_err bits as in
 * kv_decode_attention: a bad block id (its page's keys are skipped), a
 * seq_lens entry outside [0, max_blocks * 16] (that sequence's outputs are
 * empty), a bad scale (all outputs empty).  Asynchronous on `stream`;
 * ordinary stream ordering (no early start behind a write). */
kvq_status kv_prefill_attention(int32_t fmt, const void* q, const kvq_cache* cache,
                                const int32_t* block_table, int32_t max_blocks,
                                const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_tokens,
                                int32_t num_q_heads, const float* d_k_scale,
                                const float* d_v_scale, float sm_scale, float* out, float* lse,
                                int32_t* d_err, kvq_stream stream);

/* Self-test of the bounded wait behind every mbarrier wait in the library's
 * kernels (no attention computed).  One warp waits on an mbarrier phase:
 * with arrive != 0 the phase is completed first and the wait succeeds; with
 * arrive = 0 nothing completes it, the wait gives up after about two seconds
 * and KVQ_DERR_TIMEOUT is set in *d_err (device int32, caller-zeroed).  The
 * context stays usable either way.  KVQ_ERR_INVALID_ARG if d_err is NULL.
 * Asynchronous on `stream`. */
kvq_status kvq_selftest_bounded_wait(int32_t* d_err, int32_t arrive, kvq_stream stream);

/* kv_decode_attention without a caller workspace, for callers that cannot
 * allocate device memory when they run a decode step (their device memory
 * belongs to a fixed pool they must not bypass, they may not pay a
 * cudaMalloc's latency and implicit synchronisation there, or their host
 * hands them no scratch).  The pages' method has no counterpart of this call;
 * it only changes where the scratch lives.
 *   - Arguments and results are those of kv_decode_attention, minus the
 *     workspace.  The call allocates nothing (no cudaMalloc, cudaFree or
 *     allocating library routine).
 *   - The scratch is one 8 MiB device array inside the library, held by every
 *     GPU that loads the library until the process exits.  A problem whose
 *     kv_decode_workspace_size exceeds 8 MiB returns KVQ_ERR_WORKSPACE and
 *     launches nothing.
 *   - The first call on a device looks the array's device address up (once,
 *     with that device current); make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one array and clears the part it
 *     uses before launching (an extra memset on the stream).  Calls that
 *     overlap on the GPU (different streams, no ordering between them) race
 *     on the array and give wrong results; order them on one stream. */
kvq_status kv_decode_attention_static_ws(int32_t fmt, const void* q, const kvq_cache* cache,
                                         const int32_t* block_table, int32_t max_blocks,
                                         const int32_t* seq_lens, int32_t num_seqs,
                                         int32_t num_q_heads, int32_t max_seq_len,
                                         int32_t num_splits, const float* d_k_scale,
                                         const float* d_v_scale, float sm_scale, float* out,
                                         float* lse, int32_t* d_err, kvq_stream stream);

/* Dequantise the cache at the listed PHYSICAL slots (int64 [n]) into fp32
 * k_out, v_out [n][num_kv_heads][head_dim] (for checking; not on the decode
 * path).  Slots outside the cache set KVQ_DERR_SLOT and their rows are left
 * untouched. */
kvq_status kv_dequantize(int32_t fmt, const kvq_cache* cache, const int64_t* slots, int64_t n,
                         const float* d_k_scale, const float* d_v_scale, float* k_out,
                         float* v_out, int32_t* d_err, kvq_stream stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
