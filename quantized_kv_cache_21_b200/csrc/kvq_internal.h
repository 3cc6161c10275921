// kvq_internal.h -- launch interfaces shared by the C-ABI layer and the
// kernel translation units (host side only).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <atomic>

namespace kvq {

struct DecodeParams {
  const uint16_t* q;          // [B][Hq][D] bf16
  const int32_t* block_table; // [B][max_blocks]
  const int32_t* seq_lens;    // [B]
  const float* k_scale;       // device scalar (FP8: s, NVFP4: g; PQ3: 136-float parameter block)
  const float* v_scale;
  const uint8_t* kc;          // cache buffers (PQ3 pages are fetched by address)
  const uint8_t* vc;
  const float* q_scale;       // FP8 attention only: device scalar, E4M3 scale of q
  const float* prob_scale;    // FP8 attention only: device scalar, E4M3 scale of P
  float* out;                 // [B][Hq][D]
  float* lse;                 // [B][Hq] or null
  float* ws_part;             // [units + ctas][16 + 8 D] per-CTA partials (slot u + cta)
  unsigned* ws_cnt;           // [units] arrival counters (zero between launches)
  int* d_err;
  int64_t num_blocks;
  int max_blocks;
  int B, Hq, Hkv, G, n_groups;
  int units;                  // B * Hkv * n_groups (sequence, KV head, group of 8 q heads)
  int pmax;                   // pages per unit in the work partition: ceil(max_seq_len / 16),
                              // plus merge_pages of empty padding when units straddle CTAs
  int max_seq_len;
  int window;                 // > 0: attend to each sequence's last `window` tokens only
  float sm_scale;
};

struct DecodeConfig {
  int warps;        // warps per CTA
  int stages;       // shared-memory ring stages per CTA
  int stage_bytes;  // bytes per stage
  size_t smem_bytes;
  int part_floats;  // floats of one (m, l, o) partial for 8 heads
  int merge_pages;  // pages a CTA scans in about the time a unit boundary inside
                    // its range costs it (the segment merge, the next unit's start)
};

// Per-(format, head_dim) kernel configuration; false if unsupported.
bool decode_config(int fmt, int D, DecodeConfig* cfg);
// Launch the decode kernel on `ctas` persistent CTAs.  fp8_qp: the FP8
// attention variant (FP8 cache only; E4M3 Q and P on E4M3 tensor-core MMAs).
cudaError_t launch_decode(int fmt, int D, const CUtensorMap* maps, const DecodeParams& p,
                          int ctas, cudaStream_t stream, bool fp8_qp = false);

struct PrefillParams {
  const uint16_t* q;          // [B][Tq][Hq][D] bf16: the Tq newest tokens of each sequence
  const int32_t* block_table; // [B][max_blocks]
  const int32_t* seq_lens;    // [B], cached tokens including the chunk
  const uint8_t* kc;          // cache pages [num_blocks][Hkv][head page]
  const uint8_t* vc;
  const float* k_scale;       // device scalar (FP8: s, NVFP4: g); unused for BF16
  const float* v_scale;
  float* out;                 // [B][Tq][Hq][D]
  float* lse;                 // [B][Tq][Hq] or null
  int* d_err;
  int64_t num_blocks;
  int max_blocks;
  int B, Tq, Hq, Hkv, G;
  int QT;                     // query tokens per CTA (rows per CTA / G)
  int n_qblk;                 // ceil(Tq / QT)
  float sm_scale;
};

// Rows ((query token, query head) pairs of one KV head) per prefill CTA.
int prefill_rows();
cudaError_t launch_prefill(int fmt, int D, const PrefillParams& p, int64_t ctas,
                           cudaStream_t stream);

struct QuantParams {
  const uint16_t* k;
  const uint16_t* v;
  int64_t T;
  int H, D;
  const int64_t* slot_mapping;
  const int32_t* block_table;  // null: physical slots
  int num_seqs, max_blocks;
  int64_t num_blocks;
  uint8_t* kc;
  uint8_t* vc;
  const float* k_scale;
  const float* v_scale;
  int* d_err;
};
cudaError_t launch_quantize(int fmt, const QuantParams& p, cudaStream_t stream);

cudaError_t launch_dequantize(int fmt, const uint8_t* kc, const uint8_t* vc, int64_t num_blocks,
                              int H, int D, const int64_t* slots, int64_t n, const float* ks,
                              const float* vs, float* ko, float* vo, int* d_err,
                              cudaStream_t stream);

cudaError_t launch_absmax(const uint16_t* x, int64_t n, float* d_amax, cudaStream_t stream);
cudaError_t launch_scale(int fmt, const float* d_amax, float* d_scale, cudaStream_t stream);

int num_sms();

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device: `done` is the kernel's own per-device-ordinal flag
// array (kMaxDevices entries, zero-initialised).  The attribute belongs to the
// device's context, so a kernel launched on a second GPU sets it there again;
// concurrent first calls may both set it, which is harmless.
constexpr int kMaxDevices = 64;
cudaError_t ensure_smem_attr(const void* func, size_t bytes, std::atomic<bool>* done);
// Sets the text kvq_last_error() returns on this thread.
void set_last_error(const char* msg);

}  // namespace kvq
