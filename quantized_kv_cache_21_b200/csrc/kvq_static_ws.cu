// kvq_static_ws.cu -- decode attention without caller-provided workspace.
//
// kv_decode_attention needs a scratch workspace for its split merges, which
// the caller normally allocates.  Some callers cannot allocate device memory
// at the point where they run a decode step: a runtime whose device memory is
// owned by a fixed-size pool it must not bypass, a code path that may not
// pay the synchronisation and latency a cudaMalloc can bring, or a plugin
// host that hands out no scratch.  For them this file keeps one fixed-size
// scratch array in the library itself (a file-scope __device__ array, so
// every GPU that loads the library holds it until the process exits) and
// offers kv_decode_attention_static_ws, which allocates nothing.
#include <stdio.h>

#include <mutex>

#include "kvq.h"
#include "kvq_internal.h"

namespace {

// Largest workspace the static entry point serves (8 MiB per GPU).  That
// covers up to about 1,800 (sequence, KV head) units at head_dim 128.
constexpr size_t kStaticScratchBytes = size_t(8) << 20;

static __device__ __align__(256) unsigned char g_kvq_scratch[kStaticScratchBytes];

// Device address of g_kvq_scratch per device ordinal, looked up once with
// that device current (in host code the array's name is only a stand-in,
// never a device address).
constexpr int kMaxDevices = 64;
void* g_scratch_ptr[kMaxDevices] = {};
std::mutex g_scratch_mu;

kvq_status scratch_for_current_device(void** out) {
  char msg[160];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "cudaGetDevice: %s", cudaGetErrorString(e));
    kvq::set_last_error(msg);
    return KVQ_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    snprintf(msg, sizeof(msg), "device ordinal %d out of range", dev);
    kvq::set_last_error(msg);
    return KVQ_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_kvq_scratch);
    if (e != cudaSuccess || !p) {
      snprintf(msg, sizeof(msg), "cudaGetSymbolAddress: %s", cudaGetErrorString(e));
      kvq::set_last_error(msg);
      return KVQ_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kv_decode_attention_static_ws(
    int32_t fmt, const void* q, const kvq_cache* cache, const int32_t* block_table,
    int32_t max_blocks, const int32_t* seq_lens, int32_t num_seqs, int32_t num_q_heads,
    int32_t max_seq_len, int32_t num_splits, const float* d_k_scale, const float* d_v_scale,
    float sm_scale, float* out, float* lse, int32_t* d_err, kvq_stream stream) {
  if (!cache) {
    kvq::set_last_error("cache is NULL");
    return KVQ_ERR_INVALID_ARG;
  }
  size_t need = 0;
  kvq_status s = kv_decode_workspace_size(fmt, num_seqs, num_q_heads, cache->num_kv_heads,
                                          cache->head_dim, max_seq_len, num_splits, &need);
  if (s != KVQ_OK) return s;
  if (need > kStaticScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof(msg),
             "problem needs %zu bytes of workspace; the built-in scratch holds %zu (use "
             "kv_decode_attention with a caller workspace)",
             need, kStaticScratchBytes);
    kvq::set_last_error(msg);
    return KVQ_ERR_WORKSPACE;
  }
  void* scratch = nullptr;
  if (need > 0) {
    s = scratch_for_current_device(&scratch);
    if (s != KVQ_OK) return s;
    // The arrival counters in the workspace must start at zero; a call that
    // ended early could have left them otherwise, so clear the used part.
    cudaError_t e = cudaMemsetAsync(scratch, 0, need, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) {
      kvq::set_last_error(cudaGetErrorString(e));
      return KVQ_ERR_CUDA;
    }
  }
  return kv_decode_attention(fmt, q, cache, block_table, max_blocks, seq_lens, num_seqs,
                             num_q_heads, max_seq_len, num_splits, d_k_scale, d_v_scale, sm_scale,
                             out, lse, scratch, need, d_err, stream);
}
