// kvq_decode_static.cu — decode attention for callers that cannot allocate device memory.
//
// kvq_decode_attention needs a caller-provided workspace for its split-K partial
// results and arrival counters.  Some callers have no way to provide one: a serving
// engine whose memory pool has already claimed all device memory, a plugin running
// inside a host framework that owns every allocation, or a latency-critical path that
// must not call cudaMalloc (which can synchronize the device).  For them this file
// keeps one fixed scratch buffer in the library itself, as a file-scope __device__
// array that every GPU loading the library holds until the process exits.
//
// Host code never names the array's address directly (its host-side name is only a
// stand-in); the device address is looked up with cudaGetSymbolAddress once per
// device, with that device current, and passed to the kernel as an ordinary pointer.
#include <mutex>

#include "kvq_internal.cuh"

namespace {

constexpr size_t kScratchBytes = KVQ_STATIC_SCRATCH_BYTES;

__device__ __align__(256) uint8_t g_decode_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[64];  // device address of g_decode_scratch, per device ordinal

kvq_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return KVQ_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return KVQ_ERR_CUDA;
    }
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_static(const kvq_config* cfg, const void* pool, int64_t pool_pages,
                                                  const void* q, int32_t batch, const int32_t* page_table,
                                                  int32_t max_pages, const int32_t* num_pages, const void* res_k,
                                                  const void* res_v, const int32_t* res_len, float sm_scale,
                                                  float* out, int32_t* err, cudaStream_t stream) {
  // every argument is checked before the scratch is touched or anything is enqueued
  const kvq_status s = kvq::decode_check_args(cfg, pool, pool_pages, q, batch, page_table, max_pages, num_pages,
                                              res_k, res_v, res_len, out);
  if (s != KVQ_OK) return s;
  void* scratch = nullptr;
  if (batch == 0) {
    // nothing to compute: only look the scratch up, so that a caller can resolve it
    // (and, with lazy module loading, have the module loaded) before its own memory
    // pool claims the device and before any stream capture
    return scratch_address(&scratch);
  }
  const size_t need = kvq_decode_workspace_bytes(cfg, batch, max_pages);
  if (need == 0 || need > kScratchBytes) return KVQ_ERR_CAPACITY;
  const kvq_status a = scratch_address(&scratch);
  if (a != KVQ_OK) return a;
  // The scratch keeps whatever the previous call left.  The arrival counters (the
  // last batch * num_kv_heads 32-bit words of the used region) must start at zero;
  // a completed call leaves them at zero, an interrupted one may not, so clear them.
  const size_t cnt_bytes = size_t(batch) * size_t(cfg->num_kv_heads) * sizeof(uint32_t);
  if (cudaMemsetAsync(static_cast<uint8_t*>(scratch) + (need - cnt_bytes), 0, cnt_bytes, stream) != cudaSuccess)
    return KVQ_ERR_CUDA;
  return kvq_decode_attention(cfg, pool, pool_pages, q, batch, page_table, max_pages, num_pages, res_k, res_v,
                              res_len, sm_scale, out, scratch, kScratchBytes, err, stream);
}
