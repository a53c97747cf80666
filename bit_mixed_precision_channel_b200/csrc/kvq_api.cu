// kvq_api.cu — the C ABI of include/kvq.h: host-side argument checks and launches.
#include <algorithm>
#include <cstdint>

#include "kvq_internal.cuh"

namespace kvq {

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// SM count of the current device, looked up once per device (148 when no device is
// visible, so that workspace sizes can be computed on a machine without a GPU).
static int sm_count() {
  static int cached[64];
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return 148;
  }
  n = __atomic_load_n(&cached[dev], __ATOMIC_ACQUIRE);
  if (n > 0) return n;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 148;
  }
  __atomic_store_n(&cached[dev], n, __ATOMIC_RELEASE);
  return n;
}

// Decode workspace: one partial slot per (CTA, unit) pair that can occur — CTA i and
// unit u write slot i + u — then one arrival counter per unit.
struct Plan {
  int ctas;
  size_t part_bytes, cnt_bytes;
};

static Plan decode_plan(const kvq_config* cfg, int batch) {
  const int gqa = cfg->num_q_heads / cfg->num_kv_heads;
  const size_t units = size_t(batch) * cfg->num_kv_heads;
  Plan pl;
  pl.ctas = sm_count() * decode_ctas_per_sm(gqa, cfg->dtype, cfg->num_boost / 16, cfg->page_tokens);
  pl.part_bytes = (size_t(pl.ctas) + units) * gqa * (kHeadDim + 4) * sizeof(float);
  pl.part_bytes = (pl.part_bytes + 255) / 256 * 256;
  pl.cnt_bytes = units * sizeof(uint32_t);
  return pl;
}

// Every host-side check of a decode call except the workspace (shared by the
// workspace and static-scratch entry points, so both reject the same calls before
// enqueuing anything).
kvq_status decode_check_args(const kvq_config* cfg, const void* pool, int64_t pool_pages, const void* q,
                             int32_t batch, const int32_t* page_table, int32_t max_pages, const int32_t* num_pages,
                             const void* res_k, const void* res_v, const int32_t* res_len, const float* out) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (batch < 0 || max_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!pool || pool_pages <= 0 || !q || !num_pages || !res_k || !res_v || !res_len || !out) return KVQ_ERR_INVALID_ARG;
  if (max_pages > 0 && !page_table) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(pool) || !aligned16(q) || !aligned16(res_k) || !aligned16(res_v)) return KVQ_ERR_INVALID_ARG;
  // the kernel's work line (32-token groups, weighted 16-token residual pieces and a
  // merge weight per (sequence, kv head)) is indexed with 32-bit integers
  const long long line = (long long)batch * cfg->num_kv_heads *
                         ((long long)max_pages * (cfg->page_tokens / 32) +
                          (long long)kDecodePieceWeight * ((cfg->page_tokens + 15) / 16) + kDecodeMergeWeight);
  if (line >= (1ll << 31)) return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

}  // namespace kvq

using namespace kvq;

static kvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument (null pointer, inconsistent sizes or misaligned buffer)";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration (shape or precision without a kernel)";
    case KVQ_ERR_CUDA: return "CUDA runtime error";
    case KVQ_ERR_CAPACITY: return "workspace too small";
  }
  return "unknown status";
}

kvq_status kvq_check_config(const kvq_config* cfg) {
  if (!cfg) return KVQ_ERR_INVALID_ARG;
  if (cfg->head_dim <= 0 || cfg->num_q_heads <= 0 || cfg->num_kv_heads <= 0 || cfg->page_tokens <= 0 ||
      cfg->key_group <= 0 || cfg->num_boost < 0)
    return KVQ_ERR_INVALID_ARG;
  if (cfg->num_q_heads % cfg->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  if (cfg->page_tokens % cfg->key_group != 0) return KVQ_ERR_INVALID_ARG;
  if (cfg->num_boost > cfg->head_dim || cfg->num_boost % 16 != 0) return KVQ_ERR_INVALID_ARG;
  const int gqa = cfg->num_q_heads / cfg->num_kv_heads;
  if (cfg->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (gqa != 1 && gqa != 2 && gqa != 4 && gqa != 8) return KVQ_ERR_UNSUPPORTED;
  if (cfg->page_tokens != 32 && cfg->page_tokens != 64 && cfg->page_tokens != 128) return KVQ_ERR_UNSUPPORTED;
  if (cfg->key_group != 32) return KVQ_ERR_UNSUPPORTED;
  if (cfg->key_bits != 2 || cfg->boost_bits != 4 || cfg->value_bits != 2) return KVQ_ERR_UNSUPPORTED;
  if (cfg->num_boost != 0 && cfg->num_boost != 16 && cfg->num_boost != 32 && cfg->num_boost != 64 &&
      cfg->num_boost != 128)
    return KVQ_ERR_UNSUPPORTED;
  if (cfg->dtype != KVQ_F16 && cfg->dtype != KVQ_BF16) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

kvq_status kvq_page_layout(const kvq_config* cfg, kvq_layout* out) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (!out) return KVQ_ERR_INVALID_ARG;
  const Layout L = make_layout(cfg->page_tokens, cfg->head_dim, cfg->num_boost, cfg->key_group);
  out->k_codes = L.k_codes;
  out->kb_codes = L.kb_codes;
  out->v_codes = L.v_codes;
  out->k_scale = L.k_scale;
  out->k_zero = L.k_zero;
  out->kb_scale = L.kb_scale;
  out->v_scale = L.v_scale;
  out->v_zero = L.v_zero;
  out->boost_idx = L.boost_idx;
  out->payload_bytes = L.payload;
  out->record_bytes = L.record;
  return KVQ_OK;
}

size_t kvq_page_bytes(const kvq_config* cfg) {
  if (kvq_check_config(cfg) != KVQ_OK) return 0;
  return make_layout(cfg->page_tokens, cfg->head_dim, cfg->num_boost, cfg->key_group).record;
}

static kvq_status quantize_common(const kvq_config* cfg, kvq_source k, kvq_source v, int mode,
                                  const int32_t* dst_pages, int32_t n_pages, void* pool, int64_t pool_pages,
                                  int32_t* err, cudaStream_t stream, const kvq_boost_options* opts = nullptr) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (n_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (n_pages == 0) return KVQ_OK;
  if (!dst_pages || !pool || pool_pages <= 0 || !aligned16(pool)) return KVQ_ERR_INVALID_ARG;
  auto bad_src = [](const kvq_source& x) {
    return !x.src || !aligned16(x.src) || x.page_stride % 8 || x.token_stride % 8 || x.head_stride % 8 ||
           x.page_stride < 0 || x.token_stride < 0 || x.head_stride < 0;
  };
  if ((mode & (kModeSelect | kModeKeys)) && bad_src(k)) return KVQ_ERR_INVALID_ARG;
  if ((mode & kModeValues) && bad_src(v)) return KVQ_ERR_INVALID_ARG;
  QuantParams p{};
  p.k_src = static_cast<const uint16_t*>(k.src);
  p.v_src = static_cast<const uint16_t*>(v.src);
  p.k_page_stride = k.page_stride;
  p.k_tok_stride = k.token_stride;
  p.k_head_stride = k.head_stride;
  p.v_page_stride = v.page_stride;
  p.v_tok_stride = v.token_stride;
  p.v_head_stride = v.head_stride;
  p.dst_pages = dst_pages;
  p.pool = static_cast<uint8_t*>(pool);
  p.pool_pages = pool_pages;
  p.Hkv = cfg->num_kv_heads;
  p.P = cfg->page_tokens;
  p.k = cfg->num_boost;
  p.L = make_layout(cfg->page_tokens, cfg->head_dim, cfg->num_boost, cfg->key_group);
  p.err = err;
  p.mode = mode;
  p.flush = 0;
  if (opts) {
    p.qw = opts->query_weight;
    p.kh = opts->boost_per_head;
  }
  return cuda_status(launch_quantize(p, n_pages, cfg->dtype, stream));
}

kvq_status kvq_quantize_pages_ex(const kvq_config* cfg, kvq_source k, kvq_source v, const int32_t* dst_pages,
                                 int32_t n_pages, void* pool, int64_t pool_pages, const kvq_boost_options* opts,
                                 int32_t* err, cudaStream_t stream) {
  return quantize_common(cfg, k, v, kModeSelect | kModeKeys | kModeValues, dst_pages, n_pages, pool, pool_pages,
                         err, stream, opts);
}

kvq_status kvq_select_boost_channels(const kvq_config* cfg, kvq_source k, const int32_t* dst_pages,
                                     int32_t n_pages, void* pool, int64_t pool_pages, int32_t* err,
                                     cudaStream_t stream) {
  return quantize_common(cfg, k, kvq_source{}, kModeSelect, dst_pages, n_pages, pool, pool_pages, err, stream);
}

kvq_status kvq_quantize_page_keys(const kvq_config* cfg, kvq_source k, const int32_t* dst_pages, int32_t n_pages,
                                  void* pool, int64_t pool_pages, int32_t* err, cudaStream_t stream) {
  return quantize_common(cfg, k, kvq_source{}, kModeKeys, dst_pages, n_pages, pool, pool_pages, err, stream);
}

kvq_status kvq_quantize_values(const kvq_config* cfg, kvq_source v, const int32_t* dst_pages, int32_t n_pages,
                               void* pool, int64_t pool_pages, int32_t* err, cudaStream_t stream) {
  return quantize_common(cfg, kvq_source{}, v, kModeValues, dst_pages, n_pages, pool, pool_pages, err, stream);
}

kvq_status kvq_quantize_pages(const kvq_config* cfg, kvq_source k, kvq_source v, const int32_t* dst_pages,
                              int32_t n_pages, void* pool, int64_t pool_pages, int32_t* err, cudaStream_t stream) {
  return quantize_common(cfg, k, v, kModeSelect | kModeKeys | kModeValues, dst_pages, n_pages, pool, pool_pages,
                         err, stream);
}

kvq_status kvq_append_token(const kvq_config* cfg, int32_t batch, const void* k_new, const void* v_new,
                            void* res_k, void* res_v, int32_t* res_len, int32_t* err, cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (batch < 0) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!k_new || !v_new || !res_k || !res_v || !res_len) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(res_k) || !aligned16(res_v)) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_append(k_new, v_new, res_k, res_v, res_len, batch, cfg->num_kv_heads,
                                   cfg->page_tokens, err, stream));
}

kvq_status kvq_flush_residual_ex(const kvq_config* cfg, int32_t batch, const void* res_k, const void* res_v,
                                 int32_t* res_len, const int32_t* new_page, int32_t* page_table, int32_t max_pages,
                                 int32_t* num_pages, void* pool, int64_t pool_pages, const kvq_boost_options* opts,
                                 int32_t* err, cudaStream_t stream);

kvq_status kvq_flush_residual(const kvq_config* cfg, int32_t batch, const void* res_k, const void* res_v,
                              int32_t* res_len, const int32_t* new_page, int32_t* page_table, int32_t max_pages,
                              int32_t* num_pages, void* pool, int64_t pool_pages, int32_t* err,
                              cudaStream_t stream) {
  return kvq_flush_residual_ex(cfg, batch, res_k, res_v, res_len, new_page, page_table, max_pages, num_pages, pool,
                               pool_pages, nullptr, err, stream);
}

kvq_status kvq_append_flush(const kvq_config* cfg, int32_t batch, const void* k_new, const void* v_new, void* res_k,
                            void* res_v, int32_t* res_len, const int32_t* new_page, int32_t* page_table,
                            int32_t max_pages, int32_t* num_pages, void* pool, int64_t pool_pages,
                            const kvq_boost_options* opts, int32_t* counters, int32_t* err, cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (batch < 0 || max_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!k_new || !v_new || !res_k || !res_v || !res_len || !new_page || !page_table || !num_pages || !pool ||
      pool_pages <= 0 || !counters)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(res_k) || !aligned16(res_v) || !aligned16(pool))
    return KVQ_ERR_INVALID_ARG;
  const int P = cfg->page_tokens, Hkv = cfg->num_kv_heads, D = cfg->head_dim;
  QuantParams p{};
  p.k_src = static_cast<const uint16_t*>(res_k);
  p.v_src = static_cast<const uint16_t*>(res_v);
  p.k_page_stride = p.v_page_stride = (long long)Hkv * P * D;
  p.k_tok_stride = p.v_tok_stride = D;
  p.k_head_stride = p.v_head_stride = (long long)P * D;
  p.dst_pages = new_page;
  p.pool = static_cast<uint8_t*>(pool);
  p.pool_pages = pool_pages;
  p.Hkv = Hkv;
  p.P = P;
  p.k = cfg->num_boost;
  p.L = make_layout(P, D, cfg->num_boost, cfg->key_group);
  p.err = err;
  p.mode = kModeSelect | kModeKeys | kModeValues;
  p.max_pages = max_pages;
  if (opts) {
    p.qw = opts->query_weight;
    p.kh = opts->boost_per_head;
  }
  p.append = 1;
  p.k_new = static_cast<const uint16_t*>(k_new);
  p.v_new = static_cast<const uint16_t*>(v_new);
  p.res_k = static_cast<uint16_t*>(res_k);
  p.res_v = static_cast<uint16_t*>(res_v);
  p.res_len_w = res_len;
  p.num_pages_w = num_pages;
  p.page_table = page_table;
  p.counters = counters;
  return cuda_status(launch_quantize(p, batch, cfg->dtype, stream));
}

kvq_status kvq_flush_residual_ex(const kvq_config* cfg, int32_t batch, const void* res_k, const void* res_v,
                                 int32_t* res_len, const int32_t* new_page, int32_t* page_table, int32_t max_pages,
                                 int32_t* num_pages, void* pool, int64_t pool_pages, const kvq_boost_options* opts,
                                 int32_t* err, cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (batch < 0 || max_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!res_k || !res_v || !res_len || !new_page || !page_table || !num_pages || !pool || pool_pages <= 0)
    return KVQ_ERR_INVALID_ARG;
  if (!aligned16(res_k) || !aligned16(res_v) || !aligned16(pool)) return KVQ_ERR_INVALID_ARG;
  const int P = cfg->page_tokens, Hkv = cfg->num_kv_heads, D = cfg->head_dim;
  QuantParams p{};
  p.k_src = static_cast<const uint16_t*>(res_k);
  p.v_src = static_cast<const uint16_t*>(res_v);
  p.k_page_stride = p.v_page_stride = (long long)Hkv * P * D;
  p.k_tok_stride = p.v_tok_stride = D;
  p.k_head_stride = p.v_head_stride = (long long)P * D;
  p.dst_pages = new_page;
  p.pool = static_cast<uint8_t*>(pool);
  p.pool_pages = pool_pages;
  p.Hkv = Hkv;
  p.P = P;
  p.k = cfg->num_boost;
  p.L = make_layout(P, D, cfg->num_boost, cfg->key_group);
  p.err = err;
  p.mode = kModeSelect | kModeKeys | kModeValues;
  p.flush = 1;
  p.res_len = res_len;
  p.num_pages = num_pages;
  p.max_pages = max_pages;
  if (opts) {
    p.qw = opts->query_weight;
    p.kh = opts->boost_per_head;
  }
  cudaError_t e = launch_quantize(p, batch, cfg->dtype, stream);
  if (e != cudaSuccess) return KVQ_ERR_CUDA;
  return cuda_status(launch_flush_commit(res_len, new_page, page_table, max_pages, num_pages, pool_pages, batch, P,
                                         stream));
}

size_t kvq_decode_workspace_bytes(const kvq_config* cfg, int32_t batch, int32_t max_pages) {
  if (kvq_check_config(cfg) != KVQ_OK || batch < 0 || max_pages < 0) return 0;
  const Plan pl = decode_plan(cfg, batch);
  return pl.part_bytes + pl.cnt_bytes;
}

kvq_status kvq_decode_attention(const kvq_config* cfg, const void* pool, int64_t pool_pages, const void* q,
                                int32_t batch, const int32_t* page_table, int32_t max_pages,
                                const int32_t* num_pages, const void* res_k, const void* res_v,
                                const int32_t* res_len, float sm_scale, float* out, void* workspace,
                                size_t workspace_bytes, int32_t* err, cudaStream_t stream) {
  const kvq_status s = decode_check_args(cfg, pool, pool_pages, q, batch, page_table, max_pages, num_pages, res_k,
                                         res_v, res_len, out);
  if (s != KVQ_OK) return s;
  if (batch == 0) return KVQ_OK;
  if (!workspace || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
  const Plan pl = decode_plan(cfg, batch);
  if (workspace_bytes < pl.part_bytes + pl.cnt_bytes) return KVQ_ERR_CAPACITY;
  const int gqa = cfg->num_q_heads / cfg->num_kv_heads;
  DecodeParams p{};
  p.pool = static_cast<const uint8_t*>(pool);
  p.pool_pages = pool_pages;
  p.Hkv = cfg->num_kv_heads;
  p.P = cfg->page_tokens;
  p.k = cfg->num_boost;
  p.KB = cfg->num_boost / 16;
  p.L = make_layout(cfg->page_tokens, cfg->head_dim, cfg->num_boost, cfg->key_group);
  p.q = static_cast<const uint16_t*>(q);
  p.batch = batch;
  p.Hq = cfg->num_q_heads;
  p.page_table = page_table;
  p.max_pages = max_pages;
  p.num_pages = num_pages;
  p.res_k = static_cast<const uint16_t*>(res_k);
  p.res_v = static_cast<const uint16_t*>(res_v);
  p.res_len = res_len;
  p.c_log2 = sm_scale * 1.4426950408889634f;
  p.out = out;
  p.part = static_cast<float*>(workspace);
  p.cnt = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + pl.part_bytes);
  p.n_ctas = pl.ctas;
  p.n_sms = sm_count();
  p.err = err;
  return cuda_status(launch_decode(p, gqa, cfg->dtype, stream));
}

size_t kvq_prefill_workspace_bytes(const kvq_config* cfg, int32_t L) {
  if (kvq_check_config(cfg) != KVQ_OK || L < 0) return 0;
  return (2 * size_t(cfg->num_q_heads) * size_t(L) * sizeof(float) + 255) / 256 * 256;
}

kvq_status kvq_prefill_attention(const kvq_config* cfg, const void* q, const void* k, const void* v, int32_t L,
                                 float sm_scale, float* out, float* scores, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (L < 0) return KVQ_ERR_INVALID_ARG;
  if (L == 0) return KVQ_OK;
  if (!q || !k || !v || !out || !scores || !workspace) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(workspace))
    return KVQ_ERR_INVALID_ARG;
  if (workspace_bytes < kvq_prefill_workspace_bytes(cfg, L)) return KVQ_ERR_CAPACITY;
  return cuda_status(launch_prefill(q, k, v, L, cfg->num_q_heads, cfg->num_kv_heads, sm_scale, cfg->dtype, out,
                                    static_cast<float*>(workspace), scores, stream));
}

kvq_status kvq_retain_tokens(const kvq_config* cfg, const float* scores, int32_t L, int32_t n_heavy, int32_t n_recent,
                             int32_t* keep, int32_t* n_keep, cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (L < 0 || n_heavy < 0 || n_recent < 0) return KVQ_ERR_INVALID_ARG;
  if (L == 0) return KVQ_OK;
  if (!scores || !keep || !n_keep) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_retain(scores, L, cfg->num_kv_heads, n_heavy, n_recent, keep, n_keep, stream));
}

kvq_status kvq_gather_tokens(const kvq_config* cfg, const void* k, const void* v, int32_t L, const int32_t* keep,
                             int32_t n, void* k_out, void* v_out, int32_t* err, cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (L < 0 || n < 0 || n > L) return KVQ_ERR_INVALID_ARG;
  if (n == 0) return KVQ_OK;
  if (!k || !v || !keep || !k_out || !v_out) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_out) || !aligned16(v_out)) return KVQ_ERR_INVALID_ARG;
  return cuda_status(launch_gather(k, v, cfg->num_kv_heads, L, keep, n, k_out, v_out, err, stream));
}

size_t kvq_dense_page_bytes(const kvq_config* cfg) {
  if (kvq_check_config(cfg) != KVQ_OK) return 0;
  return size_t(2) * cfg->page_tokens * cfg->head_dim * 2;
}

kvq_status kvq_decode_attention_dense(const kvq_config* cfg, const void* pool, int64_t pool_pages, const void* q,
                                      int32_t batch, const int32_t* page_table, int32_t max_pages,
                                      const int32_t* seq_len, float sm_scale, float* out, void* workspace,
                                      size_t workspace_bytes, int32_t* err, cudaStream_t stream) {
  const kvq_status s = kvq_check_config(cfg);
  if (s != KVQ_OK) return s;
  if (batch < 0 || max_pages < 0) return KVQ_ERR_INVALID_ARG;
  if (batch == 0) return KVQ_OK;
  if (!pool || pool_pages <= 0 || !q || !seq_len || !out || !workspace) return KVQ_ERR_INVALID_ARG;
  if (max_pages > 0 && !page_table) return KVQ_ERR_INVALID_ARG;
  if (!aligned16(pool) || !aligned16(q) || !aligned16(workspace)) return KVQ_ERR_INVALID_ARG;
  // pieces of 16 tokens are numbered with 16 bits; the work line is indexed with 32
  const long long tokens = (long long)max_pages * cfg->page_tokens;
  if (tokens > 16ll * 65535) return KVQ_ERR_INVALID_ARG;
  if ((long long)batch * cfg->num_kv_heads * (kDecodePieceWeight * ((tokens + 15) / 16) + kDecodeMergeWeight) >=
      (1ll << 31))
    return KVQ_ERR_INVALID_ARG;
  const Plan pl = decode_plan(cfg, batch);
  if (workspace_bytes < pl.part_bytes + pl.cnt_bytes) return KVQ_ERR_CAPACITY;
  DecodeParams p{};
  p.pool = static_cast<const uint8_t*>(pool);
  p.pool_pages = pool_pages;
  p.Hkv = cfg->num_kv_heads;
  p.P = cfg->page_tokens;
  p.k = cfg->num_boost;
  p.KB = cfg->num_boost / 16;
  p.L = make_layout(cfg->page_tokens, cfg->head_dim, cfg->num_boost, cfg->key_group);
  p.q = static_cast<const uint16_t*>(q);
  p.batch = batch;
  p.Hq = cfg->num_q_heads;
  p.page_table = page_table;
  p.max_pages = max_pages;
  p.seq_len = seq_len;
  p.c_log2 = sm_scale * 1.4426950408889634f;
  p.out = out;
  p.part = static_cast<float*>(workspace);
  p.cnt = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + pl.part_bytes);
  p.n_ctas = pl.ctas;
  p.n_sms = sm_count();
  p.err = err;
  return cuda_status(launch_decode(p, cfg->num_q_heads / cfg->num_kv_heads, cfg->dtype, stream));
}

}  // extern "C"
