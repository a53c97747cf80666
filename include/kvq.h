/*
 * kvq.h — C ABI of the 2-bit mixed-precision KV cache with fused decode attention.
 *
 * What the library computes
 * -------------------------
 * Keys are quantized asymmetrically (min/max, scale + zero point) per channel over
 * groups of consecutive tokens; values are quantized per token over the head
 * dimension.  This split of quantization axes is the KIVI scheme (aibr.jp article on
 * "KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache", section 3 "core
 * technical elements": Keys per channel, Values per token, asymmetric quantization,
 * a full-precision residual of recent tokens, and streaming append into the
 * quantized cache).  On top of it sits Kitty's Dynamic Channel-wise Precision Boost
 * (fugumt.com summary of "Kitty: Accurate and Efficient 2-bit KV Cache Quantization
 * with Dynamic Channel-wise Precision Boost", Abstract; and the notes.yuuk.io wiki
 * page "KVキャッシュ量子化", open questions): the Key channels are ranked by magnitude,
 * a small fraction of them is kept at 4 bits, and every mixed-precision Key page is
 * stored as two uniform 2-bit tensors so that dequantization stays uniform and the
 * page stays coalesced.  Decode attention reads the packed pages directly and
 * dequantizes inside the attention kernel (MiniKV summary on f-binder, section
 * "proposed method": 2-bit KV expanded inside the fused attention matmul).
 *
 * Where the pages leave a step open the library takes one fixed reading; every
 * such reading is listed in this header next to the call it affects.
 *
 * Quantizer (shared by keys, boosted keys and values)
 * ---------------------------------------------------
 * For a group x[0..n) of dtype values and a bit width b:
 *   mn = min x, mx = max x                         (exact; compared after widening to fp32)
 *   s32 = fp32(mx - mn) / (2^b - 1)                (fp32, round-to-nearest-even divide)
 *   scale = s32 rounded toward +infinity to dtype   (so scale*(2^b-1) >= mx-mn)
 *   zero  = mn                                      (stored in dtype, exact; a zero minimum as +0)
 *   code  = clamp(rint(fp32(x - zero) / fp32(scale)), 0, 2^b-1)
 *           (fp32 subtract, fp32 divide, rint = round half to even); code = 0 if scale == 0
 *   dequantized value = code * scale + zero
 * Inputs are assumed finite.
 *
 * Boost-channel selection (per physical page and KV head)
 *   score_c = max over the page's tokens of |K[t][c]|; the num_boost channels with the
 *   largest score are boosted, ties going to the lower channel index; the indices are
 *   stored in ascending order.
 *
 * Keys (per channel c, per group g of key_group consecutive tokens of the page)
 *   normal channel : 2-bit code -> plane A; plane-A scale = scale, plane-A zero = mn.
 *   boosted channel: 4-bit code4 with scale s4 and zero mn; hi = code4 >> 2 -> plane A,
 *                    lo = code4 & 3 -> plane B row j (j = rank of c in boost_idx);
 *                    plane-A scale = 4*s4 (exact), plane-A zero = mn; plane-B scale = s4,
 *                    plane-B zero = 0.  Hence K^ = hi*(4*s4) + mn + lo*s4 = code4*s4 + mn.
 * Values (per token t): 2-bit code over the head_dim channels of that token.
 *
 * Page record (one per physical page and KV head), P = page_tokens, D = head_dim,
 * k = num_boost, G = key_group, S = dtype (2 bytes).  Sections follow one another
 * without gaps, in this order:
 *   k_codes   uint32 [P][D/16]   plane A, token-major; word (t, w) = channels 16w..16w+15 of token t
 *   kb_codes  uint32 [P][k/16]   plane B, token-major; word (t, w) = boosted rows 16w..16w+15
 *   v_codes   uint32 [P*D/16]    values, in the fragment order described below
 *   k_scale   S [P/G][D]         plane-A scale per (group, key scale position)
 *   k_zero    S [P/G][D]         plane-A zero  per (group, key scale position)
 *   kb_scale  S [P/G][k]         plane-B scale per (group, boosted row)
 *   v_scale   S [P]              value scale per value scale position
 *   v_zero    S [P]              value zero  per value scale position
 *   boost_idx uint8 [k]          boosted channels, ascending
 * The record stride (kvq_page_bytes) rounds the payload up to a multiple of 128 bytes;
 * the padding bytes are never read.
 * Keys are packed along channels and values along tokens — the contraction axis of
 * q.K^T and of p.V respectively — so that the decode kernel can feed codes straight
 * into its matrix products with the scales folded into the other operand.  Elements
 * are stored in the order in which the decode kernel's matrix-fragment lanes consume
 * them, and inside a 32-bit word so that one masked byte holds the two codes of one
 * fragment register.  Element e = 8a + 2b + f of a word (a, f in {0,1}, b in 0..3)
 * occupies bits 8b + 4f + 2a; position p of a row is element p % 16 of word p / 16.
 *   key channel c = 16s + 8r + 2q + f  (s 0..7, r, f 0..1, q 0..3)
 *       plane-A code row:      position 32q + 4s + 2r + f
 *       k_scale / k_zero rows: position 32*(s>>1) + 8q + 4*(s&1) + 2r + f
 *   boosted row j = 16s + 8r + 2q + f -> plane-B row position 4*KB*q + 4s + 2r + f, KB = k/16
 *   value code of token t = 32g + 16a + 8u + 2q + f and channel c = 16m + 8v + w
 *       (a, u, v, f 0..1, q 0..3, w 0..7, m 0..7): element 8a + 2(2u + v) + f of word
 *       ((2g + (m>>2))*32 + 4w + q)*4 + (m&3)
 *   v_scale / v_zero of token t = 32g + 8u + w (u 0..3, w 0..7): position 32g + 4w + u
 *   kb_scale and boost_idx are in natural order.
 *
 * Pool: uint8 pool[pool_pages][num_kv_heads][kvq_page_bytes(cfg)], 256-byte aligned base.
 * Residual window: dtype res_k/res_v[batch][num_kv_heads][page_tokens][head_dim];
 *   res_len[b] tokens of sequence b are valid (0 <= res_len[b] <= page_tokens).
 * Page table: int32 page_table[batch][max_pages]; the first num_pages[b] entries are
 *   the physical pages of sequence b in token order.
 *
 * Ownership, streams and errors
 * -----------------------------
 * Every buffer is allocated and owned by the caller; every pointer argument is a
 * device pointer (16-byte aligned where it is read in vectors).  Every call is enqueued on the
 * given stream and returns before the device work finishes.  Arguments are checked
 * on the host before any launch; on a failed check nothing is enqueued and the
 * status says why.  Faults that only the device can see (a page id outside the pool,
 * a full residual window, a full page table) set bits of the optional device word
 * *err (KVQ_DEV_ERR_* flags, OR-ed atomically; pass NULL to ignore) and the offending
 * work item is skipped; outputs of a call that raised a device error are undefined.
 * No kernel traps.  The library's only global state is a per-device record of the
 * SM count and of the kernel attributes it has already set (thread-safe).
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

/* Every entry point is exported with default visibility; the rest of the library is hidden. */
#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID_ARG = 1,  /* null pointer, inconsistent sizes, bad page count         */
  KVQ_ERR_UNSUPPORTED = 2,  /* a shape or precision this build has no kernel for         */
  KVQ_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed                */
  KVQ_ERR_CAPACITY = 4      /* workspace too small                                        */
} kvq_status;

typedef enum { KVQ_F16 = 0, KVQ_BF16 = 1 } kvq_dtype;

/* Device-side error flags OR-ed into *err. */
#define KVQ_DEV_ERR_PAGE_RANGE   1  /* a page id in a table or destination list is outside the pool */
#define KVQ_DEV_ERR_RESIDUAL     2  /* append into a full residual window                            */
#define KVQ_DEV_ERR_TABLE_FULL   4  /* flush with no free page-table slot or no destination page      */
#define KVQ_DEV_ERR_TIMEOUT      8  /* a bounded wait for an asynchronous copy gave up                */
#define KVQ_DEV_ERR_LENGTH      16  /* num_pages[b], res_len[b] or a per-head boost count out of range */
#define KVQ_DEV_ERR_RANGE       32  /* decode: an operand outside the range the kernel carries (see
                                       kvq_decode_attention, "Precision")                             */

/* Shape and precision of one attention layer's KV cache.
 * Supported: head_dim 128; num_q_heads / num_kv_heads in {1, 2, 4, 8};
 * page_tokens in {32, 64, 128}; key_group 32; key_bits 2, boost_bits 4, value_bits 2;
 * num_boost in {0, 16, 32, 64, 128} (0% .. 100% of the channels; 12.5% and 25% are the
 * ratios the method is run with); dtype KVQ_F16 or KVQ_BF16
 * (keys, values, queries, residual, scales and zeros all use dtype). */
typedef struct {
  int32_t head_dim;
  int32_t num_q_heads;
  int32_t num_kv_heads;
  int32_t page_tokens;
  int32_t key_group;
  int32_t key_bits;
  int32_t boost_bits;
  int32_t value_bits;
  int32_t num_boost;
  int32_t dtype;
} kvq_config;

/* Byte offsets of the sections of one page record (see the layout above). */
typedef struct {
  size_t k_codes, kb_codes, v_codes, k_scale, k_zero, kb_scale, v_scale, v_zero, boost_idx;
  size_t payload_bytes;  /* bytes actually used by the sections                 */
  size_t record_bytes;   /* stride between records = payload rounded up to 128  */
} kvq_layout;

/* Human-readable text for a status code (static storage, never NULL). */
KVQ_API const char* kvq_status_string(kvq_status s);

/* Checks a configuration without touching the GPU. */
KVQ_API kvq_status kvq_check_config(const kvq_config* cfg);

/* Fills *out with the record layout of cfg. Host only; no CUDA call. */
KVQ_API kvq_status kvq_page_layout(const kvq_config* cfg, kvq_layout* out);

/* Record stride in bytes for cfg, or 0 if cfg is not supported. */
KVQ_API size_t kvq_page_bytes(const kvq_config* cfg);

/* Source of whole pages for the quantize calls.  Element (page i, token t, kv head h,
 * channel c) is read at src[i*page_stride + t*token_stride + h*head_stride + c]
 * (strides in elements of dtype).  For a token-major prompt [tokens][Hkv][D] use
 * page_stride = P*Hkv*D, token_stride = Hkv*D, head_stride = D. */
typedef struct {
  const void* src;
  int64_t page_stride;
  int64_t token_stride;
  int64_t head_stride;
} kvq_source;

/* a1 — Dynamic Channel-wise Precision Boost selection (Kitty abstract; wiki open
 * question on the magnitude-based channel heuristic).  For each of the n_pages pages
 * of k and each KV head, ranks the channels by max |K| over the page and writes the
 * num_boost highest (ties to the lower index) in ascending order into the boost_idx
 * section of record (dst_pages[i], h).  dst_pages: device int32[n_pages]. */
KVQ_API kvq_status kvq_select_boost_channels(const kvq_config* cfg, kvq_source k,
                                     const int32_t* dst_pages, int32_t n_pages,
                                     void* pool, int64_t pool_pages, int32_t* err,
                                     cudaStream_t stream);

/* a2 — per-channel Key quantization with the two-plane split (KIVI per-channel keys;
 * Kitty abstract: each mixed-precision Key page becomes two unified 2-bit tensors).
 * Reads boost_idx from the destination records (written by
 * kvq_select_boost_channels) and writes k_codes, kb_codes, k_scale, k_zero, kb_scale. */
KVQ_API kvq_status kvq_quantize_page_keys(const kvq_config* cfg, kvq_source k,
                                  const int32_t* dst_pages, int32_t n_pages,
                                  void* pool, int64_t pool_pages, int32_t* err,
                                  cudaStream_t stream);

/* a3 — per-token Value quantization (KIVI section 3).  Writes v_codes, v_scale, v_zero. */
KVQ_API kvq_status kvq_quantize_values(const kvq_config* cfg, kvq_source v,
                               const int32_t* dst_pages, int32_t n_pages,
                               void* pool, int64_t pool_pages, int32_t* err,
                               cudaStream_t stream);

/* a1+a2+a3 in one pass over each page: the same bytes as the three calls above. */
KVQ_API kvq_status kvq_quantize_pages(const kvq_config* cfg, kvq_source k, kvq_source v,
                              const int32_t* dst_pages, int32_t n_pages,
                              void* pool, int64_t pool_pages, int32_t* err,
                              cudaStream_t stream);

/* Options of the boost-channel choice, for kvq_quantize_pages_ex and
 * kvq_flush_residual_ex (NULL options, or NULL fields, give the plain calls' behaviour).
 *  query_weight   — query-aware ranking (MixKVQ summary on fugumt.com, Abstract: key
 *                   channels chosen by intrinsic quantization difficulty together with
 *                   query relevance).  Reading: device float[num_kv_heads][head_dim] of
 *                   non-negative relevance weights w (for example the mean |q| of a
 *                   channel over the query heads of the kv head and recent steps); a
 *                   channel's score is fp32(w_c * fp32(max_t K - min_t K)) over the page
 *                   (its range, which sets its 2-bit error), the highest scores are
 *                   boosted, ties to the lower channel index.  NULL: magnitude (max |K|).
 *  boost_per_head — per-head boost count (notes.yuuk.io wiki "KVキャッシュ量子化", open
 *                   questions: per-head or adaptive boost ratios).  Device int32
 *                   [num_kv_heads], each in [0, num_boost]: head h boosts that many
 *                   channels; the record keeps its num_boost plane-B rows and the unused
 *                   ones (codes, scales, indices) are zero, so decode attention reads
 *                   them unchanged and they add nothing.  A count outside the range sets
 *                   KVQ_DEV_ERR_LENGTH and is clamped.  NULL: num_boost for every head. */
typedef struct {
  const float* query_weight;
  const int32_t* boost_per_head;
} kvq_boost_options;

/* kvq_quantize_pages with boost options. */
KVQ_API kvq_status kvq_quantize_pages_ex(const kvq_config* cfg, kvq_source k, kvq_source v,
                                         const int32_t* dst_pages, int32_t n_pages,
                                         void* pool, int64_t pool_pages, const kvq_boost_options* opts,
                                         int32_t* err, cudaStream_t stream);

/* a4 — streaming append into the full-precision residual window (KIVI section 3:
 * recent tokens stay in full precision and new tokens are appended without touching
 * quantized pages).  k_new, v_new: dtype [batch][Hkv][D].  For every b, writes the
 * token at position res_len[b] of res_k/res_v and increments res_len[b].  A sequence
 * whose window is already full (res_len[b] == page_tokens) is skipped and raises
 * KVQ_DEV_ERR_RESIDUAL: flush first. */
KVQ_API kvq_status kvq_append_token(const kvq_config* cfg, int32_t batch,
                            const void* k_new, const void* v_new,
                            void* res_k, void* res_v, int32_t* res_len,
                            int32_t* err, cudaStream_t stream);

/* a5 — residual flush.  Reading: the window is flushed when it holds a whole page
 * (res_len[b] == page_tokens); the flush quantizes the window as one page (a1-a3)
 * into physical page new_page[b], appends that page to the page table
 * (page_table[b][num_pages[b]] = new_page[b], num_pages[b] += 1) and empties the
 * window (res_len[b] = 0).  Sequences whose window is not full are left untouched.
 * new_page: device int32[batch], the page the host reserves for b (ignored unless b
 * flushes; a negative id or a full table raises KVQ_DEV_ERR_TABLE_FULL and skips b).
 * The caller decides which sequences will flush (it issued the appends), so the call
 * needs no device-to-host read and can be captured in a CUDA graph. */
KVQ_API kvq_status kvq_flush_residual(const kvq_config* cfg, int32_t batch,
                              const void* res_k, const void* res_v, int32_t* res_len,
                              const int32_t* new_page, int32_t* page_table,
                              int32_t max_pages, int32_t* num_pages,
                              void* pool, int64_t pool_pages, int32_t* err,
                              cudaStream_t stream);

/* kvq_flush_residual with boost options (the flushed pages' channel choice). */
KVQ_API kvq_status kvq_flush_residual_ex(const kvq_config* cfg, int32_t batch,
                                         const void* res_k, const void* res_v, int32_t* res_len,
                                         const int32_t* new_page, int32_t* page_table,
                                         int32_t max_pages, int32_t* num_pages,
                                         void* pool, int64_t pool_pages, const kvq_boost_options* opts,
                                         int32_t* err, cudaStream_t stream);

/* a4 + a5 in one launch: for every b, kvq_append_token's append followed by
 * kvq_flush_residual(_ex)'s flush of a window the append filled (KIVI section 3: the
 * streaming append, and the residual quantized once a whole page has accumulated).  The
 * arguments are those two calls' arguments together; the final window, lengths, page
 * table, records and error bits equal what the two calls would leave, including a window
 * that was already full (KVQ_DEV_ERR_RESIDUAL, then flushed if new_page[b] is valid).
 * One CTA per (sequence, KV head, keys | values) appends its row and quantizes its part;
 * the last of a sequence's CTAs to finish updates res_len, num_pages and page_table, so
 * no CTA sees a length another has already changed.
 * counters: device int32[batch], zero before the first call (clear once after
 * allocating); every call leaves them zero.  opts may be NULL.  Errors as for the two
 * calls; a NULL pointer or misaligned buffer returns KVQ_ERR_INVALID_ARG. */
KVQ_API kvq_status kvq_append_flush(const kvq_config* cfg, int32_t batch,
                                    const void* k_new, const void* v_new,
                                    void* res_k, void* res_v, int32_t* res_len,
                                    const int32_t* new_page, int32_t* page_table,
                                    int32_t max_pages, int32_t* num_pages,
                                    void* pool, int64_t pool_pages, const kvq_boost_options* opts,
                                    int32_t* counters, int32_t* err, cudaStream_t stream);

/* Scratch bytes kvq_decode_attention needs for (cfg, batch, max_pages) on the current
 * device (max_pages does not change it).  The workspace holds the partial softmax
 * states of sequences split across CTAs (one slot per pair of CTA and (sequence, KV
 * head) that can meet) and one 32-bit counter per (sequence, KV head).  The counters
 * must be zero before the first call (clear the whole workspace once after allocating
 * it); every call leaves them zero again.  Without a visible device the size assumes
 * the largest possible grid. */
KVQ_API size_t kvq_decode_workspace_bytes(const kvq_config* cfg, int32_t batch, int32_t max_pages);

/* a6 + a7 — decode attention over the paged, packed cache plus the residual window
 * (Kitty abstract: page dequantization kernels over a page-centric layout; MiniKV
 * proposed method: dequantization fused into the attention matmuls).  For every
 * sequence b and query head h (KV head h / (Hq/Hkv)):
 *   out[b][h] = softmax(sm_scale * q[b][h] . K^T) V
 * over the num_pages[b] quantized pages of page_table[b] (dequantized inside the
 * kernel) followed by the res_len[b] residual tokens.  All (sequence, KV head) token
 * ranges are laid end to end and cut into equal shares, one per resident CTA, so the
 * work per SM is the same whatever the sequence lengths; a range split across CTAs is
 * merged by log-sum-exp in the same launch (no second kernel).
 * q: dtype [batch][Hq][D]; out: fp32 [batch][Hq][D]; sm_scale normally 1/sqrt(D).
 * workspace: device, >= kvq_decode_workspace_bytes(cfg, batch, max_pages) bytes,
 * see kvq_decode_workspace_bytes for its zero-counter contract.
 * A sequence with no tokens at all (num_pages[b] == 0 and res_len[b] == 0) gets an
 * all-zero output row.
 * Precision and range: the codes enter the tensor-core products exactly; the scales are
 * folded into the other operand, carried as an fp16 high part plus an fp16 low part, and
 * products accumulate in fp32.  Each query head enters as q * 2^-e with e >= 0 the
 * smallest power of two above max |q| (e = 0 when |q| < 1), so a folded key operand
 * never exceeds its key scale: for fp16 caches no folded operand can overflow.  The
 * value operand p * sV is carried as p * sV * 2^-F with a per-warp exponent F that grows
 * before a value scale could overflow it.  bf16 caches: key scales and zero points enter
 * the products as fp16 — exact down to 2^-14, with an absolute error below 2^-25 under
 * it; a key scale or zero point above 65504 in magnitude (keys of magnitude above about
 * 10^5), or a query above 2^24, is outside the supported range and sets
 * KVQ_DEV_ERR_RANGE (the output is then undefined), as does any non-finite input. */
KVQ_API kvq_status kvq_decode_attention(const kvq_config* cfg, const void* pool, int64_t pool_pages,
                                const void* q, int32_t batch,
                                const int32_t* page_table, int32_t max_pages,
                                const int32_t* num_pages,
                                const void* res_k, const void* res_v, const int32_t* res_len,
                                float sm_scale, float* out,
                                void* workspace, size_t workspace_bytes,
                                int32_t* err, cudaStream_t stream);

/* ---- MiniKV prefill: attention with cumulative scores, token retention, gather ----
 * MiniKV summary (f-binder), "proposed method": the prompt is processed at prefill, the
 * KV states to keep are chosen by cumulative attention score — heavy hitters — together
 * with a recent window (25% of the budget each by default), and a two-stage selective
 * flash-attention kernel returns the attention output and those scores in linear memory.
 * The kept tokens are then quantized like any other (keys per channel, values per token).
 * Reading: causal attention over the L prompt tokens; the cumulative score of key token
 * j of KV head h is the attention it receives, summed over all query positions and over
 * the query heads of h. */

/* Workspace bytes of kvq_prefill_attention: the log2-sum-exp of every query row and the
 * cumulative scores of every query head (fp32 [num_q_heads][L] each). */
KVQ_API size_t kvq_prefill_workspace_bytes(const kvq_config* cfg, int32_t L);

/* q: dtype [L][num_q_heads][head_dim]; k, v: dtype [L][num_kv_heads][head_dim];
 * out: fp32 [L][num_q_heads][head_dim], out[i][h] = sum_{j <= i} softmax_j(sm_scale
 * q_i . k_j) v_j (KV head h / (Hq/Hkv)); scores: fp32 [num_kv_heads][L] cumulative
 * attention scores.  Two kernels (output and row log2-sum-exp; then the scores, by
 * recomputing K Q^T per key block), memory linear in L.  Products in the cache dtype,
 * fp32 accumulate; bf16 probabilities are carried as a high and a low bf16 part. */
KVQ_API kvq_status kvq_prefill_attention(const kvq_config* cfg, const void* q, const void* k, const void* v,
                                         int32_t L, float sm_scale, float* out, float* scores,
                                         void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Token retention per KV head: the last n_recent positions plus the n_heavy positions of
 * highest score among the others (ties to the lower position), written ascending to
 * keep[h][0 .. n_keep[h]) (keep: device int32 [num_kv_heads][L], n_keep: device int32
 * [num_kv_heads]; n_keep[h] = min(L, n_heavy + n_recent)).  Scores are the fp32 values of
 * kvq_prefill_attention (non-negative); the decision is taken on them as given. */
KVQ_API kvq_status kvq_retain_tokens(const kvq_config* cfg, const float* scores, int32_t L,
                                     int32_t n_heavy, int32_t n_recent, int32_t* keep, int32_t* n_keep,
                                     cudaStream_t stream);

/* The kept tokens compacted, token-major: k_out[t][h] = k[keep[h][t]][h] (and v) for
 * t < n, every KV head keeping n tokens (n = n_keep[h] of kvq_retain_tokens).  k_out and
 * v_out are dtype [n][num_kv_heads][head_dim], the source layout of kvq_quantize_pages.
 * A kept position outside [0, L) sets KVQ_DEV_ERR_LENGTH and copies token 0. */
KVQ_API kvq_status kvq_gather_tokens(const kvq_config* cfg, const void* k, const void* v, int32_t L,
                                     const int32_t* keep, int32_t n, void* k_out, void* v_out,
                                     int32_t* err, cudaStream_t stream);

/* Bytes of one (page, KV head) record of a dense cache: K rows then V rows, dtype
 * [2][page_tokens][head_dim]; 0 if cfg is not supported. */
KVQ_API size_t kvq_dense_page_bytes(const kvq_config* cfg);

/* Decode attention over an unquantized (fp16 / bf16) paged cache, on the same kernel,
 * work line and split-K merge as kvq_decode_attention: the comparison point of the 2-bit
 * cache (KIVI article on aibr.jp, section 4, and the Kitty summary's Abstract compare
 * against full-precision KV; this call is that baseline on this hardware).
 * pool: dtype [pool_pages][num_kv_heads][2][page_tokens][head_dim] (K rows, V rows);
 * page_table: int32 [batch][max_pages]; seq_len: device int32 [batch], tokens of each
 * sequence (0 <= seq_len[b] <= max_pages * page_tokens, the first ceil(seq_len[b] /
 * page_tokens) table entries valid); q, out, sm_scale, workspace (the size
 * kvq_decode_workspace_bytes gives), err and stream as for kvq_decode_attention.
 * Products run in the cache dtype with fp32 accumulation; num_boost and key_group of cfg
 * are not used.  max_pages * page_tokens must not exceed 1048560. */
KVQ_API kvq_status kvq_decode_attention_dense(const kvq_config* cfg, const void* pool, int64_t pool_pages,
                                              const void* q, int32_t batch,
                                              const int32_t* page_table, int32_t max_pages,
                                              const int32_t* seq_len, float sm_scale, float* out,
                                              void* workspace, size_t workspace_bytes,
                                              int32_t* err, cudaStream_t stream);

/* Size of the library's built-in decode scratch (see kvq_decode_attention_static). */
#define KVQ_STATIC_SCRATCH_BYTES (16u << 20)

/* Decode attention without a caller workspace, for callers that cannot allocate
 * device memory: a serving engine whose memory pool already holds all of the GPU, a
 * plugin whose host framework owns every device allocation, or a latency-critical
 * path that must not call cudaMalloc because it may synchronize the device.  (The
 * web pages on the method have no counterpart of this call; it is a property of this
 * library's interface only.)
 * Same arguments, results and error behaviour as kvq_decode_attention, minus the
 * workspace: the split-K partials and arrival counters live in a static device buffer
 * of KVQ_STATIC_SCRATCH_BYTES (16 MiB) inside the library, which every GPU that loads
 * the library keeps until the process exits.  Shapes that need more than that
 * (kvq_decode_workspace_bytes(cfg, batch, max_pages) > KVQ_STATIC_SCRATCH_BYTES) are
 * rejected with KVQ_ERR_CAPACITY before anything is enqueued.
 * The call allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 * The first call on each device looks up the buffer's device address
 * (cudaGetSymbolAddress) with that device current.  With lazy module loading (the CUDA
 * default since 12.2) that lookup is also what loads the library's device code and
 * commits the buffer's memory, so it can fail with KVQ_ERR_CUDA on a device whose memory
 * is already taken: call once with batch = 0 (every other argument may be NULL or zero
 * except cfg) early — before the caller's pool claims the device and outside any stream
 * capture; that call only resolves the buffer.  The address is cached per device for the
 * life of the process: after cudaDeviceReset or a re-created primary context the entry
 * point must not be called again on that device.
 * Each call clears the buffer's arrival counters on `stream` before the kernel runs; the
 * rest keeps the previous call's contents.  All calls on a device share the one buffer,
 * so two calls whose executions overlap on the GPU (different streams without ordering
 * between them) race and give undefined results.  Invalid arguments are rejected before
 * the buffer is looked up or cleared, exactly as kvq_decode_attention rejects them. */
KVQ_API kvq_status kvq_decode_attention_static(const kvq_config* cfg, const void* pool, int64_t pool_pages,
                                               const void* q, int32_t batch,
                                               const int32_t* page_table, int32_t max_pages,
                                               const int32_t* num_pages,
                                               const void* res_k, const void* res_v, const int32_t* res_len,
                                               float sm_scale, float* out, int32_t* err, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
