/*
 * kvq_oracle.c — TEST INFRASTRUCTURE, not part of the product.
 *
 * A plain, slow CPU restatement of the 2-bit mixed-precision KV cache and of decode
 * attention over it.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load this library; the product path never does.  It shares no code,
 * header, table or constant with the CUDA library: the record layout, the packing
 * and every formula are written out again here from their definitions.
 *
 * Sources (web pages on the method):
 *  - aibr.jp article on KIVI, section 3 (core technical elements): asymmetric
 *    quantization, Keys per channel, Values per token, full-precision residual of
 *    recent tokens, streaming append.
 *  - fugumt.com summary of Kitty (arXiv 2511.18643), Abstract: channels of the Key
 *    cache are ranked and a small fraction kept at higher precision; each
 *    mixed-precision Key page is stored as two uniform 2-bit tensors.
 *  - notes.yuuk.io wiki page "KVキャッシュ量子化", open questions: the ranking is a
 *    magnitude heuristic; boost ratios 12.5% and 25%.
 *  - f-binder summary of MiniKV, section "proposed method": keys grouped along
 *    channels, values per token, 2-bit codes expanded inside the attention matmul.
 * The pages print no formula.  The readings taken here (min/max asymmetric
 * quantizer with scale = (max-min)/(2^b-1) rounded up to the storage type, zero =
 * min, round half to even, clamp; magnitude = max |x| over the page; ties to the
 * lower channel; 4-bit code = 4*hi + lo) are the plainest ones and are the same
 * readings the library documents.
 *
 * Arithmetic: the quantizer works in fp32 with one rounding per operation, in the
 * order written (build with -ffp-contract=off, no fast-math), because its fp32
 * decisions fix integer codes.  Dequantization and attention work in fp64, where
 * code*scale + zero of two 16-bit values is exact.
 *
 * Every function below states which part of the method it follows.  Parity pins for
 * each function live in the tests (brute force, closed forms, library routines).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define DT_F16 0
#define DT_BF16 1

/* ---------------------------------------------------------------- 16-bit float types */

/* IEEE binary16 bits -> value (exact). */
static double f16_value(uint16_t h) {
  int sign = (h >> 15) & 1;
  int e = (h >> 10) & 0x1f;
  int m = h & 0x3ff;
  double v;
  if (e == 0)
    v = ldexp((double)m, -24);
  else if (e == 31)
    v = m ? NAN : INFINITY;
  else
    v = ldexp((double)(m + 1024), e - 25);
  return sign ? -v : v;
}

/* bfloat16 bits -> value (exact): the upper half of an IEEE binary32. */
static double bf16_value(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, 4);
  return (double)f;
}

static double dt_value(uint16_t bits, int dtype) {
  return dtype == DT_BF16 ? bf16_value(bits) : f16_value(bits);
}

/* Rounds a finite double to the 16-bit type.  mode 0: nearest, ties to even;
 * mode 1: toward +infinity.  Written from the format definitions: a value is an
 * integer multiple of the quantum of its binade (or of the subnormal quantum). */
static uint16_t dt_round(double x, int dtype, int mode) {
  const int man_bits = dtype == DT_BF16 ? 7 : 10;
  const int emin = dtype == DT_BF16 ? -126 : -14;  /* exponent of the smallest normal */
  const int emax = dtype == DT_BF16 ? 127 : 15;
  const int bias = dtype == DT_BF16 ? 127 : 15;
  const int exp_field_max = dtype == DT_BF16 ? 255 : 31;
  uint16_t sign = 0;
  double a = x;
  if (x < 0 || (x == 0 && signbit(x))) {
    sign = 1;
    a = -x;
  }
  if (a == 0) return (uint16_t)(sign << 15);
  int e2;
  frexp(a, &e2);          /* a = f * 2^e2 with f in [0.5, 1) */
  int e = e2 - 1;         /* a in [2^e, 2^(e+1)) */
  if (e < emin) e = emin; /* subnormal range shares the quantum of the smallest binade */
  double quantum = ldexp(1.0, e - man_bits);
  double n = a / quantum; /* exact: scaling by a power of two */
  double r;
  if (mode == 0) {
    r = nearbyint(n);     /* default rounding mode: half to even */
  } else {
    /* toward +inf: magnitude up for positive numbers, down for negative ones */
    r = sign ? floor(n) : ceil(n);
  }
  double v = r * quantum;
  double maxv = ldexp((double)((2 << man_bits) - 1), emax - man_bits);
  if (v > maxv) {
    /* overflow: nearest gives inf beyond the halfway point; upward gives +inf for
     * positive values (negative values cannot round up in magnitude here) */
    return (uint16_t)((sign << 15) | (exp_field_max << man_bits));
  }
  if (v == 0) return (uint16_t)(sign << 15);
  /* encode the exact value v */
  frexp(v, &e2);
  e = e2 - 1;
  uint16_t bits;
  if (e < emin) {
    bits = (uint16_t)(v / ldexp(1.0, emin - man_bits));
  } else {
    uint32_t m = (uint32_t)(v / ldexp(1.0, e - man_bits)) - (1u << man_bits);
    bits = (uint16_t)(((uint32_t)(e + bias) << man_bits) | m);
  }
  return (uint16_t)((sign << 15) | bits);
}

double kvqo_value(uint16_t bits, int dtype) { return dt_value(bits, dtype); }
uint16_t kvqo_round_nearest(double x, int dtype) { return dt_round(x, dtype, 0); }
uint16_t kvqo_round_up(double x, int dtype) { return dt_round(x, dtype, 1); }

/* ------------------------------------------------------------------------ quantizer */

/* Asymmetric min/max quantization of one group (KIVI section 3: asymmetric
 * quantization).  x: n values given as 16-bit patterns of dtype, read with stride.
 * Writes n codes, the stored scale and zero (16-bit patterns).  fp32 arithmetic,
 * one rounding per operation:
 *   mn, mx       = min and max of the group
 *   s32          = (mx - mn) / (2^bits - 1)
 *   scale        = s32 rounded toward +inf to dtype
 *   zero         = mn (a zero minimum is stored as +0)
 *   code         = clamp(rint((x - zero) / scale), 0, 2^bits - 1); 0 when scale == 0 */
void kvqo_quant_group(const uint16_t* x, int n, long stride, int bits, int dtype,
                      uint8_t* codes, uint16_t* scale_bits, uint16_t* zero_bits) {
  float mn = (float)dt_value(x[0], dtype);
  float mx = mn;
  for (int i = 1; i < n; ++i) {
    float v = (float)dt_value(x[i * stride], dtype);
    if (v < mn) mn = v;
    if (v > mx) mx = v;
  }
  const int qmax = (1 << bits) - 1;
  volatile float range = mx - mn;
  volatile float s32 = range / (float)qmax;
  uint16_t sb = dt_round((double)s32, dtype, 1);
  float scale = (float)dt_value(sb, dtype);
  uint16_t zb = mn == 0.0f ? 0 : dt_round((double)mn, dtype, 0);
  float zero = (float)dt_value(zb, dtype);
  for (int i = 0; i < n; ++i) {
    int code = 0;
    if (scale != 0.0f) {
      float v = (float)dt_value(x[i * stride], dtype);
      volatile float d = v - zero;
      volatile float t = d / scale;
      float r = rintf(t);
      if (r < 0.0f) r = 0.0f;
      if (r > (float)qmax) r = (float)qmax;
      code = (int)r;
    }
    codes[i] = (uint8_t)code;
  }
  *scale_bits = sb;
  *zero_bits = zb;
}

/* --------------------------------------------------------------------- page layout */

typedef struct {
  long k_codes, kb_codes, v_codes, k_scale, k_zero, kb_scale, v_scale, v_zero, boost_idx;
  long payload, record;
} layout_t;

/* Section order and sizes of one (page, KV head) record; see the library's ABI
 * description of the page record.  P tokens, D channels, k boosted rows, G group. */
static layout_t make_layout(int P, int D, int k, int G) {
  layout_t L;
  long off = 0;
  L.k_codes = off;   off += (long)P * (D / 16) * 4;
  L.kb_codes = off;  off += (long)P * (k / 16) * 4;
  L.v_codes = off;   off += (long)D * (P / 16) * 4;
  L.k_scale = off;   off += (long)(P / G) * D * 2;
  L.k_zero = off;    off += (long)(P / G) * D * 2;
  L.kb_scale = off;  off += (long)(P / G) * k * 2;
  L.v_scale = off;   off += (long)P * 2;
  L.v_zero = off;    off += (long)P * 2;
  L.boost_idx = off; off += k;
  L.payload = off;
  L.record = (off + 127) / 128 * 128;
  return L;
}

void kvqo_layout(int P, int D, int k, int G, long* out /* 11 entries */) {
  layout_t L = make_layout(P, D, k, G);
  long v[11] = {L.k_codes, L.kb_codes, L.v_codes, L.k_scale, L.k_zero, L.kb_scale,
                L.v_scale, L.v_zero, L.boost_idx, L.payload, L.record};
  memcpy(out, v, sizeof v);
}

/* Bit position of element e (0..15) inside a 32-bit code word.  Writing
 * e = 8a + 2b + f (a, f in {0,1}, b in 0..3), element e occupies bits 8b + 4f + 2a:
 * byte b holds elements 2b, 2b+1 (a = 0) in the low two bits of its two nibbles and
 * elements 8+2b, 9+2b (a = 1) in the high two bits. */
static int elem_shift(int e) {
  const int a = e >> 3, b = (e >> 1) & 3, f = e & 1;
  return 8 * b + 4 * f + 2 * a;
}

/* Storage position of key channel c (0..127) inside a plane-A row and inside the
 * plane-A scale and zero rows.  Writing c = 16s + 8r + 2q + f (s in 0..7, r, f in
 * {0,1}, q in 0..3), the position is 32q + 4s + 2r + f. */
static int key_pos(int c) {
  const int s = c >> 4, r = (c >> 3) & 1, q = (c >> 1) & 3, f = c & 1;
  return 32 * q + 4 * s + 2 * r + f;
}

/* Storage position of boosted row j (0..k-1) inside a plane-B row, KB = k/16:
 * j = 16s + 8r + 2q + f -> 4*KB*q + 4s + 2r + f. */
static int boost_pos(int j, int KB) {
  const int s = j >> 4, r = (j >> 3) & 1, q = (j >> 1) & 3, f = j & 1;
  return 4 * KB * q + 4 * s + 2 * r + f;
}

/* Storage position of key channel c inside the plane-A scale and zero rows:
 * c = 16s + 8r + 2q + f -> 32*(s >> 1) + 8q + 4*(s & 1) + 2r + f. */
static int key_meta_pos(int c) {
  const int s = c >> 4, r = (c >> 3) & 1, q = (c >> 1) & 3, f = c & 1;
  return 32 * (s >> 1) + 8 * q + 4 * (s & 1) + 2 * r + f;
}

/* Slot (16 * word + element) of the value code of token t (0..P-1) and channel c
 * (0..127) inside the value-code section.  Writing t = 32g + 16a + 8u + 2q + f and
 * c = 16m + 8v + w (a, u, v, f in {0,1}, q in 0..3, w in 0..7, m in 0..7), the code is
 * element 8a + 2(2u + v) + f of word ((2g + (m >> 2)) * 32 + 4w + q) * 4 + (m & 3). */
static int value_slot(int t, int c) {
  const int g = t >> 5, a = (t >> 4) & 1, u = (t >> 3) & 1, q = (t >> 1) & 3, f = t & 1;
  const int m = c >> 4, v = (c >> 3) & 1, w = c & 7;
  const int word = ((2 * g + (m >> 2)) * 32 + 4 * w + q) * 4 + (m & 3);
  return 16 * word + 8 * a + 2 * (2 * u + v) + f;
}

/* Storage position of token t inside the value scale and zero rows:
 * t = 32g + 8u + w (u in 0..3, w in 0..7) -> 32g + 4w + u. */
static int value_meta_pos(int t) {
  const int g = t >> 5, u = (t >> 3) & 3, w = t & 7;
  return 32 * g + 4 * w + u;
}

int kvqo_elem_shift(int e) { return elem_shift(e); }
int kvqo_key_pos(int c) { return key_pos(c); }
int kvqo_boost_pos(int j, int KB) { return boost_pos(j, KB); }
int kvqo_key_meta_pos(int c) { return key_meta_pos(c); }
int kvqo_value_slot(int t, int c) { return value_slot(t, c); }
int kvqo_value_meta_pos(int t) { return value_meta_pos(t); }

/* Writes / reads the 2-bit code at storage position pos of row `row` (words_per_row
 * words of 16 elements each). */
static void put2(uint32_t* words, int row, int words_per_row, int pos, unsigned code) {
  words[row * words_per_row + pos / 16] |= (uint32_t)(code & 3u) << elem_shift(pos % 16);
}

static unsigned get2(const uint32_t* words, int row, int words_per_row, int pos) {
  return (words[row * words_per_row + pos / 16] >> elem_shift(pos % 16)) & 3u;
}

/* Same for a section addressed by slot = 16 * word + element. */
static void put2s(uint32_t* words, int slot, unsigned code) {
  words[slot / 16] |= (uint32_t)(code & 3u) << elem_shift(slot % 16);
}

static unsigned get2s(const uint32_t* words, int slot) {
  return (words[slot / 16] >> elem_shift(slot % 16)) & 3u;
}

/* -------------------------------------------------------------- boost selection (a1) */

/* Dynamic Channel-wise Precision Boost selection (Kitty abstract; wiki: magnitude
 * heuristic).  score_c = max_t |K[t][c]| over the page; the k channels with the
 * highest score, ties to the lower index, returned in ascending channel order. */
void kvqo_select_boost(const uint16_t* K, long tok_stride, int P, int D, int k, int dtype,
                       uint8_t* idx) {
  double* score = (double*)malloc(sizeof(double) * D);
  char* taken = (char*)calloc(D, 1);
  for (int c = 0; c < D; ++c) {
    double s = 0.0;
    for (int t = 0; t < P; ++t) {
      double a = fabs(dt_value(K[t * tok_stride + c], dtype));
      if (a > s) s = a;
    }
    score[c] = s;
  }
  /* k rounds of "pick the best remaining channel" */
  for (int r = 0; r < k; ++r) {
    int best = -1;
    for (int c = 0; c < D; ++c) {
      if (taken[c]) continue;
      if (best < 0 || score[c] > score[best]) best = c;  /* strict: lower index wins ties */
    }
    taken[best] = 1;
  }
  int j = 0;
  for (int c = 0; c < D; ++c)
    if (taken[c]) idx[j++] = (uint8_t)c;
  free(score);
  free(taken);
}

/* Query-aware selection (MixKVQ summary on fugumt.com, Abstract: key channels are
 * ranked by their intrinsic quantization difficulty together with their relevance to
 * the query).  Reading: the difficulty of channel c is its range over the page,
 * r_c = fl32(max_t K[t][c] - min_t K[t][c]) (the 2-bit step, and so the error, grows
 * with it); the relevance is a caller-given weight w_c >= 0 (for example the mean |q_c|
 * of the query heads that share the KV head); score_c = fl32(w_c * r_c), each in fp32
 * with one rounding.  The n channels with the highest score are boosted, ties to the
 * lower channel index, returned in ascending channel order. */
void kvqo_select_boost_query(const uint16_t* K, long tok_stride, int P, int D, int n, const float* w,
                             int dtype, uint8_t* idx) {
  float* score = (float*)malloc(sizeof(float) * D);
  char* taken = (char*)calloc(D, 1);
  for (int c = 0; c < D; ++c) {
    float mn = (float)dt_value(K[c], dtype), mx = mn;
    for (int t = 1; t < P; ++t) {
      const float v = (float)dt_value(K[t * tok_stride + c], dtype);
      if (v < mn) mn = v;
      if (v > mx) mx = v;
    }
    volatile float range = mx - mn;
    volatile float sc = w[c] * range;
    score[c] = sc;
  }
  for (int r = 0; r < n; ++r) {
    int best = -1;
    for (int c = 0; c < D; ++c) {
      if (taken[c]) continue;
      if (best < 0 || score[c] > score[best]) best = c;  /* strict: lower index wins ties */
    }
    taken[best] = 1;
  }
  int j = 0;
  for (int c = 0; c < D; ++c)
    if (taken[c]) idx[j++] = (uint8_t)c;
  free(score);
  free(taken);
}

/* ------------------------------------------------------------- page quantization */

/* Quantizes one page of one KV head into a record (a1 + a2 + a3).
 * K, V: [P][D] 16-bit patterns with token stride tok_stride (elements).
 * rec: record_bytes bytes; padding is left zero. */
void kvqo_quantize_page_ex(const uint16_t* K, const uint16_t* V, long tok_stride, int P, int D,
                           int G, int k, int n_boost, const float* w, int dtype, uint8_t* rec);

void kvqo_quantize_page(const uint16_t* K, const uint16_t* V, long tok_stride, int P, int D,
                        int G, int k, int dtype, uint8_t* rec) {
  kvqo_quantize_page_ex(K, V, tok_stride, P, D, G, k, k, NULL, dtype, rec);
}

/* The same with the options of the per-head boost count and the query-aware ranking:
 * the record is laid out for k plane-B rows, but only n_boost <= k channels are boosted
 * (rows n_boost..k-1 of plane B, their scales and their boost indices stay zero, so they
 * add nothing to a dequantized key); w = NULL ranks by magnitude, otherwise by
 * kvqo_select_boost_query. */
void kvqo_quantize_page_ex(const uint16_t* K, const uint16_t* V, long tok_stride, int P, int D,
                           int G, int k, int n_boost, const float* w, int dtype, uint8_t* rec) {
  layout_t L = make_layout(P, D, k, G);
  memset(rec, 0, (size_t)L.record);
  uint32_t* kA = (uint32_t*)(rec + L.k_codes);
  uint32_t* kB = (uint32_t*)(rec + L.kb_codes);
  uint32_t* vq = (uint32_t*)(rec + L.v_codes);
  uint16_t* ks = (uint16_t*)(rec + L.k_scale);
  uint16_t* kz = (uint16_t*)(rec + L.k_zero);
  uint16_t* kbs = (uint16_t*)(rec + L.kb_scale);
  uint16_t* vs = (uint16_t*)(rec + L.v_scale);
  uint16_t* vz = (uint16_t*)(rec + L.v_zero);
  uint8_t* bidx = rec + L.boost_idx;

  /* a1: boosted channels */
  if (w)
    kvqo_select_boost_query(K, tok_stride, P, D, n_boost, w, dtype, bidx);
  else
    kvqo_select_boost(K, tok_stride, P, D, n_boost, dtype, bidx);
  int* row_of = (int*)malloc(sizeof(int) * D); /* plane-B row of a boosted channel, else -1 */
  for (int c = 0; c < D; ++c) row_of[c] = -1;
  for (int j = 0; j < n_boost; ++j) row_of[bidx[j]] = j;

  /* a2: keys, per channel and per group of G tokens */
  uint8_t* codes = (uint8_t*)malloc((size_t)(P > D ? P : D));
  const int kw = D / 16, kbw = k / 16;
  for (int g = 0; g < P / G; ++g) {
    for (int c = 0; c < D; ++c) {
      const uint16_t* col = K + (long)g * G * tok_stride + c;
      uint16_t sb, zb;
      int j = row_of[c];
      const int pc = key_pos(c);
      if (j < 0) {
        kvqo_quant_group(col, G, tok_stride, 2, dtype, codes, &sb, &zb);
        for (int t = 0; t < G; ++t) put2(kA, g * G + t, kw, pc, codes[t]);
        ks[g * D + key_meta_pos(c)] = sb;
      } else {
        kvqo_quant_group(col, G, tok_stride, 4, dtype, codes, &sb, &zb);
        for (int t = 0; t < G; ++t) {
          put2(kA, g * G + t, kw, pc, codes[t] >> 2);
          put2(kB, g * G + t, kbw, boost_pos(j, kbw), codes[t] & 3);
        }
        /* plane A carries the high bits with four times the 4-bit scale (exact) */
        ks[g * D + key_meta_pos(c)] = dt_round(4.0 * dt_value(sb, dtype), dtype, 0);
        kbs[g * k + j] = sb;
      }
      kz[g * D + key_meta_pos(c)] = zb;
    }
  }

  /* a3: values, per token over all D channels */
  for (int t = 0; t < P; ++t) {
    uint16_t sb, zb;
    kvqo_quant_group(V + (long)t * tok_stride, D, 1, 2, dtype, codes, &sb, &zb);
    for (int c = 0; c < D; ++c) put2s(vq, value_slot(t, c), codes[c]);
    vs[value_meta_pos(t)] = sb;
    vz[value_meta_pos(t)] = zb;
  }
  free(codes);
  free(row_of);
}

/* Dequantizes a record in fp64: Khat, Vhat [P][D].  K^ = A-code * A-scale + A-zero
 * (+ B-code * B-scale for boosted channels); V^ = code * scale + zero. */
void kvqo_dequantize_page(const uint8_t* rec, int P, int D, int G, int k, int dtype,
                          double* Khat, double* Vhat) {
  layout_t L = make_layout(P, D, k, G);
  const uint32_t* kA = (const uint32_t*)(rec + L.k_codes);
  const uint32_t* kB = (const uint32_t*)(rec + L.kb_codes);
  const uint32_t* vq = (const uint32_t*)(rec + L.v_codes);
  const uint16_t* ks = (const uint16_t*)(rec + L.k_scale);
  const uint16_t* kz = (const uint16_t*)(rec + L.k_zero);
  const uint16_t* kbs = (const uint16_t*)(rec + L.kb_scale);
  const uint16_t* vs = (const uint16_t*)(rec + L.v_scale);
  const uint16_t* vz = (const uint16_t*)(rec + L.v_zero);
  const uint8_t* bidx = rec + L.boost_idx;
  const int kw = D / 16, kbw = k / 16;
  if (Khat) {
    for (int t = 0; t < P; ++t) {
      int g = t / G;
      for (int c = 0; c < D; ++c) {
        const int pm = key_meta_pos(c);
        unsigned a = get2(kA, t, kw, key_pos(c));
        Khat[t * D + c] = a * dt_value(ks[g * D + pm], dtype) + dt_value(kz[g * D + pm], dtype);
      }
      for (int j = 0; j < k; ++j) {
        unsigned b = get2(kB, t, kbw, boost_pos(j, kbw));
        Khat[t * D + bidx[j]] += b * dt_value(kbs[g * k + j], dtype);
      }
    }
  }
  if (Vhat) {
    for (int t = 0; t < P; ++t)
      for (int c = 0; c < D; ++c) {
        unsigned v = get2s(vq, value_slot(t, c));
        const int pv = value_meta_pos(t);
        Vhat[t * D + c] = v * dt_value(vs[pv], dtype) + dt_value(vz[pv], dtype);
      }
  }
}

/* ------------------------------------------------------------------ decode attention */

/* Decode attention for one sequence and one KV head (fp64): the quantized pages
 * listed in pages[0..n_pages) (token order) followed by res_len residual tokens;
 * q: [gqa][D] 16-bit patterns of the query heads sharing this KV head.
 *   out[h] = sum_t softmax_t(sm_scale * q_h . K^_t) V^_t
 * Two plain passes: scores over every token, then the weighted sum of values.
 * pool is the base of record (0, head) layout: record (p, head) lives at
 * pool + (p * Hkv + head) * record_bytes.  out: [gqa][D]. */
void kvqo_decode_unit(const uint8_t* pool, int Hkv, int head, const int32_t* pages, int n_pages,
                      const uint16_t* res_k, const uint16_t* res_v, int res_len,
                      const uint16_t* q, int gqa, int P, int D, int G, int k, int dtype,
                      double sm_scale, double* out) {
  layout_t L = make_layout(P, D, k, G);
  long n_tok = (long)n_pages * P + res_len;
  for (int i = 0; i < gqa * D; ++i) out[i] = 0.0;
  if (n_tok == 0) return;
  double* scores = (double*)malloc(sizeof(double) * gqa * n_tok);
  double* Kh = (double*)malloc(sizeof(double) * P * D);
  double* Vh = (double*)malloc(sizeof(double) * P * D);
  double* qd = (double*)malloc(sizeof(double) * gqa * D);
  for (int i = 0; i < gqa * D; ++i) qd[i] = dt_value(q[i], dtype);

  /* pass 1: scores */
  for (int p = 0; p < n_pages; ++p) {
    const uint8_t* rec = pool + ((long)pages[p] * Hkv + head) * L.record;
    kvqo_dequantize_page(rec, P, D, G, k, dtype, Kh, NULL);
    for (int t = 0; t < P; ++t)
      for (int h = 0; h < gqa; ++h) {
        double s = 0.0;
        for (int c = 0; c < D; ++c) s += qd[h * D + c] * Kh[t * D + c];
        scores[h * n_tok + (long)p * P + t] = s * sm_scale;
      }
  }
  for (int t = 0; t < res_len; ++t)
    for (int h = 0; h < gqa; ++h) {
      double s = 0.0;
      for (int c = 0; c < D; ++c) s += qd[h * D + c] * dt_value(res_k[(long)t * D + c], dtype);
      scores[h * n_tok + (long)n_pages * P + t] = s * sm_scale;
    }
  /* softmax with the maximum subtracted */
  for (int h = 0; h < gqa; ++h) {
    double* s = scores + (long)h * n_tok;
    double m = s[0];
    for (long t = 1; t < n_tok; ++t)
      if (s[t] > m) m = s[t];
    double l = 0.0;
    for (long t = 0; t < n_tok; ++t) {
      s[t] = exp(s[t] - m);
      l += s[t];
    }
    for (long t = 0; t < n_tok; ++t) s[t] /= l;
  }
  /* pass 2: probability-weighted values */
  for (int p = 0; p < n_pages; ++p) {
    const uint8_t* rec = pool + ((long)pages[p] * Hkv + head) * L.record;
    kvqo_dequantize_page(rec, P, D, G, k, dtype, NULL, Vh);
    for (int h = 0; h < gqa; ++h)
      for (int t = 0; t < P; ++t) {
        double pt = scores[h * n_tok + (long)p * P + t];
        for (int c = 0; c < D; ++c) out[h * D + c] += pt * Vh[t * D + c];
      }
  }
  for (int h = 0; h < gqa; ++h)
    for (int t = 0; t < res_len; ++t) {
      double pt = scores[h * n_tok + (long)n_pages * P + t];
      for (int c = 0; c < D; ++c) out[h * D + c] += pt * dt_value(res_v[(long)t * D + c], dtype);
    }
  free(scores);
  free(Kh);
  free(Vh);
  free(qd);
}

/* ------------------------------------------------------- prefill with token retention */

/* Prefill attention with cumulative attention scores (MiniKV summary on f-binder,
 * section "proposed method": the prompt is processed at prefill, the tokens to keep are
 * chosen by cumulative attention score, and a two-stage selective flash-attention
 * kernel returns the usual attention output together with those scores in linear
 * memory).  Reading: causal self-attention over the L prompt tokens; for query head h
 * (KV head h / gqa) and position i,
 *   O[i][h] = sum_{j <= i} softmax_j(sm_scale * q_i . k_j) v_j,
 * and the cumulative score of key token j of KV head kvh is the attention it receives,
 * summed over every query position and over the gqa query heads of that KV head:
 *   A[kvh][j] = sum_{h in kvh} sum_{i >= j} P_h[i][j].
 * Q: [L][Hq][D], K and V: [L][Hkv][D] 16-bit patterns; O: [L][Hq][D], A: [Hkv][L] (fp64). */
void kvqo_prefill_attention(const uint16_t* Q, const uint16_t* K, const uint16_t* V, int L, int Hq, int Hkv,
                            int D, int dtype, double sm_scale, double* O, double* A) {
  const int gqa = Hq / Hkv;
  double* s = (double*)malloc(sizeof(double) * (L > 0 ? L : 1));
  for (int i = 0; i < Hkv * L; ++i) A[i] = 0.0;
  for (int h = 0; h < Hq; ++h) {
    const int kvh = h / gqa;
    for (int i = 0; i < L; ++i) {
      double m = -INFINITY;
      for (int j = 0; j <= i; ++j) {
        double d = 0.0;
        for (int c = 0; c < D; ++c)
          d += dt_value(Q[((long)i * Hq + h) * D + c], dtype) * dt_value(K[((long)j * Hkv + kvh) * D + c], dtype);
        s[j] = d * sm_scale;
        if (s[j] > m) m = s[j];
      }
      double l = 0.0;
      for (int j = 0; j <= i; ++j) {
        s[j] = exp(s[j] - m);
        l += s[j];
      }
      double* o = O + ((long)i * Hq + h) * D;
      for (int c = 0; c < D; ++c) o[c] = 0.0;
      for (int j = 0; j <= i; ++j) {
        const double p = s[j] / l;
        A[(long)kvh * L + j] += p;
        for (int c = 0; c < D; ++c) o[c] += p * dt_value(V[((long)j * Hkv + kvh) * D + c], dtype);
      }
    }
  }
  free(s);
}

/* Token retention (MiniKV summary, "proposed method": heavy hitters by cumulative
 * attention score and a recent window, 25% of the budget each by default).  Reading:
 * the last n_recent positions are kept; among the other positions the n_heavy with the
 * highest score are kept, ties to the lower position.  Writes the kept positions in
 * ascending order and returns their number (min(L, n_recent + n_heavy)). */
int kvqo_retain(const double* A, int L, int n_heavy, int n_recent, int32_t* keep) {
  if (n_recent > L) n_recent = L;
  const int cut = L - n_recent;  /* positions [cut, L) are the recent window */
  if (n_heavy > cut) n_heavy = cut;
  char* taken = (char*)calloc(L > 0 ? L : 1, 1);
  for (int r = 0; r < n_heavy; ++r) {
    int best = -1;
    for (int j = 0; j < cut; ++j) {
      if (taken[j]) continue;
      if (best < 0 || A[j] > A[best]) best = j;  /* strict: lower position wins ties */
    }
    taken[best] = 1;
  }
  int n = 0;
  for (int j = 0; j < L; ++j)
    if (j >= cut || taken[j]) keep[n++] = j;
  free(taken);
  return n;
}
