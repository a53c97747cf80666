// kvq_decode_impl.cuh — decode attention over the paged 2-bit cache on the fifth-
// generation tensor cores (tcgen05) of sm_100a.  Kernel templates;
// kvq_decode_<dtype>_g<GQA>.cu instantiate them, kvq_decode.cu holds the host side.
//
// Workers.  A CTA holds two warpgroups of 128 threads, and each warpgroup is an
// independent worker: it owns a ring of shared-memory stages, a region of tensor
// memory, its shared-memory operand buffers and its own range of the work line.  The
// two warpgroups of a CTA never wait for one another between the prologue and the
// end of the kernel.
//
// Work line.  Every (sequence b, kv head h) is a unit; its items are its pages in
// 128-token stages (1, 2 or 4 records), then its residual tokens in pieces of 32.
// Item weights: a stage weighs 4, a residual piece kPieceWeight, and a unit's end adds
// kMergeWeight.  The units are laid end to end and the line is cut into one equal
// range per worker; a worker takes the items that start in its range.  A worker that
// ends a unit it did not see whole writes a partial softmax state; the last
// contributor of a unit merges the partials (log-sum-exp) in the same launch.
//
// Arithmetic of a 128-token page stage (thread t of the warpgroup is token t for keys
// and channel t for values; tensor-memory lane t belongs to the same thread):
//   keys   A_K[t][c]    = codes of plane A (c < 128) and plane B (c >= 128) as
//                         fp16 0.5 * code (the FP4 conversion), written to tensor memory
//          B_s[c][n]    = q'_h[c] * sA[c][g] split into fp16 (hi, lo), n = (g, part, h)
//          B_b[j][n]    = q'_h[idx(j)] * sB[j][g], the same for plane B
//          B_z[c][n]    = q'_h[c] * zA[c][g]
//          S[t][n]      = A_K x (B_s ; B_b) + 0.5 x B_z      (all fp32 in tensor memory)
//   so that 2 * (S[t][g(t), hi, h] + S[t][g(t), lo, h]) = q'_h . K^_t exactly up to fp32
//   rounding.  q' = q * 2^-e_h with e_h chosen per (unit, head) so that |q'| < 1: the
//   folded operands then never exceed the key scales (fp16 caches cannot overflow).
//   values A_V[c][t]    = 0.5 * value code of token t, channel c (tensor memory)
//          B_p[t][n]    = p_h[t] * sV[t] * 2^-F split into fp16 (hi, lo), n = (part, h)
//          O[c][n]     += A_V x B_p                          (fp32, across the unit)
//   and the value zero points and the softmax sum stay per thread:
//          zv_h += p_h[t] * zV[t],   l_h += p_h[t].
// Online softmax (log2 units) with a running maximum M_h per worker that moves only
// when a logit exceeds it by more than kLazy; then every thread rescales its own
// partial sums and its own lane of O.  F (>= 0) keeps p * sV * 2^-F below 2^15.
// Residual pieces use the raw key and value rows (cache dtype) as A with B = q'
// (exact) and B = 0.5 * p * 2^-F; their products run in the cache dtype.
//
// Synchronisation inside a worker: two warpgroup barriers per item (operands ready
// for the QK product; probabilities ready for the PV product, which also ORs the
// "maximum must move" votes), tcgen05 commits to two mbarriers, and one bulk-copy
// mbarrier per stage.  Every mbarrier wait is bounded; a timeout sets
// KVQ_DEV_ERR_TIMEOUT and the worker stops after waiting (bounded) for its copies and
// products in flight.
#pragma once
#include <algorithm>

#include "kvq_internal.cuh"
#include "kvq_tc.cuh"

namespace kvq {
namespace dec {

constexpr int kWG = 2;                   // workers (warpgroups) per CTA
constexpr int kThreads = 128 * kWG;
constexpr int kStageBytes = 16384;       // one 128-token page stage or one residual piece
constexpr int kPieceTokens = 32;         // residual tokens per piece
constexpr int kResV = 8192;              // value rows of a residual piece in its stage
constexpr int kSegItems = 64;            // items listed per segment
constexpr int kSeqCache = 512;           // sequences whose lengths the prologue keeps
constexpr float kLazy = 8.0f;            // log2 margin before the running maximum moves
constexpr int kPieceWeight = kDecodePieceWeight;
constexpr int kMergeWeight = kDecodeMergeWeight;
constexpr int kSmemPerWorker = 104 * 1024;

// Compile-time offsets of one record (the same values as make_layout).
template <int P, int KB>
struct Rec {
  static constexpr int k = 16 * KB;
  static constexpr uint32_t k_codes = 0;
  static constexpr uint32_t kb_codes = k_codes + P * 32;
  static constexpr uint32_t v_codes = kb_codes + P * KB * 4;
  static constexpr uint32_t k_scale = v_codes + P * 32;
  static constexpr uint32_t k_zero = k_scale + (P / 32) * 256;
  static constexpr uint32_t kb_scale = k_zero + (P / 32) * 256;
  static constexpr uint32_t v_scale = kb_scale + (P / 32) * k * 2;
  static constexpr uint32_t v_zero = v_scale + P * 2;
  static constexpr uint32_t boost_idx = v_zero + P * 2;
  static constexpr uint32_t payload = boost_idx + k;
  static constexpr uint32_t record = (payload + 127u) / 128u * 128u;
};

constexpr int round16(int x) { return (x + 15) / 16 * 16; }
constexpr int cmax(int a, int b) { return a > b ? a : b; }
constexpr int cmin(int a, int b) { return a < b ? a : b; }

// Shapes, tensor-memory columns and shared-memory offsets of one instantiation.
template <int GQA, int KB, int P>
struct Cfg {
  static constexpr int PPS = 128 / P;                  // pages per stage
  static constexpr int NG = P / 32;                    // key groups per page
  static constexpr int NQK = cmax(16, 8 * GQA);        // QK columns: 4 groups x (hi, lo) x heads
  static constexpr int LBO_QK = NQK / 8 * 128;
  static constexpr int LBO_PV = 256;                   // PV / residual-QK B operands: N = 16
  static constexpr int AQ = 64 + 8 * KB;               // key A columns
  static constexpr int AV = 64;                        // value A columns
  static constexpr int COLS_SPLIT = round16(AQ + AV + NQK + 16);
  static constexpr bool SPLIT = 16 + kWG * COLS_SPLIT <= 512;  // separate key and value A regions
  static constexpr int COLS = SPLIT ? COLS_SPLIT : round16(cmax(AQ, AV) + NQK + 16);
  static constexpr int C_AQ = 0, C_AV = SPLIT ? AQ : 0, C_S = SPLIT ? AQ + AV : cmax(AQ, AV), C_O = C_S + NQK;
  static_assert(16 + kWG * COLS <= 512, "tensor memory");
  // shared memory of one worker
  static constexpr int BQK = 128 * NQK * 2;
  static constexpr int BQB = 16 * KB * NQK * 2;
  static constexpr int FIXED = 2 * BQK + BQB + 4096 + 4096 + 128 * GQA * 2;
  static constexpr int NS = cmin(4, (kSmemPerWorker - FIXED) / (kStageBytes + GQA * 256));
  static_assert(NS >= 2, "shared memory");
  static constexpr int O_RING = 0;
  static constexpr int O_Q = O_RING + NS * kStageBytes;
  static constexpr int O_BQK = O_Q + NS * GQA * 256;
  static constexpr int O_BZ = O_BQK + BQK;
  static constexpr int O_BQB = O_BZ + BQK;
  static constexpr int O_BPV = O_BQB + BQB;
  static constexpr int O_BQR = O_BPV + 4096;
  static constexpr int O_QH = O_BQR + 4096;
  static constexpr int BYTES = (O_QH + 128 * GQA * 2 + 1023) / 1024 * 1024;
  static_assert(BYTES <= kSmemPerWorker, "shared memory");
};

// ---------------------------------------------------------------- small helpers

__device__ __forceinline__ void wg_sync(int wg) { asm volatile("bar.sync %0, 128;" ::"r"(wg + 1) : "memory"); }
// Barrier of the warpgroup that also returns the OR of `pred` over its threads.
__device__ __forceinline__ bool wg_sync_or(int wg, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, 128, p;\n\tselp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(wg + 1)
      : "memory");
  return r != 0;
}

__device__ __forceinline__ uint32_t u16_at(const uint8_t* p) { return *reinterpret_cast<const uint16_t*>(p); }

// A 16-bit value of the cache dtype as fp32 (exact).
__device__ __forceinline__ float t_to_f(uint32_t b, __half) { return __half2float(__ushort_as_half(uint16_t(b))); }
__device__ __forceinline__ float t_to_f(uint32_t b, __nv_bfloat16) { return __uint_as_float(b << 16); }
// A 16-bit value of the cache dtype as an fp16 pair (x, x): exact for fp16; for bf16
// exact inside fp16's normal range.
__device__ __forceinline__ uint32_t t_bcast_h2(uint32_t b, __half) { return (b & 0xffffu) | (b << 16); }
__device__ __forceinline__ uint32_t t_bcast_h2(uint32_t b, __nv_bfloat16) {
  const float x = __uint_as_float(b << 16);
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(x));
  return d;
}
// Two floats as a pair of the given 16-bit type (low half = a).
__device__ __forceinline__ uint32_t pack2(float a, float b, __half) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}
__device__ __forceinline__ uint32_t pack2(float a, float b, __nv_bfloat16) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(b), "f"(a));
  return d;
}
__device__ __forceinline__ float2 unpack2(uint32_t u, __half) { return __half22float2(u32_as_h2(u)); }
__device__ __forceinline__ float2 unpack2(uint32_t u, __nv_bfloat16) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
// (hi, lo) pairs of (a, b) in the 16-bit type U: hi = U(x), lo = U(x - hi).
template <typename U>
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack2(a, b, U());
  const float2 h = unpack2(hi, U());
  lo = pack2(a - h.x, b - h.y, U());
}
// Products q * s of an fp16 query pair and a broadcast fp16 scale, as (hi, lo) fp16
// pairs: hi = fp16(q s), lo = q s - hi (exact: the rest of a product of two fp16 values).
__device__ __forceinline__ void fold2(uint32_t q2, uint32_t s2, uint32_t& hi, uint32_t& lo) {
  const __half2 q = u32_as_h2(q2), s = u32_as_h2(s2);
  const __half2 h = __hmul2(q, s);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__hfma2(q, s, __hneg2(h)));
}
__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // e in [-126, 127]

// Folded operand row of one key group: GQA heads x (hi, lo) as GQA 32-bit words.
// Layout n = part * GQA + h (GQA >= 2: hi pairs then lo pairs); GQA 1: (hi, lo).
template <int GQA>
struct GroupRow {
  uint32_t w[GQA];
};
template <int GQA>
__device__ __forceinline__ GroupRow<GQA> fold_group(const uint32_t (&q2)[(GQA + 1) / 2], uint32_t s2) {
  GroupRow<GQA> r;
  if constexpr (GQA == 1) {
    uint32_t hi, lo;
    fold2(q2[0], s2, hi, lo);
    r.w[0] = (hi & 0xffffu) | (lo << 16);
  } else {
#pragma unroll
    for (int i = 0; i < GQA / 2; ++i) fold2(q2[i], s2, r.w[i], r.w[GQA / 2 + i]);
  }
  return r;
}
// Stores the four group rows of one K-row (channel or boosted row) of a QK B operand:
// the GQA words of group g start at column 2 * GQA * g.
template <int GQA, int LBO>
__device__ __forceinline__ void store_qk_row(uint8_t* B, int row, const GroupRow<GQA> (&g)[4]) {
  uint32_t v[4 * GQA];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < GQA; ++j) v[GQA * i + j] = g[i].w[j];
  uint8_t* base = B + (row >> 3) * LBO + (row & 7) * 16;
#pragma unroll
  for (int c = 0; c < GQA; ++c)
    *reinterpret_cast<uint4*>(base + c * 128) = make_uint4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
}
// Stores one K-row of an N = 16 B operand (probabilities or the residual query):
// `words` 32-bit words (2 * words values) from column 0 on; the other columns are zero.
template <int NW>
__device__ __forceinline__ void store_n16_row(uint8_t* B, int row, const uint32_t (&v)[NW]) {
  uint8_t* base = B + (row >> 3) * 256 + (row & 7) * 16;
  if constexpr (NW <= 4) {
    uint32_t x[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < NW; ++i) x[i] = v[i];
    *reinterpret_cast<uint4*>(base) = make_uint4(x[0], x[1], x[2], x[3]);
  } else {
    *reinterpret_cast<uint4*>(base) = make_uint4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<uint4*>(base + 128) = make_uint4(v[4], v[5], v[6], v[7]);
  }
}

// Converts one code word (16 codes) to 8 tensor-memory columns of fp16 pairs, in
// natural element order: column 4a + b holds elements 8a + 2b (low) and 8a + 2b + 1.
__device__ __forceinline__ void word_to_cols(uint32_t w, uint32_t* c) {
  e2m1_pairs(code_pass(w, 0), c[0], c[1], c[2], c[3]);
  e2m1_pairs(code_pass(w, 1), c[4], c[5], c[6], c[7]);
}

// ---------------------------------------------------------------- work line

struct Cursor {
  int b, h, k;
  int np, rl, nst, nres;  // pages, residual tokens, page stages, residual pieces of b
  int s, ubase;           // start weight of item k and of the unit
};

template <int P>
__device__ __forceinline__ int unit_weight_of(int np, int rl) {
  const int items = np * (P / 32) + kPieceWeight * ((rl + kPieceTokens - 1) / kPieceTokens);
  return items > 0 ? items + kMergeWeight : 0;
}

// Unit weight of sequence b (-1 when its lengths are invalid), with its pages and
// residual tokens (0 when invalid).
template <int P>
__device__ __forceinline__ int seq_weight(const DecodeParams& p, int b, int& np, int& rl) {
  np = __ldcg(p.num_pages + b);
  rl = __ldcg(p.res_len + b);
  if (np < 0 || np > p.max_pages || rl < 0 || rl > P) {
    np = 0;
    rl = 0;
    return -1;
  }
  return unit_weight_of<P>(np, rl);
}

template <int P>
__device__ __forceinline__ int unit_weight(const Cursor& c) {
  return unit_weight_of<P>(c.np, c.rl);
}

__device__ __forceinline__ int owner_of(int s, int W, int C) { return int(floor(double(s) * C / W)); }
__device__ __forceinline__ int range_start(int i, int W, int C) { return int(ceil(double(W) * i / C)); }

// Partial softmax state of one (worker, unit) slot and head: unnormalised output [128],
// then the maximum and the sum (floats 128, 129), padded to 16 bytes.
constexpr int kPartStride = kHeadDim + 4;

enum : uint32_t { kDescRes = 1u << 8, kDescFirst = 1u << 9, kDescLast = 1u << 10 };

struct ItemDesc {
  uint32_t w;   // bits 0-7: pages in the stage or residual tokens; kDescRes, kDescFirst,
                // kDescLast; bits 16-31: stage or piece index within the unit
  int b, h;
  uint32_t io;  // first and last contributing worker of the unit (low, high 16 bits)
};

struct UnitSpan {
  int off, b, h, k0, n, np, rl, first, last;
  uint32_t io;
};

// Lengths the prologue keeps for the whole CTA.
struct CtaCtl {
  uint32_t tmem;
  int red[kThreads / 32];
  int2 seq[kSeqCache];   // (pages, residual tokens) of sequence b (b < kSeqCache)
  int b0[kWG], base0[kWG];
};

// Control state of one worker.
template <int P>
struct WgCtl {
  uint64_t full[4];
  uint64_t bar_s, bar_pv;
  Cursor cur;
  int nseg, more, nspan, issued, abort_flag;
  float red[4][24];
  UnitSpan span[16];
  ItemDesc desc[kSegItems];
  int ids[kSegItems][128 / P];
};

// Pages and residual tokens of sequence b (from the CTA cache when it holds b).
template <int P>
__device__ __forceinline__ int seq_info(const DecodeParams& p, const CtaCtl& cc, int b, int& np, int& rl) {
  if (b < kSeqCache) {
    const int2 v = cc.seq[b];
    np = v.x;
    rl = v.y;
    return unit_weight_of<P>(np, rl);
  }
  return max(0, seq_weight<P>(p, b, np, rl));
}

template <int P>
__device__ __forceinline__ void cursor_load_seq(const DecodeParams& p, const CtaCtl& cc, Cursor& c) {
  while (c.b < p.batch && seq_info<P>(p, cc, c.b, c.np, c.rl) == 0) ++c.b;
  if (c.b >= p.batch) c.np = c.rl = 0;
  c.nst = (c.np * P + 127) / 128;
  c.nres = (c.rl + kPieceTokens - 1) / kPieceTokens;
}

// Moves the cursor from offset `ou` of its unit to the first item that starts at or
// after it, or to the first item of the next unit.
template <int P>
__device__ __forceinline__ void cursor_seek(const DecodeParams& p, const CtaCtl& cc, Cursor& c, int ou) {
  if (c.nst > 0 && ou <= 4 * (c.nst - 1)) {
    c.k = (ou + 3) / 4;
    c.s = c.ubase + 4 * c.k;
    return;
  }
  const int j = max(0, (ou - c.np * (P / 32) + kPieceWeight - 1) / kPieceWeight);
  if (j < c.nres) {
    c.k = c.nst + j;
    c.s = c.ubase + c.np * (P / 32) + kPieceWeight * j;
    return;
  }
  c.s = c.ubase + unit_weight<P>(c);
  c.ubase = c.s;
  c.k = 0;
  if (++c.h < p.Hkv) return;
  c.h = 0;
  ++c.b;
  cursor_load_seq<P>(p, cc, c);
}

// Lists the next segment of the worker's items (all 128 threads of the worker).
template <int P>
__device__ __forceinline__ void build_segment(const DecodeParams& p, const CtaCtl& cc, WgCtl<P>& wc, int hi,
                                              int W, int C, int wt, int wg, bool worker_first) {
  constexpr int PPC = 128 / P, GPP = P / 32;
  if (wt == 0) {
    Cursor c = wc.cur;
    int n = 0, ns = 0;
    while (c.s < hi && n < kSegItems && ns < 16) {
      const int nitems = c.nst + c.nres;
      int kend = nitems;
      const int kst = min(c.nst, max(0, hi - c.ubase + 3) / 4);
      if (kst < c.nst) {
        kend = kst;
      } else {
        const int r0 = c.ubase + c.np * GPP;
        kend = c.nst + min(c.nres, max(0, (hi - r0 + kPieceWeight - 1) / kPieceWeight));
      }
      const int cnt = min(kend - c.k, kSegItems - n);
      UnitSpan& sp = wc.span[ns];
      sp.off = n;
      sp.b = c.b;
      sp.h = c.h;
      sp.k0 = c.k;
      sp.n = cnt;
      sp.np = c.np;
      sp.rl = c.rl;
      sp.first = (c.k == 0) || (worker_first && n == 0);
      sp.last = (c.k + cnt == kend);
      const int uw = unit_weight<P>(c);
      const int last_start =
          c.ubase + uw - kMergeWeight - (c.nres > 0 ? kPieceWeight : (c.np - (c.nst - 1) * PPC) * GPP);
      sp.io = uint32_t(owner_of(c.ubase, W, C)) | (uint32_t(owner_of(last_start, W, C)) << 16);
      n += cnt;
      ++ns;
      c.k += cnt;
      worker_first = false;
      if (c.k == nitems) {
        c.s = c.ubase + uw;
        c.ubase = c.s;
        c.k = 0;
        if (++c.h == p.Hkv) {
          c.h = 0;
          ++c.b;
          cursor_load_seq<P>(p, cc, c);
        }
      } else if (c.k == kend) {
        c.s = hi;  // the range ends inside this unit
      } else {
        c.s = c.ubase + (c.k < c.nst ? 4 * c.k : c.np * GPP + kPieceWeight * (c.k - c.nst));
      }
    }
    wc.cur = c;
    wc.nseg = n;
    wc.nspan = ns;
    wc.more = c.s < hi;
  }
  wg_sync(wg);
  const int n = wc.nseg, ns = wc.nspan;
  for (int t = wt; t < n; t += 128) {
    int si = 0;
    while (si + 1 < ns && wc.span[si + 1].off <= t) ++si;
    const UnitSpan& sp = wc.span[si];
    const int k = sp.k0 + (t - sp.off);
    const int nst = (sp.np * P + 127) / 128;
    ItemDesc d;
    d.b = sp.b;
    d.h = sp.h;
    d.io = sp.io;
    uint32_t w = 0;
    if (sp.first && t == sp.off) w |= kDescFirst;
    if (sp.last && t == sp.off + sp.n - 1) w |= kDescLast;
    if (k < nst) {
      const int npg = min(PPC, sp.np - k * PPC);
      w |= uint32_t(npg) | (uint32_t(k) << 16);
      for (int i = 0; i < npg; ++i) {
        int id = __ldcg(p.page_table + size_t(sp.b) * p.max_pages + k * PPC + i);
        if (id < 0 || id >= p.pool_pages) {
          flag_error(p.err, KVQ_DEV_ERR_PAGE_RANGE);
          id = 0;
        }
        wc.ids[t][i] = id;
      }
    } else {
      const int j = k - nst;
      w |= uint32_t(min(kPieceTokens, sp.rl - kPieceTokens * j)) | kDescRes | (uint32_t(j) << 16);
    }
    d.w = w;
    wc.desc[t] = d;
  }
  wg_sync(wg);
}

// Issues the copies of segment item t (global item number x) into stage x % NS: the
// page records or the residual rows, and the unit's query heads with its first item.
// One thread.
template <int GQA, int KB, int P>
__device__ __forceinline__ void issue_item(const DecodeParams& p, WgCtl<P>& wc, uint8_t* ws, int x, int t,
                                           uint64_t policy) {
  using R = Rec<P, KB>;
  using C = Cfg<GQA, KB, P>;
  const ItemDesc d = wc.desc[t];
  const int st = x % C::NS, n = d.w & 0xff;
  const bool res = d.w & kDescRes, first = d.w & kDescFirst;
  uint8_t* sb = ws + C::O_RING + st * kStageBytes;
  const uint32_t bytes = (res ? 2u * uint32_t(n) * 256u : uint32_t(n) * R::payload) + (first ? GQA * 256u : 0u);
  tc::fence_async_smem();
  mbar_arrive_expect_tx(&wc.full[st], bytes);
  if (!res) {
    for (int i = 0; i < n; ++i)
      bulk_g2s(sb + i * R::record, p.pool + (size_t(wc.ids[t][i]) * p.Hkv + d.h) * R::record, R::payload,
               &wc.full[st], policy);
  } else {
    const size_t row0 = (size_t(d.b) * p.Hkv + d.h) * P + size_t(kPieceTokens) * (d.w >> 16);
    bulk_g2s(sb, p.res_k + row0 * kHeadDim, uint32_t(n) * 256u, &wc.full[st], policy);
    bulk_g2s(sb + kResV, p.res_v + row0 * kHeadDim, uint32_t(n) * 256u, &wc.full[st], policy);
  }
  if (first) {
    const uint16_t* src = p.q + (size_t(d.b) * p.Hq + size_t(d.h) * GQA) * kHeadDim;
    bulk_g2s(ws + C::O_Q + st * GQA * 256, src, GQA * 256u, &wc.full[st], policy);
  }
  ++wc.issued;
}

// Merges heads h0 .. h0 + HC - 1 of the nc partial states at pu (log-sum-exp) into outu.
// One warp; lane i holds channels 4i .. 4i + 3.
template <int HC>
__device__ __forceinline__ void merge_heads(const float* pu, size_t slot, int nc, int h0, float* outu, int lane) {
  float Mh[HC], Lh[HC];
  float4 Oh[HC];
#pragma unroll
  for (int h = 0; h < HC; ++h) Mh[h] = -INFINITY;
  for (int i = lane; i < nc; i += 32)
#pragma unroll
    for (int h = 0; h < HC; ++h) Mh[h] = fmaxf(Mh[h], __ldcg(pu + i * slot + (h0 + h) * kPartStride + kHeadDim));
#pragma unroll
  for (int h = 0; h < HC; ++h) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) Mh[h] = fmaxf(Mh[h], __shfl_xor_sync(kFull, Mh[h], off));
    Lh[h] = 0.0f;
    Oh[h] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll 4
  for (int i = 0; i < nc; ++i) {
    const float* pi = pu + i * slot + h0 * kPartStride;
    float mi[HC], li[HC];
    float4 oi[HC];
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      mi[h] = __ldcg(pi + h * kPartStride + kHeadDim);
      li[h] = __ldcg(pi + h * kPartStride + kHeadDim + 1);
      oi[h] = __ldcg(reinterpret_cast<const float4*>(pi + h * kPartStride) + lane);
    }
#pragma unroll
    for (int h = 0; h < HC; ++h) {
      const float f = Mh[h] == -INFINITY ? 0.0f : ex2(mi[h] - Mh[h]);
      Lh[h] += f * li[h];
      Oh[h].x += f * oi[h].x;
      Oh[h].y += f * oi[h].y;
      Oh[h].z += f * oi[h].z;
      Oh[h].w += f * oi[h].w;
    }
  }
#pragma unroll
  for (int h = 0; h < HC; ++h) {
    const float inv = Lh[h] > 0.0f ? 1.0f / Lh[h] : 0.0f;
    reinterpret_cast<float4*>(outu + (h0 + h) * kHeadDim)[lane] =
        make_float4(Oh[h].x * inv, Oh[h].y * inv, Oh[h].z * inv, Oh[h].w * inv);
  }
}

__device__ __forceinline__ uint32_t atomic_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}

// ---------------------------------------------------------------- one worker

// Per-thread softmax state of the current unit.
template <int GQA>
struct State {
  float M[GQA];   // running maximum (log2 units), the same in every thread of the worker
  float l[GQA];   // this thread's share of the softmax sum
  float zv[GQA];  // this thread's share of sum p * value zero point
  int F;          // value-operand exponent
  float vlim;     // 2^(7 + F): value scales at or above it need a larger F
  float fsc;      // 2^-F
  bool pv;        // O holds products of this unit
};

template <typename T, int GQA, int KB, int P>
__device__ __forceinline__ void worker_run(const DecodeParams& p, const CtaCtl& cc, WgCtl<P>& wc, uint8_t* ws,
                                           uint32_t tmem, int W, int Cw, int worker, int wg, int wt) {
  using R = Rec<P, KB>;
  using C = Cfg<GQA, KB, P>;
  constexpr bool BF = std::is_same<T, __nv_bfloat16>::value;
  constexpr int NQ2 = (GQA + 1) / 2;
  constexpr uint32_t ID_QK = tc::idesc_f16(C::NQK, false);
  constexpr uint32_t ID_PV = tc::idesc_f16(16, false);
  constexpr uint32_t ID_RES = tc::idesc_f16(16, BF);
  const int wwarp = wt >> 5, lane = wt & 31;
  const uint32_t tbase = tmem + 16 + uint32_t(wg * C::COLS);  // this worker's columns
  const uint32_t tl = tc::lane_addr(tbase, wwarp, 0);          // this thread's lane quarter
  const uint32_t t_ones = tmem;                                // columns 0..7: fp16 0.5
  uint8_t* const bqk = ws + C::O_BQK;
  uint8_t* const bz = ws + C::O_BZ;
  uint8_t* const bqb = ws + C::O_BQB;
  uint8_t* const bpv = ws + C::O_BPV;
  uint8_t* const bqr = ws + C::O_BQR;
  uint16_t* const qh = reinterpret_cast<uint16_t*>(ws + C::O_QH);
  const uint32_t a_bqk = smem_addr(bqk), a_bz = smem_addr(bz), a_bqb = smem_addr(bqb), a_bpv = smem_addr(bpv),
                 a_bqr = smem_addr(bqr);
  const uint64_t policy = l2_evict_first_policy();
  const int lo = range_start(worker, W, Cw), hi = range_start(worker + 1, W, Cw);

  // locate the first item: the prologue found the sequence holding position lo
  if (wt == 0) {
    Cursor c;
    c.b = cc.b0[wg];
    seq_info<P>(p, cc, c.b, c.np, c.rl);
    c.nst = (c.np * P + 127) / 128;
    c.nres = (c.rl + kPieceTokens - 1) / kPieceTokens;
    c.k = 0;
    const int wseq = unit_weight<P>(c);
    const int off = lo - cc.base0[wg];
    c.h = off / wseq;
    c.ubase = cc.base0[wg] + c.h * wseq;
    cursor_seek<P>(p, cc, c, off - c.h * wseq);
    wc.cur = c;
    wc.issued = 0;
    wc.abort_flag = 0;
  }
  wg_sync(wg);

  State<GQA> stt;
  uint32_t q2[NQ2];    // this thread's channel of q' as fp16 pairs (heads 2i, 2i + 1)
  float cq[GQA], cr[GQA];  // logit factors: pages (2 * c * 2^e), residual (c * 2^e)
  int x = 0;               // items of this worker so far
  uint32_t ps = 0, ppv = 0;  // parities of bar_s and bar_pv
  bool pv_pending = false;   // a PV product was issued and not yet waited for
  bool worker_first = true;
  bool failed = false;

  auto wait_pv = [&]() {
    if (pv_pending) {
      if (!mbar_wait_bounded(&wc.bar_pv, ppv)) failed = true;
      __syncwarp();
      ppv ^= 1u;
      pv_pending = false;
    }
  };

  while (true) {
    build_segment<P>(p, cc, wc, hi, W, Cw, wt, wg, worker_first);
    worker_first = false;
    const int nseg = wc.nseg;
    if (wt == 0)
      for (int t = 0; t < min(C::NS, nseg); ++t) issue_item<GQA, KB, P>(p, wc, ws, x + t, t, policy);
    for (int t = 0; t < nseg; ++t) {
      const int xi = x + t, st = xi % C::NS;
      const uint32_t par = uint32_t(xi / C::NS) & 1u;
      const ItemDesc d = wc.desc[t];
      const uint8_t* sb = ws + C::O_RING + st * kStageBytes;
      const bool res = d.w & kDescRes;
      const int n = d.w & 0xff;
      if (!mbar_wait_bounded(&wc.full[st], par)) failed = true;
      __syncwarp();

      // ---------------------------------------------------------- unit start
      if (d.w & kDescFirst) {
        const uint8_t* qs = ws + C::O_Q + st * GQA * 256;
        float qf[GQA];
#pragma unroll
        for (int h = 0; h < GQA; ++h) qf[h] = t_to_f(u16_at(qs + h * 256 + 2 * wt), T());
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          const uint32_t mb = __reduce_max_sync(kFull, __float_as_uint(fabsf(qf[h])));
          if (lane == 0) wc.red[wwarp][h] = __uint_as_float(mb);
        }
        wg_sync(wg);
        float qp[GQA];
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          const float m = fmaxf(fmaxf(wc.red[0][h], wc.red[1][h]), fmaxf(wc.red[2][h], wc.red[3][h]));
          // |q'| = |q| * 2^-e < 1; e kept inside the normal exponent range
          int e = m > 0.0f ? int((__float_as_uint(m) >> 23) & 0xff) - 126 : 0;
          e = min(max(e, -125), 125);
          qp[h] = qf[h] * pow2f(-e);
          cq[h] = 2.0f * p.c_log2 * pow2f(e);
          cr[h] = p.c_log2 * pow2f(e);
        }
        if constexpr (GQA == 1) {
          q2[0] = pack2(qp[0], 0.0f, __half());
        } else {
#pragma unroll
          for (int i = 0; i < GQA / 2; ++i) q2[i] = pack2(qp[2 * i], qp[2 * i + 1], __half());
        }
        // q' in fp16 for the plane-B gathers, in the cache dtype for the residual product
#pragma unroll
        for (int h = 0; h < GQA; ++h) qh[wt * GQA + h] = __half_as_ushort(__float2half_rn(qp[h]));
        {
          uint32_t v[(GQA + 1) / 2];
          if constexpr (GQA == 1) {
            v[0] = pack2(qp[0], 0.0f, T());
          } else {
#pragma unroll
            for (int i = 0; i < GQA / 2; ++i) v[i] = pack2(qp[2 * i], qp[2 * i + 1], T());
          }
          store_n16_row(bqr, wt, v);
        }
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          stt.M[h] = -INFINITY;
          stt.l[h] = 0.0f;
          stt.zv[h] = 0.0f;
        }
        stt.F = 0;
        stt.vlim = 128.0f;
        stt.fsc = 1.0f;
        stt.pv = false;
        tc::fence_async_smem();
        wg_sync(wg);  // q' visible to every thread (plane B) and, through the fence, to the products
      }

      float L[GQA];     // this thread's token logits (log2 units), -inf when masked
      float sv = 0.0f;  // value scale of the token (pages)
      float zvt = 0.0f; // value zero point of the token (pages)
      bool valid;
      if (!res) {
        // ---------------------------------------------------------- page stage
        const int npg = n;
        const int r_t = wt / P, tk = wt % P;  // record and token of this thread's token
        valid = r_t < npg;
        if (!C::SPLIT) wait_pv();  // the value product still reads the shared A region
        {
          // keys of token wt: plane A words (two blocks of four), plane B words
          const uint8_t* rk = sb + r_t * R::record;
          const uint4 a0 = lds128(rk + R::k_codes + 16 * tk);
          const uint4 a1 = lds128(rk + R::k_codes + 16 * P + 16 * tk);
          uint32_t cv[32];
          word_to_cols(a0.x, cv);
          word_to_cols(a0.y, cv + 8);
          word_to_cols(a0.z, cv + 16);
          word_to_cols(a0.w, cv + 24);
          tc::st<32>(tl + C::C_AQ, cv);
          word_to_cols(a1.x, cv);
          word_to_cols(a1.y, cv + 8);
          word_to_cols(a1.z, cv + 16);
          word_to_cols(a1.w, cv + 24);
          tc::st<32>(tl + C::C_AQ + 32, cv);
          if constexpr (KB == 1) {
            uint32_t cb[8];
            word_to_cols(lds32(rk + R::kb_codes + 4 * tk), cb);
            tc::st<8>(tl + C::C_AQ + 64, cb);
          } else if constexpr (KB == 2) {
            const uint2 b0 = lds64(rk + R::kb_codes + 8 * tk);
            uint32_t cb[16];
            word_to_cols(b0.x, cb);
            word_to_cols(b0.y, cb + 8);
            tc::st<16>(tl + C::C_AQ + 64, cb);
          } else if constexpr (KB >= 4) {
#pragma unroll
            for (int blk = 0; blk < KB / 4; ++blk) {
              const uint4 b0 = lds128(rk + R::kb_codes + blk * 16 * P + 16 * tk);
              word_to_cols(b0.x, cv);
              word_to_cols(b0.y, cv + 8);
              word_to_cols(b0.z, cv + 16);
              word_to_cols(b0.w, cv + 24);
              tc::st<32>(tl + C::C_AQ + 64 + 32 * blk, cv);
            }
          }
        }
        {
          // folded query of channel wt: plane-A scales and zero points, 4 groups
          uint32_t sbits[4], zbits[4];
          if constexpr (P == 128) {
            const uint2 s = lds64(sb + R::k_scale + 8 * wt), z = lds64(sb + R::k_zero + 8 * wt);
            sbits[0] = s.x; sbits[1] = s.x >> 16; sbits[2] = s.y; sbits[3] = s.y >> 16;
            zbits[0] = z.x; zbits[1] = z.x >> 16; zbits[2] = z.y; zbits[3] = z.y >> 16;
          } else if constexpr (P == 64) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const uint32_t s = lds32(sb + r * R::record + R::k_scale + 4 * wt);
              const uint32_t z = lds32(sb + r * R::record + R::k_zero + 4 * wt);
              sbits[2 * r] = s; sbits[2 * r + 1] = s >> 16;
              zbits[2 * r] = z; zbits[2 * r + 1] = z >> 16;
            }
          } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              sbits[r] = u16_at(sb + r * R::record + R::k_scale + 2 * wt);
              zbits[r] = u16_at(sb + r * R::record + R::k_zero + 2 * wt);
            }
          }
          GroupRow<GQA> gs[4], gz[4];
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            // groups of records past the stage's pages hold stale bytes: zero operands
            const bool gv = (g / C::NG) < npg;
            gs[g] = fold_group<GQA>(q2, gv ? t_bcast_h2(sbits[g] & 0xffffu, T()) : 0u);
            gz[g] = fold_group<GQA>(q2, gv ? t_bcast_h2(zbits[g] & 0xffffu, T()) : 0u);
          }
          store_qk_row<GQA, C::LBO_QK>(bqk, wt, gs);
          store_qk_row<GQA, C::LBO_QK>(bz, wt, gz);
        }
        if constexpr (KB > 0) {
          if (wt < 16 * KB) {
            // plane B: boosted row wt of each record, with that record's channel index
            GroupRow<GQA> gb[4];
#pragma unroll
            for (int r = 0; r < C::PPS; ++r) {
              const uint8_t* rr = sb + r * R::record;
              const bool rv = r < npg;
              const int ch = rv ? (rr[R::boost_idx + wt] & 127) : 0;
              uint32_t qb[NQ2];
              if constexpr (GQA == 1) {
                qb[0] = qh[ch];
              } else if constexpr (GQA == 2) {
                qb[0] = lds32(qh + 2 * ch);
              } else if constexpr (GQA == 4) {
                const uint2 v = lds64(qh + 4 * ch);
                qb[0] = v.x;
                qb[1] = v.y;
              } else {
                const uint4 v = lds128(qh + 8 * ch);
                qb[0] = v.x;
                qb[1] = v.y;
                qb[2] = v.z;
                qb[3] = v.w;
              }
#pragma unroll
              for (int g2 = 0; g2 < C::NG; ++g2) {
                const uint32_t sbb = rv ? u16_at(rr + R::kb_scale + (wt * C::NG + g2) * 2) : 0u;
                gb[r * C::NG + g2] = fold_group<GQA>(qb, rv ? t_bcast_h2(sbb, T()) : 0u);
              }
            }
            store_qk_row<GQA, C::LBO_QK>(bqb, wt, gb);
          }
        }
        tc::wait_st();
        tc::fence_async_smem();
        tc::fence_before();
        failed = wg_sync_or(wg, failed);
        if (failed) break;
        if (wt == 0) {
          tc::fence_after();
          const uint32_t dS = tbase + C::C_S;
#pragma unroll
          for (int s = 0; s < 8; ++s)
            tc::mma(dS, tbase + C::C_AQ + 8 * s, tc::smem_desc(a_bqk + s * 2 * C::LBO_QK, C::LBO_QK, 128), ID_QK,
                    s > 0);
#pragma unroll
          for (int s = 0; s < KB; ++s)
            tc::mma(dS, tbase + C::C_AQ + 64 + 8 * s, tc::smem_desc(a_bqb + s * 2 * C::LBO_QK, C::LBO_QK, 128),
                    ID_QK, 1);
#pragma unroll
          for (int s = 0; s < 8; ++s)
            tc::mma(dS, t_ones, tc::smem_desc(a_bz + s * 2 * C::LBO_QK, C::LBO_QK, 128), ID_QK, 1);
          tc::commit(&wc.bar_s);
        }
        if (!mbar_wait_bounded(&wc.bar_s, ps)) failed = true;
        __syncwarp();
        ps ^= 1u;
        tc::fence_after();
        // logits of token wt: its group's columns (group = warp of the worker)
        uint32_t sr[2 * GQA];
        if constexpr (GQA == 4) {
          tc::ld<8>(tl + C::C_S + wwarp * 8, sr);
        } else if constexpr (GQA == 8) {
          tc::ld<16>(tl + C::C_S + wwarp * 16, sr);
        } else if constexpr (GQA == 2) {
          tc::ld<4>(tl + C::C_S + wwarp * 4, sr);
        } else {
          tc::ld<2>(tl + C::C_S + wwarp * 2, sr);
        }
        // values of channel wt -> A_V (after the previous value product has finished)
        if (C::SPLIT) wait_pv();
        {
          uint32_t cv[32];
          if constexpr (P == 128) {
            const uint4 v0 = lds128(sb + R::v_codes + 16 * wt), v1 = lds128(sb + R::v_codes + 2048 + 16 * wt);
            word_to_cols(v0.x, cv);
            word_to_cols(v0.y, cv + 8);
            word_to_cols(v0.z, cv + 16);
            word_to_cols(v0.w, cv + 24);
            tc::st<32>(tl + C::C_AV, cv);
            word_to_cols(v1.x, cv);
            word_to_cols(v1.y, cv + 8);
            word_to_cols(v1.z, cv + 16);
            word_to_cols(v1.w, cv + 24);
            tc::st<32>(tl + C::C_AV + 32, cv);
          } else if constexpr (P == 64) {
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const uint4 v0 = lds128(sb + r * R::record + R::v_codes + 16 * wt);
              word_to_cols(v0.x, cv);
              word_to_cols(v0.y, cv + 8);
              word_to_cols(v0.z, cv + 16);
              word_to_cols(v0.w, cv + 24);
              tc::st<32>(tl + C::C_AV + 32 * r, cv);
            }
          } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const uint2 v0 = lds64(sb + r * R::record + R::v_codes + 8 * wt);
              uint32_t c16[16];
              word_to_cols(v0.x, c16);
              word_to_cols(v0.y, c16 + 8);
              tc::st<16>(tl + C::C_AV + 16 * r, c16);
            }
          }
        }
        // the token's value scale and zero point
        {
          const uint8_t* rv = sb + r_t * R::record;
          sv = valid ? t_to_f(u16_at(rv + R::v_scale + 2 * tk), T()) : 0.0f;
          zvt = valid ? t_to_f(u16_at(rv + R::v_zero + 2 * tk), T()) : 0.0f;
        }
        tc::wait_ld();
#pragma unroll
        for (int h = 0; h < GQA; ++h)
          L[h] = valid ? (__uint_as_float(sr[h]) + __uint_as_float(sr[GQA + h])) * cq[h] : -INFINITY;
      } else {
        // ---------------------------------------------------------- residual piece
        valid = wt < n;
        if (!C::SPLIT) wait_pv();
        if (wwarp == 0) {
          // key row `lane` of the piece (rows >= n are stale and masked below)
          const uint8_t* kr = sb + lane * 256;
          uint32_t cv[32];
#pragma unroll
          for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint4 v = lds128(kr + half * 128 + 16 * i);
              cv[4 * i] = v.x;
              cv[4 * i + 1] = v.y;
              cv[4 * i + 2] = v.z;
              cv[4 * i + 3] = v.w;
            }
            tc::st<32>(tl + C::C_AQ + 32 * half, cv);
          }
        }
        tc::wait_st();
        tc::fence_before();
        failed = wg_sync_or(wg, failed);
        if (failed) break;
        if (wt == 0) {
          tc::fence_after();
#pragma unroll
          for (int s = 0; s < 8; ++s)
            tc::mma(tbase + C::C_S, tbase + C::C_AQ + 8 * s, tc::smem_desc(a_bqr + s * 512, 256, 128), ID_RES, s > 0);
          tc::commit(&wc.bar_s);
        }
        if (!mbar_wait_bounded(&wc.bar_s, ps)) failed = true;
        __syncwarp();
        ps ^= 1u;
        tc::fence_after();
        uint32_t sr[GQA];
        if (wwarp == 0) {
          if constexpr (GQA == 1) {
            tc::ld<1>(tl + C::C_S, sr);
          } else if constexpr (GQA == 2) {
            tc::ld<2>(tl + C::C_S, sr);
          } else if constexpr (GQA == 4) {
            tc::ld<4>(tl + C::C_S, sr);
          } else {
            tc::ld<8>(tl + C::C_S, sr);
          }
        }
        // values: channel wt of the piece's n tokens -> A_V columns 0..15
        if (C::SPLIT) wait_pv();
        {
          uint32_t cv[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const uint32_t v0 = 2 * i < n ? u16_at(sb + kResV + (2 * i) * 256 + 2 * wt) : 0u;
            const uint32_t v1 = 2 * i + 1 < n ? u16_at(sb + kResV + (2 * i + 1) * 256 + 2 * wt) : 0u;
            cv[i] = v0 | (v1 << 16);
          }
          tc::st<16>(tl + C::C_AV, cv);
        }
        if (wwarp == 0) tc::wait_ld();
#pragma unroll
        for (int h = 0; h < GQA; ++h) L[h] = valid ? __uint_as_float(sr[h]) * cr[h] : -INFINITY;
      }

      // ---------------------------------------------------------- softmax, PV operand
      bool ex = valid && !(sv < stt.vlim);
#pragma unroll
      for (int h = 0; h < GQA; ++h) ex |= !(L[h] <= stt.M[h] + kLazy);
      float pr[GQA];
      auto write_pv_row = [&]() {
#pragma unroll
        for (int h = 0; h < GQA; ++h) pr[h] = valid ? ex2(L[h] - stt.M[h]) : 0.0f;
        if (!res) {
          float xv[GQA];
#pragma unroll
          for (int h = 0; h < GQA; ++h) xv[h] = pr[h] * sv * stt.fsc;
          uint32_t v[GQA];
          if constexpr (GQA == 1) {
            uint32_t hi, lo;
            split2<__half>(xv[0], 0.0f, hi, lo);
            v[0] = (hi & 0xffffu) | (lo << 16);
          } else {
#pragma unroll
            for (int i = 0; i < GQA / 2; ++i) split2<__half>(xv[2 * i], xv[2 * i + 1], v[i], v[GQA / 2 + i]);
          }
          store_n16_row(bpv, wt, v);
        } else if (wwarp == 0) {
          float xv[GQA];
#pragma unroll
          for (int h = 0; h < GQA; ++h) xv[h] = 0.5f * pr[h] * stt.fsc;
          uint32_t v[GQA];
          if constexpr (GQA == 1) {
            uint32_t hi, lo;
            split2<T>(xv[0], 0.0f, hi, lo);
            v[0] = (hi & 0xffffu) | (lo << 16);
          } else {
#pragma unroll
            for (int i = 0; i < GQA / 2; ++i) split2<T>(xv[2 * i], xv[2 * i + 1], v[i], v[GQA / 2 + i]);
          }
          store_n16_row(bpv, wt, v);
        }
      };
      write_pv_row();
      tc::wait_st();
      tc::fence_async_smem();
      tc::fence_before();
      const bool any = wg_sync_or(wg, ex || failed);
      if (any) {
        failed = wg_sync_or(wg, failed);
        if (failed) break;
        // ---- slow path: the running maximum or the value exponent moves
        float mx[GQA];
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          float v = L[h];
          if (v != v || v == INFINITY) {  // NaN or +inf: an operand left the supported range
            flag_error(p.err, KVQ_DEV_ERR_RANGE);
            v = -INFINITY;
            L[h] = -INFINITY;
          }
          mx[h] = v;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) mx[h] = fmaxf(mx[h], __shfl_xor_sync(kFull, mx[h], off));
        }
        float svm = valid ? sv : 0.0f;
        if (!(svm < INFINITY)) {
          flag_error(p.err, KVQ_DEV_ERR_RANGE);
          svm = 0.0f;
          sv = 0.0f;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) svm = fmaxf(svm, __shfl_xor_sync(kFull, svm, off));
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < GQA; ++h) wc.red[wwarp][h] = mx[h];
          wc.red[wwarp][GQA] = svm;
        }
        wg_sync(wg);
        float alpha[GQA];
        int Fn = stt.F;
        {
          const float s4 = fmaxf(fmaxf(wc.red[0][GQA], wc.red[1][GQA]), fmaxf(wc.red[2][GQA], wc.red[3][GQA]));
          if (s4 >= stt.vlim) {
            // s4 in [2^e, 2^(e+1)): F = e - 6 keeps s4 * 2^(8 - F) below 2^15
            const int e = int((__float_as_uint(s4) >> 23) & 0xff) - 127;
            Fn = max(stt.F, min(e - 6, 120));
          }
        }
        const float beta = pow2f(stt.F - Fn);
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          const float mp = fmaxf(fmaxf(wc.red[0][h], wc.red[1][h]), fmaxf(wc.red[2][h], wc.red[3][h]));
          const float Mn = fmaxf(stt.M[h], mp);
          alpha[h] = stt.M[h] == -INFINITY ? 0.0f : ex2(stt.M[h] - Mn);
          stt.M[h] = Mn;
          stt.l[h] *= alpha[h];
          stt.zv[h] *= alpha[h];
        }
        if (stt.pv) {
          // rescale this thread's lane of O (the last value product has completed)
          wait_pv();
          uint32_t o[16];
          tc::ld<16>(tl + C::C_O, o);
          tc::wait_ld();
#pragma unroll
          for (int h = 0; h < GQA; ++h) {
            const float f = alpha[h] * beta;
            o[h] = __float_as_uint(__uint_as_float(o[h]) * f);
            o[GQA + h] = __float_as_uint(__uint_as_float(o[GQA + h]) * f);
          }
          tc::st<16>(tl + C::C_O, o);
        }
        stt.F = Fn;
        stt.vlim = pow2f(min(7 + Fn, 127));
        stt.fsc = pow2f(-Fn);
        write_pv_row();
        tc::wait_st();
        tc::fence_async_smem();
        tc::fence_before();
        wg_sync(wg);  // also keeps wc.red from being overwritten early
      }
      // ---------------------------------------------------------- PV product
      if (wt == 0) {
        tc::fence_after();
        if (!res) {
#pragma unroll
          for (int s = 0; s < 8; ++s)
            tc::mma(tbase + C::C_O, tbase + C::C_AV + 8 * s, tc::smem_desc(a_bpv + s * 512, 256, 128), ID_PV,
                    (stt.pv || s > 0) ? 1u : 0u);
        } else {
#pragma unroll
          for (int s = 0; s < 2; ++s)
            tc::mma(tbase + C::C_O, tbase + C::C_AV + 8 * s, tc::smem_desc(a_bpv + s * 512, 256, 128), ID_RES,
                    (stt.pv || s > 0) ? 1u : 0u);
        }
        tc::commit(&wc.bar_pv);
        // the stage is free (every thread has passed the barrier above): refill it
        if (t + C::NS < nseg) issue_item<GQA, KB, P>(p, wc, ws, xi + C::NS, t + C::NS, policy);
      }
      pv_pending = true;
      stt.pv = true;
#pragma unroll
      for (int h = 0; h < GQA; ++h) {
        stt.l[h] += pr[h];
        stt.zv[h] = fmaf(pr[h], zvt, stt.zv[h]);
      }

      // ---------------------------------------------------------- unit end
      if (d.w & kDescLast) {
        wait_pv();
        tc::fence_after();
        uint32_t o[16];
        tc::ld<16>(tl + C::C_O, o);
        float ls[GQA], zs[GQA];
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          ls[h] = stt.l[h];
          zs[h] = stt.zv[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            ls[h] += __shfl_xor_sync(kFull, ls[h], off);
            zs[h] += __shfl_xor_sync(kFull, zs[h], off);
          }
        }
        if (lane == 0) {
#pragma unroll
          for (int h = 0; h < GQA; ++h) {
            wc.red[wwarp][h] = ls[h];
            wc.red[wwarp][8 + h] = zs[h];
          }
        }
        tc::wait_ld();
        wg_sync(wg);
        const int u = d.b * p.Hkv + d.h;
        const int i0 = int(d.io & 0xffffu), i1 = int(d.io >> 16);
        const bool sole = i0 == i1;
        float* outu = p.out + (size_t(d.b) * p.Hq + size_t(d.h) * GQA) * kHeadDim;
        float* part_me = p.part + (size_t(worker) + u) * GQA * kPartStride;
        const float of = pow2f(stt.F + 1);
#pragma unroll
        for (int h = 0; h < GQA; ++h) {
          const float Lh = wc.red[0][h] + wc.red[1][h] + wc.red[2][h] + wc.red[3][h];
          const float Zh = wc.red[0][8 + h] + wc.red[1][8 + h] + wc.red[2][8 + h] + wc.red[3][8 + h];
          const float O = (__uint_as_float(o[h]) + __uint_as_float(o[GQA + h])) * of + Zh;
          if (sole) {
            outu[h * kHeadDim + wt] = Lh > 0.0f ? O / Lh : 0.0f;
          } else {
            float* pp = part_me + h * kPartStride;
            pp[wt] = O;
            if (wt == 0) {
              pp[kHeadDim] = stt.M[h];
              pp[kHeadDim + 1] = Lh;
            }
          }
        }
        stt.pv = false;
        if (!sole) {
          // the last of the contributors i0..i1 merges their partials.  The barrier
          // orders every thread's partial writes before the counter update (a release
          // at device scope); the merging worker acquires it.
          wg_sync(wg);
          if (wt == 0) wc.red[0][23] = __int_as_float(int(atomic_add_acq_rel_gpu(p.cnt + u, 1u)));
          wg_sync(wg);
          const int nc = i1 - i0 + 1;
          if (__float_as_int(wc.red[0][23]) == nc - 1) {
            const float* pu = p.part + (size_t(i0) + u) * GQA * kPartStride;
            for (int h = wwarp; h < GQA; h += 4) merge_heads<1>(pu, size_t(GQA) * kPartStride, nc, h, outu, lane);
            if (wt == 0) p.cnt[u] = 0u;  // ready for the next launch
          }
        }
        wg_sync(wg);  // wc.red is reused by the next unit
      }
    }
    if (failed) break;
    x += nseg;
    if (!wc.more) break;
  }

  if (failed) {
    // a wait gave up: flag it, then wait (bounded) for this worker's copies and
    // products in flight before the shared and tensor memory are released
    if (wt == 0) {
      flag_error(p.err, KVQ_DEV_ERR_TIMEOUT);
      const int issued = wc.issued;
      for (int y = max(0, issued - C::NS); y < issued; ++y)
        mbar_wait_bounded(&wc.full[y % C::NS], uint32_t(y / C::NS) & 1u);
    }
    if (pv_pending) mbar_wait_bounded(&wc.bar_pv, ppv);
  }
}

// ---------------------------------------------------------------- the kernel

template <typename T, int GQA, int KB, int P>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const __grid_constant__ DecodeParams p) {
  using C = Cfg<GQA, KB, P>;
  extern __shared__ __align__(1024) uint8_t smem[];
  __shared__ CtaCtl cc;
  __shared__ WgCtl<P> wctl[kWG];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wg = tid >> 7, wt = tid & 127;
  const int cta = blockIdx.x;
  pdl_wait();

  // ---------------------------------------------------------------- 1. the weight line
  // Total weight W, and the lengths of the first kSeqCache sequences.
  int W = 0;
  for (int base = 0; base < p.batch; base += kThreads) {
    const int b = base + tid;
    int x = 0;
    if (b < p.batch) {
      int np, rl;
      const int w = seq_weight<P>(p, b, np, rl);
      if (w < 0 && cta == 0) flag_error(p.err, KVQ_DEV_ERR_LENGTH);
      if (w <= 0 && b % p.n_ctas == cta) {  // nothing to attend to: the output is 0
        float4* o = reinterpret_cast<float4*>(p.out + size_t(b) * p.Hq * kHeadDim);
        for (int i = 0; i < p.Hq * kHeadDim / 4; ++i) o[i] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      x = max(w, 0) * p.Hkv;
      if (b < kSeqCache) cc.seq[b] = make_int2(np, rl);
    }
    int incl = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) cc.red[warp] = incl;
    __syncthreads();
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) W += cc.red[w];
    __syncthreads();
  }
  if (W == 0) return;
  const int n_workers = p.n_ctas * kWG;
  const int Cw = min(n_workers, max(1, W / 4));  // every range at least one stage long
  if (cta * kWG >= Cw) return;

  // ---------------------------------------------------------------- 2. locate the ranges
  // Sequence holding the first position of each worker's range: a second scan of the
  // weights (from the cache where it holds them).
  if (tid < kWG) {
    cc.b0[tid] = -1;
    cc.base0[tid] = 0;
  }
  {
    int run = 0;
    for (int base = 0; base < p.batch; base += kThreads) {
      const int b = base + tid;
      int x = 0;
      if (b < p.batch) {
        int np, rl;
        x = (b < kSeqCache ? unit_weight_of<P>(cc.seq[b].x, cc.seq[b].y) : max(seq_weight<P>(p, b, np, rl), 0)) *
            p.Hkv;
      }
      int incl = x;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(kFull, incl, off);
        if (lane >= off) incl += y;
      }
      __syncthreads();  // the previous round's reads of cc.red are done
      if (lane == 31) cc.red[warp] = incl;
      __syncthreads();
      int start = run + incl - x;
      for (int w = 0; w < warp; ++w) start += cc.red[w];
#pragma unroll
      for (int w = 0; w < kThreads / 32; ++w) run += cc.red[w];
#pragma unroll
      for (int g = 0; g < kWG; ++g) {
        const int pos = range_start(cta * kWG + g, W, Cw);
        if (x > 0 && start <= pos && pos < start + x) {
          cc.b0[g] = b;
          cc.base0[g] = start;
        }
      }
    }
  }

  // ---------------------------------------------------------------- 3. resources
  if (warp == 0) tc::alloc(&cc.tmem, 512);
  if (tid == 0) {
    for (int g = 0; g < kWG; ++g) {
      for (int s = 0; s < 4; ++s) mbar_init(&wctl[g].full[s], 1);
      mbar_init(&wctl[g].bar_s, 1);
      mbar_init(&wctl[g].bar_pv, 1);
    }
    fence_mbar_init();
  }
  // operand buffers start at zero (their padding columns are never written again)
  for (int g = 0; g < kWG; ++g) {
    uint4* z = reinterpret_cast<uint4*>(smem + g * C::BYTES + C::O_BQK);
    for (int i = tid; i < (C::O_QH - C::O_BQK) / 16; i += kThreads) z[i] = make_uint4(0u, 0u, 0u, 0u);
  }
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  const uint32_t tmem = cc.tmem;
  if (warp < 4) {
    // columns 0..7 of every lane: fp16 0.5, the A operand of the zero-point product
    uint32_t h[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) h[i] = 0x38003800u;
    tc::st<8>(tc::lane_addr(tmem, warp, 0), h);
    tc::wait_st();
  }
  tc::fence_async_smem();
  tc::fence_before();
  __syncthreads();
  tc::fence_after();
  // the grid fills every SM: the next kernel in the stream may be scheduled now
  pdl_trigger();

  // ---------------------------------------------------------------- 4. the workers
  const int worker = cta * kWG + wg;
  if (worker < Cw && cc.b0[wg] >= 0)
    worker_run<T, GQA, KB, P>(p, cc, wctl[wg], smem + wg * C::BYTES, tmem, W, Cw, worker, wg, wt);

  // ---------------------------------------------------------------- 5. leave
  tc::fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::fence_after();
    tc::dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- per-instantiation host side

template <typename T, int GQA, int KB, int P>
constexpr int smem_bytes() {
  return kWG * Cfg<GQA, KB, P>::BYTES;
}

template <typename T, int GQA, int KB, int P>
cudaError_t prepare_decode() {
  static int seen[64];
  return ensure_dynamic_smem(decode_kernel<T, GQA, KB, P>, smem_bytes<T, GQA, KB, P>(), seen);
}

// Calls f.template operator()<KB, P>() for one (kb, P).
template <typename F>
cudaError_t dispatch_kb_p(int kb, int P, F&& f) {
#define KVQ_P(K)                                     \
  switch (P) {                                       \
    case 32: return f.template operator()<K, 32>();   \
    case 64: return f.template operator()<K, 64>();   \
    case 128: return f.template operator()<K, 128>(); \
  }                                                  \
  return cudaErrorInvalidValue;
  switch (kb) {
    case 0: { KVQ_P(0) }
    case 1: { KVQ_P(1) }
    case 2: { KVQ_P(2) }
    case 4: { KVQ_P(4) }
    case 8: { KVQ_P(8) }
  }
  return cudaErrorInvalidValue;
#undef KVQ_P
}

template <typename T, int GQA>
struct DecodeOcc {
  int* n;
  template <int KB, int P>
  cudaError_t operator()() {
    cudaError_t e = prepare_decode<T, GQA, KB, P>();
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, decode_kernel<T, GQA, KB, P>, kThreads,
                                                         smem_bytes<T, GQA, KB, P>());
  }
};

template <typename T, int GQA>
struct DecodeRun {
  const DecodeParams& p;
  cudaStream_t stream;
  template <int KB, int P>
  cudaError_t operator()() {
    if (p.L.record != Rec<P, KB>::record || p.L.payload != Rec<P, KB>::payload) return cudaErrorInvalidValue;
    cudaError_t e = prepare_decode<T, GQA, KB, P>();
    if (e != cudaSuccess) return e;
    return launch_pdl(decode_kernel<T, GQA, KB, P>, dim3(p.n_ctas), dim3(kThreads), smem_bytes<T, GQA, KB, P>(),
                      stream, p);
  }
};

}  // namespace dec

// One translation unit per (dtype, GQA) defines these two entry points.
#define KVQ_DECODE_INSTANCE(NAME, T, GQA)                                                       \
  cudaError_t decode_occupancy_##NAME(int kb, int P, int* n) {                                 \
    return dec::dispatch_kb_p(kb, P, dec::DecodeOcc<T, GQA>{n});                                \
  }                                                                                             \
  cudaError_t decode_launch_##NAME(const DecodeParams& p, cudaStream_t stream) {               \
    return dec::dispatch_kb_p(p.KB, p.P, dec::DecodeRun<T, GQA>{p, stream});                    \
  }

}  // namespace kvq
