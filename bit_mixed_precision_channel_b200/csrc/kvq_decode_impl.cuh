// kvq_decode_impl.cuh — decode attention over the paged 2-bit cache, sm_100a.
// Kernel templates; kvq_decode_<dtype>_g<GQA>.cu instantiate them, kvq_decode.cu
// holds the host side.
//
// Work decomposition (balanced streaming).  Every (sequence b, kv head h) is a unit;
// its items are its pages, grouped into 128-token stages (1, 2 or 4 pages), followed by
// its residual tokens in pieces of 16.  Item weights count 32-token groups (a full
// stage weighs 4, a residual piece kPieceWeight, the merge at a unit's end kMergeWeight,
// all as measured).  Units are laid end to end in (b, h) order and
// the resulting weight line is cut into one equal range per CTA, one CTA per resident
// slot of the GPU (SMs x CTAs per SM); a CTA processes the items that start inside its
// range, so every SM receives the same amount of work whatever the sequence lengths.
// A CTA that finishes a unit writes either the output (when it saw the whole unit) or a
// partial (max, sum, unnormalised output); the last contributor of a unit merges the
// partials (log-sum-exp), so there is no second launch.
//
// Data movement.  A 3-stage shared-memory ring holds page records (one cp.async.bulk per
// record, L2 evict-first hint) or residual pieces (16-byte cp.async into padded rows,
// zero-filled past the last token); a unit's query heads travel with its first item.
// Completion is tracked with "full" mbarriers and every wait is bounded.  Warp 0 issues
// the first three items of a segment; afterwards the warp that releases a stage last
// (an acquire-release counter per stage) refills it with the item three places ahead.
// Each warp owns one 32-token group of a page stage and runs its own online softmax;
// warps meet only at the end of a unit.
//
// Arithmetic.  The 2-bit codes never become scaled values.  The scales are folded into
// the other operand of each product, and the codes go to the tensor cores as they are
// (Kitty abstract: page dequantization kernels; MiniKV proposed method: dequantization
// fused into the attention matmul):
//   q.k_t = sum_c codeA[t,c] (q_c sA_c) + sum_j codeB[t,j] (q_idx(j) sB_j) + sum_c q_c zA_c
//   sum_t p_t v_t[c] = sum_t codeV[t,c] (p_t sV_t) + sum_t p_t zV_t
// Codes reach the tensor cores exactly as 0.5 * code through the FP4 (e2m1) conversion;
// the folded operands are carried as fp16 high and low parts (hi = fp16(x),
// lo = fp16(x - hi)).  The eight columns of an m16n8k16 product hold four query heads,
// each as an adjacent (hi, lo) column pair, so a lane's two accumulator columns are the
// two parts of one head: the logits need no shuffle, and the (hi, lo) pair of
// p * sV is one register that movmatrix turns into the B fragment of the PV product.
#pragma once
#include <algorithm>

#include "kvq_internal.cuh"

namespace kvq {

constexpr int kStages = 3;
constexpr int kDecodeThreads = 128;
constexpr int kResRowBytes = 272;  // residual row in shared memory: 256 bytes + 16 pad
constexpr int kPieceTokens = 16;   // residual tokens per item
constexpr int kPieceWeight = kDecodePieceWeight;
constexpr int kMergeWeight = kDecodeMergeWeight;

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

// Dynamic shared memory of one CTA: kStages stages (page records, or the K and V rows
// of a residual piece), then the merge buffer [4 warps][GQA][128] fp32.
template <int GQA, int P, int KB>
struct Smem {
  static constexpr uint32_t body = std::max<uint32_t>((128 / P) * Rec<P, KB>::record, 2 * kPieceTokens * kResRowBytes);
  static constexpr uint32_t stage = (body + 127u) / 128u * 128u;
  static constexpr uint32_t merge = kStages * stage;
  static constexpr uint32_t bytes = merge + 4u * GQA * 128u * 4u;
};

// ---------------------------------------------------------------- operand builders

// One part of the folded query operand, chosen per lane without a branch:
// hfma2(q, s, -fp16(q*s) * m) is fp16(q*s) for m = 0 (hi lanes) and the exact rest
// q*s - fp16(q*s) for m = 1 (lo lanes); the product of two fp16 values is exact in fp32.
__device__ __forceinline__ uint32_t fold_one(uint32_t q2, uint32_t s2, uint32_t negmask, __half) {
  const __half2 q = u32_as_h2(q2), s = u32_as_h2(s2);
  const __half2 h = __hmul2(q, s);
  return h2_as_u32(__hfma2(q, s, __hmul2(h, u32_as_h2(negmask))));
}
// Two cache-dtype values as an fp16 pair.  bf16 values are exact in fp16 inside its
// normal range (8 significant bits fit in 11), which is where the kernel carries bf16
// queries, scales and zero points: the folded products then use the fp16 path above.
__device__ __forceinline__ uint32_t to_f16x2(uint32_t x, __half) { return x; }
__device__ __forceinline__ uint32_t to_f16x2(uint32_t x, __nv_bfloat16) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(__uint_as_float(x & 0xffff0000u)), "f"(__uint_as_float(x << 16)));
  return d;
}

// A query pair of the cache dtype scaled by 2^-e, as fp16: for fp16 one exact product
// (2^-e >= 2^-24 is an fp16 number); for bf16 through fp32, so that queries beyond
// fp16's range are scaled before they are rounded.
__device__ __forceinline__ uint32_t scale_q2(uint32_t q2, uint32_t sbq, float, __half) {
  return h2_as_u32(__hmul2(u32_as_h2(q2), u32_as_h2(sbq)));
}
__device__ __forceinline__ uint32_t scale_q2(uint32_t q2, uint32_t, float sc, __nv_bfloat16) {
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(__uint_as_float(q2 & 0xffff0000u) * sc), "f"(__uint_as_float(q2 << 16) * sc));
  return d;
}

// (hi, lo) of x as one register: low half = hi, high half = lo.
__device__ __forceinline__ uint32_t hilo(float x, __half) {
  const float hf = __half2float(__float2half_rn(x));
  uint32_t d;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(x - hf), "f"(hf));
  return d;
}
__device__ __forceinline__ uint32_t hilo(float x, __nv_bfloat16) {
  const float hf = __bfloat162float(__float2bfloat16_rn(x));
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(x - hf), "f"(hf));
  return d;
}

// Two 16-bit values of a register as floats.
__device__ __forceinline__ float2 t2_to_float2(uint32_t u, __half) { return __half22float2(u32_as_h2(u)); }
__device__ __forceinline__ float2 t2_to_float2(uint32_t u, __nv_bfloat16) {
  return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}

// ---------------------------------------------------------------- per-warp state

template <int NT>
struct WarpState {
  float o[8][NT][4];  // PV accumulator: rows = channels 16*mc + g (+8), cols (hi, lo) of head qd + 4*nt
  float m[NT], l[NT], zv[NT];
  // value exponent: the PV operand carries p * sV * 2^-F, and F grows (rescaling o) before
  // a value scale could push p * sV * 2^-F past fp16's range (p < 2^8 by the lazy maximum)
  int F;
  float fsc;   // 2^-F
  float vlim;  // 2^(7 + F): value scales at or above it need a larger F
};

// Query pairs of this lane in fp16: head (g/2) + 4 nt, channels 16 s + 2 qd (+1) for
// j = 0 and 8 more for j = 1.  They are the B column g of the code products (with the
// part g % 2 chosen by negmask) and, stored as register quads, the A operand of the
// zero-point product, whose rows are heads:
//   NT = 2: quad s = {q(0,s,0), q(1,s,0), q(0,s,1), q(1,s,1)}: rows g / g+8 = heads
//           g/2 and g/2 + 4 at k-step s;
//   NT = 1: quad i = {q(0,i,0), q(0,i+4,0), q(0,i,1), q(0,i+4,1)}: rows g / g+8 = head
//           g/2 at k-steps i and i + 4.
template <int NT>
struct LaneQ {
  uint32_t qa[NT == 2 ? 8 : 4][4];
  uint32_t negmask;  // fp16x2 -1 for lo-part lanes (odd g), 0 otherwise
  // The query enters the products as q' = q * 2^-e_h, e_h >= 0 the smallest power of two
  // with max_c |q_h[c]| < 2^e_h (0 when the query is already below 1), so that a folded
  // key operand q' * scale never exceeds the scale: no fp16 overflow for fp16 caches.
  float cl[NT];      // sm_scale * log2(e) * 2^e of the logit head qd + 4 nt
  uint32_t sbq[NT];  // fp16x2 2^-e of the B-column head (g / 2) + 4 nt (plane-B gathers)
  float sq[NT];      // the same 2^-e as a float
  __device__ __forceinline__ uint32_t& qv(int nt, int s, int j) {
    return NT == 2 ? qa[s][2 * j + nt] : qa[s & 3][2 * j + (s >> 2)];
  }
  __device__ __forceinline__ uint32_t qv(int nt, int s, int j) const {
    return NT == 2 ? qa[s][2 * j + nt] : qa[s & 3][2 * j + (s >> 2)];
  }
};

template <int NT>
__device__ __forceinline__ void reset_state(WarpState<NT>& st) {
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) st.o[mc][nt][i] = 0.0f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    st.m[nt] = -INFINITY;
    st.l[nt] = 0.0f;
    st.zv[nt] = 0.0f;
  }
  st.F = 0;
  st.fsc = 1.0f;
  st.vlim = 128.0f;
}

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // e in [-126, 127]

// Raises the value exponent F of this warp so that a value scale sv stays below 2^(7+F)
// (warp-uniform call); o is rescaled by 2^(F_old - F_new).  A scale that is not finite
// means an input outside the supported range: flagged, and F stays.
template <int NT>
__device__ __forceinline__ void raise_value_exponent(WarpState<NT>& st, float sv, int32_t* err) {
  float m = sv < INFINITY ? sv : 0.0f;
  if (!(sv < INFINITY)) flag_error(err, KVQ_DEV_ERR_RANGE);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, off));
  if (!(m >= st.vlim)) return;
  // m in [2^e, 2^(e+1)): F = e - 6 keeps m * 2^(8 - F) below 2^15
  const int e = int((__float_as_uint(m) >> 23) & 0xff) - 127;
  const int Fn = max(st.F, min(e - 6, 100));
  const float beta = pow2f(st.F - Fn);
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) st.o[mc][nt][i] *= beta;
  st.F = Fn;
  st.fsc = pow2f(-Fn);
  st.vlim = pow2f(min(7 + Fn, 127));
}

// Online-softmax update from MT x 2 logits per head part of this lane (log2 units).  The
// running maximum moves only when a logit exceeds it by more than 8, so probabilities
// stay below 2^8 and most groups skip the rescale of the accumulators.
template <int NT, int MT>
__device__ __forceinline__ void softmax_step(WarpState<NT>& st, const float (&L)[MT][NT][2], int32_t* err) {
  // the lanes' own maxima decide whether any head can move; only then are they reduced
  float mx[NT];
  bool big = false;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mx[nt] = L[0][nt][0];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) mx[nt] = fmaxf(mx[nt], fmaxf(L[mt][nt][0], L[mt][nt][1]));
    big |= !(mx[nt] <= st.m[nt] + 8.0f);  // also true for a NaN logit
  }
  if (!__any_sync(kFull, big)) return;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
    if (!(mx[nt] < INFINITY) && mx[nt] != -INFINITY) flag_error(err, KVQ_DEV_ERR_RANGE);
  float alpha[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mx[nt] = fmaxf(mx[nt], __shfl_xor_sync(kFull, mx[nt], 4));
    mx[nt] = fmaxf(mx[nt], __shfl_xor_sync(kFull, mx[nt], 8));
    mx[nt] = fmaxf(mx[nt], __shfl_xor_sync(kFull, mx[nt], 16));
    alpha[nt] = 1.0f;
    if (mx[nt] > st.m[nt] + 8.0f) {
      alpha[nt] = ex2(st.m[nt] - mx[nt]);  // 0 on the first group (m = -inf)
      st.m[nt] = mx[nt];
      st.l[nt] *= alpha[nt];
      st.zv[nt] *= alpha[nt];
    }
  }
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) st.o[mc][nt][i] *= alpha[nt];
}

// ---------------------------------------------------------------- one quantized group

// Tokens [32 grp, 32 grp + 32) of the page record `rec` (shared memory), for the lane
// (g, qd): QK^T over planes A and B and the zero points, online softmax, then PV.
template <typename T, int GQA, int KB, int P>
__device__ __forceinline__ void page_group(const uint8_t* rec, int grp, const LaneQ<(GQA > 4 ? 2 : 1)>& lq,
                                           const uint16_t* qs, WarpState<(GQA > 4 ? 2 : 1)>& st, int lane,
                                           int32_t* err) {
  constexpr int NT = GQA > 4 ? 2 : 1;
  using R = Rec<P, KB>;
  const int g = lane >> 2, qd = lane & 3;
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;

  // -- plane A: rows 32 grp + 16 mt + 8 r + g, words 2qd and 2qd+1 (channels of k-steps
  //    0..3 and 4..7); scales of k-steps 2i, 2i+1 are 16 bytes at 64 i + 16 qd --
  const uint8_t* kA = rec + R::k_codes + (32 * grp + g) * 32 + 8 * qd;
  uint2 w[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) w[mt][r] = lds64(kA + (16 * mt + 8 * r) * 32);
  const uint8_t* ksc = rec + R::k_scale + grp * 256 + 16 * qd;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint4 sc = lds128(ksc + 64 * i);
    uint32_t c[2][2][4];  // [mt][row][byte]: byte 2jj + r -> k-step 2i + jj, A register (r ? 2 : 0) + row
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int r = 0; r < 2; ++r)
        e2m1_pairs(code_pass((i >> 1) ? w[mt][r].y : w[mt][r].x, i & 1), c[mt][r][0], c[mt][r][1], c[mt][r][2],
                   c[mt][r][3]);
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int s = 2 * i + jj;
      uint32_t b[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        b[nt][0] = fold_one(lq.qv(nt, s, 0), to_f16x2(jj ? sc.z : sc.x, T()), lq.negmask, __half());
        b[nt][1] = fold_one(lq.qv(nt, s, 1), to_f16x2(jj ? sc.w : sc.y, T()), lq.negmask, __half());
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t a[4] = {c[mt][0][2 * jj], c[mt][1][2 * jj], c[mt][0][2 * jj + 1], c[mt][1][2 * jj + 1]};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a, b[nt][0], b[nt][1], __half());
      }
    }
  }

  // -- plane B: low bits of the boosted channels; rows 16s + 8r + 2qd + f of this lane sit
  //    at positions 4 KB qd + 4s + 2r + f of each token row --
  if constexpr (KB > 0) {
    const uint8_t* kB = rec + R::kb_codes;
    const uint8_t* idx = rec + R::boost_idx;
    const uint8_t* kbsc = rec + R::kb_scale + grp * (32 * KB);
    // k-steps in pairs: the codes of two k-steps sit in one word of each token row, so at
    // most 16 code registers are live whatever KB is
    constexpr int SP = KB == 1 ? 1 : 2;
#pragma unroll
    for (int sp = 0; sp < KB; sp += SP) {
      uint32_t cb[2][2][SP][2];  // [mt][row][s - sp][r]
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int rr = 0; rr < 2; ++rr) {
          const uint8_t* row = kB + (32 * grp + 16 * mt + g + 8 * rr) * KB * 4;
          if constexpr (KB == 1) {
            const uint32_t x = code_pass(lds32(row), qd >> 1) >> (16 * (qd & 1));
            cb[mt][rr][0][0] = e2m1_pair_lo(x);
            cb[mt][rr][0][1] = e2m1_pair_lo(x >> 8);
          } else {
            const int pos = 4 * KB * qd + 4 * sp;
            const uint32_t x = code_pass(lds32(row + (pos >> 4) * 4), (pos >> 3) & 1);
            e2m1_pairs(x, cb[mt][rr][0][0], cb[mt][rr][0][1], cb[mt][rr][SP - 1][0], cb[mt][rr][SP - 1][1]);
          }
        }
#pragma unroll
      for (int ss = 0; ss < SP; ++ss) {
        const int s = sp + ss;
        const int j0 = 16 * s + 2 * qd, j1 = j0 + 8;
        // indices are < 128 in any record the library wrote; the mask keeps a corrupt
        // record from reading outside the query rows
        const int i00 = idx[j0] & 127, i01 = idx[j0 + 1] & 127, i10 = idx[j1] & 127, i11 = idx[j1 + 1] & 127;
        const uint32_t s0 = to_f16x2(lds32(kbsc + j0 * 2), T()), s1 = to_f16x2(lds32(kbsc + j1 * 2), T());
        uint32_t b[NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          const int hB = (g >> 1) + 4 * nt;
          uint32_t q0 = 0u, q1 = 0u;
          if (hB < GQA) {
            const uint16_t* qh = qs + hB * kHeadDim;
            q0 = uint32_t(qh[i00]) | (uint32_t(qh[i01]) << 16);
            q1 = uint32_t(qh[i10]) | (uint32_t(qh[i11]) << 16);
          }
          // the gathered query scaled to q' = q * 2^-e (exact unless q' is an fp16 subnormal)
          b[nt][0] = fold_one(scale_q2(q0, lq.sbq[nt], lq.sq[nt], T()), s0, lq.negmask, __half());
          b[nt][1] = fold_one(scale_q2(q1, lq.sbq[nt], lq.sq[nt], T()), s1, lq.negmask, __half());
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t a[4] = {cb[mt][0][ss][0], cb[mt][1][ss][0], cb[mt][0][ss][1], cb[mt][1][ss][1]};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a, b[nt][0], b[nt][1], __half());
        }
      }
    }
  }

  // -- zero points: Z[h] = sum_c q[h][c] * zA[c], with the query quads as A (rows are
  //    heads) and the zero points as B (every column the same); the 16 bytes at
  //    64 i + 16 qd are the B pairs of k-steps 2i and 2i+1 --
  float zh[NT];
  {
    const uint8_t* kz = rec + R::k_zero + grp * 256 + 16 * qd;
    float z0[4] = {0.f, 0.f, 0.f, 0.f}, z1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 zz = lds128(kz + 64 * i);
      const uint32_t b0[2] = {to_f16x2(zz.x, T()), to_f16x2(zz.z, T())};
      const uint32_t b1[2] = {to_f16x2(zz.y, T()), to_f16x2(zz.w, T())};
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int s = 2 * i + jj;
        if constexpr (NT == 2) {
          mma_16816(z0, lq.qa[s], b0[jj], b1[jj], __half());  // rows g: head g/2, g+8: head g/2 + 4
        } else if (s < 4) {
          mma_16816(z0, lq.qa[s], b0[jj], b1[jj], __half());  // rows g: k-step s
        } else {
          mma_16816(z1, lq.qa[s - 4], b0[jj], b1[jj], __half());  // rows g+8: k-step s
        }
      }
    }
    // this lane holds Z of head g/2 (+4); head qd (+4) sits in lane 8 qd
    if constexpr (NT == 2) {
      zh[0] = __shfl_sync(kFull, z0[0], 8 * qd);
      zh[1] = __shfl_sync(kFull, z0[2], 8 * qd);
    } else {
      zh[0] = __shfl_sync(kFull, z0[0] + z1[2], 8 * qd);
    }
  }

  // -- logits (log2 units) of tokens 16 mt + 8 r + g for head qd + 4 nt; the code
  //    products carry a factor 0.5, and the query its scale 2^-e --
  float L[2][NT][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 2; ++r)
        L[mt][nt][r] = fmaf(acc[mt][nt][2 * r] + acc[mt][nt][2 * r + 1], lq.cl[nt] * kCodeScale, zh[nt] * lq.cl[nt]);
  softmax_step<NT, 2>(st, L, err);

  // -- probabilities times the value scales, as (hi, lo) pairs -> B operand of PV.
  //    Value scale/zero positions 32 grp + 4 g + u hold tokens 8u + g --
  const uint2 vsr = lds64(rec + R::v_scale + (32 * grp + 4 * g) * 2);
  const uint2 vzr = lds64(rec + R::v_zero + (32 * grp + 4 * g) * 2);
  const float2 s01 = t2_to_float2(vsr.x, T()), s23 = t2_to_float2(vsr.y, T());
  const float2 z01 = t2_to_float2(vzr.x, T()), z23 = t2_to_float2(vzr.y, T());
  const float sv[4] = {s01.x, s01.y, s23.x, s23.y}, zv[4] = {z01.x, z01.y, z23.x, z23.y};
  if (__any_sync(kFull, !(fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3])) < st.vlim)))
    raise_value_exponent(st, fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3])), err);
  uint32_t pb[2][NT][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int u = 2 * mt + r;
        const float pr = ex2(L[mt][nt][r] - st.m[nt]);
        st.l[nt] += pr;
        st.zv[nt] = fmaf(pr, zv[u], st.zv[nt]);
        pb[mt][nt][r] = movmatrix_trans(hilo(pr * sv[u] * st.fsc, __half()));
      }

  // -- P V: words ((2 grp + n) * 32 + lane) * 4 + mm hold channel tile 4n + mm of this
  //    lane; pass ks of a word is k-step ks, bytes in A-register order --
  const uint8_t* vq = rec + R::v_codes + (64 * grp + lane) * 16;
  const uint4 v0 = lds128(vq), v1 = lds128(vq + 512);
  const uint32_t vw[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      uint32_t a[4];
      e2m1_pairs(code_pass(vw[mc], ks), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(st.o[mc][nt], a, pb[ks][nt][0], pb[ks][nt][1], __half());
    }
}

// ---------------------------------------------------------------- residual tokens

// One piece of n <= 16 residual tokens staged in shared memory as K rows then V rows
// (272-byte rows; rows n..15 hold zeros).  The PV operand carries 0.5 * p so
// that the accumulator stays in the units of the code products.
template <typename T, int GQA>
__device__ __forceinline__ void residual_piece(const uint8_t* Kr, const uint8_t* Vr, int n, const uint16_t* qs,
                                               WarpState<(GQA > 4 ? 2 : 1)>& st, int lane, float c_log2,
                                               int32_t* err) {
  constexpr int NT = GQA > 4 ? 2 : 1;
  const int g = lane >> 2, li = lane >> 3, lr = lane & 7;
  const bool lo = g & 1;  // lo-part columns get no query: the raw query is exact
  float acc[NT][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[nt][i] = 0.0f;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    uint32_t a[4];
    ldmatrix_x4(a, smem_addr(Kr + (lr + 8 * (li & 1)) * kResRowBytes + (16 * s + 8 * (li >> 1)) * 2));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      // the raw query in the cache dtype (exact); lo-part columns get none
      const int hB = (g >> 1) + 4 * nt, qd = lane & 3;
      const bool use = !lo && hB < GQA;
      const uint32_t b0 = use ? lds32(qs + hB * kHeadDim + 16 * s + 2 * qd) : 0u;
      const uint32_t b1 = use ? lds32(qs + hB * kHeadDim + 16 * s + 2 * qd + 8) : 0u;
      mma_16816(acc[nt], a, b0, b1, T());
    }
  }
  float L[1][NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int r = 0; r < 2; ++r)
      L[0][nt][r] = (g + 8 * r) < n ? (acc[nt][2 * r] + acc[nt][2 * r + 1]) * c_log2 : -INFINITY;
  softmax_step<NT, 1>(st, L, err);
  uint32_t pb[NT][2];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt)
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const float pr = ex2(L[0][nt][r] - st.m[nt]);
      st.l[nt] += pr;
      pb[nt][r] = movmatrix_trans(hilo(0.5f * pr * st.fsc, T()));
    }
#pragma unroll
  for (int mc = 0; mc < 8; ++mc) {
    uint32_t a[4];
    ldmatrix_x4_trans(a, smem_addr(Vr + (lr + 8 * (li >> 1)) * kResRowBytes + (16 * mc + 8 * (li & 1)) * 2));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_16816(st.o[mc][nt], a, pb[nt][0], pb[nt][1], T());
  }
}

// ---------------------------------------------------------------- work items

// Position on the weight line: unit (b, h), item k of the unit, start weight s.  Every
// warp walks the same sequence of items, so the loop structure (and every barrier in
// it) is identical in all warps even when a copy fails.  Weights are 32-bit: the host
// rejects shapes whose line could reach 2^31.
struct Cursor {
  int b, h, k;
  int np, rl, nst, nres;  // pages, residual tokens, page stages, residual pieces of b
  int s, ubase;           // start weight of item k and of the unit
};

// Unit weight of sequence b (-1 when its lengths are invalid), with its pages and
// residual tokens (0 when invalid).
// In dense mode (p.seq_len set) a sequence has no quantized pages: all its tokens are
// read as raw rows through its page table, in the residual pieces' path.
template <int P>
__device__ __forceinline__ int seq_weight(const DecodeParams& p, int b, int& np, int& rl) {
  if (p.seq_len) {
    np = 0;
    rl = __ldcg(p.seq_len + b);
  } else {
    np = __ldcg(p.num_pages + b);
    rl = __ldcg(p.res_len + b);
  }
  if (np < 0 || np > p.max_pages || rl < 0 || rl > (p.seq_len ? p.max_pages * P : P)) {
    np = 0;
    rl = 0;
    return -1;
  }
  const int items = np * (P / 32) + kPieceWeight * ((rl + kPieceTokens - 1) / kPieceTokens);
  return items > 0 ? items + kMergeWeight : 0;
}

template <int P>
__device__ __forceinline__ void cursor_load_seq(const DecodeParams& p, Cursor& c) {
  // skip sequences without items; c.b == batch marks the end of the line
  while (c.b < p.batch) {
    if (seq_weight<P>(p, c.b, c.np, c.rl) > 0) break;
    ++c.b;
  }
  if (c.b >= p.batch) c.np = c.rl = 0;
  c.nst = (c.np * P + 127) / 128;
  c.nres = (c.rl + kPieceTokens - 1) / kPieceTokens;
}

// Weight of item k of the current unit: pages of the stage x groups per page, or 1.
template <int P>
__device__ __forceinline__ int item_weight(const Cursor& c) {
  if (c.k < c.nst) return min(128 / P, c.np - c.k * (128 / P)) * (P / 32);
  return kPieceWeight;
}
// Weight of a unit: its items, then the merge weight (0 for a unit without items).
template <int P>
__device__ __forceinline__ int unit_weight(const Cursor& c) {
  const int items = c.np * (P / 32) + kPieceWeight * c.nres;
  return items > 0 ? items + kMergeWeight : 0;
}

template <int P>
__device__ __forceinline__ int unit_weight_of(int2 v) {
  const int items = v.x * (P / 32) + kPieceWeight * ((v.y + kPieceTokens - 1) / kPieceTokens);
  return items > 0 ? items + kMergeWeight : 0;
}

template <int P>
__device__ __forceinline__ void cursor_next(const DecodeParams& p, Cursor& c) {
  c.s += item_weight<P>(c);
  if (++c.k < c.nst + c.nres) return;
  c.k = 0;
  c.s += kMergeWeight;
  c.ubase = c.s;
  if (++c.h < p.Hkv) return;
  c.h = 0;
  ++c.b;
  cursor_load_seq<P>(p, c);
}

// CTA that owns weight position s: the one whose range [ceil(W i / C), ceil(W (i+1) / C))
// contains it.
// Both are exact in double: the products stay below 2^53 and a quotient that is not an
// integer is at least 1/(W C) away from one, far above the rounding error.
__device__ __forceinline__ int owner_cta(int s, int W, int C) { return int(floor(double(s) * C / W)); }
__device__ __forceinline__ int range_start(int i, int W, int C) { return int(ceil(double(W) * i / C)); }

// Range index of CTA b.  The grid fills every resident slot at once and the hardware puts
// CTA b on SM b mod S (S SMs, n = c * S CTAs), so SM s holds CTAs s, s + S, s + 2S, ...
// Consecutive ranges are about a fifth of a unit long on the 8B-shaped layer, and S of
// them span almost a whole number of units: CTAs s + jS would hold ranges at the same phase
// of their units (all page stages, or all unit ends) and some SMs would get the heavy mix
// four times.  Rotating block j of S ranges by j puts an SM's ranges j ranges apart in
// phase.  (Any other placement only changes which ranges share an SM.)
__device__ __forceinline__ int range_of_cta(int b, int n, int S) {
  if (S <= 0 || n % S != 0) return b;
  const int j = b / S, s = b - j * S;
  return (s + j) % S + j * S;
}

// Owners of positions on the weight line: the line is cut into Cs equal ranges and CTA
// i owns range i.  Every range is at least 4 long, so every owner between a unit's
// first and last owner holds an item of the unit.
struct Owners {
  int W, Cs;
  __device__ __forceinline__ int of(int s) const { return owner_cta(s, W, Cs); }
};

// Partial softmax state of one (CTA, unit) slot and head: unnormalised output [128],
// then the maximum and the sum (floats 128, 129), padded to 16 bytes.
constexpr int kPartStride = kHeadDim + 4;

// Moves the cursor from offset `ou` of its unit to the first item that starts at or
// after it, or to the first item of the next unit.
template <int P>
__device__ __forceinline__ void cursor_seek(const DecodeParams& p, Cursor& c, int ou) {
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
  cursor_load_seq<P>(p, c);
}


__device__ __forceinline__ void named_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Shared-memory atomic add with acquire-release semantics at CTA scope.
__device__ __forceinline__ int atomic_add_acq_rel_cta(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.s32 %0, [%1], %2;" : "=r"(old) : "r"(smem_addr(p)), "r"(v) : "memory");
  return old;
}

// Device-scope atomic add with acquire-release semantics.
__device__ __forceinline__ uint32_t atomic_add_acq_rel_gpu(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}


// ---------------------------------------------------------------- item descriptors

// A CTA walks its range in segments of up to kSegItems items.  Before a segment, the
// CTA lists its items in shared memory (all threads, page ids loaded in parallel), so
// that issuing the copies of an item and consuming it need no further bookkeeping.
constexpr int kSegItems = 128;
constexpr int kSeqCache = 128;  // (pages, residual) of the sequences from the first one on

enum : uint32_t { kDescRes = 1u << 8, kDescFirst = 1u << 9, kDescLast = 1u << 10 };

struct ItemDesc {
  uint32_t w;   // bits 0-7: pages in the stage or residual tokens; kDescRes, kDescFirst,
                // kDescLast; bits 11-12: query slot; bits 16-31: stage or piece index
  int b, h;     // unit
  uint32_t io;  // first and last contributing CTA of the unit (low, high 16 bits), kDescLast only
};

// Unit spans of one segment, found by one thread walking the line.
struct UnitSpan {
  int off;        // first item of the span within the segment
  int b, h, k0;   // unit and its first item in the span
  int n;          // items of the span
  int np, rl;
  int first, last;  // span starts / ends the unit's part in this CTA
  int qslot;
  uint32_t io;
};

// Pages and residual tokens of sequence b: from the cache filled during the scan, else
// from global memory.  Returns the unit weight (0 for empty or invalid lengths).
template <int P>
__device__ __forceinline__ int seq_info(const DecodeParams& p, int b, int b0, const int2* s_seq, int& np, int& rl) {
  if (b0 >= 0 && b - b0 >= 0 && b - b0 < kSeqCache) {
    const int2 v = s_seq[b - b0];
    np = v.x;
    rl = v.y;
    return unit_weight_of<P>(v);
  }
  return max(0, seq_weight<P>(p, b, np, rl));
}

// ---------------------------------------------------------------- the kernel

// Shared state of one CTA besides the stages.
template <int GQA, int P>
struct CtaShared {
  uint64_t full_bar[kStages];  // stage filled (bulk-copy bytes landed)
  int rel[kStages];            // warps that released the stage's current item
  int red[4];
  int b0, base0, abort_flag, issued, arrived;
  int tail_u;         // unit whose split merge waits for the end of the range, or -1
  uint32_t tail_io;   // its first and last contributors
  int pref[kSeqCache];         // exclusive prefix of the weights (x kv heads), one-pass case
  int nseg, more, nspan, uord, qslot_cont;
  Cursor cur;                  // first item of the next segment
  float m[4][GQA], l[4][GQA], zv[4][GQA];
  int2 seq[kSeqCache];
  UnitSpan span[32];
  ItemDesc desc[kSegItems];
  int ids[kSegItems][128 / P];
  __align__(16) uint16_t q[3][GQA * kHeadDim];  // query heads of the last 3 units
};

// Lists the next segment of this CTA's items (all threads).  One thread walks the units
// from sh.cur; then every thread fills one descriptor and loads its page ids.
template <int GQA, int KB, int P>
__device__ __forceinline__ void build_segment(const DecodeParams& p, CtaShared<GQA, P>& sh, int hi, const Owners& ow,
                                              int tid, bool one_pass) {
  constexpr int PPC = 128 / P, GPP = P / 32;
  if (tid == 0) {
    Cursor c = sh.cur;
    int n = 0, ns = 0, uord = sh.uord, qcont = sh.qslot_cont;
    const bool cta_first = sh.uord < 0;  // no unit started yet: the range's first segment
    while (c.s < hi && n < kSegItems && ns < 32) {
      const int nitems = c.nst + c.nres;
      // items of the unit that start before hi
      int kend = nitems;
      const int kst = min(c.nst, max(0, hi - c.ubase + 3) / 4);
      if (kst < c.nst) {
        kend = kst;
      } else {
        const int r0 = c.ubase + c.np * GPP;
        kend = c.nst + min(c.nres, max(0, (hi - r0 + kPieceWeight - 1) / kPieceWeight));
      }
      const int cnt = min(kend - c.k, kSegItems - n);
      UnitSpan& sp = sh.span[ns];
      sp.off = n;
      sp.b = c.b;
      sp.h = c.h;
      sp.k0 = c.k;
      sp.n = cnt;
      sp.np = c.np;
      sp.rl = c.rl;
      sp.first = (c.k == 0) || (cta_first && n == 0);
      sp.last = (c.k + cnt == kend);
      if (sp.first) qcont = (++uord) % 3;
      sp.qslot = qcont;
      const int uw = unit_weight<P>(c);
      const int last_start =
          c.ubase + uw - kMergeWeight - (c.nres > 0 ? kPieceWeight : (c.np - (c.nst - 1) * PPC) * GPP);
      sp.io = uint32_t(ow.of(c.ubase)) | (uint32_t(ow.of(last_start)) << 16);
      n += cnt;
      ++ns;
      c.k += cnt;
      if (c.k == nitems) {
        c.s = c.ubase + uw;
        c.ubase = c.s;
        c.k = 0;
        if (++c.h == p.Hkv) {
          c.h = 0;
          ++c.b;
          // next sequence with items
          while (c.b < p.batch && seq_info<P>(p, c.b, one_pass ? 0 : sh.b0, sh.seq, c.np, c.rl) == 0) ++c.b;
          if (c.b >= p.batch) c.np = c.rl = 0;
          c.nst = (c.np * P + 127) / 128;
          c.nres = (c.rl + kPieceTokens - 1) / kPieceTokens;
        }
      } else if (c.k == kend) {
        c.s = hi;  // the range ends inside this unit
      } else {
        c.s = c.ubase + (c.k < c.nst ? 4 * c.k : c.np * GPP + kPieceWeight * (c.k - c.nst));
      }
    }
    sh.cur = c;
    sh.nseg = n;
    sh.nspan = ns;
    sh.more = c.s < hi;
    sh.uord = uord;
    sh.qslot_cont = qcont;
  }
  __syncthreads();
  const int n = sh.nseg, ns = sh.nspan;
  for (int t = tid; t < n; t += kDecodeThreads) {
    int si = 0;
    while (si + 1 < ns && sh.span[si + 1].off <= t) ++si;
    const UnitSpan& sp = sh.span[si];
    const int k = sp.k0 + (t - sp.off);
    const int nst = (sp.np * P + 127) / 128;
    ItemDesc d;
    d.b = sp.b;
    d.h = sp.h;
    d.io = sp.io;
    uint32_t w = uint32_t(sp.qslot) << 11;
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
        sh.ids[t][i] = id;
      }
    } else {
      const int j = k - nst;
      w |= uint32_t(min(kPieceTokens, sp.rl - kPieceTokens * j)) | kDescRes | (uint32_t(j) << 16);
    }
    sh.desc[t] = d;
    sh.desc[t].w = w;
  }
  __syncthreads();
}

// Issues the copies of item x (descriptor slot t of the segment) into stage x % kStages:
// the page records or residual rows, and the unit's query heads with its first item.
// All lanes of the calling warp take part.
template <int GQA, int KB, int P>
__device__ __forceinline__ void issue_item(const DecodeParams& p, CtaShared<GQA, P>& sh, uint8_t* smem, int x, int t,
                                           uint64_t policy, int lane) {
  using R = Rec<P, KB>;
  using S = Smem<GQA, P, KB>;
  const ItemDesc d = sh.desc[t];
  const int st = x % kStages, n = d.w & 0xff;
  const bool res = d.w & kDescRes, first = d.w & kDescFirst;
  uint8_t* sb = smem + st * S::stage;
  const uint32_t bytes = (res ? 0u : uint32_t(n) * R::payload) + (first ? GQA * 256u : 0u);
  if (lane == 0) {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (!res) mbar_arrive_expect_tx(&sh.full_bar[st], bytes);
    atomicAdd(&sh.issued, 1);
  }
  __syncwarp();
  if (!res) {
    if (lane < n)
      bulk_g2s(sb + lane * R::record, p.pool + (size_t(sh.ids[t][lane]) * p.Hkv + d.h) * R::record, R::payload,
               &sh.full_bar[st], policy);
  } else {
    // residual rows: 16-byte asynchronous copies into the padded rows, zero-filled past
    // the last token; each lane's copies arrive on the stage's barrier when they land
    const int t0 = kPieceTokens * int(d.w >> 16);
    const uint16_t* kr;
    const uint16_t* vr;
    if (p.seq_len) {
      // dense: page t0 / P of the sequence holds K rows then V rows ([2][P][128]); a piece
      // never crosses a page (P is a multiple of the piece length)
      int id = __ldcg(p.page_table + size_t(d.b) * p.max_pages + t0 / P);
      if (id < 0 || id >= p.pool_pages) {
        if (lane == 0) flag_error(p.err, KVQ_DEV_ERR_PAGE_RANGE);
        id = 0;
      }
      kr = reinterpret_cast<const uint16_t*>(p.pool) + ((size_t(id) * p.Hkv + d.h) * 2 * P + t0 % P) * kHeadDim;
      vr = kr + size_t(P) * kHeadDim;
    } else {
      kr = p.res_k + ((size_t(d.b) * p.Hkv + d.h) * P + t0) * kHeadDim;
      vr = p.res_v + ((size_t(d.b) * p.Hkv + d.h) * P + t0) * kHeadDim;
    }
#pragma unroll 4
    for (int i = lane; i < 2 * kPieceTokens * 16; i += 32) {
      const int which = i >> 8, row = (i >> 4) & 15, chunk = i & 15;
      const uint16_t* src = (which ? vr : kr) + (row < n ? row : 0) * kHeadDim + chunk * 8;
      cp_async16(sb + (which * kPieceTokens + row) * kResRowBytes + chunk * 16, src, row < n ? 16u : 0u);
    }
    cp_async_arrive(&sh.full_bar[st]);
  }
  if (res) {
    // every lane's asynchronous arrival is registered: now the one expected arrival
    __syncwarp();
    if (lane == 0) mbar_arrive_expect_tx(&sh.full_bar[st], bytes);
    __syncwarp();
  }
  if (first && lane == 31) {
    const uint16_t* src = p.q + (size_t(d.b) * p.Hq + size_t(d.h) * GQA) * kHeadDim;
    bulk_g2s(sh.q[(d.w >> 11) & 3], src, GQA * 256u, &sh.full_bar[st], policy);
  }
}

// Merges heads h0 .. h0 + HC - 1 of the nc partial states at pu (log-sum-exp) into outu.
// One warp; lane i holds channels 4i .. 4i + 3.
template <int HC, int UNROLL>
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
  // every contributor's loads of a batch are in flight together
#pragma unroll UNROLL
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

// One warp: counts this contributor in for unit u and, if it is the last of the
// contributors i0..i1, merges their partial states (log-sum-exp) into the output.
// (Written out rather than through merge_heads: inlined into the item loop, the helper
// changes the loop's register allocation enough to spill at 128 registers.)
template <int GQA>
__device__ __forceinline__ void merge_partials(const DecodeParams& p, int u, int i0, int i1, float* outu, int lane) {
  uint32_t arrived = 0;
  if (lane == 0) arrived = atomic_add_acq_rel_gpu(p.cnt + u, 1u);
  arrived = __shfl_sync(kFull, arrived, 0);
  const int nc = i1 - i0 + 1;
  if (arrived != uint32_t(nc - 1)) return;
  const float* pu = p.part + (size_t(i0) + u) * GQA * kPartStride;
  const size_t slot = size_t(GQA) * kPartStride;  // floats per contributor
  // up to four heads at a time, so that every contributor's loads are in flight together
  constexpr int HC = GQA < 4 ? GQA : 4;
#pragma unroll
  for (int h0 = 0; h0 < GQA; h0 += HC) {
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
  if (lane == 0) p.cnt[u] = 0u;  // ready for the next launch
}

// The same with the whole CTA, for a unit end that is the CTA's last item (all four
// warps are free): thread 96 counts in; if the CTA is the last contributor, warp w
// merges heads w, w + 4, ...
template <int GQA>
__device__ __noinline__ void merge_partials_cta(const DecodeParams& p, int* flag, int u, int i0, int i1, float* outu,
                                                   int warp, int lane) {
  const int nc = i1 - i0 + 1;
  if (warp == 3 && lane == 0) *flag = int(atomic_add_acq_rel_gpu(p.cnt + u, 1u));
  named_sync();  // the count (and, through it, the other contributors' partials) is seen by all
  if (*flag != nc - 1) return;
  const float* pu = p.part + (size_t(i0) + u) * GQA * kPartStride;
  for (int h = warp; h < GQA; h += 4) merge_heads<1, 8>(pu, size_t(GQA) * kPartStride, nc, h, outu, lane);
  if (warp == 3 && lane == 0) p.cnt[u] = 0u;  // ready for the next launch
}

template <typename T, int GQA, int KB, int P>
__global__ void __launch_bounds__(kDecodeThreads, (GQA <= 4 ? 4 : 2))
    decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NT = GQA > 4 ? 2 : 1;
  using R = Rec<P, KB>;
  using S = Smem<GQA, P, KB>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ CtaShared<GQA, P> sh;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, qd = lane & 3;
  const int cta = range_of_cta(blockIdx.x, p.n_ctas, p.n_sms);
  // the grid fills every resident slot at once, so the next kernel in the stream may be
  // scheduled right away: its CTAs take the slots this grid releases
  pdl_wait();
  pdl_trigger();

  // ---------------------------------------------------------------- 1. the weight line
  // Total weight W; with one sequence per thread (batch <= 128) the per-sequence prefix
  // and lengths stay in shared memory for locating any position later.
  int W = 0, x0 = 0, np0 = 0, rl0 = 0;
  const bool one_pass = p.batch <= kDecodeThreads;
  for (int base = 0; base < p.batch; base += kDecodeThreads) {
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
      np0 = np;
      rl0 = rl;
    }
    x0 = x;
    int incl = x;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(kFull, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) sh.red[warp] = incl;
    __syncthreads();
    if (one_pass) {
      int before = 0;
      for (int w = 0; w < warp; ++w) before += sh.red[w];
      if (b < p.batch) {
        sh.pref[b] = before + incl - x;
        sh.seq[b] = make_int2(np0, rl0);
      }
    }
    W += sh.red[0] + sh.red[1] + sh.red[2] + sh.red[3];
    __syncthreads();
  }
  if (W == 0) return;

  // At most W/4 CTAs take part, so that every range is at least one full stage long.
  Owners ow;
  ow.W = W;
  ow.Cs = min(p.n_ctas, max(1, W / 4));
  if (cta >= ow.Cs) return;
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sh.full_bar[s], 1);
      sh.rel[s] = 0;
    }
    fence_mbar_init();
    sh.abort_flag = 0;
    sh.issued = 0;
    sh.tail_u = -1;
  }

  // Moves sh.cur to the first item at or after position pos (all threads).
  auto locate = [&](int pos) {
    if (one_pass) {
      __syncthreads();
      if (tid < p.batch) {
        const int st0 = sh.pref[tid], w = unit_weight_of<P>(sh.seq[tid]) * p.Hkv;
        if (w > 0 && st0 <= pos && pos < st0 + w) {
          sh.b0 = tid;
          sh.base0 = st0;
        }
      }
    } else {
      int run = 0;
      for (int base = 0; base < p.batch; base += kDecodeThreads) {
        const int b = base + tid;
        int x = 0;
        if (b < p.batch) x = max(seq_weight<P>(p, b, np0, rl0), 0) * p.Hkv;
        int incl = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(kFull, incl, off);
          if (lane >= off) incl += y;
        }
        if (lane == 31) sh.red[warp] = incl;
        __syncthreads();
        int before = run;
        for (int w = 0; w < warp; ++w) before += sh.red[w];
        const int end = before + incl, start = end - x;
        if (x > 0 && start <= pos && pos < end) {
          sh.b0 = b;
          sh.base0 = start;
        }
        run += sh.red[0] + sh.red[1] + sh.red[2] + sh.red[3];
        __syncthreads();
      }
      // lengths of the sequences from the located one on
      for (int i = tid; i < kSeqCache && sh.b0 + i < p.batch; i += kDecodeThreads) {
        int np, rl;
        seq_weight<P>(p, sh.b0 + i, np, rl);
        sh.seq[i] = make_int2(np, rl);
      }
    }
    __syncthreads();
    if (tid == 0) {
      Cursor c;
      c.b = sh.b0;
      const int2 v = sh.seq[one_pass ? sh.b0 : 0];
      c.np = v.x;
      c.rl = v.y;
      c.nst = (c.np * P + 127) / 128;
      c.nres = (c.rl + kPieceTokens - 1) / kPieceTokens;
      c.k = 0;
      const int wseq = unit_weight<P>(c);
      const int off = pos - sh.base0;
      c.h = off / wseq;
      c.ubase = sh.base0 + c.h * wseq;
      cursor_seek<P>(p, c, off - c.h * wseq);
      sh.cur = c;
      sh.uord = -1;
      sh.qslot_cont = 0;
    }
    __syncthreads();
  };

  // ---------------------------------------------------------------- 2. items
  LaneQ<NT> lq;
  WarpState<NT> st;
  float* sO = reinterpret_cast<float*>(smem + S::merge);  // [4][GQA][128]
  const uint64_t policy = l2_evict_first_policy();
  int x = 0;  // items of this CTA so far
  const int owner = cta;
  const int lo = range_start(cta, ow.W, ow.Cs), hi = range_start(cta + 1, ow.W, ow.Cs);
  {
    locate(lo);
    while (true) {
      build_segment<GQA, P>(p, sh, hi, ow, tid, one_pass);
      const int nseg = sh.nseg;
      if (warp == 0)
        for (int t = 0; t < min(kStages, nseg); ++t) issue_item<GQA, KB, P>(p, sh, smem, x + t, t, policy, lane);
      int stg = x % kStages;
      uint32_t par = uint32_t(x / kStages) & 1u;
      for (int t = 0; t < nseg; ++t) {
        const int xi = x + t;
        const ItemDesc d = sh.desc[t];
        bool ok = !*reinterpret_cast<volatile int*>(&sh.abort_flag);
        if (ok && !mbar_wait_bounded(&sh.full_bar[stg], par)) {
          if (lane == 0) flag_error(p.err, KVQ_DEV_ERR_TIMEOUT);
          sh.abort_flag = 1;
          ok = false;
        }
        ok = __all_sync(kFull, ok);
        const uint8_t* sb = smem + stg * S::stage;
        const uint16_t* qs = sh.q[(d.w >> 11) & 3];
        const int n = d.w & 0xff;
        if (d.w & kDescFirst) {
          // query scale exponent of every head (each warp computes all of them)
          int eh[GQA];
#pragma unroll
          for (int h = 0; h < GQA; ++h) {
            const uint2 v = lds64(qs + h * kHeadDim + 4 * lane);
            const float2 a = t2_to_float2(v.x, T()), b2 = t2_to_float2(v.y, T());
            const float m = fmaxf(fmaxf(fabsf(a.x), fabsf(a.y)), fmaxf(fabsf(b2.x), fabsf(b2.y)));
            const uint32_t mb = __reduce_max_sync(kFull, __float_as_uint(m));
            const int e = int((mb >> 23) & 0xff) - 126;  // max |q| < 2^e
            if (e > 24 && lane == 0) flag_error(p.err, KVQ_DEV_ERR_RANGE);
            eh[h] = min(max(e, 0), 24);
          }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const int hB = (g >> 1) + 4 * nt, hL = qd + 4 * nt;
            int eB = 0, eL = 0;
#pragma unroll
            for (int h = 0; h < GQA; ++h) {
              eB = h == hB ? eh[h] : eB;
              eL = h == hL ? eh[h] : eL;
            }
            lq.cl[nt] = p.c_log2 * pow2f(eL);
            const float sc = pow2f(-eB);
            lq.sbq[nt] = h2_as_u32(__float2half2_rn(sc));
            lq.sq[nt] = sc;
#pragma unroll
            for (int s = 0; s < 8; ++s) {
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                uint32_t x = 0u;
                if (hB < GQA) {
                  const float2 v = t2_to_float2(lds32(qs + hB * kHeadDim + 16 * s + 2 * qd + 8 * j), T());
                  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(x) : "f"(v.y * sc), "f"(v.x * sc));
                }
                lq.qv(nt, s, j) = x;
              }
            }
          }
          lq.negmask = (g & 1) ? 0xbc00bc00u : 0u;  // fp16x2 (-1, -1) on lo-part lanes
          reset_state(st);
        }
        if (ok) {
          if (!(d.w & kDescRes)) {
            const int pw = (32 * warp) / P, grp = ((32 * warp) % P) / 32;
            if (pw < n) page_group<T, GQA, KB, P>(sb + pw * R::record, grp, lq, qs, st, lane, p.err);
          } else if (int(d.w >> 16) % 4 == warp) {
            residual_piece<T, GQA>(sb, sb + kPieceTokens * kResRowBytes, n, qs, st, lane, p.c_log2, p.err);
          }
        }
        // release the stage; the last warp to release it refills it with item xi + kStages
        __syncwarp();
        int prev = 0;
        if (lane == 0) prev = atomic_add_acq_rel_cta(&sh.rel[stg], 1);
        prev = __shfl_sync(kFull, prev, 0);
        if (prev == 3) {
          if (lane == 0) sh.rel[stg] = 0;
          if (t + kStages < nseg) issue_item<GQA, KB, P>(p, sh, smem, xi + kStages, t + kStages, policy, lane);
        }
        if (++stg == kStages) {
          stg = 0;
          par ^= 1u;
        }

        if (d.w & kDescLast) {
          // ---- merge the four warps' states for this unit
          named_sync();  // the previous merge no longer reads the merge buffer
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            float l = st.l[nt], zv = st.zv[nt];
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) {
              l += __shfl_xor_sync(kFull, l, off);
              zv += __shfl_xor_sync(kFull, zv, off);
            }
            const int head = qd + 4 * nt;
            if (g == 0 && head < GQA) {
              sh.m[warp][head] = st.m[nt];
              sh.l[warp][head] = l;
              sh.zv[warp][head] = zv;
            }
            if (head < GQA) {
#pragma unroll
              for (int mc = 0; mc < 8; ++mc)
#pragma unroll
                for (int r = 0; r < 2; ++r)
                  sO[(warp * GQA + head) * kHeadDim + 16 * mc + g + 8 * r] =
                      (st.o[mc][nt][2 * r] + st.o[mc][nt][2 * r + 1]) * pow2f(st.F);
            }
          }
          named_sync();
          const int u = d.b * p.Hkv + d.h;
          const int i0 = int(d.io & 0xffffu), i1 = int(d.io >> 16);
          const bool sole = i0 == i1;
          float* outu = p.out + (size_t(d.b) * p.Hq + size_t(d.h) * GQA) * kHeadDim;
          float* part_me = p.part + (size_t(owner) + u) * GQA * kPartStride;
          for (int e = tid; e < GQA * kHeadDim; e += kDecodeThreads) {
            const int h = e >> 7, ch = e & 127;
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < 4; ++w) M = fmaxf(M, sh.m[w][h]);
            float Ls = 0.0f, O = 0.0f;
            if (M != -INFINITY) {
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                const float f = ex2(sh.m[w][h] - M);
                Ls += f * sh.l[w][h];
                O += f * (kCodeScale * sO[(w * GQA + h) * kHeadDim + ch] + sh.zv[w][h]);
              }
            }
            if (sole) {
              outu[e] = Ls > 0.0f ? O / Ls : 0.0f;
            } else {
              float* pp = part_me + h * kPartStride;
              pp[ch] = O;
              if (ch == 0) {
                pp[kHeadDim] = M;
                pp[kHeadDim + 1] = Ls;
              }
            }
          }
          if (!sole) {
            // ---- split merge: the last of the contributors i0..i1 merges their partials.
            // The barrier orders every thread's partial writes before the counter update,
            // which is a release at device scope; the merging CTA acquires it.
            named_sync();
            if (t == nseg - 1 && !sh.more) {
              // the CTA's last item: all warps merge, after the loop
              if (tid == 0) {
                sh.tail_u = u;
                sh.tail_io = d.io;
              }
            } else if (warp == 3) {
              merge_partials<GQA>(p, u, i0, i1, outu, lane);
            }
          }
        }
      }
      x += nseg;
      if (!sh.more) break;
      __syncthreads();  // every item of the segment is consumed before its slots are reused
    }
  }

  named_sync();
  if (sh.tail_u >= 0) {
    const int u = sh.tail_u, b = u / p.Hkv, h = u - b * p.Hkv;
    const uint32_t io = sh.tail_io;
    merge_partials_cta<GQA>(p, &sh.arrived, u, int(io & 0xffffu), int(io >> 16),
                            p.out + (size_t(b) * p.Hq + size_t(h) * GQA) * kHeadDim, warp, lane);
  }

  // ---------------------------------------------------------------- 3. leave
  __syncthreads();
  if (sh.abort_flag && warp == 0) {
    // copies may still be in flight after a timeout: wait for them (bounded) before the
    // shared memory is released; the output is undefined and the error word says why
    const int issued = sh.issued;
    for (int y = max(0, issued - kStages); y < issued; ++y) {
      if (lane == 0) mbar_wait_bounded(&sh.full_bar[y % kStages], uint32_t(y / kStages) & 1u);
    }
  }
}

// ---------------------------------------------------------------- per-instantiation host side

template <typename T, int GQA, int KB, int P>
cudaError_t prepare_decode() {
  static int seen[64];
  return ensure_dynamic_smem(decode_kernel<T, GQA, KB, P>, int(Smem<GQA, P, KB>::bytes), seen);
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
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, decode_kernel<T, GQA, KB, P>, kDecodeThreads,
                                                         Smem<GQA, P, KB>::bytes);
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
    return launch_pdl(decode_kernel<T, GQA, KB, P>, dim3(p.n_ctas), dim3(kDecodeThreads), Smem<GQA, P, KB>::bytes,
                      stream, p);
  }
};

// One translation unit per (dtype, GQA) defines these two entry points.
#define KVQ_DECODE_INSTANCE(NAME, T, GQA)                                                       \
  cudaError_t decode_occupancy_##NAME(int kb, int P, int* n) {                                 \
    return dispatch_kb_p(kb, P, DecodeOcc<T, GQA>{n});                                          \
  }                                                                                             \
  cudaError_t decode_launch_##NAME(const DecodeParams& p, cudaStream_t stream) {               \
    return dispatch_kb_p(p.KB, p.P, DecodeRun<T, GQA>{p, stream});                              \
  }

}  // namespace kvq
