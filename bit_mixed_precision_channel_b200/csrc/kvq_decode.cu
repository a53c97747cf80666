// kvq_decode.cu — decode attention over the paged 2-bit cache, sm_100a.
//
// One CTA = (sequence b, kv head, split of the page list); 4 warps.  Pages stream
// through a 4-stage shared-memory ring filled by the bulk-copy engine (one
// cp.async.bulk per page record, completion on a "full" mbarrier, L2 evict-first
// hint); a stage holds 128 tokens (1, 2 or 4 pages).  Each warp owns one 32-token key
// group of the stage, keeps its own online-softmax state and releases the stage on an
// "empty" mbarrier, so warps run decoupled; thread 0 refills released stages.  The
// warps' states are merged in shared memory at the end, and the splits of a sequence
// are merged by the last CTA to finish (log-sum-exp merge, no second launch).
//
// The 2-bit codes never become floating-point values with a scale applied.  The
// scales are folded into the other operand of each product, and the codes go to the
// tensor cores as they are (Kitty abstract: page dequantization kernels with uniform
// 2-bit dequantization; MiniKV proposed method: dequantization fused into the matmul):
//   q.k_t   = sum_c code_A[t,c] * (q_c * sA_{g,c}) + sum_j code_B[t,j] * (q_{idx_j} * sB_{g,j})
//             + sum_c q_c * zA_{g,c}
//   sum_t p_t v_t[c] = sum_t code_V[t,c] * (p_t * sV_t) + sum_t p_t * zV_t
// With the 4-bit boosted channels stored as two 2-bit planes, the boosted low bits
// are simply k more rows of the same contraction.  The folded operands are carried
// as a high and a low fp16 part (hi = fp16(x), lo = fp16(x - hi)), so the products
// keep ~22 bits; codes reach the tensor cores exactly (as 0.5 * code through the FP4
// conversion, the 0.5 undone afterwards).  Matrix shapes per warp and 32-token group:
// QK^T = [32 tokens x (128 + k) channels] x [(128 + k) x 8 columns],
// PV = [128 channels x 32 tokens] x [32 tokens x 8 columns], where the 8 columns hold
// the hi and lo parts of up to 4 query heads (two column tiles for 8 heads).
#include <algorithm>

#include "kvq_internal.cuh"

namespace kvq {

constexpr int kStages = 4;
constexpr int kDecodeThreads = 128;
constexpr int kResRowBytes = 272;    // residual row in shared memory: 256 bytes + 16 pad
constexpr int kResRoundTokens = 64;  // residual tokens staged per round (16 per warp)

// ---------------------------------------------------------------- operand builders

// Query-side operand of one k-step pair: hi = fp16(q*s) and lo = fp16(q*s - hi).
// For fp16 data the product of two fp16 values is exact in 22 bits; hmul2 rounds it
// once and hfma2 returns the rest.
__device__ __forceinline__ void fold_hilo(uint32_t q2, uint32_t s2, uint32_t& hi, uint32_t& lo, __half) {
  const __half2 q = u32_as_h2(q2), s = u32_as_h2(s2);
  const __half2 h = __hmul2(q, s);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__hfma2(q, s, __hneg2(h)));
}
__device__ __forceinline__ void fold_hilo(uint32_t q2, uint32_t s2, uint32_t& hi, uint32_t& lo,
                                          __nv_bfloat16) {
  // bf16 x bf16 is exact in fp32 (16 significant bits); split it into two fp16 parts
  const float q0 = __uint_as_float(q2 << 16), q1 = __uint_as_float(q2 & 0xffff0000u);
  const float s0 = __uint_as_float(s2 << 16), s1 = __uint_as_float(s2 & 0xffff0000u);
  const float x0 = q0 * s0, x1 = q1 * s1;
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
}

// For GQA <= 4 one column tile carries hi (columns 0..3) and lo (columns 4..7):
// hfma2(q, s, -hi * m) with m = 0 or 1 per lane gives either part without a branch.
__device__ __forceinline__ uint32_t fold_one(uint32_t q2, uint32_t s2, uint32_t negmask, __half) {
  const __half2 q = u32_as_h2(q2), s = u32_as_h2(s2);
  const __half2 h = __hmul2(q, s);
  return h2_as_u32(__hfma2(q, s, __hmul2(h, u32_as_h2(negmask))));
}
__device__ __forceinline__ uint32_t fold_one(uint32_t q2, uint32_t s2, uint32_t negmask, __nv_bfloat16) {
  uint32_t hi, lo;
  fold_hilo(q2, s2, hi, lo, __nv_bfloat16());
  return negmask ? lo : hi;
}

// fp16 hi/lo split of two fp32 values (probability-side operand of the code planes).
__device__ __forceinline__ void split_f16(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __half2 h = __floats2half2_rn(x0, x1);
  const float2 hf = __half22float2(h);
  hi = h2_as_u32(h);
  lo = h2_as_u32(__floats2half2_rn(x0 - hf.x, x1 - hf.y));
}
// Same in the residual's 16-bit type (its values are the other operand there).
__device__ __forceinline__ void split_t(float x0, float x1, uint32_t& hi, uint32_t& lo, __half) {
  split_f16(x0, x1, hi, lo);
}
__device__ __forceinline__ void split_t(float x0, float x1, uint32_t& hi, uint32_t& lo, __nv_bfloat16) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
  const float2 hf = __bfloat1622float2(h);
  hi = bf2_as_u32(h);
  lo = bf2_as_u32(__floats2bfloat162_rn(x0 - hf.x, x1 - hf.y));
}

__device__ __forceinline__ float t_to_float(uint16_t b, __half) { return __half2float(__ushort_as_half(b)); }
__device__ __forceinline__ float t_to_float(uint16_t b, __nv_bfloat16) { return __uint_as_float(uint32_t(b) << 16); }

// ---------------------------------------------------------------- per-warp state

template <int GQA>
struct WarpState {
  static constexpr int NT = GQA <= 4 ? 1 : 2;
  float o[8][NT][4];  // PV accumulator: rows = channels 16*mc + g (+8), cols 2*qd, 2*qd+1
  float m[2], l[2], zv[2];
};

// Per-lane constants of the query-side operand.
struct LaneQ {
  uint32_t qv[8][2];  // q pairs of this lane's B column for k-step s: channels 16s+2qd(+1), +8
  uint32_t negmask;   // fp16x2 -1 for the lo-part columns (GQA <= 4), 0 otherwise
  float zmul;         // weight of this lane's zero-point column in the logits
};

// Online-softmax update from the logits of MT 16-token tiles held by this lane
// (rows g, g+8 of each tile; heads hc0, hc1).  Logits are in log2 units.  The running
// maximum moves only when a logit exceeds it by more than 8, so probabilities stay
// below 2^8 and most groups skip the rescale of the accumulators.
template <int GQA, int MT>
__device__ __forceinline__ void softmax_step(WarpState<GQA>& st, const float (&L)[MT][4]) {
  float mx[2] = {L[0][0], L[0][1]};
#pragma unroll
  for (int mt = 0; mt < MT; ++mt) {
    mx[0] = fmaxf(mx[0], fmaxf(L[mt][0], L[mt][2]));
    mx[1] = fmaxf(mx[1], fmaxf(L[mt][1], L[mt][3]));
  }
  float alpha[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) mx[j] = fmaxf(mx[j], __shfl_xor_sync(kFull, mx[j], off));
    if (mx[j] > st.m[j] + 8.0f) {
      alpha[j] = ex2(st.m[j] - mx[j]);  // 0 on the first group (m = -inf)
      st.m[j] = mx[j];
      st.l[j] *= alpha[j];
      st.zv[j] *= alpha[j];
    } else {
      alpha[j] = 1.0f;
    }
  }
  if (!__all_sync(kFull, alpha[0] == 1.0f && alpha[1] == 1.0f)) {
#pragma unroll
    for (int mc = 0; mc < 8; ++mc)
#pragma unroll
      for (int nt = 0; nt < WarpState<GQA>::NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) st.o[mc][nt][i] *= alpha[i & 1];
  }
}

// ---------------------------------------------------------------- one quantized group

// Processes tokens [t0, t0+32) of the page record `rec` (in shared memory).
// KB = boosted channels / 16.
template <typename T, int GQA, int KB>
__device__ __forceinline__ void page_group(const DecodeParams& p, const uint8_t* rec, int t0, const LaneQ& lq,
                                           const uint16_t* q_s, int hB, bool validB, WarpState<GQA>& st, int g,
                                           int qd) {
  constexpr int NT = WarpState<GQA>::NT;
  const int grp = t0 >> 5;
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[mt][nt][i] = 0.0f;

  // -- q . K^T over plane A: this lane's codes are words 2qd, 2qd+1 of each token row,
  //    its scales positions 32qd .. 32qd+31 of the group's scale row --
  const uint8_t* kA = rec + p.L.k_codes;
  const uint4* psc = reinterpret_cast<const uint4*>(rec + p.L.k_scale + (grp * kHeadDim + 32 * qd) * 2);
  uint2 w[2][2];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int r = 0; r < 2; ++r) w[mt][r] = lds64(kA + ((t0 + 16 * mt + g + 8 * r) * 8 + 2 * qd) * 4);
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    uint32_t sc[8];
    {
      const uint4 a = psc[2 * half], b = psc[2 * half + 1];
      sc[0] = a.x; sc[1] = a.y; sc[2] = a.z; sc[3] = a.w;
      sc[4] = b.x; sc[5] = b.y; sc[6] = b.z; sc[7] = b.w;
    }
#pragma unroll
    for (int pass = 0; pass < 2; ++pass) {
      uint32_t c[2][2][4];  // [mt][row][byte]: byte 2j + r -> k-step 4*half + 2*pass + j, reg r
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const uint32_t word = half ? w[mt][r].y : w[mt][r].x;
          e2m1_pairs(code_pass(word, pass), c[mt][r][0], c[mt][r][1], c[mt][r][2], c[mt][r][3]);
        }
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int s = 4 * half + 2 * pass + jj, sl = 2 * pass + jj;
        uint32_t b[NT][2];
        if constexpr (NT == 1) {
          b[0][0] = fold_one(lq.qv[s][0], sc[2 * sl], lq.negmask, T());
          b[0][1] = fold_one(lq.qv[s][1], sc[2 * sl + 1], lq.negmask, T());
        } else {
          fold_hilo(lq.qv[s][0], sc[2 * sl], b[0][0], b[1][0], T());
          fold_hilo(lq.qv[s][1], sc[2 * sl + 1], b[0][1], b[1][1], T());
        }
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const uint32_t a[4] = {c[mt][0][2 * jj], c[mt][1][2 * jj], c[mt][0][2 * jj + 1], c[mt][1][2 * jj + 1]};
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a, b[nt][0], b[nt][1], __half());
        }
      }
    }
  }
  // -- plane B: low bits of the boosted channels; rows 16s + 8r + 2qd + f of this lane
  //    sit at positions 4*KB*qd + 4s + 2r + f of each token row --
  if constexpr (KB > 0) {
    const uint8_t* kB = rec + p.L.kb_codes;
    const uint8_t* idx = rec + p.L.boost_idx;
    const uint8_t* kbsc = rec + p.L.kb_scale + grp * (16 * KB) * 2;
    const uint16_t* qh = q_s + hB * kHeadDim;
    uint32_t cb[2][2][KB][2];  // [mt][row][s][r]
#pragma unroll
    for (int mt = 0; mt < 2; ++mt)
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        const uint8_t* row = kB + (t0 + 16 * mt + g + 8 * rr) * KB * 4;
        if constexpr (KB == 1) {
          // positions 4qd .. 4qd+3: word 0, pass qd >> 1, bytes 2(qd & 1), +1
          const uint32_t x = code_pass(lds32(row), qd >> 1) >> (16 * (qd & 1));
          cb[mt][rr][0][0] = e2m1_pair_lo(x);
          cb[mt][rr][0][1] = e2m1_pair_lo(x >> 8);
        } else {
          // k-steps s, s+1 (s even) share a word and a pass: bytes 0..3
#pragma unroll
          for (int s = 0; s < KB; s += 2) {
            const int pos = 4 * KB * qd + 4 * s;
            const uint32_t x = code_pass(lds32(row + (pos >> 4) * 4), (pos >> 3) & 1);
            e2m1_pairs(x, cb[mt][rr][s][0], cb[mt][rr][s][1], cb[mt][rr][s + 1][0], cb[mt][rr][s + 1][1]);
          }
        }
      }
#pragma unroll
    for (int s = 0; s < KB; ++s) {
      const int j0 = 16 * s + 2 * qd, j1 = j0 + 8;
      uint32_t q0 = 0, q1 = 0;
      if (validB) {
        // indices are < 128 in any record the library wrote; the mask keeps a corrupt
        // record from reading outside the query rows
        q0 = uint32_t(qh[idx[j0] & 127]) | (uint32_t(qh[idx[j0 + 1] & 127]) << 16);
        q1 = uint32_t(qh[idx[j1] & 127]) | (uint32_t(qh[idx[j1 + 1] & 127]) << 16);
      }
      const uint32_t s0 = lds32(kbsc + j0 * 2), s1 = lds32(kbsc + j1 * 2);
      uint32_t b[NT][2];
      if constexpr (NT == 1) {
        b[0][0] = fold_one(q0, s0, lq.negmask, T());
        b[0][1] = fold_one(q1, s1, lq.negmask, T());
      } else {
        fold_hilo(q0, s0, b[0][0], b[1][0], T());
        fold_hilo(q1, s1, b[0][1], b[1][1], T());
      }
#pragma unroll
      for (int mt = 0; mt < 2; ++mt) {
        const uint32_t a[4] = {cb[mt][0][s][0], cb[mt][1][s][0], cb[mt][0][s][1], cb[mt][1][s][1]};
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) mma_16816(acc[mt][nt], a, b[nt][0], b[nt][1], __half());
      }
    }
  }
  // -- zero-point term: Z[h] = sum_c q[h][c] * zA[g][c] (all rows of A equal) --
  float z[4] = {0.f, 0.f, 0.f, 0.f};
  {
    const uint4* pz = reinterpret_cast<const uint4*>(rec + p.L.k_zero + (grp * kHeadDim + 32 * qd) * 2);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint4 zz = pz[i];
      const uint32_t zr[4] = {zz.x, zz.y, zz.z, zz.w};
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int s = 2 * i + u;
        const uint32_t a[4] = {zr[2 * u], zr[2 * u], zr[2 * u + 1], zr[2 * u + 1]};
        mma_16816(z, a, lq.qv[s][0], lq.qv[s][1], T());
      }
    }
  }
  // -- logits (log2 units); code products carry a factor 0.5 --
  const float ccode = p.c_log2 * kCodeScale;
  float L[2][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v;
      if constexpr (NT == 1) {
        v = fmaf(acc[mt][0][i], ccode, z[i & 1] * lq.zmul);
        v += __shfl_xor_sync(kFull, v, 2);
      } else {
        v = fmaf(acc[mt][0][i] + acc[mt][1][i], ccode, z[i & 1] * lq.zmul);
      }
      L[mt][i] = v;
    }
  softmax_step<GQA, 2>(st, L);

  // -- probabilities, folded with the value scales, as the B operand of PV --
  const uint16_t* vs = reinterpret_cast<const uint16_t*>(rec + p.L.v_scale);
  const uint16_t* vz = reinterpret_cast<const uint16_t*>(rec + p.L.v_zero);
  uint32_t pb[2][NT][2];
  const bool loC = qd >= 2;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int ta = t0 + 16 * mt + g, tb = ta + 8;
    const float sa = t_to_float(vs[ta], T()), sb = t_to_float(vs[tb], T());
    const float za = t_to_float(vz[ta], T()), zb = t_to_float(vz[tb], T());
    const float p00 = ex2(L[mt][0] - st.m[0]), p01 = ex2(L[mt][1] - st.m[1]);
    const float p10 = ex2(L[mt][2] - st.m[0]), p11 = ex2(L[mt][3] - st.m[1]);
    st.l[0] += p00 + p10;
    st.l[1] += p01 + p11;
    st.zv[0] += p00 * za + p10 * zb;
    st.zv[1] += p01 * za + p11 * zb;
    uint32_t th, tl, bh, bl;
    split_f16(p00 * sa, p01 * sa, th, tl);
    split_f16(p10 * sb, p11 * sb, bh, bl);
    if constexpr (NT == 1) {
      pb[mt][0][0] = movmatrix_trans(loC ? tl : th);
      pb[mt][0][1] = movmatrix_trans(loC ? bl : bh);
    } else {
      pb[mt][0][0] = movmatrix_trans(th);
      pb[mt][0][1] = movmatrix_trans(bh);
      pb[mt][1][0] = movmatrix_trans(tl);
      pb[mt][1][1] = movmatrix_trans(bl);
    }
  }
  // -- P V: word 2*grp + qd/2 of each channel row holds this lane's 8 tokens (pass qd&1) --
  const uint8_t* vq = rec + p.L.v_codes + (2 * grp + (qd >> 1)) * 4;
  const int rowb = (p.P >> 4) * 4;  // bytes per channel row
  const int vpass = qd & 1;
#pragma unroll
  for (int mc = 0; mc < 8; ++mc) {
    uint32_t ca[4], cbv[4];
    e2m1_pairs(code_pass(lds32(vq + (16 * mc + g) * rowb), vpass), ca[0], ca[1], ca[2], ca[3]);
    e2m1_pairs(code_pass(lds32(vq + (16 * mc + g + 8) * rowb), vpass), cbv[0], cbv[1], cbv[2], cbv[3]);
#pragma unroll
    for (int ks = 0; ks < 2; ++ks) {
      const uint32_t a[4] = {ca[2 * ks], cbv[2 * ks], ca[2 * ks + 1], cbv[2 * ks + 1]};
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_16816(st.o[mc][nt], a, pb[ks][nt][0], pb[ks][nt][1], __half());
    }
  }
}

// ---------------------------------------------------------------- residual tokens

// Tokens [tok0, tok0+16) of the residual window, staged in shared memory at rows
// row0.. (rows of 272 B); rows at or beyond rl are zero and masked out of the softmax.
template <typename T, int GQA>
__device__ __forceinline__ void residual_tile(const DecodeParams& p, const uint8_t* Kr, const uint8_t* Vr,
                                              int row0, int tok0, int rl, const LaneQ& lq, bool loB, bool validB,
                                              WarpState<GQA>& st, int lane, int g, int qd) {
  constexpr int NT = WarpState<GQA>::NT;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const bool useq = validB && !loB;
  const int li = lane >> 3, lr = lane & 7;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    uint32_t a[4];
    const int row = row0 + lr + 8 * (li & 1);
    const int col = 16 * s + 8 * (li >> 1);
    ldmatrix_x4(a, smem_addr(Kr + row * kResRowBytes + col * 2));
    mma_16816(acc, a, useq ? lq.qv[s][0] : 0u, useq ? lq.qv[s][1] : 0u, T());
  }
  float L[1][4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float v = acc[i] * p.c_log2;
    if constexpr (NT == 1) v += __shfl_xor_sync(kFull, v, 2);
    const int tok = tok0 + g + 8 * (i >> 1);
    L[0][i] = tok < rl ? v : -INFINITY;
  }
  softmax_step<GQA, 1>(st, L);
  uint32_t pb[NT][2];
  const bool loC = qd >= 2;
  {
    const float p00 = ex2(L[0][0] - st.m[0]), p01 = ex2(L[0][1] - st.m[1]);
    const float p10 = ex2(L[0][2] - st.m[0]), p11 = ex2(L[0][3] - st.m[1]);
    st.l[0] += p00 + p10;
    st.l[1] += p01 + p11;
    uint32_t th, tl, bh, bl;
    split_t(p00, p01, th, tl, T());
    split_t(p10, p11, bh, bl, T());
    if constexpr (NT == 1) {
      pb[0][0] = movmatrix_trans(loC ? tl : th);
      pb[0][1] = movmatrix_trans(loC ? bl : bh);
    } else {
      pb[0][0] = movmatrix_trans(th);
      pb[0][1] = movmatrix_trans(bh);
      pb[1][0] = movmatrix_trans(tl);
      pb[1][1] = movmatrix_trans(bl);
    }
  }
#pragma unroll
  for (int mc = 0; mc < 8; ++mc) {
    uint32_t a[4];
    const int row = row0 + lr + 8 * (li >> 1);
    const int col = 16 * mc + 8 * (li & 1);
    ldmatrix_x4_trans(a, smem_addr(Vr + row * kResRowBytes + col * 2));
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) mma_16816(st.o[mc][nt], a, pb[nt][0], pb[nt][1], T());
  }
}

// ---------------------------------------------------------------- the kernel

template <typename T, int GQA, int KB>
__global__ void __launch_bounds__(kDecodeThreads, (GQA <= 4 ? 4 : 2))
    decode_kernel(const __grid_constant__ DecodeParams p) {
  constexpr int NT = WarpState<GQA>::NT;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ __align__(8) uint64_t full_bar[kStages];   // stage filled (bulk-copy bytes landed)
  __shared__ __align__(8) uint64_t empty_bar[kStages];  // stage released by all 4 warps
  __shared__ __align__(16) uint16_t q_s[GQA * kHeadDim];
  __shared__ float s_m[4][GQA], s_l[4][GQA], s_zv[4][GQA];
  __shared__ int s_abort, s_last;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, qd = lane & 3;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;

  const int np = p.num_pages[b], rl = p.res_len[b];
  if (np < 0 || np > p.max_pages || rl < 0 || rl > p.P) {
    if (tid == 0 && split == 0) flag_error(p.err, KVQ_DEV_ERR_LENGTH);
    return;
  }
  const int nsplit = max(1, (np + p.pps - 1) / p.pps);
  if (split >= nsplit) return;
  const int pg0 = split * p.pps;
  const int npg = max(0, min(np, pg0 + p.pps) - pg0);
  const bool own_res = (split == nsplit - 1) && rl > 0;

  uint8_t* main = smem;
  int* s_pages = reinterpret_cast<int*>(smem + p.main_bytes);
  for (int i = tid; i < npg; i += kDecodeThreads) {
    int id = p.page_table[size_t(b) * p.max_pages + pg0 + i];
    if (id < 0 || id >= p.pool_pages) {
      flag_error(p.err, KVQ_DEV_ERR_PAGE_RANGE);
      id = 0;
    }
    s_pages[i] = id;
  }
  {
    const uint4* qg = reinterpret_cast<const uint4*>(p.q + (size_t(b) * p.Hq + size_t(kvh) * GQA) * kHeadDim);
    for (int i = tid; i < GQA * kHeadDim / 8; i += kDecodeThreads) reinterpret_cast<uint4*>(q_s)[i] = qg[i];
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 4);
    }
    fence_mbar_init();
    s_abort = 0;
  }
  __syncthreads();

  const int ppc = 128 / p.P;
  const int n_chunks = (npg + ppc - 1) / ppc;
  const uint64_t policy = l2_evict_first_policy();
  auto issue = [&](int c) {
    const int st = c % kStages, first = c * ppc, nv = min(ppc, npg - first);
    mbar_arrive_expect_tx(&full_bar[st], uint32_t(nv) * p.payload);
    for (int i = 0; i < nv; ++i) {
      const uint8_t* src = p.pool + (size_t(s_pages[first + i]) * p.Hkv + kvh) * p.rec_bytes;
      bulk_g2s(main + st * p.stage_bytes + i * p.rec_bytes, src, p.payload, &full_bar[st], policy);
    }
  };
  // Thread 0 keeps the ring full: chunk x goes to stage x % kStages once the chunk
  // x - kStages that used the stage before has been released by all four warps.
  // It blocks only when a chunk up to `need` is not issued yet; further chunks up to
  // `ahead` are issued if their stage is already free.
  int issued = 0;
  auto refill = [&](int need, int ahead) -> bool {
    while (issued < n_chunks && issued <= ahead) {
      if (issued >= kStages) {
        const uint32_t par = uint32_t(issued / kStages - 1) & 1u;
        uint64_t* eb = &empty_bar[issued % kStages];
        if (issued <= need) {
          if (!mbar_wait_bounded(eb, par)) return false;
        } else if (!mbar_test_wait(eb, par)) {
          break;
        }
      }
      issue(issued++);
    }
    return true;
  };
  if (tid == 0) refill(-1, kStages - 1);

  // query fragments of this lane's B column (head hB; lo part for columns 4..7 when GQA <= 4)
  const int hB = GQA <= 4 ? (g & 3) : g;
  const bool loB = GQA <= 4 && g >= 4;
  const bool validB = hB < GQA;
  LaneQ lq;
#pragma unroll
  for (int s = 0; s < 8; ++s) {
    lq.qv[s][0] = validB ? lds32(q_s + hB * kHeadDim + 16 * s + 2 * qd) : 0u;
    lq.qv[s][1] = validB ? lds32(q_s + hB * kHeadDim + 16 * s + 2 * qd + 8) : 0u;
  }
  lq.negmask = loB ? 0xbc00bc00u : 0u;             // fp16x2 (-1, -1) or (0, 0)
  lq.zmul = (NT == 2 || qd < 2) ? p.c_log2 : 0.0f;  // lo columns carry no zero-point term

  WarpState<GQA> st;
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int i = 0; i < 4; ++i) st.o[mc][nt][i] = 0.0f;
  st.m[0] = st.m[1] = -INFINITY;
  st.l[0] = st.l[1] = st.zv[0] = st.zv[1] = 0.0f;

  // ---------------------------------------------------------------- page stream
  const int pi = (32 * warp) / p.P, t0 = (32 * warp) % p.P;
  for (int c = 0; c < n_chunks; ++c) {
    if (tid == 0 && !refill(c, c + kStages - 1)) {
      flag_error(p.err, KVQ_DEV_ERR_TIMEOUT);
      s_abort = 1;
      break;
    }
    const int stg = c % kStages;
    if (!mbar_wait_bounded(&full_bar[stg], uint32_t(c / kStages) & 1u)) {
      flag_error(p.err, KVQ_DEV_ERR_TIMEOUT);
      s_abort = 1;
      break;
    }
    if (c * ppc + pi < npg)
      page_group<T, GQA, KB>(p, main + stg * p.stage_bytes + pi * p.rec_bytes, t0, lq, q_s, hB, validB, st, g,
                             qd);
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty_bar[stg]);
  }
  __syncthreads();
  if (s_abort) {
    // drain the copies that may still be in flight (bounded), then leave; the
    // output is undefined and the error word says why
    if (tid == 0)
      for (int x = max(0, issued - kStages); x < issued; ++x)
        mbar_wait_bounded(&full_bar[x % kStages], uint32_t(x / kStages) & 1u);
    __syncthreads();
    return;
  }
  // page results carry the 0.5 of the code encoding; bring them to real units
  if (npg > 0) {
#pragma unroll
    for (int mc = 0; mc < 8; ++mc)
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) st.o[mc][nt][i] *= kCodeScale;
  }

  // ---------------------------------------------------------------- residual window
  if (own_res) {
    uint8_t* Kr = main;
    uint8_t* Vr = main + kResRoundTokens * kResRowBytes;
    const uint8_t* gk = reinterpret_cast<const uint8_t*>(p.res_k + (size_t(b) * p.Hkv + kvh) * p.P * kHeadDim);
    const uint8_t* gv = reinterpret_cast<const uint8_t*>(p.res_v + (size_t(b) * p.Hkv + kvh) * p.P * kHeadDim);
    for (int base = 0; base < rl; base += kResRoundTokens) {
      const int rows = min(kResRoundTokens, (rl - base + 15) & ~15);  // whole 16-row tiles
      for (int i = tid; i < rows * 32; i += kDecodeThreads) {
        const int which = i / (rows * 16), j = i % (rows * 16), t = j >> 4, c16 = j & 15;
        const int tok = base + t;
        const uint8_t* src = (which ? gv : gk) + tok * 256 + c16 * 16;
        uint8_t* dst = (which ? Vr : Kr) + t * kResRowBytes + c16 * 16;
        cp_async16(dst, tok < rl ? src : gk, tok < rl ? 16u : 0u);
      }
      cp_async_wait_all();
      __syncthreads();
      if (16 * warp < rows)
        residual_tile<T, GQA>(p, Kr, Vr, 16 * warp, base + 16 * warp, rl, lq, loB, validB, st, lane, g, qd);
      __syncthreads();
    }
  }

  // ---------------------------------------------------------------- merge the 4 warps
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      st.l[j] += __shfl_xor_sync(kFull, st.l[j], off);
      st.zv[j] += __shfl_xor_sync(kFull, st.zv[j], off);
    }
  __syncthreads();  // shared ring / residual rows are free
  float* sO = reinterpret_cast<float*>(main);  // [4][GQA][128]
  const int hq = NT == 1 ? 2 * (qd & 1) : 2 * qd;  // first head of this lane's columns
  const bool writer = NT == 2 || qd < 2;
#pragma unroll
  for (int mc = 0; mc < 8; ++mc)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float v;
      if constexpr (NT == 1) {
        v = st.o[mc][0][i];
        v += __shfl_xor_sync(kFull, v, 2);  // hi columns + lo columns
      } else {
        v = st.o[mc][0][i] + st.o[mc][1][i];
      }
      const int head = hq + (i & 1), ch = 16 * mc + g + 8 * (i >> 1);
      if (writer && head < GQA) sO[(warp * GQA + head) * kHeadDim + ch] = v;
    }
  if (g == 0 && writer) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int head = hq + j;
      if (head < GQA) {
        s_m[warp][head] = st.m[j];
        s_l[warp][head] = st.l[j];
        s_zv[warp][head] = st.zv[j];
      }
    }
  }
  __syncthreads();

  float* part_base = p.part + ((size_t(b) * p.Hkv + kvh) * p.max_splits) * GQA * (2 + kHeadDim);
  for (int e = tid; e < GQA * kHeadDim; e += kDecodeThreads) {
    const int h = e >> 7, c = e & 127;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) M = fmaxf(M, s_m[w][h]);
    float Ls = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = ex2(s_m[w][h] - M);
        Ls += f * s_l[w][h];
        O += f * (sO[(w * GQA + h) * kHeadDim + c] + s_zv[w][h]);
      }
    }
    if (nsplit == 1) {
      p.out[(size_t(b) * p.Hq + size_t(kvh) * GQA + h) * kHeadDim + c] = Ls > 0.0f ? O / Ls : 0.0f;
    } else {
      float* pp = part_base + (size_t(split) * GQA + h) * (2 + kHeadDim);
      if (c == 0) {
        pp[0] = M;
        pp[1] = Ls;
      }
      pp[2 + c] = O;
    }
  }
  if (nsplit == 1) return;

  // ---------------------------------------------------------------- split merge (last CTA)
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const uint32_t prev = atomicAdd(p.cnt + size_t(b) * p.Hkv + kvh, 1u);
    s_last = prev == uint32_t(nsplit - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int e = tid; e < GQA * kHeadDim; e += kDecodeThreads) {
    const int h = e >> 7, c = e & 127;
    float M = -INFINITY;
    for (int s = 0; s < nsplit; ++s) M = fmaxf(M, __ldcg(part_base + (size_t(s) * GQA + h) * (2 + kHeadDim)));
    float Ls = 0.0f, O = 0.0f;
    if (M != -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const float* pp = part_base + (size_t(s) * GQA + h) * (2 + kHeadDim);
        const float f = ex2(__ldcg(pp) - M);
        Ls += f * __ldcg(pp + 1);
        O += f * __ldcg(pp + 2 + c);
      }
    }
    p.out[(size_t(b) * p.Hq + size_t(kvh) * GQA + h) * kHeadDim + c] = Ls > 0.0f ? O / Ls : 0.0f;
  }
  if (tid == 0) p.cnt[size_t(b) * p.Hkv + kvh] = 0u;  // ready for the next launch
}

// ---------------------------------------------------------------- host side

// Pages per split.  Resident CTAs (SMs x CTAs per SM) form a wave; the plan
// minimises waves x (pages per CTA + 2), the 2 standing for the startup of a CTA
// (page-table read and first copy latency) in units of one page of streaming.
SplitPlan plan_splits(int units, int max_pages, int slots) {
  SplitPlan best{max(max_pages, 1), 1};
  if (max_pages <= 1 || units <= 0) return best;
  double best_cost = 1e300;
  const int min_splits = (max_pages + 2047) / 2048;  // page-id list fits in 8 KB of shared memory
  for (int s = max(1, min_splits); s <= min(max_pages, 64); ++s) {
    const int pps = (max_pages + s - 1) / s;
    const int se = (max_pages + pps - 1) / pps;
    const long long ctas = 1ll * units * se;
    const long long waves = (ctas + slots - 1) / slots;
    const double cost = double(waves) * (pps + 2);
    if (cost < best_cost - 1e-9) {
      best_cost = cost;
      best = {pps, se};
    }
  }
  return best;
}

// Calls f.template operator()<T, GQA, KB>() for the instantiation of a configuration.
template <typename F>
cudaError_t dispatch(int gqa, int dtype, int kb, F&& f) {
#define KVQ_KB(T, G)                                 \
  switch (kb) {                                      \
    case 0: return f.template operator()<T, G, 0>(); \
    case 1: return f.template operator()<T, G, 1>(); \
    case 2: return f.template operator()<T, G, 2>(); \
    case 4: return f.template operator()<T, G, 4>(); \
    case 8: return f.template operator()<T, G, 8>(); \
  }                                                  \
  return cudaErrorInvalidValue;
#define KVQ_GQA(T)           \
  switch (gqa) {             \
    case 1: { KVQ_KB(T, 1) } \
    case 2: { KVQ_KB(T, 2) } \
    case 4: { KVQ_KB(T, 4) } \
    case 8: { KVQ_KB(T, 8) } \
  }                          \
  return cudaErrorInvalidValue;
  if (dtype == KVQ_BF16) {
    KVQ_GQA(__nv_bfloat16)
  } else {
    KVQ_GQA(__half)
  }
#undef KVQ_GQA
#undef KVQ_KB
}

// Raises the dynamic shared-memory limit of one decode instantiation (once per size).
template <typename T, int GQA, int KB>
cudaError_t prepare_decode(size_t smem_bytes) {
  static int seen[64];
  return ensure_dynamic_smem(decode_kernel<T, GQA, KB>, int(smem_bytes), seen);
}

struct OccupancyQuery {
  size_t smem;
  int* n;
  template <typename T, int GQA, int KB>
  cudaError_t operator()() {
    cudaError_t e = prepare_decode<T, GQA, KB>(smem);
    if (e != cudaSuccess) return e;
    return cudaOccupancyMaxActiveBlocksPerMultiprocessor(n, decode_kernel<T, GQA, KB>, kDecodeThreads, smem);
  }
};

// Resident decode CTAs per SM for this configuration (2 when it cannot be queried,
// e.g. without a device).
int decode_ctas_per_sm(int gqa, int dtype, int kb, size_t smem_bytes) {
  int n = 0;
  if (dispatch(gqa, dtype, kb, OccupancyQuery{smem_bytes, &n}) != cudaSuccess || n <= 0) {
    cudaGetLastError();
    return 2;
  }
  return n;
}

size_t decode_main_bytes(int P, int GQA, uint32_t rec_bytes) {
  const size_t stage = size_t(128 / P) * rec_bytes;
  size_t m = kStages * stage;
  m = std::max(m, size_t(kResRoundTokens) * 2 * kResRowBytes);
  m = std::max(m, size_t(4) * GQA * kHeadDim * 4);
  return (m + 127) / 128 * 128;
}

struct DecodeLaunch {
  const DecodeParams& p;
  cudaStream_t stream;
  template <typename T, int GQA, int KB>
  cudaError_t operator()() {
    const size_t smem = size_t(p.main_bytes) + size_t(p.pps) * 4;
    cudaError_t e = prepare_decode<T, GQA, KB>(smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(p.max_splits, p.Hkv, p.batch);
    decode_kernel<T, GQA, KB><<<grid, kDecodeThreads, smem, stream>>>(p);
    return cudaGetLastError();
  }
};

cudaError_t launch_decode(const DecodeParams& p, int gqa, int dtype, cudaStream_t stream) {
  if (p.batch <= 0) return cudaSuccess;
  return dispatch(gqa, dtype, p.KB, DecodeLaunch{p, stream});
}

}  // namespace kvq
